// Pieces shared by the tensor-core GEMM kernels (gemm_tc.cu, gemm_nf4.cu):
// the tile raster of the pair-CTA kernels, its host-side choice of group
// size, and the epilogue store of one accumulator row segment.
#pragma once

#include "common.cuh"

namespace qnf4 {

// Tile order of the pair kernels: groups of `group` consecutive tiles along M
// (along_n = 0) or N (along_n = 1) sweep the other dimension, so the panels of
// one group stay in L2 while the other operand streams past once per group.
__device__ __forceinline__ void pair_tile_coords(int t, int m_tiles, int n_tiles, int group, int along_n, int& mb,
                                                 int& nb) {
  const int g_tiles = along_n ? n_tiles : m_tiles, o_tiles = along_n ? m_tiles : n_tiles;
  const int per_group = group * o_tiles;
  const int gi = t / per_group, first = gi * group;
  const int gsize = min(group, g_tiles - first), local = t - gi * per_group;
  const int gpos = first + local % gsize, opos = local / gsize;
  mb = along_n ? opos : gpos;
  nb = along_n ? gpos : opos;
}

struct RasterChoice {
  int group;
  int along_n;
};

// Group as many 256-wide panels as `budget` bytes keep resident, along the
// dimension that makes the HBM traffic smallest:
//   along M: a_total + b_total * ceil(m_tiles / gm)   (A panels resident)
//   along N: b_total + a_total * ceil(n_tiles / gn)   (B panels resident)
// a_panel / b_panel: bytes one 256-wide panel of each operand reads from HBM.
inline RasterChoice choose_raster(int64_t m_tiles, int64_t n_tiles, double a_panel, double b_panel, double budget) {
  auto fit = [&](double panel, int64_t tiles) {
    int64_t g = panel > 0 ? static_cast<int64_t>(budget / panel) : tiles;
    if (g < 1) g = 1;
    return g < tiles ? g : tiles;
  };
  const int64_t gm = fit(a_panel, m_tiles), gn = fit(b_panel, n_tiles);
  const double a_total = a_panel * static_cast<double>(m_tiles), b_total = b_panel * static_cast<double>(n_tiles);
  const double traffic_m = a_total + b_total * static_cast<double>((m_tiles + gm - 1) / gm);
  const double traffic_n = b_total + a_total * static_cast<double>((n_tiles + gn - 1) / gn);
  RasterChoice c;
  c.along_n = traffic_n < traffic_m ? 1 : 0;
  c.group = static_cast<int>(c.along_n ? gn : gm);
  return c;
}

// Store 32 consecutive fp32 accumulator columns of one output row as bf16
// (D row-major [M][N]); with `accumulate` the existing bf16 values are added
// in fp32 first.  Columns past N are skipped.
__device__ __forceinline__ void store_row32_bf16(const uint32_t (&v)[32], uint16_t* __restrict__ D, int row, int col,
                                                 int M, int N, int accumulate) {
  if (row >= M || col >= N) return;
  uint16_t* dst = D + static_cast<int64_t>(row) * N + col;
  if (col + 32 <= N) {
    uint32_t pk[16];
    if (accumulate) {
      const uint4* old = reinterpret_cast<const uint4*>(dst);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const uint4 o = old[q4];
        const uint32_t ow[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int idx = q4 * 8 + e * 2;
          pk[q4 * 4 + e] = pack_bf16x2(__uint_as_float(v[idx]) + bf16_bits_to_float(ow[e] & 0xFFFF),
                                       __uint_as_float(v[idx + 1]) + bf16_bits_to_float(ow[e] >> 16));
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
    }
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) d4[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      if (col + e < N) {
        float val = __uint_as_float(v[e]);
        if (accumulate) val += bf16_bits_to_float(dst[e]);
        dst[e] = static_cast<uint16_t>(pack_bf16x2(val, 0.0f) & 0xFFFF);
      }
    }
  }
}

}  // namespace qnf4
