// Rank-r side products of the LoRA linear layer (sm_100a).
//
// With G = dY, U = X A^T and V = G B, the page "QLoRA: NF4 storage, gradients
// and local integration" (gradient paragraph after the teaching program)
// gives dB = s G^T U, dA = s V^T X and the rank-r parts of Y and dX.  All of
// these touch one large activation (X or dY, [M, C] bf16) and a matrix with
// only r <= 64 columns, so they are HBM-bound streams:
//
//  skinny_kernel   out[m][j] = sum_c In[m][c] * Wt(j, c)  (U and V): each CTA
//                  streams 64 rows of In through a cp.async ring and the warp
//                  tensor-core MMA; outputs fp32 plus the bf16 forms the
//                  consumers need (s*out for the main GEMMs' extra rank step,
//                  a hi + lo bf16 split that keeps ~16 mantissa bits for the
//                  gradient reductions).
//  colsum_kernel   part[z][c][j] = sum_{m in split z} In[m][c] * S[m][j]
//                  (dB with In = dY, S = U; dA with In = X, S = V), then
//                  colsum_reduce_kernel adds the splits in a fixed order and
//                  applies s.  Deterministic: no atomics.
#include "common.cuh"
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kTileRows = 64;  // rows of In per CTA (skinny) / per step (colsum)
constexpr int kTileCols = 64;  // columns (c) per pipeline step
constexpr int kStages = 4;
constexpr int kTileBytes = kTileRows * 128;  // one [64][64] bf16 tile

// Byte offset of 16-byte chunk `ch` of row `row` in a [64][64] bf16 tile
// stored with an XOR swizzle (conflict-free ldmatrix).
__device__ __forceinline__ uint32_t swz(int row, int ch) {
  return static_cast<uint32_t>(row * 128 + ((ch ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint16_t to_bf16(float v) { return static_cast<uint16_t>(pack_bf16x2(v, 0.0f) & 0xFFFF); }

}  // namespace

// ---------------------------------------------------------------------------
// skinny: out[m][j] = sum_c In[m][c] * Wt(j, c)
// ---------------------------------------------------------------------------
template <bool kRowLayout>
__global__ void __launch_bounds__(128) skinny_kernel(const uint16_t* __restrict__ In, int64_t M, int64_t C,
                                                     const uint16_t* __restrict__ Wt, int r, SkinnyOut out) {
  extern __shared__ __align__(128) uint8_t smem_dyn[];
  uint8_t(*s_in)[kTileBytes] = reinterpret_cast<uint8_t(*)[kTileBytes]>(smem_dyn);
  uint8_t(*s_w)[kTileBytes] = reinterpret_cast<uint8_t(*)[kTileBytes]>(smem_dyn + kStages * kTileBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kTileRows;
  const int nsteps = static_cast<int>((C + kTileCols - 1) / kTileCols);
  const int ntiles = (r + 7) / 8;

  auto load_stage = [&](int step, int buf) {
    const int64_t c0 = static_cast<int64_t>(step) * kTileCols;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + i * 128;  // 512 chunks of 16 B
      const int row = idx >> 3, ch = idx & 7;
      const int64_t m = m0 + row, c = c0 + ch * 8;
      const bool ok = m < M && c < C;
      cp_async_16(s_in[buf] + swz(row, ch), ok ? In + m * C + c : In, ok);
      if constexpr (kRowLayout) {  // Wt = Wr [r][C]: tile rows j
        const bool okw = row < r && c < C;
        cp_async_16(s_w[buf] + swz(row, ch), okw ? Wt + static_cast<int64_t>(row) * C + c : Wt, okw);
      } else {  // Wt = Wc [C][64] (zero padded beyond r): tile rows c
        const int64_t cr = c0 + row;
        const bool okw = cr < C;
        cp_async_16(s_w[buf] + swz(row, ch), okw ? Wt + cr * kRankPad + ch * 8 : Wt, okw);
      }
    }
  };

  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < nsteps) load_stage(s, s);
    cp_async_commit();
  }
  for (int step = 0; step < nsteps; ++step) {
    const int buf = step % kStages;
    if (step + kStages - 1 < nsteps) load_stage(step + kStages - 1, (step + kStages - 1) % kStages);
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    __syncthreads();
    const uint32_t in_base = smem_u32(s_in[buf]);
    const uint32_t w_base = smem_u32(s_w[buf]);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t afr[4];
      {
        const int row = warp * 16 + (lane & 15);
        const int ch = kk * 2 + (lane >> 4);
        ldmatrix_x4(afr, in_base + swz(row, ch));
      }
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        if (nt >= ntiles) break;
        uint32_t bfr[4];
        const int mat = lane >> 3, rr = lane & 7;
        if constexpr (kRowLayout) {
          // matrices: (j nt, k lo), (j nt, k hi), (j nt+1, k lo), (j nt+1, k hi)
          const int j = (nt + (mat >> 1)) * 8 + rr;
          const int ch = kk * 2 + (mat & 1);
          ldmatrix_x4(bfr, w_base + swz(j, ch));
        } else {
          // rows c, columns j: transposed 8x8 loads
          const int c = kk * 16 + (mat & 1) * 8 + rr;
          const int ch = nt + (mat >> 1);
          ldmatrix_x4_trans(bfr, w_base + swz(c, ch));
        }
        const uint32_t b0[2] = {bfr[0], bfr[1]};
        mma_bf16_16816(acc[nt], afr, b0);
        if (nt + 1 < ntiles) {
          const uint32_t b1[2] = {bfr[2], bfr[3]};
          mma_bf16_16816(acc[nt + 1], afr, b1);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int64_t m = m0 + warp * 16 + g + half * 8;
    if (m >= M) continue;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int j = nt * 8 + 2 * t;
      float v0 = nt < ntiles && j < r ? acc[nt][half * 2] : 0.0f;
      float v1 = nt < ntiles && j + 1 < r ? acc[nt][half * 2 + 1] : 0.0f;
      if (out.o32) *reinterpret_cast<float2*>(out.o32 + m * kRankPad + j) = make_float2(v0, v1);
      if (out.os) *reinterpret_cast<uint32_t*>(out.os + m * kRankPad + j) = pack_bf16x2(out.scale * v0, out.scale * v1);
      if (out.ohi) {
        const uint32_t hi = pack_bf16x2(v0, v1);
        const float r0 = v0 - bf16_bits_to_float(hi & 0xFFFF);
        const float r1 = v1 - bf16_bits_to_float(hi >> 16);
        *reinterpret_cast<uint32_t*>(out.ohi + m * kRankPad + j) = hi;
        *reinterpret_cast<uint32_t*>(out.olo + m * kRankPad + j) = pack_bf16x2(r0, r1);
      }
      if (out.obf) {
        if (j < r) out.obf[m * r + j] = to_bf16(v0);
        if (j + 1 < r) out.obf[m * r + j + 1] = to_bf16(v1);
      }
    }
  }
}

cudaError_t launch_skinny(const uint16_t* In, int64_t M, int64_t C, const uint16_t* Wt, bool wt_is_rc, int r,
                          const SkinnyOut& out, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>((M + kTileRows - 1) / kTileRows);
  const int smem = 2 * kStages * kTileBytes;
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(skinny_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    cudaFuncSetAttribute(skinny_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    configured = true;
  }
  if (wt_is_rc)
    skinny_kernel<true><<<grid, 128, smem, stream>>>(In, M, C, Wt, r, out);
  else
    skinny_kernel<false><<<grid, 128, smem, stream>>>(In, M, C, Wt, r, out);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// colsum: part[z][c][j] = sum_{m in split z} In[m][c] * (hi[m][j] + lo[m][j])
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) colsum_kernel(const uint16_t* __restrict__ In, int64_t M, int64_t C,
                                                     const uint16_t* __restrict__ hi, const uint16_t* __restrict__ lo,
                                                     int r, int splits, float* __restrict__ part) {
  extern __shared__ __align__(128) uint8_t smem_dyn[];
  uint8_t(*s_in)[kTileBytes] = reinterpret_cast<uint8_t(*)[kTileBytes]>(smem_dyn);
  uint8_t(*s_hi)[kTileBytes] = reinterpret_cast<uint8_t(*)[kTileBytes]>(smem_dyn + kStages * kTileBytes);
  uint8_t(*s_lo)[kTileBytes] = reinterpret_cast<uint8_t(*)[kTileBytes]>(smem_dyn + 2 * kStages * kTileBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kTileCols;
  const int z = blockIdx.y;
  const int64_t msteps_total = (M + kTileRows - 1) / kTileRows;
  const int64_t s_begin = msteps_total * z / splits, s_end = msteps_total * (z + 1) / splits;
  const int nsteps = static_cast<int>(s_end - s_begin);
  const int ntiles = (r + 7) / 8;

  auto load_stage = [&](int step, int buf) {
    const int64_t mb = (s_begin + step) * kTileRows;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + i * 128;
      const int row = idx >> 3, ch = idx & 7;
      const int64_t m = mb + row, c = c0 + ch * 8;
      const bool ok = m < M && c < C;
      cp_async_16(s_in[buf] + swz(row, ch), ok ? In + m * C + c : In, ok);
      const bool okm = m < M;
      cp_async_16(s_hi[buf] + swz(row, ch), okm ? hi + m * kRankPad + ch * 8 : hi, okm);
      cp_async_16(s_lo[buf] + swz(row, ch), okm ? lo + m * kRankPad + ch * 8 : lo, okm);
    }
  };

  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < nsteps) load_stage(s, s);
    cp_async_commit();
  }
  for (int step = 0; step < nsteps; ++step) {
    const int buf = step % kStages;
    if (step + kStages - 1 < nsteps) load_stage(step + kStages - 1, (step + kStages - 1) % kStages);
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    __syncthreads();
    const uint32_t in_base = smem_u32(s_in[buf]);
    const uint32_t hi_base = smem_u32(s_hi[buf]);
    const uint32_t lo_base = smem_u32(s_lo[buf]);
    const int mat = lane >> 3, rr = lane & 7;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {  // 16 tokens per MMA step
      // A = In^T (rows c, k = m): transposed loads of the [m][c] tile.
      uint32_t afr[4];
      {
        const int m = kk * 16 + (mat >> 1) * 8 + rr;
        const int ch = warp * 2 + (mat & 1);
        ldmatrix_x4_trans(afr, in_base + swz(m, ch));
      }
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        if (nt >= ntiles) break;
        const int m = kk * 16 + (mat & 1) * 8 + rr;
        const int ch = nt + (mat >> 1);
        uint32_t bh[4], bl[4];
        ldmatrix_x4_trans(bh, hi_base + swz(m, ch));
        ldmatrix_x4_trans(bl, lo_base + swz(m, ch));
        {
          const uint32_t b0[2] = {bh[0], bh[1]};
          const uint32_t b1[2] = {bl[0], bl[1]};
          mma_bf16_16816(acc[nt], afr, b0);
          mma_bf16_16816(acc[nt], afr, b1);
        }
        if (nt + 1 < ntiles) {
          const uint32_t b0[2] = {bh[2], bh[3]};
          const uint32_t b1[2] = {bl[2], bl[3]};
          mma_bf16_16816(acc[nt + 1], afr, b0);
          mma_bf16_16816(acc[nt + 1], afr, b1);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int64_t c = c0 + warp * 16 + g + half * 8;
    if (c >= C) continue;
    float* dst = part + (static_cast<int64_t>(z) * C + c) * kRankPad;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int j = nt * 8 + 2 * t;
      const float v0 = nt < ntiles ? acc[nt][half * 2] : 0.0f;
      const float v1 = nt < ntiles ? acc[nt][half * 2 + 1] : 0.0f;
      *reinterpret_cast<float2*>(dst + j) = make_float2(v0, v1);
    }
  }
}

__global__ void colsum_reduce_kernel(const float* __restrict__ part, int64_t C, int r, int splits, float scale,
                                     float* __restrict__ dst, int dst_rc) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // over C * r
  if (i >= C * r) return;
  int64_t c, j;
  if (dst_rc) {  // dst [r][C]: consecutive threads walk c
    j = i / C;
    c = i % C;
  } else {  // dst [C][r]
    c = i / r;
    j = i % r;
  }
  float s = 0.0f;
  for (int z = 0; z < splits; ++z) s += part[(static_cast<int64_t>(z) * C + c) * kRankPad + j];
  dst[dst_rc ? j * C + c : c * r + j] = scale * s;
}

int colsum_splits(int64_t M, int64_t C) {
  const int64_t ctiles = (C + kTileCols - 1) / kTileCols;
  const int64_t msteps = (M + kTileRows - 1) / kTileRows;
  int64_t s = (2 * 148 + ctiles - 1) / ctiles;
  if (s > msteps) s = msteps;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

size_t colsum_partial_bytes(int64_t M, int64_t C) {
  return static_cast<size_t>(colsum_splits(M, C)) * static_cast<size_t>(C) * kRankPad * sizeof(float);
}

cudaError_t launch_colsum(const uint16_t* In, int64_t M, int64_t C, const uint16_t* hi, const uint16_t* lo, int r,
                          float scale, float* part, float* dst, bool dst_rc, cudaStream_t stream) {
  const int splits = colsum_splits(M, C);
  dim3 grid(static_cast<unsigned>((C + kTileCols - 1) / kTileCols), static_cast<unsigned>(splits));
  const int smem = 3 * kStages * kTileBytes;
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(colsum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    configured = true;
  }
  colsum_kernel<<<grid, 128, smem, stream>>>(In, M, C, hi, lo, r, splits, part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t total = C * r;
  colsum_reduce_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(part, C, r, splits, scale, dst,
                                                                                       dst_rc ? 1 : 0);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// pad: dst[row][j] = src(row, j) for j < r, 0 for r <= j < 64
// ---------------------------------------------------------------------------
__global__ void pad_rank_kernel(const uint16_t* __restrict__ src, int src_transposed, int64_t rows, int r,
                                uint16_t* __restrict__ dst) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= rows * kRankPad) return;
  const int64_t row = i / kRankPad;
  const int j = static_cast<int>(i % kRankPad);
  uint16_t v = 0;
  if (j < r) v = src_transposed ? src[static_cast<int64_t>(j) * rows + row] : src[row * r + j];
  dst[i] = v;
}

cudaError_t launch_pad_rank(const uint16_t* src, bool src_transposed, int64_t rows, int r, uint16_t* dst,
                            cudaStream_t stream) {
  const int64_t total = rows * kRankPad;
  pad_rank_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(src, src_transposed ? 1 : 0, rows,
                                                                                  r, dst);
  return cudaGetLastError();
}

}  // namespace qnf4
