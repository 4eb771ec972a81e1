// Rank-r side products of the LoRA linear layer (sm_100a).
//
// With G = dY, U = X A^T and V = G B, the page "QLoRA: NF4 storage, gradients
// and local integration" (gradient paragraph after the teaching program)
// gives dB = s G^T U, dA = s V^T X and the rank-r parts of Y and dX.  All of
// these touch one large activation (X or dY, [M, C] bf16) and a matrix with
// only r <= 64 columns, so they are HBM-bound streams:
//
//  skinny_kernel   out[m][j] = sum_c In[m][c] * Wt(j, c)  (U and V): each CTA
//                  streams 64 rows of In through a TMA ring into the warp
//                  tensor-core MMA; outputs fp32 plus the bf16 forms the
//                  consumers need (s*out for the main GEMMs' extra rank step,
//                  a hi + lo bf16 split that keeps ~16 mantissa bits for the
//                  gradient reductions).
//  colsum_kernel   part[z][c][j] = sum_{m in split z} In[m][c] * S[m][j]
//                  (dA with In = X, S = V), then colsum_reduce_kernel adds
//                  the splits in a fixed order and applies s.
//  vdb_finalize_kernel  after the backward's one pass over G (vdb_tc.cu:
//                  V = G B and the dB partials G^T U on the tensor cores),
//                  forms s*V, the hi/lo split of V and dB = s * (sum of the
//                  partials).
// The two reductions that precede a 4-bit GEMM (skinny_finalize_kernel for U
// in the forward, vdb_finalize_kernel in the backward) also run the GEMM's
// block-scale job (BlockScalesJob) on further threads of their launch.
// Deterministic: every sum runs in a fixed order; no atomics.
#include "common.cuh"
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kTileRows = 64;   // rows of In per tile
constexpr int kTileCols = 64;   // columns (c) per tile
// Ring depth and residency: a 4-deep ring (40-48 KB of shared memory) lets
// four CTAs share an SM, four TMA-issuing threads per SM instead of two with an
// 8-deep ring; that moved the side kernels of a 7B layer step from 1.17 to
// 1.07 ms (the same bytes in flight, more issuers).
constexpr int kStages = 3;      // TMA ring depth (several CTAs per SM keep more tiles in flight)
constexpr int kCtasPerSm = 4;   // grid sizing target (148 SMs)
constexpr int kInTile = kTileRows * 128;  // one [64][64] bf16 tile, 128B-swizzled
constexpr int kThreads = 160;   // warp 0: TMA producer; warps 1-4: MMA consumers

// Byte offset of 16-byte chunk `ch` of row `row` in a [64][64] bf16 tile stored
// in the TMA 128-byte swizzle layout (chunk index XOR row % 8; base 1024-aligned).
__device__ __forceinline__ uint32_t swz(int row, int ch) {
  return static_cast<uint32_t>(row * 128 + ((ch ^ (row & 7)) << 4));
}

struct PipeBarriers {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  int abort_flag;
};

// Cross-proxy fence for this CTA's shared memory: orders the executing
// thread's earlier accesses through the generic proxy (ldmatrix, ld.shared)
// against its later accesses through the async proxy (TMA writes), and the
// reverse.  The PTX memory model orders accesses to the same bytes made
// through different proxies only across such a fence; the mbarrier
// release/acquire of a stage orders the generic proxy alone.  The stages here
// are read by ldmatrix and refilled by TMA, so every reading thread runs it
// after its last read of a stage and before the stage is released.
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

}  // namespace

// ---------------------------------------------------------------------------
// skinny: part[z][m][j] = sum_{c in split z} In[m][c] * Wt(j, c)
// ---------------------------------------------------------------------------
// Grid (ceil(M/64), splits).  One thread of warp 0 streams the CTA's tiles of
// In (64 rows x 64 columns, TMA, 128-byte swizzle) and of Wt (r16 rows of
// A, or 64 rows x r16 columns of the padded B) through a kStages-deep ring;
// warps 1-4 each own 16 rows and run the warp MMAs.  skinny_finalize_kernel adds
// the splits in order and writes the outputs.
template <bool kRowLayout, int NT>
__global__ void __launch_bounds__(kThreads) skinny_kernel(const __grid_constant__ CUtensorMap tmIn,
                                                          const __grid_constant__ CUtensorMap tmW, int64_t M,
                                                          int64_t C, int splits, float* __restrict__ part,
                                                          int* status) {
  constexpr int kR16 = NT * 8;
  constexpr int kSmallTile = 128 * kR16;
  constexpr int kStage = kInTile + kSmallTile;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  PipeBarriers* bars = reinterpret_cast<PipeBarriers*>(smem + kStages * kStage);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kTileRows;
  const int z = blockIdx.y;
  const int64_t steps_total = (C + kTileCols - 1) / kTileCols;
  const int64_t s_begin = steps_total * z / splits;
  const int nsteps = static_cast<int>(steps_total * (z + 1) / splits - s_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 4);
    }
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % kStages, u = i / kStages;
        if (i >= kStages && !mbar_wait(&bars->empty[s], (u - 1) & 1, abort_flag, status)) break;
        uint8_t* st = smem + s * kStage;
        const int c = static_cast<int>((s_begin + i) * kTileCols);
        mbar_arrive_expect_tx(&bars->full[s], kStage);
        tma_load_2d(st, &tmIn, &bars->full[s], c, static_cast<int>(m0));
        if constexpr (kRowLayout)
          tma_load_2d(st + kInTile, &tmW, &bars->full[s], c, 0);  // A rows 0..r16-1, columns c..c+63
        else
          tma_load_2d(st + kInTile, &tmW, &bars->full[s], 0, c);  // padded B rows c..c+63, columns 0..r16-1
        issued = i + 1;
      }
      for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
        mbar_wait_teardown(&bars->full[i % kStages], (i / kStages) & 1, status);
    }
    return;
  }

  const int cw = warp - 1;  // consumer warp: rows 16cw .. 16cw+15
  float acc[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

  const int mat = lane >> 3, rr = lane & 7;
  for (int i = 0; i < nsteps; ++i) {
    const int s = i % kStages, u = i / kStages;
    if (!mbar_wait(&bars->full[s], u & 1, abort_flag, status)) break;
    const uint32_t in_base = smem_u32(smem + s * kStage);
    const uint32_t w_base = in_base + kInTile;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t afr[4];
      ldmatrix_x4(afr, in_base + swz(cw * 16 + (lane & 15), kk * 2 + (lane >> 4)));
#pragma unroll
      for (int nt = 0; nt < NT; nt += 2) {
        uint32_t bfr[4];
        if constexpr (kRowLayout) {
          // matrices: (j nt, k lo), (j nt, k hi), (j nt+1, k lo), (j nt+1, k hi)
          ldmatrix_x4(bfr, w_base + swz((nt + (mat >> 1)) * 8 + rr, kk * 2 + (mat & 1)));
        } else {
          // rows c (pitch 2*r16 bytes), columns j: transposed 8x8 loads
          const int c = kk * 16 + (mat & 1) * 8 + rr;
          ldmatrix_x4_trans(bfr, w_base + c * (2 * kR16) + (nt + (mat >> 1)) * 16);
        }
        const uint32_t b0[2] = {bfr[0], bfr[1]};
        const uint32_t b1[2] = {bfr[2], bfr[3]};
        mma_bf16_16816(acc[nt], afr, b0);
        mma_bf16_16816(acc[nt + 1], afr, b1);
      }
    }
    fence_proxy_async_shared();  // this warp's ldmatrix reads of stage s before its TMA refill
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->empty[s]);
  }

  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int64_t m = m0 + cw * 16 + g + half * 8;
    if (m >= M) continue;
    float* dst = part + (static_cast<int64_t>(z) * M + m) * kRankPad;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      *reinterpret_cast<float2*>(dst + nt * 8 + 2 * t) = make_float2(acc[nt][half * 2], acc[nt][half * 2 + 1]);
  }
}

// out(m, j) = sum_z part[z][m][j] (fixed order); j >= r gives 0.
// Threads past the M * 32 pairs run out.bs (the GEMM's block scales) when set.
__global__ void skinny_finalize_kernel(const float* __restrict__ part, int64_t M, int r, int splits, SkinnyOut out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // over M * 32 pairs
  if (i >= M * (kRankPad / 2)) {
    const int64_t q = i - M * (kRankPad / 2);
    if (out.bs.out != nullptr && q < out.bs.groups) block_scales_group(out.bs, q);
    return;
  }
  const int64_t m = i / (kRankPad / 2);
  const int j = static_cast<int>(i % (kRankPad / 2)) * 2;
  float v0 = 0.0f, v1 = 0.0f;
  if (j < r) {
    for (int z = 0; z < splits; ++z) {
      const float2 p = *reinterpret_cast<const float2*>(part + (static_cast<int64_t>(z) * M + m) * kRankPad + j);
      v0 += p.x;
      v1 += p.y;
    }
    if (j + 1 >= r) v1 = 0.0f;
  }
  if (out.o32) {
    if (j < r) out.o32[m * out.o32_ld + j] = v0;
    if (j + 1 < r) out.o32[m * out.o32_ld + j + 1] = v1;
  }
  if (out.os) *reinterpret_cast<uint32_t*>(out.os + m * kRankPad + j) = pack_bf16x2(out.scale * v0, out.scale * v1);
  if (out.ohi) {
    const uint32_t hi = pack_bf16x2(v0, v1);
    const float r0 = v0 - bf16_bits_to_float(hi & 0xFFFF);
    const float r1 = v1 - bf16_bits_to_float(hi >> 16);
    *reinterpret_cast<uint32_t*>(out.ohi + m * kRankPad + j) = hi;
    *reinterpret_cast<uint32_t*>(out.olo + m * kRankPad + j) = pack_bf16x2(r0, r1);
  }
}

// hi/lo bf16 split of a compact fp32 [M][r] matrix into [M][64] (zero padded).
__global__ void split_hilo_kernel(const float* __restrict__ src, int64_t M, int r, uint16_t* __restrict__ hi,
                                  uint16_t* __restrict__ lo) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= M * (kRankPad / 2)) return;
  const int64_t m = i / (kRankPad / 2);
  const int j = static_cast<int>(i % (kRankPad / 2)) * 2;
  const float v0 = j < r ? src[m * r + j] : 0.0f;
  const float v1 = j + 1 < r ? src[m * r + j + 1] : 0.0f;
  const uint32_t h = pack_bf16x2(v0, v1);
  *reinterpret_cast<uint32_t*>(hi + m * kRankPad + j) = h;
  *reinterpret_cast<uint32_t*>(lo + m * kRankPad + j) =
      pack_bf16x2(v0 - bf16_bits_to_float(h & 0xFFFF), v1 - bf16_bits_to_float(h >> 16));
}

int skinny_splits(int64_t M, int64_t C) {
  const int64_t mtiles = (M + kTileRows - 1) / kTileRows;
  const int64_t steps = (C + kTileCols - 1) / kTileCols;
  int64_t s = (kCtasPerSm * 148 + mtiles - 1) / mtiles;
  if (s > steps) s = steps;
  if (s > 64) s = 64;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

size_t skinny_partial_bytes(int64_t M, int64_t C) {
  return static_cast<size_t>(skinny_splits(M, C)) * static_cast<size_t>(M) * kRankPad * sizeof(float);
}

template <bool kRowLayout, int NT>
cudaError_t launch_skinny_nt(const CUtensorMap& tin, const CUtensorMap& tw, int64_t M, int64_t C, int splits,
                             float* part, int* status, cudaStream_t stream) {
  constexpr int kStage = kInTile + 128 * NT * 8;
  constexpr int smem = 1024 + kStages * kStage + static_cast<int>(sizeof(PipeBarriers));
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static DeviceOnce configured;
  e = configured.run(dev, [] {
    return cudaFuncSetAttribute(skinny_kernel<kRowLayout, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>((M + kTileRows - 1) / kTileRows), static_cast<unsigned>(splits));
  skinny_kernel<kRowLayout, NT><<<grid, kThreads, smem, stream>>>(tin, tw, M, C, splits, part, status);
  return cudaGetLastError();
}

cudaError_t launch_skinny(const uint16_t* In, int64_t M, int64_t C, const uint16_t* Wt, bool wt_is_rc, int r,
                          int64_t ldw, float* part, const SkinnyOut& out, int* status, cudaStream_t stream) {
  const int splits = skinny_splits(M, C);
  const int nt = ((r + 15) / 16) * 2;
  CUtensorMap tin, tw;
  if (!encode_tensor_map_2d(&tin, In, M, C, kTileRows, kTileCols)) return cudaErrorInvalidValue;
  if (wt_is_rc) {
    if (!encode_tensor_map_2d(&tw, Wt, r, C, nt * 8, kTileCols)) return cudaErrorInvalidValue;
  } else {
    if (!encode_tensor_map_2d(&tw, Wt, C, r, kTileCols, nt * 8, false, ldw)) return cudaErrorInvalidValue;
  }
  cudaError_t e;
  if (wt_is_rc) {
    e = nt == 2   ? launch_skinny_nt<true, 2>(tin, tw, M, C, splits, part, status, stream)
        : nt == 4 ? launch_skinny_nt<true, 4>(tin, tw, M, C, splits, part, status, stream)
        : nt == 6 ? launch_skinny_nt<true, 6>(tin, tw, M, C, splits, part, status, stream)
                  : launch_skinny_nt<true, 8>(tin, tw, M, C, splits, part, status, stream);
  } else {
    e = nt == 2   ? launch_skinny_nt<false, 2>(tin, tw, M, C, splits, part, status, stream)
        : nt == 4 ? launch_skinny_nt<false, 4>(tin, tw, M, C, splits, part, status, stream)
        : nt == 6 ? launch_skinny_nt<false, 6>(tin, tw, M, C, splits, part, status, stream)
                  : launch_skinny_nt<false, 8>(tin, tw, M, C, splits, part, status, stream);
  }
  if (e != cudaSuccess) return e;
  const int64_t total = M * (kRankPad / 2) + (out.bs.out != nullptr ? out.bs.groups : 0);
  skinny_finalize_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(part, M, r, splits, out);
  return cudaGetLastError();
}

cudaError_t launch_split_hilo(const float* src, int64_t M, int r, uint16_t* hi, uint16_t* lo, cudaStream_t stream) {
  const int64_t total = M * (kRankPad / 2);
  split_hilo_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(src, M, r, hi, lo);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// colsum: part[z][c][j] = sum_{m in split z} In[m][c] * (hi[m][j] + lo[m][j])
// ---------------------------------------------------------------------------
// Grid (ceil(C/64), splits).  Warp 0 streams tiles of In (64 tokens x 64
// columns, 128-byte swizzle) and the matching 64 x r16 tiles of the hi / lo
// split of S through a kStages-deep TMA ring; warps 1-4 each own 16 columns:
// A = In^T by transposed 8x8 loads, B = hi and lo.
template <int NT>
__global__ void __launch_bounds__(kThreads) colsum_kernel(const __grid_constant__ CUtensorMap tmIn,
                                                          const __grid_constant__ CUtensorMap tmHi,
                                                          const __grid_constant__ CUtensorMap tmLo, int64_t M,
                                                          int64_t C, int splits, float* __restrict__ part,
                                                          int* status) {
  constexpr int kR16 = NT * 8;
  constexpr int kSTile = 128 * kR16;  // [64 tokens][r16] bf16
  constexpr int kStage = kInTile + 2 * kSTile;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  PipeBarriers* bars = reinterpret_cast<PipeBarriers*>(smem + kStages * kStage);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kTileCols;
  const int z = blockIdx.y;
  const int64_t steps_total = (M + kTileRows - 1) / kTileRows;
  const int64_t s_begin = steps_total * z / splits;
  const int nsteps = static_cast<int>(steps_total * (z + 1) / splits - s_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 4);
    }
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % kStages, u = i / kStages;
        if (i >= kStages && !mbar_wait(&bars->empty[s], (u - 1) & 1, abort_flag, status)) break;
        uint8_t* st = smem + s * kStage;
        const int m = static_cast<int>((s_begin + i) * kTileRows);
        mbar_arrive_expect_tx(&bars->full[s], kStage);
        tma_load_2d(st, &tmIn, &bars->full[s], static_cast<int>(c0), m);
        tma_load_2d(st + kInTile, &tmHi, &bars->full[s], 0, m);
        tma_load_2d(st + kInTile + kSTile, &tmLo, &bars->full[s], 0, m);
        issued = i + 1;
      }
      for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
        mbar_wait_teardown(&bars->full[i % kStages], (i / kStages) & 1, status);
    }
    return;
  }

  const int cw = warp - 1;  // consumer warp: columns 16cw .. 16cw+15
  float acc[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

  const int mat = lane >> 3, rr = lane & 7;
  for (int i = 0; i < nsteps; ++i) {
    const int s = i % kStages, u = i / kStages;
    if (!mbar_wait(&bars->full[s], u & 1, abort_flag, status)) break;
    const uint32_t in_base = smem_u32(smem + s * kStage);
    const uint32_t hi_base = in_base + kInTile;
    const uint32_t lo_base = hi_base + kSTile;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {  // 16 tokens per MMA step
      // A = In^T (rows c, k = m): transposed loads of the [m][c] tile.
      uint32_t afr[4];
      ldmatrix_x4_trans(afr, in_base + swz(kk * 16 + (mat >> 1) * 8 + rr, cw * 2 + (mat & 1)));
      const int m = kk * 16 + (mat & 1) * 8 + rr;
#pragma unroll
      for (int nt = 0; nt < NT; nt += 2) {
        const uint32_t off = m * (2 * kR16) + (nt + (mat >> 1)) * 16;
        uint32_t bh[4], bl[4];
        ldmatrix_x4_trans(bh, hi_base + off);
        ldmatrix_x4_trans(bl, lo_base + off);
        const uint32_t h0[2] = {bh[0], bh[1]}, l0[2] = {bl[0], bl[1]};
        const uint32_t h1[2] = {bh[2], bh[3]}, l1[2] = {bl[2], bl[3]};
        mma_bf16_16816(acc[nt], afr, h0);
        mma_bf16_16816(acc[nt], afr, l0);
        mma_bf16_16816(acc[nt + 1], afr, h1);
        mma_bf16_16816(acc[nt + 1], afr, l1);
      }
    }
    fence_proxy_async_shared();  // this warp's ldmatrix reads of stage s before its TMA refill
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->empty[s]);
  }

  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int64_t c = c0 + cw * 16 + g + half * 8;
    if (c >= C) continue;
    float* dst = part + (static_cast<int64_t>(z) * C + c) * kRankPad;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      *reinterpret_cast<float2*>(dst + nt * 8 + 2 * t) = make_float2(acc[nt][half * 2], acc[nt][half * 2 + 1]);
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
  int64_t s = (kCtasPerSm * 148 + ctiles - 1) / ctiles;
  if (s > msteps) s = msteps;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

size_t colsum_partial_bytes(int64_t M, int64_t C) {
  return static_cast<size_t>(colsum_splits(M, C)) * static_cast<size_t>(C) * kRankPad * sizeof(float);
}

template <int NT>
cudaError_t launch_colsum_nt(const CUtensorMap& tin, const CUtensorMap& thi, const CUtensorMap& tlo, int64_t M,
                             int64_t C, int splits, float* part, int* status, cudaStream_t stream) {
  constexpr int kStage = kInTile + 2 * 128 * NT * 8;
  constexpr int smem = 1024 + kStages * kStage + static_cast<int>(sizeof(PipeBarriers));
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static DeviceOnce configured;
  e = configured.run(dev, [] {
    return cudaFuncSetAttribute(colsum_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>((C + kTileCols - 1) / kTileCols), static_cast<unsigned>(splits));
  colsum_kernel<NT><<<grid, kThreads, smem, stream>>>(tin, thi, tlo, M, C, splits, part, status);
  return cudaGetLastError();
}

cudaError_t launch_colsum(const uint16_t* In, int64_t M, int64_t C, const uint16_t* hi, const uint16_t* lo, int r,
                          float scale, float* part, float* dst, bool dst_rc, int* status, cudaStream_t stream) {
  const int splits = colsum_splits(M, C);
  const int nt = ((r + 15) / 16) * 2;
  CUtensorMap tin, thi, tlo;
  if (!encode_tensor_map_2d(&tin, In, M, C, kTileRows, kTileCols)) return cudaErrorInvalidValue;
  if (!encode_tensor_map_2d(&thi, hi, M, kRankPad, kTileRows, nt * 8, false)) return cudaErrorInvalidValue;
  if (!encode_tensor_map_2d(&tlo, lo, M, kRankPad, kTileRows, nt * 8, false)) return cudaErrorInvalidValue;
  cudaError_t e = nt == 2   ? launch_colsum_nt<2>(tin, thi, tlo, M, C, splits, part, status, stream)
                  : nt == 4 ? launch_colsum_nt<4>(tin, thi, tlo, M, C, splits, part, status, stream)
                  : nt == 6 ? launch_colsum_nt<6>(tin, thi, tlo, M, C, splits, part, status, stream)
                            : launch_colsum_nt<8>(tin, thi, tlo, M, C, splits, part, status, stream);
  if (e != cudaSuccess) return e;
  const int64_t total = C * r;
  colsum_reduce_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(part, C, r, splits, scale, dst,
                                                                                       dst_rc ? 1 : 0);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// vdb reduction: the partials of the tensor-core V / dB pass (vdb_tc.cu)
// ---------------------------------------------------------------------------
// V (fp32) = sum over column blocks of vpart, written as s*V (bf16, [M][64]
// zero padded) and its hi / lo split; dB[c][j] = scale * sum over token
// blocks of dbpart.  Threads [0, M*32) take pairs of V, the rest dB entries.
__global__ void vdb_finalize_kernel(const float* __restrict__ vpart, int ncb, const float* __restrict__ dbpart,
                                    int ntb, int64_t M, int64_t N, int r, int r16, float scale,
                                    uint16_t* __restrict__ vs, uint16_t* __restrict__ vhi, uint16_t* __restrict__ vlo,
                                    float* __restrict__ dB, BlockScalesJob bs) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nv = M * (kRankPad / 2);
  if (i < nv) {
    const int64_t m = i / (kRankPad / 2);
    const int j = static_cast<int>(i % (kRankPad / 2)) * 2;
    float v0 = 0.0f, v1 = 0.0f;
    if (j < r) {
      for (int z = 0; z < ncb; ++z) {
        const float2 p = *reinterpret_cast<const float2*>(vpart + (static_cast<int64_t>(z) * M + m) * r16 + j);
        v0 += p.x;
        v1 += p.y;
      }
      if (j + 1 >= r) v1 = 0.0f;
    }
    *reinterpret_cast<uint32_t*>(vs + m * kRankPad + j) = pack_bf16x2(scale * v0, scale * v1);
    const uint32_t hi = pack_bf16x2(v0, v1);
    *reinterpret_cast<uint32_t*>(vhi + m * kRankPad + j) = hi;
    *reinterpret_cast<uint32_t*>(vlo + m * kRankPad + j) =
        pack_bf16x2(v0 - bf16_bits_to_float(hi & 0xFFFF), v1 - bf16_bits_to_float(hi >> 16));
    return;
  }
  const int64_t k = i - nv;
  const int64_t ndb = dB != nullptr ? N * r : 0;
  if (k >= ndb) {  // the GEMM's block scales, when set
    if (bs.out != nullptr && k - ndb < bs.groups) block_scales_group(bs, k - ndb);
    return;
  }
  const int64_t c = k / r;
  const int j = static_cast<int>(k % r);
  float s = 0.0f;
  for (int z = 0; z < ntb; ++z) s += dbpart[(static_cast<int64_t>(z) * N + c) * r16 + j];
  dB[c * r + j] = scale * s;
}

cudaError_t launch_vdb_finalize(const float* vpart, int ncb, const float* dbpart, int ntb, int64_t M, int64_t N,
                                int r, float scale, uint16_t* vs, uint16_t* vhi, uint16_t* vlo, float* dB,
                                const BlockScalesJob& bs, cudaStream_t stream) {
  const int64_t total =
      M * (kRankPad / 2) + (dB != nullptr ? N * r : 0) + (bs.out != nullptr ? bs.groups : 0);
  vdb_finalize_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(vpart, ncb, dbpart, ntb, M, N,
                                                                                       r, 16, scale, vs, vhi, vlo, dB,
                                                                                       bs);
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
