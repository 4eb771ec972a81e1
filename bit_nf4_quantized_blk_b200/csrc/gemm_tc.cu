// Tensor-core GEMM for the training-shaped LoRA linear (sm_100a, tcgen05).
//
//   D[M][N] (+)= A[M][K] B[N][K]^T + A2[M][64] B2[N][64]^T
//
// Forward: A = X, B = W_hat (dequantized NF4 weight), A2 = s (X A^T) padded
// to 64 columns, B2 = the LoRA B padded.  Backward-input: A = dY, B = W_hat^T,
// A2 = s (dY B), B2 = A^T ("QLoRA: NF4 storage, gradients and local
// integration": Y = X Qhat(W)^T + s X A^T B^T, dX = G Qhat(W) + s G B A).
// The rank-r product is one more pipeline step that issues ceil(r/16)
// K=16 MMAs into the same accumulator.
//
// Two kernels: the pair-CTA kernel below (256 x 256 tiles on CTA pairs, used
// whenever pair clusters can be scheduled) and this one-CTA kernel.
// Persistent CTAs (one per SM) compute 128 x 256 tiles with a 4-stage TMA ring:
//   warp 0      TMA producer (one elected thread), 128B-swizzled tiles
//   warp 1      TMEM allocation + MMA issue (one thread): tcgen05.mma
//               kind::f16, M=128 N=256 K=16, fp32 accumulators in TMEM,
//               double-buffered so the epilogue overlaps the next tile
//   warps 2-5   epilogue: tcgen05.ld 32 columns at a time -> bf16 -> global
// Every barrier wait is bounded (see common.cuh); a timeout aborts the CTA,
// which then waits (bounded) for its copies and MMAs in flight and frees its
// tensor memory before returning.  No TMA or bulk load uses cluster
// multicast: every CTA loads its own tiles.  The pair kernel's
// tcgen05.commit does carry .multicast::cluster, which is an mbarrier arrive
// delivered to both CTAs of the pair on this GPU, not a load.
//
// These kernels read a dense bf16 weight (the dequantized copy).  The linear
// calls use them for the dense-weight ablation arm and as the fallback where
// pair clusters cannot be scheduled; the default path is gemm_nf4.cu, which
// decodes the 4-bit weight inside the GEMM.
#include "common.cuh"
#include "gemm_common.cuh"
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_TILE = BM * BK * 2;  // 16 KB
constexpr int B_TILE = BN * BK * 2;  // 32 KB
constexpr int TMEM_COLS = 512;       // two 128 x 256 fp32 accumulators
constexpr int kGroupM = 16;          // M tiles per raster group
constexpr int SMEM_BYTES = 1024 + STAGES * (A_TILE + B_TILE) + 256;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Resolved once per process (a thread-safe static initialisation; nullptr if
// the driver does not provide it).
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return static_cast<EncodeTiledFn>(nullptr);
  }();
  return fn;
}

}  // namespace

// bf16 row-major [rows][cols] (cols contiguous, row pitch ld elements), box
// box_rows x box_cols, 128-byte swizzle (or none), zero fill outside the tensor.
bool encode_tensor_map_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                          uint32_t box_cols, bool swizzle128, uint64_t ld) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t gdim[2] = {cols, rows};
  const cuuint64_t gstride[1] = {(ld ? ld : cols) * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major [rows][cols] tensor of 1-byte (uint8) or 4-byte (fp32) elements,
// row pitch `ld` elements, box box_rows x box_cols, no swizzle, zero fill
// outside the tensor.
bool encode_tensor_map_2d_plain(CUtensorMap* map, const void* base, int elem_bytes, uint64_t rows, uint64_t cols,
                                uint64_t ld, uint32_t box_rows, uint32_t box_cols) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr || (elem_bytes != 1 && elem_bytes != 4)) return false;
  const cuuint64_t gdim[2] = {cols, rows};
  const cuuint64_t gstride[1] = {ld * static_cast<uint64_t>(elem_bytes)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return fn(map, elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
            const_cast<void*>(base), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tile order: groups of kGroupM consecutive M tiles sweep the N tiles, so the
// CTAs resident at one time share a few A row panels and a few B row panels
// (both stay in L2 instead of being re-read from HBM every wave).
__device__ __forceinline__ void tile_coords(int t, int m_tiles, int n_tiles, int& mb, int& nb) {
  const int per_group = kGroupM * n_tiles;
  const int group = t / per_group;
  const int first_m = group * kGroupM;
  const int gsize = min(kGroupM, m_tiles - first_m);
  const int local = t - group * per_group;
  mb = first_m + local % gsize;
  nb = local / gsize;
}

// Persistent: one CTA per SM loops over output tiles.  The TMA ring runs
// across tile boundaries; the accumulator is double-buffered in TMEM (2 x 256
// columns) so the epilogue of one tile overlaps the main loop of the next.
//
// kBMN selects the B operand's major-ness.  K-major: B tiles are 256 rows (N)
// of 64 K elements, one TMA box.  MN-major: B is stored [K][N] (N
// contiguous, e.g. the weight [d_out, d_in] read as W^T); a stage holds four
// 64 (K) x 64 (N) boxes 8 KB apart, described with LBO = 8 KB between N
// groups and SBO = 1 KB between 8-row K groups.
template <bool kBMN>
__global__ void __launch_bounds__(192, 1)
    gemm_tn_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2, int M, int N,
                   int num_k, int r_steps, uint16_t* __restrict__ D, int accumulate, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_TILE;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * B_TILE);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;     // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (M + BM - 1) / BM, n_tiles = (N + BN - 1) / BN;
  const int total_tiles = m_tiles * n_tiles;
  const int k_iters = num_k + (r_steps > 0 ? 1 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      if (r_steps > 0) {
        tma_prefetch_desc(&tmA2);
        tma_prefetch_desc(&tmB2);
      }
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, m_tiles, n_tiles, mb, nb);
        const int m0 = mb * BM, n0 = nb * BN;
        for (int i = 0; i < k_iters; ++i, ++it) {
          const int s = it % STAGES, u = it / STAGES;
          if (it >= STAGES && !mbar_wait(&empty[s], (u - 1) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          if constexpr (!kBMN) {
            mbar_arrive_expect_tx(&full[s], A_TILE + B_TILE);
            if (i < num_k) {
              tma_load_2d(sA + s * A_TILE, &tmA, &full[s], i * BK, m0);
              tma_load_2d(sB + s * B_TILE, &tmB, &full[s], i * BK, n0);
            } else {
              tma_load_2d(sA + s * A_TILE, &tmA2, &full[s], 0, m0);
              tma_load_2d(sB + s * B_TILE, &tmB2, &full[s], 0, n0);
            }
          } else {
            if (i < num_k) {
              mbar_arrive_expect_tx(&full[s], A_TILE + B_TILE);
              tma_load_2d(sA + s * A_TILE, &tmA, &full[s], i * BK, m0);
              for (int j = 0; j < BN / 64; ++j)
                tma_load_2d(sB + s * B_TILE + j * 8192, &tmB, &full[s], n0 + 64 * j, i * BK);
            } else {
              // rank step: B2 is [r][N]; boxes of r16 rows at the same 8 KB spacing
              mbar_arrive_expect_tx(&full[s], A_TILE + (BN / 64) * r_steps * 16 * 128);
              tma_load_2d(sA + s * A_TILE, &tmA2, &full[s], 0, m0);
              for (int j = 0; j < BN / 64; ++j)
                tma_load_2d(sB + s * B_TILE + j * 8192, &tmB2, &full[s], n0 + 64 * j, 0);
            }
          }
        }
      }
      // Teardown: every issued copy must have landed before shared memory is released.
      for (int i = (it > STAGES ? it - STAGES : 0); i < it; ++i)
        mbar_wait_teardown(&full[i % STAGES], (i / STAGES) & 1, status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, BN, kBMN);
      int it = 0, tl = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++tl) {
        const int buf = tl & 1, use = tl >> 1;
        if (use > 0 && !mbar_wait(&acc_empty[buf], (use - 1) & 1, abort_flag, status)) break;
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(buf * BN);
        for (int i = 0; i < k_iters; ++i, ++it) {
          const int s = it % STAGES, u = it / STAGES;
          if (!mbar_wait(&full[s], u & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nsteps = i < num_k ? BK / 16 : r_steps;
          const uint64_t adesc = smem_desc_k128(smem_u32(sA + s * A_TILE));
          const uint64_t bdesc = kBMN ? smem_desc_mn128(smem_u32(sB + s * B_TILE), 8192, 1024)
                                      : smem_desc_k128(smem_u32(sB + s * B_TILE));
          // One K=16 step: A (K-major) +32 bytes inside the swizzle atom;
          // B +32 bytes (K-major) or +2 atoms of 8 rows = 2048 bytes (MN-major).
          const uint32_t bstep = kBMN ? (2048 >> 4) : 2;
          for (int kk = 0; kk < nsteps; ++kk)
            tc_mma_bf16_ss(acc, adesc + 2 * kk, bdesc + bstep * kk, idesc, (i > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        if (ok) tc_commit(&acc_full[buf]);
      }
      // Every MMA must be complete before the tensor memory is released.
      tc_commit(drain);
      mbar_wait_teardown(drain, 0, status);
    }
  } else {
    // Epilogue warps 2..5 own TMEM lane quadrants (warp % 4).
    const int q = warp & 3;
    int tl = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++tl) {
      const int buf = tl & 1, use = tl >> 1;
      // The tcgen05.ld below is warp-collective: take the decision warp-uniformly.
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], use & 1, abort_flag, status) ? 1 : 0) != 0;
      if (!ok) break;
      tc_fence_after();
      int mb, nb;
      tile_coords(t, m_tiles, n_tiles, mb, nb);
      const int row = mb * BM + q * 32 + lane;
      const uint32_t acc = tmem + static_cast<uint32_t>(buf * BN) + (static_cast<uint32_t>(q * 32) << 16);
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(acc + c * 32, v);
        tmem_wait_ld();
        store_row32_bf16(v, D, row, nb * BN + c * 32, M, N, accumulate);
      }
      // Hand the accumulator buffer back to the MMA warp.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Pair-CTA variant: a cluster of 2 CTAs computes 256 x 256 tiles with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16).  Each CTA loads its
// 128 rows of A and its 128 rows (N) of B per stage (32 KB instead of 48 KB,
// six stages), so the pair reads half of B per CTA and the shared-memory
// operand traffic per FLOP drops by a third.
//   warp 0      TMA producer of this CTA's halves; the transaction bytes of
//               both CTAs complete on the even CTA's stage barrier, which
//               the even CTA's producer arms with the pair's total
//   warp 1      TMEM allocation (both CTAs); in the even CTA, MMA issue
//   warps 2-5   epilogue of this CTA's 128 accumulator rows
// The MMA's commits reach both CTAs (multicast commit); the epilogue warps of
// both CTAs hand the accumulator back to the even CTA by remote arrive.
// ---------------------------------------------------------------------------

namespace {
constexpr int BM2 = 128;                 // rows of A per CTA (256 per pair)
constexpr int BN2 = 256;                 // N per tile; each CTA loads 128 rows of B
constexpr int BNH = BN2 / 2;
constexpr int STAGES2 = 6;
constexpr int A_TILE2 = BM2 * BK * 2;    // 16 KB
constexpr int B_TILE2 = BNH * BK * 2;    // 16 KB
constexpr size_t kL2PanelBudget = size_t(48) << 20;  // bytes of operand panels kept resident per group
constexpr int SMEM2_BYTES = 1024 + STAGES2 * (A_TILE2 + B_TILE2) + 512;
}  // namespace

template <bool kBMN>
__global__ void __launch_bounds__(192, 1)
    gemm_tn2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2, int M, int N,
                    int num_k, int r_steps, uint16_t* __restrict__ D, int accumulate, int* status, int group,
                    int along_n) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES2 * A_TILE2;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES2 * B_TILE2);
  uint64_t* empty = full + STAGES2;
  uint64_t* acc_full = empty + STAGES2;    // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2], even CTA
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t rank = cluster_ctarank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (M + 2 * BM2 - 1) / (2 * BM2), n_tiles = (N + BN2 - 1) / BN2;
  const int total_tiles = m_tiles * n_tiles;
  const int pair = static_cast<int>(cluster_id_x()), npairs = static_cast<int>(num_clusters_x());
  const int k_iters = num_k + (r_steps > 0 ? 1 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES2; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 8);  // 4 epilogue warps x 2 CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      if (r_steps > 0) {
        tma_prefetch_desc(&tmA2);
        tma_prefetch_desc(&tmB2);
      }
      // Stage barriers of the even CTA, in the cluster address space.
      const uint32_t full0 = map_to_cta(&full[0], 0);
      int it = 0;
      bool ok = true;
      for (int t = pair; t < total_tiles && ok; t += npairs) {
        int mb, nb;
        pair_tile_coords(t, m_tiles, n_tiles, group, along_n, mb, nb);
        const int m0 = mb * 2 * BM2 + static_cast<int>(rank) * BM2;
        const int n0 = nb * BN2 + static_cast<int>(rank) * BNH;
        for (int i = 0; i < k_iters; ++i, ++it) {
          const int s = it % STAGES2, u = it / STAGES2;
          if (it >= STAGES2 && !mbar_wait(&empty[s], (u - 1) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8u * static_cast<uint32_t>(s);
          if constexpr (!kBMN) {
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * (A_TILE2 + B_TILE2));
            if (i < num_k) {
              tma_load_2d_pair(sA + s * A_TILE2, &tmA, fb, i * BK, m0);
              tma_load_2d_pair(sB + s * B_TILE2, &tmB, fb, i * BK, n0);
            } else {
              tma_load_2d_pair(sA + s * A_TILE2, &tmA2, fb, 0, m0);
              tma_load_2d_pair(sB + s * B_TILE2, &tmB2, fb, 0, n0);
            }
          } else {
            if (i < num_k) {
              if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * (A_TILE2 + B_TILE2));
              tma_load_2d_pair(sA + s * A_TILE2, &tmA, fb, i * BK, m0);
              for (int j = 0; j < BNH / 64; ++j)
                tma_load_2d_pair(sB + s * B_TILE2 + j * 8192, &tmB, fb, n0 + 64 * j, i * BK);
            } else {
              if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * (A_TILE2 + (BNH / 64) * r_steps * 16 * 128));
              tma_load_2d_pair(sA + s * A_TILE2, &tmA2, fb, 0, m0);
              for (int j = 0; j < BNH / 64; ++j)
                tma_load_2d_pair(sB + s * B_TILE2 + j * 8192, &tmB2, fb, n0 + 64 * j, 0);
            }
          }
        }
      }
      // Teardown: the copies into this CTA's shared memory must have landed
      // before it goes.  The even CTA waits on its stage barriers (they count
      // both CTAs' bytes).  The odd CTA cannot wait on them; on the normal path
      // the even CTA consumed every stage before the final handshake, and
      // after an abort the odd CTA gives its copies in flight 100 us.
      if (rank == 0) {
        for (int i = (it > STAGES2 ? it - STAGES2 : 0); i < it; ++i)
          mbar_wait_teardown(&full[i % STAGES2], (i / STAGES2) & 1, status);
      } else if (!ok) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 100000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_bf16_f32(2 * BM2, BN2, kBMN);
      int it = 0, tl = 0;
      bool ok = true;
      for (int t = pair; t < total_tiles && ok; t += npairs, ++tl) {
        const int buf = tl & 1, use = tl >> 1;
        if (use > 0 && !mbar_wait_cluster(&acc_empty[buf], (use - 1) & 1, abort_flag, status)) break;
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(buf * BN2);
        for (int i = 0; i < k_iters; ++i, ++it) {
          const int s = it % STAGES2, u = it / STAGES2;
          if (!mbar_wait_cluster(&full[s], u & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nsteps = i < num_k ? BK / 16 : r_steps;
          const uint64_t adesc = smem_desc_k128(smem_u32(sA + s * A_TILE2));
          const uint64_t bdesc = kBMN ? smem_desc_mn128(smem_u32(sB + s * B_TILE2), 8192, 1024)
                                      : smem_desc_k128(smem_u32(sB + s * B_TILE2));
          const uint32_t bstep = kBMN ? (2048 >> 4) : 2;
          for (int kk = 0; kk < nsteps; ++kk)
            tc_mma_bf16_ss_pair(acc, adesc + 2 * kk, bdesc + bstep * kk, idesc, (i > 0 || kk > 0) ? 1u : 0u);
          tc_commit_pair(&empty[s], 0x3);
        }
        if (ok) tc_commit_pair(&acc_full[buf], 0x3);
      }
      // Every MMA (which also reads the odd CTA's shared memory) must be
      // complete before the pair's tensor memory and shared memory go.
      tc_commit_pair(drain, 0x1);
      mbar_wait_teardown(drain, 0, status);
    }
  } else {
    // Epilogue warps 2..5 own TMEM lane quadrants (warp % 4).
    const int q = warp & 3;
    const uint32_t acc_empty0 = map_to_cta(&acc_empty[0], 0);
    int tl = 0;
    for (int t = pair; t < total_tiles; t += npairs, ++tl) {
      const int buf = tl & 1, use = tl >> 1;
      const bool ok =
          __all_sync(0xffffffffu, mbar_wait_cluster(&acc_full[buf], use & 1, abort_flag, status) ? 1 : 0) != 0;
      if (!ok) break;
      tc_fence_after();
      int mb, nb;
      pair_tile_coords(t, m_tiles, n_tiles, group, along_n, mb, nb);
      const int row = mb * 2 * BM2 + static_cast<int>(rank) * BM2 + q * 32 + lane;
      const uint32_t acc = tmem + static_cast<uint32_t>(buf * BN2) + (static_cast<uint32_t>(q * 32) << 16);
      for (int c = 0; c < BN2 / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(acc + c * 32, v);
        tmem_wait_ld();
        store_row32_bf16(v, D, row, nb * BN2 + c * 32, M, N, accumulate);
      }
      // Hand the accumulator buffer back to the even CTA's MMA thread.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0 + 8u * static_cast<uint32_t>(buf));
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the pair's MMAs are complete; no remote signal is in flight
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

namespace {

// One device's answer for max_pair_clusters.
template <bool kBMN>
int query_pair_clusters() {
  if (cudaFuncSetAttribute(gemm_tn2_kernel<kBMN>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM2_BYTES) !=
      cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = SMEM2_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_tn2_kernel<kBMN>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  return n;
}

// Pair clusters that can be resident at once on the current device (0: the
// pair kernel cannot run there).  Sets the kernel's shared-memory limit on
// the device as it first asks.
template <bool kBMN>
int max_pair_clusters(int dev) {
  static DeviceValue cached;
  return cached.get(dev, [] { return query_pair_clusters<kBMN>(); });
}

template <bool kBMN>
cudaError_t launch_pair(const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap& tA2, const CUtensorMap& tB2,
                        const GemmArgs& a, int num_k, int r_steps, int clusters, cudaStream_t stream) {
  const int64_t m_tiles = (a.M + 2 * BM2 - 1) / (2 * BM2), n_tiles = (a.N + BN2 - 1) / BN2;
  const int64_t tiles = m_tiles * n_tiles;
  const int pairs = static_cast<int>(tiles < clusters ? tiles : clusters);
  // A 256-wide panel of either operand holds 256 x K bf16.
  const double panel = 256.0 * static_cast<double>(a.K) * 2.0;
  const RasterChoice rc = choose_raster(m_tiles, n_tiles, panel, panel, static_cast<double>(kL2PanelBudget));
  const int group = rc.group, along_n = rc.along_n;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = SMEM2_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_tn2_kernel<kBMN>, tA, tB, tA2, tB2, static_cast<int>(a.M), static_cast<int>(a.N),
                            num_k, r_steps, a.D, a.accumulate, a.status, group, along_n);
}

}  // namespace

cudaError_t launch_gemm_tn(const GemmArgs& a, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static DeviceOnce configured;
  e = configured.run(dev, [] {
    cudaError_t r = cudaFuncSetAttribute(gemm_tn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (r == cudaSuccess)
      r = cudaFuncSetAttribute(gemm_tn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    return r;
  });
  if (e != cudaSuccess) return e;
  const int clusters = a.b_mn_major ? max_pair_clusters<true>(dev) : max_pair_clusters<false>(dev);
  const bool pair = clusters > 0;
  // B (and B2) boxes: the pair kernel loads 128 rows of N per CTA.
  const uint32_t bn_box = pair ? static_cast<uint32_t>(BNH) : static_cast<uint32_t>(BN);
  CUtensorMap tA, tB, tA2, tB2;
  if (!encode_tensor_map_2d(&tA, a.A, a.M, a.K, BM, BK)) return cudaErrorInvalidValue;
  if (a.b_mn_major) {
    if (!encode_tensor_map_2d(&tB, a.B, a.K, a.N, BK, 64)) return cudaErrorInvalidValue;  // B stored [K][N]
  } else {
    if (!encode_tensor_map_2d(&tB, a.B, a.N, a.K, bn_box, BK, true, a.ldb)) return cudaErrorInvalidValue;
  }
  int r_steps = 0;
  if (a.A2 != nullptr && a.r > 0) {
    r_steps = (a.r + 15) / 16;
    if (!encode_tensor_map_2d(&tA2, a.A2, a.M, kRankPad, BM, BK)) return cudaErrorInvalidValue;
    if (a.b_mn_major) {
      // B2 stored [r][N]
      if (!encode_tensor_map_2d(&tB2, a.B2, a.r, a.N, static_cast<uint32_t>(16 * r_steps), 64))
        return cudaErrorInvalidValue;
    } else {
      // B2 stored [N][ldb2] with r valid columns (zero filled up to 64)
      if (!encode_tensor_map_2d(&tB2, a.B2, a.N, a.r, bn_box, BK, true, a.ldb2)) return cudaErrorInvalidValue;
    }
  } else {
    tA2 = tA;
    tB2 = tB;
  }
  const int num_k = static_cast<int>((a.K + BK - 1) / BK);
  if (pair) {
    return a.b_mn_major ? launch_pair<true>(tA, tB, tA2, tB2, a, num_k, r_steps, clusters, stream)
                        : launch_pair<false>(tA, tB, tA2, tB2, a, num_k, r_steps, clusters, stream);
  }
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  const int64_t tiles = ((a.M + BM - 1) / BM) * ((a.N + BN - 1) / BN);
  const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
  if (a.b_mn_major)
    gemm_tn_kernel<true><<<grid, 192, SMEM_BYTES, stream>>>(tA, tB, tA2, tB2, static_cast<int>(a.M),
                                                            static_cast<int>(a.N), num_k, r_steps, a.D, a.accumulate,
                                                            a.status);
  else
    gemm_tn_kernel<false><<<grid, 192, SMEM_BYTES, stream>>>(tA, tB, tA2, tB2, static_cast<int>(a.M),
                                                             static_cast<int>(a.N), num_k, r_steps, a.D, a.accumulate,
                                                             a.status);
  return cudaGetLastError();
}

}  // namespace qnf4
