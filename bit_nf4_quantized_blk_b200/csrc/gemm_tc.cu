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
// One CTA computes a 128 x 256 tile with a 4-stage TMA ring:
//   warp 0      TMA producer (one elected thread), 128B-swizzled tiles
//   warp 1      TMEM allocation + MMA issue (one thread): tcgen05.mma
//               kind::f16, M=128 N=256 K=16, fp32 accumulator in TMEM
//   warps 2-5   epilogue: tcgen05.ld 32 columns at a time -> bf16 -> global
// Every barrier wait is bounded (see common.cuh); a timeout aborts the CTA,
// which then waits (bounded) for its copies and MMAs in flight and frees its
// tensor memory before returning.  No cluster multicast is used.
#include "common.cuh"
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_TILE = BM * BK * 2;  // 16 KB
constexpr int B_TILE = BN * BK * 2;  // 32 KB
constexpr int TMEM_COLS = 256;
constexpr int SMEM_BYTES = 1024 + STAGES * (A_TILE + B_TILE) + 256;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace

// bf16 row-major [rows][cols] (cols contiguous), box box_rows x box_cols,
// 128-byte swizzle, zero fill outside the tensor.
bool encode_tensor_map_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                          uint32_t box_cols) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t gdim[2] = {cols, rows};
  const cuuint64_t gstride[1] = {cols * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

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
  uint64_t* acc_full = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int total = num_k + (r_steps > 0 ? 1 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
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
      int issued = 0;
      for (int i = 0; i < total; ++i) {
        const int s = i % STAGES, u = i / STAGES;
        if (i >= STAGES && !mbar_wait(&empty[s], (u - 1) & 1, abort_flag, status)) break;
        mbar_arrive_expect_tx(&full[s], A_TILE + B_TILE);
        if (i < num_k) {
          tma_load_2d(sA + s * A_TILE, &tmA, &full[s], i * BK, m0);
          tma_load_2d(sB + s * B_TILE, &tmB, &full[s], i * BK, n0);
        } else {
          tma_load_2d(sA + s * A_TILE, &tmA2, &full[s], 0, m0);
          tma_load_2d(sB + s * B_TILE, &tmB2, &full[s], 0, n0);
        }
        issued = i + 1;
      }
      // Teardown: every issued copy must have landed before shared memory is released.
      for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
        mbar_wait_teardown(&full[i % STAGES], (i / STAGES) & 1, status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, BN);
      for (int i = 0; i < total; ++i) {
        const int s = i % STAGES, u = i / STAGES;
        if (!mbar_wait(&full[s], u & 1, abort_flag, status)) break;
        tc_fence_after();
        const int nsteps = i < num_k ? BK / 16 : r_steps;
        const uint64_t adesc = smem_desc_k128(smem_u32(sA + s * A_TILE));
        const uint64_t bdesc = smem_desc_k128(smem_u32(sB + s * B_TILE));
        for (int kk = 0; kk < nsteps; ++kk) {
          // +32 bytes (16 bf16 of K) inside the 128-byte swizzle atom
          tc_mma_bf16_ss(tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&empty[s]);
      }
      tc_commit(acc_full);
      // The accumulator must be complete before the tensor memory is released.
      mbar_wait_teardown(acc_full, 0, status);
    }
  } else {
    // Epilogue warps 2..5 own TMEM lane quadrants (warp % 4).
    // The tcgen05.ld below is warp-collective: take the decision warp-uniformly.
    const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, status) ? 1 : 0) != 0;
    tc_fence_after();
    if (ok) {
      const int q = warp & 3;
      const int row = m0 + q * 32 + lane;
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + c * 32, v);
        tmem_wait_ld();
        const int col = n0 + c * 32;
        if (row >= M || col >= N) continue;
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
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

cudaError_t launch_gemm_tn(const GemmArgs& a, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  CUtensorMap tA, tB, tA2, tB2;
  if (!encode_tensor_map_2d(&tA, a.A, a.M, a.K, BM, BK)) return cudaErrorInvalidValue;
  if (!encode_tensor_map_2d(&tB, a.B, a.N, a.K, BN, BK)) return cudaErrorInvalidValue;
  int r_steps = 0;
  if (a.A2 != nullptr && a.r > 0) {
    if (!encode_tensor_map_2d(&tA2, a.A2, a.M, kRankPad, BM, BK)) return cudaErrorInvalidValue;
    if (!encode_tensor_map_2d(&tB2, a.B2, a.N, kRankPad, BN, BK)) return cudaErrorInvalidValue;
    r_steps = (a.r + 15) / 16;
  } else {
    tA2 = tA;
    tB2 = tB;
  }
  const int num_k = static_cast<int>((a.K + BK - 1) / BK);
  dim3 grid(static_cast<unsigned>((a.N + BN - 1) / BN), static_cast<unsigned>((a.M + BM - 1) / BM));
  gemm_tn_kernel<<<grid, 192, SMEM_BYTES, stream>>>(tA, tB, tA2, tB2, static_cast<int>(a.M), static_cast<int>(a.N),
                                                     num_k, r_steps, a.D, a.accumulate, a.status);
  return cudaGetLastError();
}

}  // namespace qnf4
