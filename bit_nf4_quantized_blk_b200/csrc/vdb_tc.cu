// V = dY B and the dB partials dY^T U from one pass over dY, on the
// tensor cores (sm_100a, tcgen05, one CTA per MMA).
//
// "QLoRA: NF4 storage, gradients and local integration", section "Exact CPU
// teaching quantizer and adapter gradient path": with U = X A^T,
//   dB = s dY^T U        [N][r]
//   V  = dY B            [M][r]   (dA = s V^T X and the dX rank term use it)
// Both products read dY, the largest operand of the LoRA side work; here
// every dY tile is loaded once and feeds both.
//
// A stage is one 128-token x 128-column tile of dY (two 64-column TMA boxes,
// 128-byte swizzle) with the matching tiles of B^T [16][N] and of the hi / lo
// bf16 split of U^T [16][M].  The tile is read by two MMA chains:
//   V:  D[128 tokens][16] += dY tile (A, K-major: rows = tokens, K = columns)
//                            x B^T tile (B, K-major)
//   dB: D[128 columns][16] += dY tile read as A MN-major (M = columns,
//                             K = tokens) x U^T hi tile, then x U^T lo tile
// CTA (zc, zm) covers up to kVtCT column tiles x a range of token tiles,
// token-tile major.  The V accumulator (16 TMEM columns) is double-buffered
// and drained to the partial vpart[zc][m][16] after each token tile; the dB
// accumulators (16 columns per column tile) live across the CTA's token
// tiles and are drained to dbpart[zm][n][16] at the end.  Two CTAs share an
// SM (two-stage rings): two producer threads keep the SM's TMA busier than one
// with a four-stage ring did (0.89 -> 0.83 ms for the step's side family).
// Partial sums are
// reduced in a fixed order by vdb_finalize_kernel (no atomics).
//
// Warps: 0 TMA producer; 1 TMEM allocation and MMA issue; 2-5 epilogue
// (TMEM lane quadrant = warp % 4).  Every barrier wait is bounded.
#include "common.cuh"
#include "device_once.h"
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kVtTok = 128;                    // tokens per tile
constexpr int kVtCol = 128;                    // dY columns per tile
constexpr int kVtStages = 2;                   // two CTAs share an SM (two producers in flight)
constexpr int kVtPerSm = 2;
constexpr int kVtGTile = kVtTok * kVtCol * 2;  // 32 KB: two [128][64] boxes
constexpr int kVtGBox = kVtGTile / 2;          // 16 KB
constexpr int kVtSmall = 16 * kVtCol * 2;      // 4 KB: two [16][64] boxes
constexpr int kVtSmallBox = kVtSmall / 2;      // 2 KB
constexpr int kVtStage = kVtGTile + 3 * kVtSmall;  // 44 KB
constexpr int kVtCTMax = 8;                    // column tiles per CTA
constexpr int kVtThreads = 192;
constexpr uint32_t kVtTmemCols = 256;          // V: 2 x 16, dB: up to 8 x 16
constexpr int kVtSmem = 1024 + kVtStages * kVtStage + 256;

struct VtBarriers {
  uint64_t full[kVtStages];
  uint64_t empty[kVtStages];
  uint64_t v_full[2];
  uint64_t v_empty[2];
  uint64_t db_full;
  uint64_t drain;
  uint32_t tmem;
  int abort_flag;
};

__device__ __forceinline__ bool vt_warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag, status);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok) (void)mbar_try_wait(bar, parity);
  return ok;
}

// tcgen05.wait::ld that hands the loaded registers on, so no use of them can
// be scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])
               :
               : "memory");
}

// 16 fp32 columns of one accumulator row to dst (16-byte aligned).
__device__ __forceinline__ void store16(float* dst, const uint32_t (&v)[16]) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d4[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]), __uint_as_float(v[4 * q + 2]),
                        __uint_as_float(v[4 * q + 3]));
}

}  // namespace

__global__ void __launch_bounds__(kVtThreads, kVtPerSm)
    vdb_tc_kernel(const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmBt,
                  const __grid_constant__ CUtensorMap tmUh, const __grid_constant__ CUtensorMap tmUl, int64_t M,
                  int64_t N, int ct, int tt, float* __restrict__ vpart, float* __restrict__ dbpart, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  VtBarriers* bars = reinterpret_cast<VtBarriers*>(smem + kVtStages * kVtStage);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int zc = blockIdx.x, zm = blockIdx.y;
  const int ctiles = static_cast<int>((N + kVtCol - 1) / kVtCol);
  const int mtiles = static_cast<int>((M + kVtTok - 1) / kVtTok);
  const int tc0 = zc * ct, tm0 = zm * tt;
  const int ntc = min(ct, ctiles - tc0), ntm = min(tt, mtiles - tm0);
  const int nsteps = ntc * ntm;  // step i: token tile i / ntc, column tile i % ntc

  if (threadIdx.x == 0) {
    for (int s = 0; s < kVtStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->v_full[b], 1);
      mbar_init(&bars->v_empty[b], 4);  // the four epilogue warps
    }
    mbar_init(&bars->db_full, 1);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem, kVtTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % kVtStages, u = i / kVtStages;
        if (i >= kVtStages && !mbar_wait(&bars->empty[s], (u - 1) & 1, abort_flag, status)) break;
        uint8_t* st = smem + s * kVtStage;
        const int c = (tc0 + i % ntc) * kVtCol, m = (tm0 + i / ntc) * kVtTok;
        mbar_arrive_expect_tx(&bars->full[s], kVtStage);
        tma_load_2d(st, &tmG, &bars->full[s], c, m);
        tma_load_2d(st + kVtGBox, &tmG, &bars->full[s], c + 64, m);
        tma_load_2d(st + kVtGTile, &tmBt, &bars->full[s], c, 0);
        tma_load_2d(st + kVtGTile + kVtSmallBox, &tmBt, &bars->full[s], c + 64, 0);
        tma_load_2d(st + kVtGTile + kVtSmall, &tmUh, &bars->full[s], m, 0);
        tma_load_2d(st + kVtGTile + kVtSmall + kVtSmallBox, &tmUh, &bars->full[s], m + 64, 0);
        tma_load_2d(st + kVtGTile + 2 * kVtSmall, &tmUl, &bars->full[s], m, 0);
        tma_load_2d(st + kVtGTile + 2 * kVtSmall + kVtSmallBox, &tmUl, &bars->full[s], m + 64, 0);
        issued = i + 1;
      }
      // Every copy into shared memory has landed before the CTA can exit.
      for (int i = (issued > kVtStages ? issued - kVtStages : 0); i < issued; ++i)
        mbar_wait_teardown(&bars->full[i % kVtStages], (i / kVtStages) & 1, status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // V: A K-major (tokens x columns), B K-major; dB: A MN-major (columns
      // x tokens), B K-major.  M = 128, N = 16.
      constexpr uint32_t idesc_v = idesc_bf16_f32(128, 16);
      constexpr uint32_t idesc_db = idesc_bf16_f32(128, 16) | (1u << 15);
      bool ok = true;
      for (int i = 0; i < nsteps && ok; ++i) {
        const int s = i % kVtStages, u = i / kVtStages;
        const int tm = i / ntc, tc = i % ntc, vb = tm & 1;
        if (tc == 0 && tm >= 2 && !mbar_wait(&bars->v_empty[vb], ((tm - 2) >> 1) & 1, abort_flag, status)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&bars->full[s], u & 1, abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * kVtStage);
        // dY tile as the MN-major A of dB: 64-column groups 16 KB apart
        // (the two boxes), 8-token groups 1 KB apart; a K = 16 step is 16
        // tokens = 2 KB.
        const uint64_t g_mn = smem_desc_mn128(st, kVtGBox, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t box = static_cast<uint32_t>(kk >> 2), sub = static_cast<uint32_t>(kk & 3);
          // V: K = 16 columns at kk * 16 (box kk / 4, +32 bytes per step inside it).
          const uint64_t a_v = smem_desc_k128(st + box * kVtGBox) + 2 * sub;
          const uint64_t b_v = smem_desc_k128(st + kVtGTile + box * kVtSmallBox) + 2 * sub;
          tc_mma_bf16_ss(tmem + static_cast<uint32_t>(vb * 16), a_v, b_v, idesc_v, (tc > 0 || kk > 0) ? 1u : 0u);
          // dB: K = 16 tokens at kk * 16.
          const uint64_t a_db = g_mn + static_cast<uint64_t>(kk) * (2048 >> 4);
          const uint64_t b_hi = smem_desc_k128(st + kVtGTile + kVtSmall + box * kVtSmallBox) + 2 * sub;
          const uint64_t b_lo = smem_desc_k128(st + kVtGTile + 2 * kVtSmall + box * kVtSmallBox) + 2 * sub;
          const uint32_t acc_db = tmem + 32u + static_cast<uint32_t>(tc * 16);
          tc_mma_bf16_ss(acc_db, a_db, b_hi, idesc_db, (tm > 0 || kk > 0) ? 1u : 0u);
          tc_mma_bf16_ss(acc_db, a_db, b_lo, idesc_db, 1u);
        }
        tc_commit(&bars->empty[s]);
        if (tc == ntc - 1) tc_commit(&bars->v_full[vb]);
      }
      if (ok) tc_commit(&bars->db_full);
      tc_commit(&bars->drain);
      mbar_wait_teardown(&bars->drain, 0, status);
    }
  } else {
    // Epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31.
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    bool ok = true;
    for (int tm = 0; tm < ntm && ok; ++tm) {
      const int vb = tm & 1;
      ok = vt_warp_wait(&bars->v_full[vb], (tm >> 1) & 1, abort_flag, status);
      if (!ok) break;
      tc_fence_after();
      uint32_t v[16];
      tmem_ld_32x32b_x16(tmem + lane_off + static_cast<uint32_t>(vb * 16), v);
      tmem_wait_ld16(v);
      const int64_t m = static_cast<int64_t>(tm0 + tm) * kVtTok + q * 32 + lane;
      if (m < M) store16(vpart + (static_cast<int64_t>(zc) * M + m) * 16, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->v_empty[vb]);
    }
    if (ok && vt_warp_wait(&bars->db_full, 0, abort_flag, status)) {
      tc_fence_after();
      for (int tc = 0; tc < ntc; ++tc) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem + lane_off + 32u + static_cast<uint32_t>(tc * 16), v);
        tmem_wait_ld16(v);
        const int64_t n = static_cast<int64_t>(tc0 + tc) * kVtCol + q * 32 + lane;
        if (n < N) store16(dbpart + (static_cast<int64_t>(zm) * N + n) * 16, v);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kVtTmemCols);
  }
}

// The three rank-16 transposes of one call in one launch: B^T [16][N] from
// B [N][ldb], and U^T hi / lo [16][ldm] from uhi / ulo [M][64];
// dst[j][row] = src[row][j] for j < r, 0 for r <= j < 16.  Consecutive
// threads take consecutive rows of one j, so the stores are contiguous.
__global__ void rank16_transpose3_kernel(const uint16_t* __restrict__ B, int64_t ldb, int64_t N,
                                         const uint16_t* __restrict__ uhi, const uint16_t* __restrict__ ulo,
                                         const float* __restrict__ u32, int64_t M, int64_t ldm, int r,
                                         uint16_t* __restrict__ bt, uint16_t* __restrict__ uht,
                                         uint16_t* __restrict__ ult) {
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint16_t* src;
  uint16_t* dst;
  int64_t ld, rows, ldd;
  if (i < 16 * N) {
    src = B, dst = bt, ld = ldb, rows = N, ldd = N;
  } else if (u32 != nullptr) {
    // The saved fp32 U [M][r]: each thread forms both halves of one element,
    // hi = bf16(u) and lo = bf16(u - hi).
    i -= 16 * N;
    if (i >= 16 * M) return;
    const int j = static_cast<int>(i / M);
    const int64_t row = i % M;
    const float v = j < r ? u32[row * r + j] : 0.0f;
    const uint32_t h = pack_bf16x2(v, 0.0f) & 0xFFFFu;
    uht[j * ldm + row] = static_cast<uint16_t>(h);
    ult[j * ldm + row] = static_cast<uint16_t>(pack_bf16x2(v - bf16_bits_to_float(h), 0.0f) & 0xFFFFu);
    return;
  } else {
    i -= 16 * N;
    if (i >= 32 * M) return;
    const bool lo = i >= 16 * M;
    if (lo) i -= 16 * M;
    src = lo ? ulo : uhi, dst = lo ? ult : uht, ld = kRankPad, rows = M, ldd = ldm;
  }
  const int j = static_cast<int>(i / rows);
  const int64_t row = i % rows;
  dst[j * ldd + row] = j < r ? src[row * ld + j] : static_cast<uint16_t>(0);
}

VdbTcGrid vdb_tc_grid(int64_t M, int64_t N) {
  // Sized for one wave of two CTAs per SM on a 148-SM B200 (a device with
  // fewer SMs runs the same grid in more waves; the workspace size depends
  // on shapes only).
  constexpr int sms = 148 * kVtPerSm;
  const int64_t ctiles = (N + kVtCol - 1) / kVtCol, mtiles = (M + kVtTok - 1) / kVtTok;
  // As many column tiles per CTA as keep every SM busy (fewer for narrow
  // weights), then the token tiles split to about one wave.
  int ct = kVtCTMax;
  while (ct > 1 && ((ctiles + ct - 1) / ct) * mtiles < sms) ct /= 2;
  VdbTcGrid g;
  g.ct = ct;
  g.ncb = static_cast<int>((ctiles + ct - 1) / ct);
  int64_t ntb = sms / g.ncb;  // no second, partial wave
  if (ntb < 1) ntb = 1;
  if (ntb > mtiles) ntb = mtiles;
  g.tt = static_cast<int>((mtiles + ntb - 1) / ntb);
  g.ntb = static_cast<int>((mtiles + g.tt - 1) / g.tt);
  return g;
}

size_t vdb_tc_partial_bytes(int64_t M, int64_t N) {
  const VdbTcGrid g = vdb_tc_grid(M, N);
  return (static_cast<size_t>(g.ncb) * static_cast<size_t>(M) + static_cast<size_t>(g.ntb) * static_cast<size_t>(N)) *
         16 * sizeof(float);
}

cudaError_t launch_vdb_tc(const uint16_t* G, int64_t M, int64_t N, const uint16_t* B, int64_t ldb,
                          const uint16_t* uhi, const uint16_t* ulo, const float* u32, int r, float scale, float* part,
                          uint16_t* bt, uint16_t* uht, uint16_t* ult, uint16_t* vs, uint16_t* vhi, uint16_t* vlo,
                          float* dB, const BlockScalesJob& bs, int* status, cudaStream_t stream) {
  if (r < 1 || r > 16) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static DeviceOnce configured;
  e = configured.run(dev, [] {
    return cudaFuncSetAttribute(vdb_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kVtSmem);
  });
  if (e != cudaSuccess) return e;
  // B^T [16][N] and the hi / lo split of U^T [16][ldm]: the MMAs' K-major
  // B operands.
  const int64_t ldm = vdb_tc_ldm(M);
  const int64_t items = 16 * N + (u32 != nullptr ? 16 : 32) * M;
  rank16_transpose3_kernel<<<static_cast<unsigned>((items + 255) / 256), 256, 0, stream>>>(B, ldb, N, uhi, ulo, u32, M,
                                                                                          ldm, r, bt, uht, ult);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap tg, tbt, tuh, tul;
  if (!encode_tensor_map_2d(&tg, G, M, N, kVtTok, 64)) return cudaErrorInvalidValue;
  if (!encode_tensor_map_2d(&tbt, bt, 16, N, 16, 64)) return cudaErrorInvalidValue;
  if (!encode_tensor_map_2d(&tuh, uht, 16, M, 16, 64, true, ldm)) return cudaErrorInvalidValue;
  if (!encode_tensor_map_2d(&tul, ult, 16, M, 16, 64, true, ldm)) return cudaErrorInvalidValue;
  const VdbTcGrid g = vdb_tc_grid(M, N);
  float* vpart = part;
  float* dbpart = part + static_cast<int64_t>(g.ncb) * M * 16;
  vdb_tc_kernel<<<dim3(static_cast<unsigned>(g.ncb), static_cast<unsigned>(g.ntb)), kVtThreads, kVtSmem, stream>>>(
      tg, tbt, tuh, tul, M, N, g.ct, g.tt, vpart, dbpart, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_vdb_finalize(vpart, g.ncb, dbpart, g.ntb, M, N, r, scale, vs, vhi, vlo, dB, bs, stream);
}

}  // namespace qnf4
