// Training-shaped GEMM of the QLoRA linear with the 4-bit weight decoded
// inside the kernel (sm_100a, tcgen05 pair-CTA MMAs).
//
//   forward         Y  [M][N_w] = X  [M][K_w] W_hat^T + (s U) B^T
//   backward-input  dX [M][K_w] = dY [M][N_w] W_hat   + (s V) A
//
// "QLoRA Deep Dive: 4-bit NormalFloat & Double Quantization Internals",
// section "The Quantization Process in QLoRA": a block's 4-bit codes and its
// constant are loaded, multiplied back and used directly in the computation;
// "FT-02: QLoRA -- Fine-Tuning with Quantization", section "Reading the
// result: the three lines that decide memory": the frozen weight stays in 4
// bits and is dequantized on the fly in every forward (and backward) pass.
// The gradient formulas are those of "QLoRA: NF4 storage, gradients and local
// integration", section "Exact CPU teaching quantizer and adapter gradient
// path".
//
// The dense bf16 weight never exists in HBM: each stage of the weight operand
// is decoded from its packed codes and block-scale codes straight into the
// 128-byte-swizzled shared-memory layout the tensor core reads.  One stage
// covers 64 values of the reduction, and in both directions one 128-byte row
// of the stage tile is exactly one quantization block (64 consecutive values
// of one weight row), so a decoding thread owns one block per stage:
//   forward  (B operand K-major):  tile row = weight row n, the 64 values of
//            block (n, k0 / 64);
//   backward (B operand MN-major): tile row = reduction index n, 64 output
//            columns k0..k0+63 of weight row n = block (n, k0 / 64).
// Decoded values are bf16(fp32(L[code] * a)) with the block scale
// a = fp32(fp32(t * c2) + mu) (t = fp32(q / 127) for int8 codes, the E4M3
// value for FP8 codes) or the stored fp32 absmax -- the same bits the dense
// dequantize entry point writes.  The thread first forms the block's 16
// possible bf16 values (16 multiplies, 8 conversions), splits them into a
// low-byte and a high-byte table of four registers each, and then looks up
// four codes at a time with byte permutes whose selectors are the packed
// nibbles themselves (bit 3 of a code picks the upper half of the table).
//
// Pair-CTA layout (cluster of 2, 512 x 256 output tile per pair):
//   Each decoded weight stage feeds the MMAs of two 256-row halves of A, so
//   every decoded value serves 512 rows of the activations; decoding then
//   takes half the share of the SM's issue slots and shared-memory port that
//   a 256-row tile would.  The two halves' accumulators fill tensor memory
//   (2 x 256 columns), so the accumulator is single-buffered: the epilogue
//   drains it while the producers already fill the next tile's stages.
//   warp 0      TMA producer of this CTA's 2 x 128 rows of A (X or dY) per
//               stage, and of the rank step's tiles; the even CTA arms the
//               stage's barrier (full) with both CTAs' bytes
//   warp 1      TMEM allocation (both CTAs); in the even CTA, MMA issue:
//               tcgen05.mma.cta_group::2 kind::f16, M = 256, N = 256, K = 16,
//               one accumulator per half
//   warps 2-5   epilogue of this CTA's 2 x 128 accumulator rows (each lane
//               one row; 32-byte stores, so a lane writes whole sectors)
//   warps 6-8, 10-12, 14, 15
//               weight decoders: two groups of four warps take alternate
//               stages; each thread reads its block's codes and scale from
//               the code ring, decodes the block into the stage's tile,
//               fences its shared-memory writes for the async proxy, and its
//               warp arrives on the even CTA's stage barrier (full) with a
//               CTA-scope arrive (mbar_arrive_remote)
//   warp 9      code ring producer: per stage, this CTA's packed codes and
//               decoded block scales by TMA into a 4-slot ring
//   warp 13     idle
// No decoder shares the MMA warp's scheduler (warp % 4 == 1): decoders there
// take issue slots from the MMA issue and slow the tensor pipe by 10-15%;
// only the light code-ring producer and one epilogue warp sit beside it.
// Tiles are whole (512 rows) except in a last partial wave that would use at
// most half of the pairs: those tiles are split into their two 256-row
// halves, which run on twice as many pairs in half the time.
// A stage is complete when its copies have landed and the eight decode warps
// of the pair have arrived: one barrier, so the MMA issuer checks one phase
// per stage.  The issuer is a single thread whose scalar work between two
// stages' MMAs delays the tensor pipe, so its loop is kept lean: the slot
// descriptors are the slot-0 descriptors plus constant offsets, and a full
// stage's eight MMAs are unrolled.  At teardown the even producer waits for the
// last stages' phases (so for the copies of both CTAs) and then signals the
// odd CTA (`drained`), which waits for that before its shared memory can go.
// The rank-r LoRA term is one more pipeline step of ceil(r/16) MMAs into the
// same accumulator, its operands loaded by TMA.  No TMA load uses cluster
// multicast; the MMA's tcgen05.commit is delivered to both CTAs of the pair
// (an mbarrier arrive, not a load).  Every barrier wait is bounded in time
// (common.cuh).
#include "common.cuh"
#include "gemm_common.cuh"
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int BM = 128;          // rows of A per CTA and half (256 per pair and half)
constexpr int kHalves = 2;       // 256-row halves of A per pair tile
constexpr int BN = 256;          // output columns per pair tile
constexpr int BNH = BN / 2;      // B rows (forward) / output columns (backward) per CTA
constexpr int BK = 64;           // reduction values per stage (one quantization block)
constexpr int STAGES = 4;
constexpr int A_TILE = BM * BK * 2;          // 16 KB per half
constexpr int A_STAGE = kHalves * A_TILE;    // 32 KB
constexpr int B_TILE = BNH * BK * 2;         // 16 KB
constexpr int TMEM_COLS = 512;               // one 128 x 256 fp32 accumulator per half, per CTA
constexpr int kDecodeGroups = 2;
constexpr int kFirstDecodeWarp = 6;
constexpr int kCodeWarp = 9;     // producer of the code ring
constexpr int kThreads = 32 * 16;
// Decoder index 0..7 of a warp (-1: not a decoder): warps 6..15 except those
// on the MMA warp's scheduler (9, 13).
__device__ __forceinline__ int decoder_index(int warp) {
  return (warp < kFirstDecodeWarp || (warp & 3) == 1) ? -1 : (warp - kFirstDecodeWarp) - ((warp - 5) >> 2);
}
constexpr int kDecodedArrivals = 2 * 4;    // the four decode warps of each CTA that handle a stage
// Code ring (per CTA): a stage's packed codes (4 KB) and decoded block scales
// (fp32 boxes of 4 blocks per weight row: 2 KB forward, 1 KB backward).
constexpr int kCodeStages = 4;             // a multiple of kDecodeGroups: a slot always serves one group
constexpr int CODE_SLOT = 6144;
constexpr int kCodeBytes = 4096;
constexpr int SMEM_BYTES = 1024 + STAGES * (A_STAGE + B_TILE) + kCodeStages * CODE_SLOT + 512;
static_assert(kCodeStages % kDecodeGroups == 0, "a code slot must always serve the same decode group");
constexpr size_t kL2PanelBudget = size_t(48) << 20;

// A pair's work item t: pair tile t of the raster whole, or (from full_tiles
// on) one 256-row half of a tile of the last wave.  mh0 is its first 256-row
// block of A, nh the number of 256-row blocks (0: past the end of A).
struct WorkItem {
  int mh0, nb, nh;
};

__device__ __forceinline__ WorkItem work_item(int t, const Nf4GemmParams& p, int m_tiles, int n_tiles, int m256) {
  int tile = t, half = -1;
  if (t >= p.full_tiles) {
    tile = p.full_tiles + ((t - p.full_tiles) >> 1);
    half = (t - p.full_tiles) & 1;
  }
  int mb, nb;
  pair_tile_coords(tile, m_tiles, n_tiles, p.group, p.along_n, mb, nb);
  WorkItem w;
  w.nb = nb;
  if (half < 0) {
    w.mh0 = kHalves * mb;
    w.nh = min(kHalves, m256 - w.mh0);
  } else {
    w.mh0 = kHalves * mb + half;
    w.nh = w.mh0 < m256 ? 1 : 0;
  }
  return w;
}

// tcgen05.wait::ld that also hands the loaded registers on, so no use of
// them can be scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Four bf16 values from four 4-bit codes: `m` holds the codes' low three bits
// in its four low nibbles (the permute selectors), `h` their bit 3 (0 / 1 per
// nibble).  lo*/hi* are the low and high bytes of the 16-entry value table.
__device__ __forceinline__ void lookup4(uint32_t m, uint32_t h, uint32_t lo0, uint32_t lo1, uint32_t lo2, uint32_t lo3,
                                        uint32_t hi0, uint32_t hi1, uint32_t hi2, uint32_t hi3, uint32_t& out01,
                                        uint32_t& out23) {
  const uint32_t upper = prmt(0x0000FF00u, 0u, h);  // byte i = 0xFF where code i >= 8
  const uint32_t lo = (prmt(lo0, lo1, m) & ~upper) | (prmt(lo2, lo3, m) & upper);
  const uint32_t hi = (prmt(hi0, hi1, m) & ~upper) | (prmt(hi2, hi3, m) & upper);
  out01 = prmt(lo, hi, 0x5140u);  // value 0 in the low half, value 1 in the high half
  out23 = prmt(lo, hi, 0x7362u);
}

// Decode one quantization block (64 codes in w, element 2i in the low nibble
// of byte i) with scale `a` into a 128-byte row of a 128B-swizzled tile at
// shared address `row`: 16-byte chunk j (values 8j..8j+7) goes to chunk
// position j ^ sw.
__device__ __forceinline__ void decode_block_to_smem(uint32_t row, uint32_t sw, const uint32_t (&w)[8], float a,
                                                     const float (&L)[16]) {
  uint32_t P[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) P[i] = pack_bf16x2(__fmul_rn(L[2 * i], a), __fmul_rn(L[2 * i + 1], a));
  // P[i] bytes: (lo 2i, hi 2i, lo 2i+1, hi 2i+1)
  const uint32_t lo0 = prmt(P[0], P[1], 0x6420u), lo1 = prmt(P[2], P[3], 0x6420u);
  const uint32_t lo2 = prmt(P[4], P[5], 0x6420u), lo3 = prmt(P[6], P[7], 0x6420u);
  const uint32_t hi0 = prmt(P[0], P[1], 0x7531u), hi1 = prmt(P[2], P[3], 0x7531u);
  const uint32_t hi2 = prmt(P[4], P[5], 0x7531u), hi3 = prmt(P[6], P[7], 0x7531u);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t m = w[j] & 0x77777777u;
    const uint32_t h = (w[j] >> 3) & 0x11111111u;
    uint32_t o0, o1, o2, o3;
    lookup4(m, h, lo0, lo1, lo2, lo3, hi0, hi1, hi2, hi3, o0, o1);
    lookup4(m >> 16, h >> 16, lo0, lo1, lo2, lo3, hi0, hi1, hi2, hi3, o2, o3);
    st_shared_v4(row + ((static_cast<uint32_t>(j) ^ sw) << 4), o0, o1, o2, o3);
  }
}


// Store 32 fp32 accumulator columns of one output row as bf16 with two
// 32-byte stores (D rows 32-byte aligned: N % 16 == 0, 32-byte aligned base).
// A segment that reaches past column N takes the element-wise path.
__device__ __forceinline__ void store_row32_bf16_wide(const uint32_t (&v)[32], uint16_t* __restrict__ D, int row,
                                                      int col, int M, int N) {
  if (row >= M || col >= N) return;
  if (col + 32 > N) {
    store_row32_bf16(v, D, row, col, M, N, 0);
    return;
  }
  uint32_t lo[8], hi[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    lo[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
    hi[e] = pack_bf16x2(__uint_as_float(v[16 + 2 * e]), __uint_as_float(v[16 + 2 * e + 1]));
  }
  uint16_t* dst = D + static_cast<int64_t>(row) * N + col;
  st_stream_v8(dst, lo);
  st_stream_v8(dst + 16, hi);
}

__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "r"(addr) : "memory");
}

__device__ __forceinline__ float ld_shared_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// Warp-wide bounded wait: lane 0 polls (the other lanes idle at the shuffle,
// so a waiting warp takes few issue slots), then every lane acquires the
// completed phase itself.  Returns false (warp-uniformly) on abort / timeout.
// `suspend`: lane 0's tries may suspend it (a long wait beside the MMA warp).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                                          uint64_t lim, bool cluster, bool suspend = false) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0)
    ok = suspend   ? mbar_wait_suspend(bar, parity, cluster, abort_flag, status, lim)
         : cluster ? mbar_wait_cluster(bar, parity, abort_flag, status, lim)
                   : mbar_wait(bar, parity, abort_flag, status, lim);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok) {
    if (cluster)
      (void)mbar_try_wait_cluster(bar, parity);
    else
      (void)mbar_try_wait(bar, parity);
  }
  return ok;
}

}  // namespace

template <bool kBwd>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_nf4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                    const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmP,
                    const __grid_constant__ CUtensorMap tmS, const __grid_constant__ Nf4GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE;
  uint8_t* sC = sB + STAGES * B_TILE;    // code ring
  uint64_t* full = reinterpret_cast<uint64_t*>(sC + kCodeStages * CODE_SLOT);  // even CTA: copies + decode warps
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;    // the accumulators hold a finished tile
  uint64_t* acc_empty = acc_full + 1;     // even CTA: both CTAs' epilogues drained them
  uint64_t* drain = acc_empty + 1;
  uint64_t* drained = drain + 1;          // odd CTA: every copy of the pair has landed
  uint64_t* never = drained + 1;          // diagnostic: a barrier nothing arrives at
  uint64_t* cfull = never + 1;            // [kCodeStages] code ring: TMA bytes landed
  uint64_t* cempty = cfull + kCodeStages; // [kCodeStages] code ring: the group's four warps read the slot
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cempty + kCodeStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t rank = cluster_ctarank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = p.M, N = p.N, num_k = p.num_k, r_steps = p.r_steps;
  const int m256 = (M + 2 * BM - 1) / (2 * BM);
  const int m_tiles = (m256 + kHalves - 1) / kHalves, n_tiles = (N + BN - 1) / BN;
  const int items = p.items;
  const int pair = static_cast<int>(cluster_id_x()), npairs = static_cast<int>(num_clusters_x());
  const int k_iters = num_k + (r_steps > 0 ? 1 : 0);
  int* status = p.status;
  const uint64_t lim = p.wait_limit_ns;  // pipeline waits (teardown waits keep the full limit)

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1 + kDecodedArrivals);  // the producer's expect-tx arrive and the decode warps
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);  // 4 epilogue warps x 2 CTAs
    mbar_init(drain, 1);
    mbar_init(drained, 1);
    mbar_init(never, 1);
    for (int c = 0; c < kCodeStages; ++c) {
      mbar_init(&cfull[c], 1);
      mbar_init(&cempty[c], 4);
    }
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
      if (r_steps > 0) {
        tma_prefetch_desc(&tmA2);
        tma_prefetch_desc(&tmB2);
      }
      const uint32_t full0 = map_to_cta(&full[0], 0);
      int it = 0;
      bool ok = true;
      for (int t = pair; t < items && ok; t += npairs) {
        const WorkItem wi = work_item(t, p, m_tiles, n_tiles, m256);
        if (wi.nh == 0) continue;
        const int m0 = wi.mh0 * 2 * BM + static_cast<int>(rank) * BM;  // this CTA's rows of the first half
        const int n0 = wi.nb * BN + static_cast<int>(rank) * BNH;
        for (int i = 0; i < k_iters; ++i, ++it) {
          const int s = it % STAGES, u = it / STAGES;
          if (it >= STAGES && !mbar_wait(&empty[s], (u - 1) & 1, abort_flag, status, lim)) {
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8u * static_cast<uint32_t>(s);
          uint8_t* const a_st = sA + s * A_STAGE;
          if (i < num_k) {
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * wi.nh * A_TILE);
            for (int h = 0; h < wi.nh; ++h) tma_load_2d_pair(a_st + h * A_TILE, &tmA, fb, i * BK, m0 + h * 2 * BM);
          } else if constexpr (!kBwd) {
            // rank step: A2 = s U [M][64], B2 = LoRA B [N_w][r] (zero filled to 64)
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * (wi.nh * A_TILE + B_TILE));
            for (int h = 0; h < wi.nh; ++h) tma_load_2d_pair(a_st + h * A_TILE, &tmA2, fb, 0, m0 + h * 2 * BM);
            tma_load_2d_pair(sB + s * B_TILE, &tmB2, fb, 0, n0);
          } else {
            // rank step: A2 = s V [M][64], B2 = LoRA A [r][K_w] as MN-major boxes
            if (rank == 0)
              mbar_arrive_expect_tx(&full[s], 2 * (wi.nh * A_TILE + (BNH / 64) * r_steps * 16 * 128));
            for (int h = 0; h < wi.nh; ++h) tma_load_2d_pair(a_st + h * A_TILE, &tmA2, fb, 0, m0 + h * 2 * BM);
            for (int j = 0; j < BNH / 64; ++j)
              tma_load_2d_pair(sB + s * B_TILE + j * 8192, &tmB2, fb, n0 + 64 * j, 0);
          }
        }
      }
      // Teardown: the copies into both CTAs' shared memory must have landed
      // before either goes.  Every copy of a stage completes on the even
      // CTA's copy barrier, so the even producer waits for the last stages
      // it armed (both CTAs' bytes) and then tells the odd CTA, which waits
      // for that word.  (Both producers wait on the same released stages, so
      // they stop after the same number of issued stages.)
      if (rank == 0) {
        for (int i = (it > STAGES ? it - STAGES : 0); i < it; ++i)
          mbar_wait_teardown(&full[i % STAGES], (i / STAGES) & 1, status);
        mbar_arrive_cluster(map_to_cta(drained, 1));
      } else {
        mbar_wait_teardown(drained, 0, status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_bf16_f32(2 * BM, BN, kBwd);
      // Stage descriptors: the start-address field (bits 0..13, address >> 4)
      // of slot s is the slot-0 descriptor's plus the slot's offset >> 4
      // (shared addresses stay below 256 KB, so the field cannot overflow).
      const uint64_t a_desc0 = smem_desc_k128(smem_u32(sA));
      const uint64_t b_desc0 = kBwd ? smem_desc_mn128(smem_u32(sB), 8192, 1024) : smem_desc_k128(smem_u32(sB));
      constexpr uint32_t kAStage16 = A_STAGE >> 4, kATile16 = A_TILE >> 4, kBTile16 = B_TILE >> 4;
      // One K = 16 step: A (K-major) +32 bytes inside the swizzle atom;
      // B +32 bytes (K-major) or +2 atoms of 8 rows = 2048 bytes (MN-major).
      constexpr uint32_t kBStep = kBwd ? (2048 >> 4) : 2;
      int it = 0, tl = 0;
      // Diagnostic launch: the issuer first waits on a barrier nothing
      // arrives at, so its wait runs out and the whole pair takes the abort
      // path (every other wait then ends on the abort flag or its own limit).
      bool ok = !p.debug_stall || mbar_wait(never, 0, abort_flag, status, lim);
      for (int t = pair; t < items && ok; t += npairs) {
        const WorkItem wi = work_item(t, p, m_tiles, n_tiles, m256);
        if (wi.nh == 0) continue;
        if (tl > 0 && !mbar_wait_cluster(acc_empty, (tl - 1) & 1, abort_flag, status, lim)) break;
        ++tl;
        tc_fence_after();
        const bool two = wi.nh == 2;
        for (int i = 0; i < k_iters; ++i, ++it) {
          const uint32_t s = static_cast<uint32_t>(it) % STAGES, u = static_cast<uint32_t>(it) / STAGES;
          if (!mbar_wait_cluster(&full[s], u & 1, abort_flag, status, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = a_desc0 + s * kAStage16, bd = b_desc0 + s * kBTile16;
          if (i > 0 && i < num_k) {  // a full stage after the first: four K steps per half
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) tc_mma_bf16_ss_pair(tmem, ad + 2 * kk, bd + kBStep * kk, idesc, 1u);
            if (two) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                tc_mma_bf16_ss_pair(tmem + BN, ad + kATile16 + 2 * kk, bd + kBStep * kk, idesc, 1u);
            }
          } else {  // the tile's first stage (accumulators start over) or the rank step
            const int nsteps = i < num_k ? BK / 16 : r_steps;
            for (int h = 0; h < wi.nh; ++h)
              for (int kk = 0; kk < nsteps; ++kk)
                tc_mma_bf16_ss_pair(tmem + static_cast<uint32_t>(h * BN), ad + h * kATile16 + 2 * kk,
                                    bd + kBStep * kk, idesc, (i > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit_pair(&empty[s], 0x3);
        }
        if (ok) tc_commit_pair(acc_full, 0x3);
      }
      // Every MMA (which also reads the odd CTA's shared memory) must be
      // complete before the pair's tensor memory and shared memory go.
      tc_commit_pair(drain, 0x1);
      mbar_wait_teardown(drain, 0, status);
    }
  } else if (warp < kFirstDecodeWarp) {
    // Epilogue warps 2..5 own TMEM lane quadrants (warp % 4).
    const int q = warp & 3;
    const uint32_t acc_empty0 = map_to_cta(acc_empty, 0);
    int tl = 0;
    for (int t = pair; t < items; t += npairs) {
      const WorkItem wi = work_item(t, p, m_tiles, n_tiles, m256);
      if (wi.nh == 0) continue;
      // The tile's whole main loop passes meanwhile; warp 5 shares the MMA
      // warp's scheduler, so the waiting lane sleeps between tries.
      const bool ok = warp_wait(acc_full, tl & 1, abort_flag, status, lim, true, true);
      ++tl;
      if (!ok) break;
      tc_fence_after();
      const int col0 = wi.nb * BN;
      for (int h = 0; h < wi.nh; ++h) {
        const int row = (wi.mh0 + h) * 2 * BM + static_cast<int>(rank) * BM + q * 32 + lane;
        const uint32_t acc = tmem + static_cast<uint32_t>(h * BN) + (static_cast<uint32_t>(q * 32) << 16);
        // Two chunks of 32 columns in flight: the next chunk's load overlaps
        // this chunk's conversion and stores.
        uint32_t va[32], vb[32];
        tmem_ld_32x32b_x32(acc, va);
#pragma unroll
        for (int c = 0; c < BN / 32; c += 2) {
          tmem_wait_ld_regs(va);
          tmem_ld_32x32b_x32(acc + (c + 1) * 32, vb);
          if (p.wide_store)
            store_row32_bf16_wide(va, p.D, row, col0 + c * 32, M, N);
          else
            store_row32_bf16(va, p.D, row, col0 + c * 32, M, N, p.accumulate);
          tmem_wait_ld_regs(vb);
          if (c + 2 < BN / 32) tmem_ld_32x32b_x32(acc + (c + 2) * 32, va);
          if (p.wide_store)
            store_row32_bf16_wide(vb, p.D, row, col0 + (c + 1) * 32, M, N);
          else
            store_row32_bf16(vb, p.D, row, col0 + (c + 1) * 32, M, N, p.accumulate);
        }
      }
      // Hand the accumulators back to the even CTA's MMA thread.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0);
    }
  } else if (warp != kCodeWarp) {
    // Weight decoders.  Group g takes the pipeline steps it with
    // it % kDecodeGroups == g; thread `tid` writes one 128-byte row of the
    // stage's B tile from its block's codes and scale in the code ring.  No
    // decoder thread loads from global memory, so its release-arrives never
    // wait on loads in flight.
    const int dw = decoder_index(warp);
    if (dw >= 0) {  // (warp 13 idles)
      const int grp = dw >> 2;
      const int tid = ((dw & 3) << 5) | lane;
      const uint32_t row_off = kBwd ? static_cast<uint32_t>((tid >> 6) * 8192 + (tid & 63) * 128)
                                    : static_cast<uint32_t>(tid * 128);
      const uint32_t sw = static_cast<uint32_t>(tid & 7);
      // this thread's codes (32 bytes) and scale in a code slot
      const uint32_t code_off = kBwd ? static_cast<uint32_t>((tid >> 6) * 2048 + (tid & 63) * 32)
                                     : static_cast<uint32_t>(tid * 32);
      const uint32_t scale_row = kBwd ? static_cast<uint32_t>(kCodeBytes + (tid & 63) * 16)
                                      : static_cast<uint32_t>(kCodeBytes + tid * 16);
      float L[16];
  #pragma unroll
      for (int j = 0; j < 16; ++j) L[j] = codebook_level(p.codebook, j);
      const int64_t kblocks = p.Kw / kBlock;
      const uint32_t decoded0 = map_to_cta(&full[0], 0);
      const uint32_t sB0 = smem_u32(sB), sC0 = smem_u32(sC);
      int it = 0;
      bool ok = true;
      for (int t = pair; t < items && ok; t += npairs) {
        const WorkItem wi = work_item(t, p, m_tiles, n_tiles, m256);
        if (wi.nh == 0) continue;
        const int64_t nh0 = static_cast<int64_t>(wi.nb) * BN + static_cast<int64_t>(rank) * BNH;
        const int64_t base = kBwd ? nh0 / kBlock : nh0;
        for (int i = 0; i < k_iters; ++i, ++it) {
          if (it % kDecodeGroups != grp) continue;
          const int c = it % kCodeStages, cu = it / kCodeStages;
          const int s = it % STAGES, u = it / STAGES;
          if (i < num_k) {
            // this thread's block: valid row and column, else a zero row
            bool valid;
            uint32_t kq;  // the block's column within its 4-block scale box
            if constexpr (!kBwd) {
              valid = base + tid < p.Nw;
              kq = static_cast<uint32_t>(i & 3);
            } else {
              const int64_t kb = base + (tid >> 6);
              valid = static_cast<int64_t>(i) * BK + (tid & 63) < p.Nw && kb < kblocks;
              kq = static_cast<uint32_t>(kb & 3);
            }
            if (!warp_wait(&cfull[c], cu & 1, abort_flag, status, lim, false)) {
              ok = false;
              break;
            }
            const uint32_t slot = sC0 + static_cast<uint32_t>(c * CODE_SLOT);
            uint32_t w[8];
            ld_shared_v4(slot + code_off, w[0], w[1], w[2], w[3]);
            ld_shared_v4(slot + code_off + 16, w[4], w[5], w[6], w[7]);
            const float a = ld_shared_f32(slot + scale_row + 4 * kq);
            if (it >= STAGES && !warp_wait(&empty[s], (u - 1) & 1, abort_flag, status, lim, false)) {
              ok = false;
              break;
            }
            const uint32_t row = sB0 + static_cast<uint32_t>(s * B_TILE) + row_off;
            if (valid) {
              decode_block_to_smem(row, sw, w, a, L);
            } else {
  #pragma unroll
              for (int j = 0; j < 8; ++j) st_shared_v4(row + (static_cast<uint32_t>(j) << 4), 0u, 0u, 0u, 0u);
            }
            // One proxy fence orders this thread's code-slot reads before the
            // slot's next TMA refill and its tile writes before the MMA's reads.
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive_remote(decoded0 + 8u * static_cast<uint32_t>(s));
              mbar_arrive(&cempty[c]);
            }
          } else {
            // The rank step: its operands come by TMA.  Every stage still gets
            // this warp's arrivals, so the barriers' phases follow the slots' uses.
            if (!warp_wait(&cfull[c], cu & 1, abort_flag, status, lim, false) ||
                (it >= STAGES && !warp_wait(&empty[s], (u - 1) & 1, abort_flag, status, lim, false))) {
              ok = false;
              break;
            }
            if (lane == 0) {
              mbar_arrive_remote(decoded0 + 8u * static_cast<uint32_t>(s));
              mbar_arrive(&cempty[c]);
            }
          }
        }
      }
    }
  } else {
    // Code ring producer (lane 0): per pipeline step, this CTA's packed codes
    // and decoded block scales by TMA into slot it % kCodeStages, as soon as
    // the decode group that read the slot's previous contents released it.
    if (lane == 0) {
      tma_prefetch_desc(&tmP);
      tma_prefetch_desc(&tmS);
      int it = 0;
      bool ok = true;
      for (int t = pair; t < items && ok; t += npairs) {
        const WorkItem wi = work_item(t, p, m_tiles, n_tiles, m256);
        if (wi.nh == 0) continue;
        const int n_half = wi.nb * BN + static_cast<int>(rank) * BNH;  // forward: first weight row; backward: first column
        for (int i = 0; i < k_iters; ++i, ++it) {
          const int c = it % kCodeStages, cu = it / kCodeStages;
          // (this warp shares the MMA warp's scheduler: it sleeps between tries)
          if (it >= kCodeStages && !mbar_wait_suspend(&cempty[c], (cu - 1) & 1, false, abort_flag, status, lim)) {
            ok = false;
            break;
          }
          uint8_t* slot = sC + c * CODE_SLOT;
          if (i >= num_k) {
            mbar_arrive(&cfull[c]);  // the rank step carries no codes
          } else if constexpr (!kBwd) {
            mbar_arrive_expect_tx(&cfull[c], kCodeBytes + BNH * 16);
            tma_load_2d<1>(slot, &tmP, &cfull[c], i * 32, n_half, status);                          // [128 rows][32 B]
            tma_load_2d<4>(slot + kCodeBytes, &tmS, &cfull[c], i & ~3, n_half, status);             // [128 rows][4 scales]
          } else {
            const int n0 = i * BK, kb0 = n_half / kBlock;
            mbar_arrive_expect_tx(&cfull[c], kCodeBytes + BK * 16);
            tma_load_2d<1>(slot, &tmP, &cfull[c], n_half / 2, n0, status);                          // [64 rows][32 B]
            tma_load_2d<1>(slot + 2048, &tmP, &cfull[c], n_half / 2 + 32, n0, status);              // the next block
            tma_load_2d<4>(slot + kCodeBytes, &tmS, &cfull[c], kb0 & ~3, n0, status);               // [64 rows][4 scales]
          }
        }
      }
      // Teardown: every copy into the code ring has landed.
      for (int i = (it > kCodeStages ? it - kCodeStages : 0); i < it; ++i)
        mbar_wait_teardown(&cfull[i % kCodeStages], (i / kCodeStages) & 1, status);
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

template <bool kBwd>
int query_nf4_clusters() {
  if (cudaFuncSetAttribute(gemm_nf4_kernel<kBwd>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
      cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_nf4_kernel<kBwd>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  return n;
}

// Pair clusters of the decoding kernel that fit at once on the current device
// (0: it cannot run there); sets the kernel's shared-memory limit on the
// device as it first asks.
template <bool kBwd>
int nf4_pair_clusters(int dev) {
  static DeviceValue cached;
  return cached.get(dev, [] { return query_nf4_clusters<kBwd>(); });
}

}  // namespace

cudaError_t launch_gemm_nf4(const Nf4GemmArgs& a, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool bwd = a.backward != 0;
  const int clusters = bwd ? nf4_pair_clusters<true>(dev) : nf4_pair_clusters<false>(dev);
  if (clusters <= 0) return cudaErrorNotSupported;
  const WeightView& w = a.w;
  // GEMM view: D [M][N] = A [M][K] op(W_hat) + A2 B2
  const int64_t N = bwd ? w.cols : w.rows;
  const int64_t K = bwd ? w.rows : w.cols;
  CUtensorMap tA, tA2, tB2, tP, tS;
  if (!encode_tensor_map_2d(&tA, a.A, a.M, K, BM, BK)) return cudaErrorInvalidValue;
  // Code ring sources: the packed codes [N_w][K_w / 2] bytes and the decoded
  // block scales [N_w][ld] fp32 (a.scales, written by launch_block_scales).
  const uint32_t code_rows = bwd ? BK : BNH;
  const int64_t sld = block_scales_ld(w.cols);
  if (a.scales == nullptr) return cudaErrorInvalidValue;
  if (!encode_tensor_map_2d_plain(&tP, w.packed, 1, w.rows, w.cols / 2, w.cols / 2, code_rows, 32))
    return cudaErrorInvalidValue;
  if (!encode_tensor_map_2d_plain(&tS, a.scales, 4, w.rows, sld, sld, code_rows, 4)) return cudaErrorInvalidValue;
  int r_steps = 0;
  if (a.A2 != nullptr && a.r > 0) {
    r_steps = (a.r + 15) / 16;
    if (!encode_tensor_map_2d(&tA2, a.A2, a.M, kRankPad, BM, BK)) return cudaErrorInvalidValue;
    if (bwd) {
      // LoRA A [r][K_w]: boxes of 16 * r_steps rows x 64 columns (MN-major B2)
      if (!encode_tensor_map_2d(&tB2, a.B2, a.r, N, static_cast<uint32_t>(16 * r_steps), 64))
        return cudaErrorInvalidValue;
    } else {
      // LoRA B [N_w][ldb2] with r valid columns, zero filled to 64
      if (!encode_tensor_map_2d(&tB2, a.B2, N, a.r, BNH, BK, true, a.ldb2)) return cudaErrorInvalidValue;
    }
  } else {
    tA2 = tA;
    tB2 = tA;
  }
  Nf4GemmParams p{};
  p.packed = w.packed;
  p.qscale = w.qscale;
  p.c2 = w.c2;
  p.mu = w.mu;
  p.absmax = w.absmax;
  p.codebook = w.codebook;
  p.scale_format = w.scale_format;
  p.Nw = w.rows;
  p.Kw = w.cols;
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(N);
  p.num_k = static_cast<int>((K + BK - 1) / BK);
  p.r_steps = r_steps;
  p.D = a.D;
  p.accumulate = a.accumulate;
  p.status = a.status;
  p.wait_limit_ns = a.wait_limit_ns ? a.wait_limit_ns : kWaitLimitNs;
  p.debug_stall = a.debug_stall;
  p.wide_store = !a.accumulate && N % 16 == 0 && (reinterpret_cast<uintptr_t>(a.D) & 31) == 0;
  const int64_t m256 = (a.M + 2 * BM - 1) / (2 * BM);
  const int64_t m_tiles = (m256 + kHalves - 1) / kHalves, n_tiles = (N + BN - 1) / BN;
  const int64_t tiles = m_tiles * n_tiles;
  // Whole tiles fill complete waves of the pairs; a last partial wave that
  // would occupy at most half of them is split into half tiles, so it takes
  // half a wave's time.
  const int64_t rem = tiles % clusters;
  const int64_t split = (rem > 0 && 2 * rem <= clusters) ? rem : 0;
  const int64_t items = tiles + split;
  if (items > 0x7FFFFFFF) return cudaErrorInvalidValue;
  p.full_tiles = static_cast<int>(tiles - split);
  p.items = static_cast<int>(items);
  const int pairs = static_cast<int>(items < clusters ? items : clusters);
  // HBM bytes of one tile-wide panel: A (bf16 activations) 2 B per value;
  // the weight 0.5 B of codes + 1/64 B of scale codes per value.
  const double a_panel = static_cast<double>(kHalves * 2 * BM) * static_cast<double>(K) * 2.0;
  const double b_panel = 256.0 * static_cast<double>(K) * (0.5 + 1.0 / 64.0);
  const RasterChoice rc = choose_raster(m_tiles, n_tiles, a_panel, b_panel, static_cast<double>(kL2PanelBudget));
  p.group = rc.group;
  p.along_n = rc.along_n;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (bwd) return cudaLaunchKernelEx(&cfg, gemm_nf4_kernel<true>, tA, tA2, tB2, tP, tS, p);
  return cudaLaunchKernelEx(&cfg, gemm_nf4_kernel<false>, tA, tA2, tB2, tP, tS, p);
}

}  // namespace qnf4
