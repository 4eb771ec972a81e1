// Decode-shaped LoRA linear forward, M <= 16 tokens (sm_100a).
//
//   Y = X W_hat^T + s (X A^T) B^T       ("QLoRA: NF4 storage, gradients and
//   local integration", FrozenNF4LoRA.forward; "FT-02: QLoRA -- Fine-Tuning
//   with Quantization", section "4. The LoRA mechanics the API wraps")
//
// The packed weight (0.5 B per weight) is the only large operand, so the path
// is HBM-bound: it streams the codes once and never writes a dequantized
// copy.  Up to three kernels:
//
//   xa_part_kernel   only when K > 4096: U partials, each CTA reduces
//                    X A^T over 1024 of K with warp MMAs ([P][16][64] fp32);
//                    it releases the GEMV at once (programmatic dependent
//                    launch).  For K <= 4096 the GEMV computes U itself from
//                    the X fragments it holds (one launch per call).
//   gemv_kernel      persistent, one CTA per SM, which owns a contiguous
//                    range of 16-row tiles.  Each of its 16 warps owns one
//                    quarter-kilo slice of K (4 blocks of 64; X held in
//                    registers as MMA fragments) and walks every tile of the
//                    CTA: a private ring of 16-byte cp.async copies keeps its
//                    next 2 tile slices in flight (rows padded in shared
//                    memory so the fragment loads never conflict), nibble
//                    pairs are decoded through a byte -> bf16x2 table,
//                    m16n8k16 MMAs accumulate each block and the decoded
//                    block scale is applied to the block's fp32 partial.
//                    Each tile's partial goes to the reduction buffer; after
//                    2 (M > 8) or 4 tiles one cross-warp reduction (two CTA
//                    barriers) sums the 16 slices, adds the rank-r term
//                    s U B^T (the CTA's B rows copied once) and stores Y as
//                    bf16.  No barrier sits inside a tile, so each warp
//                    overlaps the latency of one tile's loads, lookups and
//                    MMAs with the next.
//   gemv_finalize    only when K > 4096: sums the per-chunk fp32 partials and
//                    adds the rank-r term.
//
// The dequantized weight used is bf16(L[code]) * a, with the decoded block
// scale a applied in fp32 to the block's partial sum (the dequantizer and the
// training path round fp32(L[code] * a) to bf16 instead; the difference is one
// bf16 rounding of the weight).
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kGvWarps = 16;
constexpr int kGvThreads = kGvWarps * 32;
constexpr int kGvRows = 16;                  // weight rows per tile (MMA m = 16)
constexpr int kGvWarpBlocks = 4;             // 64-blocks of K per warp and chunk
constexpr int kGvUnitBlocks = kGvWarps * kGvWarpBlocks;  // 64 blocks = 4096 of K per chunk
constexpr int kGvDepth = 2;                  // tile slices in flight per warp
constexpr int kGvSlicePitch = kGvWarpBlocks * kBlock / 2 + 32;  // 160 B per row of a slice
constexpr int kGvSliceBytes = kGvRows * kGvSlicePitch;          // 2560 B
constexpr int kGvPartFloats = 512;           // partials per warp and pass: tiles x token tiles x 32 lanes x 4
constexpr int kGvRedWarpBytes = kGvPartFloats * 4 + 16;         // one warp's partials, padded
constexpr int kGvBBytes = 16384;             // B rows of the CTA, when they fit

// Shared memory.  The byte -> bf16x2 table sits at shared-window address
// 0x10000 (64 KB): entry (byte, lane) is at 0x10000 | byte << 8 | lane << 2,
// formed from the packed word by one permute, so a lookup is two
// instructions and every lane reads its own bank.  Region A (below the table,
// after the dynamic base) holds the reduction buffer, U, small tables and the
// B rows; region C (above the table) the warps' copy rings.
constexpr uint32_t kLutWindow = 0x10000;
constexpr int kRedOff = 0;                                        // [16 warps][kGvRedWarpBytes]
constexpr int kUOff = kRedOff + kGvWarps * kGvRedWarpBytes;      // [16][64] fp32
constexpr int kQdivOff = kUOff + kGemvMaxM * kRankPad * 4;        // [256] fp32
constexpr int kLevOff = kQdivOff + 256 * 4;                       // [16] fp32 levels
constexpr int kBOff = kLevOff + 16 * 4;                           // [rows][ldb] bf16
constexpr int kRegionA = kBOff + kGvBBytes;
constexpr uint32_t kRingWindow = 2 * kLutWindow;                  // [16 warps][depth][slice]
constexpr int kGvSmemBytes = static_cast<int>(kRingWindow) + kGvWarps * kGvDepth * kGvSliceBytes;

static_assert(kBOff % 16 == 0 && kGvSliceBytes % 16 == 0 && kGvRedWarpBytes % 16 == 0, "copy alignment");
static_assert(kRegionA + 4096 <= static_cast<int>(kLutWindow), "region A must leave room for the dynamic base");
static_assert(kGvSmemBytes <= 227 * 1024, "shared memory budget");

constexpr int kXaWarps = 16;  // U partial kernel: one 64-wide K block per warp


// Table entry for byte J of `word`: `lane_base` = 0x10000 | 4 * lane; the
// permute keeps its bytes 0, 2, 3 and puts byte J of `word` in byte 1.  The
// load is left non-volatile so it schedules freely; its address depends on
// `word`, which is read after the stage's barrier completes.
template <int J>
__device__ __forceinline__ uint32_t lut_pair(uint32_t word, uint32_t lane_base) {
  uint32_t addr, v;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(addr) : "r"(lane_base), "r"(word), "n"(0x3240 + 0x10 * J));
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// 16-byte copy global -> shared (32-bit shared address), no predicate.
__device__ __forceinline__ void cp_async_16_full(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ uint2 ld_shared_v2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// 16 consecutive bf16 of row `row` starting at element k (zeros if !valid).
__device__ __forceinline__ void load16(const uint16_t* base, int64_t ld, int row, int64_t k, bool valid,
                                       uint32_t (&w)[8]) {
  uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
  if (valid) {
    const uint4* p = reinterpret_cast<const uint4*>(base + static_cast<int64_t>(row) * ld + k);
    a = __ldg(p);
    b = __ldg(p + 1);
  }
  w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
  w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
}

}  // namespace

// Fragment k-map shared by both kernels.  In a 64-wide block, lane
// (g = lane/4, t = lane%4) holds k = 16t .. 16t+15 of its row; k16 step s
// takes k = 16t + 4s + {0,1} into fragment slots {2t, 2t+1} and
// 16t + 4s + {2,3} into slots {2t+8, 2t+9}.  Both operands of every MMA use
// the same map, so each block's 64 products are each taken exactly once.

// U partials: Upart[p][m][j] = sum over k in [1024p, 1024p + 1024) of
// X[m][k] A[j][k] (m < 16, j < 64; zeros beyond M and r).
__global__ void __launch_bounds__(kXaWarps * 32) xa_part_kernel(const uint16_t* __restrict__ X,
                                                                const uint16_t* __restrict__ A, int M, int64_t K,
                                                                int r, float* __restrict__ Upart) {
  pdl_launch_dependents();
  extern __shared__ float s_xa[];  // [16 warps][16][64]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int64_t kb = static_cast<int64_t>(blockIdx.x) * kXaWarps + warp;
  float acc[8][4];
#pragma unroll
  for (int jt = 0; jt < 8; ++jt)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[jt][c] = 0.0f;
  if (kb * kBlock < K) {
    const int64_t k0 = kb * kBlock + 16 * t;
    uint32_t xa[8], xb[8];
    load16(X, K, g, k0, g < M, xa);
    load16(X, K, g + 8, k0, g + 8 < M, xb);
#pragma unroll
    for (int jt = 0; jt < 8; ++jt) {
      if (8 * jt < r) {
        uint32_t aw[8];
        load16(A, K, 8 * jt + g, k0, 8 * jt + g < r, aw);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint32_t af[4] = {xa[2 * s], xb[2 * s], xa[2 * s + 1], xb[2 * s + 1]};
          const uint32_t bf[2] = {aw[2 * s], aw[2 * s + 1]};
          mma_bf16_16816(acc[jt], af, bf);
        }
      }
    }
  }
  float* mine = s_xa + warp * (kGemvMaxM * kRankPad);
#pragma unroll
  for (int jt = 0; jt < 8; ++jt) {
    *reinterpret_cast<float2*>(&mine[g * kRankPad + 8 * jt + 2 * t]) = make_float2(acc[jt][0], acc[jt][1]);
    *reinterpret_cast<float2*>(&mine[(g + 8) * kRankPad + 8 * jt + 2 * t]) = make_float2(acc[jt][2], acc[jt][3]);
  }
  __syncthreads();
  for (int e = tid; e < kGemvMaxM * kRankPad; e += kXaWarps * 32) {
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < kXaWarps; ++w) v += s_xa[w * (kGemvMaxM * kRankPad) + e];
    Upart[static_cast<int64_t>(blockIdx.x) * (kGemvMaxM * kRankPad) + e] = v;
  }
}

// Sum of the U partials into shared memory U_s[16][64]; the first CTA also
// writes the caller's fp32 copy U_out [M][r].
__device__ __forceinline__ void gather_u(const GemvParams& p, float* U_s, int tid, int nthreads) {
  for (int e = tid; e < kGemvMaxM * kRankPad; e += nthreads) {
    float v = 0.0f;
    for (int q = 0; q < p.n_upart; ++q) v += p.upart[static_cast<int64_t>(q) * (kGemvMaxM * kRankPad) + e];
    U_s[e] = v;
    const int m = e / kRankPad, j = e % kRankPad;
    if (blockIdx.x == 0 && p.U_out != nullptr && m < p.M && j < p.r) p.U_out[m * p.r + j] = v;
  }
}

// Position of one work item of a CTA: chunk c of K, tile `tile` of rows.
struct GvCursor {
  int c, tile;
  __device__ __forceinline__ void next(int t0, int t1) {
    if (++tile == t1) {
      tile = t0;
      ++c;
    }
  }
};

// Decode-shaped forward.  The weight tile is the MMA's A operand (16 rows x
// 16 k), X the B operand (8 tokens; two token tiles for 9..16 tokens).  Lane
// (g, t) reads 8 bytes of rows g and g+8 per block and decodes four nibble
// pairs per k16 step; every tile runs the same straight-line code (no branch
// inside a tile: pieces past the end are zero-filled copies, blocks past the
// end of K meet zero X fragments).
template <bool kM16, bool kScales32>
__global__ void __launch_bounds__(kGvThreads, 1) gemv_kernel(const __grid_constant__ GemvParams p) {
  constexpr int NT = kM16 ? 2 : 1;  // token tiles of 8
  constexpr int P = kM16 ? 2 : 4;   // tiles per reduction pass
  static_assert(P * NT * 32 * 4 == kGvPartFloats, "partials layout");
  extern __shared__ __align__(16) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  if (base + kRegionA > kLutWindow) {  // the layout needs the dynamic base below 0x10000 - kRegionA
    if (threadIdx.x == 0) raise_status(p.status, QLORA_ERR_UNSUPPORTED);
    return;
  }
  float* const s_u = reinterpret_cast<float*>(smem + kUOff);
  float* const s_qdiv = reinterpret_cast<float*>(smem + kQdivOff);
  float* const s_lev = reinterpret_cast<float*>(smem + kLevOff);
  uint16_t* const s_b = reinterpret_cast<uint16_t*>(smem + kBOff);
  uint32_t* const lut = reinterpret_cast<uint32_t*>(smem + (kLutWindow - base));
  float* const red = reinterpret_cast<float*>(smem + kRedOff);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int64_t N = p.N, K = p.K;
  const int64_t nbk = K / kBlock;
  const int nchunk = static_cast<int>((nbk + kGvUnitBlocks - 1) / kGvUnitBlocks);
  const int tiles = static_cast<int>((N + kGvRows - 1) / kGvRows);
  const int t0 = static_cast<int>(static_cast<int64_t>(tiles) * blockIdx.x / gridDim.x);
  const int t1 = static_cast<int>(static_cast<int64_t>(tiles) * (blockIdx.x + 1) / gridDim.x);
  const int items = (t1 - t0) * nchunk;  // chunk-major: all tiles of chunk 0, then chunk 1, ...
  const bool single = nchunk == 1;
  const int64_t row_lo = static_cast<int64_t>(t0) * kGvRows;
  const int64_t row_hi = static_cast<int64_t>(t1) * kGvRows < N ? static_cast<int64_t>(t1) * kGvRows : N;
  const bool b_smem = single && (row_hi - row_lo) * p.ldb * 2 <= kGvBBytes;
  uint8_t* const ring = smem + (kRingWindow - base) + warp * (kGvDepth * kGvSliceBytes);

  // The CTA's B rows (one commit group, the first of every thread).
  if (b_smem) {
    const int pieces = static_cast<int>((row_hi - row_lo) * p.ldb / 8);  // 16-byte pieces
    const uint8_t* src = reinterpret_cast<const uint8_t*>(p.B + row_lo * p.ldb);
    for (int i = tid; i < pieces; i += kGvThreads) cp_async_16(smem + kBOff + i * 16, src + i * 16, true);
  }
  cp_async_commit();

  // This warp's slice of item i: rows tile*16 .. +16, blocks c*64 + 4*warp
  // .. +4, eight 16-byte pieces per row (zero-filled past N, past K or past
  // the last item); one commit group per item and thread.  Lane piece h is
  // row (lane >> 3) + 4h, 16-byte column lane & 7 of the slice, so the
  // source is one running pointer plus fixed strides: it advances by one
  // tile per item and, after the CTA's last tile, to the next 4096-wide chunk
  // of K.
  const int ntile = t1 - t0;
  const int64_t tile_bytes = static_cast<int64_t>(kGvRows) * (K / 2);
  const int64_t rows4_bytes = 4 * (K / 2);
  const int prow = lane >> 3, pcol = lane & 7;
  const uint8_t* isrc = p.packed + static_cast<int64_t>(t0) * tile_bytes + warp * (kGvWarpBlocks * kBlock / 2) +
                        prow * (K / 2) + pcol * 16;
  const uint32_t slot_lane = static_cast<uint32_t>(prow * kGvSlicePitch + pcol * 16);
  const uint32_t ring_lane = smem_u32(ring) + slot_lane;
  // An item is full (every piece of the slice valid) unless it is the ragged
  // last tile of the weight or a chunk where this warp's 4 blocks run past K.
  const int ragged_tile = N % kGvRows != 0 ? tiles - 1 : -1;
  const int full_chunks = nbk >= kGvWarpBlocks * (warp + 1)
                              ? static_cast<int>((nbk - kGvWarpBlocks * (warp + 1)) / kGvUnitBlocks) + 1
                              : 0;
  int i_tile = 0, i_chunk = 0, issued = 0;
  auto issue_next = [&]() {
    const bool live = issued < items;
    const uint32_t dst = ring_lane + (issued & (kGvDepth - 1)) * kGvSliceBytes;
    // A checks build also tests that the four unpredicated copies stay inside
    // the packed weight (else it takes the predicated path).
    if (live && t0 + i_tile != ragged_tile && i_chunk < full_chunks &&
        qlora_checked(p.status, isrc >= p.packed && isrc + 3 * rows4_bytes + 16 <= p.packed + N * (K / 2))) {
#pragma unroll
      for (int h = 0; h < 4; ++h) cp_async_16_full(dst + h * 4 * kGvSlicePitch, isrc + h * rows4_bytes);
    } else {
      const int rows_left = static_cast<int>(N - static_cast<int64_t>(t0 + i_tile) * kGvRows);
      const int rem = static_cast<int>(nbk - i_chunk * kGvUnitBlocks) - kGvWarpBlocks * warp;
      const bool col_ok = live && pcol < 2 * rem;
      uint8_t* slot = ring + (issued & (kGvDepth - 1)) * kGvSliceBytes + slot_lane;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const bool v = col_ok && prow + 4 * h < rows_left;
        cp_async_16(slot + h * 4 * kGvSlicePitch, v ? isrc + h * rows4_bytes : p.packed, v);
      }
    }
    if (live) {
      if (++i_tile == ntile) {
        i_tile = 0;
        ++i_chunk;
        isrc += kGvUnitBlocks * kBlock / 2 - static_cast<int64_t>(ntile - 1) * tile_bytes;
      } else {
        isrc += tile_bytes;
      }
    }
    ++issued;
    cp_async_commit();
  };
#pragma unroll 1
  for (int i = 0; i < kGvDepth; ++i) issue_next();

  if (tid < 16) s_lev[tid] = codebook_level(p.codebook, tid);
  if (tid < 256) s_qdiv[tid] = scale_table_entry(p.scale_format, tid);
  __syncthreads();
  // lut[byte][64 words]: word `lane` = (L[byte & 15], L[byte >> 4]) as bf16.
  for (int i = tid; i < 256 * 32; i += kGvThreads) {
    const int byte = i >> 5, l = i & 31;
    lut[byte * 64 + l] = pack_bf16x2(s_lev[byte & 15], s_lev[byte >> 4]);
  }

  const float mu = kScales32 ? 0.0f : *p.mu;
  const uint32_t lane_base = kLutWindow | (static_cast<uint32_t>(lane) * 4);
  const uint32_t ring_frag = smem_u32(ring) + static_cast<uint32_t>(g * kGvSlicePitch + 8 * t);
  // Scales this lane decodes per item: row lane%16 of the tile, blocks
  // 4 warp + lane/16 and 4 warp + lane/16 + 2; the lanes holding rows g and
  // g+8 hand them over by shuffle.  The block index runs like the copy
  // source: + 16 nbk per tile, to the next chunk after the last tile.
  const int frow = lane & 15, fblk = kGvWarpBlocks * warp + (lane >> 4);
  int64_t fgb = (static_cast<int64_t>(t0) * kGvRows + frow) * nbk + fblk;
  int f_tile = 0, f_chunk = 0, fetched = 0;
  int qv[kGvDepth][2];
  float c2v[kGvDepth][2];
  auto fetch = [&](int slot) {
    const bool live = fetched < items;
    // fp32 scales: t(127) = 1, "c2" is the block's absmax and mu = 0, so the
    // decode below returns the absmax itself.
    if (live && t0 + f_tile != ragged_tile && f_chunk < full_chunks) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        qv[slot][e] = kScales32 ? 127 : p.qscale[fgb + 2 * e];
        c2v[slot][e] = __ldg(p.c2 + (kScales32 ? fgb + 2 * e : (fgb + 2 * e) >> 8));
      }
    } else {
      const bool row_ok = live && static_cast<int64_t>(t0 + f_tile) * kGvRows + frow < N;
      const int blk = f_chunk * kGvUnitBlocks + fblk;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool v = row_ok && blk + 2 * e < nbk;
        const int64_t gb = v ? fgb + 2 * e : 0;
        const int q = kScales32 ? 127 : p.qscale[gb];
        const float c2 = __ldg(p.c2 + (kScales32 ? gb : gb >> 8));
        qv[slot][e] = v ? q : 0;
        c2v[slot][e] = v ? c2 : 0.0f;
      }
    }
    if (live) {
      if (++f_tile == ntile) {
        f_tile = 0;
        ++f_chunk;
        fgb += kGvUnitBlocks - static_cast<int64_t>(ntile - 1) * kGvRows * nbk;
      } else {
        fgb += kGvRows * nbk;
      }
    }
    ++fetched;
  };
#pragma unroll
  for (int i = 0; i < kGvDepth; ++i) fetch(i);

  // X fragments of the current chunk (B operand of k16 step s of block b:
  // words 2s, 2s+1 of the lane's 16 k of token g (+8 for the second tile).
  uint32_t xf[NT][kGvWarpBlocks][8];
  int x_chunk = -1;
  __syncthreads();  // table complete

  GvCursor cc{0, t0};
  bool first_reduce = true;
  int item = 0;
  // One pass: np consecutive tiles of chunk cc.c, then one cross-warp
  // reduction.  The tile loop is not unrolled (one tile body of code keeps the
  // instruction cache warm); each tile's fp32 partial goes to its slot of the
  // reduction buffer as soon as the tile is done.
  const uint32_t red_lane = smem_u32(red) + static_cast<uint32_t>(warp * kGvRedWarpBytes + lane * 16);
  auto run_pass = [&](int np) {
    const int c = cc.c, tile0 = cc.tile;
#pragma unroll 1
    for (int j = 0; j < np; ++j) {
      float acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;
      const float a_lo = __fadd_rn(__fmul_rn(s_qdiv[qv[0][0] + 128], c2v[0][0]), mu);
      const float a_hi = __fadd_rn(__fmul_rn(s_qdiv[qv[0][1] + 128], c2v[0][1]), mu);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        qv[0][e] = qv[1][e];
        c2v[0][e] = c2v[1][e];
      }
      fetch(1);
      cp_async_wait<kGvDepth - 1>();  // this item (this lane's pieces)
      __syncwarp();                   // ... and the other lanes' pieces
      const uint32_t sl = ring_frag + (item & (kGvDepth - 1)) * kGvSliceBytes;
#pragma unroll
      for (int b = 0; b < kGvWarpBlocks; ++b) {
        const uint2 wa = ld_shared_v2(sl + b * 32);
        const uint2 wb = ld_shared_v2(sl + 8 * kGvSlicePitch + b * 32);
        float d[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) d[nt][e] = 0.0f;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const uint32_t xa = k4 < 2 ? wa.x : wa.y, xb = k4 < 2 ? wb.x : wb.y;
          uint32_t a[4];
          if (k4 & 1) {
            a[0] = lut_pair<2>(xa, lane_base);
            a[1] = lut_pair<2>(xb, lane_base);
            a[2] = lut_pair<3>(xa, lane_base);
            a[3] = lut_pair<3>(xb, lane_base);
          } else {
            a[0] = lut_pair<0>(xa, lane_base);
            a[1] = lut_pair<0>(xb, lane_base);
            a[2] = lut_pair<1>(xa, lane_base);
            a[3] = lut_pair<1>(xb, lane_base);
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const uint32_t bx[2] = {xf[nt][b][2 * k4], xf[nt][b][2 * k4 + 1]};
            mma_16816(d[nt], a, bx);
          }
        }
        // D rows g and g+8 are weight rows g and g+8 of the tile.
        const float sv = b < 2 ? a_lo : a_hi;
        const float s_g = __shfl_sync(0xffffffffu, sv, g + 16 * (b & 1));
        const float s_g8 = __shfl_sync(0xffffffffu, sv, g + 8 + 16 * (b & 1));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          acc[nt][0] = fmaf(s_g, d[nt][0], acc[nt][0]);
          acc[nt][1] = fmaf(s_g, d[nt][1], acc[nt][1]);
          acc[nt][2] = fmaf(s_g8, d[nt][2], acc[nt][2]);
          acc[nt][3] = fmaf(s_g8, d[nt][3], acc[nt][3]);
        }
      }
      // This tile's partial: slot [tile j][token tile][lane][4] of the warp's buffer.
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(red_lane + (j * NT + nt) * 512),
                     "f"(acc[nt][0]), "f"(acc[nt][1]), "f"(acc[nt][2]), "f"(acc[nt][3])
                     : "memory");
      __syncwarp();  // the slot is read; refill it
      issue_next();
      ++item;
    }

    // Cross-warp reduction: thread tau sums float tau of the 16 warps'
    // partials ([tile][token tile][lane][4]).
    __syncthreads();
    if (first_reduce) {
      // K > 4096: the U partials of the preceding kernel (programmatic
      // launch) must be complete before this grid ends (the finalize kernel
      // reads them).  For K <= 4096 this kernel computed U itself, no kernel
      // precedes by programmatic launch and the wait returns at once.
      pdl_wait_prior();
      first_reduce = false;
    }
    if (tid < np * NT * 128) {
      float y = 0.0f;
#pragma unroll
      for (int w = 0; w < kGvWarps; ++w) y += red[w * (kGvRedWarpBytes / 4) + tid];
      const int comp = tid & 3, ls = (tid >> 2) & 31, rest = tid >> 7;
      const int nt = rest % NT, j = rest / NT;
      const int row = (ls >> 2) + 8 * (comp >> 1);
      const int tok = 2 * (ls & 3) + (comp & 1) + 8 * nt;
      const int64_t n = static_cast<int64_t>(tile0 + j) * kGvRows + row;
      if (tok < p.M && n < N) {
        if (single) {
          float l = 0.0f;
          const uint16_t* brow = b_smem ? s_b + (n - row_lo) * p.ldb : p.B + n * p.ldb;
          for (int jj = 0; jj < p.r; ++jj) l = fmaf(s_u[tok * kRankPad + jj], bf16_bits_to_float(brow[jj]), l);
          y = fmaf(p.scale, l, y);
          p.Y[static_cast<int64_t>(tok) * N + n] = static_cast<uint16_t>(pack_bf16x2(y, 0.0f) & 0xFFFFu);
        } else {
          p.ypart[(static_cast<int64_t>(c) * kGemvMaxM + tok) * N + n] = y;
        }
      }
    }
    __syncthreads();  // the reduction buffer is free again
#pragma unroll 1
    for (int j = 0; j < np; ++j) cc.next(t0, t1);
  };

  // U = X A^T when K fits one chunk: warp w multiplies its K slice of X (the
  // fragments in registers, as the MMA's 16-row operand: tokens g, g + 8) by
  // the same slice of A (8 columns of U per MMA); the 16 warps' partials are
  // summed through the reduction buffer, up to four 8-column groups per
  // round, into U in shared memory.  The first CTA also writes U_out.
  auto compute_u = [&]() {
    const int n_jt = (p.r + 7) / 8;
#pragma unroll 1
    for (int jt0 = 0; jt0 < n_jt; jt0 += 4) {
      const int njt = n_jt - jt0 < 4 ? n_jt - jt0 : 4;
#pragma unroll 1
      for (int jj = 0; jj < njt; ++jj) {
        const int j = 8 * (jt0 + jj) + g;
        float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int b = 0; b < kGvWarpBlocks; ++b) {
          const int64_t blk = kGvWarpBlocks * warp + b;
          uint32_t aw[8];
          load16(p.A, K, j, blk * kBlock + 16 * t, blk < nbk && j < p.r, aw);
#pragma unroll
          for (int s4 = 0; s4 < 4; ++s4) {
            const uint32_t af[4] = {xf[0][b][2 * s4], NT > 1 ? xf[NT - 1][b][2 * s4] : 0u, xf[0][b][2 * s4 + 1],
                                    NT > 1 ? xf[NT - 1][b][2 * s4 + 1] : 0u};
            const uint32_t bf[2] = {aw[2 * s4], aw[2 * s4 + 1]};
            mma_16816(d, af, bf);
          }
        }
        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(red_lane + jj * 512), "f"(d[0]), "f"(d[1]),
                     "f"(d[2]), "f"(d[3])
                     : "memory");
      }
      __syncthreads();
      if (tid < njt * 128) {
        float u = 0.0f;
#pragma unroll
        for (int w = 0; w < kGvWarps; ++w) u += red[w * (kGvRedWarpBytes / 4) + tid];
        const int comp = tid & 3, ls = (tid >> 2) & 31, jj = tid >> 7;
        const int tok = (ls >> 2) + 8 * (comp >> 1);
        const int j = 8 * (jt0 + jj) + 2 * (ls & 3) + (comp & 1);
        s_u[tok * kRankPad + j] = u;
        if (blockIdx.x == 0 && p.U_out != nullptr && tok < p.M && j < p.r) p.U_out[tok * p.r + j] = u;
      }
      __syncthreads();
    }
  };

  for (int i0 = 0; i0 < items;) {
    const int np = (t1 - cc.tile) < P ? (t1 - cc.tile) : P;
    if (cc.c != x_chunk) {
      const int64_t blkw = static_cast<int64_t>(cc.c) * kGvUnitBlocks + kGvWarpBlocks * warp;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int b = 0; b < kGvWarpBlocks; ++b) {
          const int tok = g + 8 * nt;
          load16(p.X, K, tok, (blkw + b) * kBlock + 16 * t, blkw + b < nbk && tok < p.M, xf[nt][b]);
        }
      x_chunk = cc.c;
      if (single) compute_u();
    }
    run_pass(np);
    i0 += np;
  }
  cp_async_wait<0>();
}

// K > 4096: Y[m][n] = sum over chunks of the fp32 partials + s (U B^T)[m][n].
__global__ void __launch_bounds__(256) gemv_finalize_kernel(const __grid_constant__ GemvParams p) {
  __shared__ float s_u[kGemvMaxM * kRankPad];
  gather_u(p, s_u, threadIdx.x, 256);
  __syncthreads();
  const int64_t N = p.N;
  const int nchunk = static_cast<int>((p.K / kBlock + kGvUnitBlocks - 1) / kGvUnitBlocks);
  const int64_t pairs = static_cast<int64_t>(p.M) * (N / 2);
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; e < pairs;
       e += static_cast<int64_t>(gridDim.x) * 256) {
    const int m = static_cast<int>(e / (N / 2));
    const int64_t n = (e % (N / 2)) * 2;
    float y0 = 0.0f, y1 = 0.0f;
    for (int cc = 0; cc < nchunk; ++cc) {
      const float2 v = *reinterpret_cast<const float2*>(p.ypart + (static_cast<int64_t>(cc) * kGemvMaxM + m) * N + n);
      y0 += v.x;
      y1 += v.y;
    }
    float l0 = 0.0f, l1 = 0.0f;
    for (int j = 0; j < p.r; ++j) {
      const float uj = s_u[m * kRankPad + j];
      l0 = fmaf(uj, bf16_bits_to_float(p.B[n * p.ldb + j]), l0);
      l1 = fmaf(uj, bf16_bits_to_float(p.B[(n + 1) * p.ldb + j]), l1);
    }
    y0 = fmaf(p.scale, l0, y0);
    y1 = fmaf(p.scale, l1, y1);
    *reinterpret_cast<uint32_t*>(p.Y + static_cast<int64_t>(m) * N + n) = pack_bf16x2(y0, y1);
  }
}

int gemv_upart_count(int64_t K) { return static_cast<int>((K / kBlock + kXaWarps - 1) / kXaWarps); }
int gemv_chunks(int64_t K) { return static_cast<int>((K / kBlock + kGvUnitBlocks - 1) / kGvUnitBlocks); }

int gemv_launches(int64_t K, int /*M*/) { return gemv_chunks(K) > 1 ? 3 : 1; }

cudaError_t launch_gemv(const GemvParams& p, cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static DeviceOnce configured;
  e = configured.run(dev, [] {
    cudaError_t r = cudaSuccess;
    for (auto fn : {gemv_kernel<true, false>, gemv_kernel<false, false>, gemv_kernel<true, true>,
                    gemv_kernel<false, true>})
      if (r == cudaSuccess) r = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kGvSmemBytes);
    if (r == cudaSuccess)
      r = cudaFuncSetAttribute(xa_part_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kXaWarps * kGemvMaxM * kRankPad * 4);
    return r;
  });
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;

  // K <= 4096: the GEMV computes U itself from the X fragments it holds (a
  // separate U kernel before it cost about 4 us per call when calls follow
  // one another); otherwise U partials come from the first kernel, which
  // releases the GEMV at once (programmatic launch) and finishes while the
  // GEMV streams its tiles.
  const bool fused_u = gemv_chunks(p.K) == 1;
  if (!fused_u) {
    xa_part_kernel<<<p.n_upart, kXaWarps * 32, kXaWarps * kGemvMaxM * kRankPad * 4, stream>>>(p.X, p.A, p.M, p.K,
                                                                                            p.r, p.upart);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }

  const int64_t tiles = (p.N + kGvRows - 1) / kGvRows;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles < sms ? tiles : sms));
  cfg.blockDim = dim3(kGvThreads);
  cfg.dynamicSmemBytes = kGvSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = fused_u ? 0 : 1;
  if (p.scale_format == kScalesFp32)
    e = p.M > 8 ? cudaLaunchKernelEx(&cfg, gemv_kernel<true, true>, p)
                : cudaLaunchKernelEx(&cfg, gemv_kernel<false, true>, p);
  else
    e = p.M > 8 ? cudaLaunchKernelEx(&cfg, gemv_kernel<true, false>, p)
                : cudaLaunchKernelEx(&cfg, gemv_kernel<false, false>, p);
  if (e != cudaSuccess || gemv_chunks(p.K) == 1) return e;
  const int64_t pairs = static_cast<int64_t>(p.M) * (p.N / 2);
  const int64_t blocks = (pairs + 255) / 256;
  gemv_finalize_kernel<<<static_cast<unsigned>(blocks < 4 * sms ? blocks : 4 * sms), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace qnf4
