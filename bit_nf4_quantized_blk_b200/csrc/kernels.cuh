// Kernel parameter blocks and host-side launchers shared by the library's
// translation units.
#pragma once

#include "common.cuh"
#include "device_once.h"

namespace qnf4 {

// ---------------------------------------------------------------------------
// Quantize + double quantize (quantize.cu)
// ---------------------------------------------------------------------------

constexpr int kMaxQuantBatch = 128;  // tensors per launch (kernel parameter block)

struct QuantBatchParams {
  int count;
  int64_t total_chunks;
  int64_t chunk_begin[kMaxQuantBatch + 1];  // prefix sums of chunks per tensor
  int64_t n_blocks[kMaxQuantBatch];
  const void* W[kMaxQuantBatch];          // fp32, bf16 or fp16 (in_dtype)
  uint8_t* packed[kMaxQuantBatch];
  int8_t* qscale[kMaxQuantBatch];
  float* c2[kMaxQuantBatch];
  float* mu[kMaxQuantBatch];
  float* absmax_out[kMaxQuantBatch];      // fp32 scales: the tensor's block absmax array
  int in_dtype;                           // QLORA_INPUT_*
  int codebook;                           // QLORA_CODEBOOK_* (one per launch)
  int scale_format;                       // QLORA_SCALES_* (one per launch)
  // workspace
  float* absmax;        // [total_chunks * 256] first-level scales, slot per chunk
  double* chunk_sum;    // [total_chunks]
  int* chunk_exp;       // [2 * total_chunks] min / max exponent field per chunk
  unsigned* counters;   // [count], zero on entry
  int* status;          // device status word, zero on entry
  Nf4DecisionTable table;
};

cudaError_t launch_quantize_batch(const QuantBatchParams& p, cudaStream_t stream);

// ---------------------------------------------------------------------------
// Dequantize (dequant.cu)
// ---------------------------------------------------------------------------

struct WeightView {
  const uint8_t* packed;
  const int8_t* qscale;
  const float* c2;
  const float* mu;
  int64_t rows, cols;
  int codebook;          // QLORA_CODEBOOK_*
  int scale_format;      // QLORA_SCALES_*
  const float* absmax;   // fp32 block scales (QLORA_SCALES_FP32)
};

// Block scale blk of a weight; mu is *w.mu read once by the caller (0 for
// fp32 scales).
__device__ __forceinline__ float weight_block_scale(const WeightView& w, int64_t blk, float mu) {
  if (w.scale_format == kScalesFp32) return w.absmax[blk];
  return decode_scale_value(scale_code_value(w.scale_format, w.qscale[blk]), w.c2[blk / kDqBlock], mu);
}

__device__ __forceinline__ float weight_mu(const WeightView& w) {
  return w.scale_format == kScalesFp32 ? 0.0f : *w.mu;
}

// The 4-bit GEMM's decoded block scales, fp32 [rows][ld] (pad columns 0),
// as a job of `groups` four-block groups that runs on spare threads of
// another small kernel's launch (or alone, launch_block_scales).  out null:
// no job.
struct BlockScalesJob {
  WeightView w;
  float* out;
  int64_t ld, groups;
};

// Group q: blocks 4 (q % (ld / 4)) .. + 3 of row q / (ld / 4), one 16-byte store.
__device__ __forceinline__ void block_scales_group(const BlockScalesJob& j, int64_t q) {
  const int64_t per_row = j.ld / 4;
  const int64_t n = q / per_row, kb0 = (q - n * per_row) * 4;
  const int64_t kblocks = j.w.cols / kBlock;
  const float mu = weight_mu(j.w);
  float v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = kb0 + i < kblocks ? weight_block_scale(j.w, n * kblocks + kb0 + i, mu) : 0.0f;
  *reinterpret_cast<float4*>(j.out + n * j.ld + kb0) = make_float4(v[0], v[1], v[2], v[3]);
}

// Entry i of a 256-entry table of scale-code values t(q), q = i - 128 the
// int8 view of the stored code: fp32(q / 127) for int8 codes, the E4M3 value
// for FP8 codes.  With fp32 scales the table is the int8 one and the kernels
// decode with q = 127 (t = 1 exactly), c2 = the block absmax and mu = 0, so
// that fp32(fp32(t c2) + mu) is the absmax itself.
__device__ __forceinline__ float scale_table_entry(int format, int i) {
  const int q = i - 128;
  return format == kScalesDqFp8 ? e4m3_to_float(static_cast<uint32_t>(q) & 0xFFu)
                                : __fdiv_rn(static_cast<float>(q), 127.0f);
}

constexpr int kMaxDequantBatch = 128;

struct DequantBatchParams {
  int count;
  int64_t total_seg;                        // 2 KB packed segments in the batch
  int64_t begin_seg[kMaxDequantBatch + 1];  // prefix sums of segments per tensor
  int64_t n_units[kMaxDequantBatch];        // 16-byte packed units per tensor
  const uint8_t* packed[kMaxDequantBatch];
  const int8_t* qscale[kMaxDequantBatch];
  const float* c2[kMaxDequantBatch];
  const float* mu[kMaxDequantBatch];
  const float* absmax[kMaxDequantBatch];   // fp32 scales
  int codebook[kMaxDequantBatch];          // QLORA_CODEBOOK_*
  int scale_format[kMaxDequantBatch];      // QLORA_SCALES_*
  void* out[kMaxDequantBatch];
};

cudaError_t launch_dequant_batch(const DequantBatchParams& p, int out_fp32, cudaStream_t stream);
// Decoded fp32 block scales [rows][block_scales_ld(cols)] (16-byte aligned output).
int64_t block_scales_ld(int64_t cols);
BlockScalesJob block_scales_job(const WeightView& w, float* out);
cudaError_t launch_block_scales(const WeightView& w, float* out, cudaStream_t stream);
cudaError_t launch_dequant_transposed(const WeightView& w, uint16_t* out, cudaStream_t stream);

// ---------------------------------------------------------------------------
// Merged weight W + s B A (merge.cu)
// ---------------------------------------------------------------------------

cudaError_t launch_merge(const WeightView& w, const uint16_t* A, const uint16_t* B, int r, float scale, void* out,
                         int out_fp32, cudaStream_t stream);

// ---------------------------------------------------------------------------
// Decode-shaped dequant-GEMV (gemv.cu), M <= 16
// ---------------------------------------------------------------------------

constexpr int kGemvMaxM = 16;

struct GemvParams {
  const uint8_t* packed;
  const int8_t* qscale;
  const float* c2;       // fp32 scales: the block absmax array
  const float* mu;
  int codebook;          // QLORA_CODEBOOK_*
  int scale_format;      // QLORA_SCALES_*
  int64_t N, K;          // weight [N][K]; N % 8 == 0, K % 64 == 0
  const uint16_t* X;     // [M][K] bf16
  int M;                 // 1 .. 16
  const uint16_t* A;     // [r][K] bf16
  const uint16_t* B;     // [N][ldb] bf16, r valid columns; 16-byte aligned
  int ldb, r;
  float scale;
  float* upart;          // [n_upart][16][64] fp32 scratch
  int n_upart;           // gemv_upart_count(K)
  float* U_out;          // [M][r] fp32, may be null
  uint16_t* Y;           // [M][N] bf16
  float* ypart;          // [gemv_chunks(K)][16][N] fp32 scratch (K > 4096 only)
  int* status;
};

int gemv_upart_count(int64_t K);
int gemv_chunks(int64_t K);
int gemv_launches(int64_t K, int M);
// Y[m][n] = sum_k X[m][k] W[n][k] + s * sum_j (X A^T)[m][j] B[n][j].
cudaError_t launch_gemv(const GemvParams& p, cudaStream_t stream);

// ---------------------------------------------------------------------------
// Skinny LoRA side products (lora_side.cu)
// ---------------------------------------------------------------------------

// out[m][j] = sum_c In[m][c] * Wt(j, c) for j < r, with Wt(j, c) = Wr[j][c]
// (row layout [r, C]) or Wc[c][j] (column layout [C][ldw], r valid columns;
// ldw * 2 bytes a multiple of 16).
// `part` is split scratch of skinny_partial_bytes(M, C).  Writes
//   o32   fp32 [M][o32_ld] (j < r)                   (may be null)
//   os    [M][64] bf16 of scale * out, zero padded   (may be null)
//   ohi / olo [M][64] bf16 split of out (hi + lo ~ fp32) (may be null)
struct SkinnyOut {
  float* o32;
  int64_t o32_ld;
  uint16_t* os;
  uint16_t* ohi;
  uint16_t* olo;
  float scale;
  BlockScalesJob bs;  // run on further threads of the reduction's launch (out null: none)
};
int skinny_splits(int64_t M, int64_t C);
size_t skinny_partial_bytes(int64_t M, int64_t C);
cudaError_t launch_skinny(const uint16_t* In, int64_t M, int64_t C, const uint16_t* Wt, bool wt_is_rc, int r,
                          int64_t ldw, float* part, const SkinnyOut& out, int* status, cudaStream_t stream);
// hi/lo bf16 split of a compact fp32 [M][r] matrix into [M][64] buffers.
cudaError_t launch_split_hilo(const float* src, int64_t M, int r, uint16_t* hi, uint16_t* lo, cudaStream_t stream);

// Column sums over tokens: out(c, j) = scale * sum_m In[m][c] * (hi[m][j] + lo[m][j]).
// part: [ms][C][64] fp32 partials; then written to dst as [C][r] (dst_rc = false)
// or [r][C] (dst_rc = true).
int colsum_splits(int64_t M, int64_t C);
size_t colsum_partial_bytes(int64_t M, int64_t C);
cudaError_t launch_colsum(const uint16_t* In, int64_t M, int64_t C, const uint16_t* hi, const uint16_t* lo, int r,
                          float scale, float* part, float* dst, bool dst_rc, int* status, cudaStream_t stream);

// Both rank-r products of the backward from one pass over G = dY [M][N]
// (vdb_tc.cu, ranks 1..kVdbMaxRank; wider ranks use launch_skinny +
// launch_colsum): V = G B written as vs = s*V (bf16 [M][64]) and its hi / lo
// split (vhi, vlo, [M][64]); dB = scale * G^T (uhi + ulo) into dB [N][r] (may
// be null).  B is [N][ldb] bf16 with r valid columns.
constexpr int kVdbMaxRank = 16;
// The pass writes partials [ncb][M][16] and [ntb][N][16] fp32 (`part`, vdb_tc_partial_bytes
// bytes); bt [16][N], uht and ult [16][vdb_tc_ldm(M)] are bf16 scratch for
// B^T and the transposed U split.  U comes either as the hi / lo split
// (uhi / ulo [M][64], as launch_skinny writes it; u32 null) or as the saved
// fp32 U [M][r] (u32; uhi / ulo unused), which the transposes split
// themselves.
struct VdbTcGrid {
  int ct, tt, ncb, ntb;  // column / token tiles per CTA; column / token blocks
};
VdbTcGrid vdb_tc_grid(int64_t M, int64_t N);
size_t vdb_tc_partial_bytes(int64_t M, int64_t N);
inline int64_t vdb_tc_ldm(int64_t M) { return (M + 7) / 8 * 8; }  // 16-byte rows for TMA
// `bs`: a block-scales job run in the reduction's launch (out null: none).
cudaError_t launch_vdb_tc(const uint16_t* G, int64_t M, int64_t N, const uint16_t* B, int64_t ldb,
                          const uint16_t* uhi, const uint16_t* ulo, const float* u32, int r, float scale, float* part,
                          uint16_t* bt, uint16_t* uht, uint16_t* ult, uint16_t* vs, uint16_t* vhi, uint16_t* vlo,
                          float* dB, const BlockScalesJob& bs, int* status, cudaStream_t stream);
// The fixed-order reduction of vdb partials [ncb][M][16] and [ntb][N][16],
// plus the block-scales job `bs` on further threads.
cudaError_t launch_vdb_finalize(const float* vpart, int ncb, const float* dbpart, int ntb, int64_t M, int64_t N,
                                int r, float scale, uint16_t* vs, uint16_t* vhi, uint16_t* vlo, float* dB,
                                const BlockScalesJob& bs, cudaStream_t stream);

// Copy a bf16 [rows][r] matrix into [rows][64] zero padded, optionally from
// the transposed source [r][rows].
cudaError_t launch_pad_rank(const uint16_t* src, bool src_transposed, int64_t rows, int r, uint16_t* dst,
                            cudaStream_t stream);

// ---------------------------------------------------------------------------
// tcgen05 GEMM (gemm_tc.cu):  D[M][N] (+)= A[M][K] B[N][K]^T + A2[M][64] B2[N][64]^T
// ---------------------------------------------------------------------------
struct GemmArgs {
  const uint16_t* A;   // [M][K]
  const uint16_t* B;   // K-major: [N][ldb] (ldb = 0: K);  MN-major: [K][N]
  const uint16_t* A2;  // [M][64] bf16, zero padded beyond r; null: no rank step
  const uint16_t* B2;  // K-major: [N][ldb2] with r valid columns;  MN-major: [r][N]
  int64_t M, N, K;
  int r;               // rank of the extra product (<= 64)
  uint16_t* D;
  int accumulate;      // D += ... instead of D = ...
  int* status;
  int b_mn_major;      // 0: B and B2 K-major; 1: B and B2 MN-major
  int64_t ldb, ldb2;   // row pitches (elements) of K-major B / B2 (0: dense)
};
cudaError_t launch_gemm_tn(const GemmArgs& a, cudaStream_t stream);

// ---------------------------------------------------------------------------
// tcgen05 GEMM with the 4-bit weight decoded in the kernel (gemm_nf4.cu):
//   forward   D [M][N_w] = A [M][K_w] W_hat^T + A2 [M][64] B2^T  (B2 = LoRA B [N_w][ldb2])
//   backward  D [M][K_w] = A [M][N_w] W_hat   + A2 [M][64] B2    (B2 = LoRA A [r][K_w])
// ---------------------------------------------------------------------------
struct Nf4GemmArgs {
  WeightView w;
  const float* scales; // decoded block scales [N_w][block_scales_ld(K_w)] (launch_block_scales)
  const uint16_t* A;   // X (forward) or dY (backward), bf16 row-major
  const uint16_t* A2;  // [M][64] bf16 s*U or s*V, zero padded beyond r; null: no rank step
  const uint16_t* B2;  // see above
  int64_t M;
  int r;
  int64_t ldb2;        // row pitch (elements) of the forward's B2
  uint16_t* D;
  int accumulate;      // D += ... instead of D = ...
  int* status;
  int backward;        // 0: forward, 1: backward-input
  // Diagnostics (zero in every product call): a wait limit for the pipeline
  // waits (0: the default one second) and debug_stall = 1 to hold the MMA
  // issuer on a barrier nothing arrives at, so the abort path runs.
  uint64_t wait_limit_ns;
  int debug_stall;
};

// Kernel parameters (the launcher fills them from Nf4GemmArgs).
struct Nf4GemmParams {
  const uint8_t* packed;
  const int8_t* qscale;
  const float* c2;
  const float* mu;
  const float* absmax;
  int codebook, scale_format;
  int64_t Nw, Kw;      // weight [N_w][K_w]
  int M, N, num_k, r_steps;
  uint16_t* D;
  int accumulate;
  int* status;
  int group, along_n;  // tile raster
  int wide_store;      // output rows 32-byte aligned and no accumulation: 32-byte stores
  int full_tiles;      // pair tiles taken whole; the ones after them are split into two halves
  int items;           // work items: full_tiles whole tiles, then the halves
  uint64_t wait_limit_ns;
  int debug_stall;
};

// Returns cudaErrorNotSupported when pair clusters of the kernel cannot be
// scheduled on the current device (the caller then takes the dense path).
cudaError_t launch_gemm_nf4(const Nf4GemmArgs& a, cudaStream_t stream);

// Driver entry point used to encode TMA descriptors (resolved once).
bool encode_tensor_map_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                          uint32_t box_cols, bool swizzle128 = true, uint64_t ld = 0);
// uint8 (elem_bytes 1) or fp32 (4) row-major tensor, pitch ld elements, no swizzle.
bool encode_tensor_map_2d_plain(CUtensorMap* map, const void* base, int elem_bytes, uint64_t rows, uint64_t cols,
                                uint64_t ld, uint32_t box_rows, uint32_t box_cols);

// ---------------------------------------------------------------------------
// Barrier ring self-test (selftest.cu)
// ---------------------------------------------------------------------------

// result (device int[3]) is cleared, then receives the wrong / read counts and
// the timeout status of the ring kernel.
cudaError_t launch_mbarrier_ring_selftest(int stages, int consumers, int iters, uint64_t limit_ns, int* result,
                                          cudaStream_t stream);
// *result = QLORA_ERR_CHECK when the device code was built with QLORA_CHECKS, else 0.
cudaError_t launch_checks_selftest(int* result, cudaStream_t stream);

}  // namespace qnf4
