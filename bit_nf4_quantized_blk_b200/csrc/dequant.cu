// 4-bit dequantization to dense bf16 / fp32 (sm_100a).
//
// Method: "QLoRA Deep Dive: 4-bit NormalFloat & Double Quantization
// Internals", section "The Quantization Process in QLoRA" (load the 4-bit
// codes and the block constant, multiply, cast to bf16); "QLoRA: NF4 storage,
// gradients and local integration", ``dequantize_nf4`` of the teaching
// program.  Block scale decode a = fp32(fp32(t * c2) + mu) (t = fp32(q/127)
// for int8 codes, the E4M3 value for FP8 codes) or the stored fp32 absmax;
// weight fp32(L[code] * a) with L the NF4 or FP4 codebook; bf16 output
// rounds that value to nearest even.
//
// HBM-bound: 0.5 B of codes + 1/64 B of scale codes read and 2 B (bf16) or
// 4 B (fp32) written per weight.
#include "common.cuh"
#include "kernels.cuh"

namespace qnf4 {

namespace {

__device__ __forceinline__ void fill_pair_table(float2* tab, int codebook) {
  for (int b = threadIdx.x; b < 256; b += blockDim.x)
    tab[b] = make_float2(codebook_level(codebook, b & 15), codebook_level(codebook, b >> 4));
}

}  // namespace

__device__ __forceinline__ int find_tensor_seg(const DequantBatchParams& p, int64_t seg) {
  int lo = 0, hi = p.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.begin_seg[mid] <= seg) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// One warp per 2 KB segment of packed codes (4096 weights): lane t loads the
// 16-byte units t, t+32, t+64, t+96 of the segment (every load instruction of
// the warp reads 512 contiguous bytes, all four are in flight together) and
// writes each unit's 32 outputs with 256-bit stores (whole sectors).  Level
// lookup by shuffle: lane l holds L[l % 16], and a shuffle reads its source
// lane modulo 32, so `word >> 4i` selects L[nibble i] with no masking and no
// shared-memory table.
//
// kAnyFormat = false: every tensor of the batch is NF4 with int8 scale codes
// (the default format), decoded without the per-tensor format dispatch.
template <bool kFp32, bool kAnyFormat>
__global__ void __launch_bounds__(256) dequant_kernel(const __grid_constant__ DequantBatchParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t gseg = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (gseg >= p.total_seg) return;
  const int t = find_tensor_seg(p, gseg);
  const float level = kAnyFormat ? codebook_level(p.codebook[t], lane & 15) : nf4_level(lane & 15);
  const int64_t seg = gseg - p.begin_seg[t];
  const int64_t n_units = p.n_units[t];
  const uint4* __restrict__ packed = reinterpret_cast<const uint4*>(p.packed[t]);
  const int fmt = kAnyFormat ? p.scale_format[t] : kScalesDqInt8;
  const float mu = fmt == kScalesFp32 ? 0.0f : *p.mu[t];
  uint4 pk[4];
  float a[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int64_t u = seg * 128 + lane + 32 * q;
    pk[q] = make_uint4(0, 0, 0, 0);
    a[q] = 0.0f;
    if (u < n_units) pk[q] = ld_stream_u4(packed + u);
  }
  // Scales of the four units (two units per 64-weight block); one uniform
  // branch on the format, the loads of each branch issued together.
  if (kAnyFormat && fmt == kScalesFp32) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t u = seg * 128 + lane + 32 * q;
      if (u < n_units) a[q] = p.absmax[t][u >> 1];
    }
  } else {
    int qv[4];
    float c2v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t u = seg * 128 + lane + 32 * q;
      qv[q] = 0;
      c2v[q] = 0.0f;
      if (u < n_units) {
        qv[q] = p.qscale[t][u >> 1];
        c2v[q] = p.c2[t][(u >> 1) / kDqBlock];
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t u = seg * 128 + lane + 32 * q;
      if (u < n_units)
        a[q] = kAnyFormat ? decode_scale_value(scale_code_value(fmt, static_cast<int8_t>(qv[q])), c2v[q], mu)
                          : decode_scale(qv[q], c2v[q], mu);
    }
  }
  // Every lane takes part in the shuffles; units past the end are skipped
  // only at the stores.
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int64_t u = seg * 128 + lane + 32 * q;
    const bool live = u < n_units;
    const uint32_t words[4] = {pk[q].x, pk[q].y, pk[q].z, pk[q].w};
    if constexpr (kFp32) {
      float* o = static_cast<float*>(p.out[t]) + u * 32;
#pragma unroll
      for (int h = 0; h < 4; ++h) {  // 8 weights (one word) per 32-byte store
        uint32_t vals[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float lv = __shfl_sync(0xffffffffu, level, static_cast<int>(words[h] >> (4 * i)));
          vals[i] = __float_as_uint(__fmul_rn(lv, a[q]));
        }
        if (live) st_stream_v8(o + 8 * h, vals);
      }
    } else {
      uint16_t* o = static_cast<uint16_t*>(p.out[t]) + u * 32;
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // 16 weights (two words) per 32-byte store
        uint32_t pr[8];
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          const uint32_t w = words[2 * h + (b >> 2)] >> (8 * (b & 3));
          const float lo = __shfl_sync(0xffffffffu, level, static_cast<int>(w));
          const float hi = __shfl_sync(0xffffffffu, level, static_cast<int>(w >> 4));
          pr[b] = pack_bf16x2(__fmul_rn(lo, a[q]), __fmul_rn(hi, a[q]));
        }
        if (live) st_stream_v8(o + 16 * h, pr);
      }
    }
  }
}

// Transposed bf16 output out[k][n] = W_hat[n][k]: one CTA per 64 x 64 tile
// (exactly one block per row of the tile), staged through shared memory.
__global__ void __launch_bounds__(256) dequant_transposed_kernel(WeightView w, uint16_t* __restrict__ out) {
  __shared__ float2 s_pair[256];
  __shared__ __align__(16) uint16_t s_t[64][64];  // [k][n]
  fill_pair_table(s_pair, w.codebook);
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * 64;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * 64;
  const int tid = threadIdx.x;
  const int nn = tid & 63;         // row of the weight tile
  const int kq = (tid >> 6) * 16;  // 16 weights of that row
  const int64_t n = n0 + nn;
  __syncthreads();
  uint32_t lo = 0, hi = 0;
  float a = 0.0f;
  if (n < w.rows) {
    const int64_t blk = (n * w.cols + k0) / kBlock;
    a = weight_block_scale(w, blk, weight_mu(w));
    const uint2 pk = *reinterpret_cast<const uint2*>(w.packed + (n * w.cols + k0 + kq) / 2);
    lo = pk.x;
    hi = pk.y;
  }
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    const uint32_t byte = ((b < 4 ? lo : hi) >> (8 * (b & 3))) & 0xFF;
    const float2 lv = s_pair[byte];
    const uint32_t pr = pack_bf16x2(__fmul_rn(lv.x, a), __fmul_rn(lv.y, a));
    s_t[kq + 2 * b][nn] = static_cast<uint16_t>(pr & 0xFFFF);
    s_t[kq + 2 * b + 1][nn] = static_cast<uint16_t>(pr >> 16);
  }
  __syncthreads();
  const int kk = tid >> 2;        // output row within the tile
  const int nc = (tid & 3) * 16;  // 16 outputs of that row
  const int64_t k = k0 + kk;
  if (k >= w.cols) return;
  uint16_t* dst = out + k * w.rows + n0 + nc;
  if (n0 + nc + 16 <= w.rows) {
    const uint4* src = reinterpret_cast<const uint4*>(&s_t[kk][nc]);
    reinterpret_cast<uint4*>(dst)[0] = src[0];
    reinterpret_cast<uint4*>(dst)[1] = src[1];
  } else {
    for (int j = 0; j < 16; ++j)
      if (n0 + nc + j < w.rows) dst[j] = s_t[kk][nc + j];
  }
}

// Decoded block scales of a weight as an fp32 [rows][ld] array (ld >= cols /
// 64; the pad columns are 0), read by the 4-bit GEMM's tile producer: the same
// a = fp32(fp32(t * c2) + mu), or the stored fp32 absmax, that every decoder
// of this library applies.  Four blocks per thread (one 16-byte store;
// block_scales_group).  The linear calls usually run this job on spare
// threads of the U or V reduction that precedes the GEMM; this kernel runs
// it alone.
__global__ void __launch_bounds__(256) block_scales_kernel(BlockScalesJob j) {
  const int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // 4-column group
  if (q < j.groups) block_scales_group(j, q);
}

int64_t block_scales_ld(int64_t cols) { return (cols / kBlock + 3) / 4 * 4; }

BlockScalesJob block_scales_job(const WeightView& w, float* out) {
  BlockScalesJob j;
  j.w = w;
  j.out = out;
  j.ld = block_scales_ld(w.cols);
  j.groups = w.rows * (j.ld / 4);
  return j;
}

cudaError_t launch_block_scales(const WeightView& w, float* out, cudaStream_t stream) {
  const BlockScalesJob j = block_scales_job(w, out);
  block_scales_kernel<<<static_cast<unsigned>((j.groups + 255) / 256), 256, 0, stream>>>(j);
  return cudaGetLastError();
}

cudaError_t launch_dequant_batch(const DequantBatchParams& p, int out_fp32, cudaStream_t stream) {
  if (p.total_seg <= 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((p.total_seg + 7) / 8);  // 8 warps per CTA
  bool any_format = false;
  for (int i = 0; i < p.count; ++i)
    any_format |= p.codebook[i] != QLORA_CODEBOOK_NF4 || p.scale_format[i] != kScalesDqInt8;
  if (out_fp32) {
    if (any_format) dequant_kernel<true, true><<<grid, 256, 0, stream>>>(p);
    else dequant_kernel<true, false><<<grid, 256, 0, stream>>>(p);
  } else {
    if (any_format) dequant_kernel<false, true><<<grid, 256, 0, stream>>>(p);
    else dequant_kernel<false, false><<<grid, 256, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_dequant_transposed(const WeightView& w, uint16_t* out, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>(w.cols / 64), static_cast<unsigned>((w.rows + 63) / 64));
  dequant_transposed_kernel<<<grid, 256, 0, stream>>>(w, out);
  return cudaGetLastError();
}

}  // namespace qnf4
