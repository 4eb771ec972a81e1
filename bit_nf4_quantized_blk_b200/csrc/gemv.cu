// Decode-shaped LoRA linear forward, M <= 16 tokens (sm_100a).
//
//   Y = X W_hat^T + s (X A^T) B^T       ("QLoRA: NF4 storage, gradients and
//   local integration", FrozenNF4LoRA.forward; "FT-02: QLoRA -- Fine-Tuning
//   with Quantization", section "4. The LoRA mechanics the API wraps")
//
// The packed weight (0.5 B per weight) is the only large operand, so the
// kernel is HBM-bound: it streams the codes once with 128-bit loads and never
// writes a dequantized copy.  One CTA owns 16 weight rows; its 8 warps split
// K into 128-wide segments.  In a segment each lane loads 16 bytes of two
// rows (rows g and g+8, k = 32t .. 32t+31 of the segment, g = lane/4,
// t = lane%4) and turns them directly into the A fragments of eight
// m16n8k16 tensor-core steps; X supplies the B fragments.  Because a dot
// product is invariant under a common permutation of k, the lane's 32
// consecutive k values are mapped onto the fragment's k slots in whatever
// order makes both loads contiguous: step s takes bytes 2s and 2s+1, i.e.
// physical k = 32t + 4s + {0,1} for fragment slots {2t, 2t+1} and
// 32t + 4s + {2,3} for slots {2t+8, 2t+9}; the X fragment is read with the
// same map (four consecutive bf16 per step).  Each lane's 32 k values lie in
// one 64-weight block, so one decoded scale serves them.
//
// Dequantized values are bit-identical to the dequantizer: fp32(L[c] * a)
// rounded to bf16.  The rank-r term uses fp32 U = X A^T (computed by
// small_xa_kernel, overlapped through programmatic dependent launch) and is
// added in the fp32 epilogue after the cross-warp reduction.
#include "common.cuh"
#include "kernels.cuh"

namespace qnf4 {

namespace {
constexpr int kGvWarps = 8;
constexpr int kSegK = 128;     // k per segment
constexpr int kSegBatch = 4;   // segments loaded ahead per warp
}  // namespace

__global__ void __launch_bounds__(256) small_xa_kernel(const uint16_t* __restrict__ X, const uint16_t* __restrict__ A,
                                                       int M, int K, int r, float* __restrict__ U32,
                                                       float* __restrict__ U_out) {
  pdl_launch_dependents();
  __shared__ float s_red[8][kGemvMaxM];
  const int j = blockIdx.x;  // rank index
  const int tid = threadIdx.x;
  float acc[kGemvMaxM];
#pragma unroll
  for (int m = 0; m < kGemvMaxM; ++m) acc[m] = 0.0f;
  for (int k = tid * 8; k < K; k += 256 * 8) {
    const uint4 av = *reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j) * K + k);
    const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
    for (int m = 0; m < kGemvMaxM; ++m) {
      if (m < M) {
        const uint4 xv = *reinterpret_cast<const uint4*>(X + static_cast<int64_t>(m) * K + k);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[m] = fmaf(bf16_bits_to_float(xw[q] & 0xFFFF), bf16_bits_to_float(aw[q] & 0xFFFF), acc[m]);
          acc[m] = fmaf(bf16_bits_to_float(xw[q] >> 16), bf16_bits_to_float(aw[q] >> 16), acc[m]);
        }
      }
    }
  }
  const int warp = tid >> 5, lane = tid & 31;
#pragma unroll
  for (int m = 0; m < kGemvMaxM; ++m) {
    float v = acc[m];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_red[warp][m] = v;
  }
  __syncthreads();
  if (tid < M) {
    float u = 0.0f;
    for (int w = 0; w < 8; ++w) u += s_red[w][tid];
    U32[tid * kRankPad + j] = u;
    if (U_out != nullptr) U_out[tid * r + j] = u;
  }
}

__device__ __forceinline__ uint32_t dq_pair(const float2* lut, uint32_t byte, float a) {
  const float2 lv = lut[byte];
  return pack_bf16x2(__fmul_rn(lv.x, a), __fmul_rn(lv.y, a));
}

template <bool kTwoTiles>
__global__ void __launch_bounds__(256) gemv_kernel(WeightView w, const uint16_t* __restrict__ X, int M,
                                                   const uint16_t* __restrict__ B, int r, float scale,
                                                   const float* __restrict__ U32, uint16_t* __restrict__ Y) {
  __shared__ float2 s_lut[256];
  __shared__ float s_red[kGvWarps][16][16];  // [warp][row][token]
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  for (int b = tid; b < 256; b += 256) s_lut[b] = make_float2(nf4_level(b & 15), nf4_level(b >> 4));

  const int64_t N = w.rows, K = w.cols;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 16;
  const int64_t row0 = n0 + g, row1 = n0 + g + 8;
  const bool v0 = row0 < N, v1 = row1 < N;
  const int64_t kb = K / kBlock;  // blocks per row
  const float mu = *w.mu;
  const int nseg = static_cast<int>((K + kSegK - 1) / kSegK);
  __syncthreads();

  float acc[2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

  for (int sb = warp; sb < nseg; sb += kGvWarps * kSegBatch) {
    uint4 wr0[kSegBatch], wr1[kSegBatch];
    float a0[kSegBatch], a1[kSegBatch];
    // Issue all weight loads of this batch first.
#pragma unroll
    for (int u = 0; u < kSegBatch; ++u) {
      const int seg = sb + u * kGvWarps;
      const int64_t k = static_cast<int64_t>(seg) * kSegK + 32 * t;
      const bool kv = seg < nseg && k < K;
      wr0[u] = (kv && v0) ? ld_stream_u4(w.packed + (row0 * K + k) / 2) : make_uint4(0, 0, 0, 0);
      wr1[u] = (kv && v1) ? ld_stream_u4(w.packed + (row1 * K + k) / 2) : make_uint4(0, 0, 0, 0);
      a0[u] = 0.0f;
      a1[u] = 0.0f;
      if (kv && v0) {
        const int64_t blk = row0 * kb + k / kBlock;
        a0[u] = decode_scale(w.qscale[blk], w.c2[blk / kDqBlock], mu);
      }
      if (kv && v1) {
        const int64_t blk = row1 * kb + k / kBlock;
        a1[u] = decode_scale(w.qscale[blk], w.c2[blk / kDqBlock], mu);
      }
    }
#pragma unroll
    for (int u = 0; u < kSegBatch; ++u) {
      const int seg = sb + u * kGvWarps;
      const int64_t k = static_cast<int64_t>(seg) * kSegK + 32 * t;
      const bool kv = seg < nseg && k < K;
      // X fragments: 32 consecutive k of token g (tile 0) and token g+8 (tile 1).
      uint32_t x0[16], x1[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (kv && g < M) v = __ldg(reinterpret_cast<const uint4*>(X + static_cast<int64_t>(g) * K + k) + q);
        x0[4 * q] = v.x; x0[4 * q + 1] = v.y; x0[4 * q + 2] = v.z; x0[4 * q + 3] = v.w;
        if constexpr (kTwoTiles) {
          uint4 v2 = make_uint4(0, 0, 0, 0);
          if (kv && g + 8 < M) v2 = __ldg(reinterpret_cast<const uint4*>(X + static_cast<int64_t>(g + 8) * K + k) + q);
          x1[4 * q] = v2.x; x1[4 * q + 1] = v2.y; x1[4 * q + 2] = v2.z; x1[4 * q + 3] = v2.w;
        }
      }
      const uint32_t w0[4] = {wr0[u].x, wr0[u].y, wr0[u].z, wr0[u].w};
      const uint32_t w1[4] = {wr1[u].x, wr1[u].y, wr1[u].z, wr1[u].w};
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint32_t word0 = w0[s >> 1], word1 = w1[s >> 1];
        const int sh = (s & 1) * 16;
        uint32_t afr[4];
        afr[0] = dq_pair(s_lut, (word0 >> sh) & 0xFF, a0[u]);        // row g,   slots 2t, 2t+1
        afr[1] = dq_pair(s_lut, (word1 >> sh) & 0xFF, a1[u]);        // row g+8, slots 2t, 2t+1
        afr[2] = dq_pair(s_lut, (word0 >> (sh + 8)) & 0xFF, a0[u]);  // row g,   slots 2t+8, 2t+9
        afr[3] = dq_pair(s_lut, (word1 >> (sh + 8)) & 0xFF, a1[u]);  // row g+8, slots 2t+8, 2t+9
        const uint32_t b0[2] = {x0[2 * s], x0[2 * s + 1]};
        mma_bf16_16816(acc[0], afr, b0);
        if constexpr (kTwoTiles) {
          const uint32_t b1[2] = {x1[2 * s], x1[2 * s + 1]};
          mma_bf16_16816(acc[1], afr, b1);
        }
      }
    }
  }

  // Cross-warp reduction: D fragment (row g / g+8, tokens 2t, 2t+1 of each tile).
#pragma unroll
  for (int tile = 0; tile < 2; ++tile) {
    s_red[warp][g][tile * 8 + 2 * t] = acc[tile][0];
    s_red[warp][g][tile * 8 + 2 * t + 1] = acc[tile][1];
    s_red[warp][g + 8][tile * 8 + 2 * t] = acc[tile][2];
    s_red[warp][g + 8][tile * 8 + 2 * t + 1] = acc[tile][3];
  }
  __syncthreads();
  // U comes from the preceding small_xa_kernel.
  pdl_wait_prior();
  const int row = tid & 15, tok = tid >> 4;
  const int64_t n = n0 + row;
  if (tok < M && n < N) {
    float y = 0.0f;
#pragma unroll
    for (int wv = 0; wv < kGvWarps; ++wv) y += s_red[wv][row][tok];
    float l = 0.0f;
    for (int j = 0; j < r; ++j) l = fmaf(U32[tok * kRankPad + j], bf16_bits_to_float(B[n * r + j]), l);
    y = fmaf(scale, l, y);
    Y[static_cast<int64_t>(tok) * N + n] = static_cast<uint16_t>(pack_bf16x2(y, 0.0f) & 0xFFFF);
  }
}

cudaError_t launch_small_xa(const uint16_t* X, const uint16_t* A, int M, int K, int r, float* U32, float* U_out,
                            cudaStream_t stream) {
  small_xa_kernel<<<r, 256, 0, stream>>>(X, A, M, K, r, U32, U_out);
  return cudaGetLastError();
}

cudaError_t launch_gemv(const WeightView& w, const uint16_t* X, int M, const uint16_t* B, int r, float scale,
                        const float* U32, uint16_t* Y, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((w.rows + 15) / 16));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (M > 8) return cudaLaunchKernelEx(&cfg, gemv_kernel<true>, w, X, M, B, r, scale, U32, Y);
  return cudaLaunchKernelEx(&cfg, gemv_kernel<false>, w, X, M, B, r, scale, U32, Y);
}

}  // namespace qnf4
