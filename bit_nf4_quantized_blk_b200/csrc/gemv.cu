// Decode-shaped LoRA linear forward, M <= 16 tokens (sm_100a).
//
//   Y = X W_hat^T + s (X A^T) B^T       ("QLoRA: NF4 storage, gradients and
//   local integration", FrozenNF4LoRA.forward; "FT-02: QLoRA -- Fine-Tuning
//   with Quantization", section "4. The LoRA mechanics the API wraps")
//
// The packed weight (0.5 B per weight) is the only large operand, so the
// kernel is HBM-bound: it streams the codes once and never writes a
// dequantized copy; the tensor cores (warp MMA, m16n8k16) do the products.
// The dequantized weight it uses is bf16(L[code]) * a, with the block scale a
// applied in fp32 to each block's partial sum (the training path and the
// dequantizer round fp32(L[code] * a) to bf16 instead; the difference is one
// bf16 rounding).  The rank-r term uses fp32 U = X A^T (small_xa_kernel,
// overlapped through programmatic dependent launch) and is added in the fp32
// epilogue after the cross-warp reduction.
#include "common.cuh"
#include "kernels.cuh"

namespace qnf4 {

namespace {
__device__ __forceinline__ uint32_t ld_shared_u32_lut(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
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

// One CTA owns 32 weight rows (two 16-row MMA tiles); its 4 warps split the
// row's 64-weight blocks.  Inside a block, lane (g = lane/4, t = lane%4)
// loads 8 bytes of each of its 4 rows (k = 16t .. 16t+15 of the block) and
// runs 4 k16 steps per row tile: step s takes bytes 2s and 2s+1, i.e.
// physical k = 16t + 4s + {0,1} for fragment slots {2t, 2t+1} and
// 16t + 4s + {2,3} for slots {2t+8, 2t+9}; X is read with the same map.  A
// block's MMAs accumulate bf16 levels L[code] into a fresh fp32 fragment that
// is then scaled by the block's decoded scale and added to the running sum.
// Levels come from a byte -> (L[lo], L[hi]) bf16 pair table replicated once
// per lane (table[byte][lane]), so the lookups never conflict.
template <bool kTwoTok>
__global__ void __launch_bounds__(128) gemv_kernel(WeightView w, const uint16_t* __restrict__ X, int M,
                                                   const uint16_t* __restrict__ B, int r, float scale,
                                                   const float* __restrict__ U32, uint16_t* __restrict__ Y) {
  extern __shared__ uint32_t s_lut[];        // [256][32] bf16 pairs (32 KB)
  __shared__ float s_red[4][32][16];          // [warp][row][token]
  __shared__ float s_qdiv[256];               // fp32(q / 127) for q = -128 .. 127
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  for (int e = tid; e < 256; e += 128) {
    const uint32_t pr = pack_bf16x2(nf4_level(e & 15), nf4_level(e >> 4));
    for (int l = 0; l < 32; ++l) s_lut[e * 32 + l] = pr;
    s_qdiv[e] = __fdiv_rn(static_cast<float>(e - 128), 127.0f);
  }

  const int64_t N = w.rows, K = w.cols;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int64_t kb = K / kBlock;  // blocks per row
  const int64_t b_begin = kb * warp / 4, b_end = kb * (warp + 1) / 4;
  const float mu = *w.mu;
  // Rows of this lane: g, g+8 (tile 0), 16+g, 24+g (tile 1); row (t) is the one
  // whose scale this lane decodes and shares.
  int64_t rows[4];
  bool rv[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    rows[i] = n0 + g + 8 * i;
    rv[i] = rows[i] < N;
  }
  const int64_t my_row = n0 + g + 8 * t;
  const bool my_rv = my_row < N;
  const uint32_t lut_lane = smem_u32(s_lut) + lane * 4;
  __syncthreads();

  float acc[2][2][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][b][c] = 0.0f;

  // Weights and scale codes of the next kAhead blocks stay in flight.
  constexpr int kAhead = 4;
  const int nblk = static_cast<int>(b_end - b_begin);
  uint2 wv[kAhead][4];
  int qv[kAhead];
  float c2v[kAhead];
  auto prefetch = [&](int j, int slot) {
#pragma unroll
    for (int i = 0; i < 4; ++i) wv[slot][i] = make_uint2(0, 0);
    qv[slot] = 0;
    c2v[slot] = 0.0f;
    if (j >= nblk) return;
    const int64_t b = b_begin + j;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (rv[i]) {
        const uint2* src = reinterpret_cast<const uint2*>(w.packed + (rows[i] * K + b * kBlock) / 2) + t;
        asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                     : "=r"(wv[slot][i].x), "=r"(wv[slot][i].y)
                     : "l"(src));
      }
    }
    if (my_rv) {
      const int64_t blk = my_row * kb + b;
      qv[slot] = w.qscale[blk];
      c2v[slot] = w.c2[blk / kDqBlock];
    }
  };
#pragma unroll
  for (int u = 0; u < kAhead; ++u) prefetch(u, u);

  for (int j0 = 0; j0 < nblk; j0 += kAhead) {
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      const int j = j0 + u;
      if (j < nblk) {
        const int64_t b = b_begin + j;
        // Decoded scale of row my_row, shared with the 4 lanes of the quad.
        const float a_mine = my_rv ? __fadd_rn(__fmul_rn(s_qdiv[qv[u] + 128], c2v[u]), mu) : 0.0f;
        float av[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = __shfl_sync(0xffffffffu, a_mine, (lane & ~3) | i);
        // X fragments: 16 consecutive k of token g (tile 0) and g+8 (tile 1).
        uint32_t xf[2][8];
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
          const int tok = g + 8 * tt;
          uint4 x0 = make_uint4(0, 0, 0, 0), x1 = make_uint4(0, 0, 0, 0);
          if ((tt == 0 || kTwoTok) && tok < M) {
            const uint4* xs = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(tok) * K + b * kBlock + 16 * t);
            x0 = __ldg(xs);
            x1 = __ldg(xs + 1);
          }
          xf[tt][0] = x0.x; xf[tt][1] = x0.y; xf[tt][2] = x0.z; xf[tt][3] = x0.w;
          xf[tt][4] = x1.x; xf[tt][5] = x1.y; xf[tt][6] = x1.z; xf[tt][7] = x1.w;
        }
        uint2 cur[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) cur[i] = wv[u][i];
        prefetch(j + kAhead, u);
#pragma unroll
        for (int rt = 0; rt < 2; ++rt) {
          float d[2][4];
#pragma unroll
          for (int tt = 0; tt < 2; ++tt)
#pragma unroll
            for (int c = 0; c < 4; ++c) d[tt][c] = 0.0f;
          const uint2 lo = cur[2 * rt], hi = cur[2 * rt + 1];  // rows g(+16rt), g+8(+16rt)
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const uint32_t wl = s < 2 ? lo.x : lo.y, wh = s < 2 ? hi.x : hi.y;
            const int sh = (s & 1) * 16;
            uint32_t afr[4];
            afr[0] = ld_shared_u32_lut(lut_lane + ((wl >> sh) & 0xFF) * 128);
            afr[1] = ld_shared_u32_lut(lut_lane + ((wh >> sh) & 0xFF) * 128);
            afr[2] = ld_shared_u32_lut(lut_lane + ((wl >> (sh + 8)) & 0xFF) * 128);
            afr[3] = ld_shared_u32_lut(lut_lane + ((wh >> (sh + 8)) & 0xFF) * 128);
            const uint32_t b0[2] = {xf[0][2 * s], xf[0][2 * s + 1]};
            mma_bf16_16816(d[0], afr, b0);
            if constexpr (kTwoTok) {
              const uint32_t b1[2] = {xf[1][2 * s], xf[1][2 * s + 1]};
              mma_bf16_16816(d[1], afr, b1);
            }
          }
#pragma unroll
          for (int tt = 0; tt < (kTwoTok ? 2 : 1); ++tt) {
            acc[rt][tt][0] = fmaf(av[2 * rt], d[tt][0], acc[rt][tt][0]);
            acc[rt][tt][1] = fmaf(av[2 * rt], d[tt][1], acc[rt][tt][1]);
            acc[rt][tt][2] = fmaf(av[2 * rt + 1], d[tt][2], acc[rt][tt][2]);
            acc[rt][tt][3] = fmaf(av[2 * rt + 1], d[tt][3], acc[rt][tt][3]);
          }
        }
      }
    }
  }

  // Cross-warp reduction.  D fragment: rows g / g+8 of the tile, tokens 2t, 2t+1.
#pragma unroll
  for (int rt = 0; rt < 2; ++rt)
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      s_red[warp][16 * rt + g][tt * 8 + 2 * t] = acc[rt][tt][0];
      s_red[warp][16 * rt + g][tt * 8 + 2 * t + 1] = acc[rt][tt][1];
      s_red[warp][16 * rt + g + 8][tt * 8 + 2 * t] = acc[rt][tt][2];
      s_red[warp][16 * rt + g + 8][tt * 8 + 2 * t + 1] = acc[rt][tt][3];
    }
  __syncthreads();
  // U comes from the preceding small_xa_kernel.
  pdl_wait_prior();
  for (int o = tid; o < 32 * 16; o += 128) {
    const int row = o & 31, tok = o >> 5;
    const int64_t n = n0 + row;
    if (tok >= M || n >= N) continue;
    float y = s_red[0][row][tok] + s_red[1][row][tok] + s_red[2][row][tok] + s_red[3][row][tok];
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
  constexpr int kLutBytes = 256 * 32 * 4;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemv_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((w.rows + 31) / 32));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = kLutBytes;
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
