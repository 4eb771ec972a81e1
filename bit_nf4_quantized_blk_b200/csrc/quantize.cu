// NF4 blockwise quantization and double quantization (sm_100a).
//
// Method: "QLoRA: NF4 storage, gradients and local integration", sections
// "NF4: nonuniform reconstruction levels", "Double quantization: correct the
// scale arithmetic" and "Exact CPU teaching quantizer and adapter gradient
// path"; "QLoRA Deep Dive: 4-bit NormalFloat & Double Quantization
// Internals", section "2. Squeezing More Memory: Double Quantization (DQ)".
//
// Two kernels per batch of tensors:
//
//  quantize_chunks  one CTA per chunk of 256 blocks (16384 weights).  Each
//                   group of 8 lanes owns one 64-weight block: 256-bit loads,
//                   absmax by three xor-shuffles, IEEE fp32 division by the
//                   absmax (by 1 for an all-zero block; a reciprocal multiply
//                   with an exact-division fallback next to a threshold),
//                   nearest level from a
//                   129-cell decision table, eight codes packed into one
//                   32-bit word (even element in the low nibble).  The CTA
//                   then forms the fp64 sum of its 256 block scales and the
//                   last CTA of each tensor forms the tensor's mean offset.
//  dq_chunks        one warp per chunk: d = a - mu, c2 = max|d|,
//                   q = rint(fp32(fp32(d / c2) * 127)) (0 where c2 == 0).
//
// The mean is defined as a strictly sequential fp64 sum (inside each chunk,
// then over chunk sums).  When the exponents of the summed values span few
// enough binades every partial sum is exact in fp64, so a tree reduction
// gives the same bits; the kernels check that bound and fall back to a
// sequential loop when it does not hold.
#include "common.cuh"
#include "kernels.cuh"

namespace qnf4 {

namespace {

__device__ __forceinline__ int find_tensor(const QuantBatchParams& p, int64_t chunk) {
  int lo = 0, hi = p.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.chunk_begin[mid] <= chunk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Effective biased exponent of a non-negative finite fp32 (subnormals count
// as exponent 1, whose unit is the same 2^-149).
__device__ __forceinline__ int exp_field(float v) {
  const int e = static_cast<int>((__float_as_uint(v) >> 23) & 0xFF);
  return e == 0 ? 1 : e;
}

__device__ __forceinline__ int ceil_log2(int64_t n) {
  int b = 0;
  while ((int64_t{1} << b) < n) ++b;
  return b;
}

// True when n values whose exponents lie in [emin, emax] sum exactly in fp64
// in any order: all are multiples of 2^(emin-150) and every partial sum stays
// below 2^(emax-126) * n, which needs (emax - emin) + 24 + ceil(log2 n) <= 53.
__device__ __forceinline__ bool fp64_sum_is_exact(int emin, int emax, int64_t n) {
  if (emin > emax) return true;  // no nonzero value
  return (emax - emin) + 24 + ceil_log2(n) <= 53;
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint32_t nf4_code(float x, const float2* tab) {
  const int cell = __float2int_rz(x * 64.0f) + 64;  // x * 64 is exact
  const float2 e = tab[cell];
  return static_cast<uint32_t>(__float_as_int(e.y) + (x >= e.x ? 1 : 0));
}

// Code of w / a without a division per weight.  x' = fp32(w * rcp) with
// rcp = RN(1/a) differs from the correctly rounded quotient fp32(w / a) by
// less than 2^-22 |x|, so both fall on the same side of every decision
// threshold unless x' lies within that distance of one.  Every threshold is
// far (> 2^-14 relative) from the cell edges (checked when the table is
// built), so the only threshold that can lie that close is the one of x's
// cell; when |x' - thr| <= 2^-19 |thr| the exact IEEE quotient decides.
__device__ __forceinline__ uint32_t nf4_code_scaled(float w, float a, float rcp, const float2* tab) {
  const float xa = w * rcp;
  const int cell = __float2int_rz(xa * 64.0f) + 64;
  const float2 e = tab[cell];
  uint32_t code = static_cast<uint32_t>(__float_as_int(e.y) + (xa >= e.x ? 1 : 0));
  if (fabsf(xa - e.x) <= fabsf(e.x) * 0x1p-19f) code = nf4_code(__fdiv_rn(w, a), tab);
  return code;
}

}  // namespace

__global__ void __launch_bounds__(256) quantize_chunks_kernel(const __grid_constant__ QuantBatchParams p) {
  __shared__ float2 s_tab[129];
  __shared__ float s_absmax[kDqBlock];
  __shared__ double s_red[8];
  __shared__ int s_ered[16];
  __shared__ int s_last;

  const int tid = threadIdx.x;
  const int64_t g = blockIdx.x;
  const int t = find_tensor(p, g);
  const int64_t local_chunk = g - p.chunk_begin[t];
  const int64_t nb = p.n_blocks[t];
  const int64_t blk0 = local_chunk * kDqBlock;
  const int nblk = static_cast<int>(((nb - blk0) < kDqBlock ? (nb - blk0) : int64_t{kDqBlock}));
  const float* __restrict__ W = p.W[t];
  uint32_t* __restrict__ packed = reinterpret_cast<uint32_t*>(p.packed[t]);

  if (tid < 129) s_tab[tid] = make_float2(p.table.thr[tid], __int_as_float(p.table.base[tid]));

  const int grp = tid >> 3;  // 32 groups of 8 lanes
  const int l = tid & 7;     // lane in group: weights 8l .. 8l+7 of the block

  // Issue every load of this thread first (8 blocks x 32 bytes).
  float v[8][8];
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int b = it * 32 + grp;
    if (b < nblk) {
      ld_stream_v8(W + (blk0 + b) * kBlock + l * 8, v[it]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[it][i] = 0.0f;
    }
  }
  __syncthreads();  // decision table ready

  float nonfinite = 0.0f;  // becomes NaN if any input is NaN or +-Inf
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int b = it * 32 + grp;
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      m = fmaxf(m, fabsf(v[it][i]));
      nonfinite = fmaf(v[it][i], 0.0f, nonfinite);
    }
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
    const float div = (m == 0.0f) ? 1.0f : m;  // zero-block convention
    uint32_t word = 0;
    if (div >= 0x1p-125f && div <= 0x1p125f) {  // 1/div is a normal fp32
      const float rcp = __frcp_rn(div);
#pragma unroll
      for (int i = 7; i >= 0; --i) word = word * 16u + nf4_code_scaled(v[it][i], div, rcp, s_tab);
    } else {
#pragma unroll
      for (int i = 7; i >= 0; --i) word = word * 16u + nf4_code(__fdiv_rn(v[it][i], div), s_tab);
    }
    if (b < nblk) {
      packed[(blk0 + b) * (kBlock / 8) + l] = word;
      if (l == 0) {
        s_absmax[b] = m;
        p.absmax[g * kDqBlock + b] = m;
      }
    }
  }
  if (!(nonfinite == 0.0f)) raise_status(p.status, QLORA_ERR_NONFINITE);
  __syncthreads();

  // ---- fp64 sum of this chunk's block scales -------------------------------
  const float av = tid < nblk ? s_absmax[tid] : 0.0f;
  int emin = av > 0.0f ? exp_field(av) : 1 << 20;
  int emax = av > 0.0f ? exp_field(av) : -(1 << 20);
  emin = __reduce_min_sync(0xffffffffu, emin);
  emax = __reduce_max_sync(0xffffffffu, emax);
  const double wsum = warp_sum_f64(static_cast<double>(av));
  const int warp = tid >> 5, lane = tid & 31;
  if (lane == 0) {
    s_red[warp] = wsum;
    s_ered[warp] = emin;
    s_ered[8 + warp] = emax;
  }
  __syncthreads();
  if (tid == 0) {
    int cmin = s_ered[0], cmax = s_ered[8];
    double s = 0.0;
    for (int w = 0; w < 8; ++w) {
      cmin = min(cmin, s_ered[w]);
      cmax = max(cmax, s_ered[8 + w]);
      s += s_red[w];
    }
    if (!fp64_sum_is_exact(cmin, cmax, nblk)) {
      s = 0.0;  // the definition: left to right
      for (int b = 0; b < nblk; ++b) s += static_cast<double>(s_absmax[b]);
    }
    p.chunk_sum[g] = s;
    p.chunk_exp[2 * g] = cmin;
    p.chunk_exp[2 * g + 1] = cmax;
    __threadfence();
    const unsigned n_chunks = static_cast<unsigned>(p.chunk_begin[t + 1] - p.chunk_begin[t]);
    const unsigned ticket = atomicAdd(&p.counters[t], 1u);
    s_last = (ticket == n_chunks - 1) ? 1 : 0;
  }
  __syncthreads();
  if (!s_last) return;

  // ---- last CTA of tensor t: the mean offset ---------------------------------
  __threadfence();
  const int64_t c0 = p.chunk_begin[t], c1 = p.chunk_begin[t + 1];
  double part = 0.0;
  int tmin = 1 << 20, tmax = -(1 << 20);
  for (int64_t c = c0 + tid; c < c1; c += 256) {
    part += __ldcg(&p.chunk_sum[c]);
    tmin = min(tmin, __ldcg(&p.chunk_exp[2 * c]));
    tmax = max(tmax, __ldcg(&p.chunk_exp[2 * c + 1]));
  }
  part = warp_sum_f64(part);
  tmin = __reduce_min_sync(0xffffffffu, tmin);
  tmax = __reduce_max_sync(0xffffffffu, tmax);
  __syncthreads();
  if (lane == 0) {
    s_red[warp] = part;
    s_ered[warp] = tmin;
    s_ered[8 + warp] = tmax;
  }
  __syncthreads();
  if (tid == 0) {
    int gmin = s_ered[0], gmax = s_ered[8];
    double s = 0.0;
    for (int w = 0; w < 8; ++w) {
      gmin = min(gmin, s_ered[w]);
      gmax = max(gmax, s_ered[8 + w]);
      s += s_red[w];
    }
    if (!fp64_sum_is_exact(gmin, gmax, nb)) {
      s = 0.0;  // the definition: chunk sums left to right
      for (int64_t c = c0; c < c1; ++c) s += __ldcg(&p.chunk_sum[c]);
    }
    *p.mu[t] = __double2float_rn(s / static_cast<double>(nb));
    p.counters[t] = 0u;
  }
}

__global__ void __launch_bounds__(256) dq_chunks_kernel(const __grid_constant__ QuantBatchParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * 8 + warp;
  if (g >= p.total_chunks) return;
  const int t = find_tensor(p, g);
  const int64_t local_chunk = g - p.chunk_begin[t];
  const int64_t nb = p.n_blocks[t];
  const int nblk = static_cast<int>(((nb - local_chunk * kDqBlock) < kDqBlock ? (nb - local_chunk * kDqBlock) : int64_t{kDqBlock}));
  const float mu = __ldcg(p.mu[t]);

  float d[8];
  float m = 0.0f;
  const float* a = p.absmax + g * kDqBlock + lane * 8;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool valid = lane * 8 + i < nblk;
    d[i] = valid ? __fsub_rn(__ldcg(a + i), mu) : 0.0f;
    m = fmaxf(m, fabsf(d[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float c2 = m;

  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int q = 0;
    if (c2 != 0.0f) q = static_cast<int>(rintf(__fmul_rn(__fdiv_rn(d[i], c2), 127.0f)));
    const uint32_t byte = static_cast<uint32_t>(q) & 0xFFu;
    if (i < 4) lo |= byte << (8 * i); else hi |= byte << (8 * (i - 4));
  }
  int8_t* qs = p.qscale[t] + local_chunk * kDqBlock + lane * 8;
  if (lane * 8 + 8 <= nblk) {
    *reinterpret_cast<uint2*>(qs) = make_uint2(lo, hi);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (lane * 8 + i < nblk) qs[i] = static_cast<int8_t>(((i < 4 ? lo >> (8 * i) : hi >> (8 * (i - 4)))) & 0xFF);
  }
  if (lane == 0) p.c2[t][local_chunk] = c2;
}

cudaError_t launch_quantize_batch(const QuantBatchParams& p, cudaStream_t stream) {
  if (p.total_chunks <= 0) return cudaSuccess;
  quantize_chunks_kernel<<<static_cast<unsigned>(p.total_chunks), 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dq_chunks_kernel<<<static_cast<unsigned>((p.total_chunks + 7) / 8), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace qnf4
