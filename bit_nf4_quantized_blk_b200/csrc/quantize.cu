// NF4 blockwise quantization and double quantization (sm_100a).
//
// Method: "QLoRA: NF4 storage, gradients and local integration", sections
// "NF4: nonuniform reconstruction levels", "Double quantization: correct the
// scale arithmetic" and "Exact CPU teaching quantizer and adapter gradient
// path"; "QLoRA Deep Dive: 4-bit NormalFloat & Double Quantization
// Internals", section "2. Squeezing More Memory: Double Quantization (DQ)".
//
// Three kernels per batch of tensors (the first alone for fp32 scales):
//
//  quantize_codes   persistent, one CTA per SM over the chunks of 256 blocks
//                   (16384 weights).  Each group of 8 lanes owns one 64-weight
//                   block: 256-bit streaming loads (the next chunk in flight),
//                   absmax by three xor-shuffles, IEEE fp32 division by the
//                   absmax (by 1 for an all-zero block; a reciprocal multiply
//                   with an exact-division fallback next to a threshold),
//                   nearest level from a 130-cell decision table (one 16-byte
//                   lookup per weight), eight codes packed into one 32-bit
//                   word (even element in the low nibble).
//  chunk_sums       one warp per chunk: the fp64 sum of its 256 block scales;
//                   the last warp of each tensor forms the tensor's mean offset.
//  dq_chunks        one warp per chunk: d = a - mu, c2 = max|d|,
//                   q = rint(fp32(fp32(d / c2) * 127)) (int8 codes) or the
//                   E4M3 code of fp32(d / c2) (FP8 codes); 0 where c2 == 0.
//
// Variants: fp32, bf16 or fp16 input weights (16-bit ones widen exactly to
// fp32 on load); the NF4 or FP4 codebook ("FT-02: QLoRA -- Fine-Tuning with
// Quantization", "Exercise 3: NF4 vs FP4 at equal memory").
//
// The mean is defined as a strictly sequential fp64 sum (inside each chunk,
// then over chunk sums).  When the exponents of the summed values span few
// enough binades every partial sum is exact in fp64, so a tree reduction
// gives the same bits; the kernels check that bound and fall back to a
// sequential loop when it does not hold.
#include <type_traits>

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

__device__ __forceinline__ uint4 ld_shared_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// Hardware reciprocal (at most 1 ulp from 1/x for a normal x whose
// reciprocal is normal).
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kQWarps = 16;  // 64 groups of 8 lanes
constexpr int kQThreads = kQWarps * 32;

// Per decision cell, one 16-byte entry per lane (conflict-free): the band
// [lo, hi] = 64 T (1 -+ 2^-19) around the cell's threshold T, 64 T itself and
// the cell's base position; lo = hi = thr = 256 (never reached) in a cell
// without a threshold.
constexpr int kCellEntries = kDecisionCells * 32;
constexpr int kQuantSmemBytes = kCellEntries * 16;

// 8 consecutive 16-bit weights with one 128-bit streaming load, widened to
// fp32 exactly (bf16: the bits are the top half of the fp32; fp16: IEEE
// half to single conversion).
template <int kIn>
__device__ __forceinline__ void ld_stream_16bit_v8(const uint16_t* p, float (&v)[8]) {
  uint32_t u[4];
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3])
               : "l"(p));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (kIn == QLORA_INPUT_BF16) {
      v[2 * i] = __uint_as_float(u[i] << 16);
      v[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    } else {
      v[2 * i] = __half2float(__ushort_as_half(static_cast<unsigned short>(u[i] & 0xFFFFu)));
      v[2 * i + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(u[i] >> 16)));
    }
  }
}

__device__ __forceinline__ void chunk_bounds(const QuantBatchParams& p, int64_t g, int& t, int64_t& blk0, int& nblk) {
  t = find_tensor(p, g);
  blk0 = (g - p.chunk_begin[t]) * kDqBlock;
  const int64_t rem = p.n_blocks[t] - blk0;
  nblk = static_cast<int>(rem < kDqBlock ? rem : int64_t{kDqBlock});
}

// Tensor, first block and block count of chunk g (nblk = 0 past the batch).
// A CTA visits its chunks in increasing order, so the tensor index only moves
// forward from the previous chunk's.
struct ChunkInfo {
  int t, nblk;
  int64_t blk0;
};

__device__ __forceinline__ ChunkInfo next_chunk_info(const QuantBatchParams& p, int64_t g, int& t_cursor) {
  ChunkInfo ci{t_cursor, 0, 0};
  if (g < p.total_chunks) {
    while (t_cursor + 1 < p.count && p.chunk_begin[t_cursor + 1] <= g) ++t_cursor;
    ci.t = t_cursor;
    ci.blk0 = (g - p.chunk_begin[ci.t]) * kDqBlock;
    const int64_t rem = p.n_blocks[ci.t] - ci.blk0;
    ci.nblk = static_cast<int>(rem < kDqBlock ? rem : int64_t{kDqBlock});
  }
  return ci;
}

// Weights 8l .. 8l+7 of blocks grp, grp + 64, grp + 128, grp + 192 of a
// chunk (zeros past the tensor or the batch), with 256-bit (fp32) or 128-bit
// (16-bit inputs) streaming loads.
template <int kIn>
__device__ __forceinline__ void load_chunk(const QuantBatchParams& p, const ChunkInfo& ci, int grp, int l,
                                           float (&v)[4][8]) {
  const int t = ci.t, nblk = ci.nblk;
  const int64_t blk0 = ci.blk0;
  using In = std::conditional_t<kIn == QLORA_INPUT_FP32, float, uint16_t>;
  const In* src = static_cast<const In*>(p.W[t]) + (blk0 + grp) * kBlock + l * 8;
#pragma unroll
  for (int rep = 0; rep < 4; ++rep) {
    if (rep * 64 + grp < nblk) {
      if constexpr (kIn == QLORA_INPUT_FP32)
        ld_stream_v8(src + rep * 64 * kBlock, v[rep]);
      else
        ld_stream_16bit_v8<kIn>(src + rep * 64 * kBlock, v[rep]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[rep][i] = 0.0f;
    }
  }
}

}  // namespace

// Codes and block absmax.  Persistent: one CTA per SM walks the chunks (256
// blocks = 16384 weights) of the batch.  Every lane streams its share of the
// next chunk into registers (256-bit loads) while it codes the current one.
// Each group of 8 lanes owns a block: absmax by three xor-shuffles, then per
// weight x' = w * (64 / a) with the hardware reciprocal.  x' is within
// 2^-21 |x| of the correctly rounded 64 * fp32(w / a), so it lies on the same
// side of the cell's threshold unless it falls inside the cell's band
// (2^-19 relative around the threshold); a lane with such a weight recodes
// its 8 weights from the IEEE quotient (so does a block whose 64/a is not a
// normal fp32).  Every threshold is > 2^-14 (relative) from its cell's edges
// (checked on the host), so no other threshold can be that close.
//
// kFp4: the FP4 codebook's table uses floor cells (c = floor(64 x) + 65) and
// yields positions among its 15 distinct levels; fp4_codes_of maps each
// word of positions to codes.  NF4: trunc cells (c = trunc(64 x) + 64),
// positions are the codes.  kScales32: the block absmax goes to the tensor's
// fp32 scale array (no double quantization), else to the chunk's workspace
// slots.
template <int kIn, bool kFp4, bool kScales32>
__global__ void __launch_bounds__(kQThreads, 1) quantize_codes_kernel(const __grid_constant__ QuantBatchParams p) {
  extern __shared__ uint4 s_cell[];  // [kDecisionCells cells][32 lanes]
  const int tid = threadIdx.x, lane = tid & 31;
  const int grp = tid >> 3;  // 64 groups of 8 lanes
  const int l = tid & 7;     // lane in group: weights 8l .. 8l+7 of the block

  float cur[4][8], nxt[4][8];
  int t_cursor = 0;
  ChunkInfo cur_ci = next_chunk_info(p, blockIdx.x, t_cursor);
  load_chunk<kIn>(p, cur_ci, grp, l, cur);

  for (int i = tid; i < kCellEntries; i += kQThreads) {
    const int c = i >> 5;
    const float thr = p.table.thr[c];
    float t64 = 256.0f, lo = 256.0f, hi = 256.0f;
    if (thr < 2.0f) {
      t64 = thr * 64.0f;
      const float tol = fabsf(t64) * 0x1p-19f;
      lo = t64 - tol;
      hi = t64 + tol;
    }
    s_cell[i] = make_uint4(__float_as_uint(lo), __float_as_uint(hi), __float_as_uint(t64),
                           static_cast<uint32_t>(p.table.base[c]));
  }
  __syncthreads();

  // NF4: cell 64 <-> trunc(x64) = 0; FP4: cell 65 <-> floor(x64) = 0.
  const uint32_t cell_addr0 = smem_u32(&s_cell[(kFp4 ? 65 : 64) * 32 + lane]);
  auto cell_of = [](float x64) {
    return static_cast<uint32_t>(kFp4 ? __float2int_rd(x64) : __float2int_rz(x64)) * 512u;
  };
  float nonfinite = 0.0f;  // becomes NaN if any input is NaN or +-Inf
  for (int64_t g = blockIdx.x; g < p.total_chunks; g += gridDim.x) {
    const ChunkInfo nxt_ci = next_chunk_info(p, g + gridDim.x, t_cursor);
    load_chunk<kIn>(p, nxt_ci, grp, l, nxt);
    const int t = cur_ci.t, nblk = cur_ci.nblk;
    const int64_t blk0 = cur_ci.blk0;
    uint32_t* __restrict__ packed = reinterpret_cast<uint32_t*>(p.packed[t]);
#pragma unroll
    for (int rep = 0; rep < kDqBlock / 64; ++rep) {
      const int b = rep * 64 + grp;
      float (&v)[8] = cur[rep];
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        m = fmaxf(m, fabsf(v[i]));
        nonfinite = fmaf(v[i], 0.0f, nonfinite);
      }
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
      const float div = (m == 0.0f) ? 1.0f : m;  // zero-block convention
      uint32_t word = 0;
      bool risky = false;  // some weight fell inside its cell's band
      const bool fast = div >= 0x1p-121f && div <= 0x1p119f;  // 64 / div is a normal fp32
      const float rcp64 = fast ? rcp_approx(div) * 64.0f : 0.0f;
#pragma unroll
      for (int i = 7; i >= 0; --i) {
        const float x64 = __fmul_rn(v[i], rcp64);
        const uint4 e = ld_shared_u4(cell_addr0 + cell_of(x64));
        const bool above_lo = x64 >= __uint_as_float(e.x);
        const bool above_hi = x64 > __uint_as_float(e.y);
        word = word * 16u + e.w + (above_lo ? 1u : 0u);
        risky |= above_lo != above_hi;
      }
      if (__any_sync(0xffffffffu, !fast || risky)) {
        if (!fast || risky) {
          // Recode this lane's 8 weights from the IEEE quotients.
          word = 0;
#pragma unroll
          for (int i = 7; i >= 0; --i) {
            const float x64 = __fdiv_rn(v[i], div) * 64.0f;  // exact scaling
            const uint4 e = ld_shared_u4(cell_addr0 + cell_of(x64));
            word = word * 16u + e.w + (x64 >= __uint_as_float(e.z) ? 1u : 0u);
          }
        }
      }
      if constexpr (kFp4) word = fp4_codes_of(word);
      if (b < nblk) {
        packed[(blk0 + b) * (kBlock / 8) + l] = word;
        if (l == 0) {
          if constexpr (kScales32)
            p.absmax_out[t][blk0 + b] = m;
          else
            p.absmax[g * kDqBlock + b] = m;
        }
      }
    }
#pragma unroll
    for (int rep = 0; rep < 4; ++rep)
#pragma unroll
      for (int i = 0; i < 8; ++i) cur[rep][i] = nxt[rep][i];
    cur_ci = nxt_ci;
  }
  if (!(nonfinite == 0.0f)) raise_status(p.status, QLORA_ERR_NONFINITE);
}

// fp64 sums of the block scales, one warp per chunk, then the tensor's mean
// offset by the last warp to finish a chunk of that tensor.  The definition
// is the left-to-right sum; the tree sums here are taken only when every
// partial sum is exact (see fp64_sum_is_exact), otherwise one lane loops.
__global__ void __launch_bounds__(256) chunk_sums_kernel(const __grid_constant__ QuantBatchParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (g >= p.total_chunks) return;
  int t, nblk;
  int64_t blk0;
  chunk_bounds(p, g, t, blk0, nblk);
  const float* a = p.absmax + g * kDqBlock;
  double part = 0.0;
  int emin = 1 << 20, emax = -(1 << 20);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int b = lane * 8 + i;
    const float v = b < nblk ? __ldcg(a + b) : 0.0f;
    part += static_cast<double>(v);
    if (v > 0.0f) {
      emin = min(emin, exp_field(v));
      emax = max(emax, exp_field(v));
    }
  }
  // Each lane's 8-term partial is exact whenever the whole chunk's sum is.
  part = warp_sum_f64(part);
  emin = __reduce_min_sync(0xffffffffu, emin);
  emax = __reduce_max_sync(0xffffffffu, emax);
  unsigned last = 0;
  if (lane == 0) {
    if (!fp64_sum_is_exact(emin, emax, nblk)) {
      part = 0.0;  // the definition: left to right (loads batched 8 ahead)
      for (int b0 = 0; b0 < nblk; b0 += 8) {
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = b0 + i < nblk ? __ldcg(a + b0 + i) : 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (b0 + i < nblk) part += static_cast<double>(v[i]);
      }
    }
    p.chunk_sum[g] = part;
    p.chunk_exp[2 * g] = emin;
    p.chunk_exp[2 * g + 1] = emax;
    __threadfence();
    const unsigned n_chunks = static_cast<unsigned>(p.chunk_begin[t + 1] - p.chunk_begin[t]);
    last = atomicAdd(&p.counters[t], 1u) == n_chunks - 1 ? 1u : 0u;
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __threadfence();
  const int64_t c0 = p.chunk_begin[t], c1 = p.chunk_begin[t + 1];
  const int64_t nb = p.n_blocks[t];
  double sum = 0.0;
  int tmin = 1 << 20, tmax = -(1 << 20);
  // Loads batched 8 deep per lane: the chunk sums sit in L2, and one
  // dependent round trip per chunk would dominate the kernel.
  for (int64_t cb = c0 + lane; cb < c1; cb += 32 * 8) {
    double v[8];
    int2 e[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t c = cb + 32 * i;
      v[i] = c < c1 ? __ldcg(&p.chunk_sum[c]) : 0.0;
      e[i] = c < c1 ? __ldcg(reinterpret_cast<const int2*>(p.chunk_exp) + c) : make_int2(1 << 20, -(1 << 20));
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      sum += v[i];
      tmin = min(tmin, e[i].x);
      tmax = max(tmax, e[i].y);
    }
  }
  sum = warp_sum_f64(sum);
  tmin = __reduce_min_sync(0xffffffffu, tmin);
  tmax = __reduce_max_sync(0xffffffffu, tmax);
  if (lane == 0) {
    if (!fp64_sum_is_exact(tmin, tmax, nb)) {
      sum = 0.0;  // the definition: chunk sums left to right (loads batched 8 ahead)
      for (int64_t cb = c0; cb < c1; cb += 8) {
        double v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = cb + i < c1 ? __ldcg(&p.chunk_sum[cb + i]) : 0.0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (cb + i < c1) sum += v[i];
      }
    }
    *p.mu[t] = __double2float_rn(sum / static_cast<double>(nb));
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

  uint32_t bytes[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) bytes[i] = 0;
  if (c2 != 0.0f) {
    if (p.scale_format == kScalesDqFp8) {
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        // E4M3 pair, round to nearest even (|d / c2| <= 1: no saturation);
        // the first source operand goes to the upper byte.
        uint16_t pair;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
            : "=h"(pair)
            : "f"(__fdiv_rn(d[i + 1], c2)), "f"(__fdiv_rn(d[i], c2)));
        bytes[i] = pair & 0xFFu;
        bytes[i + 1] = pair >> 8;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        bytes[i] = static_cast<uint32_t>(static_cast<int>(rintf(__fmul_rn(__fdiv_rn(d[i], c2), 127.0f)))) & 0xFFu;
    }
  }
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t byte = bytes[i];
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

namespace {

template <int kIn, bool kFp4, bool kScales32>
cudaError_t launch_codes(const QuantBatchParams& p, unsigned grid, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static DeviceOnce configured;
  e = configured.run(dev, [] {
    return cudaFuncSetAttribute(quantize_codes_kernel<kIn, kFp4, kScales32>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kQuantSmemBytes);
  });
  if (e != cudaSuccess) return e;
  quantize_codes_kernel<kIn, kFp4, kScales32><<<grid, kQThreads, kQuantSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

template <int kIn, bool kFp4>
cudaError_t launch_codes_scales(const QuantBatchParams& p, unsigned grid, cudaStream_t stream) {
  return p.scale_format == kScalesFp32 ? launch_codes<kIn, kFp4, true>(p, grid, stream)
                                       : launch_codes<kIn, kFp4, false>(p, grid, stream);
}

template <int kIn>
cudaError_t launch_codes_for(const QuantBatchParams& p, unsigned grid, cudaStream_t stream) {
  return p.codebook == QLORA_CODEBOOK_FP4 ? launch_codes_scales<kIn, true>(p, grid, stream)
                                          : launch_codes_scales<kIn, false>(p, grid, stream);
}

}  // namespace

cudaError_t launch_quantize_batch(const QuantBatchParams& p, cudaStream_t stream) {
  if (p.total_chunks <= 0) return cudaSuccess;
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  const unsigned grid = static_cast<unsigned>(p.total_chunks < sms ? p.total_chunks : sms);
  cudaError_t e = p.in_dtype == QLORA_INPUT_BF16   ? launch_codes_for<QLORA_INPUT_BF16>(p, grid, stream)
                  : p.in_dtype == QLORA_INPUT_FP16 ? launch_codes_for<QLORA_INPUT_FP16>(p, grid, stream)
                                                   : launch_codes_for<QLORA_INPUT_FP32>(p, grid, stream);
  if (e != cudaSuccess) return e;
  if (p.scale_format == kScalesFp32) return cudaSuccess;  // no double quantization
  const unsigned warps_grid = static_cast<unsigned>((p.total_chunks + 7) / 8);
  chunk_sums_kernel<<<warps_grid, 256, 0, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dq_chunks_kernel<<<warps_grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace qnf4
