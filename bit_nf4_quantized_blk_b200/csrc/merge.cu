// Merged weight of a LoRA-adapted NF4 layer (sm_100a):
//
//   out[n][k] = Qhat(W)[n][k] + s * sum_j B[n][j] A[j][k]
//
// "FT-02: QLoRA -- Fine-Tuning with Quantization", section "4. The LoRA
// mechanics the API wraps" (the merged dense layer W0 + (alpha/r) B A
// computes the two-branch output); "QLoRA: NF4 storage, gradients and local
// integration", section "Merge changes the operator: test it explicitly"
// (merge into the dequantized Qhat(W); requantizing the merge adds
// Qhat(M) - M, which is the quantize entry point applied to the fp32 output
// of this one).
//
// The operation streams the packed codes in (0.52 bytes per weight) and the
// dense result out (2 or 4 bytes per weight): it is HBM-bound once the rank-r
// product costs less than the traffic.  That product is a dense contraction
// over j, so it runs on the tensor cores: each warp owns one 64-column
// quantization-block stripe, keeps the stripe's A operand (r x 64, bf16) in
// registers for every row tile it visits, and per 16-row tile issues
// 8 * ceil(r / 16) m16n8k16 MMAs with fp32 accumulation.  The columns are
// dealt to the MMAs so that lane t of a quad ends up with the 16 contiguous
// columns 16t .. 16t+15 of its rows: column slot 2t + e of 8-column group i
// is weight column 16t + 2i + e.  A lane therefore loads exactly the 8 code
// bytes it decodes (one 8-byte load per row) and stores its outputs straight
// from registers, 32 bytes of a row per store (a whole sector per lane, whole
// lines per warp), with no shared-memory staging.  The
// decode (NF4 level by a lane shuffle, fp32 block scale) and
// out = fma(s, BA, Qhat(W)) run in the accumulator layout.  Loads of the next
// tile (codes, scale codes, B rows) are issued before the current tile's
// arithmetic.  Pairs of B columns are loaded as one word where B allows it
// (4-byte aligned, even r).
#include "common.cuh"
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kMergeWarps = 4;  // warps per CTA: 4 adjacent 64-column stripes
constexpr int kMergeThreads = 32 * kMergeWarps;

// Inputs of one 16-row tile for one lane: rows g and g + 8 of the tile.
template <int kSteps>
struct MergeTileIn {
  uint2 code[2];           // codes of the row's columns 16t .. 16t+15 in the stripe (8 bytes)
  int q[2];                // scale codes
  float c2[2];             // second-level scales
  uint32_t bf[kSteps][4];  // MMA A operand: B rows of the tile, bf16 pairs
};

// Columns j, j + 1 of a B row as one bf16 pair (zero at j >= r).  kPair32:
// the row is 4-byte aligned and r even, so the pair is one aligned word.
template <bool kPair32>
__device__ __forceinline__ uint32_t b_pair(const uint16_t* __restrict__ brow, int j, int r) {
  if constexpr (kPair32) {
    return j < r ? __ldg(reinterpret_cast<const uint32_t*>(brow + j)) : 0u;
  } else {
    const uint32_t lo = j < r ? brow[j] : 0u;
    const uint32_t hi = j + 1 < r ? brow[j + 1] : 0u;
    return lo | (hi << 16);
  }
}

template <int kSteps, bool kPair32>
__device__ __forceinline__ void merge_load_tile(MergeTileIn<kSteps>& in, const WeightView& w,
                                                const uint16_t* __restrict__ B, int r, int64_t n0, int stripe,
                                                int g, int t) {
  const int64_t N = w.rows, K = w.cols, kb = K / kBlock;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t n = n0 + g + 8 * h;
    const bool ok = n < N;
    const int64_t nn = ok ? n : 0;
    const uint2* src = reinterpret_cast<const uint2*>(w.packed) + nn * (K / 16) + 4 * stripe + t;
    const int64_t blk = nn * kb + stripe;
    in.code[h] = ok ? __ldg(src) : make_uint2(0, 0);
    if (w.scale_format == kScalesFp32) {  // t = 1, c2 = the absmax (see scale_table_entry)
      in.q[h] = 127;
      in.c2[h] = ok ? __ldg(w.absmax + blk) : 0.0f;
    } else {
      in.q[h] = ok ? static_cast<int>(w.qscale[blk]) : 0;
      in.c2[h] = ok ? __ldg(w.c2 + (blk >> 8)) : 0.0f;  // 256 scales per chunk
    }
    const uint16_t* brow = B + nn * r;
#pragma unroll
    for (int s = 0; s < kSteps; ++s) {
      in.bf[s][h] = ok ? b_pair<kPair32>(brow, 16 * s + 2 * t, r) : 0u;
      in.bf[s][2 + h] = ok ? b_pair<kPair32>(brow, 16 * s + 2 * t + 8, r) : 0u;
    }
  }
}

// d = a b (the accumulator starts at zero).
__device__ __forceinline__ void mma_16816_zero(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "f"(0.0f));
}

}  // namespace

template <int kSteps, bool kFp32, bool kPair32>
__global__ void __launch_bounds__(kMergeThreads, kSteps == 1 ? 4 : (kSteps == 2 ? 3 : 2))
    merge_kernel(WeightView w, const uint16_t* __restrict__ A, const uint16_t* __restrict__ B, int r, float scale,
                 void* __restrict__ out, bool wide32) {
  __shared__ float s_qdiv[256];  // scale-code values t(q), q = -128 .. 127

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  for (int i = threadIdx.x; i < 256; i += kMergeThreads) s_qdiv[i] = scale_table_entry(w.scale_format, i);
  __syncthreads();
  const int64_t N = w.rows, K = w.cols;
  const int stripe = blockIdx.x * kMergeWarps + warp;
  if (stripe >= K / kBlock) return;  // whole warp; no block-wide barrier below
  const int64_t c0 = static_cast<int64_t>(stripe) * kBlock;
  const float level = codebook_level(w.codebook, lane & 15);
  const float mu = weight_mu(w);

  // MMA B operand: the stripe's A columns, fragment (k = j, n = column slot
  // g of group i), slot g holding column 16 (g / 2) + 2i + g % 2.
  uint32_t af[kSteps][8][2];
#pragma unroll
  for (int s = 0; s < kSteps; ++s)
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = 16 * s + 2 * t + 8 * h;
        const uint16_t* col = A + c0 + 16 * (g >> 1) + 2 * i + (g & 1);
        const uint32_t lo = j < r ? col[static_cast<int64_t>(j) * K] : 0u;
        const uint32_t hi = j + 1 < r ? col[static_cast<int64_t>(j + 1) * K] : 0u;
        af[s][i][h] = lo | (hi << 16);
      }

  const int64_t n_tiles = (N + 15) / 16;

  // One 16-row tile: per 8-column group i an MMA, then for rows g and g + 8
  // the lane's columns 16t + 2i, 16t + 2i + 1 (byte i of its 8 code bytes,
  // low nibble first): decode, fma, and every 16 bytes of output a store.
  auto process = [&](const MergeTileIn<kSteps>& in, int64_t n0) {
    float sc[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) sc[h] = __fadd_rn(__fmul_rn(s_qdiv[in.q[h] + 128], in.c2[h]), mu);
    constexpr int kGroupsPerStore = kFp32 ? 4 : 8;  // 32 bytes per store and row
    uint32_t o[2][8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float d[4];
      mma_16816_zero(d, in.bf[0], af[0][i]);
#pragma unroll
      for (int s = 1; s < kSteps; ++s) mma_16816(d, in.bf[s], af[s][i]);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // The shuffle reads the source lane from the low five bits; lanes
        // hold L[lane % 16], so the high bits need no mask.
        const uint32_t x = (i < 4 ? in.code[h].x : in.code[h].y) >> (8 * (i & 3));
        const float l0 = __shfl_sync(0xffffffffu, level, static_cast<int>(x));
        const float l1 = __shfl_sync(0xffffffffu, level, static_cast<int>(x >> 4));
        const float m0 = fmaf(scale, d[2 * h], __fmul_rn(l0, sc[h]));
        const float m1 = fmaf(scale, d[2 * h + 1], __fmul_rn(l1, sc[h]));
        if constexpr (kFp32) {
          o[h][2 * (i & 3)] = __float_as_uint(m0);
          o[h][2 * (i & 3) + 1] = __float_as_uint(m1);
        } else {
          o[h][i] = pack_bf16x2(m0, m1);
        }
      }
      if (i % kGroupsPerStore == kGroupsPerStore - 1) {
        // 32 bytes of the row: a full sector per lane and eight whole lines
        // per warp (two 16-byte stores when the output is only 16-byte
        // aligned).
        const int piece = i / kGroupsPerStore;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int64_t n = n0 + g + 8 * h;
          if (n < N) {
            uint8_t* dst = static_cast<uint8_t*>(out) + (n * K + c0 + 16 * t) * (kFp32 ? 4 : 2) + 32 * piece;
            if (wide32) {
              st_stream_v8(dst, o[h]);
            } else {
              *reinterpret_cast<uint4*>(dst) = make_uint4(o[h][0], o[h][1], o[h][2], o[h][3]);
              *reinterpret_cast<uint4*>(dst + 16) = make_uint4(o[h][4], o[h][5], o[h][6], o[h][7]);
            }
          }
        }
      }
    }
  };

  // 16-row tiles of this warp: blockIdx.y, +gridDim.y, ... (the CTAs of one
  // grid row cover whole rows of the weight at a time).  Two register
  // buffers alternate: the next tile's loads are in flight while the current
  // one is computed.
  MergeTileIn<kSteps> buf0, buf1;
  const int64_t step = gridDim.y;
  int64_t tile = blockIdx.y;
  if (tile < n_tiles) merge_load_tile<kSteps, kPair32>(buf0, w, B, r, tile * 16, stripe, g, t);
  while (tile < n_tiles) {
    if (tile + step < n_tiles) merge_load_tile<kSteps, kPair32>(buf1, w, B, r, (tile + step) * 16, stripe, g, t);
    process(buf0, tile * 16);
    tile += step;
    if (tile >= n_tiles) break;
    if (tile + step < n_tiles) merge_load_tile<kSteps, kPair32>(buf0, w, B, r, (tile + step) * 16, stripe, g, t);
    process(buf1, tile * 16);
    tile += step;
  }
}

namespace {

// One wave: as many CTAs as fit on the GPU at once, each walking its row
// tiles with a stride of grid rows.
template <int kSteps, bool kFp32, bool kPair32>
cudaError_t launch_merge_kernel(const WeightView& w, const uint16_t* A, const uint16_t* B, int r, float scale,
                                void* out, cudaStream_t stream) {
  // Resident CTAs on the device, queried once per device and instantiation.
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static DeviceValue resident;
  const int ctas = resident.get(dev, [dev, &e] {
    int sms = 0, per_sm = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, merge_kernel<kSteps, kFp32, kPair32>, kMergeThreads,
                                                        0);
    if (e != cudaSuccess) return -1;
    return sms * (per_sm > 0 ? per_sm : 1);
  });
  if (ctas < 0) return e;
  const int64_t gx = (w.cols / kBlock + kMergeWarps - 1) / kMergeWarps;
  const int64_t n_tiles = (w.rows + 15) / 16;
  int64_t gy = (static_cast<int64_t>(ctas) + gx - 1) / gx;
  if (gy > n_tiles) gy = n_tiles;
  if (gy > 65535) gy = 65535;
  if (gy < 1) gy = 1;
  const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  const bool wide32 = (reinterpret_cast<uintptr_t>(out) & 31) == 0;
  merge_kernel<kSteps, kFp32, kPair32><<<grid, kMergeThreads, 0, stream>>>(w, A, B, r, scale, out, wide32);
  return cudaGetLastError();
}

template <int kSteps>
cudaError_t launch_merge_steps(const WeightView& w, const uint16_t* A, const uint16_t* B, int r, float scale,
                               void* out, int out_fp32, cudaStream_t stream) {
  const bool pair32 = (reinterpret_cast<uintptr_t>(B) & 3) == 0 && r % 2 == 0;
  if (pair32)
    return out_fp32 ? launch_merge_kernel<kSteps, true, true>(w, A, B, r, scale, out, stream)
                    : launch_merge_kernel<kSteps, false, true>(w, A, B, r, scale, out, stream);
  return out_fp32 ? launch_merge_kernel<kSteps, true, false>(w, A, B, r, scale, out, stream)
                  : launch_merge_kernel<kSteps, false, false>(w, A, B, r, scale, out, stream);
}

}  // namespace

cudaError_t launch_merge(const WeightView& w, const uint16_t* A, const uint16_t* B, int r, float scale, void* out,
                         int out_fp32, cudaStream_t stream) {
  switch ((r + 15) / 16) {
    case 1: return launch_merge_steps<1>(w, A, B, r, scale, out, out_fp32, stream);
    case 2: return launch_merge_steps<2>(w, A, B, r, scale, out, out_fp32, stream);
    case 3: return launch_merge_steps<3>(w, A, B, r, scale, out, out_fp32, stream);
    default: return launch_merge_steps<4>(w, A, B, r, scale, out, out_fp32, stream);
  }
}

}  // namespace qnf4
