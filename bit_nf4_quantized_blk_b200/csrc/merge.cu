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
// 8 * ceil(r / 16) m16n8k16 MMAs with fp32 accumulation.  The decode of the
// codes (NF4 level by a lane shuffle, fp32 block scale) and
// out = fma(s, BA, Qhat(W)) run in the accumulator layout; a per-warp shared
// tile turns the two-column fragments into 16-byte row-contiguous stores.
// Loads of the next tile (codes, scale codes, B rows) are issued before the
// current tile's arithmetic.  Pairs of B columns are loaded as one word
// where B allows it (4-byte aligned, even r).
#include "common.cuh"
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kMergeWarps = 4;  // warps per CTA: 4 adjacent 64-column stripes
constexpr int kMergeThreads = 32 * kMergeWarps;

// Inputs of one 16-row tile for one lane: rows g and g + 8 of the tile.
template <int kSteps>
struct MergeTileIn {
  uint4 code[2][2];        // the row's 64 codes (32 bytes) in the stripe
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
    const uint4* src = reinterpret_cast<const uint4*>(w.packed) + nn * (K / 32) + 2 * stripe;
    const int64_t blk = nn * kb + stripe;
    in.code[h][0] = ok ? __ldg(src) : make_uint4(0, 0, 0, 0);
    in.code[h][1] = ok ? __ldg(src + 1) : make_uint4(0, 0, 0, 0);
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
                 void* __restrict__ out) {
  // Output staging: 16 rows per warp, padded so that the fragment stores hit
  // 32 distinct banks (bf16: 36-word pitch; fp32: 72-word pitch, 8-byte stores
  // in half-warp phases).
  constexpr int kPitch = kFp32 ? 288 : 144;
  __shared__ __align__(16) uint8_t s_out[kMergeWarps][16 * kPitch];
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

  // MMA B operand: the stripe's A columns, fragment (k = j, n = column).
  uint32_t af[kSteps][8][2];
#pragma unroll
  for (int s = 0; s < kSteps; ++s)
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = 16 * s + 2 * t + 8 * h;
        const uint16_t* col = A + c0 + 8 * i + g;
        const uint32_t lo = j < r ? col[static_cast<int64_t>(j) * K] : 0u;
        const uint32_t hi = j + 1 < r ? col[static_cast<int64_t>(j + 1) * K] : 0u;
        af[s][i][h] = lo | (hi << 16);
      }

  uint8_t* stage = s_out[warp];
  const int64_t n_tiles = (N + 15) / 16;

  // One 16-row tile: MMA per 8-column group, decode, fma, stage, store.
  auto process = [&](const MergeTileIn<kSteps>& in, int64_t n0) {
    float sc[2];
    uint32_t words[2][8];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      sc[h] = __fadd_rn(__fmul_rn(s_qdiv[in.q[h] + 128], in.c2[h]), mu);
      words[h][0] = in.code[h][0].x, words[h][1] = in.code[h][0].y;
      words[h][2] = in.code[h][0].z, words[h][3] = in.code[h][0].w;
      words[h][4] = in.code[h][1].x, words[h][5] = in.code[h][1].y;
      words[h][6] = in.code[h][1].z, words[h][7] = in.code[h][1].w;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float d[4];
      mma_16816_zero(d, in.bf[0], af[0][i]);
#pragma unroll
      for (int s = 1; s < kSteps; ++s) mma_16816(d, in.bf[s], af[s][i]);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // Columns 8i + 2t and 8i + 2t + 1 are byte t of word i (low nibble
        // first).  The shuffle reads the source lane from the low five bits;
        // lanes hold L[lane % 16], so the high bits need no mask.
        const uint32_t x = words[h][i] >> (8 * t);
        const float l0 = __shfl_sync(0xffffffffu, level, static_cast<int>(x));
        const float l1 = __shfl_sync(0xffffffffu, level, static_cast<int>(x >> 4));
        const float m0 = fmaf(scale, d[2 * h], __fmul_rn(l0, sc[h]));
        const float m1 = fmaf(scale, d[2 * h + 1], __fmul_rn(l1, sc[h]));
        const int row = g + 8 * h;
        if constexpr (kFp32) {
          *reinterpret_cast<float2*>(stage + row * kPitch + 32 * i + 8 * t) = make_float2(m0, m1);
        } else {
          *reinterpret_cast<uint32_t*>(stage + row * kPitch + 16 * i + 4 * t) = pack_bf16x2(m0, m1);
        }
      }
    }
    __syncwarp();
    constexpr int kChunksPerRow = kFp32 ? 16 : 8;  // 16-byte pieces of a 64-column row
#pragma unroll
    for (int k = 0; k < kChunksPerRow / 2; ++k) {
      const int q = lane + 32 * k;
      const int row = q / kChunksPerRow, ch = q % kChunksPerRow;
      const uint4 v = *reinterpret_cast<const uint4*>(stage + row * kPitch + 16 * ch);
      const int64_t n = n0 + row;
      if (n < N) {
        if constexpr (kFp32)
          *reinterpret_cast<uint4*>(static_cast<float*>(out) + n * K + c0 + 4 * ch) = v;
        else
          *reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + n * K + c0 + 8 * ch) = v;
      }
    }
    __syncwarp();
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
  merge_kernel<kSteps, kFp32, kPair32><<<grid, kMergeThreads, 0, stream>>>(w, A, B, r, scale, out);
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
