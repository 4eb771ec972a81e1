// C ABI of the QLoRA NF4 library: argument checks, workspace layout and the
// launch sequences of quantize / dequantize / linear forward / backward.
//
// The host never computes any part of the method's results: it checks
// arguments, carves the caller's workspace and enqueues kernels.  The one
// table it builds, the decision cells of the nearest-level search, is derived
// here from the codebook of "QLoRA: NF4 storage, gradients and local
// integration" (section "Exact CPU teaching quantizer and adapter gradient
// path") with the same fp32 rule the definition uses.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"
#include "kernels.cuh"

using namespace qnf4;

namespace {

// ---------------------------------------------------------------------------
// Decision table
// ---------------------------------------------------------------------------

// Nearest level of x by the definition: fp32 distances |x - L_j|, the lowest
// code wins a tie.  Host fp32 arithmetic (SSE, no contraction) is IEEE.
int host_nearest_code(int codebook, float x) {
  int best = 0;
  volatile float bd = std::fabs(x - codebook_level(codebook, 0));
  for (int j = 1; j < 16; ++j) {
    volatile float d = std::fabs(x - codebook_level(codebook, j));
    if (d < bd) {
      bd = d;
      best = j;
    }
  }
  return best;
}

int64_t ordered_key(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return (u >> 31) ? -static_cast<int64_t>(u & 0x7FFFFFFFu) : static_cast<int64_t>(u);
}

float from_key(int64_t k) {
  const uint32_t u = k >= 0 ? static_cast<uint32_t>(k) : (0x80000000u | static_cast<uint32_t>(-k));
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// The codebook's distinct levels in increasing order, each with the code the
// tie rule picks for it (NF4: 16 levels, positions = codes; FP4: 15, +0 and
// -0 being one value whose code is 0).
struct SortedLevels {
  int n = 0;
  float level[16];
  int code[16];
  int pos_of_code[16];
};

SortedLevels sorted_levels(int codebook) {
  SortedLevels s;
  int order[16];
  for (int j = 0; j < 16; ++j) order[j] = j;
  std::sort(order, order + 16, [&](int a, int b) {
    const float la = codebook_level(codebook, a), lb = codebook_level(codebook, b);
    return la < lb || (la == lb && a < b);
  });
  for (int i = 0; i < 16; ++i) {
    const int c = order[i];
    const float l = codebook_level(codebook, c);
    if (s.n > 0 && s.level[s.n - 1] == l) {  // equal value: the lower code (first in order) stays
      s.pos_of_code[c] = s.n - 1;
      continue;
    }
    s.level[s.n] = l;
    s.code[s.n] = c;
    s.pos_of_code[c] = s.n;
    ++s.n;
  }
  return s;
}

int host_position(int codebook, const SortedLevels& s, float x) {
  return s.pos_of_code[host_nearest_code(codebook, x)];
}

// The n - 1 decision thresholds: T_j is the smallest fp32 x whose nearest
// level has position >= j (the choice between neighbouring levels flips once
// between them).
void derive_thresholds(int codebook, const SortedLevels& s, float (&T)[16]) {
  T[0] = -INFINITY;
  for (int j = 1; j < s.n; ++j) {
    int64_t lo = ordered_key(s.level[j - 1]), hi = ordered_key(s.level[j]);
    while (hi - lo > 1) {
      const int64_t mid = lo + (hi - lo) / 2;
      if (host_position(codebook, s, from_key(mid)) >= j) hi = mid; else lo = mid;
    }
    T[j] = from_key(hi);
  }
}

// Cells of x in [-1, 1]; each is an interval of fp32 values [xlo, xhi] that
// holds at most one threshold, so pos(x) = base[c] + (x >= thr[c]).
//   NF4 (trunc cells): c = trunc(64 x) + 64, c = 0 .. 128 (cell 64 is
//   (-1/64, 1/64)).  FP4 (floor cells): c = floor(64 x) + 65, c = 1 .. 128
//   cover [k/64, (k+1)/64), k = c - 65; cells 0 and 129 take the products a
//   rounding below -64 or at 64 (x = -1, x = 1).  Verified against the
//   definition at every cell edge and around every threshold.
bool build_decision_table(int codebook, Nf4DecisionTable* tab) {
  const SortedLevels s = sorted_levels(codebook);
  float T[16];
  derive_thresholds(codebook, s, T);
  const bool floor_cells = codebook == QLORA_CODEBOOK_FP4;
  int cells_with_threshold = 0;
  for (int c = 0; c < kDecisionCells; ++c) {
    float xlo, xhi;
    if (floor_cells) {
      const int k = c - 65;
      if (k < -64) {
        xlo = xhi = -1.0f;
      } else if (k >= 64) {
        xlo = xhi = 1.0f;
      } else {
        xlo = static_cast<float>(k) / 64.0f;
        xhi = std::nextafter(static_cast<float>(k + 1) / 64.0f, -INFINITY);
      }
    } else {
      const int t = c - 64;
      if (t > 64) {  // not addressed by trunc cells
        xlo = xhi = 1.0f;
      } else if (t >= 1) {
        xlo = static_cast<float>(t) / 64.0f;
        xhi = t == 64 ? 1.0f : std::nextafter(static_cast<float>(t + 1) / 64.0f, -INFINITY);
      } else if (t == 0) {
        xlo = std::nextafter(-1.0f / 64.0f, INFINITY);
        xhi = std::nextafter(1.0f / 64.0f, -INFINITY);
      } else {
        xlo = t == -64 ? -1.0f : std::nextafter(static_cast<float>(t - 1) / 64.0f, INFINITY);
        xhi = static_cast<float>(t) / 64.0f;
      }
    }
    int base = 0, inside = 0;
    float thr = 4.0f;  // no threshold in this cell: a value no x in [-1, 1] reaches
    for (int j = 1; j < s.n; ++j) {
      if (T[j] <= xlo) ++base;
      else if (T[j] <= xhi) {
        thr = T[j];
        ++inside;
      }
    }
    if (inside > 1) return false;
    // The quantize kernel's reciprocal fast path needs every threshold well
    // inside its cell (relative gap > 2^-14 to both cell edges).
    if (inside && (thr - xlo < std::fabs(thr) * 0x1p-14f || xhi - thr < std::fabs(thr) * 0x1p-14f)) return false;
    tab->thr[c] = thr;
    tab->base[c] = base;
    auto pos_of = [&](float x) { return base + (x >= thr ? 1 : 0); };
    if (pos_of(xlo) != host_position(codebook, s, xlo) || pos_of(xhi) != host_position(codebook, s, xhi)) return false;
    if (inside) {
      if (pos_of(thr) != host_position(codebook, s, thr)) return false;
      const float below = std::nextafter(thr, -INFINITY);
      if (pos_of(below) != host_position(codebook, s, below)) return false;
      if (thr != T[base + 1]) return false;  // the cell's threshold is the next one above its base
      ++cells_with_threshold;
    }
  }
  // every threshold sits inside exactly one cell
  if (cells_with_threshold != s.n - 1) return false;
  // the kernel's position -> code mapping (identity for NF4)
  for (int i = 0; i < s.n; ++i)
    if ((floor_cells ? fp4_code_of_position(i) : i) != s.code[i]) return false;
  return true;
}

const Nf4DecisionTable* decision_table(int codebook) {
  static Nf4DecisionTable tab[2];
  static bool ok[2] = {false, false};
  static std::once_flag once[2];
  if (codebook != QLORA_CODEBOOK_NF4 && codebook != QLORA_CODEBOOK_FP4) return nullptr;
  std::call_once(once[codebook], [codebook] { ok[codebook] = build_decision_table(codebook, &tab[codebook]); });
  return ok[codebook] ? &tab[codebook] : nullptr;
}

// ---------------------------------------------------------------------------
// Kernel timing (instrumentation): CUDA events around each launch family.
// ---------------------------------------------------------------------------

enum Family { kFamQuant, kFamDequant, kFamGemv, kFamSide, kFamGemm, kFamMerge, kFamCount };
const char* const kFamNames[kFamCount] = {"quantize", "dequant", "gemv", "side", "gemm", "merge"};

// Shared by every host thread: `mu` guards the event pool and the records.
struct TimingState {
  std::mutex mu;
  std::atomic<bool> enabled{false};
  std::vector<cudaEvent_t> pool;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pending[kFamCount];
  double ms[kFamCount] = {};
  int64_t launches[kFamCount] = {};
};

TimingState& timing() {
  static TimingState t;
  return t;
}

// An event from the pool, or a new one (nullptr if none can be created).
// The caller holds T.mu.
cudaEvent_t take_event_locked(TimingState& T) {
  if (!T.pool.empty()) {
    cudaEvent_t e = T.pool.back();
    T.pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Brackets the kernels enqueued during its lifetime with two events.  An
// event that cannot be taken or recorded drops the record, never the launch.
class Timed {
 public:
  Timed(Family fam, cudaStream_t s, int kernels = 1) : fam_(fam), s_(s), kernels_(kernels) {
    TimingState& T = timing();
    if (!T.enabled.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lock(T.mu);
    start_ = take_event_locked(T);
    if (start_ != nullptr && cudaEventRecord(start_, s_) != cudaSuccess) {
      T.pool.push_back(start_);
      start_ = nullptr;
    }
  }
  ~Timed() {
    if (start_ == nullptr) return;
    TimingState& T = timing();
    std::lock_guard<std::mutex> lock(T.mu);
    cudaEvent_t stop = take_event_locked(T);
    if (stop == nullptr || cudaEventRecord(stop, s_) != cudaSuccess) {
      T.pool.push_back(start_);
      if (stop != nullptr) T.pool.push_back(stop);
      return;
    }
    T.pending[fam_].push_back({start_, stop});
    T.launches[fam_] += kernels_;
  }
  Timed(const Timed&) = delete;
  Timed& operator=(const Timed&) = delete;

 private:
  Family fam_;
  cudaStream_t s_;
  int kernels_;
  cudaEvent_t start_ = nullptr;
};

// ---------------------------------------------------------------------------
// Helpers
// ---------------------------------------------------------------------------

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

qlora_status from_cuda(cudaError_t e) { return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

qlora_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return QLORA_ERR_CUDA;
  return (major == 10 && minor == 0) ? QLORA_OK : QLORA_ERR_UNSUPPORTED;
}

qlora_status check_weight(const qlora_nf4_weight* w) {
  if (w == nullptr) return QLORA_ERR_INVALID_ARG;
  if (w->rows < 1 || w->cols < kBlock || w->cols % kBlock != 0) return QLORA_ERR_INVALID_ARG;
  if (w->rows > (int64_t{1} << 40) / w->cols) return QLORA_ERR_UNSUPPORTED;
  if (w->codebook != QLORA_CODEBOOK_NF4 && w->codebook != QLORA_CODEBOOK_FP4) return QLORA_ERR_INVALID_ARG;
  if (w->scale_format != kScalesDqInt8 && w->scale_format != kScalesDqFp8 && w->scale_format != kScalesFp32)
    return QLORA_ERR_INVALID_ARG;
  if (!w->packed) return QLORA_ERR_INVALID_ARG;
  if (!aligned(w->packed, 16)) return QLORA_ERR_ALIGNMENT;
  if (w->scale_format == kScalesFp32) {
    if (!w->absmax) return QLORA_ERR_INVALID_ARG;
    if (!aligned(w->absmax, 16)) return QLORA_ERR_ALIGNMENT;
    return QLORA_OK;
  }
  if (!w->qscale || !w->c2 || !w->mu) return QLORA_ERR_INVALID_ARG;
  if (!aligned(w->qscale, 16) || !aligned(w->c2, 4) || !aligned(w->mu, 4)) return QLORA_ERR_ALIGNMENT;
  return QLORA_OK;
}

// Input weights: fp32 needs 32-byte alignment (256-bit loads), bf16 / fp16 16.
qlora_status check_input(const void* W, int32_t in_dtype) {
  if (W == nullptr) return QLORA_ERR_INVALID_ARG;
  if (in_dtype != QLORA_INPUT_FP32 && in_dtype != QLORA_INPUT_BF16 && in_dtype != QLORA_INPUT_FP16)
    return QLORA_ERR_INVALID_ARG;
  return aligned(W, in_dtype == QLORA_INPUT_FP32 ? 32 : 16) ? QLORA_OK : QLORA_ERR_ALIGNMENT;
}

int64_t n_chunks_of(int64_t rows, int64_t cols) {
  const int64_t nb = rows * cols / kBlock;
  return (nb + kDqBlock - 1) / kDqBlock;
}

// Quantize workspace: [status 256 B][counters][absmax][chunk sums][chunk exponents]
struct QuantWs {
  size_t counters, absmax, sums, exps, total;
};

constexpr QuantWs quant_ws_layout(int count, int64_t chunks) {
  QuantWs l{};
  size_t off = kWsHeader;
  l.counters = off;
  off = align_up(off + sizeof(unsigned) * kMaxQuantBatch, 256);
  l.absmax = off;
  off = align_up(off + sizeof(float) * kDqBlock * static_cast<size_t>(chunks), 256);
  l.sums = off;
  off = align_up(off + sizeof(double) * static_cast<size_t>(chunks), 256);
  l.exps = off;
  off = align_up(off + 2 * sizeof(int) * static_cast<size_t>(chunks), 256);
  l.total = off;
  (void)count;
  return l;
}

// Largest number of chunks any launch group of a batch holds.
int64_t max_group_chunks(const qlora_nf4_weight* outs, int32_t count) {
  int64_t best = 0;
  for (int32_t g0 = 0; g0 < count; g0 += kMaxQuantBatch) {
    int64_t c = 0;
    for (int32_t i = g0; i < count && i < g0 + kMaxQuantBatch; ++i) c += n_chunks_of(outs[i].rows, outs[i].cols);
    if (c > best) best = c;
  }
  return best;
}

// Linear workspace layout.
struct LinearWs {
  size_t wbf, scales, us, uhi, ulo, vs, vhi, vlo, bpad, part, skpart, vdbpart, bt, uht, ult, gu, gy, total;
};

LinearWs linear_ws_layout(int64_t M, int64_t N, int64_t K, bool dense) {
  LinearWs l;
  size_t off = kWsHeader;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  const size_t mr = static_cast<size_t>(M) * kRankPad;
  // The dense bf16 copy of the weight exists only on the dense-weight path
  // (the backward's GEMM runs at every M).
  l.wbf = take(dense ? static_cast<size_t>(N) * static_cast<size_t>(K) * 2 : 0);
  // Decoded block scales for the fused GEMM's tile producer (1/16 B per weight).
  l.scales = take(dense ? 0 : static_cast<size_t>(N) * static_cast<size_t>(block_scales_ld(K)) * sizeof(float));
  l.us = take(mr * 2);
  l.uhi = take(mr * 2);
  l.ulo = take(mr * 2);
  l.vs = take(mr * 2);
  l.vhi = take(mr * 2);
  l.vlo = take(mr * 2);
  l.bpad = take(static_cast<size_t>(N) * kRankPad * 2);
  const size_t p1 = colsum_partial_bytes(M, N), p2 = colsum_partial_bytes(M, K);
  l.part = take(p1 > p2 ? p1 : p2);
  const size_t s1 = skinny_partial_bytes(M, N), s2 = skinny_partial_bytes(M, K);
  l.skpart = take(s1 > s2 ? s1 : s2);
  // The tensor-core V / dB pass: its partials and the transposed B and U split.
  const bool vdb = M > kGemvMaxM;
  l.vdbpart = take(vdb ? vdb_tc_partial_bytes(M, N) : 0);
  l.bt = take(vdb ? static_cast<size_t>(16) * static_cast<size_t>(N) * 2 : 0);
  l.uht = take(vdb ? static_cast<size_t>(16) * static_cast<size_t>(vdb_tc_ldm(M)) * 2 : 0);
  l.ult = take(vdb ? static_cast<size_t>(16) * static_cast<size_t>(vdb_tc_ldm(M)) * 2 : 0);
  // Decode path (M <= 16): U partials and, for K > 4096, per-chunk fp32 outputs.
  const bool decode = M <= kGemvMaxM;
  l.gu = take(decode ? static_cast<size_t>(gemv_upart_count(K)) * kGemvMaxM * kRankPad * 4 : 0);
  l.gy = take(decode && gemv_chunks(K) > 1
                  ? static_cast<size_t>(gemv_chunks(K)) * kGemvMaxM * static_cast<size_t>(N) * 4
                  : 0);
  l.total = off;
  return l;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// Tensor i of a dequant batch.
void set_dequant_tensor(DequantBatchParams& p, int i, const qlora_nf4_weight& w, void* out) {
  p.n_units[i] = w.rows * w.cols / 32;
  p.packed[i] = w.packed;
  p.qscale[i] = w.qscale;
  p.c2[i] = w.c2;
  p.mu[i] = w.mu;
  p.absmax[i] = w.absmax;
  p.codebook[i] = w.codebook;
  p.scale_format[i] = w.scale_format;
  p.out[i] = out;
}

// A one-tensor dequant batch (the dense bf16 weight of the linear paths).
void dequant_one(DequantBatchParams& p, const qlora_nf4_weight* w, void* out) {
  std::memset(&p, 0, sizeof(p));
  p.count = 1;
  set_dequant_tensor(p, 0, *w, out);
  p.begin_seg[1] = p.total_seg = (p.n_units[0] + 127) / 128;
}

WeightView view_of(const qlora_nf4_weight* w) {
  return WeightView{w->packed, w->qscale, w->c2, w->mu, w->rows, w->cols, w->codebook, w->scale_format, w->absmax};
}

// Shapes the linear paths take: M >= 1 tokens, N (rows) a multiple of 8, K
// (cols) a multiple of 64, rank 1..64; and sizes within the kernels' 32-bit
// indices and TMA coordinates: M * 64 < 2^31, N and K < 2^31, N * K <= 2^40.
qlora_status check_linear_shape(int64_t M, int64_t N, int64_t K, int32_t r) {
  if (M < 1 || N < 1 || N % 8 != 0 || K < kBlock || K % kBlock != 0 || r < 1 || r > kMaxRank)
    return QLORA_ERR_INVALID_ARG;
  if (M > (int64_t{1} << 31) / kRankPad || N > INT32_MAX || K > INT32_MAX || N > (int64_t{1} << 40) / K)
    return QLORA_ERR_UNSUPPORTED;
  return QLORA_OK;
}

// Weight path of the tensor-core linear calls (process-wide, read once per call).
std::atomic<int> g_weight_path{QLORA_WEIGHT_PATH_FUSED};

bool dense_weight_path() { return g_weight_path.load(std::memory_order_relaxed) == QLORA_WEIGHT_PATH_DENSE; }

qlora_status check_linear_args(const qlora_nf4_weight* w, int64_t M, int32_t r, size_t ws_bytes, const void* ws,
                               bool dense) {
  qlora_status st = check_weight(w);
  if (st != QLORA_OK) return st;
  st = check_linear_shape(M, w->rows, w->cols, r);
  if (st != QLORA_OK) return st;
  if (ws == nullptr || !aligned(ws, 256)) return ws == nullptr ? QLORA_ERR_WORKSPACE : QLORA_ERR_ALIGNMENT;
  if (ws_bytes < linear_ws_layout(M, w->rows, w->cols, dense).total) return QLORA_ERR_WORKSPACE;
  return QLORA_OK;
}

// The 4-bit weight decoded inside the tensor-core GEMM.
// The 4-bit weight decoded inside the tensor-core GEMM; its decoded block
// scales (`scales`, workspace) are written first by a small pre-pass.
// `scales_written`: the caller's preceding reduction kernel already wrote the
// block scales (a BlockScalesJob on its spare threads); otherwise a pre-pass
// launch writes them here.
cudaError_t launch_linear_gemm_nf4(const qlora_nf4_weight* w, float* scales, const uint16_t* A, int64_t M,
                                   const uint16_t* A2, const uint16_t* B2, int r, int64_t ldb2, uint16_t* D,
                                   int accumulate, int* status, bool backward, cudaStream_t s, bool scales_written,
                                   uint64_t wait_limit_ns = 0, int debug_stall = 0) {
  if (!scales_written) {
    const cudaError_t e = launch_block_scales(view_of(w), scales, s);
    if (e != cudaSuccess) return e;
  }
  Nf4GemmArgs g{};
  g.w = view_of(w);
  g.scales = scales;
  g.A = A;
  g.A2 = A2;
  g.B2 = B2;
  g.M = M;
  g.r = r;
  g.ldb2 = ldb2;
  g.D = D;
  g.accumulate = accumulate;
  g.status = status;
  g.backward = backward ? 1 : 0;
  g.wait_limit_ns = wait_limit_ns;
  g.debug_stall = debug_stall;
  return launch_gemm_nf4(g, s);
}

qlora_status gemm_status(cudaError_t e) { return e == cudaErrorNotSupported ? QLORA_ERR_UNSUPPORTED : from_cuda(e); }

}  // namespace

// ===========================================================================
// Exported entry points
// ===========================================================================

extern "C" const char* qlora_status_string(qlora_status status) {
  switch (status) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument";
    case QLORA_ERR_ALIGNMENT: return "misaligned pointer";
    case QLORA_ERR_NONFINITE: return "non-finite value in the weight";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_TIMEOUT: return "device-side wait timed out";
    case QLORA_ERR_UNSUPPORTED: return "unsupported device or size";
    case QLORA_ERR_CHECK: return "a debug-build index or alignment check failed";
  }
  return "unknown status";
}

extern "C" qlora_status qlora_nf4_sizes(int64_t rows, int64_t cols, size_t* packed_bytes, size_t* n_blocks,
                                        size_t* n_chunks, size_t* ws_bytes) {
  if (rows < 1 || cols < kBlock || cols % kBlock != 0) return QLORA_ERR_INVALID_ARG;
  if (rows > (int64_t{1} << 40) / cols) return QLORA_ERR_UNSUPPORTED;
  const int64_t n = rows * cols;
  if (packed_bytes) *packed_bytes = static_cast<size_t>(n / 2);
  if (n_blocks) *n_blocks = static_cast<size_t>(n / kBlock);
  if (n_chunks) *n_chunks = static_cast<size_t>(n_chunks_of(rows, cols));
  if (ws_bytes) *ws_bytes = quant_ws_layout(1, n_chunks_of(rows, cols)).total;
  return QLORA_OK;
}

extern "C" size_t qlora_nf4_quantize_batched_ws_bytes(const qlora_nf4_weight* outs, int32_t count) {
  if (outs == nullptr || count < 1) return 0;
  for (int32_t i = 0; i < count; ++i)
    if (outs[i].rows < 1 || outs[i].cols < kBlock || outs[i].cols % kBlock != 0) return 0;
  return quant_ws_layout(count, max_group_chunks(outs, count)).total;
}

extern "C" qlora_status qlora_nf4_quantize_batched_ex(const void* const* W, int32_t in_dtype,
                                                      const qlora_nf4_weight* outs, int32_t count, void* ws,
                                                      size_t ws_bytes, int32_t* d_status, void* stream) {
  if (W == nullptr || outs == nullptr || count < 1) return QLORA_ERR_INVALID_ARG;
  for (int32_t i = 0; i < count; ++i) {
    qlora_status st = check_weight(&outs[i]);
    if (st != QLORA_OK) return st;
    if (outs[i].codebook != outs[0].codebook || outs[i].scale_format != outs[0].scale_format)
      return QLORA_ERR_INVALID_ARG;  // one format per call
    st = check_input(W[i], in_dtype);
    if (st != QLORA_OK) return st;
  }
  if (ws == nullptr) return QLORA_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return QLORA_ERR_ALIGNMENT;
  const QuantWs lay = quant_ws_layout(count, max_group_chunks(outs, count));
  if (ws_bytes < lay.total) return QLORA_ERR_WORKSPACE;
  if (d_status != nullptr && !aligned(d_status, 4)) return QLORA_ERR_ALIGNMENT;
  qlora_status st = check_device();
  if (st != QLORA_OK) return st;
  const Nf4DecisionTable* tab = decision_table(outs[0].codebook);
  if (tab == nullptr) return QLORA_ERR_UNSUPPORTED;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = d_status != nullptr ? d_status : at<int>(ws, 0);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), s);
  if (e != cudaSuccess) return from_cuda(e);

  QuantBatchParams p;
  for (int32_t g0 = 0; g0 < count; g0 += kMaxQuantBatch) {
    std::memset(&p, 0, sizeof(p));
    const int n = (count - g0 < kMaxQuantBatch) ? count - g0 : kMaxQuantBatch;
    p.count = n;
    int64_t c = 0;
    for (int i = 0; i < n; ++i) {
      const qlora_nf4_weight& o = outs[g0 + i];
      p.chunk_begin[i] = c;
      p.n_blocks[i] = o.rows * o.cols / kBlock;
      p.W[i] = W[g0 + i];
      p.packed[i] = o.packed;
      p.qscale[i] = o.qscale;
      p.c2[i] = o.c2;
      p.mu[i] = o.mu;
      c += n_chunks_of(o.rows, o.cols);
    }
    p.chunk_begin[n] = c;
    p.total_chunks = c;
    p.in_dtype = in_dtype;
    p.codebook = outs[0].codebook;
    p.scale_format = outs[0].scale_format;
    p.absmax = at<float>(ws, lay.absmax);
    for (int i = 0; i < n; ++i) p.absmax_out[i] = outs[g0 + i].absmax;
    p.chunk_sum = at<double>(ws, lay.sums);
    p.chunk_exp = at<int>(ws, lay.exps);
    p.counters = at<unsigned>(ws, lay.counters);
    p.status = status;
    p.table = *tab;
    e = cudaMemsetAsync(p.counters, 0, sizeof(unsigned) * kMaxQuantBatch, s);
    if (e != cudaSuccess) return from_cuda(e);
    {
      // The codes kernel, then (double-quantized formats) the chunk sums and the DQ codes.
      Timed tm(kFamQuant, s, p.scale_format == kScalesFp32 ? 1 : 3);
      e = launch_quantize_batch(p, s);
    }
    if (e != cudaSuccess) return from_cuda(e);
  }
  if (d_status != nullptr) return QLORA_OK;
  int32_t h = 0;
  e = cudaMemcpyAsync(&h, status, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return from_cuda(e);
  return static_cast<qlora_status>(h);
}

extern "C" qlora_status qlora_nf4_quantize_batched(const float* const* W, const qlora_nf4_weight* outs, int32_t count,
                                                   void* ws, size_t ws_bytes, int32_t* d_status, void* stream) {
  return qlora_nf4_quantize_batched_ex(reinterpret_cast<const void* const*>(W), QLORA_INPUT_FP32, outs, count, ws,
                                       ws_bytes, d_status, stream);
}

extern "C" qlora_status qlora_nf4_quantize_ex(const void* W, int32_t in_dtype, const qlora_nf4_weight* out, void* ws,
                                              size_t ws_bytes, int32_t* d_status, void* stream) {
  if (out == nullptr) return QLORA_ERR_INVALID_ARG;
  const void* const ws_list[1] = {W};
  return qlora_nf4_quantize_batched_ex(ws_list, in_dtype, out, 1, ws, ws_bytes, d_status, stream);
}

extern "C" qlora_status qlora_nf4_quantize(const float* W, const qlora_nf4_weight* out, void* ws, size_t ws_bytes,
                                           int32_t* d_status, void* stream) {
  return qlora_nf4_quantize_ex(W, QLORA_INPUT_FP32, out, ws, ws_bytes, d_status, stream);
}

extern "C" qlora_status qlora_nf4_dequantize_batched(const qlora_nf4_weight* weights, void* const* outs, int32_t count,
                                                     int32_t out_dtype, void* stream) {
  if (weights == nullptr || outs == nullptr || count < 1) return QLORA_ERR_INVALID_ARG;
  if (out_dtype != 0 && out_dtype != 1) return QLORA_ERR_INVALID_ARG;
  for (int32_t i = 0; i < count; ++i) {
    const qlora_status st = check_weight(&weights[i]);
    if (st != QLORA_OK) return st;
    if (outs[i] == nullptr) return QLORA_ERR_INVALID_ARG;
    if (!aligned(outs[i], 32)) return QLORA_ERR_ALIGNMENT;  // 256-bit stores
  }
  qlora_status st = check_device();
  if (st != QLORA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DequantBatchParams p;
  for (int32_t g0 = 0; g0 < count; g0 += kMaxDequantBatch) {
    std::memset(&p, 0, sizeof(p));
    const int n = (count - g0 < kMaxDequantBatch) ? count - g0 : kMaxDequantBatch;
    p.count = n;
    int64_t c = 0;
    for (int i = 0; i < n; ++i) {
      const qlora_nf4_weight& w = weights[g0 + i];
      p.begin_seg[i] = c;
      set_dequant_tensor(p, i, w, outs[g0 + i]);
      c += (p.n_units[i] + 127) / 128;
    }
    p.begin_seg[n] = c;
    p.total_seg = c;
    cudaError_t e;
    {
      Timed tm(kFamDequant, s);
      e = launch_dequant_batch(p, out_dtype, s);
    }
    if (e != cudaSuccess) return from_cuda(e);
  }
  return QLORA_OK;
}

extern "C" qlora_status qlora_nf4_dequantize(const qlora_nf4_weight* w, void* out, int32_t out_dtype,
                                             int32_t transpose, void* stream) {
  if (transpose != 0 && transpose != 1) return QLORA_ERR_INVALID_ARG;
  if (!transpose) {
    void* const outs[1] = {out};
    return qlora_nf4_dequantize_batched(w, outs, 1, out_dtype, stream);
  }
  qlora_status st = check_weight(w);
  if (st != QLORA_OK) return st;
  if (out == nullptr || out_dtype != 0) return QLORA_ERR_INVALID_ARG;
  if (w->rows % 8 != 0) return QLORA_ERR_INVALID_ARG;
  if (!aligned(out, 16)) return QLORA_ERR_ALIGNMENT;
  st = check_device();
  if (st != QLORA_OK) return st;
  Timed tm(kFamDequant, static_cast<cudaStream_t>(stream));
  return from_cuda(launch_dequant_transposed(view_of(w), static_cast<uint16_t*>(out), static_cast<cudaStream_t>(stream)));
}

extern "C" qlora_status qlora_merge(const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B, int32_t r,
                                    float scale, void* out, int32_t out_dtype, void* stream) {
  qlora_status st = check_weight(w);
  if (st != QLORA_OK) return st;
  if (A == nullptr || B == nullptr || out == nullptr) return QLORA_ERR_INVALID_ARG;
  if (r < 1 || r > kMaxRank || (out_dtype != 0 && out_dtype != 1) || !std::isfinite(scale))
    return QLORA_ERR_INVALID_ARG;
  if (!aligned(A, 2) || !aligned(B, 2) || !aligned(out, 16)) return QLORA_ERR_ALIGNMENT;
  st = check_device();
  if (st != QLORA_OK) return st;
  Timed tm(kFamMerge, static_cast<cudaStream_t>(stream));
  return from_cuda(launch_merge(view_of(w), A, B, r, scale, out, out_dtype, static_cast<cudaStream_t>(stream)));
}

extern "C" size_t qlora_linear_ws_bytes(int64_t M, int64_t N, int64_t K, int32_t r) {
  if (check_linear_shape(M, N, K, r) != QLORA_OK) return 0;
  return linear_ws_layout(M, N, K, dense_weight_path()).total;
}

extern "C" qlora_status qlora_linear_set_weight_path(int32_t path) {
  if (path != QLORA_WEIGHT_PATH_FUSED && path != QLORA_WEIGHT_PATH_DENSE) return QLORA_ERR_INVALID_ARG;
  g_weight_path.store(path, std::memory_order_relaxed);
  return QLORA_OK;
}

extern "C" int32_t qlora_linear_weight_path(void) { return g_weight_path.load(std::memory_order_relaxed); }

extern "C" qlora_status qlora_workspace_reset(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes < kWsHeader) return QLORA_ERR_WORKSPACE;
  return from_cuda(cudaMemsetAsync(ws, 0, kWsHeader, static_cast<cudaStream_t>(stream)));
}

extern "C" qlora_status qlora_workspace_status(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes < kWsHeader) return QLORA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(int32_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return from_cuda(e);
  return static_cast<qlora_status>(h);
}

namespace {

// Diagnostic settings of the fused GEMM (all zero in product calls).
struct GemmDiagnostics {
  uint64_t wait_limit_ns;
  int debug_stall;
};

qlora_status linear_fwd(const qlora_nf4_weight* w, const uint16_t* X, int64_t M, const uint16_t* A, const uint16_t* B,
                        int32_t r, float scale, uint16_t* Y, float* U_out, void* ws, size_t ws_bytes, void* stream,
                        const GemmDiagnostics& diag) {
  const bool dense = dense_weight_path() && !diag.debug_stall;
  qlora_status st = check_linear_args(w, M, r, ws_bytes, ws, dense);
  if (st != QLORA_OK) return st;
  if (!X || !A || !B || !Y) return QLORA_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(A, 16) || !aligned(B, 2) || !aligned(Y, 16) || (U_out && !aligned(U_out, 4)))
    return QLORA_ERR_ALIGNMENT;
  if (!std::isfinite(scale)) return QLORA_ERR_INVALID_ARG;
  st = check_device();
  if (st != QLORA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t N = w->rows, K = w->cols;
  const LinearWs lay = linear_ws_layout(M, N, K, dense);
  int* status = at<int>(ws, 0);
  cudaError_t e;
  if (M <= kGemvMaxM) {
    GemvParams gp{};
    gp.packed = w->packed;
    gp.qscale = w->qscale;
    gp.c2 = w->scale_format == kScalesFp32 ? w->absmax : w->c2;  // fp32 scales: the absmax array
    gp.mu = w->mu;
    gp.codebook = w->codebook;
    gp.scale_format = w->scale_format;
    gp.N = N;
    gp.K = K;
    gp.X = X;
    gp.M = static_cast<int>(M);
    gp.A = A;
    gp.r = r;
    gp.scale = scale;
    gp.upart = at<float>(ws, lay.gu);
    gp.n_upart = gemv_upart_count(K);
    gp.U_out = U_out;
    gp.Y = Y;
    gp.ypart = at<float>(ws, lay.gy);
    gp.status = status;
    // B rows travel with each weight tile as one bulk copy, which needs a
    // 16-byte aligned source; otherwise a zero-padded copy [N][64] is used.
    const bool b_direct = aligned(B, 16) || gemv_chunks(K) > 1;
    gp.B = b_direct ? B : at<uint16_t>(ws, lay.bpad);
    gp.ldb = b_direct ? r : kRankPad;
    if (!b_direct) {
      Timed tm(kFamSide, s);
      e = launch_pad_rank(B, false, N, r, at<uint16_t>(ws, lay.bpad), s);
      if (e != cudaSuccess) return from_cuda(e);
    }
    Timed tm(kFamGemv, s, gemv_launches(K, static_cast<int>(M)));
    return from_cuda(launch_gemv(gp, s));
  }
  // Tensor-core path: U = X A^T, padded B if needed, GEMM with the rank-r
  // step; the GEMM decodes the 4-bit weight itself, or, on the dense-weight
  // path, reads a bf16 copy dequantized first into the workspace.
  if (dense) {
    DequantBatchParams p;
    dequant_one(p, w, at<uint16_t>(ws, lay.wbf));
    Timed tm(kFamDequant, s);
    e = launch_dequant_batch(p, 0, s);
    if (e != cudaSuccess) return from_cuda(e);
  }
  SkinnyOut so{};
  so.o32 = U_out;
  so.o32_ld = r;
  so.os = at<uint16_t>(ws, lay.us);
  so.scale = scale;
  // The fused GEMM's block scales ride in the U reduction's launch.
  if (!dense) so.bs = block_scales_job(view_of(w), at<float>(ws, lay.scales));
  // The caller's B [N, r] feeds the rank step directly when its rows are
  // 16-byte multiples; otherwise a zero-padded copy [N, 64] does.
  const bool b_direct = (r % 8) == 0 && aligned(B, 16);
  {
    Timed tm(kFamSide, s, b_direct ? 2 : 3);
    e = launch_skinny(X, M, K, A, true, r, 0, at<float>(ws, lay.skpart), so, status, s);
    if (e == cudaSuccess && !b_direct) e = launch_pad_rank(B, false, N, r, at<uint16_t>(ws, lay.bpad), s);
  }
  if (e != cudaSuccess) return from_cuda(e);
  const uint16_t* B2 = b_direct ? B : at<uint16_t>(ws, lay.bpad);
  const int64_t ldb2 = b_direct ? r : kRankPad;
  if (!dense) {
    Timed tm(kFamGemm, s, 1);  // the block scales came with the U reduction
    return gemm_status(launch_linear_gemm_nf4(w, at<float>(ws, lay.scales), X, M, at<uint16_t>(ws, lay.us), B2, r,
                                              ldb2, Y, 0, status, false, s, true, diag.wait_limit_ns,
                                              diag.debug_stall));
  }
  GemmArgs g{};
  g.A = X;
  g.B = at<uint16_t>(ws, lay.wbf);
  g.A2 = at<uint16_t>(ws, lay.us);
  g.B2 = B2;
  g.ldb2 = ldb2;
  g.M = M;
  g.N = N;
  g.K = K;
  g.r = r;
  g.D = Y;
  g.accumulate = 0;
  g.status = status;
  Timed tm(kFamGemm, s);
  return from_cuda(launch_gemm_tn(g, s));
}

}  // namespace

extern "C" qlora_status qlora_linear_fwd(const qlora_nf4_weight* w, const uint16_t* X, int64_t M, const uint16_t* A,
                                         const uint16_t* B, int32_t r, float scale, uint16_t* Y, float* U_out,
                                         void* ws, size_t ws_bytes, void* stream) {
  return linear_fwd(w, X, M, A, B, r, scale, Y, U_out, ws, ws_bytes, stream, GemmDiagnostics{0, 0});
}

extern "C" qlora_status qlora_linear_fwd_stall_diagnostic(const qlora_nf4_weight* w, const uint16_t* X, int64_t M,
                                                          const uint16_t* A, const uint16_t* B, int32_t r,
                                                          float scale, uint16_t* Y, void* ws, size_t ws_bytes,
                                                          int32_t wait_limit_us, void* stream) {
  if (M <= kGemvMaxM || wait_limit_us < 1 || wait_limit_us > 1000000) return QLORA_ERR_INVALID_ARG;
  return linear_fwd(w, X, M, A, B, r, scale, Y, nullptr, ws, ws_bytes, stream,
                    GemmDiagnostics{static_cast<uint64_t>(wait_limit_us) * 1000ull, 1});
}

extern "C" qlora_status qlora_selftest_mbarrier_ring(int32_t stages, int32_t consumers, int32_t iters,
                                                     int32_t wait_limit_us, int32_t* d_result, void* stream) {
  if (stages < 1 || stages > 8 || consumers < 0 || consumers > 4 || iters < 1 || iters > (1 << 24) ||
      wait_limit_us < 1 || wait_limit_us > 1000000 || d_result == nullptr)
    return QLORA_ERR_INVALID_ARG;
  if (!aligned(d_result, 4)) return QLORA_ERR_ALIGNMENT;
  const qlora_status st = check_device();
  if (st != QLORA_OK) return st;
  return from_cuda(launch_mbarrier_ring_selftest(stages, consumers, iters, static_cast<uint64_t>(wait_limit_us) * 1000ull,
                                                 d_result, static_cast<cudaStream_t>(stream)));
}

extern "C" qlora_status qlora_selftest_checks(int32_t* d_result, void* stream) {
  if (d_result == nullptr) return QLORA_ERR_INVALID_ARG;
  if (!aligned(d_result, 4)) return QLORA_ERR_ALIGNMENT;
  const qlora_status st = check_device();
  if (st != QLORA_OK) return st;
  return from_cuda(launch_checks_selftest(d_result, static_cast<cudaStream_t>(stream)));
}

extern "C" qlora_status qlora_linear_bwd(const qlora_nf4_weight* w, const uint16_t* X, const uint16_t* dY, int64_t M,
                                         const uint16_t* A, const uint16_t* B, int32_t r, float scale, const float* U,
                                         uint16_t* dX, int32_t accumulate, float* dA, float* dB, void* ws,
                                         size_t ws_bytes, void* stream) {
  const bool dense = dense_weight_path();
  qlora_status st = check_linear_args(w, M, r, ws_bytes, ws, dense);
  if (st != QLORA_OK) return st;
  if (!X || !dY || !A || !B) return QLORA_ERR_INVALID_ARG;
  if (accumulate != 0 && accumulate != 1) return QLORA_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(dY, 16) || !aligned(A, 16) || !aligned(B, 2) || (dX && !aligned(dX, 16)) ||
      (dA && !aligned(dA, 4)) || (dB && !aligned(dB, 4)) || (U && !aligned(U, 4)))
    return QLORA_ERR_ALIGNMENT;
  if (!std::isfinite(scale)) return QLORA_ERR_INVALID_ARG;
  st = check_device();
  if (st != QLORA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t N = w->rows, K = w->cols;
  const LinearWs lay = linear_ws_layout(M, N, K, dense);
  int* status = at<int>(ws, 0);
  cudaError_t e;

  const bool b_direct = (r % 8) == 0 && aligned(B, 16);
  // B [N, r] feeds the rank-r kernels directly when its rows are 16-byte
  // multiples, else through a zero-padded copy [N, 64].
  if (!b_direct) {
    Timed tm(kFamSide, s);
    e = launch_pad_rank(B, false, N, r, at<uint16_t>(ws, lay.bpad), s);
    if (e != cudaSuccess) return from_cuda(e);
  }
  const uint16_t* Bk = b_direct ? B : at<uint16_t>(ws, lay.bpad);
  const int64_t ldbk = b_direct ? r : kRankPad;
  // U = X A^T as a bf16 hi/lo pair (from the saved fp32 U, or recomputed).
  auto u_hilo = [&]() -> cudaError_t {
    if (U != nullptr) {
      Timed tm(kFamSide, s);
      return launch_split_hilo(U, M, r, at<uint16_t>(ws, lay.uhi), at<uint16_t>(ws, lay.ulo), s);
    }
    SkinnyOut uo{};
    uo.ohi = at<uint16_t>(ws, lay.uhi);
    uo.olo = at<uint16_t>(ws, lay.ulo);
    uo.scale = 1.0f;
    Timed tm(kFamSide, s, 2);
    return launch_skinny(X, M, K, A, true, r, 0, at<float>(ws, lay.skpart), uo, status, s);
  };
  BlockScalesJob bs{};  // the dX GEMM's block scales, when a kernel before it carries them
  if (dB != nullptr && r <= kVdbMaxRank && M > kGemvMaxM) {
    // V = dY B (s*V for the dX rank step, hi/lo for dA) and dB = s dY^T U in one pass over dY.
    // A saved fp32 U goes straight to the rank transposes, which split it
    // themselves; otherwise U is recomputed as its hi/lo split first.
    if (U == nullptr) {
      e = u_hilo();
      if (e != cudaSuccess) return from_cuda(e);
    }
    // The dX GEMM's block scales ride in the pass's reduction launch.
    if (dX != nullptr && !dense) bs = block_scales_job(view_of(w), at<float>(ws, lay.scales));
    Timed tm(kFamSide, s, 3);  // the rank transposes, the pass, the reduction
    e = launch_vdb_tc(dY, M, N, Bk, ldbk, at<uint16_t>(ws, lay.uhi), at<uint16_t>(ws, lay.ulo), U, r, scale,
                      at<float>(ws, lay.vdbpart), at<uint16_t>(ws, lay.bt), at<uint16_t>(ws, lay.uht),
                      at<uint16_t>(ws, lay.ult), at<uint16_t>(ws, lay.vs), at<uint16_t>(ws, lay.vhi),
                      at<uint16_t>(ws, lay.vlo), dB, bs, status, s);
    if (e != cudaSuccess) return from_cuda(e);
  } else {
    // V = dY B (bf16 s*V for the dX rank step; hi/lo split for dA).
    SkinnyOut vo{};
    vo.os = at<uint16_t>(ws, lay.vs);
    vo.ohi = at<uint16_t>(ws, lay.vhi);
    vo.olo = at<uint16_t>(ws, lay.vlo);
    vo.scale = scale;
    {
      Timed tm(kFamSide, s, 2);
      e = launch_skinny(dY, M, N, Bk, false, r, ldbk, at<float>(ws, lay.skpart), vo, status, s);
    }
    if (e != cudaSuccess) return from_cuda(e);
    if (dB != nullptr) {  // dB = s dY^T U
      e = u_hilo();
      if (e != cudaSuccess) return from_cuda(e);
      Timed tm(kFamSide, s, 2);
      e = launch_colsum(dY, M, N, at<uint16_t>(ws, lay.uhi), at<uint16_t>(ws, lay.ulo), r, scale,
                        at<float>(ws, lay.part), dB, false, status, s);
      if (e != cudaSuccess) return from_cuda(e);
    }
  }
  if (dX != nullptr && !dense) {  // dX = dY W_hat + s V A, W_hat decoded in the GEMM, A [r, K] MN-major
    const bool scales_written = bs.out != nullptr;
    Timed tm(kFamGemm, s, scales_written ? 1 : 2);  // (block-scale pre-pass +) GEMM
    e = launch_linear_gemm_nf4(w, at<float>(ws, lay.scales), dY, M, at<uint16_t>(ws, lay.vs), A, r, 0, dX, accumulate,
                               status, true, s, scales_written);
    if (e != cudaSuccess) return gemm_status(e);
  }
  if (dX != nullptr && dense) {  // dense-weight path: W_hat [N, K] and A [r, K] read as MN-major operands
    DequantBatchParams p;
    dequant_one(p, w, at<uint16_t>(ws, lay.wbf));
    {
      Timed tm(kFamDequant, s);
      e = launch_dequant_batch(p, 0, s);
    }
    if (e != cudaSuccess) return from_cuda(e);
    GemmArgs g{};
    g.A = dY;
    g.B = at<uint16_t>(ws, lay.wbf);
    g.A2 = at<uint16_t>(ws, lay.vs);
    g.B2 = A;
    g.b_mn_major = 1;
    g.M = M;
    g.N = K;
    g.K = N;
    g.r = r;
    g.D = dX;
    g.accumulate = accumulate;
    g.status = status;
    {
      Timed tm(kFamGemm, s);
      e = launch_gemm_tn(g, s);
    }
    if (e != cudaSuccess) return from_cuda(e);
  }
  if (dA != nullptr) {  // dA = s V^T X
    {
      Timed tm(kFamSide, s, 2);
      e = launch_colsum(X, M, K, at<uint16_t>(ws, lay.vhi), at<uint16_t>(ws, lay.vlo), r, scale,
                        at<float>(ws, lay.part), dA, true, status, s);
    }
    if (e != cudaSuccess) return from_cuda(e);
  }
  return QLORA_OK;
}

extern "C" qlora_status qlora_timing_enable(int32_t enable) {
  TimingState& T = timing();
  std::lock_guard<std::mutex> lock(T.mu);
  if (enable) {
    for (int f = 0; f < kFamCount; ++f) {
      for (auto& pr : T.pending[f]) {
        T.pool.push_back(pr.first);
        T.pool.push_back(pr.second);
      }
      T.pending[f].clear();
      T.ms[f] = 0.0;
      T.launches[f] = 0;
    }
  }
  T.enabled.store(enable != 0, std::memory_order_relaxed);
  return QLORA_OK;
}

extern "C" qlora_status qlora_timing_read(const char* family, double* total_ms, int64_t* launches) {
  if (family == nullptr) return QLORA_ERR_INVALID_ARG;
  int f = -1;
  for (int i = 0; i < kFamCount; ++i)
    if (std::strcmp(family, kFamNames[i]) == 0) f = i;
  if (f < 0) return QLORA_ERR_INVALID_ARG;
  TimingState& T = timing();
  std::lock_guard<std::mutex> lock(T.mu);
  // Every pending pair is consumed, so a failed pair is neither counted nor
  // read again; the first failure is returned after the others are summed.
  cudaError_t first_error = cudaSuccess;
  for (auto& pr : T.pending[f]) {
    float ms = 0.0f;
    cudaError_t e = cudaEventSynchronize(pr.second);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, pr.first, pr.second);
    if (e == cudaSuccess)
      T.ms[f] += ms;
    else if (first_error == cudaSuccess)
      first_error = e;
    T.pool.push_back(pr.first);
    T.pool.push_back(pr.second);
  }
  T.pending[f].clear();
  if (total_ms) *total_ms = T.ms[f];
  if (launches) *launches = T.launches[f];
  return from_cuda(first_error);
}

// ===========================================================================
// Quantize without a caller-provided workspace
// ===========================================================================
//
// qlora_nf4_quantize needs ~1 KB of device scratch per 16384 weights (block
// scales, chunk sums, a counter and a status word) which the caller normally
// provides as a workspace.  qlora_nf4_quantize_noalloc takes that scratch from
// the static device array below instead, so a caller that cannot allocate
// device memory can still quantize.  The array is sized for tensors of up to
// kNoAllocMaxWeights weights; every GPU that loads this library holds it
// until the process exits.
namespace {

constexpr int64_t kNoAllocMaxWeights = int64_t{1} << 26;  // 67,108,864 weights per call
constexpr int64_t kNoAllocMaxChunks = kNoAllocMaxWeights / kChunkWeights;
constexpr QuantWs kNoAllocLayout = quant_ws_layout(1, kNoAllocMaxChunks);

// Device scratch shared by every qlora_nf4_quantize_noalloc call on a device.
static __device__ __align__(256) unsigned char g_quant_scratch[kNoAllocLayout.total];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_scratch[kNoAllocMaxDevices] = {};

// Device address of g_quant_scratch on the current device, resolved once per
// device.  In host code the array's name only stands for the symbol; the
// address the kernels need comes from cudaGetSymbolAddress.
qlora_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return QLORA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_scratch[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_quant_scratch);
    if (e != cudaSuccess || p == nullptr) return QLORA_ERR_CUDA;
    g_noalloc_scratch[dev] = p;
  }
  *out = g_noalloc_scratch[dev];
  return QLORA_OK;
}

}  // namespace

extern "C" qlora_status qlora_nf4_quantize_noalloc(const float* W, const qlora_nf4_weight* out, int32_t* d_status,
                                                   void* stream) {
  qlora_status st = check_weight(out);
  if (st != QLORA_OK) return st;
  if (W == nullptr) return QLORA_ERR_INVALID_ARG;
  if (out->rows > kNoAllocMaxWeights / out->cols) return QLORA_ERR_UNSUPPORTED;  // beyond the static scratch
  if (!aligned(W, 32)) return QLORA_ERR_ALIGNMENT;
  if (d_status != nullptr && !aligned(d_status, 4)) return QLORA_ERR_ALIGNMENT;
  st = check_device();
  if (st != QLORA_OK) return st;
  const Nf4DecisionTable* tab = decision_table(out->codebook);
  if (tab == nullptr) return QLORA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != QLORA_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = d_status != nullptr ? d_status : at<int>(scratch, 0);
  // The scratch keeps the previous call's contents: clear what must start at zero.
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(at<unsigned>(scratch, kNoAllocLayout.counters), 0, sizeof(unsigned), s);
  if (e != cudaSuccess) return from_cuda(e);

  QuantBatchParams p;
  std::memset(&p, 0, sizeof(p));
  p.count = 1;
  p.chunk_begin[0] = 0;
  p.chunk_begin[1] = p.total_chunks = n_chunks_of(out->rows, out->cols);
  p.n_blocks[0] = out->rows * out->cols / kBlock;
  p.W[0] = W;
  p.packed[0] = out->packed;
  p.qscale[0] = out->qscale;
  p.c2[0] = out->c2;
  p.mu[0] = out->mu;
  p.in_dtype = QLORA_INPUT_FP32;
  p.codebook = out->codebook;
  p.scale_format = out->scale_format;
  p.absmax = at<float>(scratch, kNoAllocLayout.absmax);
  p.absmax_out[0] = out->absmax;
  p.chunk_sum = at<double>(scratch, kNoAllocLayout.sums);
  p.chunk_exp = at<int>(scratch, kNoAllocLayout.exps);
  p.counters = at<unsigned>(scratch, kNoAllocLayout.counters);
  p.status = status;
  p.table = *tab;
  {
    Timed tm(kFamQuant, s, 2);
    e = launch_quantize_batch(p, s);
  }
  if (e != cudaSuccess) return from_cuda(e);
  if (d_status != nullptr) return QLORA_OK;
  int32_t h = 0;
  e = cudaMemcpyAsync(&h, status, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return from_cuda(e);
  return static_cast<qlora_status>(h);
}
