// Phase-parity self-test of the shared-memory barrier ring that the
// pipelined kernels use (mbarrier init, arrive, parity wait and the bounded
// wait with its timeout).  The pages have no counterpart: this checks the
// library's synchronisation, not a step of the method.
//
// One CTA of 1 + C warps.  Lane 0 of warp 0 produces `iters` values into a
// ring of `stages` shared slots; lane 0 of each of the C consumer warps reads
// every value in order.  full[s] (one arrival) publishes slot s, empty[s] (C
// arrivals) hands it back; the waits take the phase parity of the pass
// (i / stages) exactly as the GEMM, side and V/dB rings do.  With C = 0 the
// producer's second pass waits on an empty barrier nothing arrives at, so its
// bounded wait runs out and records QLORA_ERR_TIMEOUT.
#include "common.cuh"
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kRingMaxStages = 8;

__global__ void __launch_bounds__(160) mbarrier_ring_kernel(int stages, int iters, int consumers, uint64_t limit_ns,
                                                            int* result) {
  __shared__ uint64_t full[kRingMaxStages], empty[kRingMaxStages];
  __shared__ int slot[kRingMaxStages];
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], consumers > 0 ? consumers : 1);
      slot[s] = 0;
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (lane != 0) return;
  volatile int* vslot = slot;
  int wrong = 0, read = 0;
  if (warp == 0) {
    for (int i = 0; i < iters; ++i) {
      const int s = i % stages, u = i / stages;
      if (i >= stages && !mbar_wait(&empty[s], (u - 1) & 1, &abort_flag, result + 2, limit_ns)) break;
      vslot[s] = i + 1;
      mbar_arrive(&full[s]);  // release: the slot's value before the phase completes
    }
  } else {
    for (int i = 0; i < iters; ++i) {
      const int s = i % stages, u = i / stages;
      if (!mbar_wait(&full[s], u & 1, &abort_flag, result + 2, limit_ns)) break;
      if (vslot[s] != i + 1) ++wrong;
      ++read;
      mbar_arrive(&empty[s]);
    }
  }
  atomicAdd(result, wrong);
  atomicAdd(result + 1, read);
}

// One thread runs a test that always fails: a library built with
// QLORA_CHECKS records QLORA_ERR_CHECK in *result, the default build (where
// the test compiles away) leaves the 0 written before.
__global__ void checks_probe_kernel(int* result) { qlora_checked(result, false); }

}  // namespace

cudaError_t launch_checks_selftest(int* result, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(result, 0, sizeof(int), stream);
  if (e != cudaSuccess) return e;
  checks_probe_kernel<<<1, 1, 0, stream>>>(result);
  return cudaGetLastError();
}

cudaError_t launch_mbarrier_ring_selftest(int stages, int consumers, int iters, uint64_t limit_ns, int* result,
                                          cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(result, 0, 3 * sizeof(int), stream);
  if (e != cudaSuccess) return e;
  mbarrier_ring_kernel<<<1, 32 * (1 + consumers), 0, stream>>>(stages, iters, consumers, limit_ns, result);
  return cudaGetLastError();
}

}  // namespace qnf4
