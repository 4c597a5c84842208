// wait_timeout_probe.cu -- test-only library: exercises the bounded mbarrier wait the prefill kernel uses.
//
// One thread initialises an mbarrier that nothing ever arrives on and waits for its first phase with a short
// limit. The wait must give up, raise the abort flag and OR the timeout bit into the status word, and the
// kernel must return normally, leaving the context usable. No fault, trap or endless loop is involved.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../head_sparse_paged_b200/csrc/sm100_ptx.cuh"

namespace {
__global__ void wait_never_completes(int32_t* status, int32_t* result, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    segpaged::ptx::mbar_init(&bar, 1);
    segpaged::ptx::mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = segpaged::ptx::mbar_wait(&bar, 0, &abort_flag, status, 4, limit_ns);
    result[0] = ok ? 1 : 0;
    result[1] = abort_flag;
  }
}
__global__ void add_one(int32_t* x) { x[2] += 1; }
}  // namespace

extern "C" int segpaged_test_wait_timeout(int32_t* status_dev, int32_t* result_dev, uint64_t limit_ns) {
  wait_never_completes<<<1, 32>>>(status_dev, result_dev, limit_ns);
  if (cudaGetLastError() != cudaSuccess) return -1;
  add_one<<<1, 1>>>(result_dev);   // the context still runs work after the timed-out wait
  if (cudaDeviceSynchronize() != cudaSuccess) return -2;
  return 0;
}
