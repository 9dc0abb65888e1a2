// Self-test of the bounded-wait mechanism (kda_selftest_bounded_wait).
//
// Every wait of the library's kernels on an mbarrier (asynchronous copies, tensor-
// core operations) polls a bounded number of times; when the limit runs out the
// kernel stops waiting, raises a device flag and finishes, so that a lost
// completion shows up as a status (kda_device_status) instead of a hung GPU.  This
// kernel exercises that path on purpose: one thread waits on an mbarrier phase
// that nothing completes, gives up after `polls` polls and raises its own flag.
#include "kda_common.cuh"
#include "sm100.cuh"

namespace kda {

// Set by the self-test kernel when its (never completed) wait gives up.
__device__ int g_selftest_timeout = 0;

namespace {
using namespace sm100;

__global__ void kda_selftest_wait_kernel(uint32_t polls) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);                 // one arrival expected; none is ever made
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, polls)) atomicExch(&g_selftest_timeout, 1);
}

}  // namespace

cudaError_t launch_selftest_wait(uint32_t polls, cudaStream_t stream) {
  kda_selftest_wait_kernel<<<1, 32, 0, stream>>>(polls);
  note_launches(1);
  return cudaGetLastError();
}

// Reads (and with reset clears) g_selftest_timeout; host side of kda_device_status.
cudaError_t take_selftest_timeout(int* flag, bool reset) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_selftest_timeout, sizeof(int));
  if (e == cudaSuccess && reset && v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_selftest_timeout, &zero, sizeof(int));
  }
  *flag = v;
  return e;
}

}  // namespace kda
