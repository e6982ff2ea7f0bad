// ivit_selftest.cu -- a kernel that makes a bounded wait run out, so that the
// failure path (status word, ivit_stream_status, a usable context afterwards)
// can be tested without faulting or hanging a GPU.
#include "ivit_common.cuh"
#include "ivit_internal.h"
#include "../../include/ivit_selftest.h"

namespace ivit {
namespace {

// One warp; lane 0 initialises an mbarrier expecting one arrival and waits
// for its first phase, which nothing completes.  mbar_wait gives up after the
// wait budget, records the timeout in *status and returns false.
__global__ void __launch_bounds__(32) wait_timeout_kernel(int* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    (void)mbar_wait(&bar, 0, status);
  }
}

}  // namespace
}  // namespace ivit

extern "C" ivit_status ivit_selftest_wait_timeout(ivit_stream_t stream) {
  ivit::DeviceCtx dc;
  const ivit_status st = ivit::device_ctx(&dc);
  if (st != IVIT_OK) return st;
  ivit::wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(dc.status);
  ivit::note_launch();
  return cudaGetLastError() == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}
