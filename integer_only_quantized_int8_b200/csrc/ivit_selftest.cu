// ivit_selftest.cu -- diagnostics: a kernel that makes a bounded wait run out,
// so that the failure path (status word, ivit_stream_status, a usable context
// afterwards) can be tested without faulting or hanging a GPU; and a probe of
// the integer throughput of the instruction mix the Shiftmax passes issue,
// which gives the attention kernels their measured roof.
#include <atomic>

#include "ivit_common.cuh"
#include "ivit_internal.h"
#include "../../include/ivit_selftest.h"

namespace ivit {
namespace {
// (kernel << 32) | index of the pending withhold request, 0 when none
std::atomic<uint64_t> g_withhold{0};
}  // namespace

int32_t take_withhold(int kernel) {
  uint64_t cur = g_withhold.load(std::memory_order_relaxed);
  while (cur != 0 && (int)(cur >> 32) == kernel) {
    if (g_withhold.compare_exchange_weak(cur, 0, std::memory_order_acq_rel)) return (int32_t)(uint32_t)cur;
  }
  return -1;
}
}  // namespace ivit

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

// The Shiftmax mix: per step of each of kIntChains independent chains, the
// integer operations a score goes through on the CUDA cores (I-ViT section
// 3.3): the logit requant by mul.hi, the two-sided saturation, the offset
// from the row maximum, the table index and the ShiftExp table load from
// shared memory, the row-sum add, and a shift and add that feed the next
// step (so no chain is loop-invariant).  kIntOpsPerStep counts them.
constexpr int kIntChains = 8;
constexpr int kIntOpsPerStep = 10;
constexpr int kIntThreads = 256;

__global__ void __launch_bounds__(kIntThreads) int_rate_kernel(int32_t iters, int32_t bq, int32_t* sink) {
  __shared__ int32_t tab[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) tab[i] = 1000 - 3 * i;
  __syncthreads();
  int32_t a[kIntChains], s[kIntChains];
#pragma unroll
  for (int k = 0; k < kIntChains; ++k) {
    a[k] = (int32_t)(threadIdx.x * 7919u + blockIdx.x * 104729u + k * 15485863u);
    s[k] = 0;
  }
  const int32_t lo = -128, hi = 127, mx = 127;
  for (int32_t it = 0; it < iters; ++it) {
#pragma unroll
    for (int k = 0; k < kIntChains; ++k) {
      int32_t t = __mulhi(a[k], bq);                      // 1 requant multiply
      t = max(t, lo);                                     // 2 saturation
      t = min(t, hi);                                     // 3
      const int32_t d = mx - t;                           // 4 offset from the row maximum
      const int32_t e = tab[d & 255];                     // 5 index, 6 table load
      s[k] += e;                                          // 7 row sum
      a[k] += (e >> 1) + it;                              // 8 shift, 9-10 adds
    }
  }
  int32_t r = 0;
#pragma unroll
  for (int k = 0; k < kIntChains; ++k) r ^= s[k] ^ a[k];
  for (int o = 16; o > 0; o >>= 1) r ^= __shfl_xor_sync(0xffffffffu, r, o);
  if ((threadIdx.x & 31) == 0) atomicXor(sink + blockIdx.x, r);
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

extern "C" ivit_status ivit_selftest_int_rate(int32_t iters, int32_t* sink, int32_t sink_len, int64_t* ops,
                                              ivit_stream_t stream) {
  if (iters < 1 || !sink || !ops) return IVIT_ERR_INVALID_ARG;
  ivit::DeviceCtx dc;
  const ivit_status st = ivit::device_ctx(&dc);
  if (st != IVIT_OK) return st;
  const int grid = dc.num_sms * 4;  // 32 warps per SM
  if (sink_len < grid) return IVIT_ERR_INVALID_ARG;
  *ops = (int64_t)grid * ivit::kIntThreads * (int64_t)iters * ivit::kIntChains * ivit::kIntOpsPerStep;
  ivit::int_rate_kernel<<<grid, ivit::kIntThreads, 0, (cudaStream_t)stream>>>(iters, 0x2b8e5f31, sink);
  ivit::note_launch();
  return cudaGetLastError() == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}

extern "C" ivit_status ivit_selftest_withhold(int32_t kernel, int32_t index) {
  if ((kernel != ivit::kWithholdGemm && kernel != ivit::kWithholdAttention) || index < 0) return IVIT_ERR_INVALID_ARG;
  ivit::g_withhold.store(((uint64_t)(uint32_t)kernel << 32) | (uint32_t)index, std::memory_order_release);
  return IVIT_OK;
}
