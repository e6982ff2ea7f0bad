// ivit_static_scratch.cu -- an encoder-block forward that allocates nothing.
//
// Some callers cannot allocate device memory at all, not even a workspace to
// pass in: an inference-server plugin whose host hands it no allocator, code
// running inside a framework whose caching allocator has already reserved
// the whole device (so a direct cudaMalloc fails or fragments the pool), and
// latency-critical loops that cannot afford cudaMalloc/cudaFree, which may
// synchronise the whole device.  For them the intermediates of the block
// live in one fixed-size array of device memory that this library defines at
// file scope; the caller passes only the inputs, the outputs and the weights.
//
// The array exists once per GPU that loads this library and stays allocated
// until the process exits.  In host code its name is only a host-side stand-in,
// so its device address is looked up with cudaGetSymbolAddress, once per
// device, with that device current, on the first call made on that device.
#include <mutex>

#include "ivit_common.cuh"
#include "ivit_internal.h"

namespace {

constexpr size_t kScratchBytes = IVIT_STATIC_SCRATCH_BYTES;
constexpr int kMaxScratchDevices = 64;

// Intermediates of ivit_block_forward_static (LN output, QKV, context, first
// residual sum, fc1 + ShiftGELU output), shared by every call on a device.
static __device__ __align__(256) unsigned char g_block_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxScratchDevices] = {};

// Device address of g_block_scratch on the current device (set up once).
ivit_status scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxScratchDevices) return IVIT_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_block_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();  // leave no error behind for the next launch check
      return IVIT_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return IVIT_OK;
}

}  // namespace

extern "C" ivit_status ivit_block_forward_static(const ivit_block_params* p, const int8_t* x, int8_t* y,
                                                 int32_t B, int32_t N, ivit_stream_t stream) {
  // the checks of ivit_block_forward, in its order, then the array's capacity
  ivit_status st = ivit::check_block_args(p, x, y, B, N);
  if (st != IVIT_OK || B == 0 || N == 0) return st;
  if (ivit_block_workspace_bytes(B, N, p->D, p->Dm) > kScratchBytes) return IVIT_ERR_UNSUPPORTED;
  ivit::DeviceCtx dc;
  if ((st = ivit::device_ctx(&dc)) != IVIT_OK) return st;  // not an sm_100 device: UNSUPPORTED
  void* scratch = nullptr;
  if ((st = scratch_address(dc.device, &scratch)) != IVIT_OK) return st;
  // Every intermediate is written in full before it is read, so nothing in the
  // array has to start at zero and nothing is cleared between calls.
  return ivit_block_forward(p, x, y, scratch, kScratchBytes, B, N, stream);
}
