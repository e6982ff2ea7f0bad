// ivit_internal.h -- launchers shared between the operator files and the C ABI.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/ivit.h"

namespace ivit {

enum EpiMode : int { kEpiPlain = 0, kEpiResidual = 1, kEpiGelu = 2 };

struct GeluParams {
  int32_t I0, M, k_out;
  ivit_dyadic out;
};

// Per-device context: SM count, the status word's device address.
struct DeviceCtx {
  int device;
  int num_sms;
  int* status;
};
ivit_status device_ctx(DeviceCtx* out);

// Count a kernel launch (for ivit_launch_count).
void note_launch(int n = 1);

// Diagnostics (ivit_selftest_withhold): the index at which the next launch of
// the given kernel has its producer stop, or -1; taking it clears it.
enum WithholdKernel : int { kWithholdGemm = 1, kWithholdAttention = 2 };
int32_t take_withhold(int kernel);

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel of the stream finishes; it must call pdl_wait() before
// touching that kernel's outputs or writing global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

ivit_status encode_tmap_2d_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                              uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                              CUtensorMapSwizzle swizzle);

// The host-side checks of one encoder-block call other than those of its
// workspace (parameters, alignment, sizes, attention configuration).
ivit_status check_block_args(const ivit_block_params* p, const int8_t* x, const int8_t* y, int32_t B, int32_t N);

ivit_status launch_gemm(const DeviceCtx& dc, const int8_t* X, int64_t M, int32_t K, const int8_t* W, int32_t N,
                        const int32_t* bias, const int32_t* b, const int8_t* c, int32_t out_bits, bool round,
                        EpiMode mode, const int8_t* skip, ivit_residual res, const GeluParams* gelu, int8_t* Y,
                        cudaStream_t stream);

// Whether the attention kernels take (N, k_s, I0): up to 640 keys; logits
// wider than 8 bits (ShiftExp computed, not looked up) on up to 256 keys and
// with (largest -I_p) * I0 < 2^32.
bool attention_config_supported(int32_t N, int32_t k_s, int32_t I0);

// lis: Log-Int-Softmax instead of Shiftmax (logits of at most 8 bits, M >= 15;
// k_out is then unused)
ivit_status launch_attention(const DeviceCtx& dc, const int8_t* qkv, int32_t B, int32_t N, int32_t H,
                             ivit_dyadic logit, int32_t k_s, int32_t I0, int32_t M, int32_t k_out,
                             ivit_dyadic out, int8_t* ctx, cudaStream_t stream, bool lis = false);

ivit_status launch_shiftgelu(const DeviceCtx& dc, const int8_t* x, int64_t n, const GeluParams& g, int8_t* y,
                             cudaStream_t stream);

// ShiftGELU with the row's largest exponent as I_max, x [rows x cols]
// (cols a multiple of 16).
ivit_status launch_shiftgelu_rowmax(const DeviceCtx& dc, const int8_t* x, int64_t rows, int32_t cols,
                                    const GeluParams& g, int8_t* y, cudaStream_t stream);

// I-LayerNorm of x << alpha (alpha [cols], values 0 .. 3; cols a multiple of
// 16, at most 2048; M_ln <= 20).
ivit_status launch_layernorm_ptf(const DeviceCtx& dc, const int8_t* x, int64_t rows, int32_t cols,
                                 const uint8_t* alpha, const int8_t* gamma, const int32_t* beta, int32_t F,
                                 int32_t M_ln, ivit_dyadic out, int8_t* y, cudaStream_t stream);

// Patch rows z [B*Np x C*P*P] from img [B x C x Hi x Wi] (Hi, Wi multiples of P).
ivit_status launch_im2col(const DeviceCtx& dc, const int8_t* img, int32_t B, int32_t C, int32_t Hi, int32_t Wi,
                          int32_t P, int8_t* z, cudaStream_t stream);

// Tokens x [B*(Np+1) x D] from the class token, the patch embeddings e
// [B*Np x D] and the position embedding pos [(Np+1) x D] (D a multiple of 16).
ivit_status launch_tokens(const DeviceCtx& dc, const int8_t* e, const int8_t* cls, const int8_t* pos,
                          ivit_residual add, int32_t B, int32_t Np, int32_t D, int8_t* x, cudaStream_t stream);

// t [B x D] = the first of each image's Ntok rows of x (D a multiple of 16).
ivit_status launch_gather_rows(const DeviceCtx& dc, const int8_t* x, int32_t B, int32_t Ntok, int32_t D, int8_t* t,
                               cudaStream_t stream);

ivit_status launch_layernorm(const DeviceCtx& dc, const int8_t* x, int64_t rows, int32_t cols,
                             const int8_t* gamma, const int32_t* beta, int32_t F, int32_t M_ln, ivit_dyadic out,
                             int8_t* y, cudaStream_t stream);

}  // namespace ivit
