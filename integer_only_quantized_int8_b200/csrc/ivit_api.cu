// ivit_api.cu -- the C ABI: argument validation, per-device context, TMA
// descriptor encoding and the encoder-block orchestration.  See include/ivit.h
// for the contract of every entry point.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "ivit_common.cuh"
#include "ivit_internal.h"

namespace ivit {

// One status word per device (a module-scope device variable exists once per
// device context); kernels receive its address.
__device__ int g_status_word;

static std::atomic<uint64_t> g_launches{0};
void note_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

namespace {

constexpr int kMaxDevices = 64;
struct CtxCache {
  bool ready = false;
  int num_sms = 0;
  int* status = nullptr;
  bool sm100 = false;
};
CtxCache g_ctx[kMaxDevices];
std::mutex g_ctx_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

ivit_status device_ctx(DeviceCtx* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return IVIT_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_ctx_mu);
  CtxCache& c = g_ctx[dev];
  if (!c.ready) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return IVIT_ERR_CUDA;
    c.sm100 = (prop.major == 10 && prop.minor == 0);
    c.num_sms = prop.multiProcessorCount;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_status_word) != cudaSuccess) return IVIT_ERR_CUDA;
    c.status = static_cast<int*>(addr);
    c.ready = true;
  }
  if (!c.sm100) return IVIT_ERR_UNSUPPORTED;
  out->device = dev;
  out->num_sms = c.num_sms;
  out->status = c.status;
  return IVIT_OK;
}

ivit_status encode_tmap_2d_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                              uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                              CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) return IVIT_ERR_CUDA;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? IVIT_OK : IVIT_ERR_CUDA;
}

}  // namespace ivit

using namespace ivit;

namespace {

bool valid_dyadic(ivit_dyadic d) { return d.b >= 0 && d.c >= 0 && d.c <= 31; }
bool valid_residual(ivit_residual r) {
  return r.b_skip >= 0 && r.b_branch >= 0 && r.c >= 0 && r.c <= 31;
}
bool valid_shiftmax(int32_t I0, int32_t M, int32_t k_out) {
  return I0 >= 1 && I0 <= (1 << 22) && k_out >= 1 && k_out <= 8 && M >= k_out - 1 && M <= 30;
}

ivit_status dyadic_impl(double s, int32_t* b, int32_t* c) {
  if (!std::isfinite(s) || s < 0.0 || !(s < 2147483647.5)) return IVIT_ERR_INVALID_ARG;
  for (int cc = 31; cc >= 0; --cc) {
    const double v = std::round(std::ldexp(s, cc));  // exact scaling, half away from zero
    if (v < 2147483648.0) {
      *b = (int32_t)v;
      *c = cc;
      return IVIT_OK;
    }
  }
  return IVIT_ERR_INVALID_ARG;
}

}  // namespace

extern "C" {

const char* ivit_status_string(ivit_status s) {
  switch (s) {
    case IVIT_OK:
      return "IVIT_OK";
    case IVIT_ERR_INVALID_ARG:
      return "IVIT_ERR_INVALID_ARG";
    case IVIT_ERR_UNSUPPORTED:
      return "IVIT_ERR_UNSUPPORTED";
    case IVIT_ERR_CUDA:
      return "IVIT_ERR_CUDA";
    case IVIT_ERR_TIMEOUT:
      return "IVIT_ERR_TIMEOUT";
    case IVIT_ERR_INTERNAL:
      return "IVIT_ERR_INTERNAL";
  }
  return "IVIT_ERR_UNKNOWN";
}

ivit_status ivit_dyadic_from_double(double s, ivit_dyadic* out) {
  if (!out) return IVIT_ERR_INVALID_ARG;
  int32_t b = 0, c = 0;
  ivit_status st = dyadic_impl(s, &b, &c);
  if (st != IVIT_OK) return st;
  out->b = b;
  out->c = c;
  return IVIT_OK;
}

ivit_status ivit_residual_from_double(double s_skip, double s_branch, ivit_residual* out) {
  if (!out) return IVIT_ERR_INVALID_ARG;
  int32_t b1, c1, b2, c2;
  ivit_status st = dyadic_impl(s_skip, &b1, &c1);
  if (st != IVIT_OK) return st;
  st = dyadic_impl(s_branch, &b2, &c2);
  if (st != IVIT_OK) return st;
  const int32_t c = c1 < c2 ? c1 : c2;
  out->b_skip = (int32_t)std::round(std::ldexp(s_skip, c));
  out->b_branch = (int32_t)std::round(std::ldexp(s_branch, c));
  out->c = c;
  return IVIT_OK;
}

ivit_status ivit_i0_from_scale(double S, int32_t* out) {
  if (!out || !std::isfinite(S) || !(S > 0.0)) return IVIT_ERR_INVALID_ARG;
  double v = std::round(1.0 / S);
  if (v < 1.0) v = 1.0;
  if (v > 2147483647.0) v = 2147483647.0;
  *out = (int32_t)v;
  return IVIT_OK;
}

ivit_status ivit_linear_requant(const int8_t* X, int64_t M, int32_t K, const int8_t* W, int32_t N,
                                const int32_t* bias, const int32_t* b, const int8_t* c, int32_t out_bits,
                                const int8_t* skip, ivit_residual res, int8_t* Y, ivit_stream_t stream) {
  if (!X || !W || !b || !c || !Y) return IVIT_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W) || !aligned16(b) || !aligned16(c) || !aligned16(Y) ||
      (bias && !aligned16(bias)) || (skip && !aligned16(skip)))
    return IVIT_ERR_INVALID_ARG;
  if (M < 1 || K < 16 || K % 16 != 0 || N < 16 || N % 16 != 0 || out_bits < 2 || out_bits > 8)
    return IVIT_ERR_INVALID_ARG;
  if (K > 16384 || M > 0x7fffff00LL) return IVIT_ERR_UNSUPPORTED;
  if (skip && !valid_residual(res)) return IVIT_ERR_INVALID_ARG;
  DeviceCtx dc;
  ivit_status st = device_ctx(&dc);
  if (st != IVIT_OK) return st;
  return launch_gemm(dc, X, M, K, W, N, bias, b, c, out_bits, skip ? kEpiResidual : kEpiPlain, skip, res, nullptr, Y,
                     (cudaStream_t)stream);
}

ivit_status ivit_linear_shiftgelu(const int8_t* X, int64_t M, int32_t K, const int8_t* W, int32_t N,
                                  const int32_t* bias, const int32_t* b, const int8_t* c, int32_t gelu_I0,
                                  int32_t gelu_M, int32_t gelu_k_out, ivit_dyadic gelu_out, int8_t* Y,
                                  ivit_stream_t stream) {
  if (!X || !W || !b || !c || !Y) return IVIT_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W) || !aligned16(b) || !aligned16(c) || !aligned16(Y) ||
      (bias && !aligned16(bias)))
    return IVIT_ERR_INVALID_ARG;
  if (M < 1 || K < 16 || K % 16 != 0 || N < 16 || N % 16 != 0) return IVIT_ERR_INVALID_ARG;
  if (!valid_shiftmax(gelu_I0, gelu_M, gelu_k_out) || !valid_dyadic(gelu_out)) return IVIT_ERR_INVALID_ARG;
  if (K > 16384 || M > 0x7fffff00LL) return IVIT_ERR_UNSUPPORTED;
  DeviceCtx dc;
  ivit_status st = device_ctx(&dc);
  if (st != IVIT_OK) return st;
  const GeluParams gp{gelu_I0, gelu_M, gelu_k_out, gelu_out};
  return launch_gemm(dc, X, M, K, W, N, bias, b, c, 8, kEpiGelu, nullptr, ivit_residual{0, 0, 0}, &gp, Y,
                     (cudaStream_t)stream);
}

ivit_status ivit_attention(const int8_t* qkv, int32_t B, int32_t N, int32_t H, ivit_dyadic logit, int32_t k_s,
                           int32_t I0, int32_t M, int32_t k_out, ivit_dyadic out, int8_t* ctx,
                           ivit_stream_t stream) {
  if (!qkv || !ctx || !aligned16(qkv) || !aligned16(ctx)) return IVIT_ERR_INVALID_ARG;
  if (B < 0 || N < 0 || H < 1 || k_s < 2 || k_s > 16 || !valid_shiftmax(I0, M, k_out) || !valid_dyadic(logit) ||
      !valid_dyadic(out))
    return IVIT_ERR_INVALID_ARG;
  if (N > 640 || (int64_t)B * N > 0x7fffff00LL || H > 4096 || !attention_config_supported(N, k_s, I0))
    return IVIT_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return IVIT_OK;
  DeviceCtx dc;
  ivit_status st = device_ctx(&dc);
  if (st != IVIT_OK) return st;
  return launch_attention(dc, qkv, B, N, H, logit, k_s, I0, M, k_out, out, ctx, (cudaStream_t)stream);
}

ivit_status ivit_shiftgelu(const int8_t* x, int64_t n, int32_t I0, int32_t M, int32_t k_out, ivit_dyadic out,
                           int8_t* y, ivit_stream_t stream) {
  if (n < 0 || !valid_shiftmax(I0, M, k_out) || !valid_dyadic(out)) return IVIT_ERR_INVALID_ARG;
  if (n == 0) return IVIT_OK;
  if (!x || !y || !aligned16(x) || !aligned16(y)) return IVIT_ERR_INVALID_ARG;
  DeviceCtx dc;
  ivit_status st = device_ctx(&dc);
  if (st != IVIT_OK) return st;
  GeluParams g{I0, M, k_out, out};
  return launch_shiftgelu(dc, x, n, g, y, (cudaStream_t)stream);
}

ivit_status ivit_layernorm(const int8_t* x, int64_t rows, int32_t cols, const int8_t* gamma,
                           const int32_t* beta, int32_t F, int32_t M_ln, ivit_dyadic out, int8_t* y,
                           ivit_stream_t stream) {
  if (rows < 0 || cols < 16 || cols > 2048 || cols % 16 != 0 || F < 0 || F > 14 || M_ln < F || M_ln > 23 ||
      !valid_dyadic(out))
    return IVIT_ERR_INVALID_ARG;
  if (rows == 0) return IVIT_OK;
  if (!x || !y || !gamma || !beta || !aligned16(x) || !aligned16(y) || !aligned16(gamma) || !aligned16(beta))
    return IVIT_ERR_INVALID_ARG;
  DeviceCtx dc;
  ivit_status st = device_ctx(&dc);
  if (st != IVIT_OK) return st;
  return launch_layernorm(dc, x, rows, cols, gamma, beta, F, M_ln, out, y, (cudaStream_t)stream);
}

size_t ivit_block_workspace_bytes(int32_t B, int32_t N, int32_t D, int32_t Dm) {
  if (B < 0 || N < 0 || D < 0 || Dm < 0) return 0;
  const size_t T = (size_t)B * (size_t)N;
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  // ln (T x D) | qkv (T x 3D) | ctx (T x D) | xh (T x D) | g (T x Dm)
  return up(T * D) + up(T * 3 * (size_t)D) + up(T * D) + up(T * D) + up(T * (size_t)Dm);
}

ivit_status ivit_block_forward(const ivit_block_params* p, const int8_t* x, int8_t* y, void* workspace,
                               size_t workspace_bytes, int32_t B, int32_t N, ivit_stream_t stream) {
  if (!p || !x || !y || !workspace) return IVIT_ERR_INVALID_ARG;
  if (B < 0 || N < 0 || p->H < 1 || p->D != 64 * p->H || p->Dm < 16 || p->Dm % 16 != 0 || p->D > 2048)
    return IVIT_ERR_INVALID_ARG;
  if (x == y) return IVIT_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return IVIT_OK;
  if (N > 640) return IVIT_ERR_UNSUPPORTED;
  const int32_t D = p->D, Dm = p->Dm;
  const size_t need = ivit_block_workspace_bytes(B, N, D, Dm);
  if (workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return IVIT_ERR_INVALID_ARG;
  if (!p->ln1_gamma || !p->ln1_beta || !p->w_qkv || !p->b_qkv || !p->c_qkv || !p->w_o || !p->b_o || !p->c_o ||
      !p->ln2_gamma || !p->ln2_beta || !p->w1 || !p->b1 || !p->c1 || !p->w2 || !p->b2 || !p->c2)
    return IVIT_ERR_INVALID_ARG;
  if (p->k_s < 2 || p->k_s > 16 || !valid_shiftmax(p->attn_I0, p->attn_M, p->attn_k_out) ||
      !valid_shiftmax(p->gelu_I0, p->gelu_M, p->gelu_k_out) || !valid_dyadic(p->logit) ||
      !valid_dyadic(p->attn_out) || !valid_dyadic(p->gelu_out) || !valid_dyadic(p->ln1_out) ||
      !valid_dyadic(p->ln2_out) || !valid_residual(p->res1) || !valid_residual(p->res2) || p->ln_F < 0 ||
      p->ln_F > 14 || p->ln_M < p->ln_F || p->ln_M > 23)
    return IVIT_ERR_INVALID_ARG;
  if (!attention_config_supported(N, p->k_s, p->attn_I0)) return IVIT_ERR_UNSUPPORTED;
  DeviceCtx dc;
  ivit_status st = device_ctx(&dc);
  if (st != IVIT_OK) return st;
  const int64_t T = (int64_t)B * N;
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  int8_t* ws = static_cast<int8_t*>(workspace);
  int8_t* ln = ws;
  int8_t* qkv = ln + up((size_t)T * D);
  int8_t* ctx = qkv + up((size_t)T * 3 * D);
  int8_t* xh = ctx + up((size_t)T * D);
  int8_t* g = xh + up((size_t)T * D);
  cudaStream_t s = (cudaStream_t)stream;
  const ivit_residual none{0, 0, 0};
  // a1 LN1
  if ((st = launch_layernorm(dc, x, T, D, p->ln1_gamma, p->ln1_beta, p->ln_F, p->ln_M, p->ln1_out, ln, s)) != IVIT_OK)
    return st;
  // a2 QKV
  if ((st = launch_gemm(dc, ln, T, D, p->w_qkv, 3 * D, p->bias_qkv, p->b_qkv, p->c_qkv, 8, kEpiPlain, nullptr, none,
                        nullptr, qkv, s)) != IVIT_OK)
    return st;
  // a3-a5 logits, Shiftmax, A V
  if ((st = launch_attention(dc, qkv, B, N, p->H, p->logit, p->k_s, p->attn_I0, p->attn_M, p->attn_k_out,
                             p->attn_out, ctx, s)) != IVIT_OK)
    return st;
  // a6 W^O + residual 1
  if ((st = launch_gemm(dc, ctx, T, D, p->w_o, D, p->bias_o, p->b_o, p->c_o, 8, kEpiResidual, x, p->res1, nullptr,
                        xh, s)) != IVIT_OK)
    return st;
  // a7 LN2
  if ((st = launch_layernorm(dc, xh, T, D, p->ln2_gamma, p->ln2_beta, p->ln_F, p->ln_M, p->ln2_out, ln, s)) !=
      IVIT_OK)
    return st;
  // a8 + a9 fc1 with ShiftGELU in the epilogue
  const GeluParams gp{p->gelu_I0, p->gelu_M, p->gelu_k_out, p->gelu_out};
  if ((st = launch_gemm(dc, ln, T, D, p->w1, Dm, p->bias1, p->b1, p->c1, 8, kEpiGelu, nullptr, none, &gp, g, s)) !=
      IVIT_OK)
    return st;
  // a10 fc2 + residual 2
  return launch_gemm(dc, g, T, Dm, p->w2, D, p->bias2, p->b2, p->c2, 8, kEpiResidual, xh, p->res2, nullptr, y, s);
}

ivit_status ivit_stream_status(ivit_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return IVIT_ERR_CUDA;
  DeviceCtx dc;
  ivit_status st = device_ctx(&dc);
  if (st != IVIT_OK) return st;
  int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_status_word, sizeof(int)) != cudaSuccess) return IVIT_ERR_CUDA;
  if (word != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(int)) != cudaSuccess) return IVIT_ERR_CUDA;
    return IVIT_ERR_TIMEOUT;
  }
  return IVIT_OK;
}

uint64_t ivit_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
