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
                                int32_t rounding, const int8_t* skip, ivit_residual res, int8_t* Y,
                                ivit_stream_t stream) {
  if (!X || !W || !b || !c || !Y || (rounding != 0 && rounding != 1)) return IVIT_ERR_INVALID_ARG;
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
  return launch_gemm(dc, X, M, K, W, N, bias, b, c, out_bits, rounding != 0, skip ? kEpiResidual : kEpiPlain, skip,
                     res, nullptr, Y,
                     (cudaStream_t)stream);
}

ivit_status ivit_linear_shiftgelu(const int8_t* X, int64_t M, int32_t K, const int8_t* W, int32_t N,
                                  const int32_t* bias, const int32_t* b, const int8_t* c, int32_t rounding,
                                  int32_t gelu_I0, int32_t gelu_M, int32_t gelu_k_out, ivit_dyadic gelu_out,
                                  int8_t* Y, ivit_stream_t stream) {
  if (!X || !W || !b || !c || !Y || (rounding != 0 && rounding != 1)) return IVIT_ERR_INVALID_ARG;
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
  return launch_gemm(dc, X, M, K, W, N, bias, b, c, 8, rounding != 0, kEpiGelu, nullptr, ivit_residual{0, 0, 0}, &gp,
                     Y,
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

ivit_status ivit_shiftgelu_rowmax(const int8_t* x, int64_t rows, int32_t cols, int32_t I0, int32_t M,
                                  int32_t k_out, ivit_dyadic out, int8_t* y, ivit_stream_t stream) {
  if (rows < 0 || cols < 16 || cols > 16384 || cols % 16 != 0 || !valid_shiftmax(I0, M, k_out) ||
      !valid_dyadic(out))
    return IVIT_ERR_INVALID_ARG;
  if (rows == 0) return IVIT_OK;
  if (!x || !y || !aligned16(x) || !aligned16(y)) return IVIT_ERR_INVALID_ARG;
  DeviceCtx dc;
  ivit_status st = device_ctx(&dc);
  if (st != IVIT_OK) return st;
  const GeluParams g{I0, M, k_out, out};
  return launch_shiftgelu_rowmax(dc, x, rows, cols, g, y, (cudaStream_t)stream);
}

ivit_status ivit_attention_lis(const int8_t* qkv, int32_t B, int32_t N, int32_t H, ivit_dyadic logit, int32_t k_s,
                               int32_t I0, int32_t M, ivit_dyadic out, int8_t* ctx, ivit_stream_t stream) {
  if (!qkv || !ctx || !aligned16(qkv) || !aligned16(ctx)) return IVIT_ERR_INVALID_ARG;
  if (B < 0 || N < 0 || H < 1 || k_s < 2 || k_s > 8 || I0 < 1 || I0 > (1 << 22) || M < 15 || M > 30 ||
      !valid_dyadic(logit) || !valid_dyadic(out))
    return IVIT_ERR_INVALID_ARG;
  if (N > 640 || (int64_t)B * N > 0x7fffff00LL || H > 4096) return IVIT_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return IVIT_OK;
  DeviceCtx dc;
  ivit_status st = device_ctx(&dc);
  if (st != IVIT_OK) return st;
  return launch_attention(dc, qkv, B, N, H, logit, k_s, I0, M, 8, out, ctx, (cudaStream_t)stream, true);
}

ivit_status ivit_layernorm_ptf(const int8_t* x, int64_t rows, int32_t cols, const uint8_t* alpha,
                               const int8_t* gamma, const int32_t* beta, int32_t F, int32_t M_ln, ivit_dyadic out,
                               int8_t* y, ivit_stream_t stream) {
  if (rows < 0 || cols < 16 || cols > 2048 || cols % 16 != 0 || F < 0 || F > 14 || M_ln < F || M_ln > 20 ||
      !valid_dyadic(out))
    return IVIT_ERR_INVALID_ARG;
  if (rows == 0) return IVIT_OK;
  if (!x || !y || !alpha || !gamma || !beta || !aligned16(x) || !aligned16(y) || !aligned16(alpha) ||
      !aligned16(gamma) || !aligned16(beta))
    return IVIT_ERR_INVALID_ARG;
  DeviceCtx dc;
  ivit_status st = device_ctx(&dc);
  if (st != IVIT_OK) return st;
  return launch_layernorm_ptf(dc, x, rows, cols, alpha, gamma, beta, F, M_ln, out, y, (cudaStream_t)stream);
}

size_t ivit_block_workspace_bytes(int32_t B, int32_t N, int32_t D, int32_t Dm) {
  if (B < 0 || N < 0 || D < 0 || Dm < 0) return 0;
  const size_t T = (size_t)B * (size_t)N;
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  // ln (T x D) | qkv (T x 3D) | ctx (T x D) | xh (T x D) | g (T x Dm)
  return up(T * D) + up(T * 3 * (size_t)D) + up(T * D) + up(T * D) + up(T * (size_t)Dm);
}

}  // extern "C"

// Every host-side check of one block call except those of the workspace;
// IVIT_OK means the arguments may be enqueued (or, with B or N zero, that
// there is nothing to do).
ivit_status ivit::check_block_args(const ivit_block_params* p, const int8_t* x, const int8_t* y, int32_t B,
                                   int32_t N) {
  if (!p || !x || !y) return IVIT_ERR_INVALID_ARG;
  if (B < 0 || N < 0 || p->H < 1 || p->D != 64 * p->H || p->Dm < 16 || p->Dm % 16 != 0 || p->D > 2048)
    return IVIT_ERR_INVALID_ARG;
  if (x == y) return IVIT_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return IVIT_OK;
  if (N > 640) return IVIT_ERR_UNSUPPORTED;
  if (!p->ln1_gamma || !p->ln1_beta || !p->w_qkv || !p->b_qkv || !p->c_qkv || !p->w_o || !p->b_o || !p->c_o ||
      !p->ln2_gamma || !p->ln2_beta || !p->w1 || !p->b1 || !p->c1 || !p->w2 || !p->b2 || !p->c2)
    return IVIT_ERR_INVALID_ARG;
  if (p->k_s < 2 || p->k_s > 16 || !valid_shiftmax(p->attn_I0, p->attn_M, p->attn_k_out) ||
      !valid_shiftmax(p->gelu_I0, p->gelu_M, p->gelu_k_out) || !valid_dyadic(p->logit) ||
      !valid_dyadic(p->attn_out) || !valid_dyadic(p->gelu_out) || !valid_dyadic(p->ln1_out) ||
      !valid_dyadic(p->ln2_out) || !valid_residual(p->res1) || !valid_residual(p->res2) || p->ln_F < 0 ||
      p->ln_F > 14 || p->ln_M < p->ln_F || p->ln_M > 23 || (p->linear_round != 0 && p->linear_round != 1))
    return IVIT_ERR_INVALID_ARG;
  // the kernels read and write all of these by 16-byte vector accesses or TMA
  const void* const need16[] = {x,         y,        p->ln1_gamma, p->ln1_beta, p->w_qkv, p->b_qkv,
                                p->c_qkv,  p->w_o,   p->b_o,       p->c_o,      p->ln2_gamma, p->ln2_beta,
                                p->w1,     p->b1,    p->c1,        p->w2,       p->b2,    p->c2};
  for (const void* q : need16)
    if (!aligned16(q)) return IVIT_ERR_INVALID_ARG;
  const void* const bias16[] = {p->bias_qkv, p->bias_o, p->bias1, p->bias2};  // optional
  for (const void* q : bias16)
    if (q && !aligned16(q)) return IVIT_ERR_INVALID_ARG;
  if (!attention_config_supported(N, p->k_s, p->attn_I0)) return IVIT_ERR_UNSUPPORTED;
  return IVIT_OK;
}

extern "C" {

namespace {

// Every host-side check of one block call; IVIT_OK means it may be enqueued
// (or, with B or N zero, that there is nothing to do).
ivit_status check_block(const ivit_block_params* p, const int8_t* x, const int8_t* y, const void* workspace,
                        size_t workspace_bytes, int32_t B, int32_t N) {
  if (!workspace) return IVIT_ERR_INVALID_ARG;
  const ivit_status st = check_block_args(p, x, y, B, N);
  if (st != IVIT_OK || B == 0 || N == 0) return st;
  const size_t need = ivit_block_workspace_bytes(B, N, p->D, p->Dm);
  if (workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return IVIT_ERR_INVALID_ARG;
  return IVIT_OK;
}

// Enqueues one checked block (B, N > 0).
ivit_status enqueue_block(const DeviceCtx& dc, const ivit_block_params* p, const int8_t* x, int8_t* y,
                          void* workspace, int32_t B, int32_t N, cudaStream_t s) {
  const int32_t D = p->D, Dm = p->Dm;
  const int64_t T = (int64_t)B * N;
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  int8_t* ws = static_cast<int8_t*>(workspace);
  int8_t* ln = ws;
  int8_t* qkv = ln + up((size_t)T * D);
  int8_t* ctx = qkv + up((size_t)T * 3 * D);
  int8_t* xh = ctx + up((size_t)T * D);
  int8_t* g = xh + up((size_t)T * D);
  const ivit_residual none{0, 0, 0};
  ivit_status st;
  // a1 LN1
  if ((st = launch_layernorm(dc, x, T, D, p->ln1_gamma, p->ln1_beta, p->ln_F, p->ln_M, p->ln1_out, ln, s)) != IVIT_OK)
    return st;
  // a2 QKV
  const bool rnd = p->linear_round != 0;
  if ((st = launch_gemm(dc, ln, T, D, p->w_qkv, 3 * D, p->bias_qkv, p->b_qkv, p->c_qkv, 8, rnd, kEpiPlain, nullptr, none,
                        nullptr, qkv, s)) != IVIT_OK)
    return st;
  // a3-a5 logits, Shiftmax, A V
  if ((st = launch_attention(dc, qkv, B, N, p->H, p->logit, p->k_s, p->attn_I0, p->attn_M, p->attn_k_out,
                             p->attn_out, ctx, s)) != IVIT_OK)
    return st;
  // a6 W^O + residual 1
  if ((st = launch_gemm(dc, ctx, T, D, p->w_o, D, p->bias_o, p->b_o, p->c_o, 8, rnd, kEpiResidual, x, p->res1, nullptr,
                        xh, s)) != IVIT_OK)
    return st;
  // a7 LN2
  if ((st = launch_layernorm(dc, xh, T, D, p->ln2_gamma, p->ln2_beta, p->ln_F, p->ln_M, p->ln2_out, ln, s)) !=
      IVIT_OK)
    return st;
  // a8 + a9 fc1 with ShiftGELU in the epilogue
  const GeluParams gp{p->gelu_I0, p->gelu_M, p->gelu_k_out, p->gelu_out};
  if ((st = launch_gemm(dc, ln, T, D, p->w1, Dm, p->bias1, p->b1, p->c1, 8, rnd, kEpiGelu, nullptr, none, &gp, g, s)) !=
      IVIT_OK)
    return st;
  // a10 fc2 + residual 2
  return launch_gemm(dc, g, T, Dm, p->w2, D, p->bias2, p->b2, p->c2, 8, rnd, kEpiResidual, xh, p->res2, nullptr, y,
                     s);
}

}  // namespace

ivit_status ivit_block_forward(const ivit_block_params* p, const int8_t* x, int8_t* y, void* workspace,
                               size_t workspace_bytes, int32_t B, int32_t N, ivit_stream_t stream) {
  ivit_status st = check_block(p, x, y, workspace, workspace_bytes, B, N);
  if (st != IVIT_OK || B == 0 || N == 0) return st;
  DeviceCtx dc;
  if ((st = device_ctx(&dc)) != IVIT_OK) return st;
  return enqueue_block(dc, p, x, y, workspace, B, N, (cudaStream_t)stream);
}

// ---------------------------------------------------------------------------
// steps either side of the blocks
// ---------------------------------------------------------------------------

size_t ivit_patch_embed_workspace_bytes(int32_t B, int32_t C, int32_t Hi, int32_t Wi, int32_t P, int32_t D) {
  if (B < 0 || C < 1 || P < 1 || Hi < P || Wi < P || D < 0) return 0;
  const size_t rows = (size_t)B * (size_t)(Hi / P) * (size_t)(Wi / P);
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  // patch rows (rows x C P P) | embeddings (rows x D)
  return up(rows * (size_t)C * P * P) + up(rows * (size_t)D);
}

size_t ivit_head_workspace_bytes(int32_t B, int32_t D) {
  if (B < 0 || D < 0) return 0;
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  // class tokens | their normalised copy
  return 2 * up((size_t)B * (size_t)D);
}

namespace {

ivit_status check_patch_embed(const int8_t* img, int32_t B, int32_t C, int32_t Hi, int32_t Wi, int32_t P,
                              const int8_t* W, int32_t D, const int32_t* bias, const int32_t* b, const int8_t* c,
                              int32_t rounding, const int8_t* cls, const int8_t* pos, ivit_residual pos_add, const void* workspace,
                              size_t workspace_bytes, const int8_t* x) {
  if (!img || !W || !b || !c || !cls || !pos || !x || !workspace || (rounding != 0 && rounding != 1))
    return IVIT_ERR_INVALID_ARG;
  if (!aligned16(img) || !aligned16(W) || !aligned16(b) || !aligned16(c) || !aligned16(cls) || !aligned16(pos) ||
      !aligned16(x) || (bias && !aligned16(bias)) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return IVIT_ERR_INVALID_ARG;
  if (B < 0 || C < 1 || P < 1 || Hi < P || Wi < P || Hi % P != 0 || Wi % P != 0 || D < 16 || D % 16 != 0 ||
      !valid_residual(pos_add))
    return IVIT_ERR_INVALID_ARG;
  const int64_t K = (int64_t)C * P * P;
  if (K < 16 || K % 16 != 0) return IVIT_ERR_INVALID_ARG;
  const int64_t rows = (int64_t)B * (Hi / P) * (Wi / P);
  if (K > 16384 || D > 16384 || rows + B > 0x7fffff00LL) return IVIT_ERR_UNSUPPORTED;
  if (workspace_bytes < ivit_patch_embed_workspace_bytes(B, C, Hi, Wi, P, D)) return IVIT_ERR_INVALID_ARG;
  return IVIT_OK;
}

ivit_status enqueue_patch_embed(const DeviceCtx& dc, const int8_t* img, int32_t B, int32_t C, int32_t Hi,
                                int32_t Wi, int32_t P, const int8_t* W, int32_t D, const int32_t* bias,
                                const int32_t* b, const int8_t* c, bool round, const int8_t* cls, const int8_t* pos,
                                ivit_residual pos_add, void* workspace, int8_t* x, cudaStream_t s) {
  const int32_t Np = (Hi / P) * (Wi / P), K = C * P * P;
  const int64_t rows = (int64_t)B * Np;
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  int8_t* z = static_cast<int8_t*>(workspace);
  int8_t* e = z + up((size_t)rows * K);
  ivit_status st;
  if ((st = launch_im2col(dc, img, B, C, Hi, Wi, P, z, s)) != IVIT_OK) return st;
  if ((st = launch_gemm(dc, z, rows, K, W, D, bias, b, c, 8, round, kEpiPlain, nullptr, ivit_residual{0, 0, 0}, nullptr, e,
                        s)) != IVIT_OK)
    return st;
  return launch_tokens(dc, e, cls, pos, pos_add, B, Np, D, x, s);
}

ivit_status check_head(const int8_t* x, int32_t B, int32_t Ntok, int32_t D, const int8_t* gamma,
                       const int32_t* beta, int32_t F, int32_t M_ln, ivit_dyadic ln_out, const int8_t* W,
                       int32_t Ncls, const int32_t* bias, const int32_t* b, const int8_t* c, int32_t rounding,
                       const void* workspace, size_t workspace_bytes, const int8_t* logits) {
  if (!x || !gamma || !beta || !W || !b || !c || !logits || !workspace || (rounding != 0 && rounding != 1))
    return IVIT_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(beta) || !aligned16(W) || !aligned16(b) || !aligned16(c) ||
      !aligned16(logits) || (bias && !aligned16(bias)) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return IVIT_ERR_INVALID_ARG;
  if (B < 0 || Ntok < 1 || D < 16 || D > 2048 || D % 16 != 0 || Ncls < 16 || Ncls % 16 != 0 || F < 0 || F > 14 ||
      M_ln < F || M_ln > 23 || !valid_dyadic(ln_out))
    return IVIT_ERR_INVALID_ARG;
  if ((int64_t)B * Ntok > 0x7fffff00LL) return IVIT_ERR_UNSUPPORTED;
  if (workspace_bytes < ivit_head_workspace_bytes(B, D)) return IVIT_ERR_INVALID_ARG;
  return IVIT_OK;
}

ivit_status enqueue_head(const DeviceCtx& dc, const int8_t* x, int32_t B, int32_t Ntok, int32_t D,
                         const int8_t* gamma, const int32_t* beta, int32_t F, int32_t M_ln, ivit_dyadic ln_out,
                         const int8_t* W, int32_t Ncls, const int32_t* bias, const int32_t* b, const int8_t* c,
                         bool round, void* workspace, int8_t* logits, cudaStream_t s) {
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  int8_t* t = static_cast<int8_t*>(workspace);
  int8_t* n = t + up((size_t)B * D);
  ivit_status st;
  if ((st = launch_gather_rows(dc, x, B, Ntok, D, t, s)) != IVIT_OK) return st;
  if ((st = launch_layernorm(dc, t, B, D, gamma, beta, F, M_ln, ln_out, n, s)) != IVIT_OK) return st;
  return launch_gemm(dc, n, B, D, W, Ncls, bias, b, c, 8, round, kEpiPlain, nullptr, ivit_residual{0, 0, 0}, nullptr,
                     logits,
                     s);
}

}  // namespace

ivit_status ivit_patch_embed(const int8_t* img, int32_t B, int32_t C, int32_t Hi, int32_t Wi, int32_t P,
                             const int8_t* W, int32_t D, const int32_t* bias, const int32_t* b, const int8_t* c,
                             int32_t rounding, const int8_t* cls, const int8_t* pos, ivit_residual pos_add,
                             void* workspace, size_t workspace_bytes, int8_t* x, ivit_stream_t stream) {
  ivit_status st = check_patch_embed(img, B, C, Hi, Wi, P, W, D, bias, b, c, rounding, cls, pos, pos_add, workspace,
                                     workspace_bytes, x);
  if (st != IVIT_OK || B == 0) return st;
  DeviceCtx dc;
  if ((st = device_ctx(&dc)) != IVIT_OK) return st;
  return enqueue_patch_embed(dc, img, B, C, Hi, Wi, P, W, D, bias, b, c, rounding != 0, cls, pos, pos_add,
                             workspace, x, (cudaStream_t)stream);
}

ivit_status ivit_head(const int8_t* x, int32_t B, int32_t Ntok, int32_t D, const int8_t* gamma, const int32_t* beta,
                      int32_t F, int32_t M_ln, ivit_dyadic ln_out, const int8_t* W, int32_t Ncls,
                      const int32_t* bias, const int32_t* b, const int8_t* c, int32_t rounding, void* workspace,
                      size_t workspace_bytes, int8_t* logits, ivit_stream_t stream) {
  ivit_status st = check_head(x, B, Ntok, D, gamma, beta, F, M_ln, ln_out, W, Ncls, bias, b, c, rounding, workspace,
                              workspace_bytes, logits);
  if (st != IVIT_OK || B == 0) return st;
  DeviceCtx dc;
  if ((st = device_ctx(&dc)) != IVIT_OK) return st;
  return enqueue_head(dc, x, B, Ntok, D, gamma, beta, F, M_ln, ln_out, W, Ncls, bias, b, c, rounding != 0, workspace,
                      logits, (cudaStream_t)stream);
}

size_t ivit_model_workspace_bytes(const ivit_model_params* m, int32_t B, int32_t Hi, int32_t Wi) {
  if (!m || B < 0 || m->P < 1 || Hi < m->P || Wi < m->P || m->D < 0 || m->n_blocks < 0) return 0;
  if (m->n_blocks > 0 && !m->blocks) return 0;
  const int32_t Ntok = (Hi / m->P) * (Wi / m->P) + 1;
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  size_t scratch = ivit_patch_embed_workspace_bytes(B, m->C, Hi, Wi, m->P, m->D);
  for (int32_t i = 0; i < m->n_blocks; ++i) {
    const size_t w = ivit_block_workspace_bytes(B, Ntok, m->blocks[i].D, m->blocks[i].Dm);
    if (w > scratch) scratch = w;
  }
  const size_t hw = ivit_head_workspace_bytes(B, m->D);
  if (hw > scratch) scratch = hw;
  // two token buffers, then the scratch of whichever step runs
  return 2 * up((size_t)B * Ntok * m->D) + scratch;
}

ivit_status ivit_model_forward(const ivit_model_params* m, const int8_t* img, int32_t B, int32_t Hi, int32_t Wi,
                               void* workspace, size_t workspace_bytes, int8_t* logits, ivit_stream_t stream) {
  if (!m || !img || !logits || !workspace || m->n_blocks < 0 || (m->n_blocks > 0 && !m->blocks))
    return IVIT_ERR_INVALID_ARG;
  if (B < 0 || m->P < 1 || Hi < m->P || Wi < m->P || m->D < 16) return IVIT_ERR_INVALID_ARG;
  const size_t need = ivit_model_workspace_bytes(m, B, Hi, Wi);
  if (need == 0 || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return IVIT_ERR_INVALID_ARG;
  const int32_t Ntok = (Hi / m->P) * (Wi / m->P) + 1;
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  int8_t* tok[2];
  tok[0] = static_cast<int8_t*>(workspace);
  tok[1] = tok[0] + up((size_t)B * Ntok * m->D);
  void* scratch = tok[1] + up((size_t)B * Ntok * m->D);
  const size_t scratch_bytes = workspace_bytes - 2 * up((size_t)B * Ntok * m->D);
  // every step is checked before anything is enqueued
  ivit_status st = check_patch_embed(img, B, m->C, Hi, Wi, m->P, m->w_pe, m->D, m->bias_pe, m->b_pe, m->c_pe,
                                     m->linear_round, m->cls, m->pos, m->pos_add, scratch, scratch_bytes, tok[0]);
  if (st != IVIT_OK) return st;
  for (int32_t i = 0; i < m->n_blocks; ++i) {
    if (m->blocks[i].D != m->D) return IVIT_ERR_INVALID_ARG;
    if ((st = check_block(&m->blocks[i], tok[i & 1], tok[(i + 1) & 1], scratch, scratch_bytes, B, Ntok)) != IVIT_OK)
      return st;
  }
  if ((st = check_head(tok[m->n_blocks & 1], B, Ntok, m->D, m->head_gamma, m->head_beta, m->head_ln_F, m->head_ln_M,
                       m->head_ln_out, m->w_head, m->Ncls, m->bias_head, m->b_head, m->c_head, m->linear_round,
                       scratch, scratch_bytes, logits)) != IVIT_OK)
    return st;
  if (B == 0) return IVIT_OK;
  DeviceCtx dc;
  if ((st = device_ctx(&dc)) != IVIT_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if ((st = enqueue_patch_embed(dc, img, B, m->C, Hi, Wi, m->P, m->w_pe, m->D, m->bias_pe, m->b_pe, m->c_pe,
                                m->linear_round != 0, m->cls, m->pos, m->pos_add, scratch, tok[0], s)) != IVIT_OK)
    return st;
  for (int32_t i = 0; i < m->n_blocks; ++i)
    if ((st = enqueue_block(dc, &m->blocks[i], tok[i & 1], tok[(i + 1) & 1], scratch, B, Ntok, s)) != IVIT_OK)
      return st;
  return enqueue_head(dc, tok[m->n_blocks & 1], B, Ntok, m->D, m->head_gamma, m->head_beta, m->head_ln_F,
                      m->head_ln_M, m->head_ln_out, m->w_head, m->Ncls, m->bias_head, m->b_head, m->c_head,
                      m->linear_round != 0, scratch, logits, s);
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
