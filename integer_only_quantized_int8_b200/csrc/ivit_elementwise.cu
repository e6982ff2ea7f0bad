// ivit_elementwise.cu -- the HBM-bound operators of the integer ViT block.
//
// ShiftGELU ("I-ViT: Integer-only Quantization for Efficient Vision
// Transformer Inference", section 3.4): the output depends only on the int8
// input and scalar parameters, so each CTA tabulates the 256 possible outputs
// with the integer formula and streams 16-byte vectors through the table.
//
// I-LayerNorm (same page, section 3.5): one warp per row; sums of x and x^2
// with dp4a, exact integer variance, 10 Newton steps of the integer square
// root, then the per-element normalisation, affine and dyadic requant.
#include "ivit_common.cuh"
#include "ivit_internal.h"

namespace ivit {
namespace {

constexpr int kGeluThreads = 256;

__global__ void __launch_bounds__(kGeluThreads)
    shiftgelu_kernel(const int8_t* __restrict__ x, int64_t n, GeluParams g, int8_t* __restrict__ y) {
  __shared__ int8_t tab[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x)
    tab[i] = (int8_t)shiftgelu8(i - 128, g.I0, g.M, g.k_out, g.out.b, g.out.c);
  __syncthreads();
  const int64_t nvec = n >> 4;
  const int4* xv = reinterpret_cast<const int4*>(x);
  int4* yv = reinterpret_cast<int4*>(y);
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nvec; v += (int64_t)gridDim.x * blockDim.x) {
    const int4 in = __ldcs(xv + v);  // streamed once: do not keep in L1
    const uint32_t w[4] = {(uint32_t)in.x, (uint32_t)in.y, (uint32_t)in.z, (uint32_t)in.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t r = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t idx = ((w[k] >> (8 * e)) & 0xFFu) ^ 0x80u;  // int8 -> table index x + 128
        r |= ((uint32_t)(uint8_t)tab[idx]) << (8 * e);
      }
      o[k] = r;
    }
    __stcs(yv + v, make_int4((int)o[0], (int)o[1], (int)o[2], (int)o[3]));
  }
  // ragged tail (n not a multiple of 16)
  if (blockIdx.x == 0) {
    for (int64_t i = (nvec << 4) + threadIdx.x; i < n; i += blockDim.x)
      y[i] = tab[((uint32_t)(uint8_t)x[i]) ^ 0x80u];
  }
}

constexpr int kLnWarps = 8;
constexpr int kLnMaxChunks = 4;  // 16-byte chunks per lane: cols <= 32 * 16 * 4 = 2048

// floor(a / b) for b > 0
__device__ __forceinline__ int64_t floordiv64(int64_t a, int64_t b) {
  int64_t q = a / b;
  if ((a % b) != 0 && a < 0) q -= 1;
  return q;
}

__device__ __forceinline__ int32_t isqrt_newton10(int32_t V) {
  if (V <= 0) return 0;
  const int bits = 32 - __clz(V);
  int32_t I = 1 << (bits >> 1);
#pragma unroll
  for (int it = 0; it < 10; ++it) I = (I + V / I) >> 1;
  return I;
}

__global__ void __launch_bounds__(kLnWarps * 32)
    layernorm_kernel(const int8_t* __restrict__ x, int64_t rows, int32_t cols, const int8_t* __restrict__ gamma,
                     const int32_t* __restrict__ beta, int32_t F, int32_t M_ln, ivit_dyadic out,
                     int8_t* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kLnWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int nchunk = cols >> 4;
  const int8_t* xr = x + row * cols;
  int4 v[kLnMaxChunks];
  int32_t s1 = 0, s2 = 0;
#pragma unroll
  for (int k = 0; k < kLnMaxChunks; ++k) {
    const int ci = lane + 32 * k;
    if (ci < nchunk) {
      v[k] = __ldcs(reinterpret_cast<const int4*>(xr) + ci);
      const int w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        s1 = __dp4a(w[e], 0x01010101, s1);  // sum of four signed bytes
        s2 = __dp4a(w[e], w[e], s2);        // sum of their squares
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    s2 += __shfl_xor_sync(0xffffffffu, s2, o);
  }
  // mu = floor(sum x / n); sum (x - mu)^2 = sum x^2 - 2 mu sum x + n mu^2 (exact)
  const int64_t mu = floordiv64(s1, cols);
  const int64_t sd2 = (int64_t)s2 - 2 * mu * (int64_t)s1 + (int64_t)cols * mu * mu;
  const int32_t V = (int32_t)(sd2 / cols);  // sd2 >= 0: truncation == floor
  int32_t sigma = isqrt_newton10(V);
  if (sigma < 1) sigma = 1;
  const int32_t f = (1 << M_ln) / sigma;
  const int sh = M_ln - F;
  const int32_t m32 = (int32_t)mu;
  int8_t* yr = y + row * cols;
#pragma unroll
  for (int k = 0; k < kLnMaxChunks; ++k) {
    const int ci = lane + 32 * k;
    if (ci < nchunk) {
      const int c0 = ci * 16;
      const int4 gv = __ldg(reinterpret_cast<const int4*>(gamma + c0));
      const int8_t* gb = reinterpret_cast<const int8_t*>(&gv);
      const int8_t* xb = reinterpret_cast<const int8_t*>(&v[k]);
      int32_t bt[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) *reinterpret_cast<int4*>(&bt[4 * q]) = __ldg(reinterpret_cast<const int4*>(beta + c0) + q);
      uint32_t o[4] = {0, 0, 0, 0};
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int32_t d = (int32_t)xb[e] - m32;
        const int32_t nv = (d * f) >> sh;
        const int32_t acc = nv * (int32_t)gb[e] + bt[e];
        o[e >> 2] |= ((uint32_t)requant8(acc, out.b, out.c) & 0xFFu) << (8 * (e & 3));
      }
      __stcs(reinterpret_cast<int4*>(yr) + ci, make_int4((int)o[0], (int)o[1], (int)o[2], (int)o[3]));
    }
  }
}

}  // namespace

ivit_status launch_shiftgelu(const DeviceCtx& dc, const int8_t* x, int64_t n, const GeluParams& g, int8_t* y,
                             cudaStream_t stream) {
  if (n == 0) return IVIT_OK;
  const int64_t nvec = n >> 4;
  int64_t blocks = (nvec + kGeluThreads - 1) / kGeluThreads;
  const int64_t cap = (int64_t)dc.num_sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  shiftgelu_kernel<<<(unsigned)blocks, kGeluThreads, 0, stream>>>(x, n, g, y);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}

ivit_status launch_layernorm(const DeviceCtx& dc, const int8_t* x, int64_t rows, int32_t cols,
                             const int8_t* gamma, const int32_t* beta, int32_t F, int32_t M_ln, ivit_dyadic out,
                             int8_t* y, cudaStream_t stream) {
  (void)dc;
  if (rows == 0) return IVIT_OK;
  const int64_t blocks = (rows + kLnWarps - 1) / kLnWarps;
  if (blocks > 0x7fffffff) return IVIT_ERR_UNSUPPORTED;
  layernorm_kernel<<<(unsigned)blocks, kLnWarps * 32, 0, stream>>>(x, rows, cols, gamma, beta, F, M_ln, out, y);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}

}  // namespace ivit
