// ivit_model.cu -- the data movement on either side of the encoder blocks:
// flattening image patches for the patch-embedding GEMM, assembling the
// tokens (class token, patch embeddings, position embedding), and gathering
// the class tokens for the classifier head.  The patch projection and the
// classifier are int8 linear layers of the I-ViT scheme ("I-ViT: Integer-only
// Quantization for Efficient Vision Transformer Inference", section 3.1) and
// run on the tcgen05 GEMM of ivit_gemm.cu; the position embedding joins the
// tokens through the two-scale dyadic addition of the residual connections
// (section 3.1).  All three kernels are HBM-bound copies of a few MB.
#include <climits>

#include "ivit_common.cuh"
#include "ivit_internal.h"

namespace ivit {
namespace {

constexpr int kMoveThreads = 256;

// Patch rows z [B*Np x C*P*P]: z[(b Np + py gx + px), (ch P + ky) P + kx] =
// img[b, ch, py P + ky, px P + kx].  VEC: 16 consecutive kx at a time (P and
// Wi multiples of 16, so both ends are 16-byte aligned); else one byte.
template <bool VEC>
__global__ void __launch_bounds__(kMoveThreads)
    im2col_kernel(const int8_t* __restrict__ img, int64_t n_units, int32_t C, int32_t Hi, int32_t Wi, int32_t P,
                  int32_t gx, int32_t Np, int8_t* __restrict__ z) {
  pdl_wait();  // the image may come from an earlier kernel
  pdl_launch_dependents();
  const int32_t K = C * P * P;
  const int32_t w = VEC ? 16 : 1;  // bytes per unit
  const int32_t upr = K / w;       // units per patch row
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < n_units; u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = u / upr;
    const int32_t k = (int32_t)(u - row * upr) * w;
    const int64_t b = row / Np;
    const int32_t p = (int32_t)(row - b * Np);
    const int32_t py = p / gx, px = p - (p / gx) * gx;
    const int32_t ch = k / (P * P);
    const int32_t rem = k - ch * P * P;
    const int32_t ky = rem / P, kx = rem - (rem / P) * P;
    const int64_t src = ((b * C + ch) * Hi + (int64_t)py * P + ky) * Wi + (int64_t)px * P + kx;
    if (VEC)
      *reinterpret_cast<int4*>(z + row * K + k) = __ldg(reinterpret_cast<const int4*>(img + src));
    else
      z[row * K + k] = img[src];
  }
}

// sat_8((b_u u + b_v v) >> c) on the 16 bytes of two vectors
IVIT_DEV int4 add2_vec(int4 uv, int4 vv, const ivit_residual& r) {
  const uint32_t uw[4] = {(uint32_t)uv.x, (uint32_t)uv.y, (uint32_t)uv.z, (uint32_t)uv.w};
  const uint32_t vw[4] = {(uint32_t)vv.x, (uint32_t)vv.y, (uint32_t)vv.z, (uint32_t)vv.w};
  uint32_t o[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int64_t u = (int8_t)(uw[q] >> (8 * e));
      const int64_t v = (int8_t)(vw[q] >> (8 * e));
      int64_t t = ((int64_t)r.b_skip * u + (int64_t)r.b_branch * v) >> r.c;  // arithmetic: floor
      t = t < -128 ? -128 : (t > 127 ? 127 : t);
      word |= ((uint32_t)t & 0xffu) << (8 * e);
    }
    o[q] = word;
  }
  return make_int4((int)o[0], (int)o[1], (int)o[2], (int)o[3]);
}

// x [B*(Np+1) x D]: row 0 of each image from the class token, rows 1.. from
// the patch embeddings e [B*Np x D], each joined to its position-embedding
// row by the two-scale dyadic addition.  One 16-byte vector per unit.
__global__ void __launch_bounds__(kMoveThreads)
    tokens_kernel(const int8_t* __restrict__ e, const int8_t* __restrict__ cls, const int8_t* __restrict__ pos,
                  ivit_residual add, int64_t n_units, int32_t Np, int32_t D, int8_t* __restrict__ x) {
  pdl_wait();  // the embeddings come from the patch GEMM
  pdl_launch_dependents();
  const int32_t vpr = D / 16;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < n_units; u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = u / vpr;
    const int32_t j = (int32_t)(u - row * vpr) * 16;
    const int64_t b = row / (Np + 1);
    const int32_t t = (int32_t)(row - b * (Np + 1));
    const int8_t* src = t == 0 ? cls + j : e + ((b * Np + t - 1) * D + j);
    const int4 uv = __ldg(reinterpret_cast<const int4*>(src));
    const int4 vv = __ldg(reinterpret_cast<const int4*>(pos + (int64_t)t * D + j));
    *reinterpret_cast<int4*>(x + row * D + j) = add2_vec(uv, vv, add);
  }
}

// t [B x D] = row 0 of each image's Ntok rows of x.
__global__ void __launch_bounds__(kMoveThreads)
    gather_rows_kernel(const int8_t* __restrict__ x, int64_t n_units, int32_t Ntok, int32_t D,
                       int8_t* __restrict__ t) {
  pdl_wait();  // x comes from the last block
  pdl_launch_dependents();
  const int32_t vpr = D / 16;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < n_units; u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t b = u / vpr;
    const int32_t j = (int32_t)(u - b * vpr) * 16;
    *reinterpret_cast<int4*>(t + b * D + j) = __ldg(reinterpret_cast<const int4*>(x + b * Ntok * D + j));
  }
}

unsigned move_grid(const DeviceCtx& dc, int64_t n_units) {
  int64_t blocks = (n_units + kMoveThreads - 1) / kMoveThreads;
  const int64_t cap = (int64_t)dc.num_sms * 8;
  if (blocks > cap) blocks = cap;
  return (unsigned)(blocks < 1 ? 1 : blocks);
}

}  // namespace

ivit_status launch_im2col(const DeviceCtx& dc, const int8_t* img, int32_t B, int32_t C, int32_t Hi, int32_t Wi,
                          int32_t P, int8_t* z, cudaStream_t stream) {
  const int32_t gx = Wi / P, Np = (Hi / P) * gx;
  const int64_t rows = (int64_t)B * Np;
  if (rows == 0) return IVIT_OK;
  const bool vec = P % 16 == 0 && Wi % 16 == 0;
  const int64_t n_units = rows * (int64_t)C * P * P / (vec ? 16 : 1);
  const cudaError_t e =
      vec ? launch_pdl(im2col_kernel<true>, dim3(move_grid(dc, n_units)), dim3(kMoveThreads), 0, stream, img,
                       n_units, C, Hi, Wi, P, gx, Np, z)
          : launch_pdl(im2col_kernel<false>, dim3(move_grid(dc, n_units)), dim3(kMoveThreads), 0, stream, img,
                       n_units, C, Hi, Wi, P, gx, Np, z);
  note_launch();
  return e == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}

ivit_status launch_tokens(const DeviceCtx& dc, const int8_t* e, const int8_t* cls, const int8_t* pos,
                          ivit_residual add, int32_t B, int32_t Np, int32_t D, int8_t* x, cudaStream_t stream) {
  const int64_t n_units = (int64_t)B * (Np + 1) * (D / 16);
  if (n_units == 0) return IVIT_OK;
  const cudaError_t err = launch_pdl(tokens_kernel, dim3(move_grid(dc, n_units)), dim3(kMoveThreads), 0, stream, e,
                                     cls, pos, add, n_units, Np, D, x);
  note_launch();
  return err == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}

ivit_status launch_gather_rows(const DeviceCtx& dc, const int8_t* x, int32_t B, int32_t Ntok, int32_t D, int8_t* t,
                               cudaStream_t stream) {
  const int64_t n_units = (int64_t)B * (D / 16);
  if (n_units == 0) return IVIT_OK;
  const cudaError_t err = launch_pdl(gather_rows_kernel, dim3(move_grid(dc, n_units)), dim3(kMoveThreads), 0, stream,
                                     x, n_units, Ntok, D, t);
  note_launch();
  return err == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}

}  // namespace ivit
