// ivit_elementwise.cu -- the HBM-bound operators of the integer ViT block.
//
// ShiftGELU ("I-ViT: Integer-only Quantization for Efficient Vision
// Transformer Inference", section 3.4): the output depends only on the int8
// input and scalar parameters, so each CTA tabulates the 256 possible outputs
// with the integer formula and streams 16-byte vectors through the table.
//
// I-LayerNorm (same page, section 3.5): one half-warp per row, so a whole
// activation tensor is in flight in one wave; gamma and beta staged in shared
// memory; sums of x and x^2 with dp4a, exact integer variance, 10 Newton steps
// of the integer square root, then the per-element normalisation, affine and
// dyadic requant.
#include <climits>
#include <cmath>

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
  pdl_wait();  // x comes from an earlier kernel
  pdl_launch_dependents();
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

constexpr int kLnThreads = 256;  // 16 half-warps: one row each

// floor(a / d) for 0 <= a < 2^30, d >= 1 and a quotient below 2^22.  Each of
// the conversions of a, the reciprocal of d and the product rounds with a
// relative error of at most 2^-24, so the fp32 quotient is within
// 3.01 * 2^-24 * 2^22 < 1 of a / d: its floor is the true quotient or off by
// one, and one integer correction in each direction settles it.
__device__ __forceinline__ int32_t udiv_fast(int32_t a, int32_t d) {
  int32_t q = (int32_t)((float)a * __frcp_rn((float)d));
  const int32_t r = a - q * d;
  if (r < 0) q -= 1;
  else if (r >= d) q += 1;
  return q;
}

// Integer square root by exactly 10 Newton steps I <- (I + floor(V / I)) / 2
// from I_0 = 2^floor(bits(V) / 2) (I-ViT section 3.5).
__host__ __device__ constexpr int32_t isqrt_newton10_exact(int32_t V) {
  if (V <= 0) return 0;
  int bits = 0;
  for (int32_t x = V; x; x >>= 1) ++bits;
  int32_t I = 1 << (bits >> 1);
  for (int it = 0; it < 10; ++it) I = (I + V / I) >> 1;
  return I;
}

// floor(sqrt(V)) by bisection, for the compile-time check below.
__host__ __device__ constexpr int32_t isqrt_floor_exact(int32_t V) {
  int32_t lo = 0, hi = 46341;  // hi^2 > INT32_MAX
  while (hi - lo > 1) {
    const int32_t m = (lo + hi) / 2;
    if ((int64_t)m * m <= V) lo = m; else hi = m;
  }
  return lo;
}

// The variance of int8 values is at most 127.5^2 < 16384.  Over that range the
// 10-step root equals floor(sqrt(V)) except at some V = s^2 - 1, where the
// iteration, which alternates between s - 1 and s there, stops on s.  Those s
// (all <= 128) are marked in a bit mask built at compile time from the
// iteration itself, and the whole range is checked against root-plus-mask.
constexpr int kIsqrtRange = 16384;
struct IsqrtMask {
  uint32_t w[5];  // bit s: the 10-step root of s^2 - 1 is s
};
__host__ __device__ constexpr IsqrtMask make_isqrt_mask() {
  IsqrtMask m{};
  for (int s = 1; s * s - 1 < kIsqrtRange; ++s)
    if (isqrt_newton10_exact(s * s - 1) == s) m.w[s >> 5] |= 1u << (s & 31);
  return m;
}
constexpr IsqrtMask kIsqrtMask = make_isqrt_mask();
__host__ __device__ constexpr bool isqrt_mask_matches() {
  for (int32_t V = 0; V < kIsqrtRange; ++V) {
    const int32_t r = isqrt_floor_exact(V), s = r + 1;
    const bool up = V + 1 == s * s && ((kIsqrtMask.w[s >> 5] >> (s & 31)) & 1u);
    if (isqrt_newton10_exact(V) != r + (up ? 1 : 0)) return false;
  }
  return true;
}
static_assert(isqrt_mask_matches(), "10-step root = floor(sqrt) + mask over int8 variances");

__device__ __forceinline__ int32_t isqrt_newton10(int32_t V) {
  if (V >= kIsqrtRange) return isqrt_newton10_exact(V);
  // V < 2^22: the correctly rounded single-precision root of an integer V never
  // rounds up to the next integer, so truncation gives floor(sqrt(V))
  const int32_t r = (int32_t)__fsqrt_rn((float)V), s = r + 1;  // s <= 128
  constexpr uint32_t m0 = kIsqrtMask.w[0], m1 = kIsqrtMask.w[1], m2 = kIsqrtMask.w[2], m3 = kIsqrtMask.w[3],
                     m4 = kIsqrtMask.w[4];
  const int wi = s >> 5;
  const uint32_t word = wi == 0 ? m0 : wi == 1 ? m1 : wi == 2 ? m2 : wi == 3 ? m3 : m4;
  return (V + 1 == s * s && ((word >> (s & 31)) & 1u)) ? s : r;
}

// Saturation bounds of the output requant sat_8((b acc) >> c): clamping acc to
// [lo, hi] keeps every unsaturated result and the direction of the others,
// and keeps (b acc) >> c inside int32.
__device__ __forceinline__ void out_bounds(int32_t b, int32_t c, int32_t& lo, int32_t& hi) {
  if (b == 0) {
    lo = INT_MIN;
    hi = INT_MAX;
    return;
  }
  const int64_t p2 = (int64_t)1 << c;
  const int64_t vhi = (127 * p2 + b - 1) / b;       // first acc with result >= 127
  const int64_t num = -127 * p2 - 1;                 // results <= -128: b acc <= num
  const int64_t vlo = -((-num + b - 1) / b);
  hi = (int32_t)(vhi > INT_MAX ? INT_MAX : vhi);
  lo = (int32_t)(vlo < INT_MIN ? INT_MIN : vlo);
}

__device__ __forceinline__ uint32_t pack_sat4_ln(int32_t y0, int32_t y1, int32_t y2, int32_t y3) {
  uint32_t t, d;
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(t) : "r"(y3), "r"(y2), "r"(0u));
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(y1), "r"(y0), "r"(t));
  return d;
}

// byte i of w, sign-extended (prmt in sign-replicate mode)
__device__ __forceinline__ int32_t sext_byte(uint32_t w, int i) {
  int32_t r;
  const uint32_t sel = (uint32_t)i | ((uint32_t)(8 | i) << 4) | ((uint32_t)(8 | i) << 8) | ((uint32_t)(8 | i) << 12);
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(w), "r"(sel));
  return r;
}

// I-LayerNorm with gamma and beta staged in shared memory: LPR lanes per row,
// lane l of a row holding its 16-byte chunks l, l + LPR, ... (at most CPL).
// gamma (sign-extended to 32 bits) and beta are parameters, not outputs of an
// earlier kernel, so every CTA stages them before the dependent-launch wait,
// while the previous kernel of the stream finishes.  Sums of x and x^2 come
// from dp4a; the mean and variance divisions and 2^M / sigma use an exact
// fp32 reciprocal quotient with one integer correction (udiv_fast); the root
// is isqrt_newton10; then the per-element normalisation, affine and dyadic
// requant.  CLAMP = false when the host has shown that (b acc) >> c fits
// int32 for every reachable acc; FASTQ: the requant is one mul.hi.
constexpr int kLnLanes = 16;  // a half-warp per row
template <int LPR, int CPL, bool CLAMP, bool FASTQ>
__global__ void __launch_bounds__(kLnThreads)
    layernorm_staged_kernel(const int8_t* __restrict__ x, int64_t rows, int32_t cols,
                            const int8_t* __restrict__ gamma, const int32_t* __restrict__ beta, int32_t F,
                            int32_t M_ln, ivit_dyadic out, int32_t out_bq, int8_t* __restrict__ y) {
  // gamma (sign-extended) and beta as 16-byte groups of four channels, stored
  // [q][chunk]: group q of 16-channel chunk ci at q * nchunk + ci, so the
  // lanes of a row, which hold consecutive chunks, read consecutive 16-byte
  // slots (no bank conflicts)
  extern __shared__ int4 ln_smem[];
  const int nchunk = cols >> 4;
  int4* gs = ln_smem;                 // [4][nchunk]
  int4* bs = ln_smem + 4 * nchunk;    // [4][nchunk]
  for (int i = threadIdx.x; i < cols / 4; i += blockDim.x) {
    const int ci = i >> 2, q = i & 3;
    const uint32_t g4 = __ldg(reinterpret_cast<const uint32_t*>(gamma) + i);
    gs[q * nchunk + ci] = make_int4(sext_byte(g4, 0), sext_byte(g4, 1), sext_byte(g4, 2), sext_byte(g4, 3));
    bs[q * nchunk + ci] = __ldg(reinterpret_cast<const int4*>(beta) + i);
  }
  __syncthreads();
  pdl_wait();  // x comes from an earlier kernel
  pdl_launch_dependents();
  const int hl = threadIdx.x % LPR;
  const int64_t row = (int64_t)blockIdx.x * (kLnThreads / LPR) + (threadIdx.x / LPR);
  const bool active = row < rows;
  const int8_t* xr = x + (active ? row : 0) * cols;
  int4 v[CPL];
  int32_t s1 = 0, s2 = 0;
#pragma unroll
  for (int k = 0; k < CPL; ++k) {
    const int ci = hl + LPR * k;
    if (active && ci < nchunk) {
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
  for (int o = LPR / 2; o > 0; o >>= 1) {  // reduce within each row's lanes
    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    s2 += __shfl_xor_sync(0xffffffffu, s2, o);
  }
  if (!active) return;
  const int32_t as1 = s1 < 0 ? -s1 : s1;
  const int32_t q1 = udiv_fast(as1, cols);
  const int32_t mu = s1 >= 0 ? q1 : -q1 - (as1 - q1 * cols != 0 ? 1 : 0);
  const int32_t sd2 = s2 - 2 * mu * s1 + cols * mu * mu;
  const int32_t V = udiv_fast(sd2, cols);
  int32_t sigma = isqrt_newton10(V);
  if (sigma < 1) sigma = 1;
  const int32_t f = udiv_fast(1 << M_ln, sigma);
  const int sh = M_ln - F;
  const int32_t muf = mu * f;
  int32_t lo = INT_MIN, hi = INT_MAX;
  if (CLAMP) out_bounds(out.b, out.c, lo, hi);
  int8_t* yr = y + row * cols;
#pragma unroll
  for (int k = 0; k < CPL; ++k) {
    const int ci = hl + LPR * k;
    if (ci < nchunk) {
      const uint32_t xw[4] = {(uint32_t)v[k].x, (uint32_t)v[k].y, (uint32_t)v[k].z, (uint32_t)v[k].w};
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int4 g4 = gs[q * nchunk + ci];
        const int4 b4 = bs[q * nchunk + ci];
        const int32_t gg[4] = {g4.x, g4.y, g4.z, g4.w};
        const int32_t bb[4] = {b4.x, b4.y, b4.z, b4.w};
        int32_t r[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int32_t nv = (sext_byte(xw[q], e) * f - muf) >> sh;
          int32_t acc = nv * gg[e] + bb[e];
          if (FASTQ) {
            r[e] = __mulhi(out_bq, acc);
          } else {
            if (CLAMP) acc = min(max(acc, lo), hi);
            const int64_t pr = (int64_t)out.b * acc;
            r[e] = (int32_t)__funnelshift_r((uint32_t)pr, (uint32_t)(pr >> 32), (uint32_t)out.c);
          }
        }
        o[q] = pack_sat4_ln(r[0], r[1], r[2], r[3]);
      }
      __stcs(reinterpret_cast<int4*>(yr) + ci, make_int4((int)o[0], (int)o[1], (int)o[2], (int)o[3]));
    }
  }
}

// ---------------------------------------------------------------------------
// ShiftGELU with a row maximum (I-ViT section 3.4, I_max read as the row's
// largest exponent; see include/ivit.h): one warp per row.  I_p is
// non-decreasing in x, so the row's largest exponent is I_p of the row's
// largest byte; given it, the output is a function of the int8 input alone:
// a 256-entry table, which the warp builds when its row's I_max differs
// from its previous row's (rows of a real activation rarely share one).  A
// table entry takes its two exponentials from a per-CTA ShiftExp table over
// every reachable exponent offset (built before the dependent-launch wait:
// it depends on I0 only) and one integer division.  Tables are indexed by the
// raw byte and sit on 256-byte boundaries, so a lookup address is one
// bitwise merge of the byte and the table base.  With VPL > 0 a row of at
// most 32 VPL 16-byte vectors stays in registers between the maximum and the
// lookups; VPL = 0 reads a row twice.
// ---------------------------------------------------------------------------
constexpr int kRowGeluThreads = 256;
constexpr int kRowGeluWarps = kRowGeluThreads / 32;
// I_max - I_p(x) over int8 x: I_max <= I_p(127) = 212 and I_p(-128) = -216
constexpr int kRowGeluExpSpan = 432;

__device__ __forceinline__ int32_t gelu_ip(int32_t x) { return x + (x >> 1) + (x >> 3) + (x >> 4); }

// the four signed-byte maxima of v folded into m4
__device__ __forceinline__ uint32_t vmax_int4(uint32_t m4, const int4& v) {
  return __vmaxs4(m4, __vmaxs4(__vmaxs4((uint32_t)v.x, (uint32_t)v.y), __vmaxs4((uint32_t)v.z, (uint32_t)v.w)));
}

__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// 16 table lookups, one per byte; tbase is the table's shared-memory address
// (a multiple of 256)
__device__ __forceinline__ int4 gelu_lookup16(uint32_t tbase, const int4& in) {
  const uint32_t w[4] = {(uint32_t)in.x, (uint32_t)in.y, (uint32_t)in.z, (uint32_t)in.w};
  uint32_t o[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t v0 = lds_u8(tbase | (w[k] & 0xFFu));
    const uint32_t v1 = lds_u8(tbase | ((w[k] >> 8) & 0xFFu));
    const uint32_t v2 = lds_u8(tbase | ((w[k] >> 16) & 0xFFu));
    const uint32_t v3 = lds_u8(tbase | (w[k] >> 24));
    o[k] = __byte_perm(__byte_perm(v0, v1, 0x0040u), __byte_perm(v2, v3, 0x0040u), 0x5410u);
  }
  return make_int4((int)o[0], (int)o[1], (int)o[2], (int)o[3]);
}

template <int VPL>
__global__ void __launch_bounds__(kRowGeluThreads)
    shiftgelu_rowmax_kernel(const int8_t* __restrict__ x, int64_t rows, int32_t cols, GeluParams g,
                            int8_t* __restrict__ y) {
  __shared__ __align__(256) uint8_t tabs[kRowGeluWarps][256];
  __shared__ int32_t expt[kRowGeluExpSpan];  // expt[d] = ShiftExp(-d)
  for (int d = threadIdx.x; d < kRowGeluExpSpan; d += blockDim.x) expt[d] = shift_exp(-d, g.I0);
  __syncthreads();
  pdl_wait();  // x comes from an earlier kernel
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* own = tabs[warp];
  const uint32_t tbase = smem_u32(own);
  const int nvec = cols >> 4;
  const int sh = g.M - (g.k_out - 1);
  int32_t own_imax = -1;  // the I_max the warp's table holds (none yet)
  // the table of a row with largest byte m (warp-uniform)
  auto make_table = [&](int32_t m) {
    const int32_t ipm = gelu_ip(m);
    const int32_t I_max = ipm > 0 ? ipm : 0;
    if (I_max == own_imax) return;
    __syncwarp();  // every lane is done with the previous table
    const uint32_t e2 = (uint32_t)expt[I_max];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int32_t xi = (int32_t)(int8_t)(uint8_t)(lane + 32 * j);  // entry (uint8_t) xi
      // bytes above the row's maximum never occur in the row: their entries
      // are unused, and the offset is clamped only to stay inside the table
      const uint32_t e1 = (uint32_t)expt[max(I_max - gelu_ip(xi), 0)];
      const uint32_t sum = e1 + e2;
      const uint32_t dv = (1u << g.M) / (sum > 0u ? sum : 1u);  // both exponentials 0: sigma = 0
      const int32_t sig = (int32_t)((dv * e1) >> sh);
      own[lane + 32 * j] = (uint8_t)(int8_t)requant8(xi * sig, g.out.b, g.out.c);
    }
    __syncwarp();
    own_imax = I_max;
  };
  auto warp_max = [&](uint32_t m4) {
    int32_t m = max(max((int32_t)(int8_t)m4, (int32_t)(int8_t)(m4 >> 8)),
                    max((int32_t)(int8_t)(m4 >> 16), (int32_t)(int8_t)(m4 >> 24)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    return m;
  };
  const int64_t rstep = (int64_t)gridDim.x * kRowGeluWarps;
  for (int64_t row = (int64_t)blockIdx.x * kRowGeluWarps + warp; row < rows; row += rstep) {
    const int4* xv = reinterpret_cast<const int4*>(x + row * cols);
    int4* yv = reinterpret_cast<int4*>(y + row * cols);
    if (VPL > 0) {
      int4 v[VPL > 0 ? VPL : 1];
      uint32_t m4 = 0x80808080u;  // padding vectors hold -128, which never raises the maximum
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
        const int c = lane + 32 * k;
        v[k] = c < nvec ? __ldcs(xv + c) : make_int4((int)0x80808080, (int)0x80808080, (int)0x80808080, (int)0x80808080);
        m4 = vmax_int4(m4, v[k]);
      }
      make_table(warp_max(m4));
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
        const int c = lane + 32 * k;
        if (c < nvec) __stcs(yv + c, gelu_lookup16(tbase, v[k]));
      }
    } else {
      uint32_t m4 = 0x80808080u;
      for (int c = lane; c < nvec; c += 32) m4 = vmax_int4(m4, __ldg(xv + c));
      make_table(warp_max(m4));
      for (int c = lane; c < nvec; c += 32) __stcs(yv + c, gelu_lookup16(tbase, __ldg(xv + c)));
    }
  }
}

// ---------------------------------------------------------------------------
// I-LayerNorm of an input with power-of-two channel factors (the FQ-ViT
// record's Power-of-Two Factor; see include/ivit.h): one warp per row; the
// LayerNorm input is x_i << alpha_i (|x << alpha| <= 1024).  Sums are exact
// in 32 bits for cols <= 2048 (2048 * 1024^2 < 2^31); (x - mu) f stays below
// 2^31 because the host requires M_ln <= 23 - max alpha.
// ---------------------------------------------------------------------------
constexpr int kPtfThreads = 256;

template <bool FASTQ>
__global__ void __launch_bounds__(kPtfThreads)
    layernorm_ptf_kernel(const int8_t* __restrict__ x, int64_t rows, int32_t cols, const uint8_t* __restrict__ alpha,
                         const int8_t* __restrict__ gamma, const int32_t* __restrict__ beta, int32_t F, int32_t M_ln,
                         ivit_dyadic out, int32_t out_bq, int8_t* __restrict__ y) {
  pdl_wait();  // x comes from an earlier kernel
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int nchunk = cols >> 4;
  for (int64_t row = (int64_t)blockIdx.x * (kPtfThreads / 32) + (threadIdx.x >> 5); row < rows;
       row += (int64_t)gridDim.x * (kPtfThreads / 32)) {
    const int4* xr = reinterpret_cast<const int4*>(x + row * cols);
    int32_t s1 = 0, s2 = 0;
    for (int ci = lane; ci < nchunk; ci += 32) {
      const int4 xv = __ldg(xr + ci);
      const int4 av = __ldg(reinterpret_cast<const int4*>(alpha) + ci);
      const uint32_t xw[4] = {(uint32_t)xv.x, (uint32_t)xv.y, (uint32_t)xv.z, (uint32_t)xv.w};
      const uint32_t aw[4] = {(uint32_t)av.x, (uint32_t)av.y, (uint32_t)av.z, (uint32_t)av.w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int32_t v = sext_byte(xw[q], e) << ((aw[q] >> (8 * e)) & 3u);
          s1 += v;
          s2 += v * v;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s1 += __shfl_xor_sync(0xffffffffu, s1, o);
      s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    }
    // mu = floor(sum / n); V = floor(sum (v - mu)^2 / n) = floor((s2 - 2 mu s1 + n mu^2) / n), in 64 bits
    const int64_t mu = s1 >= 0 ? (int64_t)s1 / cols : -((-(int64_t)s1 + cols - 1) / cols);
    const int64_t sd2 = (int64_t)s2 - 2 * mu * s1 + (int64_t)cols * mu * mu;
    const int32_t V = (int32_t)(sd2 / cols);  // sd2 >= 0
    int32_t sigma = isqrt_newton10(V);
    if (sigma < 1) sigma = 1;
    const int32_t f = (int32_t)((1u << M_ln) / (uint32_t)sigma);
    const int sh = M_ln - F;
    int8_t* yr = y + row * cols;
    for (int ci = lane; ci < nchunk; ci += 32) {
      const int c0 = ci * 16;
      const int4 xv = __ldg(xr + ci);
      const int4 av = __ldg(reinterpret_cast<const int4*>(alpha) + ci);
      const int4 gv = __ldg(reinterpret_cast<const int4*>(gamma + c0));
      const uint32_t xw[4] = {(uint32_t)xv.x, (uint32_t)xv.y, (uint32_t)xv.z, (uint32_t)xv.w};
      const uint32_t aw[4] = {(uint32_t)av.x, (uint32_t)av.y, (uint32_t)av.z, (uint32_t)av.w};
      const uint32_t gw[4] = {(uint32_t)gv.x, (uint32_t)gv.y, (uint32_t)gv.z, (uint32_t)gv.w};
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int4 bt = __ldg(reinterpret_cast<const int4*>(beta + c0) + q);
        const int32_t bb[4] = {bt.x, bt.y, bt.z, bt.w};
        int32_t r[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int32_t v = sext_byte(xw[q], e) << ((aw[q] >> (8 * e)) & 3u);
          const int32_t nv = ((v - (int32_t)mu) * f) >> sh;
          const int32_t acc = nv * sext_byte(gw[q], e) + bb[e];
          if (FASTQ) {
            r[e] = __mulhi(out_bq, acc);
          } else {
            const int64_t q64 = ((int64_t)out.b * acc) >> out.c;
            r[e] = (int32_t)(q64 < -128 ? -128 : (q64 > 127 ? 127 : q64));
          }
        }
        o[q] = pack_sat4_ln(r[0], r[1], r[2], r[3]);
      }
      __stcs(reinterpret_cast<int4*>(yr) + ci, make_int4((int)o[0], (int)o[1], (int)o[2], (int)o[3]));
    }
  }
}

}  // namespace

ivit_status launch_shiftgelu_rowmax(const DeviceCtx& dc, const int8_t* x, int64_t rows, int32_t cols,
                                    const GeluParams& g, int8_t* y, cudaStream_t stream) {
  if (rows == 0) return IVIT_OK;
  // rows in registers up to 32 x 8 vectors (4096 columns); one wave of
  // resident CTAs, so that each warp takes several rows and the next row's
  // load overlaps the current lookups
  const int vpl = (cols / 16 + 31) / 32;
  static int per_sm_of[6] = {0, 0, 0, 0, 0, 0};  // resident CTAs per SM of each instance (benign race: same value)
  auto run = [&](int id, void (*kernel)(const int8_t*, int64_t, int32_t, GeluParams, int8_t*)) -> cudaError_t {
    int& per_sm = per_sm_of[id];
    if (per_sm == 0 && cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kRowGeluThreads, 0) != cudaSuccess)
      return cudaErrorUnknown;
    int64_t blocks = (rows + kRowGeluWarps - 1) / kRowGeluWarps;
    const int64_t cap = (int64_t)dc.num_sms * (per_sm > 0 ? per_sm : 1);
    if (blocks > cap) blocks = cap;
    return launch_pdl(kernel, dim3((unsigned)blocks), dim3(kRowGeluThreads), 0, stream, x, rows, cols, g, y);
  };
  cudaError_t e;
  if (vpl <= 1)
    e = run(0, shiftgelu_rowmax_kernel<1>);
  else if (vpl <= 2)
    e = run(1, shiftgelu_rowmax_kernel<2>);
  else if (vpl <= 4)
    e = run(2, shiftgelu_rowmax_kernel<4>);
  else if (vpl <= 6)
    e = run(3, shiftgelu_rowmax_kernel<6>);
  else if (vpl <= 8)
    e = run(4, shiftgelu_rowmax_kernel<8>);
  else
    e = run(5, shiftgelu_rowmax_kernel<0>);
  note_launch();
  return e == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}

ivit_status launch_layernorm_ptf(const DeviceCtx& dc, const int8_t* x, int64_t rows, int32_t cols,
                                 const uint8_t* alpha, const int8_t* gamma, const int32_t* beta, int32_t F,
                                 int32_t M_ln, ivit_dyadic out, int8_t* y, cudaStream_t stream) {
  if (rows == 0) return IVIT_OK;
  const int64_t rows_per_cta = kPtfThreads / 32;
  int64_t blocks = (rows + rows_per_cta - 1) / rows_per_cta;
  const int64_t cap = (int64_t)dc.num_sms * 16;
  if (blocks > cap) blocks = cap;
  // the output requant is one mul.hi by b 2^(32 - c) when that fits a positive int32
  const bool fastq = out.c >= 1 && (int64_t)out.b < ((int64_t)1 << (out.c - 1));
  const int32_t bq = fastq ? (int32_t)((int64_t)out.b << (32 - out.c)) : 0;
  const cudaError_t e =
      fastq ? launch_pdl(layernorm_ptf_kernel<true>, dim3((unsigned)blocks), dim3(kPtfThreads), 0, stream, x, rows,
                         cols, alpha, gamma, beta, F, M_ln, out, bq, y)
            : launch_pdl(layernorm_ptf_kernel<false>, dim3((unsigned)blocks), dim3(kPtfThreads), 0, stream, x, rows,
                         cols, alpha, gamma, beta, F, M_ln, out, bq, y);
  note_launch();
  return e == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}

ivit_status launch_shiftgelu(const DeviceCtx& dc, const int8_t* x, int64_t n, const GeluParams& g, int8_t* y,
                             cudaStream_t stream) {
  if (n == 0) return IVIT_OK;
  const int64_t nvec = n >> 4;
  int64_t blocks = (nvec + kGeluThreads - 1) / kGeluThreads;
  const int64_t cap = (int64_t)dc.num_sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const cudaError_t e = launch_pdl(shiftgelu_kernel, dim3((unsigned)blocks), dim3(kGeluThreads), 0, stream, x, n, g, y);
  note_launch();
  return e == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}

ivit_status launch_layernorm(const DeviceCtx& dc, const int8_t* x, int64_t rows, int32_t cols,
                             const int8_t* gamma, const int32_t* beta, int32_t F, int32_t M_ln, ivit_dyadic out,
                             int8_t* y, cudaStream_t stream) {
  (void)dc;
  if (rows == 0) return IVIT_OK;
  const int64_t rows_per_cta = kLnThreads / kLnLanes;
  const int64_t blocks = (rows + rows_per_cta - 1) / rows_per_cta;
  if (blocks > 0x7fffffff) return IVIT_ERR_UNSUPPORTED;
  const size_t smem = (size_t)cols * 8;  // gamma and beta as int32
  const unsigned g = (unsigned)blocks;
  const int nchunk = cols / 16;
  // |n| <= 255 2^F, |gamma| <= 128, |beta| <= 2^30: when b times that bound stays
  // below 2^(30 + c), (b acc) >> c always fits int32 and the clamp is not needed
  const double amax = 255.0 * 128.0 * std::ldexp(1.0, F) + std::ldexp(1.0, 30);
  const bool clamp = amax * (double)out.b >= std::ldexp(1.0, 30 + out.c);
  // the output requant is one mul.hi by b 2^(32 - c) when that fits a positive int32
  const bool fastq = out.c >= 1 && (int64_t)out.b < ((int64_t)1 << (out.c - 1));
  const int32_t bq = fastq ? (int32_t)((int64_t)out.b << (32 - out.c)) : 0;
#define IVIT_LN_LAUNCH(CPL)                                                                                  \
  launch_pdl(fastq   ? layernorm_staged_kernel<kLnLanes, CPL, false, true>                                      \
             : clamp ? layernorm_staged_kernel<kLnLanes, CPL, true, false>                                      \
                     : layernorm_staged_kernel<kLnLanes, CPL, false, false>,                                    \
             dim3(g), dim3(kLnThreads), smem, stream, x, rows, cols, gamma, beta, F, M_ln, out, bq, y)
  cudaError_t e;
  const int cpl = (nchunk + kLnLanes - 1) / kLnLanes;
  if (cpl <= 1)
    e = IVIT_LN_LAUNCH(1);
  else if (cpl <= 2)
    e = IVIT_LN_LAUNCH(2);
  else if (cpl <= 3)
    e = IVIT_LN_LAUNCH(3);
  else if (cpl <= 4)
    e = IVIT_LN_LAUNCH(4);
  else if (cpl <= 6)
    e = IVIT_LN_LAUNCH(6);
  else if (cpl <= 8)
    e = IVIT_LN_LAUNCH(8);
  else
    e = IVIT_LN_LAUNCH(16);
#undef IVIT_LN_LAUNCH
  note_launch();
  return e == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}

}  // namespace ivit
