// ivit_gemm.cu -- INT8 linear layer with the dyadic epilogue on the 5th-gen
// tensor cores (tcgen05.mma kind::i8, TMA-fed shared memory, TMEM accumulator).
//
// Y = sat((b_j * (X W^T + bias)_ij) >> c_j), optionally followed by a residual
// addition or a ShiftGELU lookup ("I-ViT: Integer-only Quantization for
// Efficient Vision Transformer Inference", sections 3.1, 3.2 and 3.4; the
// Trio-ViT article, eqs. (1) and (12)).
//
// Design (one CTA per SM, persistent over 128 x BN output tiles):
//   warp 0      TMA producer: 128 x 128 A and BN x 128 B k-slices, 128B swizzle,
//               into a STAGES-deep ring guarded by full/empty mbarriers;
//   warp 1      allocates TMEM (2 x BN columns) and one lane issues
//               tcgen05.mma M=128 N=BN K=32; tcgen05.commit frees smem stages
//               and publishes finished accumulators;
//   warps 2-5   epilogue: tcgen05.ld 32 columns at a time, bias, dyadic
//               requant, saturation, optional residual / GELU table, 16-byte
//               stores.  Two accumulators let the epilogue of tile t overlap
//               the MMAs of tile t+1.
#include "ivit_common.cuh"
#include "ivit_internal.h"

namespace ivit {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 128;  // bytes = int8 elements per k-slice (one 128-byte swizzle row)
constexpr int kGemmThreads = 192;

struct GemmArgs {
  int64_t M;
  int32_t N, K;
  const int32_t* bias;
  const int32_t* b;
  const int8_t* c;
  int32_t lo, hi;  // saturation range of the requantised output
  const int8_t* skip;
  ivit_residual res;
  int8_t* Y;
  GeluParams gelu;
  int* status;
};

template <int BN, int STAGES>
struct GemmLayout {
  static constexpr int kABytes = kBM * kBK;
  static constexpr int kBBytes = BN * kBK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarOff = STAGES * kStageBytes;
  static constexpr int kNumBars = 2 * STAGES + 5;  // full, empty, tmem full x2, tmem empty x2, drain
  static constexpr int kSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kGeluOff = kSlotOff + 16;
  static constexpr int kBytes = kGeluOff + 256;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 bytes
};

template <int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_i8_requant_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const GemmArgs args) {
  using L = GemmLayout<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);
  int8_t* gelu_tab = reinterpret_cast<int8_t*>(smem + L::kGeluOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t M = args.M;
  const int N = args.N;
  const int m_tiles = (int)((M + kBM - 1) / kBM);
  const int n_tiles = (N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int num_kb = (args.K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (EPI == kEpiGelu) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x)
      gelu_tab[i] = (int8_t)shiftgelu8(i - 128, args.gelu.I0, args.gelu.M, args.gelu.k_out, args.gelu.out.b,
                                       args.gelu.out.c);
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(tslot, 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tslot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued = 0;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const int mb = t / n_tiles, nb = t % n_tiles;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, args.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
          uint8_t* sa = smem + stage * L::kStageBytes;
          tma_load_2d(sa, &tmA, kb * kBK, mb * kBM, &full[stage]);
          tma_load_2d(sa + L::kABytes, &tmB, kb * kBK, nb * BN, &full[stage]);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        // let the copies already in flight land before the CTA exits
        for (int i = 0; i < STAGES && i < issued; ++i) {
          stage = (stage + STAGES - 1) % STAGES;
          if (stage == STAGES - 1) phase ^= 1;
          mbar_wait(&full[stage], phase, args.status);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_i8(kBM, BN, true, true, false);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * L::kStageBytes);
          const uint32_t sb = sa + L::kABytes;
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k) {
            const uint64_t da = smem_desc(sa + k * 32, 16, 1024, kSwizzle128B);
            const uint64_t db = smem_desc(sb + k * 32, 16, 1024, kSwizzle128B);
            umma_i8(d_tmem, da, db, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      // all MMAs of this CTA have finished before TMEM is released
      umma_commit(drain);
      mbar_wait(drain, 0, args.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes [32 * quarter, 32 * quarter + 32)
    const int row_local = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      const int mb = t / n_tiles, nb = t % n_tiles;
      const bool got = mbar_wait(&tfull[acc], acc_phase, args.status);
      if (!__all_sync(0xffffffffu, got)) break;  // warp-uniform give-up
      tc_fence_after();
      const int64_t row = (int64_t)mb * kBM + row_local;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        const int col0 = nb * BN + ch * 32;
        if (col0 >= N) break;  // warp-uniform
        uint32_t r[32];
        __syncwarp();
        tmem_ld32(tbase + (uint32_t)(ch * 32), r);
        tmem_ld_wait();
        if (row < M) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int col = col0 + half * 16;
            if (col < N) {
              int32_t bb[16], bi[16];
              int8_t cc[16];
              *reinterpret_cast<int4*>(&bb[0]) = __ldg(reinterpret_cast<const int4*>(args.b + col));
              *reinterpret_cast<int4*>(&bb[4]) = __ldg(reinterpret_cast<const int4*>(args.b + col + 4));
              *reinterpret_cast<int4*>(&bb[8]) = __ldg(reinterpret_cast<const int4*>(args.b + col + 8));
              *reinterpret_cast<int4*>(&bb[12]) = __ldg(reinterpret_cast<const int4*>(args.b + col + 12));
              if (args.bias) {
                *reinterpret_cast<int4*>(&bi[0]) = __ldg(reinterpret_cast<const int4*>(args.bias + col));
                *reinterpret_cast<int4*>(&bi[4]) = __ldg(reinterpret_cast<const int4*>(args.bias + col + 4));
                *reinterpret_cast<int4*>(&bi[8]) = __ldg(reinterpret_cast<const int4*>(args.bias + col + 8));
                *reinterpret_cast<int4*>(&bi[12]) = __ldg(reinterpret_cast<const int4*>(args.bias + col + 12));
              } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) bi[i] = 0;
              }
              *reinterpret_cast<int4*>(&cc[0]) = __ldg(reinterpret_cast<const int4*>(args.c + col));
              int4 sk = make_int4(0, 0, 0, 0);
              if (EPI == kEpiResidual)
                sk = __ldg(reinterpret_cast<const int4*>(args.skip + row * N + col));
              const int8_t* skb = reinterpret_cast<const int8_t*>(&sk);
              uint32_t packed[4];
#pragma unroll
              for (int w = 0; w < 4; ++w) {
                uint32_t word = 0;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int i = w * 4 + e;
                  const int32_t v = (int32_t)r[half * 16 + i] + bi[i];
                  int32_t y = requant_bits(v, bb[i], (int32_t)cc[i], args.lo, args.hi);
                  if (EPI == kEpiResidual) y = residual8(skb[i], y, args.res.b_skip, args.res.b_branch, args.res.c);
                  if (EPI == kEpiGelu) y = gelu_tab[y + 128];
                  word |= ((uint32_t)y & 0xFFu) << (8 * e);
                }
                packed[w] = word;
              }
              *reinterpret_cast<int4*>(args.Y + row * N + col) =
                  make_int4((int)packed[0], (int)packed[1], (int)packed[2], (int)packed[3]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * BN);
  }
}

template <int BN, int STAGES, int EPI>
ivit_status run_gemm(const DeviceCtx& dc, const int8_t* X, const int8_t* W, const GemmArgs& a,
                     cudaStream_t stream) {
  using L = GemmLayout<BN, STAGES>;
  static_assert(L::kAlloc <= 227 * 1024, "shared memory budget");
  CUtensorMap tmA, tmB;
  ivit_status st = encode_tmap_2d_u8(&tmA, X, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.K, kBK, kBM,
                                     CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != IVIT_OK) return st;
  st = encode_tmap_2d_u8(&tmB, W, (uint64_t)a.K, (uint64_t)a.N, (uint64_t)a.K, kBK, BN,
                         CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != IVIT_OK) return st;
  auto kern = gemm_i8_requant_kernel<BN, STAGES, EPI>;
  static bool attr_done = false;  // benign race: the attribute value is the same
  if (!attr_done) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) != cudaSuccess)
      return IVIT_ERR_CUDA;
    attr_done = true;
  }
  const int m_tiles = (int)((a.M + kBM - 1) / kBM);
  const int n_tiles = (a.N + BN - 1) / BN;
  const int tiles = m_tiles * n_tiles;
  const int grid = tiles < dc.num_sms ? tiles : dc.num_sms;
  kern<<<grid, kGemmThreads, L::kAlloc, stream>>>(tmA, tmB, a);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}

template <int EPI>
ivit_status dispatch_bn(const DeviceCtx& dc, const int8_t* X, const int8_t* W, const GemmArgs& a,
                        cudaStream_t stream) {
  if (a.N % 256 == 0) return run_gemm<256, 4, EPI>(dc, X, W, a, stream);
  return run_gemm<128, 6, EPI>(dc, X, W, a, stream);
}

}  // namespace

ivit_status launch_gemm(const DeviceCtx& dc, const int8_t* X, int64_t M, int32_t K, const int8_t* W, int32_t N,
                        const int32_t* bias, const int32_t* b, const int8_t* c, int32_t out_bits, EpiMode mode,
                        const int8_t* skip, ivit_residual res, const GeluParams* gelu, int8_t* Y,
                        cudaStream_t stream) {
  GemmArgs a;
  a.M = M;
  a.N = N;
  a.K = K;
  a.bias = bias;
  a.b = b;
  a.c = c;
  a.lo = -(1 << (out_bits - 1));
  a.hi = (1 << (out_bits - 1)) - 1;
  a.skip = skip;
  a.res = res;
  a.Y = Y;
  a.gelu = gelu ? *gelu : GeluParams{1, 30, 8, {0, 0}};
  a.status = dc.status;
  switch (mode) {
    case kEpiPlain:
      return dispatch_bn<kEpiPlain>(dc, X, W, a, stream);
    case kEpiResidual:
      return dispatch_bn<kEpiResidual>(dc, X, W, a, stream);
    case kEpiGelu:
      return dispatch_bn<kEpiGelu>(dc, X, W, a, stream);
  }
  return IVIT_ERR_INTERNAL;
}

}  // namespace ivit
