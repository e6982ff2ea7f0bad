// ivit_gemm.cu -- INT8 linear layer with the dyadic epilogue on the 5th-gen
// tensor cores (tcgen05.mma kind::i8, TMA-fed shared memory, TMEM accumulator).
//
// Y = sat((b_j * (X W^T + bias)_ij) >> c_j), optionally followed by a residual
// addition or a ShiftGELU lookup ("I-ViT: Integer-only Quantization for
// Efficient Vision Transformer Inference", sections 3.1, 3.2 and 3.4; the
// Trio-ViT article, eqs. (1) and (12)).
//
// The accumulator is computed transposed, D = W X^T: the UMMA M dimension
// (TMEM lanes) runs over 128 output channels and N over BN tokens.  Every
// epilogue thread therefore owns one output channel of the tile and keeps that
// channel's multiplier and shift in registers.  The bias is not added per
// element: each accumulator buffer is preloaded with its next tile's bias
// (tcgen05.st) before the MMAs accumulate onto it.  When b_j < 2^(c_j - 1) (a
// requant scale below one half, the usual case) the requant
// floor(b acc / 2^c) is then one mul.hi by b 2^(32 - c); the saturating byte
// pack clips (a round-half-up variant adds half an LSB first).  A 4 x 4 byte
// transpose across lanes turns channel-major bytes into token-major 4-byte
// words.  The four warps that cover the tile's 128 channels for the same
// tokens (one per TMEM lane quarter: a "part") fill one 16-token x
// 128-channel staging slot per chunk, 128B-swizzled, and one thread of the
// part sends it out with a single TMA store of 16 rows of 128 bytes (a
// quarter as many stores as one per warp).  Where shared memory allows, two
// slot sets serve alternate tiles.  The residual's skip tile arrives the
// same way.  Each tile's channel constants are loaded and turned into its
// requant form one tile ahead.
//
// Roles (one CTA per SM, persistent over 128 x BN tiles):
//   warp 0      TMA producer: W and X k-slices of 128 bytes, 128B swizzle,
//               into a STAGES-deep ring guarded by full/empty mbarriers;
//   warps 1-2   MMA issue: warp 1 allocates TMEM (two BN-column accumulators);
//               lane 0 issues tcgen05.mma M=128 N=BN K=32.  With an even ring
//               depth lane 0 of warp 2 issues too: the two threads take
//               alternate k-slices (the even and the odd ones of the CTA's
//               whole sequence), both into the same accumulator;
//               tcgen05.commit frees smem stages and, from every issuing
//               thread, publishes finished accumulators;
//   warps 3-14  epilogue: three warps per TMEM lane quarter split the tile's
//               16-token chunks; the accumulator of tile t drains while the
//               MMAs of tile t+1 run.
//
// Why two issuing threads: one thread spends about 480 SM cycles per k-slice
// on its mbarrier wait, the four MMA issues and the commit, whatever BN is,
// while the four MMAs take 2 BN cycles on the tensor core; below BN = 256 a
// single issuer leaves the tensor core idle.  Two threads overlap that
// bookkeeping.  The integer accumulation is exact and every MMA accumulates
// (the bias is preloaded), so the order in which the two threads' MMAs land
// on the accumulator does not change the result.  The ring depth must be even
// so that each thread owns the stages of its k-slice parity: a thread then
// waits on a stage's full barrier only after its own previous use of the
// stage, never two phases ahead of it (TMA loads may complete out of order,
// and a parity wait cannot tell phase p from phase p + 2).  At BN = 256 the
// ring is three deep and a single thread keeps the tensor core busy.
#include <climits>

#include "ivit_common.cuh"
#include "ivit_internal.h"

namespace ivit {
namespace {

constexpr int kBM = 128;  // output channels per tile
constexpr int kBK = 128;  // bytes = int8 elements per k-slice (one 128-byte swizzle row)
constexpr int kEpiWarps = 12;  // three per TMEM lane quarter
constexpr int kEpiParts = kEpiWarps / 4;
constexpr int kGemmThreads = 96 + 32 * kEpiWarps;
constexpr int kSlotBytes = 16 * kBM;  // one staged chunk: 16 tokens x 128 channels

struct GemmArgs {
  int64_t M;       // tokens (rows of X and Y)
  int32_t N, K;    // output channels, reduction length
  const int32_t* bias;
  const int32_t* b;
  const int8_t* c;
  int32_t lo, hi;  // saturation range of the requantised output
  int32_t round;   // 1: the requant rounds half up (else the floor shift)
  ivit_residual res;
  GeluParams gelu;
  int* status;
  int32_t withhold;  // diagnostic: CTA 0's producer stops before this k-slice of its sequence (-1: never)
};

template <int BN, int STAGES>
struct GemmLayout {
  // MMA-issuing threads: two when each can own half of the ring's stages
  static constexpr int kIssuers = (STAGES % 2 == 0) ? 2 : 1;
  static constexpr int kABytes = kBM * kBK;
  static constexpr int kBBytes = BN * kBK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kChunks = BN / 16;
  static constexpr int kMaxPart = (kChunks + kEpiParts - 1) / kEpiParts;  // chunks of the largest part
  static constexpr int kOutOff = STAGES * kStageBytes;
  static constexpr int kPartSlots = kMaxPart * kSlotBytes;  // 1024-byte aligned, as the swizzle needs
  static constexpr int kSetBytes = kEpiParts * kPartSlots;    // one slot set: every part's chunks
  // Two slot sets, used by alternate tiles, when they fit: a tile's stores
  // then have a whole tile's time to finish reading their slots.
  static constexpr int kFixedBytes = (2 * STAGES + 5 + kEpiParts) * 8 + 16 + 256 + 1024;
  static constexpr int kSlotSets = (kOutOff + 2 * kSetBytes + kFixedBytes <= 227 * 1024) ? 2 : 1;
  static constexpr int kBarOff = kOutOff + kSlotSets * kSetBytes;
  // full, empty (STAGES each), tmem full x2, tmem empty x2, drain, one skip barrier per part
  static constexpr int kNumBars = 2 * STAGES + 5 + kEpiParts;
  static constexpr int kSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kGeluOff = kSlotOff + 16;
  static constexpr int kBytes = kGeluOff + 256;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 bytes
  // TMEM columns per accumulator buffer: BN rounded up to 32, so the second
  // buffer starts on a 32-column boundary whatever the tile width
  static constexpr int kAccCols = (BN + 31) / 32 * 32;
  static constexpr int kTmemCols = (2 * kAccCols <= 256) ? 256 : 512;
};

IVIT_DEV int32_t sat_i32(int64_t v) {
  return (int32_t)(v < (int64_t)INT_MIN ? (int64_t)INT_MIN : (v > (int64_t)INT_MAX ? (int64_t)INT_MAX : v));
}

// Per-channel constants of the requant sat((b acc) >> c), b >= 0, where acc
// already holds the bias.  floor(b acc / 2^c) is monotone in acc.  With
// bl = bit length of b, s = bl - 1 - c (so 2^s <= b / 2^c < 2^(s+1)) and
// u = 128 / 2^s (u = 1 once s >= 7), acc = u gives a result >= 128 and
// acc = -u one <= -128, while every acc in [-u, u] gives a result of magnitude
// at most max(256, b / 2^c) < 2^31.  Clamping acc to [-u, u] therefore changes
// no result inside the int8 range (nor any narrower range), sends everything
// beyond to a value that saturates the same way, and keeps the shifted result
// within int32: the saturating byte pack then finishes the job.  When even
// the largest possible |acc| (2^14 K + |bias|) keeps |b acc| below 2^(30 + c),
// the shifted result always fits int32 and the clamp is skipped.
//
// Fast form: when b < 2^(c - 1), bq = b 2^(32 - c) is a positive int32 and
// floor(b acc / 2^c) = floor(bq acc / 2^32) = mul.hi(bq, acc) exactly, for
// every int32 acc; acc stays within int32 because |acc| <= 2^14 K + |bias| <=
// 2^28 + 2^30.  b = 0 takes the fast form with bq = 0.
struct ChanConst {
  int32_t b, c, lim, bq;
  bool fast, needs_clamp;
};

IVIT_DEV ChanConst chan_const(int32_t b, int32_t c, int32_t bias, int32_t K) {
  ChanConst k;
  k.b = b;
  k.c = c;
  k.fast = b == 0 || (c >= 1 && (int64_t)b < ((int64_t)1 << (c - 1)));
  k.bq = (k.fast && b != 0) ? (int32_t)((uint32_t)b << (32 - c)) : 0;
  if (b == 0) {
    k.lim = INT_MAX;
    k.needs_clamp = false;
    return k;
  }
  const int bl = 32 - __clz(b);
  const int s = bl - 1 - c;  // 2^s <= b / 2^c < 2^(s+1)
  const int64_t u = s >= 7 ? 1 : (s >= 0 ? (128 >> s) : ((int64_t)128 << (-s)));
  k.lim = sat_i32(u);
  const int64_t vmax = (int64_t)K * 16384 + (bias < 0 ? -(int64_t)bias : (int64_t)bias);
  k.needs_clamp = vmax * (int64_t)b >= ((int64_t)1 << (30 + c));
  return k;
}

// Requant forms, chosen per warp and tile: every channel of the warp fast, or
// the 64-bit product with or without the accumulator clamp; each with the
// floor shift or, in the round-half-up variant of the linear layers, with
// 2^(c - 1) added before it.
enum ReqForm : int {
  kReqFast = 0,
  kReqWide = 1,
  kReqWideClamp = 2,
  kReqRound = 3,  // added to a form: round half up
};

// floor(b acc / 2^c) (ROUND: floor(b acc / 2^c + 1/2)).  In the wide forms
// the result fits int32 (see above; adding half an LSB changes nothing
// there), so the low word of the 64-bit shift is one funnel shift (c <= 31).
// The fast form with rounding: b acc / 2^c = bq acc / 2^32 exactly, and
// floor((bq acc + 2^31) / 2^32) is the high word plus the top bit of the low
// word.  The clamp keeps the saturation direction: acc = +-u still gives a
// result of magnitude >= 128 after rounding.
template <int REQ>
IVIT_DEV int32_t requant_acc(int32_t acc, const ChanConst& k) {
  constexpr int form = REQ % kReqRound;
  constexpr bool round = REQ >= kReqRound;
  if (form == kReqFast) {
    const int32_t hi = __mulhi(k.bq, acc);
    if (!round) return hi;
    const uint32_t lo = (uint32_t)k.bq * (uint32_t)acc;
    return hi + (int32_t)(lo >> 31);
  }
  const int32_t a = form == kReqWideClamp ? min(max(acc, -k.lim), k.lim) : acc;
  int64_t v = (int64_t)k.b * a;
  if (round && k.c > 0) v += (int64_t)1 << (k.c - 1);
  return (int32_t)__funnelshift_r((uint32_t)v, (uint32_t)(v >> 32), (uint32_t)k.c);
}

// bytes [sat8(y0), sat8(y1), sat8(y2), sat8(y3)]
IVIT_DEV uint32_t pack_sat4(int32_t y0, int32_t y1, int32_t y2, int32_t y3) {
  uint32_t t, d;
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(t) : "r"(y3), "r"(y2), "r"(0u));
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(y1), "r"(y0), "r"(t));
  return d;
}

// sign-extended byte I of w: one prmt in sign-replicate mode (the __byte_perm
// intrinsic keeps only the low three bits of each selector nibble, so the
// instruction is written out)
template <int I>
IVIT_DEV int32_t sbyte(uint32_t w) {
  constexpr uint32_t sel = (uint32_t)I | ((8u | I) << 4) | ((8u | I) << 8) | ((8u | I) << 12);
  int32_t r;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(w), "n"(sel));
  return r;
}

// 4 x 4 byte transpose among lanes 4g..4g+3: lane l enters with byte i =
// element (i, l) and leaves with byte i = element (l, i).  sel2 / sel1 are
// the lane's byte selectors, (lane & 2) ? 0x3276 : 0x5410 and
// (lane & 1) ? 0x3715 : 0x6240.
IVIT_DEV uint32_t transpose4x4(uint32_t w, uint32_t sel2, uint32_t sel1) {
  uint32_t o = __shfl_xor_sync(0xffffffffu, w, 2);
  w = __byte_perm(w, o, sel2);
  o = __shfl_xor_sync(0xffffffffu, w, 1);
  return __byte_perm(w, o, sel1);
}

// sat_8((b_skip s + b_branch y) >> c) on the four bytes of two words.  The
// sum is below 2^39 in magnitude, so once c >= 9 the shifted value fits int32:
// the low word of the funnel shift is exact and the saturating pack clips it.
template <bool FAST_RES>
IVIT_DEV uint32_t residual_word(uint32_t s, uint32_t y, const ivit_residual& res) {
  int32_t z[4];
#define IVIT_RES_BYTE(I)                                                                      \
  {                                                                                           \
    int64_t t = (int64_t)res.b_skip * sbyte<I>(s);                                            \
    t += (int64_t)res.b_branch * sbyte<I>(y);                                                 \
    if (FAST_RES) {                                                                           \
      z[I] = (int32_t)__funnelshift_r((uint32_t)t, (uint32_t)(t >> 32), (uint32_t)res.c);     \
    } else {                                                                                  \
      const int64_t q = t >> res.c;                                                           \
      z[I] = (int32_t)(q < -128 ? -128 : (q > 127 ? 127 : q));                                \
    }                                                                                         \
  }
  IVIT_RES_BYTE(0)
  IVIT_RES_BYTE(1)
  IVIT_RES_BYTE(2)
  IVIT_RES_BYTE(3)
#undef IVIT_RES_BYTE
  return pack_sat4(z[0], z[1], z[2], z[3]);
}

// Byte offset of the lane's word k (token 4k + sub of the chunk, the lane's
// channel group of four) in a 128B-swizzled 16 x 128-byte slot: 16-byte
// column c of row r sits at column c ^ (r & 7).  ofs_even / ofs_odd are the
// offsets for k = 0 and k = 1; words 2 and 3 lie 8 rows (1024 bytes) further.
IVIT_DEV uint32_t slot_ofs(int sub, int quarter, int grp, int k01) {
  const int r = 4 * k01 + sub;
  const int c = 2 * quarter + (grp >> 2);
  return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4) + ((grp & 3) << 2));
}

// One 16-token chunk of one epilogue warp: requant the 16 accumulators of this
// thread's channel (r = TMEM columns of the chunk), pack, transpose to
// token-major words, apply the residual (its skip words were staged in the
// same slot) and leave the result in the slot at the lane's offsets.
template <int EPI, bool NARROW, int REQ>
IVIT_DEV void epi_chunk(const uint32_t (&r)[16], const ChanConst& kc, const GemmArgs& args, const int8_t* gelu_tab,
                        uint8_t* slot, uint32_t ofs_even, uint32_t ofs_odd, uint32_t sel2, uint32_t sel1) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    int32_t y[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int32_t v = requant_acc<REQ>((int32_t)r[4 * k + i], kc);
      if (EPI == kEpiGelu) {
        v = min(max(v, -128), 127);
        v = gelu_tab[v + 128];
      } else if (NARROW) {
        v = min(max(v, args.lo), args.hi);
      }
      y[i] = v;
    }
    w[k] = transpose4x4(pack_sat4(y[0], y[1], y[2], y[3]), sel2, sel1);
  }
  if (EPI == kEpiResidual) {
    uint32_t s[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) s[k] = *reinterpret_cast<const uint32_t*>(slot + (k >> 1) * 1024 + ((k & 1) ? ofs_odd : ofs_even));
    if (args.res.c >= 9) {
#pragma unroll
      for (int k = 0; k < 4; ++k) w[k] = residual_word<true>(s[k], w[k], args.res);
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) w[k] = residual_word<false>(s[k], w[k], args.res);
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) *reinterpret_cast<uint32_t*>(slot + (k >> 1) * 1024 + ((k & 1) ? ofs_odd : ofs_even)) = w[k];
}

// The chunks [c_begin, c_begin + n) of one tile into the part's slots, two
// chunks' TMEM loads per wait.
template <int EPI, bool NARROW, int REQ>
IVIT_DEV void epi_tile(uint32_t tbase, int c_begin, int n, const ChanConst& kc, const GemmArgs& args,
                       const int8_t* gelu_tab, uint8_t* slots, uint32_t ofs_even, uint32_t ofs_odd, uint32_t sel2,
                       uint32_t sel1) {
  const uint32_t t0 = tbase + (uint32_t)(16 * c_begin);
  int i = 0;
  for (; i + 1 < n; i += 2) {
    uint32_t ra[16], rb[16];
    tmem_ld16(t0 + (uint32_t)(16 * i), ra);
    tmem_ld16(t0 + (uint32_t)(16 * (i + 1)), rb);
    tmem_ld_wait_regs2(ra, rb);
    epi_chunk<EPI, NARROW, REQ>(ra, kc, args, gelu_tab, slots + i * kSlotBytes, ofs_even, ofs_odd, sel2, sel1);
    epi_chunk<EPI, NARROW, REQ>(rb, kc, args, gelu_tab, slots + (i + 1) * kSlotBytes, ofs_even, ofs_odd, sel2, sel1);
  }
  if (i < n) {
    uint32_t r[16];
    tmem_ld16(t0 + (uint32_t)(16 * i), r);
    tmem_ld_wait_regs(r);
    epi_chunk<EPI, NARROW, REQ>(r, kc, args, gelu_tab, slots + i * kSlotBytes, ofs_even, ofs_odd, sel2, sel1);
  }
}

// Named barrier of the four warps of one part (ids 1..kEpiParts) that also
// returns the AND of every thread's v, so the part gives up together.
IVIT_DEV bool part_bar_and(int part, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(1 + part)
      : "memory");
  return r != 0;
}

// Preload TMEM columns [16 c_begin, 16 c_end) of this warp's lanes in one
// accumulator buffer with the bias of the lane's output channel.
IVIT_DEV void bias_fill(uint32_t tbase, int c_begin, int c_end, int32_t bias) {
  for (int cc = c_begin; cc < c_end; ++cc) tmem_st16_fill(tbase + (uint32_t)(16 * cc), (uint32_t)bias);
}

template <int BN, int STAGES, int EPI, bool NARROW>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_i8_requant_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                           const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmS,
                           const GemmArgs args) {
  using L = GemmLayout<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* skip_full = drain + 1;  // [kEpiParts]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);
  int8_t* gelu_tab = reinterpret_cast<int8_t*>(smem + L::kGeluOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t M = args.M;
  const int N = args.N;
  const int ch_tiles = (N + kBM - 1) / kBM;
  const int tok_tiles = (int)((M + BN - 1) / BN);
  const int num_tiles = ch_tiles * tok_tiles;
  const int num_kb = (args.K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], L::kIssuers);  // one commit per issuing thread
      mbar_init(&tempty[a], kEpiWarps);
    }
    mbar_init(drain, L::kIssuers);
    for (int e = 0; e < kEpiParts; ++e) mbar_init(&skip_full[e], 1);
    fence_barrier_init();
    prefetch_tensormap(&tmW);
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmY);
    if (EPI == kEpiResidual) prefetch_tensormap(&tmS);
  }
  if (EPI == kEpiGelu) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x)
      gelu_tab[i] = (int8_t)shiftgelu8(i - 128, args.gelu.I0, args.gelu.M, args.gelu.k_out, args.gelu.out.b,
                                       args.gelu.out.c);
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(tslot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tslot;
  pdl_wait();  // X and the skip tensor come from earlier kernels
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued = 0;  // k-slices loaded so far by this CTA
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const int cb = t % ch_tiles, tb = t / ch_tiles;
        for (int kb = 0; kb < num_kb; ++kb, ++issued) {
          if (!mbar_wait(&empty[stage], phase ^ 1, args.status)) {
            ok = false;
            break;
          }
          // diagnostic (ivit_selftest_withhold): this k-slice is never loaded, so
          // the MMA issuer's bounded wait for it runs out
          if (issued == args.withhold && blockIdx.x == 0) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
          uint8_t* sa = smem + stage * L::kStageBytes;
          tma_load_2d(sa, &tmW, kb * kBK, cb * kBM, &full[stage]);
          tma_load_2d(sa + L::kABytes, &tmX, kb * kBK, tb * BN, &full[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else if (warp <= 2) {
    // ------------------------------------------------------------ MMA issuers
    if (lane == 0 && warp <= L::kIssuers) {
      constexpr int kStep = L::kIssuers;
      const uint32_t idesc = idesc_i8(kBM, BN, true, true, false);
      // descriptors of stage 0, k-step 0: a stage adds kStageBytes >> 4 to the
      // low half, the B tile kABytes >> 4 and a 32-byte k-step 2, so the issue
      // loop stays a handful of instructions per MMA
      const uint64_t d0 = smem_desc(smem_u32(smem), 16, 1024, kSwizzle128B);
      const uint32_t d_lo0 = (uint32_t)d0, d_hi = (uint32_t)(d0 >> 32);
      // this thread takes every kStep-th k-slice of the CTA's sequence,
      // starting with slice warp - 1; the ring position advances kStep stages
      // per slice
      int stage = warp - 1;
      uint32_t phase = 0;
      int kb0 = warp - 1;  // this thread's first k-slice within the current tile
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        // the buffer holds this tile's bias once the epilogue has drained it
        if (!mbar_wait(&tempty[acc], acc_phase, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * L::kAccCols);
        int kb = kb0;
        for (; kb < num_kb; kb += kStep) {
          if (!mbar_wait(&full[stage], phase, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_lo = d_lo0 + (uint32_t)(stage * (L::kStageBytes >> 4));
          const uint32_t b_lo = a_lo + (uint32_t)(L::kABytes >> 4);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)  // accumulate onto the preloaded bias
            umma_i8_acc(d_tmem, a_lo + 2 * k, d_hi, b_lo + 2 * k, d_hi, idesc);
          umma_commit(&empty[stage]);
          stage += kStep;
          if (stage >= STAGES) {
            stage -= STAGES;
            phase ^= 1;
          }
        }
        if (!ok) break;
        kb0 = kb - num_kb;
        // arrives once this thread's MMAs of the tile (possibly none) are done
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
    constexpr int kChunks = L::kChunks;
    const int e = warp - 3;
    const int quarter = warp & 3;  // TMEM lanes [32 q, 32 q + 32) = channels of this warp
    const int part = e >> 2;       // which of the quarter's warps: splits the token chunks
    const int c_begin = (kChunks * part) / kEpiParts;
    const int c_end = (kChunks * (part + 1)) / kEpiParts;
    const uint32_t sel2 = (lane & 2) ? 0x3276u : 0x5410u;
    const uint32_t sel1 = (lane & 1) ? 0x3715u : 0x6240u;
    const int sub = lane & 3;   // token offset within a transposed 4 x 4 block
    const int grp = lane >> 2;  // channel group of 4 within the warp's 32 channels
    // the part's first warp stages its skip tiles and stores its outputs
    const bool part_lead = (e & 3) == 0 && lane == 0;
    uint8_t* const slots0 = smem + L::kOutOff + part * L::kPartSlots;
    int set = 0;  // slot set of the current tile
    const uint32_t ofs_even = slot_ofs(sub, quarter, grp, 0), ofs_odd = slot_ofs(sub, quarter, grp, 1);
    uint64_t* sbar = &skip_full[part];
    const uint32_t tlane = tmem_base + ((uint32_t)(quarter * 32) << 16);
    auto bias_of = [&](int t) -> int32_t {
      const int ch = (t % ch_tiles) * kBM + quarter * 32 + lane;
      return (args.bias && ch < N) ? __ldg(args.bias + ch) : 0;
    };
    // both accumulator buffers start out holding the bias of their first tile
    for (int a = 0; a < 2; ++a) {
      const int t = (int)blockIdx.x + a * (int)gridDim.x;
      if (t < num_tiles) bias_fill(tlane + (uint32_t)(a * L::kAccCols), c_begin, c_end, bias_of(t));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[a]);
    }
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t skip_phase = 0;
    // Tile coordinates advance by gridDim.x tiles without divisions: (cb, tb)
    // of the current tile, cb1 / cb2 the channel blocks one and two tiles on.
    const int step_cb = (int)gridDim.x % ch_tiles, step_tb = (int)gridDim.x / ch_tiles;
    auto advance = [&](int& cbx, int& tbx) {
      cbx += step_cb;
      tbx += step_tb;
      if (cbx >= ch_tiles) {
        cbx -= ch_tiles;
        ++tbx;
      }
    };
    int cb = (int)blockIdx.x % ch_tiles, tb = (int)blockIdx.x / ch_tiles;
    int cb1 = cb, tb1 = tb;
    advance(cb1, tb1);
    int cb2 = cb1, tb2 = tb1;
    advance(cb2, tb2);
    // This lane's channel constants (multiplier, shift, bias) are loaded one
    // tile ahead and turned into the requant form at the end of the tile
    // before, so neither their L2 latency nor their derivation sits on a
    // tile's path.
    auto load_chan = [&](int t, int cbx, int32_t& cb_b, int32_t& cb_c, int32_t& cb_bias) {
      const int chx = cbx * kBM + quarter * 32 + lane;
      const bool ok = t < num_tiles && chx < N;
      cb_b = ok ? __ldg(args.b + chx) : 0;
      cb_c = ok ? (int32_t)__ldg(args.c + chx) : 0;
      cb_bias = (ok && args.bias) ? __ldg(args.bias + chx) : 0;
    };
    auto derive = [&](int cbx, int32_t vb, int32_t vc, int32_t vbias, ChanConst& kx, int& reqx) {
      kx = cbx * kBM + quarter * 32 + lane < N ? chan_const(vb, vc, vbias, args.K) : chan_const(0, 0, 0, args.K);
      // warp-uniform requant form
      reqx = __all_sync(0xffffffffu, kx.fast) ? kReqFast
                                               : (__any_sync(0xffffffffu, kx.needs_clamp) ? kReqWideClamp : kReqWide);
    };
    int32_t nb, nc, nbias;
    load_chan(blockIdx.x, cb, nb, nc, nbias);
    ChanConst kc;
    int req;
    derive(cb, nb, nc, nbias, kc, req);
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      load_chan(t + (int)gridDim.x, cb1, nb, nc, nbias);
      const int64_t tok_base = (int64_t)tb * BN;
      const int ch_next2 = cb2 * kBM + quarter * 32 + lane;
      const int32_t next_bias =
          (args.bias && ch_next2 < N && t + 2 * (int)gridDim.x < num_tiles) ? __ldg(args.bias + ch_next2) : 0;
      int n = c_end - c_begin;  // chunks that hold at least one real token
      while (n > 0 && tok_base + 16 * (c_begin + n - 1) >= M) --n;
      const bool live = n > 0;  // the same for the part's four warps
      const int tile_ch = cb * kBM;
      uint8_t* const slots = slots0 + set * L::kSetBytes;
      if (part_lead) {
        // the slots are free again once the stores of the tile that last used
        // them have read them: the previous tile (one set), or the one before
        // it (two sets; every tile commits one bulk group, possibly empty)
        if (L::kSlotSets == 2)
          bulk_wait_read_1();
        else
          bulk_wait_read_all();
        if (EPI == kEpiResidual && live) {
          mbar_arrive_expect_tx(sbar, (uint32_t)(n * kSlotBytes));
          for (int i = 0; i < n; ++i)
            tma_load_2d(slots + i * kSlotBytes, &tmS, tile_ch, (int32_t)(tok_base + 16 * (c_begin + i)), sbar);
        }
      }
      const bool got = mbar_wait(&tfull[acc], acc_phase, args.status);
      // the whole part has its accumulator and free slots, or gives up together
      if (!part_bar_and(part, got)) {
        // the skip loads issued above still write into the slots: let them
        // land (a bounded wait) before the CTA can release its shared memory
        if (EPI == kEpiResidual && live && part_lead) mbar_wait(sbar, skip_phase, args.status);
        break;
      }
      bool got_skip = true;
      if (EPI == kEpiResidual && live) {
        got_skip = mbar_wait(sbar, skip_phase, args.status);
        skip_phase ^= 1;
      }
      tc_fence_after();
      const uint32_t tbase = tlane + (uint32_t)(acc * L::kAccCols);
#define IVIT_EPI_TILE(R) \
  epi_tile<EPI, NARROW, R>(tbase, c_begin, n, kc, args, gelu_tab, slots, ofs_even, ofs_odd, sel2, sel1)
      if (!args.round) {
        if (req == kReqFast)
          IVIT_EPI_TILE(kReqFast);
        else if (req == kReqWide)
          IVIT_EPI_TILE(kReqWide);
        else
          IVIT_EPI_TILE(kReqWideClamp);
      } else {
        if (req == kReqFast)
          IVIT_EPI_TILE(kReqFast + kReqRound);
        else if (req == kReqWide)
          IVIT_EPI_TILE(kReqWide + kReqRound);
        else
          IVIT_EPI_TILE(kReqWideClamp + kReqRound);
      }
#undef IVIT_EPI_TILE
      // staged words -> global by TMA once the part's four warps have written
      // them (rows past M and channels past N are clipped)
      fence_proxy_async_smem();
      if (!part_bar_and(part, got_skip)) break;
      if (part_lead) {
        if (live)
          for (int i = 0; i < n; ++i)
            tma_store_2d(&tmY, tile_ch, (int32_t)(tok_base + 16 * (c_begin + i)), slots + i * kSlotBytes);
        bulk_commit_group();
      }
      if (L::kSlotSets == 2) set ^= 1;
      // preload the bias of the tile that next accumulates in this buffer
      if (t + 2 * (int)gridDim.x < num_tiles) bias_fill(tbase, c_begin, c_end, next_bias);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
      // the next tile's requant form, from constants loaded during this one
      derive(cb1, nb, nc, nbias, kc, req);
      cb = cb1;
      tb = tb1;
      cb1 = cb2;
      tb1 = tb2;
      advance(cb2, tb2);
    }
    if (part_lead) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Own-tile variant: three TMEM accumulators (tile widths up to 160 tokens),
// and each of the three epilogue parts drains whole tiles -- part p takes the
// CTA's tiles p, p + 3, ... -- instead of all three parts sharing every tile.
// A tile's epilogue carries a fixed latency (the wait for the accumulator,
// the part barriers, the stores and the bias refill) besides its arithmetic;
// with three tiles draining at once those latencies overlap.  Producer and
// MMA issuers are those of gemm_i8_requant_kernel with the accumulator index
// cycling over three buffers.
// ---------------------------------------------------------------------------
constexpr int kOwnAcc = 3;

template <int BN, int STAGES>
struct OwnLayout {
  static constexpr int kIssuers = (STAGES % 2 == 0) ? 2 : 1;
  static constexpr int kABytes = kBM * kBK;
  static constexpr int kBBytes = BN * kBK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kChunks = BN / 16;
  static constexpr int kOutOff = STAGES * kStageBytes;
  static constexpr int kPartSlots = kChunks * kSlotBytes;  // a whole tile per part
  static constexpr int kBarOff = kOutOff + kEpiParts * kPartSlots;
  // full, empty (STAGES each), tmem full / empty (three each), drain, one skip barrier per part
  static constexpr int kNumBars = 2 * STAGES + 2 * kOwnAcc + 1 + kEpiParts;
  static constexpr int kSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kGeluOff = kSlotOff + 16;
  static constexpr int kBytes = kGeluOff + 256;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr int kAccCols = (BN + 31) / 32 * 32;
  static_assert(kOwnAcc * kAccCols <= 512, "three accumulators must fit the TMEM columns");
  static_assert(kAlloc <= 227 * 1024, "shared memory budget");
};

template <int BN, int STAGES, int EPI, bool NARROW>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_own_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                    const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmS,
                    const GemmArgs args) {
  using L = OwnLayout<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;      // [3]
  uint64_t* tempty = tfull + kOwnAcc;    // [3]
  uint64_t* drain = tempty + kOwnAcc;
  uint64_t* skip_full = drain + 1;       // [kEpiParts]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);
  int8_t* gelu_tab = reinterpret_cast<int8_t*>(smem + L::kGeluOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t M = args.M;
  const int N = args.N;
  const int ch_tiles = (N + kBM - 1) / kBM;
  const int tok_tiles = (int)((M + BN - 1) / BN);
  const int num_tiles = ch_tiles * tok_tiles;
  const int num_kb = (args.K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < kOwnAcc; ++a) {
      mbar_init(&tfull[a], L::kIssuers);  // one commit per issuing thread
      mbar_init(&tempty[a], 4);           // the four warps of the part that owns the buffer
    }
    mbar_init(drain, L::kIssuers);
    for (int e = 0; e < kEpiParts; ++e) mbar_init(&skip_full[e], 1);
    fence_barrier_init();
    prefetch_tensormap(&tmW);
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmY);
    if (EPI == kEpiResidual) prefetch_tensormap(&tmS);
  }
  if (EPI == kEpiGelu) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x)
      gelu_tab[i] = (int8_t)shiftgelu8(i - 128, args.gelu.I0, args.gelu.M, args.gelu.k_out, args.gelu.out.b,
                                       args.gelu.out.c);
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tslot;
  pdl_wait();  // X and the skip tensor come from earlier kernels
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued = 0;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const int cb = t % ch_tiles, tb = t / ch_tiles;
        for (int kb = 0; kb < num_kb; ++kb, ++issued) {
          if (!mbar_wait(&empty[stage], phase ^ 1, args.status)) {
            ok = false;
            break;
          }
          if (issued == args.withhold && blockIdx.x == 0) {  // diagnostic (ivit_selftest_withhold)
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
          uint8_t* sa = smem + stage * L::kStageBytes;
          tma_load_2d(sa, &tmW, kb * kBK, cb * kBM, &full[stage]);
          tma_load_2d(sa + L::kABytes, &tmX, kb * kBK, tb * BN, &full[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else if (warp <= 2) {
    // ------------------------------------------------------------ MMA issuers
    if (lane == 0 && warp <= L::kIssuers) {
      constexpr int kStep = L::kIssuers;
      const uint32_t idesc = idesc_i8(kBM, BN, true, true, false);
      const uint64_t d0 = smem_desc(smem_u32(smem), 16, 1024, kSwizzle128B);
      const uint32_t d_lo0 = (uint32_t)d0, d_hi = (uint32_t)(d0 >> 32);
      int stage = warp - 1;
      uint32_t phase = 0;
      int kb0 = warp - 1;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * L::kAccCols);
        int kb = kb0;
        for (; kb < num_kb; kb += kStep) {
          if (!mbar_wait(&full[stage], phase, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_lo = d_lo0 + (uint32_t)(stage * (L::kStageBytes >> 4));
          const uint32_t b_lo = a_lo + (uint32_t)(L::kABytes >> 4);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k) umma_i8_acc(d_tmem, a_lo + 2 * k, d_hi, b_lo + 2 * k, d_hi, idesc);
          umma_commit(&empty[stage]);
          stage += kStep;
          if (stage >= STAGES) {
            stage -= STAGES;
            phase ^= 1;
          }
        }
        if (!ok) break;
        kb0 = kb - num_kb;
        umma_commit(&tfull[acc]);
        if (++acc == kOwnAcc) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      umma_commit(drain);
      mbar_wait(drain, 0, args.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    constexpr int kChunks = L::kChunks;
    const int e = warp - 3;
    const int quarter = warp & 3;
    const int part = e >> 2;  // owns accumulator `part` and the CTA's tiles part, part + 3, ...
    const uint32_t sel2 = (lane & 2) ? 0x3276u : 0x5410u;
    const uint32_t sel1 = (lane & 1) ? 0x3715u : 0x6240u;
    const int sub = lane & 3;
    const int grp = lane >> 2;
    const bool part_lead = (e & 3) == 0 && lane == 0;
    uint8_t* const slots = smem + L::kOutOff + part * L::kPartSlots;
    const uint32_t ofs_even = slot_ofs(sub, quarter, grp, 0), ofs_odd = slot_ofs(sub, quarter, grp, 1);
    uint64_t* sbar = &skip_full[part];
    const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(part * L::kAccCols);
    const int tstep = kOwnAcc * (int)gridDim.x;  // tiles between two of this part's tiles
    auto chan_of = [&](int t) { return (t % ch_tiles) * kBM + quarter * 32 + lane; };
    // the buffer starts out holding the bias of the part's first tile
    int t = (int)blockIdx.x + part * (int)gridDim.x;
    if (t < num_tiles) {
      const int ch = chan_of(t);
      bias_fill(tbase, 0, kChunks, (args.bias && ch < N) ? __ldg(args.bias + ch) : 0);
    }
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&tempty[part]);
    uint32_t acc_phase = 0;
    uint32_t skip_phase = 0;
    // this lane's channel constants, loaded one own tile ahead
    auto load_chan = [&](int tt, int32_t& vb, int32_t& vc, int32_t& vbias) {
      const int ch = chan_of(tt);
      const bool okc = tt < num_tiles && ch < N;
      vb = okc ? __ldg(args.b + ch) : 0;
      vc = okc ? (int32_t)__ldg(args.c + ch) : 0;
      vbias = (okc && args.bias) ? __ldg(args.bias + ch) : 0;
    };
    auto derive = [&](int tt, int32_t vb, int32_t vc, int32_t vbias, ChanConst& kx, int& reqx) {
      kx = chan_of(tt) < N ? chan_const(vb, vc, vbias, args.K) : chan_const(0, 0, 0, args.K);
      reqx = __all_sync(0xffffffffu, kx.fast) ? kReqFast
                                              : (__any_sync(0xffffffffu, kx.needs_clamp) ? kReqWideClamp : kReqWide);
    };
    int32_t nb, nc, nbias;
    load_chan(t, nb, nc, nbias);
    ChanConst kc;
    int req;
    derive(t, nb, nc, nbias, kc, req);
    for (; t < num_tiles; t += tstep) {
      const int tn = t + tstep;  // this part's next tile
      load_chan(tn, nb, nc, nbias);
      const int cb = t % ch_tiles, tb = t / ch_tiles;
      const int64_t tok_base = (int64_t)tb * BN;
      int n = kChunks;  // chunks that hold at least one real token
      while (n > 0 && tok_base + 16 * (n - 1) >= M) --n;
      const bool live = n > 0;
      const int tile_ch = cb * kBM;
      if (part_lead) {
        bulk_wait_read_all();  // the part's previous stores have read its slots
        if (EPI == kEpiResidual && live) {
          mbar_arrive_expect_tx(sbar, (uint32_t)(n * kSlotBytes));
          for (int i = 0; i < n; ++i)
            tma_load_2d(slots + i * kSlotBytes, &tmS, tile_ch, (int32_t)(tok_base + 16 * i), sbar);
        }
      }
      const bool got = mbar_wait(&tfull[part], acc_phase, args.status);
      if (!part_bar_and(part, got)) {
        if (EPI == kEpiResidual && live && part_lead) mbar_wait(sbar, skip_phase, args.status);
        break;
      }
      bool got_skip = true;
      if (EPI == kEpiResidual && live) {
        got_skip = mbar_wait(sbar, skip_phase, args.status);
        skip_phase ^= 1;
      }
      tc_fence_after();
#define IVIT_OWN_TILE(R) \
  epi_tile<EPI, NARROW, R>(tbase, 0, n, kc, args, gelu_tab, slots, ofs_even, ofs_odd, sel2, sel1)
      if (!args.round) {
        if (req == kReqFast)
          IVIT_OWN_TILE(kReqFast);
        else if (req == kReqWide)
          IVIT_OWN_TILE(kReqWide);
        else
          IVIT_OWN_TILE(kReqWideClamp);
      } else {
        if (req == kReqFast)
          IVIT_OWN_TILE(kReqFast + kReqRound);
        else if (req == kReqWide)
          IVIT_OWN_TILE(kReqWide + kReqRound);
        else
          IVIT_OWN_TILE(kReqWideClamp + kReqRound);
      }
#undef IVIT_OWN_TILE
      fence_proxy_async_smem();
      if (!part_bar_and(part, got_skip)) break;
      if (part_lead) {
        if (live)
          for (int i = 0; i < n; ++i)
            tma_store_2d(&tmY, tile_ch, (int32_t)(tok_base + 16 * i), slots + i * kSlotBytes);
        bulk_commit_group();
      }
      // the buffer takes the bias of the part's next tile
      if (tn < num_tiles) bias_fill(tbase, 0, kChunks, nbias);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[part]);
      acc_phase ^= 1;
      derive(tn, nb, nc, nbias, kc, req);
    }
    if (part_lead) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int BN, int STAGES, int EPI, bool NARROW>
ivit_status run_gemm_own(const DeviceCtx& dc, const int8_t* X, const int8_t* W, const int8_t* skip, int8_t* Y,
                         const GemmArgs& a, cudaStream_t stream) {
  using L = OwnLayout<BN, STAGES>;
  CUtensorMap tmW, tmX, tmY, tmS;
  ivit_status st = encode_tmap_2d_u8(&tmW, W, (uint64_t)a.K, (uint64_t)a.N, (uint64_t)a.K, kBK, kBM,
                                     CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != IVIT_OK) return st;
  st = encode_tmap_2d_u8(&tmX, X, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.K, kBK, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != IVIT_OK) return st;
  st = encode_tmap_2d_u8(&tmY, Y, (uint64_t)a.N, (uint64_t)a.M, (uint64_t)a.N, kBM, 16, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != IVIT_OK) return st;
  if (EPI == kEpiResidual) {
    st = encode_tmap_2d_u8(&tmS, skip, (uint64_t)a.N, (uint64_t)a.M, (uint64_t)a.N, kBM, 16,
                           CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != IVIT_OK) return st;
  } else {
    tmS = tmY;  // unused
  }
  auto kern = gemm_own_kernel<BN, STAGES, EPI, NARROW>;
  static bool attr_done = false;  // benign race: the attribute value is the same
  if (!attr_done) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) != cudaSuccess)
      return IVIT_ERR_CUDA;
    attr_done = true;
  }
  const int tiles = ((a.N + kBM - 1) / kBM) * (int)((a.M + BN - 1) / BN);
  const int grid = tiles < dc.num_sms ? tiles : dc.num_sms;
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kGemmThreads), L::kAlloc, stream, tmW, tmX, tmY, tmS, a);
  note_launch();
  return e == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}

template <int BN, int STAGES, int EPI, bool NARROW>
ivit_status run_gemm(const DeviceCtx& dc, const int8_t* X, const int8_t* W, const int8_t* skip, int8_t* Y,
                     const GemmArgs& a, cudaStream_t stream) {
  using L = GemmLayout<BN, STAGES>;
  static_assert(L::kAlloc <= 227 * 1024, "shared memory budget");
  CUtensorMap tmW, tmX, tmY, tmS;
  ivit_status st = encode_tmap_2d_u8(&tmW, W, (uint64_t)a.K, (uint64_t)a.N, (uint64_t)a.K, kBK, kBM,
                                     CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != IVIT_OK) return st;
  st = encode_tmap_2d_u8(&tmX, X, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.K, kBK, BN,
                         CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != IVIT_OK) return st;
  st = encode_tmap_2d_u8(&tmY, Y, (uint64_t)a.N, (uint64_t)a.M, (uint64_t)a.N, kBM, 16, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != IVIT_OK) return st;
  if (EPI == kEpiResidual) {
    st = encode_tmap_2d_u8(&tmS, skip, (uint64_t)a.N, (uint64_t)a.M, (uint64_t)a.N, kBM, 16,
                           CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != IVIT_OK) return st;
  } else {
    tmS = tmY;  // unused
  }
  auto kern = gemm_i8_requant_kernel<BN, STAGES, EPI, NARROW>;
  static bool attr_done = false;  // benign race: the attribute value is the same
  if (!attr_done) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) != cudaSuccess)
      return IVIT_ERR_CUDA;
    attr_done = true;
  }
  const int tiles = ((a.N + kBM - 1) / kBM) * (int)((a.M + BN - 1) / BN);
  const int grid = tiles < dc.num_sms ? tiles : dc.num_sms;
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kGemmThreads), L::kAlloc, stream, tmW, tmX, tmY, tmS, a);
  note_launch();
  return e == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}

// Token-tile width: the fewest rounds of tiles over the SMs, each round
// costing the tile width plus a fixed per-tile cost of about 112 token
// columns (channel constants, bias preload, accumulator hand-off, ring
// ramp), and 20 more at BN = 256, whose three-stage ring has one MMA issuer.
// Among widths with the same number of rounds the narrowest wins; a narrower
// width that needs one more round wins only when it is much narrower.  The
// two constants are fitted to per-kernel timings of the ViT-B, ViT-L,
// DeiT-S and ViT-B/384 layers on a B200 (148 SMs), where they reproduce
// every measured preference between widths.
int pick_bn(int64_t M, int N, int num_sms) {
  static const int cands[] = {256, 224, 192, 176, 160, 128};
  const int ch_tiles = (N + kBM - 1) / kBM;
  int best = 256;
  int64_t best_cost = INT64_MAX;
  for (int bn : cands) {
    const int64_t tiles = (int64_t)ch_tiles * ((M + bn - 1) / bn);
    const int64_t rounds = (tiles + num_sms - 1) / num_sms;
    const int64_t cost = rounds * (bn + 112 + (bn == 256 ? 20 : 0));
    if (cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

// Token-tile width of the own-tile variant (three accumulators: at most 160
// tokens), by the same cost model.
int pick_bn_own(int64_t M, int N, int num_sms) {
  static const int cands[] = {160, 144, 128};
  const int ch_tiles = (N + kBM - 1) / kBM;
  int best = 160;
  int64_t best_cost = INT64_MAX;
  for (int bn : cands) {
    const int64_t tiles = (int64_t)ch_tiles * ((M + bn - 1) / bn);
    const int64_t rounds = (tiles + num_sms - 1) / num_sms;
    const int64_t cost = rounds * (bn + 112);
    if (cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

// Whether the own-tile variant takes a GEMM: where the epilogue outweighs
// the MMAs of a tile -- a short reduction (K <= 512), or the ShiftGELU
// epilogue at K <= 768.  Same-box timings of the ViT-B, ViT-L and DeiT-S
// layers (us, shared-tile / own-tile): DeiT-S (K = 384) QKV 11.1 / 9.0,
// W^O 8.9 / 7.8, fc1 16.0 / 14.0; ViT-B fc1 30.1 / 27.5; but ViT-B QKV
// 18.8 / 20.3, W^O 13.0 / 13.5, fc2 25.9 / 29.9 and every ViT-L layer were
// slower (tiles of at most 160 tokens take an extra round of tiles there).
template <int EPI>
bool use_own_tiles(int K) {
  return K <= 512 || (EPI == kEpiGelu && K <= 768);
}

template <int EPI, bool NARROW>
ivit_status dispatch_bn(const DeviceCtx& dc, const int8_t* X, const int8_t* W, const int8_t* skip, int8_t* Y,
                        const GemmArgs& a, cudaStream_t stream) {
  if (use_own_tiles<EPI>(a.K)) {
    switch (pick_bn_own(a.M, a.N, dc.num_sms)) {
      case 160:
        return run_gemm_own<160, 4, EPI, NARROW>(dc, X, W, skip, Y, a, stream);
      case 144:
        return run_gemm_own<144, 4, EPI, NARROW>(dc, X, W, skip, Y, a, stream);
      default:
        return run_gemm_own<128, 4, EPI, NARROW>(dc, X, W, skip, Y, a, stream);
    }
  }
  switch (pick_bn(a.M, a.N, dc.num_sms)) {
    case 256:
      return run_gemm<256, 3, EPI, NARROW>(dc, X, W, skip, Y, a, stream);
    case 224:
      return run_gemm<224, 4, EPI, NARROW>(dc, X, W, skip, Y, a, stream);
    case 192:
      return run_gemm<192, 4, EPI, NARROW>(dc, X, W, skip, Y, a, stream);
    case 176:
      return run_gemm<176, 4, EPI, NARROW>(dc, X, W, skip, Y, a, stream);
    case 160:
      return run_gemm<160, 4, EPI, NARROW>(dc, X, W, skip, Y, a, stream);
    default:
      return run_gemm<128, 6, EPI, NARROW>(dc, X, W, skip, Y, a, stream);
  }
}

}  // namespace

ivit_status launch_gemm(const DeviceCtx& dc, const int8_t* X, int64_t M, int32_t K, const int8_t* W, int32_t N,
                        const int32_t* bias, const int32_t* b, const int8_t* c, int32_t out_bits, bool round,
                        EpiMode mode, const int8_t* skip, ivit_residual res, const GeluParams* gelu, int8_t* Y,
                        cudaStream_t stream) {
  GemmArgs a;
  a.round = round ? 1 : 0;
  a.M = M;
  a.N = N;
  a.K = K;
  a.bias = bias;
  a.b = b;
  a.c = c;
  a.lo = -(1 << (out_bits - 1));
  a.hi = (1 << (out_bits - 1)) - 1;
  a.res = res;
  a.gelu = gelu ? *gelu : GeluParams{1, 30, 8, {0, 0}};
  a.status = dc.status;
  a.withhold = take_withhold(kWithholdGemm);
  const bool narrow = out_bits < 8;
  switch (mode) {
    case kEpiPlain:
      return narrow ? dispatch_bn<kEpiPlain, true>(dc, X, W, skip, Y, a, stream)
                    : dispatch_bn<kEpiPlain, false>(dc, X, W, skip, Y, a, stream);
    case kEpiResidual:
      return narrow ? dispatch_bn<kEpiResidual, true>(dc, X, W, skip, Y, a, stream)
                    : dispatch_bn<kEpiResidual, false>(dc, X, W, skip, Y, a, stream);
    case kEpiGelu:
      return dispatch_bn<kEpiGelu, false>(dc, X, W, skip, Y, a, stream);
  }
  return IVIT_ERR_INTERNAL;
}

}  // namespace ivit
