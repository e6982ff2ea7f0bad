// ivit_attention.cu -- fused integer attention with Shiftmax on sm_100a.
//
// Per (128-query tile, head, image) one CTA of 16 warps computes
//   S = Q K^T                 tcgen05.mma kind::i8 (s8 x s8 -> s32) into TMEM
//   L = sat_ks((b_s S) >> c_s)  dyadic logit requant, row max     (CUDA cores)
//   P = Shiftmax(L)           ShiftExp table + IntDiv, u8 probabilities
//   O = P V                   tcgen05.mma kind::i8 (u8 x s8 -> s32) into TMEM
//   ctx = sat_8((b_o O) >> c_o)
// following "I-ViT: Integer-only Quantization for Efficient Vision Transformer
// Inference", sections 3.2-3.3, and the Trio-ViT article, eqs. (1)-(3).  The
// score matrix stays on chip: S in TMEM, k_s-bit logits and u8 P in shared
// memory.  The four warps w, w + 4, w + 8, w + 12 share TMEM lane quarter
// w & 3 (query rows 32 (w & 3) .. + 31) and split every row's keys: each
// reads a quarter of the score columns, keeps a partial row maximum and sum,
// and the four partials of a row meet in shared memory.
//
// Shared memory (runtime N, keys padded to 64 for loads and 32 for the MMAs):
//   R0  Q (128 x 64 B) and K (N64 x 64 B), 64B swizzle; later reused for P
//       (128 x N32 u8, K-major, 128B swizzle, 16 KB per 128 keys)
//   V   (N64 x 64 B), 64B swizzle, read MN-major by the P V MMA
//   logits (128 rows x lstride B), exp table (2^k_s int32), the row
//   partials (4 x 128 maxima, 4 x 128 sums), barriers
#include <climits>

#include "ivit_common.cuh"
#include "ivit_internal.h"

namespace ivit {
namespace {

constexpr int kAttnSplit = 4;                   // threads (warps of one lane quarter) per query row
constexpr int kAttnThreads = 128 * kAttnSplit;  // 16 warps
constexpr int kQTile = 128;
constexpr int kHeadDim = 64;
constexpr int kMaxKeys = 640;
constexpr int kTmemCols = 256;

struct AttnArgs {
  int32_t B, N, H;
  int32_t logit_b, logit_c, ks_lo, ks_hi, k_s;
  int32_t I0, M, k_out;
  int32_t out_b, out_c;
  int32_t o_lo, o_hi;  // accumulator clamp of the output requant (see out_clamp)
  int32_t out_bq;      // b_o 2^(32 - c_o) when that fits a positive int32 (then the requant is one mul.hi), else 0
  int32_t out_fast;
  uint32_t exp_magic;  // ceil(2^32 / I0) for the arithmetic ShiftExp of logits wider than 8 bits (0 when I0 = 1)
  int8_t* ctx;
  int* status;
  int32_t withhold;  // diagnostic: CTA 0's producer stops before this local item (-1: never)
};

struct AttnLayout {
  int n64, n32, kblocks, lstride;
  int r0_bytes, v_off, logit_off, tab_off, part_off, bar_off, total;
};

__host__ __device__ inline AttnLayout attn_layout(int N) {
  AttnLayout L;
  L.n64 = (N + 63) / 64 * 64;
  L.n32 = (N + 31) / 32 * 32;
  L.kblocks = (L.n32 + 127) / 128;
  int ls = (N + 15) / 16 * 16;
  if (((ls / 16) & 1) == 0) ls += 16;  // odd multiple of 16 B: conflict-free 16 B row accesses
  L.lstride = ls;
  const int qk = kQTile * kHeadDim + L.n64 * kHeadDim;
  const int p = L.kblocks * 128 * 128;
  L.r0_bytes = (qk > p ? qk : p + 0);
  L.r0_bytes = (L.r0_bytes + 1023) / 1024 * 1024;
  L.v_off = L.r0_bytes;
  L.logit_off = L.v_off + (L.n64 * kHeadDim + 1023) / 1024 * 1024;
  L.tab_off = L.logit_off + kQTile * L.lstride;
  L.part_off = (L.tab_off + 256 * 4 + 15) / 16 * 16;
  L.bar_off = L.part_off + 2 * kAttnSplit * kQTile * 4;
  L.total = L.bar_off + 64;
  return L;
}

// 4-bit log2 code of a 16-bit probability P16 (scale 2^-15): 15 -
// round(log2 P16), clipped to [0, 15]; P16 = 0 gives 15.  round(log2 P) of an
// integer P >= 1 is floor(log2 P) + 1 exactly when P^2 >= 2^(2 floor(log2 P) + 1).
IVIT_DEV uint32_t lis_code(uint32_t p16) {
  if (p16 == 0u) return 15u;
  const uint32_t fl = 31u - (uint32_t)__clz((int)p16);
  const uint32_t r = fl + ((p16 * p16 >= (1u << (2 * fl + 1))) ? 1u : 0u);  // p16 <= 2^15: no overflow
  return r >= 15u ? 0u : 15u - r;
}

// FASTQ: the logit requant is one mul.hi by bq = b_s 2^(32 - c_s), exact
// when b_s < 2^(c_s - 1), then the k_s-bit saturation.
// LIS: Log-Int-Softmax instead of Shiftmax (see ivit_attention_lis): the row's
// 16-bit probabilities become 4-bit log2 codes k, and P V is the bit shift
// sum_j V_j 2^(15 - k_j), computed as two u8 x s8 MMAs over the planes
// 2^(7 - k) (k <= 7) and 2^(15 - k) (k >= 8), combined as 256 hi + lo.
template <bool FASTQ, bool LIS>
__global__ void __launch_bounds__(kAttnThreads)
    attention_shiftmax_kernel(const __grid_constant__ CUtensorMap tm, const AttnArgs a, const int32_t bq) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int N = a.N;
  const AttnLayout L = attn_layout(N);
  uint8_t* r0 = smem;
  uint8_t* sQ = r0;
  uint8_t* sK = r0 + kQTile * kHeadDim;
  uint8_t* sP = r0;
  uint8_t* sV = smem + L.v_off;
  int8_t* slog = reinterpret_cast<int8_t*>(smem + L.logit_off);
  int32_t* tab = reinterpret_cast<int32_t*>(smem + L.tab_off);
  uint64_t* bar_qk = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* bar_v = bar_qk + 1;
  uint64_t* bar_s = bar_qk + 2;  // [2]: S chunk in TMEM buffer b
  uint64_t* bar_o = bar_qk + 4;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar_qk + 5);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int q0 = blockIdx.x * kQTile;
  const int h = blockIdx.y;
  const int img = blockIdx.z;
  const int D = a.H * kHeadDim;
  const int row0 = img * N;  // first token row of this image in qkv / ctx
  const int nload = L.n64 / 64;
  // S is computed in chunks of up to 256 keys; with more than one chunk, two
  // TMEM buffers let the next chunk's MMA run while this one is requantised
  // (the launcher then keeps one CTA per SM, so the 512 columns are free)
  const int nchunks = (L.n32 + 255) / 256;
  const bool dbuf = nchunks >= 2;
  const uint32_t tcols = dbuf ? 2u * kTmemCols : (uint32_t)kTmemCols;

  if (tid == 0) {
    mbar_init(bar_qk, 1);
    mbar_init(bar_v, 1);
    mbar_init(&bar_s[0], 1);
    mbar_init(&bar_s[1], 1);
    mbar_init(bar_o, 1);
    fence_barrier_init();
    prefetch_tensormap(&tm);
  }
  // ShiftExp table over I_delta = -t, t in [0, 2^k_s)
  for (int t = tid; t < (1 << a.k_s); t += kAttnThreads) tab[t] = shift_exp(-t, a.I0);
  if (warp == 0) {
    __syncwarp();
    tmem_alloc(tslot, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  pdl_wait();  // Q, K and V come from the previous kernel
  pdl_launch_dependents();

  if (tid == 0) {
    mbar_arrive_expect_tx(bar_qk, (uint32_t)(kQTile * kHeadDim + nload * 64 * kHeadDim));
    tma_load_2d(sQ, &tm, h * kHeadDim, row0 + q0, bar_qk);
    tma_load_2d(sQ + 64 * kHeadDim, &tm, h * kHeadDim, row0 + q0 + 64, bar_qk);
    for (int i = 0; i < nload; ++i) tma_load_2d(sK + i * 64 * kHeadDim, &tm, D + h * kHeadDim, row0 + 64 * i, bar_qk);
    mbar_arrive_expect_tx(bar_v, (uint32_t)(nload * 64 * kHeadDim));
    for (int i = 0; i < nload; ++i)
      tma_load_2d(sV + i * 64 * kHeadDim, &tm, 2 * D + h * kHeadDim, row0 + 64 * i, bar_v);
  }

  bool ok = true;
  const int quarter = warp & 3;           // TMEM lane quarter: query rows 32 quarter .. + 31
  const int slice = warp >> 2;            // which quarter of every row's keys this thread takes
  const int row = quarter * 32 + (tid & 31);
  int32_t mx = a.ks_lo;
  int8_t* my_log = slog + row * L.lstride;
  const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
  int32_t* part_max = reinterpret_cast<int32_t*>(smem + L.part_off);  // [slice][row]
  uint32_t* part_sum = reinterpret_cast<uint32_t*>(part_max + kAttnSplit * kQTile);

  // ---- S = Q K^T in chunks of up to 256 keys, requantised to k_s-bit logits;
  // the chunk's 32-column groups go round-robin to the four slices.  Chunk c
  // lands in buffer c & 1 (dbuf) and completes phase (c >> 1) & 1 of
  // bar_s[c & 1]: one commit in flight per barrier.
  auto chunk_width = [&](int c) { return (L.n32 - c * 256) < 256 ? (L.n32 - c * 256) : 256; };
  auto issue_s = [&](int c) {  // tid 0 only
    tc_fence_after();
    const uint32_t idesc = idesc_i8(kQTile, chunk_width(c), true, true, false);
    const uint32_t qa = smem_u32(sQ);
    const uint32_t kb = smem_u32(sK + c * 256 * kHeadDim);
    const uint32_t dst = tmem + (dbuf ? (uint32_t)((c & 1) * kTmemCols) : 0u);
#pragma unroll
    for (int k = 0; k < kHeadDim / 32; ++k)
      umma_i8(dst, smem_desc(qa + k * 32, 16, 512, kSwizzle64B), smem_desc(kb + k * 32, 16, 512, kSwizzle64B), idesc,
              k != 0);
    umma_commit(&bar_s[c & 1]);
  };
  if (tid == 0) {
    if (!mbar_wait(bar_qk, 0, a.status)) ok = false;
    if (ok) issue_s(0);
  }
  for (int c = 0; c < nchunks; ++c) {
    const int w = chunk_width(c);
    // the other buffer's previous chunk was read before the last __syncthreads
    if (tid == 0 && ok && dbuf && c + 1 < nchunks) issue_s(c + 1);
    if (!mbar_wait(&bar_s[c & 1], (uint32_t)((c >> 1) & 1), a.status)) ok = false;
    ok = __all_sync(0xffffffffu, ok);  // warp-uniform: guards a warp-collective TMEM load
    tc_fence_after();
    if (ok) {
      const uint32_t t_buf = t_lane + (dbuf ? (uint32_t)((c & 1) * kTmemCols) : 0u);
      for (int cc = slice; cc < w / 32; cc += kAttnSplit) {
        uint32_t r[32];
        tmem_ld32(t_buf + (uint32_t)(cc * 32), r);
        tmem_ld_wait();
        const int j0 = c * 256 + cc * 32;
        uint32_t packed[8];
#pragma unroll
        for (int wd = 0; wd < 8; ++wd) {
          uint32_t word = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = wd * 4 + e;
            const int32_t l =
                FASTQ ? min(max(__mulhi(bq, (int32_t)r[i]), a.ks_lo), a.ks_hi)
                      : requant_bits((int32_t)r[i], a.logit_b, a.logit_c, a.ks_lo, a.ks_hi);
            if (j0 + i < N) mx = l > mx ? l : mx;
            word |= ((uint32_t)l & 0xFFu) << (8 * e);
          }
          packed[wd] = word;
        }
        // logits row is lstride >= round16(N) bytes; j0 + 32 <= n32 may pass it
        if (j0 < L.lstride)
          *reinterpret_cast<int4*>(my_log + j0) = make_int4(packed[0], packed[1], packed[2], packed[3]);
        if (j0 + 16 < L.lstride)
          *reinterpret_cast<int4*>(my_log + j0 + 16) = make_int4(packed[4], packed[5], packed[6], packed[7]);
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  // the row maximum from the four slices' partial maxima
  part_max[slice * kQTile + row] = mx;
  __syncthreads();
  mx = max(max(part_max[row], part_max[kQTile + row]), max(part_max[2 * kQTile + row], part_max[3 * kQTile + row]));

  // ---- Shiftmax row sum: e_j = ShiftExp(L_j - max) by table, over this
  // slice's 16-key units u = slice, slice + 4, ...
  // (after a timed-out wait the logits are not written: skip to zero P)
  uint32_t sum = 0;
  const int nfull = ok ? N / 16 : 0;
  for (int u = slice; u < nfull; u += kAttnSplit) {
    const int4 v = *reinterpret_cast<const int4*>(my_log + u * 16);
    const int8_t* lb = reinterpret_cast<const int8_t*>(&v);
#pragma unroll
    for (int e = 0; e < 16; ++e) sum += (uint32_t)tab[mx - (int32_t)lb[e]];
  }
  if (ok && (nfull % kAttnSplit) == slice)  // the ragged last unit
    for (int j = nfull * 16; j < N; ++j) sum += (uint32_t)tab[mx - (int32_t)my_log[j]];
  part_sum[slice * kQTile + row] = sum;
  __syncthreads();
  sum = (part_sum[row] + part_sum[kQTile + row]) + (part_sum[2 * kQTile + row] + part_sum[3 * kQTile + row]);
  if (sum == 0) sum = 1;
  const uint32_t dv = (1u << a.M) / sum;
  const int pshift = a.M - (a.k_out - 1);

  // ---- P as u8 into the K-major 128B-swizzled operand; this slice's 16-key
  // units (zero past the last key).  Shiftmax: P = (Dv e_j) >> (M - k_out + 1).
  // LIS: plane `plane` of the code k_j of P16 = (Dv e_j) >> (M - 15).
  const int rlo = row & 7;
  uint8_t* prow = sP + (row >> 3) * 1024 + rlo * 128;
  auto write_p = [&](int plane) {
    fence_proxy_async_smem();
    for (int u = slice; u < L.n32 / 16; u += kAttnSplit) {
      const int j0 = u * 16;
      uint32_t packed[4] = {0, 0, 0, 0};
      if (ok && j0 < N) {
        const int4 v = *reinterpret_cast<const int4*>(my_log + j0);
        const int8_t* lb = reinterpret_cast<const int8_t*>(&v);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          uint32_t p = 0u;
          if (j0 + e < N) {
            const uint32_t ev = (uint32_t)tab[mx - (int32_t)lb[e]];
            if (!LIS) {
              p = (dv * ev) >> pshift;
            } else {
              const uint32_t k = lis_code((dv * ev) >> (a.M - 15));
              p = plane == 0 ? (k <= 7u ? 1u << (7u - k) : 0u) : (k >= 8u ? 1u << (15u - k) : 0u);
            }
          }
          packed[e >> 2] |= p << (8 * (e & 3));
        }
      }
      const int kb = j0 >> 7;
      const int ch = (j0 & 127) >> 4;
      *reinterpret_cast<int4*>(prow + kb * 16384 + ((ch ^ rlo) << 4)) =
          make_int4(packed[0], packed[1], packed[2], packed[3]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
  };
  // ---- O = P V (one commit phase of bar_o per product)
  auto pv = [&](int phase) {
    if (tid == 0 && ok) {
      if (phase == 0 && !mbar_wait(bar_v, 0, a.status)) ok = false;
      if (ok) {
        tc_fence_after();
        const uint32_t idesc = idesc_i8(kQTile, kHeadDim, false, true, true);
        const uint32_t pa = smem_u32(sP);
        const uint32_t va = smem_u32(sV);
        for (int k = 0; k < L.n32 / 32; ++k) {
          const uint64_t da = smem_desc(pa + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024, kSwizzle128B);
          const uint64_t db = smem_desc(va + k * 32 * kHeadDim, 512, 512, kSwizzle64B);
          umma_i8(tmem, da, db, idesc, k != 0);
        }
      }
      umma_commit(bar_o);
    }
    if (!mbar_wait(bar_o, (uint32_t)phase, a.status)) ok = false;
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
  };
  write_p(0);
  pv(0);
  // slice s reads columns [16 s, 16 s + 16) of O
  uint32_t r[16];
  tmem_ld16(t_lane + (uint32_t)(slice * 16), r);
  tmem_ld_wait_regs(r);
  uint32_t rlo16[16];
  if (LIS) {
    // the low plane's product replaces the high one's in the same columns,
    // once every thread has read the high one
    tc_fence_before();
    __syncthreads();
    write_p(1);
    pv(1);
    tmem_ld16(t_lane + (uint32_t)(slice * 16), rlo16);
    tmem_ld_wait_regs(rlo16);
  }

  // ---- ctx = sat_8((b_o O) >> c_o); slice s writes columns [16 s, 16 s + 16)
  {
    const int q = q0 + row;
    if (ok && q < N) {
      int8_t* dst = a.ctx + (int64_t)(row0 + q) * D + h * kHeadDim + slice * 16;
      uint32_t packed[4];
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) {
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int32_t y;
          if (!LIS) {
            y = requant8((int32_t)r[wd * 4 + e], a.out_b, a.out_c);
          } else {
            // acc = sum_j V_j 2^(15 - k_j) = 256 hi + lo, |acc| < 2^32; (b_o acc) >> c_o in 64 bits
            const int64_t acc = 256 * (int64_t)(int32_t)r[wd * 4 + e] + (int64_t)(int32_t)rlo16[wd * 4 + e];
            const int64_t v = ((int64_t)a.out_b * acc) >> a.out_c;
            y = (int32_t)(v < -128 ? -128 : (v > 127 ? 127 : v));
          }
          word |= ((uint32_t)y & 0xFFu) << (8 * e);
        }
        packed[wd] = word;
      }
      *reinterpret_cast<int4*>(dst) = make_int4(packed[0], packed[1], packed[2], packed[3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

// ---------------------------------------------------------------------------
// Short sequences (N <= 256 keys): persistent, warp-specialised kernel.
//
// One CTA per SM walks the work items (128-query tile, head, image) with
// stride gridDim.x; local item j of a CTA belongs to softmax group j & 1.
//   warp 0      TMA producer: Q, K and V of item j into stage j % 3 of a
//               three-stage ring; a stage is released when P V of its item
//               has completed, so loads run up to two items ahead;
//   warp 1      S issuer: S = Q K^T of item j into TMEM buffer j & 1 once
//               that buffer is free and the stage has landed;
//   warp 2      P V issuer: P V of item j once its P is in shared memory.
//               Two issuing threads, each blocked on its own next event, so
//               neither softmax group waits behind the other;
//   warps 3-18  two softmax groups of eight warps;
//   warps 19-22 output readout, one per TMEM lane quarter: each item's
//               ctx = sat_8((b_o O) >> c_o), in item order, while the
//               softmax groups go on with their next items.
// S = Q K^T is N = round16(N) columns wide.
// Within an item the score row never leaves TMEM: pass 1 takes the row
// maximum of the raw int32 scores (the logit requant is monotone, so
// max L = requant(max S)); pass 2 requantises each score, looks up
// ShiftExp(L - max L) in a table replicated once per shared-memory bank (lane
// l reads copy l, so lookups never conflict), sums the row and writes the
// exponentials back into TMEM in place; pass 3 turns them into
// u8 P = (Dv e) >> (M - k_out + 1), written into the group's own
// 128B-swizzled K-major P operand.  Warps w and w + 4 of a group share TMEM
// lanes (query rows) and split the key columns; their partial maxima and sums
// meet in shared memory behind a named barrier of the group's 256 threads.
// P V lands in a 64-column region of its own when two S buffers and it fit
// the 512 TMEM columns (N <= 224), else in the first 64 columns of the
// item's S buffer, dead by then.
// ---------------------------------------------------------------------------
constexpr int kShortMaxKeys = 256;
constexpr int kTableMaxBits = 8;  // ShiftExp by table up to 8-bit logits, computed beyond

// The arithmetic ShiftExp divides n = -I_p by I0 with one mul.hi, exact while
// n I0 < 2^32.  Over k_s-bit logits |L - max L| <= 2^k_s - 1 = m, and
// -I_p = m' + ceil(m'/2) - ceil(m'/16) at |d| = m' never decreases in m', so
// its largest value is at m' = m.
inline bool shift_exp_alu_exact(int32_t k_s, int32_t I0) {
  const int64_t m = ((int64_t)1 << k_s) - 1;
  const int64_t nmax = m + (m + 1) / 2 - (m + 15) / 16;
  return nmax * (int64_t)I0 < ((int64_t)1 << 32);
}
constexpr int kRowSplit = 2;     // warps (per lane quarter) that split a query row's keys (3 measured slower)
constexpr int kSoftWarps = 4 * kRowSplit;  // per softmax group
constexpr int kSoftGroups = 2;   // groups take alternate items, one TMEM buffer each
constexpr int kLoadStages = 3;
constexpr int kReadWarps = 4;    // output readout, one per TMEM lane quarter
constexpr int kPersistThreads = 96 + 32 * kSoftWarps * kSoftGroups + 32 * kReadWarps;

struct PersistLayout {
  int n64, n32, n16, kblocks;
  int sbuf;    // TMEM column stride of the two S buffers
  int o_col;   // first TMEM column of the P V output when it has a region of its own, else -1
  int k_off, v_off, stage_bytes;  // Q at 0, K, V within a stage
  int p_off, p_bytes, tab_off, part_off, bar_off, total;
};

__host__ __device__ inline PersistLayout persist_layout(int N) {
  PersistLayout L;
  L.n64 = (N + 63) / 64 * 64;
  L.n32 = (N + 31) / 32 * 32;
  L.n16 = (N + 15) / 16 * 16;
  L.kblocks = (L.n32 + 127) / 128;
  // Two S buffers of n32 columns and a 64-column region for P V fit the 512
  // TMEM columns while n32 <= 224: a group then frees its S buffer as soon as
  // P is written, and the next S MMA overlaps P V and the output requant.
  // Beyond that P V lands in the first 64 columns of the item's S buffer.
  const bool sep = 2 * L.n32 + kHeadDim <= 512;
  L.sbuf = sep ? L.n32 : 256;
  L.o_col = sep ? 2 * L.n32 : -1;
  L.k_off = kQTile * kHeadDim;             // 8 KB
  L.v_off = L.k_off + L.n64 * kHeadDim;    // + a multiple of 4 KB
  L.stage_bytes = L.v_off + L.n64 * kHeadDim;
  L.p_off = kLoadStages * L.stage_bytes;   // a multiple of 4 KB
  L.p_bytes = L.kblocks * 128 * 128;       // 16 KB per 128 keys
  L.tab_off = L.p_off + kSoftGroups * L.p_bytes;
  L.part_off = L.tab_off + 256 * 32 * 4;
  L.bar_off = L.part_off + kSoftGroups * kRowSplit * 2 * kQTile * 4;
  L.total = L.bar_off + 24 * 8;
  return L;
}

// bytes [sat8(y0), sat8(y1), sat8(y2), sat8(y3)]
IVIT_DEV uint32_t pack_sat4_attn(int32_t y0, int32_t y1, int32_t y2, int32_t y3) {
  uint32_t t, d;
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(t) : "r"(y3), "r"(y2), "r"(0u));
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(y1), "r"(y0), "r"(t));
  return d;
}

// floor(b S / 2^c) before the k_s-bit saturation: one mul.hi when
// bq = b 2^(32 - c) fits a positive int32
template <bool FASTQ>
IVIT_DEV int32_t logit_unclamped(int32_t S, int32_t bq, int32_t b, int32_t c) {
  if (FASTQ) return __mulhi(bq, S);
  const int64_t q = ((int64_t)b * (int64_t)S) >> c;
  return (int32_t)(q < (int64_t)INT_MIN ? (int64_t)INT_MIN : (q > (int64_t)INT_MAX ? (int64_t)INT_MAX : q));
}

// bounded wait that also gives up at once when another thread has aborted
IVIT_DEV bool wait_or_abort(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitBudgetNs) {
      report_timeout(status);
      *abort_flag = 1;
      return false;
    }
  }
}

// named barrier of one softmax group (ids 1 and 2; 256 threads each)
IVIT_DEV void softmax_bar(int group) { asm volatile("bar.sync %0, %1;" ::"r"(1 + group), "n"(32 * kSoftWarps) : "memory"); }

// Streams n 16-column chunks of this warp's TMEM lanes starting at taddr,
// body(r, k) on chunk k.  Single-buffered: with 23 warps a thread has at
// most 80 registers, and the other softmax warps cover the load latency.
template <typename F>
IVIT_DEV void tmem_stream16(uint32_t taddr, int n, F&& body) {
  uint32_t r[16];
  for (int k = 0; k < n; ++k) {
    tmem_ld16(taddr + (uint32_t)(16 * k), r);
    tmem_ld_wait_regs(r);
    body(r, k);
  }
}

// As tmem_stream16 with two chunks' loads per wait, for the passes whose
// per-chunk work is light enough to keep 32 columns in registers.
template <typename F>
IVIT_DEV void tmem_stream16x2(uint32_t taddr, int n, F&& body) {
  int k = 0;
  for (; k + 1 < n; k += 2) {
    uint32_t ra[16], rb[16];
    tmem_ld16(taddr + (uint32_t)(16 * k), ra);
    tmem_ld16(taddr + (uint32_t)(16 * (k + 1)), rb);
    tmem_ld_wait_regs2(ra, rb);
    body(ra, k);
    body(rb, k + 1);
  }
  if (k < n) {
    uint32_t r[16];
    tmem_ld16(taddr + (uint32_t)(16 * k), r);
    tmem_ld_wait_regs(r);
    body(r, k);
  }
}

// ShiftExp(d), d <= 0, computed: the same steps as shift_exp, with the floor
// division of n = -I_p by I0 done as one mul.hi by ceil(2^32 / I0), which is
// exact while n I0 < 2^32 (the host checks that bound for the logit width;
// I0 = 1 divides by itself).
IVIT_DEV uint32_t shift_exp_alu(int32_t d, int32_t I0, uint32_t magic) {
  const int32_t ip = d + (d >> 1) - (d >> 4);
  const uint32_t n = (uint32_t)(-ip);
  const uint32_t q = magic != 0u ? __umulhi(n, magic) : n;
  const int32_t r = (int32_t)(n - q * (uint32_t)I0);
  const int32_t t = I0 - ((r + 1) >> 1);  // I0 + floor(-r / 2) >= 1
  return (uint32_t)t >> min(q, 31u);      // t < 2^31: a shift by 31 gives 0, as every q >= 31 must
}

// Pass 2 of one half row: e = ShiftExp(L - max L) by table (ALU: computed),
// written back to TMEM in place; returns the partial row sum.  tb = table +
// lane + 32 lmax, so tb[-32 L] = ShiftExp(L - lmax).  UPPER: some row of the
// warp has a raw logit maximum above the k_s-bit range, so the upper
// saturation is needed (otherwise every logit of the row is at most lmax
// already).
template <bool FASTQ, bool UPPER, bool ALU>
IVIT_DEV uint32_t shiftmax_pass2(uint32_t t_row, int cbase, int nvalid, int N, const int32_t* tb, int32_t lmax,
                                 int32_t bq, const AttnArgs& a) {
  uint32_t s4[4] = {0u, 0u, 0u, 0u};
  tmem_stream16(t_row + (uint32_t)cbase, nvalid, [&](uint32_t(&r)[16], int k) {
    const int col = cbase + 16 * k;
    const int lim = N - col;
    if (lim >= 16) {
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        int32_t l = max(logit_unclamped<FASTQ>((int32_t)r[e], bq, a.logit_b, a.logit_c), a.ks_lo);
        if (UPPER || !FASTQ) l = min(l, a.ks_hi);
        const uint32_t x = ALU ? shift_exp_alu(l - lmax, a.I0, a.exp_magic) : (uint32_t)tb[-32 * l];
        s4[e & 3] += x;
        r[e] = x;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        // padding keys: any index in range, then masked
        const int32_t l = min(max(logit_unclamped<FASTQ>((int32_t)r[e], bq, a.logit_b, a.logit_c), a.ks_lo), lmax);
        const uint32_t x = e < lim ? (ALU ? shift_exp_alu(l - lmax, a.I0, a.exp_magic) : (uint32_t)tb[-32 * l]) : 0u;
        s4[e & 3] += x;
        r[e] = x;
      }
    }
    tmem_st16(t_row + (uint32_t)col, r);
  });
  tmem_st_wait();
  return (s4[0] + s4[1]) + (s4[2] + s4[3]);
}

// ALU: logits wider than 8 bits, ShiftExp computed per score instead of
// looked up (the table would not fit).
template <bool FASTQ, bool ALU>
__global__ void __launch_bounds__(kPersistThreads, 1)
    attention_persist_kernel(const __grid_constant__ CUtensorMap tm, const AttnArgs a, const int32_t bq) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int N = a.N;
  const PersistLayout L = persist_layout(N);
  int32_t* tab = reinterpret_cast<int32_t*>(smem + L.tab_off);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* qkv_full = bars + 0;      // [3] Q, K and V of a stage landed
  uint64_t* stage_empty = bars + 3;   // [3] stage reusable (P V of its item done)
  uint64_t* s_full = bars + 6;        // [2] S in TMEM buffer g
  uint64_t* p_full = bars + 8;        // [2] P of group g in shared memory (one arrival per warp)
  uint64_t* o_full = bars + 10;       // [2] P V of group g's item in TMEM
  uint64_t* tmem_empty = bars + 12;   // [2] S buffer g reusable
  uint64_t* drain = bars + 14;        // all MMAs of the CTA complete (one commit per issuer)
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 15);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 16);
  uint64_t* o_empty = bars + 17;      // separate P V region read out (one arrival per readout warp)
  const bool sep_o = L.o_col >= 0;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int D = a.H * kHeadDim;
  const int qtiles = (N + kQTile - 1) / kQTile;
  const int n_items = qtiles * a.H * a.B;
  const int nload = L.n64 / 64;

  if (tid == 0) {
    for (int s = 0; s < kLoadStages; ++s) {
      mbar_init(&qkv_full[s], 1);
      mbar_init(&stage_empty[s], 1);
    }
    for (int g = 0; g < kSoftGroups; ++g) {
      mbar_init(&s_full[g], 1);
      mbar_init(&p_full[g], kSoftWarps);
      mbar_init(&o_full[g], 1);
      // freed by the softmax warps once P is written (separate P V region),
      // else by the readout warps once the output in it is read
      mbar_init(&tmem_empty[g], sep_o ? kSoftWarps : kReadWarps);
    }
    mbar_init(drain, 2);
    mbar_init(o_empty, kReadWarps);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tm);
  }
  // replicated ShiftExp table, tab[t * 32 + l] = ShiftExp(-t) for every lane l:
  // one evaluation per entry (staged in the partials area), then copies in
  // consecutive 16-byte chunks
  int32_t* stage_t = reinterpret_cast<int32_t*>(smem + L.part_off);
  if (!ALU && tid < (1 << a.k_s)) stage_t[tid] = shift_exp(-tid, a.I0);
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  for (int i4 = tid; !ALU && i4 < (8 << a.k_s); i4 += kPersistThreads) {
    const int32_t e = stage_t[i4 >> 3];
    reinterpret_cast<int4*>(tab)[i4] = make_int4(e, e, e, e);
  }
  __syncthreads();
  const uint32_t tmem = *tslot;
  pdl_wait();  // Q, K and V come from the previous kernel
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int j = 0;
      for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++j) {
        const int s = j % kLoadStages;
        const uint32_t ph = (uint32_t)((j / kLoadStages) & 1);
        if (!wait_or_abort(&stage_empty[s], ph ^ 1, a.status, abort_flag)) break;
        // diagnostic (ivit_selftest_withhold): the item's loads are never issued,
        // so the S issuer's bounded wait for them runs out
        if (j == a.withhold && blockIdx.x == 0) break;
        const int qt = item % qtiles, h = (item / qtiles) % a.H, img = item / (qtiles * a.H);
        const int row0 = img * N;
        uint8_t* st = smem + s * L.stage_bytes;
        mbar_arrive_expect_tx(&qkv_full[s], (uint32_t)(kQTile * kHeadDim + 2 * nload * 64 * kHeadDim));
        tma_load_2d(st, &tm, h * kHeadDim, row0 + qt * kQTile, &qkv_full[s]);
        tma_load_2d(st + 64 * kHeadDim, &tm, h * kHeadDim, row0 + qt * kQTile + 64, &qkv_full[s]);
        for (int i = 0; i < nload; ++i)
          tma_load_2d(st + L.k_off + i * 64 * kHeadDim, &tm, D + h * kHeadDim, row0 + 64 * i, &qkv_full[s]);
        for (int i = 0; i < nload; ++i)
          tma_load_2d(st + L.v_off + i * 64 * kHeadDim, &tm, 2 * D + h * kHeadDim, row0 + 64 * i, &qkv_full[s]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_i8(kQTile, L.n16, true, true, false);
      const int n_local = n_items > (int)blockIdx.x ? (n_items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
      for (int j = 0; j < n_local; ++j) {
        const int g = j & 1, s = j % kLoadStages;
        if (!wait_or_abort(&tmem_empty[g], (uint32_t)(((j >> 1) & 1) ^ 1), a.status, abort_flag)) break;
        if (!wait_or_abort(&qkv_full[s], (uint32_t)((j / kLoadStages) & 1), a.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t qa = smem_u32(smem + s * L.stage_bytes);
        const uint32_t ka = qa + L.k_off;
#pragma unroll
        for (int k = 0; k < kHeadDim / 32; ++k)
          umma_i8(tmem + (uint32_t)(g * L.sbuf), smem_desc(qa + k * 32, 16, 512, kSwizzle64B),
                  smem_desc(ka + k * 32, 16, 512, kSwizzle64B), idesc_s, k != 0);
        umma_commit(&s_full[g]);
      }
      // every MMA of this thread has completed before TMEM is released
      umma_commit(drain);
      mbar_wait(drain, 0, a.status);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ P V issuer
    if (lane == 0) {
      const uint32_t idesc_o = idesc_i8(kQTile, kHeadDim, false, true, true);
      const int n_local = n_items > (int)blockIdx.x ? (n_items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
      for (int j = 0; j < n_local; ++j) {
        const int g = j & 1, s = j % kLoadStages;
        if (!wait_or_abort(&p_full[g], (uint32_t)((j >> 1) & 1), a.status, abort_flag)) break;
        // the shared P V region is free once the previous item's output is read
        if (sep_o && j > 0 && !wait_or_abort(o_empty, (uint32_t)((j - 1) & 1), a.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t pa = smem_u32(smem + L.p_off + g * L.p_bytes);
        const uint32_t va = smem_u32(smem + s * L.stage_bytes + L.v_off);
        const uint32_t d_o = tmem + (uint32_t)(sep_o ? L.o_col : g * L.sbuf);
        for (int k = 0; k < L.n32 / 32; ++k)
          umma_i8(d_o, smem_desc(pa + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024, kSwizzle128B),
                  smem_desc(va + k * 32 * kHeadDim, 512, 512, kSwizzle64B), idesc_o, k != 0);
        umma_commit(&o_full[g]);
        umma_commit(&stage_empty[s]);
      }
      umma_commit(drain);
    }
  } else if (warp < 3 + kSoftWarps * kSoftGroups) {
    // ------------------------------------------------------------ softmax warps
    const int sw = warp - 3;
    const int group = sw / kSoftWarps;   // handles local items j with j % 2 == group
    const int quarter = warp & 3;
    const int half = (sw >> 2) % kRowSplit;  // which slice of the row's key chunks
    const int row = quarter * 32 + lane;  // query row of the tile = TMEM lane
    const int nc32 = L.n32 / 16;          // 16-key chunks of the MMA-padded row
    const int c_lo = (nc32 * half) / kRowSplit, c_hi = (nc32 * (half + 1)) / kRowSplit;
    const int cbase = 16 * c_lo;
    const int nch = c_hi - c_lo;
    int nvalid = 0;  // chunks of this half that hold at least one real key
    while (nvalid < nch && cbase + 16 * nvalid < N) ++nvalid;
    // [slice][max, sum][128 rows]
    int32_t* part = reinterpret_cast<int32_t*>(smem + L.part_off) + group * (kRowSplit * 2 * kQTile);
    const int rlo = row & 7;
    uint8_t* prow = smem + L.p_off + group * L.p_bytes + (row >> 3) * 1024 + rlo * 128;
    const uint32_t t_row = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(group * L.sbuf);
    const int pshift = a.M - (a.k_out - 1);
    bool ok = true;
    int j = group;
    // item = qt + qtiles (h + H img), advanced by a fixed step without divisions
    const int first = blockIdx.x + group * gridDim.x;
    const int step = kSoftGroups * gridDim.x;
    int qt = first % qtiles, h = (first / qtiles) % a.H, img = first / (qtiles * a.H);
    const int st_q = step % qtiles, st_h = (step / qtiles) % a.H, st_i = step / (qtiles * a.H);
    for (int item = first; item < n_items; item += step, j += 2) {
      const uint32_t ph = (uint32_t)((j >> 1) & 1);
      const int q0 = qt * kQTile;
      if (ok) ok = wait_or_abort(&s_full[group], ph, a.status, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      // warps whose rows all lie past the image's last token skip the passes
      const bool work = ok && (q0 + quarter * 32 < N);

      // ---- pass 1: row maximum of the raw scores over the real keys
      int32_t m4[4] = {INT_MIN, INT_MIN, INT_MIN, INT_MIN};
      if (work) {
        tmem_stream16x2(t_row + (uint32_t)cbase, nvalid, [&](uint32_t(&r)[16], int k) {
          const int lim = N - (cbase + 16 * k);
          if (lim >= 16) {
#pragma unroll
            for (int e = 0; e < 16; ++e) m4[e & 3] = max(m4[e & 3], (int32_t)r[e]);
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if (e < lim) m4[e & 3] = max(m4[e & 3], (int32_t)r[e]);
          }
        });
      }
      int32_t smax = max(max(m4[0], m4[1]), max(m4[2], m4[3]));
      part[half * 2 * kQTile + row] = smax;
      softmax_bar(group);
      smax = part[row];
#pragma unroll
      for (int sl = 1; sl < kRowSplit; ++sl) smax = max(smax, part[sl * 2 * kQTile + row]);
      const int32_t vmax = logit_unclamped<FASTQ>(smax, bq, a.logit_b, a.logit_c);
      const int32_t lmax = min(max(vmax, a.ks_lo), a.ks_hi);

      // ---- pass 2: e = ShiftExp(L - max L) back into TMEM, row sum
      uint32_t sum = 0;
      if (work) {
        const int32_t* tb = tab + lane + lmax * 32;
        if (__any_sync(0xffffffffu, vmax > a.ks_hi))
          sum = shiftmax_pass2<FASTQ, true, ALU>(t_row, cbase, nvalid, N, tb, lmax, bq, a);
        else
          sum = shiftmax_pass2<FASTQ, false, ALU>(t_row, cbase, nvalid, N, tb, lmax, bq, a);
      }
      part[half * 2 * kQTile + kQTile + row] = (int32_t)sum;
      softmax_bar(group);
      sum = 0;
#pragma unroll
      for (int sl = 0; sl < kRowSplit; ++sl) sum += (uint32_t)part[sl * 2 * kQTile + kQTile + row];
      if (sum == 0) sum = 1;  // rows that skipped the passes
      const uint32_t dv = (1u << a.M) / sum;

      // ---- pass 3: P = (Dv e) >> (M - k_out + 1) into the group's swizzled operand,
      // once the P V of the group's previous item (which read the previous P)
      // has completed
      if (j >= 2) {
        if (ok) ok = wait_or_abort(&o_full[group], (uint32_t)(((j >> 1) - 1) & 1), a.status, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
      }
      if (work && ok) {
        // (Dv e) >> pshift is one mul.hi by Dv 2^(32 - pshift) when Dv < 2^pshift
        const bool hip = pshift >= 1 && __all_sync(0xffffffffu, (uint64_t)dv < ((uint64_t)1 << pshift));
        const uint32_t dvh = hip ? dv << (32 - pshift) : 0u;
        tmem_stream16x2(t_row + (uint32_t)cbase, nvalid, [&](uint32_t(&r)[16], int k) {
          const int col = cbase + 16 * k;
          uint32_t w[4];
          if (hip) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              w[q] = __umulhi(dvh, r[4 * q]) + __umulhi(dvh, r[4 * q + 1]) * 256u +
                     __umulhi(dvh, r[4 * q + 2]) * 65536u + __umulhi(dvh, r[4 * q + 3]) * 16777216u;
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              w[q] = ((dv * r[4 * q]) >> pshift) + ((dv * r[4 * q + 1]) >> pshift) * 256u +
                     ((dv * r[4 * q + 2]) >> pshift) * 65536u + ((dv * r[4 * q + 3]) >> pshift) * 16777216u;
          }
          *reinterpret_cast<int4*>(prow + (col >> 7) * 16384 + ((((col & 127) >> 4) ^ rlo) << 4)) =
              make_int4((int)w[0], (int)w[1], (int)w[2], (int)w[3]);
        });
      }
      // chunks of padding keys (and every chunk of a skipped warp): P = 0
      for (int k = work ? nvalid : 0; k < nch; ++k) {
        const int col = cbase + 16 * k;
        *reinterpret_cast<int4*>(prow + (col >> 7) * 16384 + ((((col & 127) >> 4) ^ rlo) << 4)) =
            make_int4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&p_full[group]);
        if (sep_o) mbar_arrive(&tmem_empty[group]);  // S is consumed: the next S may land
      }

      qt += st_q;
      if (qt >= qtiles) {
        qt -= qtiles;
        ++h;
      }
      h += st_h;
      if (h >= a.H) {
        h -= a.H;
        ++img;
      }
      img += st_i;
    }
  } else {
    // ------------------------------------------------------------ readout warps
    // ctx = sat_8((b_o O) >> c_o) of every local item in order, while the
    // softmax groups go on with their next items; each warp reads the 64
    // output columns of its lane quarter's 32 query rows
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int n_local = n_items > (int)blockIdx.x ? (n_items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    bool ok = true;
    for (int j = 0; j < n_local; ++j) {
      const int g = j & 1;
      const int item = (int)blockIdx.x + j * (int)gridDim.x;
      const int qt = item % qtiles, h = (item / qtiles) % a.H, img = item / (qtiles * a.H);
      if (ok) ok = wait_or_abort(&o_full[g], (uint32_t)((j >> 1) & 1), a.status, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      const int q = qt * kQTile + row;
      if (ok && qt * kQTile + quarter * 32 < N) {  // the quarter holds at least one real row
        const uint32_t t_out =
            tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(sep_o ? L.o_col : g * L.sbuf);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          uint32_t ra[16], rb[16];
          tmem_ld16(t_out + (uint32_t)(32 * part), ra);
          tmem_ld16(t_out + (uint32_t)(32 * part + 16), rb);
          tmem_ld_wait_regs2(ra, rb);
          if (q < N) {
            uint32_t packed[8];
#pragma unroll
            for (int wd = 0; wd < 8; ++wd) {
              int32_t y[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int32_t acc = (int32_t)(wd < 4 ? ra[wd * 4 + e] : rb[(wd - 4) * 4 + e]);
                if (a.out_fast) {
                  y[e] = __mulhi(a.out_bq, acc);  // floor(b_o acc / 2^c_o), exact
                } else {
                  const int32_t ac = min(max(acc, a.o_lo), a.o_hi);
                  const int64_t v = (int64_t)a.out_b * ac;  // |v >> c| < 2^31 after the clamp
                  y[e] = (int32_t)__funnelshift_r((uint32_t)v, (uint32_t)(v >> 32), (uint32_t)a.out_c);
                }
              }
              packed[wd] = pack_sat4_attn(y[0], y[1], y[2], y[3]);
            }
            int8_t* dst = a.ctx + (int64_t)(img * N + q) * D + h * kHeadDim + part * 32;
            reinterpret_cast<int4*>(dst)[0] = make_int4(packed[0], packed[1], packed[2], packed[3]);
            reinterpret_cast<int4*>(dst)[1] = make_int4(packed[4], packed[5], packed[6], packed[7]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sep_o ? o_empty : &tmem_empty[g]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool attention_config_supported(int32_t N, int32_t k_s, int32_t I0) {
  if (N > kMaxKeys) return false;
  return k_s <= kTableMaxBits || (N <= kShortMaxKeys && shift_exp_alu_exact(k_s, I0));
}

ivit_status launch_attention(const DeviceCtx& dc, const int8_t* qkv, int32_t B, int32_t N, int32_t H,
                             ivit_dyadic logit, int32_t k_s, int32_t I0, int32_t M, int32_t k_out,
                             ivit_dyadic out, int8_t* ctx, cudaStream_t stream, bool lis) {
  if (B == 0 || N == 0) return IVIT_OK;
  if (N > kMaxKeys) return IVIT_ERR_UNSUPPORTED;
  const int64_t T = (int64_t)B * N;
  const int D = H * kHeadDim;
  CUtensorMap tm;
  ivit_status st = encode_tmap_2d_u8(&tm, qkv, (uint64_t)(3 * D), (uint64_t)T, (uint64_t)(3 * D), 64, 64,
                                     CU_TENSOR_MAP_SWIZZLE_64B);
  if (st != IVIT_OK) return st;
  AttnArgs a;
  a.B = B;
  a.N = N;
  a.H = H;
  a.logit_b = logit.b;
  a.logit_c = logit.c;
  a.k_s = k_s;
  a.ks_lo = -(1 << (k_s - 1));
  a.ks_hi = (1 << (k_s - 1)) - 1;
  a.I0 = I0;
  a.M = M;
  a.k_out = k_out;
  a.out_b = out.b;
  a.out_c = out.c;
  {
    // acc in [-u, u] with u = 128 / 2^s (2^s <= b / 2^c < 2^(s+1)) keeps every
    // unsaturated result, saturates the rest the same way and keeps
    // (b acc) >> c within int32
    if (out.b == 0) {
      a.o_lo = INT_MIN;
      a.o_hi = INT_MAX;
    } else {
      int bl = 0;
      while (bl < 31 && (out.b >> bl) != 0) ++bl;
      const int sh = bl - 1 - out.c;
      const int64_t u = sh >= 7 ? 1 : (sh >= 0 ? (128 >> sh) : ((int64_t)128 << (-sh)));
      a.o_hi = (int32_t)(u > INT_MAX ? INT_MAX : u);
      a.o_lo = -a.o_hi;
    }
  }
  a.out_fast = out.c >= 1 && (int64_t)out.b < ((int64_t)1 << (out.c - 1));
  a.out_bq = a.out_fast ? (int32_t)((int64_t)out.b << (32 - out.c)) : 0;
  // logits wider than 8 bits: arithmetic ShiftExp on the short-sequence path only
  const bool alu = k_s > kTableMaxBits;
  if (!attention_config_supported(N, k_s, I0)) return IVIT_ERR_UNSUPPORTED;
  a.exp_magic = I0 > 1 ? (uint32_t)((((uint64_t)1 << 32) + (uint64_t)I0 - 1) / (uint64_t)I0) : 0u;
  a.ctx = ctx;
  a.status = dc.status;
  a.withhold = N <= kShortMaxKeys && !lis ? take_withhold(kWithholdAttention) : -1;
  dim3 grid((unsigned)((N + kQTile - 1) / kQTile), (unsigned)H, (unsigned)B);
  if (N <= kShortMaxKeys && !lis) {
    const PersistLayout P = persist_layout(N);
    const int smem = P.total + 1024;
    // bq = b 2^(32 - c) when it fits a positive int32: the logit requant is then one mul.hi
    const bool fastq = logit.c >= 1 && (int64_t)logit.b < ((int64_t)1 << (logit.c - 1));
    const int32_t bq = fastq ? (int32_t)((int64_t)logit.b << (32 - logit.c)) : 0;
    static bool attr_persist = false;
    if (!attr_persist) {
      if (cudaFuncSetAttribute(attention_persist_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               227 * 1024) != cudaSuccess ||
          cudaFuncSetAttribute(attention_persist_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               227 * 1024) != cudaSuccess ||
          cudaFuncSetAttribute(attention_persist_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               227 * 1024) != cudaSuccess ||
          cudaFuncSetAttribute(attention_persist_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               227 * 1024) != cudaSuccess)
        return IVIT_ERR_CUDA;
      attr_persist = true;
    }
    const int64_t items = (int64_t)((N + kQTile - 1) / kQTile) * H * B;
    if (items > 0x7fffffff) return IVIT_ERR_UNSUPPORTED;
    const unsigned pgrid = (unsigned)(items < dc.num_sms ? items : dc.num_sms);
    auto kern = fastq ? (alu ? attention_persist_kernel<true, true> : attention_persist_kernel<true, false>)
                      : (alu ? attention_persist_kernel<false, true> : attention_persist_kernel<false, false>);
    const cudaError_t e = launch_pdl(kern, dim3(pgrid), dim3(kPersistThreads), smem, stream, tm, a, bq);
    note_launch();
    return e == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
  }
  const AttnLayout L = attn_layout(N);
  // at most two CTAs per SM, so that their TMEM (256 columns each) always
  // fits; one CTA per SM when S takes two 256-column buffers (N > 256)
  int smem = L.total + 1024;
  if (smem < 80 * 1024) smem = 80 * 1024;
  if (L.n32 > 256 && smem < 116 * 1024) smem = 116 * 1024;
  static int attr_bytes = 0;
  if (smem > attr_bytes) {
    if (cudaFuncSetAttribute(attention_shiftmax_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             227 * 1024) != cudaSuccess ||
        cudaFuncSetAttribute(attention_shiftmax_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             227 * 1024) != cudaSuccess ||
        cudaFuncSetAttribute(attention_shiftmax_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             227 * 1024) != cudaSuccess ||
        cudaFuncSetAttribute(attention_shiftmax_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             227 * 1024) != cudaSuccess)
      return IVIT_ERR_CUDA;
    attr_bytes = 227 * 1024;
  }
  // bq = b 2^(32 - c) when it fits a positive int32: the logit requant is then one mul.hi
  const bool fastq_long = logit.c >= 1 && (int64_t)logit.b < ((int64_t)1 << (logit.c - 1));
  const int32_t bq_long = fastq_long ? (int32_t)((int64_t)logit.b << (32 - logit.c)) : 0;
  auto kern = fastq_long ? (lis ? attention_shiftmax_kernel<true, true> : attention_shiftmax_kernel<true, false>)
                         : (lis ? attention_shiftmax_kernel<false, true> : attention_shiftmax_kernel<false, false>);
  const cudaError_t e = launch_pdl(kern, grid, dim3(kAttnThreads), smem, stream, tm, a, bq_long);
  note_launch();
  return e == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}

}  // namespace ivit
