// ivit_attention.cu -- fused integer attention with Shiftmax on sm_100a.
//
// Per (128-query tile, head, image) one CTA of 4 warps computes
//   S = Q K^T                 tcgen05.mma kind::i8 (s8 x s8 -> s32) into TMEM
//   L = sat_ks((b_s S) >> c_s)  dyadic logit requant, row max     (CUDA cores)
//   P = Shiftmax(L)           ShiftExp table + IntDiv, u8 probabilities
//   O = P V                   tcgen05.mma kind::i8 (u8 x s8 -> s32) into TMEM
//   ctx = sat_8((b_o O) >> c_o)
// following "I-ViT: Integer-only Quantization for Efficient Vision Transformer
// Inference", sections 3.2-3.3, and the Trio-ViT article, eqs. (1)-(3).  The
// score matrix stays on chip: S in TMEM, k_s-bit logits and u8 P in shared
// memory.  Thread t owns query row t of the tile (TMEM lane t), so the row
// reductions need no shuffles.
//
// Shared memory (runtime N, keys padded to 64 for loads and 32 for the MMAs):
//   R0  Q (128 x 64 B) and K (N64 x 64 B), 64B swizzle; later reused for P
//       (128 x N32 u8, K-major, 128B swizzle, 16 KB per 128 keys)
//   V   (N64 x 64 B), 64B swizzle, read MN-major by the P V MMA
//   logits (128 rows x lstride B), exp table (2^k_s int32), barriers
#include <climits>

#include "ivit_common.cuh"
#include "ivit_internal.h"

namespace ivit {
namespace {

constexpr int kAttnThreads = 128;
constexpr int kQTile = 128;
constexpr int kHeadDim = 64;
constexpr int kMaxKeys = 640;
constexpr int kTmemCols = 256;

struct AttnArgs {
  int32_t B, N, H;
  int32_t logit_b, logit_c, ks_lo, ks_hi, k_s;
  int32_t I0, M, k_out;
  int32_t out_b, out_c;
  int8_t* ctx;
  int* status;
};

struct AttnLayout {
  int n64, n32, kblocks, lstride;
  int r0_bytes, v_off, logit_off, tab_off, bar_off, total;
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
  L.bar_off = (L.tab_off + 256 * 4 + 15) / 16 * 16;
  L.total = L.bar_off + 64;
  return L;
}

__global__ void __launch_bounds__(kAttnThreads)
    attention_shiftmax_kernel(const __grid_constant__ CUtensorMap tm, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
  uint64_t* bar_s = bar_qk + 2;
  uint64_t* bar_o = bar_qk + 3;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar_qk + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int q0 = blockIdx.x * kQTile;
  const int h = blockIdx.y;
  const int img = blockIdx.z;
  const int D = a.H * kHeadDim;
  const int row0 = img * N;  // first token row of this image in qkv / ctx
  const int nload = L.n64 / 64;

  if (tid == 0) {
    mbar_init(bar_qk, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_barrier_init();
    prefetch_tensormap(&tm);
  }
  // ShiftExp table over I_delta = -t, t in [0, 2^k_s)
  for (int t = tid; t < (1 << a.k_s); t += kAttnThreads) tab[t] = shift_exp(-t, a.I0);
  if (warp == 0) {
    __syncwarp();
    tmem_alloc(tslot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

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
  int32_t mx = a.ks_lo;
  int8_t* my_log = slog + tid * L.lstride;
  const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);

  // ---- S = Q K^T in chunks of up to 256 keys, requantised to k_s-bit logits
  const int nchunks = (L.n32 + 255) / 256;
  for (int c = 0; c < nchunks; ++c) {
    const int w = (L.n32 - c * 256) < 256 ? (L.n32 - c * 256) : 256;
    if (tid == 0 && ok) {
      if (c == 0 && !mbar_wait(bar_qk, 0, a.status)) ok = false;
      if (ok) {
        tc_fence_after();
        const uint32_t idesc = idesc_i8(kQTile, w, true, true, false);
        const uint32_t qa = smem_u32(sQ);
        const uint32_t kb = smem_u32(sK + c * 256 * kHeadDim);
#pragma unroll
        for (int k = 0; k < kHeadDim / 32; ++k)
          umma_i8(tmem, smem_desc(qa + k * 32, 16, 512, kSwizzle64B), smem_desc(kb + k * 32, 16, 512, kSwizzle64B),
                  idesc, k != 0);
        umma_commit(bar_s);
      }
    }
    if (!mbar_wait(bar_s, (uint32_t)(c & 1), a.status)) ok = false;
    ok = __all_sync(0xffffffffu, ok);  // warp-uniform: guards a warp-collective TMEM load
    tc_fence_after();
    if (ok) {
      for (int cc = 0; cc < w / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(t_lane + (uint32_t)(cc * 32), r);
        tmem_ld_wait();
        const int j0 = c * 256 + cc * 32;
        uint32_t packed[8];
#pragma unroll
        for (int wd = 0; wd < 8; ++wd) {
          uint32_t word = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = wd * 4 + e;
            const int32_t l = requant_bits((int32_t)r[i], a.logit_b, a.logit_c, a.ks_lo, a.ks_hi);
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

  // ---- Shiftmax row sum: e_j = ShiftExp(L_j - max) by table
  // (after a timed-out wait the logits are not written: skip to zero P)
  uint32_t sum = 0;
  const int nfull = ok ? N / 16 : 0;
  for (int cidx = 0; cidx < nfull; ++cidx) {
    const int4 v = *reinterpret_cast<const int4*>(my_log + cidx * 16);
    const int8_t* lb = reinterpret_cast<const int8_t*>(&v);
#pragma unroll
    for (int e = 0; e < 16; ++e) sum += (uint32_t)tab[mx - (int32_t)lb[e]];
  }
  if (ok)
    for (int j = nfull * 16; j < N; ++j) sum += (uint32_t)tab[mx - (int32_t)my_log[j]];
  if (sum == 0) sum = 1;
  const uint32_t dv = (1u << a.M) / sum;
  const int pshift = a.M - (a.k_out - 1);

  // ---- P = (Dv e_j) >> (M - k_out + 1) as u8, into the K-major 128B-swizzled operand
  fence_proxy_async_smem();
  const int rlo = tid & 7;
  uint8_t* prow = sP + (tid >> 3) * 1024 + rlo * 128;
  for (int cidx = 0; cidx < L.n32 / 16; ++cidx) {
    const int j0 = cidx * 16;
    uint32_t packed[4] = {0, 0, 0, 0};
    if (ok && j0 < N) {
      const int4 v = *reinterpret_cast<const int4*>(my_log + j0);
      const int8_t* lb = reinterpret_cast<const int8_t*>(&v);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const uint32_t p = (j0 + e < N) ? (dv * (uint32_t)tab[mx - (int32_t)lb[e]]) >> pshift : 0u;
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

  // ---- O = P V
  if (tid == 0 && ok) {
    if (!mbar_wait(bar_v, 0, a.status)) ok = false;
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
  if (!mbar_wait(bar_o, 0, a.status)) ok = false;
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after();

  // ---- ctx = sat_8((b_o O) >> c_o)
  {
    uint32_t r0v[32], r1v[32];
    tmem_ld32(t_lane, r0v);
    tmem_ld32(t_lane + 32, r1v);
    tmem_ld_wait();
    const int q = q0 + tid;
    if (ok && q < N) {
      int8_t* dst = a.ctx + (int64_t)(row0 + q) * D + h * kHeadDim;
      uint32_t packed[16];
#pragma unroll
      for (int wd = 0; wd < 16; ++wd) {
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = wd * 4 + e;
          const int32_t acc = (int32_t)(i < 32 ? r0v[i] : r1v[i - 32]);
          word |= ((uint32_t)requant8(acc, a.out_b, a.out_c) & 0xFFu) << (8 * e);
        }
        packed[wd] = word;
      }
#pragma unroll
      for (int v = 0; v < 4; ++v)
        reinterpret_cast<int4*>(dst)[v] =
            make_int4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Short sequences (N <= 256 keys): the whole score row stays in TMEM.
//
// 8 warps; warps w and w + 4 read the same TMEM lanes (query rows) and split
// the key columns in two halves.  Pass 1 takes the row maximum of the raw
// int32 scores (the logit requant is monotone, so max L = requant(max S)).
// Pass 2 requantises each score, looks up ShiftExp(L - max L) in a table
// replicated once per shared-memory bank (lane l reads copy l: no bank
// conflicts), accumulates the row sum and writes the exponentials back into
// TMEM in place.  Pass 3 turns them into u8 P = (Dv e) >> (M - k_out + 1),
// written straight into the 128B-swizzled K-major operand of the P V MMA.
// ---------------------------------------------------------------------------
constexpr int kShortThreads = 256;
constexpr int kShortMaxKeys = 256;

struct ShortLayout {
  int n64, n32, kblocks;
  int r0_bytes, v_off, tab_off, part_off, bar_off, total;
};

__host__ __device__ inline ShortLayout short_layout(int N) {
  ShortLayout L;
  L.n64 = (N + 63) / 64 * 64;
  L.n32 = (N + 31) / 32 * 32;
  L.kblocks = (L.n32 + 127) / 128;
  const int qk = kQTile * kHeadDim + L.n64 * kHeadDim;
  const int p = L.kblocks * 128 * 128;
  L.r0_bytes = ((qk > p ? qk : p) + 1023) / 1024 * 1024;
  L.v_off = L.r0_bytes;
  L.tab_off = L.v_off + (L.n64 * kHeadDim + 1023) / 1024 * 1024;
  L.part_off = L.tab_off + 256 * 32 * 4;
  L.bar_off = L.part_off + 2 * 2 * kQTile * 4;
  L.total = L.bar_off + 64;
  return L;
}

// sat_ks(floor(b S / 2^c)): one mul.hi when b 2^(32-c) fits a positive int32
template <bool FASTQ>
IVIT_DEV int32_t logit_requant(int32_t S, int32_t bq, int32_t b, int32_t c, int32_t lo, int32_t hi) {
  if (FASTQ) {
    const int32_t v = __mulhi(bq, S);  // floor(bq S / 2^32), bq = b 2^(32 - c)
    return min(max(v, lo), hi);
  } else {
    return requant_bits(S, b, c, lo, hi);
  }
}

template <bool FASTQ>
__global__ void __launch_bounds__(kShortThreads, 2)
    attention_short_kernel(const __grid_constant__ CUtensorMap tm, const AttnArgs a, const int32_t bq) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int N = a.N;
  const ShortLayout L = short_layout(N);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kQTile * kHeadDim;
  uint8_t* sP = smem;
  uint8_t* sV = smem + L.v_off;
  int32_t* tab = reinterpret_cast<int32_t*>(smem + L.tab_off);
  int32_t* part = reinterpret_cast<int32_t*>(smem + L.part_off);  // [half][max, sum][128 rows]
  uint64_t* bar_qk = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* bar_v = bar_qk + 1;
  uint64_t* bar_s = bar_qk + 2;
  uint64_t* bar_o = bar_qk + 3;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar_qk + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int quarter = warp & 3;
  const int half = warp >> 2;
  const int row = quarter * 32 + lane;  // query row of the tile = TMEM lane
  const int q0 = blockIdx.x * kQTile;
  const int h = blockIdx.y;
  const int img = blockIdx.z;
  const int D = a.H * kHeadDim;
  const int row0 = img * N;
  const int nload = L.n64 / 64;
  const int hcols = L.n32 / 2;  // key columns per half (multiple of 16)

  if (tid == 0) {
    mbar_init(bar_qk, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_barrier_init();
    prefetch_tensormap(&tm);
  }
  if (warp == 0) {
    __syncwarp();
    tmem_alloc(tslot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (tid == 0) {
    mbar_arrive_expect_tx(bar_qk, (uint32_t)(kQTile * kHeadDim + nload * 64 * kHeadDim));
    tma_load_2d(sQ, &tm, h * kHeadDim, row0 + q0, bar_qk);
    tma_load_2d(sQ + 64 * kHeadDim, &tm, h * kHeadDim, row0 + q0 + 64, bar_qk);
    for (int i = 0; i < nload; ++i) tma_load_2d(sK + i * 64 * kHeadDim, &tm, D + h * kHeadDim, row0 + 64 * i, bar_qk);
    mbar_arrive_expect_tx(bar_v, (uint32_t)(nload * 64 * kHeadDim));
    for (int i = 0; i < nload; ++i)
      tma_load_2d(sV + i * 64 * kHeadDim, &tm, 2 * D + h * kHeadDim, row0 + 64 * i, bar_v);
  }
  // replicated ShiftExp table: tab[t * 32 + l] = ShiftExp(-t) for every lane l.
  // One evaluation per entry into part[] (free until pass 1), then copies
  // written as consecutive 16-byte chunks by consecutive threads (no bank
  // conflicts).
  if (tid < (1 << a.k_s)) part[tid] = shift_exp(-tid, a.I0);
  __syncthreads();
  for (int i4 = tid; i4 < (8 << a.k_s); i4 += kShortThreads) {
    const int32_t e = part[i4 >> 3];
    reinterpret_cast<int4*>(tab)[i4] = make_int4(e, e, e, e);
  }

  bool ok = true;
  if (tid == 0) {
    if (!mbar_wait(bar_qk, 0, a.status)) ok = false;
    if (ok) {
      tc_fence_after();
      const uint32_t idesc = idesc_i8(kQTile, L.n32, true, true, false);
      const uint32_t qa = smem_u32(sQ);
      const uint32_t kb = smem_u32(sK);
#pragma unroll
      for (int k = 0; k < kHeadDim / 32; ++k)
        umma_i8(tmem, smem_desc(qa + k * 32, 16, 512, kSwizzle64B), smem_desc(kb + k * 32, 16, 512, kSwizzle64B),
                idesc, k != 0);
    }
    umma_commit(bar_s);
  }
  __syncthreads();  // exp table complete
  if (!mbar_wait(bar_s, 0, a.status)) ok = false;
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after();
  const uint32_t t_row = tmem + ((uint32_t)(quarter * 32) << 16);
  const int cbase = half * hcols;

  // Warps whose 32 query rows all lie past the image's last token skip the
  // three passes (their P rows feed only outputs that are never stored).
  const bool rows_live = q0 + quarter * 32 < N;
  const bool work = ok && rows_live;
  const int nchunk = hcols / 16;

  // Each pass streams this thread's key columns in 16-column TMEM chunks with
  // the next chunk's load in flight while the current one is processed.
#define IVIT_STREAM_CHUNKS(BODY)                                          \
  {                                                                       \
    uint32_t ra[16], rb[16];                                              \
    tmem_ld16(t_row + (uint32_t)cbase, ra);                               \
    for (int k = 0; k < nchunk; k += 2) {                                 \
      tmem_ld_wait();                                                     \
      if (k + 1 < nchunk) tmem_ld16(t_row + (uint32_t)(cbase + 16 * (k + 1)), rb); \
      { uint32_t(&r)[16] = ra; const int col = cbase + 16 * k; BODY }     \
      if (k + 1 < nchunk) {                                               \
        tmem_ld_wait();                                                   \
        if (k + 2 < nchunk) tmem_ld16(t_row + (uint32_t)(cbase + 16 * (k + 2)), ra); \
        { uint32_t(&r)[16] = rb; const int col = cbase + 16 * (k + 1); BODY } \
      }                                                                   \
    }                                                                     \
  }

  // ---- pass 1: row maximum of the raw scores over the valid keys
  int32_t smax = INT_MIN;
  if (work) {
    IVIT_STREAM_CHUNKS({
      const int lim = N - col;
      if (lim >= 16) {
#pragma unroll
        for (int i = 0; i < 16; ++i) smax = max(smax, (int32_t)r[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (i < lim) smax = max(smax, (int32_t)r[i]);
      }
    })
  }
  part[half * 256 + row] = smax;
  __syncthreads();
  smax = max(part[row], part[256 + row]);
  const int32_t lmax = logit_requant<FASTQ>(smax, bq, a.logit_b, a.logit_c, a.ks_lo, a.ks_hi);

  // ---- pass 2: e = ShiftExp(L - max L) back into TMEM, row sum
  uint32_t sum = 0;
  // tb[-32 L] = ShiftExp(L - max L) from this lane's copy of the table
  const int32_t* tb = tab + lane + lmax * 32;
  if (work) {
    IVIT_STREAM_CHUNKS({
      const int lim = N - col;
      if (lim >= 16) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int32_t l = logit_requant<FASTQ>((int32_t)r[i], bq, a.logit_b, a.logit_c, a.ks_lo, a.ks_hi);
          const uint32_t e = (uint32_t)tb[-32 * l];
          sum += e;
          r[i] = e;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int32_t l = logit_requant<FASTQ>((int32_t)r[i], bq, a.logit_b, a.logit_c, a.ks_lo, a.ks_hi);
          const uint32_t e = (i < lim) ? (uint32_t)tb[-32 * l] : 0u;
          sum += e;
          r[i] = e;
        }
      }
      tmem_st16(t_row + (uint32_t)col, r);
    })
    tmem_st_wait();
  }
  part[half * 256 + 128 + row] = (int32_t)sum;
  __syncthreads();
  sum = (uint32_t)part[128 + row] + (uint32_t)part[256 + 128 + row];
  if (sum == 0) sum = 1;  // rows that skipped the passes
  const uint32_t dv = (1u << a.M) / sum;
  const int pshift = a.M - (a.k_out - 1);

  // ---- pass 3: P = (Dv e) >> (M - k_out + 1) into the swizzled operand
  fence_proxy_async_smem();
  if (work) {
    const int rlo = row & 7;
    uint8_t* prow = sP + (row >> 3) * 1024 + rlo * 128;
    IVIT_STREAM_CHUNKS({
      uint32_t w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        w[q] = ((dv * r[4 * q]) >> pshift) + ((dv * r[4 * q + 1]) >> pshift) * 256u +
               ((dv * r[4 * q + 2]) >> pshift) * 65536u + ((dv * r[4 * q + 3]) >> pshift) * 16777216u;
      *reinterpret_cast<int4*>(prow + (col >> 7) * 16384 + ((((col & 127) >> 4) ^ rlo) << 4)) =
          make_int4((int)w[0], (int)w[1], (int)w[2], (int)w[3]);
    })
  }
#undef IVIT_STREAM_CHUNKS
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  // ---- O = P V
  if (tid == 0) {
    if (ok && mbar_wait(bar_v, 0, a.status)) {
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
  if (!mbar_wait(bar_o, 0, a.status)) ok = false;
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after();

  // ---- ctx = sat_8((b_o O) >> c_o); warp half h writes columns [32 h, 32 h + 32)
  {
    uint32_t r[32];
    tmem_ld32(t_row + (uint32_t)(half * 32), r);
    tmem_ld_wait();
    const int q = q0 + row;
    if (ok && q < N) {
      int8_t* dst = a.ctx + (int64_t)(row0 + q) * D + h * kHeadDim + half * 32;
      uint32_t packed[8];
#pragma unroll
      for (int wd = 0; wd < 8; ++wd) {
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          word |= ((uint32_t)requant8((int32_t)r[wd * 4 + e], a.out_b, a.out_c) & 0xFFu) << (8 * e);
        packed[wd] = word;
      }
      reinterpret_cast<int4*>(dst)[0] = make_int4(packed[0], packed[1], packed[2], packed[3]);
      reinterpret_cast<int4*>(dst)[1] = make_int4(packed[4], packed[5], packed[6], packed[7]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

ivit_status launch_attention(const DeviceCtx& dc, const int8_t* qkv, int32_t B, int32_t N, int32_t H,
                             ivit_dyadic logit, int32_t k_s, int32_t I0, int32_t M, int32_t k_out,
                             ivit_dyadic out, int8_t* ctx, cudaStream_t stream) {
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
  a.ctx = ctx;
  a.status = dc.status;
  dim3 grid((unsigned)((N + kQTile - 1) / kQTile), (unsigned)H, (unsigned)B);
  if (N <= kShortMaxKeys) {
    const ShortLayout S = short_layout(N);
    const int smem = S.total + 1024;  // >= 80 KB: at most two CTAs (2 x 256 TMEM columns) per SM
    // bq = b 2^(32 - c) when it fits a positive int32: the logit requant is then one mul.hi
    const bool fastq = logit.c >= 1 && (int64_t)logit.b < ((int64_t)1 << (logit.c - 1));
    const int32_t bq = fastq ? (int32_t)((int64_t)logit.b << (32 - logit.c)) : 0;
    static bool attr_short = false;
    if (!attr_short) {
      if (cudaFuncSetAttribute(attention_short_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               227 * 1024) != cudaSuccess ||
          cudaFuncSetAttribute(attention_short_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               227 * 1024) != cudaSuccess)
        return IVIT_ERR_CUDA;
      attr_short = true;
    }
    if (fastq)
      attention_short_kernel<true><<<grid, kShortThreads, smem, stream>>>(tm, a, bq);
    else
      attention_short_kernel<false><<<grid, kShortThreads, smem, stream>>>(tm, a, bq);
    note_launch();
    return cudaGetLastError() == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
  }
  const AttnLayout L = attn_layout(N);
  // at most two CTAs per SM, so that their TMEM (256 columns each) always fits
  int smem = L.total + 1024;
  if (smem < 80 * 1024) smem = 80 * 1024;
  static int attr_bytes = 0;
  if (smem > attr_bytes) {
    if (cudaFuncSetAttribute(attention_shiftmax_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
        cudaSuccess)
      return IVIT_ERR_CUDA;
    attr_bytes = 227 * 1024;
  }
  attention_shiftmax_kernel<<<grid, kAttnThreads, smem, stream>>>(tm, a);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? IVIT_OK : IVIT_ERR_CUDA;
}

}  // namespace ivit
