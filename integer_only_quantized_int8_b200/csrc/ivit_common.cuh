// ivit_common.cuh -- sm_100a building blocks shared by the integer ViT kernels:
// mbarrier / TMA / tcgen05 (TMEM, UMMA) wrappers in inline PTX, bounded waits,
// and the integer helpers of the method (dyadic requant, shift-exponential).
//
// Method sources: "I-ViT: Integer-only Quantization for Efficient Vision
// Transformer Inference", sections 3.2 (dyadic arithmetic), 3.3 (Shiftmax),
// 3.4 (ShiftGELU), 3.5 (I-LayerNorm); the Trio-ViT article, eq. (12).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/ivit.h"

#define IVIT_DEV __device__ __forceinline__

namespace ivit {

// ---------------------------------------------------------------------------
// device status word (bounded waits report here instead of hanging)
// ---------------------------------------------------------------------------
enum : int { kStatusOk = 0, kStatusTimeout = 1 };

// Wait budget in nanoseconds of %globaltimer: far above any legitimate wait in
// these kernels (each finishes in well under a millisecond), far below a hang.
constexpr uint64_t kWaitBudgetNs = 1000ull * 1000ull * 1000ull;   // 1 s

IVIT_DEV uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

IVIT_DEV void report_timeout(int* status) {
  if (status) atomicExch(status, kStatusTimeout);
}

// ---------------------------------------------------------------------------
// shared-memory addresses and mbarriers
// ---------------------------------------------------------------------------
IVIT_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// The first 1024-byte-aligned byte of a dynamic shared-memory array, found by
// pointer arithmetic on the array itself: the compiler then still knows that
// the result points into shared memory, so accesses through it stay 32-bit
// ld/st.shared (a round trip through an integer makes them generic accesses
// with 64-bit address arithmetic).
IVIT_DEV uint8_t* align_smem_1024(uint8_t* raw) {
  return raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
}

IVIT_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// make barrier initialisation visible to the async proxy (TMA, tensor core)
IVIT_DEV void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

IVIT_DEV void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

IVIT_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

IVIT_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

IVIT_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, but the thread may be suspended in hardware for up to
// kSuspendHintNs while the phase is incomplete (it resumes as soon as the
// phase completes), so a waiting warp does not spin on the issue slots.
constexpr uint32_t kSuspendHintNs = 20000;
IVIT_DEV bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "n"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed.  Gives up after
// kWaitBudgetNs, records a timeout in *status and returns false.
IVIT_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitBudgetNs) {
      report_timeout(status);
      return false;
    }
  }
}

// ---------------------------------------------------------------------------
// programmatic dependent launch
// ---------------------------------------------------------------------------
// Every kernel of this library is launched so that the next kernel of the
// stream may start (and run its prologue) while this one finishes.  A kernel
// therefore calls pdl_wait() before it first touches memory that an earlier
// kernel of the stream writes, and before its own first global write; the
// wait returns once every earlier kernel has completed and its writes are
// visible.  pdl_launch_dependents() lets the next kernel be scheduled.
IVIT_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
IVIT_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor): every copy fills or drains this CTA's own shared memory
// ---------------------------------------------------------------------------
IVIT_DEV void tma_load_2d(void* smem_dst, const CUtensorMap* map, int32_t x, int32_t y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// shared -> global tile store, tracked in the issuing thread's bulk groups
IVIT_DEV void tma_store_2d(const CUtensorMap* map, int32_t x, int32_t y, const void* smem_src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(smem_u32(smem_src))
               : "memory");
}
IVIT_DEV void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// every committed store of this thread has finished reading shared memory
IVIT_DEV void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// every committed store group of this thread but the most recent one has
// finished reading shared memory
IVIT_DEV void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// every committed store of this thread has completed
IVIT_DEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

IVIT_DEV void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: TMEM allocation, UMMA issue/commit, TMEM loads
// ---------------------------------------------------------------------------
// whole warp; writes the TMEM base address into *slot (shared memory)
IVIT_DEV void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
IVIT_DEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
IVIT_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
IVIT_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
IVIT_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, kind::i8, int32 accumulate; single thread.
IVIT_DEV void umma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// As umma_i8, always accumulating, with each descriptor passed as its two
// 32-bit halves: the start address sits in the low half, so stepping through a
// stage costs one 32-bit add per operand in the issuing loop.
IVIT_DEV void umma_i8_acc(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo, uint32_t b_hi,
                          uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "setp.eq.u32 p, 1, 1;\n\t"
      "mov.b64 da, {%1, %2};\n\t"
      "mov.b64 db, {%3, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], da, db, %5, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc)
      : "memory");
}

// arrive on *bar once all previously issued tcgen05.mma of this thread complete
IVIT_DEV void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Instruction descriptor of tcgen05.mma kind::i8 (int32 accumulator):
// bits 4-5 D format (2 = s32), 7-9 A format, 10-12 B format (1 = signed,
// 0 = unsigned 8-bit), 15 / 16 A / B major (0 = K-major, 1 = MN-major),
// 17-22 N >> 3, 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N, bool a_signed, bool b_signed, bool b_mn_major) {
  return (2u << 4) | ((a_signed ? 1u : 0u) << 7) | ((b_signed ? 1u : 0u) << 10) |
         ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor (sm_100 format): start address >> 4 in bits
// 0-13, leading-dimension byte offset >> 4 in 16-29, stride-dimension byte
// offset >> 4 in 32-45, version 1 in 46-47, layout (swizzle) in 61-63.
enum : uint32_t { kSwizzleNone = 0, kSwizzle128B = 2, kSwizzle64B = 4, kSwizzle32B = 6 };

IVIT_DEV uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes, uint32_t layout) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives
// lane (base lane + i), columns [col, col + 32).
IVIT_DEV void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
IVIT_DEV void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns (thread i: lane base + i)
IVIT_DEV void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

IVIT_DEV void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
IVIT_DEV void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// tcgen05.wait::ld that also names the registers of the load it completes, so
// no use of them can be scheduled before it (for loads kept in flight while
// other registers are being worked on)
IVIT_DEV void tmem_ld_wait_regs(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}

// As tmem_ld_wait_regs, for two loads in flight.
IVIT_DEV void tmem_ld_wait_regs2(uint32_t (&a)[16], uint32_t (&b)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]), "+r"(a[7]),
                 "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]), "+r"(a[12]), "+r"(a[13]), "+r"(a[14]), "+r"(a[15]),
                 "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]), "+r"(b[6]), "+r"(b[7]),
                 "+r"(b[8]), "+r"(b[9]), "+r"(b[10]), "+r"(b[11]), "+r"(b[12]), "+r"(b[13]), "+r"(b[14]), "+r"(b[15])
               :
               : "memory");
}

// 32 lanes x 16 consecutive columns, every column of a lane set to v
IVIT_DEV void tmem_st16_fill(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1};" ::"r"(taddr),
      "r"(v)
      : "memory");
}

// ---------------------------------------------------------------------------
// integer arithmetic of the method
// ---------------------------------------------------------------------------

// sat_8((b * v) >> c), b >= 0, 0 <= c <= 31, with >> an arithmetic (floor) shift
IVIT_DEV int32_t requant8(int32_t v, int32_t b, int32_t c) {
  const int64_t p = (int64_t)b * (int64_t)v;
  const int64_t q = p >> c;
  return (int32_t)(q < -128 ? -128 : (q > 127 ? 127 : q));
}

IVIT_DEV int32_t requant_bits(int32_t v, int32_t b, int32_t c, int32_t lo, int32_t hi) {
  const int64_t q = ((int64_t)b * (int64_t)v) >> c;
  return (int32_t)(q < lo ? lo : (q > hi ? hi : q));
}

// Shift-exponential of d <= 0 at scale 1/I0 (I-ViT section 3.3):
// log2 e ~ 1.0111b (d + d/2 - d/16, floor shifts); -I_p = q I0 + r with
// 0 <= r < I0; 2^(-r/I0) ~ 1 - r/(2 I0); then a right shift by q.
IVIT_DEV int32_t shift_exp(int32_t d, int32_t I0) {
  const int32_t ip = d + (d >> 1) - (d >> 4);
  const int32_t neg = -ip;                       // >= 0
  const int32_t q = neg / I0;                    // non-negative operands: truncation == floor
  const int32_t r = neg - q * I0;
  const int32_t t = I0 - ((r + 1) >> 1);         // I0 + floor(-r / 2)
  return q >= 31 ? 0 : (t >> q);
}

// Integer sigmoid of S * I_p as a two-term Shiftmax (I-ViT section 3.4),
// exponent offset max(I_p, 0); result scale 2^-(k_out - 1).
IVIT_DEV int32_t shift_sigmoid(int32_t ip, int32_t I0, int32_t M, int32_t k_out) {
  const int32_t m = ip > 0 ? ip : 0;
  const int32_t e1 = shift_exp(ip - m, I0);
  const int32_t e2 = shift_exp(-m, I0);
  const uint32_t dv = (1u << M) / (uint32_t)(e1 + e2);
  return (int32_t)((dv * (uint32_t)e1) >> (M - (k_out - 1)));
}

// ShiftGELU of one int8 input: x * sigma(1.1011b * x), requantised to int8.
IVIT_DEV int32_t shiftgelu8(int32_t x, int32_t I0, int32_t M, int32_t k_out, int32_t b, int32_t c) {
  const int32_t ip = x + (x >> 1) + (x >> 3) + (x >> 4);
  const int32_t sig = shift_sigmoid(ip, I0, M, k_out);
  return requant8(x * sig, b, c);
}

}  // namespace ivit
