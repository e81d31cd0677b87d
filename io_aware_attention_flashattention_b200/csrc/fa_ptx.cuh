// fa_ptx.cuh -- thin inline-PTX wrappers for sm_100a: shared-memory barriers
// (mbarrier), TMA tensor loads, and the tcgen05 family (TMEM allocation, MMA,
// commit, TMEM loads/stores, fences). Every wait is bounded by a watchdog.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace fa {

// Error bits recorded in the device status word.
enum : unsigned { kStatusTimeout = 1u };

__device__ unsigned int g_status;  // per-GPU status word, read by fa_get_status()

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31; }

// Timeline trace, a profiling aid compiled only with -DFA_TRACE (never in the
// library build): lane 0 of the calling warp, in the one CTA g_trace_cta names,
// stores the SM clock of event (code < 128, a < 1024, b < 2) into its own slot of
// g_trace (plain stores, no atomics, so the trace barely perturbs the timeline),
// and the global timer into g_trace_ns for codes 0 and 99 (start and end). The
// host reads both back with cudaMemcpyFromSymbol.
#ifdef FA_TRACE
constexpr unsigned kTraceCap = 128u * 1024u * 2u;
__device__ uint32_t g_trace[kTraceCap];
__device__ unsigned long long g_trace_ns[2];
__device__ int g_trace_cta;
__device__ __forceinline__ void trace_point(uint32_t code, uint32_t a, uint32_t b) {
  if (static_cast<int>(blockIdx.x) == g_trace_cta && (threadIdx.x & 31) == 0) {
    g_trace[((code & 127u) * 1024u + (a & 1023u)) * 2u + (b & 1u)] =
        static_cast<uint32_t>(clock64());
    if (code == 0u || code == 99u) {
      unsigned long long t;
      asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
      g_trace_ns[code == 0u ? 0 : 1] = t;
    }
  }
}
// Per-CTA timeline of every CTA (up to kTraceCtas): global timer at up to 7 stages
// (slot < 7) and the SM id (slot 7), stored by whichever thread passes the stage.
constexpr unsigned kTraceCtas = 16384u;
__device__ unsigned long long g_trace_cta_ns[kTraceCtas * 8u];
__device__ __forceinline__ void trace_cta(uint32_t slot) {
  if (blockIdx.x >= kTraceCtas) return;
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  g_trace_cta_ns[blockIdx.x * 8u + (slot & 7u)] = t;
  if (slot == 0u) {
    uint32_t sm;
    asm volatile("mov.u32 %0, %smid;" : "=r"(sm));
    g_trace_cta_ns[blockIdx.x * 8u + 7u] = sm;
  }
}
#define FA_TRACE_POINT(code, a, b) ::fa::trace_point((code), (a), (b))
#define FA_TRACE_CTA(slot) ::fa::trace_cta(slot)
#else
#define FA_TRACE_POINT(code, a, b) ((void)0)
#define FA_TRACE_CTA(slot) ((void)0)
#endif

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Watchdog shared by all waits of one CTA: an abort flag in shared memory and a
// time limit. Once any wait of the CTA has run out, every later wait returns
// false at once, so the CTA drains in bounded time.
struct Watchdog {
  volatile int* abort_flag;  // shared memory
  uint64_t limit_ns;
};

// Waits until the barrier's phase with the given parity has completed. Returns
// false (after recording the timeout) if the watchdog limit ran out or another
// wait of this CTA already gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const Watchdog& wd) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*wd.abort_flag) return false;
      if (globaltimer_ns() - t0 > wd.limit_ns) {
        *wd.abort_flag = 1;
        atomicOr(&g_status, kStatusTimeout);
        return false;
      }
    }
  }
}

// ---------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled load of one box into shared memory, completing `bytes` on `bar`.
// The innermost coordinate x must be a multiple of 8 elements (16 bytes) for
// 16-bit data; callers only pass 0 or 64.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later accesses by
// the async proxy (TMA, tcgen05.mma operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05

// Allocates `ncols` TMEM columns (power of two >= 32) for the CTA; the base
// address is written to shared memory at `dst`. Executed by one full warp.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Programmatic dependent launch. Every kernel of this library is launched with
// programmatic stream serialization, so it may start while the grid before it on
// the stream is still running. pdl_wait blocks the calling thread until that grid
// has completed and its memory writes are visible (at once when there is no such
// grid); each kernel calls it before its first global memory access, read or write.
// pdl_launch_dependents lets the grid after this one start launching once every CTA
// of this grid has called it or exited; its CTAs then run their set-up and wait.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Makes the mbarrier track completion of all prior tcgen05.mma of this thread.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]; kind::f16 (bf16 operands, fp32 D).
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]; kind::f16.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// ---- elect-one forms. The whole warp executes these converged; exactly one lane
// (chosen by elect.sync inside the asm) issues the operation. Issuing from a
// converged warp keeps the operands in uniform registers; issuing from a divergent
// `if (lane == 0)` branch was measured on B200 to slow back-to-back 128x128x16 MMAs
// from 64 to 184 cycles each when two busy warps share the issuer's sub-partition
// (70 cycles with this form).

__device__ __forceinline__ void mma_ss_e(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_ts_e(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Four MMAs of one K chunk (K = 4 x 16) from one elected lane: MMA i takes the
// descriptors a0 + i * SA and b0 + i * SB (in the descriptors' 16-byte address units;
// shared-memory addresses stay below 256 KB, so the 14-bit start-address field never
// carries into the next field) and accumulates if i > 0 or acc_first is set. Fewer
// instructions in the issuing warp than four separate issues, each recomputing its
// descriptors.
template <uint32_t SA, uint32_t SB>
__device__ __forceinline__ void mma_ss_x4(uint32_t d_tmem, uint64_t a0, uint64_t b0,
                                          uint32_t idesc, uint32_t acc_first) {
  asm volatile(
      "{\n\t.reg .pred p, e, t;\n\t"
      ".reg .b32 al, ah, bl, bh, x, y;\n\t"
      ".reg .b64 a, b;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, %4, %4;\n\t"
      "mov.b64 {al, ah}, %1;\n\t"
      "mov.b64 {bl, bh}, %2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
      "add.u32 x, al, %5;\n\tadd.u32 y, bl, %8;\n\t"
      "mov.b64 a, {x, ah};\n\tmov.b64 b, {y, bh};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, t;\n\t"
      "add.u32 x, al, %6;\n\tadd.u32 y, bl, %9;\n\t"
      "mov.b64 a, {x, ah};\n\tmov.b64 b, {y, bh};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, t;\n\t"
      "add.u32 x, al, %7;\n\tadd.u32 y, bl, %10;\n\t"
      "mov.b64 a, {x, ah};\n\tmov.b64 b, {y, bh};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, t;\n\t}" ::"r"(d_tmem),
      "l"(a0), "l"(b0), "r"(idesc), "r"(acc_first), "n"(SA), "n"(2 * SA), "n"(3 * SA), "n"(SB),
      "n"(2 * SB), "n"(3 * SB)
      : "memory");
}

// The same with A in TMEM: MMA i reads A at column a_tmem + i * SA.
template <uint32_t SA, uint32_t SB>
__device__ __forceinline__ void mma_ts_x4(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0,
                                          uint32_t idesc, uint32_t acc_first) {
  asm volatile(
      "{\n\t.reg .pred p, e, t;\n\t"
      ".reg .b32 bl, bh, x, y;\n\t"
      ".reg .b64 b;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, %4, %4;\n\t"
      "mov.b64 {bl, bh}, %2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "add.u32 x, %1, %5;\n\tadd.u32 y, bl, %8;\n\tmov.b64 b, {y, bh};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [x], b, %3, t;\n\t"
      "add.u32 x, %1, %6;\n\tadd.u32 y, bl, %9;\n\tmov.b64 b, {y, bh};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [x], b, %3, t;\n\t"
      "add.u32 x, %1, %7;\n\tadd.u32 y, bl, %10;\n\tmov.b64 b, {y, bh};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [x], b, %3, t;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b0), "r"(idesc), "r"(acc_first), "n"(SA), "n"(2 * SA), "n"(3 * SA),
      "n"(SB), "n"(2 * SB), "n"(3 * SB)
      : "memory");
}

__device__ __forceinline__ void tc_commit_e(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          bar)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx_e(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;\n\t}" ::"r"(bar),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_e(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                              int x, int y, int z) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];\n\t}" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void bulk_load_e(uint32_t dst, const void* src, uint32_t bytes,
                                            uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      "\n\t}" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Warp-wide bounded wait: every lane polls, the result is the same in all lanes.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, const Watchdog& wd) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, wd));
}

// The 16-bit element types of the tensor-core paths (kind::f16 operands).
enum class Elt { BF16, F16 };

// Instruction descriptor for kind::f16 with A and B of element type E and an fp32
// accumulator. a_mn / b_mn: 1 when the operand is MN-major (else K-major).
template <Elt E>
__host__ __device__ constexpr uint32_t idesc_f32acc(int M, int N, int a_mn, int b_mn) {
  constexpr uint32_t fmt = (E == Elt::BF16) ? 1u : 0u;  // A/B format: 1 = bf16, 0 = f16
  return (1u << 4)                               // D format: f32
         | (fmt << 7)                            // A format
         | (fmt << 10)                           // B format
         | (static_cast<uint32_t>(a_mn) << 15)   // A major
         | (static_cast<uint32_t>(b_mn) << 16)   // B major
         | (static_cast<uint32_t>(N >> 3) << 17) // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);  // M / 16
}

// Shared-memory matrix descriptor, 128-byte swizzle (the layout TMA writes with
// CU_TENSOR_MAP_SWIZZLE_128B into 1024-byte aligned tiles).
//   K-major operand: rows of 64 bf16 (128 B), 8-row atoms 1024 B apart (SBO);
//                    LBO unused.
//   MN-major operand: 64-element MN chunks `lbo` bytes apart, 8-row K atoms
//                    1024 B apart (SBO).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;  // descriptor version for sm_100
  d |= 2ull << 61;  // SWIZZLE_128B
  return d;
}

// TMEM loads/stores, 32 lanes x 32-bit, repeated over consecutive columns: each
// thread of the warp owns one lane (row) and gets/gives consecutive columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- math

// 2^x on the MUFU unit (approximate, flush-to-zero).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (Blackwell f32x2 arithmetic: one instruction for two lanes of
// work on the FMA pipe).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for a pair, on the FMA and integer pipes instead of MUFU, for x <= 64.
// Range reduction in the Cody-Waite manner: adding 1.5*2^23 rounds x to the
// nearest integer j and leaves j in the low mantissa bits of the sum; f = x - j
// lies in [-0.5, 0.5]. 2^f is a degree-3 polynomial fitted to 2^f on [-0.5, 0.5]
// (least squares at Chebyshev nodes with Lawson reweighting toward the minimax
// fit; maximum relative error 7.5e-5, about 1/26 of a bf16 ulp), and j is added
// to its exponent field. x is clamped at -125 so the result stays a normal
// number: inputs below that give 2^-125 (about 2.4e-38) instead of 0.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 t = fadd2(x, make_float2(kMagic, kMagic));
  const float2 j = fadd2(t, make_float2(-kMagic, -kMagic));
  const float2 f = ffma2(j, make_float2(-1.0f, -1.0f), x);
  float2 q = ffma2(f, make_float2(0.0551716648f, 0.0551716648f),
                   make_float2(0.2426111251f, 0.2426111251f));
  q = ffma2(q, f, make_float2(0.6932609678f, 0.6932609678f));
  q = ffma2(q, f, make_float2(0.9999280572f, 0.9999280572f));
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

// Two fp32 values to a packed 16-bit pair, round-to-nearest-even; `lo` lands in
// the low half (the element with the smaller index).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
template <Elt E>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (E == Elt::BF16) return pack_bf16x2(lo, hi);
  else return pack_f16x2(lo, hi);
}

// A packed 16-bit pair back to two fp32 values (exact).
template <Elt E>
__device__ __forceinline__ float2 unpack2(uint32_t w) {
  if constexpr (E == Elt::BF16) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  } else {
    __half2 h = *reinterpret_cast<__half2*>(&w);
    return __half22float2(h);
  }
}

// ---------------------------------------------------------------- dropout RNG

// Philox-4x32-10, the counter-based generator of Salmon, Moraes, Dror and Shaw
// ("Parallel random numbers: as easy as 1, 2, 3", SC 2011): in each of ten rounds the
// words 0 and 2 are multiplied by the two round constants, the high halves of the
// products are mixed with words 1 and 3 and the round key, and the words are
// permuted; the key advances by the two Weyl constants between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    // the two 32 x 32 -> 64-bit products (one wide multiply each)
    const unsigned long long p0 = static_cast<unsigned long long>(0xD2511F53u) * c.x;
    const unsigned long long p1 = static_cast<unsigned long long>(0xCD9E8D57u) * c.z;
    c = make_uint4(static_cast<uint32_t>(p1 >> 32) ^ c.y ^ k0, static_cast<uint32_t>(p1),
                   static_cast<uint32_t>(p0 >> 32) ^ c.w ^ k1, static_cast<uint32_t>(p0));
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

// Lanes 4g..4g+3 of a warp each hold one row of a 4 x 4 matrix (lane 4g+r: a[] = row
// r); afterwards lane 4g+c holds column c (a[r] = element (r, c)). Two butterfly
// rounds; in each, paired lanes swap the two elements the other one needs.
__device__ __forceinline__ void transpose4_lanes(uint32_t (&a)[4], int u) {
#pragma unroll
  for (int d = 1; d <= 2; d <<= 1) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (j & d) continue;  // the pair (j, j + d)
      const bool hi = (u & d) != 0;
      const uint32_t recv = __shfl_xor_sync(0xffffffffu, hi ? a[j] : a[j | d], d);
      if (hi)
        a[j] = recv;
      else
        a[j | d] = recv;
    }
  }
}

// Dropout on P: key j of query row i in head bh is kept iff byte (j mod 4) of word
// (i mod 4) of philox4x32_10((j / 4, i / 4, head_base + bh, offset), seed) is at least
// `threshold` (= floor(256 p), so the drop probability is threshold / 256); kept
// values are scaled by `scale` = 256 / (256 - threshold). head_base is 0 except for a
// call on a range of a larger problem's heads, which draws that problem's masks.
struct DropoutParams {
  uint32_t threshold;
  float scale;
  uint32_t seed_lo, seed_hi, offset;
  uint32_t head_base;
};

}  // namespace fa
