// sm100_ptx.cuh -- inline-PTX building blocks for the sm_100a attention kernels:
// mbarriers with time-bounded waits, TMA tile loads, tcgen05 (TMEM allocation,
// MMA, commit, TMEM loads/stores), and the shared-memory / instruction
// descriptors that tcgen05.mma reads.
//
// Descriptor formats follow the public PTX ISA (tcgen05 "shared memory
// descriptor" and "instruction descriptor" tables).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace axis_attn {

// ------------------------------------------------------------------ status
// Device status word.  Bit 0: a bounded wait ran out.  Bit 1: a device-side
// index (a page of the decode step's block table, a sequence length) was out
// of range and was not used.  Bits 8..15: the wait site of the first timeout
// (for debugging).  Read and cleared by axis_attn_get_status().
__device__ unsigned int g_status;
// Number of bounded waits that have ever run out on this device (never
// cleared).  A launch snapshots it at entry; a change during the launch means
// that one of its own CTAs gave up, and the others stop waiting.  A timeout
// left over from an earlier launch is therefore never mistaken for one of the
// current launch, whether or not axis_attn_get_status() has been called since.
__device__ unsigned int g_timeouts;

// Upper bound on any single wait inside a kernel, in SM clock cycles (2^31,
// about 1.1 s at 1.965 GHz).  No wait in a correct run comes near it: every
// wait here is on work that the same CTA issued.  Once any CTA of a launch has
// timed out, the other CTAs of that launch stop waiting at their next check,
// so a faulty launch ends quickly instead of timing out CTA by CTA.
//
// The polling loops below touch only shared memory and the SM's own cycle
// counter on each pass; the global counter is read about every 2^16 cycles.
// (Reading global memory or %globaltimer on every pass would make a waiting
// thread notice a completed barrier up to a global round trip late.)
#ifndef AXIS_ATTN_WAIT_LIMIT_CYCLES
#define AXIS_ATTN_WAIT_LIMIT_CYCLES (1ull << 31)
#endif
#define AXIS_ATTN_STATUS_CHECK_CYCLES (1ull << 16)

// Test-only builds: AXIS_ATTN_TEST_DROP_ARRIVE = 1 makes the softmax warps of
// the forward's first query tile skip their first "P is in TMEM" arrive, 2
// makes the backward's compute warps skip their first "P^T, dS^T written"
// arrive.  The wait for that barrier phase can then never complete (the next
// arrivals come only after it), and AXIS_ATTN_TEST_SHORT_SITE gives that one
// wait site a short limit (AXIS_ATTN_TEST_SHORT_LIMIT cycles), so the failure
// path runs: the waiting MMA issuer records a timeout at its site, the other
// roles of the CTA stop on the abort flag, the other CTAs on the changed
// timeout count, copies and MMAs in flight drain, TMEM is freed, the kernel
// returns.  All three are 0 in every normal build.
#ifndef AXIS_ATTN_TEST_DROP_ARRIVE
#define AXIS_ATTN_TEST_DROP_ARRIVE 0
#endif
#ifndef AXIS_ATTN_TEST_SHORT_SITE
#define AXIS_ATTN_TEST_SHORT_SITE 0
#endif
#ifndef AXIS_ATTN_TEST_SHORT_LIMIT
#define AXIS_ATTN_TEST_SHORT_LIMIT (1ull << 22)
#endif

// Per-CTA wait control in shared memory: `abort` is raised by the first role
// that gives up (the others see it on their next poll); `epoch` is the
// launch's snapshot of g_timeouts; `watch` = 0 for drain waits (on TMA copies
// or MMAs already issued, which complete whatever other CTAs do), which
// therefore ignore the other CTAs.
struct WaitCtl {
  int abort;
  unsigned int epoch;
  unsigned int watch;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Called by one thread while the CTA initialises its barriers.
__device__ __forceinline__ void wait_ctl_init(volatile WaitCtl* c) {
  c->abort = 0;
  c->epoch = *reinterpret_cast<volatile unsigned int*>(&g_timeouts);
  c->watch = 1;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase of `bar` with parity `parity` has completed.  Gives up
// when `abort->abort` becomes non-zero (another role of the CTA gave up), when
// another CTA of the launch has timed out (unless abort->watch is 0), or after
// AXIS_ATTN_WAIT_LIMIT_CYCLES; in the last case it raises `abort->abort` and
// records the failure in g_status and g_timeouts.  Returns
// true when the phase completed.  Called by a single thread, or by all lanes
// of a warp (see wait_warp).  The poll loop reads only the barrier, the
// 32-bit SM clock and the abort flag; try_wait suspends the thread in
// hardware between polls.
__device__ __forceinline__ bool mbar_wait_loop(uint32_t bar, uint32_t parity, volatile WaitCtl* abort, int site) {
  const uint32_t t0 = (uint32_t)clock();
  uint32_t last = t0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (abort->abort) return false;
    const uint32_t now = (uint32_t)clock();
    if (now - last > AXIS_ATTN_STATUS_CHECK_CYCLES) {
      last = now;
      if (abort->watch && *reinterpret_cast<volatile unsigned int*>(&g_timeouts) != abort->epoch) {
        abort->abort = 1;  // another CTA of this launch gave up: results are void already
        return false;
      }
      const unsigned long long limit = (AXIS_ATTN_TEST_SHORT_SITE != 0 && site == AXIS_ATTN_TEST_SHORT_SITE)
                                           ? AXIS_ATTN_TEST_SHORT_LIMIT
                                           : AXIS_ATTN_WAIT_LIMIT_CYCLES;
      if (now - t0 > limit) {
        abort->abort = 1;
        // the first timeout since the report was last cleared names its site
        if ((atomicOr(&g_status, 1u) & 1u) == 0) atomicOr(&g_status, (unsigned)(site & 0xff) << 8);
        atomicAdd(&g_timeouts, 1u);
        return false;
      }
    }
  }
}

__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile WaitCtl* abort, int site) {
  return mbar_wait_loop(bar, parity, abort, site);
}

// One try_wait inline; on a miss the poll loop, out of line (INL = false: less
// code at each call site, but the compiler saves the caller's live registers
// around the call) or inline (INL = true: no call, more code).
template <bool INL = false>
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, volatile WaitCtl* abort,
                                                  int site) {
  if (mbar_try_wait(bar, parity)) return true;
  return INL ? mbar_wait_loop(bar, parity, abort, site) : mbar_wait_slow(bar, parity, abort, site);
}

// Warp-uniform bounded wait: every lane polls, and the warp proceeds only if
// all lanes saw the phase complete, so warp-collective instructions that
// follow are never reached by a partial warp.
template <bool INL = false>
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile WaitCtl* abort,
                                          int site) {
  const bool ok = mbar_wait_bounded<INL>(bar, parity, abort, site);
  return __all_sync(0xffffffffu, ok);
}

// -------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 4-D tiled load (coordinates innermost first), completion counted in bytes on `bar`.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

// 3-D tiled load (coordinates innermost first), completion counted in bytes on `bar`.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// L2 prefetch of a 4-D tile (no shared-memory destination, no completion).
__device__ __forceinline__ void tma_prefetch_4d(const CUtensorMap* map, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global [%0, {%1, %2, %3, %4}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

// Element-wise add of a shared-memory tile into global memory through the
// TMA engine (3-D tensor map; elements outside the tensor are skipped).
// Completion is tracked by bulk groups of the issuing thread.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
  asm volatile("cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until no committed bulk group is still reading shared memory.
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until every committed bulk group has completed.
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Untiled bulk copy global -> shared (16-byte aligned addresses, size % 16 == 0).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
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

// ---- MMA issue: the whole (converged) warp executes these, with warp-uniform
// operands; lane 0 issues the instruction (always the same lane: a commit
// tracks only the MMAs its own thread issued, and arrives on `bar` once all of
// them have completed).  Keeping the issuing loop warp-uniform lets descriptors
// live in uniform registers.
__device__ __forceinline__ void mma_ss_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .u32 l;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "mov.u32 l, %%laneid;\n\t"
      "setp.eq.u32 e, l, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .u32 l;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "mov.u32 l, %%laneid;\n\t"
      "setp.eq.u32 e, l, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit_w(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t.reg .u32 l;\n\t"
      "mov.u32 l, %%laneid;\n\t"
      "setp.eq.u32 e, l, 0;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns; thread t gets lane (base + t).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
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

// TMEM address of lane `lane`, column `col` relative to an allocation base.
__device__ __forceinline__ uint32_t tmem_at(uint32_t base, uint32_t lane, uint32_t col) {
  return base + (lane << 16) + col;
}

// --------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor, 128-byte swizzle.  Start address, LBO and
// SBO are in bytes (encoded >> 4); bits 46..47 = 1 (the sm_100 descriptor
// version); bits 61..63 = 2 (128B swizzle).  Tiles must sit on 1024-byte
// boundaries; a start address may be advanced inside the 128-byte row (K-major
// k-steps) because the swizzle is applied to the final address.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3fff);
  d |= (uint64_t)((lbo >> 4) & 0x3fff) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3fff) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A and B and fp32 accumulate.
// a_mn / b_mn select MN-major (1) instead of K-major (0) operands.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                       // D format: f32
         | (1u << 7)                     // A format: bf16
         | (1u << 10)                    // B format: bf16
         | ((uint32_t)a_mn << 15)        // A major
         | ((uint32_t)b_mn << 16)        // B major
         | ((uint32_t)(N >> 3) << 17)    // N / 8
         | ((uint32_t)(M >> 4) << 24);   // M / 16
}

// ------------------------------------------------------------- arithmetic
// Named barrier `id` over `count` threads (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Warp-level MMA (m16n8k16, bf16 in, fp32 accumulate) and its 8x8 matrix
// loads from shared memory: for the small decode products, where G <= 8 query
// rows would fill a tcgen05 tile to a few percent.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// d += A B for A = {a0, a1, a2, a3} (16 x 16, rows g / g + 8, columns k / k + 8)
// and B = {b0, b1} (16 x 8).
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Packed pairs of fp32 (sm_100 executes f32x2 FMA/ADD/MUL as one instruction).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// Round-to-nearest packed add (explicit .rn: the magic-number rounding below
// must not be contracted with a neighbouring multiply).
__device__ __forceinline__ uint64_t f2_add_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x for a pair of fp32 values on the FP32 and integer pipes instead of the
// MUFU: x = n + f with n = round(x) (adding 1.5 * 2^23 leaves n in the low
// mantissa bits) and f in [-1/2, 1/2]; 2^f from a degree-3 polynomial whose
// coefficients are the fp32-rounded least-maximum-relative-error fit on
// [-1/2, 1/2] by the Remez exchange (exp2_fit.py in the package reproduces
// them); n is added to the exponent field with one integer shift-add (the
// magic number's own bits shift out).  Relative error <= 7.5e-5 for
// -125 <= x <= 64 (measured on the fp32 evaluation), mean +5e-6.  x is
// clamped at -126 first, so every smaller x, -inf included, gives 2^-126
// (1.2e-38) instead of 0: below the fp32 resolution of any sum or product it
// enters here.
constexpr float EXP2_C0 = 0.999928057f, EXP2_C1 = 0.693260968f, EXP2_C2 = 0.242611125f,
                EXP2_C3 = 0.0551716685f;
__device__ __forceinline__ uint64_t f2_exp2_poly(uint64_t x2) {
  float x0, x1;
  f2_unpack(x2, x0, x1);
  const uint64_t x = f2_pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
  const uint64_t t = f2_add_rn(x, f2_pack(12582912.f, 12582912.f));
  const uint64_t n = f2_add_rn(t, f2_pack(-12582912.f, -12582912.f));
  const uint64_t f = f2_fma(n, f2_pack(-1.f, -1.f), x);
  uint64_t p = f2_fma(f2_pack(EXP2_C3, EXP2_C3), f, f2_pack(EXP2_C2, EXP2_C2));
  p = f2_fma(p, f, f2_pack(EXP2_C1, EXP2_C1));
  p = f2_fma(p, f, f2_pack(EXP2_C0, EXP2_C0));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  return f2_pack(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
                 __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_bf16x2(uint64_t x2) {
  float lo, hi;
  f2_unpack(x2, lo, hi);
  return pack_bf16x2(lo, hi);
}

}  // namespace axis_attn
