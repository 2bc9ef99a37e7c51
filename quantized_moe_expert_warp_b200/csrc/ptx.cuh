// Inline-PTX building blocks for sm_100a: mbarriers with bounded waits,
// cp.async gathers, bulk (TMA engine) copies, and the tcgen05 family
// (TMEM allocation, MMA, commit, TMEM loads/stores, fences).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "moeq4.h"

namespace moeq4 {

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ uint16_t lds16(uint32_t addr)
{
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ int lds_volatile_s32(uint32_t addr)
{
    int v;
    asm volatile("ld.volatile.shared.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// A waiting thread sleeps inside try_wait until the phase completes or the
// suspend-time hint (ns) runs out, so idle warps do not take issue slots from
// the warps doing work.  0 selects the form without a hint.
#ifndef MOEQ4_WAIT_HINT_NS
#define MOEQ4_WAIT_HINT_NS 10000000
#endif

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity, bool sleep = true,
                                              uint32_t hint_ns = (uint32_t)MOEQ4_WAIT_HINT_NS)
{
    uint32_t ok;
#if MOEQ4_WAIT_HINT_NS > 0
    if (!sleep) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        return ok != 0;
    }
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
#else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
#endif
    return ok != 0;
}

// Per-CTA abort flag shared by all roles of a persistent kernel: once one
// wait gives up, every other wait returns at once.
struct WaitCtx {
    volatile int *abort_flag;   // shared memory
    int *status;                // global status words [code, detail] (may be null)
    uint64_t t0;
    uint64_t limit;             // ns after t0 at which a wait gives up
#ifdef MOEQ4_TRACE
    uint32_t polls[16] = {};    // failed polls per call site (instrumented builds)
    uint32_t waits[16] = {};    // waits per call site that polled more than once
#endif
};

// Instrumentation hook: called once per wait that did not complete at the
// first try, with the call site and the number of further failed polls.
#ifdef MOEQ4_TRACE
#define MOEQ4_WAIT_HOOK(where, spins) \
    do {                              \
        if (spins) {                  \
            w.waits[where] += 1;      \
            w.polls[where] += spins;  \
        }                             \
    } while (0)
#else
#define MOEQ4_WAIT_HOOK(where, spins) \
    do {                              \
    } while (0)
#endif

// Call sites (bit `where`) that poll without the suspend-time hint.
#ifndef MOEQ4_NOHINT_SITES
#define MOEQ4_NOHINT_SITES 0u
#endif

// Call sites (bit `where`) whose failed polls back off with __nanosleep.
#ifndef MOEQ4_BACKOFF_SITES
#define MOEQ4_BACKOFF_SITES 0u
#endif
#ifndef MOEQ4_BACKOFF_NS
#define MOEQ4_BACKOFF_NS 128
#endif

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s: kernels here take well under 10 ms
// Word of a workspace's status block holding the caller's wait budget in
// microseconds (0: the 2 s default).
constexpr int kStatusWaitLimitWord = 20;
// Test knob word: c > 0 makes CTA c - 1 of a launch lose one of its own
// signals (a grid-barrier arrival in the decode kernel, the weight copies in
// the grouped GEMMs), so that its waits run out of the budget.  Zero in use.
constexpr int kStatusTestKnobWord = 21;

__device__ __forceinline__ bool test_knob_hits_this_cta(const int *status)
{
    return status && *(const volatile int *)(status + kStatusTestKnobWord) == (int)blockIdx.x + 1;
}

// The wait budget of a launch: the status block's word, else 2 s.
__device__ __forceinline__ uint64_t wait_limit_ns(const int *status)
{
    const int us = status ? *(const volatile int *)(status + kStatusWaitLimitWord) : 0;
    return us > 0 ? (uint64_t)us * 1000ull : kWaitLimitNs;
}
// failed try_waits between clock reads: each one may already have slept up to the hint
constexpr uint32_t kClockEvery = MOEQ4_WAIT_HINT_NS > 0 ? 1u : 64u;

// Wait for the phase of `bar` with parity `parity` to complete.  Returns
// false (after recording MOE_ERR_TIMEOUT) if the wait budget runs out or
// another role of this CTA already gave up.
// Non-blocking probe of a phase.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Polling policy.  Mode 0 (default) polls with try_wait and its suspend-time
// hint.  Mode 1 probes with test_wait and sleeps between probes for a time
// that doubles up to a cap (short on the critical path of a k-step, call
// sites 3, 4, 9, 10; longer elsewhere); it frees issue slots but wakes
// later, and measured slower on these kernels.
#ifndef MOEQ4_WAIT_MODE
#define MOEQ4_WAIT_MODE 0   // 0: try_wait loop (suspend-time hint); 1: test_wait with sleeping back-off
#endif
#ifndef MOEQ4_NS_CRIT
#define MOEQ4_NS_CRIT 32
#endif
#ifndef MOEQ4_NS_CRIT_MAX
#define MOEQ4_NS_CRIT_MAX 128
#endif
#ifndef MOEQ4_NS_BG
#define MOEQ4_NS_BG 128
#endif
#ifndef MOEQ4_NS_BG_MAX
#define MOEQ4_NS_BG_MAX 1024
#endif

__device__ __forceinline__ constexpr bool wait_site_critical(int where)
{
    return where == 3 || where == 4 || where == 9 || where == 10;
}

__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, WaitCtx &w, int where)
{
#if MOEQ4_WAIT_MODE == 1
    if (mbar_test(bar, parity))
        return true;
    const bool crit = wait_site_critical(where);
    uint32_t ns = crit ? MOEQ4_NS_CRIT : MOEQ4_NS_BG;
    const uint32_t ns_max = crit ? MOEQ4_NS_CRIT_MAX : MOEQ4_NS_BG_MAX;
    uint32_t spins = 0;
    while (true) {
        __nanosleep(ns);
        if (mbar_test(bar, parity)) {
            MOEQ4_WAIT_HOOK(where, spins);
            return true;
        }
        if (lds_volatile_s32(smem_u32((const void *)w.abort_flag)))
            return false;
        ns = ns * 2 < ns_max ? ns * 2 : ns_max;
        if ((++spins & 15u) == 0 && globaltimer_ns() - w.t0 > w.limit) {
            *w.abort_flag = 1;
            if (w.status && atomicCAS(w.status, 0, MOE_ERR_TIMEOUT) == 0)
                w.status[1] = where;
            return false;
        }
    }
#else
    const bool sleep = !((MOEQ4_NOHINT_SITES >> where) & 1u);
    // a suspended try_wait returns at the latest after its hint, so the hint
    // is capped at the budget: the budget is then checked at least that often
    const uint32_t hint = (uint32_t)(w.limit < (uint64_t)MOEQ4_WAIT_HINT_NS ? w.limit : (uint64_t)MOEQ4_WAIT_HINT_NS);
    if (mbar_try_wait(bar, parity, sleep, hint))
        return true;
    uint32_t spins = 0;
    while (true) {
        // after every failed poll: has another role given up, has the budget run out
        if (lds_volatile_s32(smem_u32((const void *)w.abort_flag)))
            return false;
        if (spins++ % kClockEvery == 0) {
            if (globaltimer_ns() - w.t0 > w.limit) {
                *w.abort_flag = 1;
                if (w.status && atomicCAS(w.status, 0, MOE_ERR_TIMEOUT) == 0)
                    w.status[1] = where;
                return false;
            }
        }
        if ((MOEQ4_BACKOFF_SITES >> where) & 1u)
            __nanosleep(MOEQ4_BACKOFF_NS);
        if (mbar_try_wait(bar, parity, sleep, hint)) {
            MOEQ4_WAIT_HOOK(where, spins);
            return true;
        }
    }
#endif
}

// One lane of a converged warp waits; the whole warp gets the result.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, WaitCtx &w, int where)
{
    int ok = 0;
    if ((threadIdx.x & 31) == 0)
        ok = mbar_wait(bar, parity, w, where) ? 1 : 0;
    return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

// A producer that stops early (a wait ran out, or another role gave up)
// still waits, with a fresh bounded budget, until the copies it issued have
// landed, so that none writes into this CTA's shared memory after it exits:
// the last `depth` of the n_issued ring slots it filled.  On the normal path
// every such phase has completed already.
__device__ __forceinline__ void drain_ring(uint64_t *full, int n_issued, int depth, int *status, int where,
                                           int *never_abort)
{
    WaitCtx wd{never_abort, status, globaltimer_ns(), kWaitLimitNs};
    for (int i = max(0, n_issued - depth); i < n_issued; ++i)
        if (!warp_wait(&full[i % depth], (i / depth) & 1, wd, where))
            break;
}

// The last `depth` phases of a ring that one thread filled, waited for by that thread.
__device__ __forceinline__ void drain_ring_lane(uint64_t *full, int n_issued, int depth, int *status, int where,
                                                int *never_abort)
{
    WaitCtx wd{never_abort, status, globaltimer_ns(), kWaitLimitNs};
    for (int i = max(0, n_issued - depth); i < n_issued; ++i)
        if (!mbar_wait(&full[i % depth], (i / depth) & 1, wd, where))
            break;
}

// True on exactly one lane of a converged warp.  Single-thread tcgen05 and
// bulk-copy instructions are issued under this predicate from a converged
// warp: issuing them from a lone divergent lane costs several times longer.
__device__ __forceinline__ bool elect_one()
{
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .b32 %%rx;\n\t.reg .pred %%px;\n\t"
        "elect.sync %%rx|%%px, %1;\n\t"
        "@%%px mov.s32 %0, 1;\n\t}"
        : "+r"(pred)
        : "r"(0xFFFFFFFFu));
    return pred != 0;
}

// Programmatic dependent launch: wait until the predecessor grid has
// finished (no-op without the launch attribute), and let the successor be
// scheduled now (it still waits for this grid to finish before it reads).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_allow_successor() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ copies

// 16-byte cp.async; src_bytes = 0 writes zeros (the source is not read).
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}

// Arrive on `bar` once all cp.async operations issued so far by this thread
// have completed (the arrival counts against the barrier's initial count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait_group()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Make generic-proxy writes to shared memory (cp.async, st.shared)
// visible to the async proxy (tcgen05.mma operand reads).
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Bulk global -> shared copy on the TMA engine, completion counted in
// bytes on `bar`.  dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Tiled 2-D tensor copy global -> shared on the TMA engine (no multicast):
// the box at element coordinates (x, y) of the tensor map, completion
// counted in bytes on `bar`.  x * element size must be a multiple of 16
// bytes; rows past the tensor's extent arrive as zeros.
__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, int x, int y, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// One TMA copy of a 3D box: (64 elements of K, rows, k-steps) of a map whose
// third dimension steps 128 bytes along a row, so the box lands as one
// 128-byte-swizzled [rows x 64] slab per k-step.
__device__ __forceinline__ void tma_load_3d(void *dst, const void *tmap, int x, int y, int z, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const void *tmap)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// ------------------------------------------------------------------ tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem], kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void mma_ts_f16(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[smem] * B[smem], kind::f16.
__device__ __forceinline__ void mma_ss_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when all tcgen05 operations issued so far by this
// thread have completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Instruction descriptor, kind::f16: bf16 A and B (K-major), fp32 D,
// M = 128, N = n (multiple of 16, 16..256).
__device__ __forceinline__ uint32_t idesc_bf16_f32(uint32_t m, uint32_t n)
{
    return (1u << 4)                 // D format: fp32
           | (1u << 7)               // A format: bf16
           | (1u << 10)              // B format: bf16
           | ((n >> 3) << 17)        // N >> 3
           | ((m >> 4) << 24);       // M >> 4
}

// The same for fp16 A and B operands (format code 0)
__device__ __forceinline__ uint32_t idesc_f16_f32(uint32_t m, uint32_t n)
{
    return (1u << 4)                 // D format: fp32
           | ((n >> 3) << 17)        // N >> 3
           | ((m >> 4) << 24);       // M >> 4
}

// Shared-memory matrix descriptor: K-major operand in the 128-byte
// swizzled layout (rows of 64 bf16 = 128 B, 8-row atoms of 1024 B).
__device__ __forceinline__ uint64_t sdesc_kmajor_sw128(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);            // start address
    d |= (uint64_t)1 << 16;                            // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;                  // stride byte offset: next 8-row atom
    d |= (uint64_t)1 << 46;                            // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;                            // swizzle: 128 B
    return d;
}

// 32 lanes x 32 bit, 16 consecutive columns, one register per column.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
        "%13, %14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ misc

__device__ __forceinline__ void record_error(int *status, int code, int detail)
{
    if (status && atomicCAS(status, 0, code) == 0)
        status[1] = detail;
}

}  // namespace moeq4
