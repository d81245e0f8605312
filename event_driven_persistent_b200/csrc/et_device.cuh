// Device-side runtime of the event-tensor megakernels (sm_100a).
//
// * PTX wrappers: mbarrier, TMA (cp.async.bulk.tensor), tcgen05 (TMEM alloc,
//   MMA, commit, ld), acquire/release atomics, %globaltimer.
// * Event counters ("Event Tensor：用“事件张量”编译动态 Megakernel",
//   §Event Tensor, §Minimal runtime): an event is an int32 counter in
//   device memory.  notify() is one atomic add with release semantics;
//   wait() spins with acquire loads until the counter reaches the event's
//   wait count.  A counter here records notifications received, starting
//   at zero, so "remaining = wait_count - counter" is the pages' count-down
//   value and an event fires when that reaches zero.  Starting from zero
//   means a run needs no initialisation pass that depends on T.
// * Every spin is bounded (time and iterations).  On expiry the thread
//   records ET_ERR_TIMEOUT plus where it was, raises the abort flag, and
//   every other spin in the grid sees the flag and returns, so the kernel
//   drains and exits normally (no trap).
// * Dynamic ready queue (§动态调度): a ring of 64-bit slots tagged with the
//   run's epoch; push reserves slots with one atomic on the tail and
//   publishes each slot with a release store; pop claims `fetch_batch`
//   consecutive slots with one atomic on the head (batched pops, as in
//   "MoE Kernel动态SM调度：从静态分配到任务池" §2.2).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "et_shared.h"

namespace et {

// ----------------------------------------------------------------- PTX ----

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smid() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
    return r;
}

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ int ld_volatile(const int* p) { return *reinterpret_cast<const volatile int*>(p); }

__device__ __forceinline__ int ld_relaxed(const int* p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
// after a relaxed load observed a released value: acquire (fence) once
__device__ __forceinline__ void fence_acquire() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Spin back-off: 148 SMs polling a few counters must not flood the L2 slice
// that holds them (which slows every other access to that slice).
// Exponential back-off between polls, 32 ns up to `cap` ns: short enough
// that a hop from one task to the next costs little, long enough that
// 148 pollers do not crowd the L2 slice of one counter.
struct Backoff {
    uint32_t ns = 32;
    uint32_t cap = 512;
    __device__ __forceinline__ explicit Backoff(uint32_t c = 512) : cap(c) {}
    __device__ __forceinline__ void pause() {
        __nanosleep(ns);
        if (ns < cap) ns <<= 1;
    }
};

// atomic add, acquire+release at GPU scope; returns the old value
__device__ __forceinline__ int atom_add_acq_rel(int* p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ int atom_add_relaxed(int* p, int v) {
    int old;
    asm volatile("atom.relaxed.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// generic-proxy writes -> later async-proxy (TMA) reads of global memory
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------- mbarrier ----

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* b, uint32_t tx) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(tx)
                 : "memory");
}
// raise the phase's expected transaction bytes without arriving
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t tx) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(tx) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* b, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(b)), "r"(parity)
        : "memory");
    return ok != 0;
}

// ------------------------------------------------------------- cp.async ----

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// the mbarrier's next phase also waits for every cp.async this thread issued
// so far (the pending count is raised now and lowered when they land)
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* b) {
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// non-blocking: has the phase with this parity completed?
__device__ __forceinline__ bool mbar_test(uint64_t* b, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(b)), "r"(parity)
        : "memory");
    return ok != 0;
}

// ----------------------------------------------------------------- TMA ----

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// -------------------------------------------------------------- tcgen05 ----

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 x bf16 -> fp32, one CTA
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// arrive on an mbarrier once every tcgen05 op issued so far by this thread completes
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
// 32 lanes x 16 consecutive fp32 columns: thread i of the warp gets lane
// (quadrant*32 + i).  The load and its wait are one asm statement: the
// destination registers of tcgen05.ld are written asynchronously and are
// only valid after tcgen05.wait::ld, so the compiler must not see them as
// defined (and schedule their uses) before the wait.
__device__ __forceinline__ void tmem_ld4_wait(uint32_t taddr, float (&v)[4]) {
    uint32_t r[4];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld16_wait(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Instruction descriptor, kind::f16: D fp32, A/B bf16, both K-major, M x N.
__device__ __forceinline__ uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Shared-memory matrix descriptor: K-major, 128-byte swizzle, rows of 128 B,
// 8-row groups 1024 B apart (stride byte offset), sm_100 descriptor version 1.
__device__ __forceinline__ uint64_t sdesc_k128(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// ------------------------------------------------------ control / errors ----



// Record the first device error of a run: the sticky status word and the
// diagnostic words in device memory, a copy of the status in mapped host
// memory (so the host sees it without a synchronisation), and the grid-wide
// abort flag every spin checks.
__device__ __forceinline__ void fail(Ctl* ctl, int code, int where, int a, int b, int c) {
    if (atomicCAS(&ctl->status, 0, code) == 0) {
        ctl->diag[0] = where;
        ctl->diag[1] = a;
        ctl->diag[2] = b;
        ctl->diag[3] = c;
        ctl->diag[4] = (int)blockIdx.x;
        ctl->diag[5] = (int)threadIdx.x;
        if (ctl->host_status) {
            *reinterpret_cast<volatile int*>(ctl->host_status) = code;
            __threadfence_system();
        }
    }
    __threadfence();
    atomicExch(&ctl->abort, 1);
}

__device__ __forceinline__ bool aborted(const Ctl* ctl) { return ld_volatile(&ctl->abort) != 0; }

// Spin budget: time limit (ns) and a hard iteration cap, whichever comes first.
constexpr uint32_t kMaxSpinIters = 1u << 26;

// wait(): spin until *ctr >= target.  false on timeout/abort.  The check
// of an event that is already complete is inline; the bounded spin is out
// of line (many call sites; the megakernel's instruction footprint matters).
static __device__ __noinline__ bool wait_geq_spin(const int* ctr, int target, Ctl* ctl, uint64_t timeout_ns, int where,
                                                  int ev) {
    uint64_t t0 = globaltimer();
    Backoff bo;
    for (uint32_t it = 1;; ++it) {
        bo.pause();
        if (ld_relaxed(ctr) >= target) {
            fence_acquire();
            return true;
        }
        if ((it & 31) == 0) {
            if (aborted(ctl)) return false;
            if (globaltimer() - t0 > timeout_ns || it > kMaxSpinIters) {
                fail(ctl, ET_ERR_TIMEOUT, where, ev, target, ld_volatile(ctr));
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool wait_geq(const int* ctr, int target, Ctl* ctl, uint64_t timeout_ns, int where, int ev) {
    if (ld_acquire(ctr) >= target) return true;
    return wait_geq_spin(ctr, target, ctl, timeout_ns, where, ev);
}

// notify(): add n with release (and acquire, so that the notifier that
// completes an event has seen every earlier producer's writes before it
// pushes consumers).  Returns the new count.
__device__ __forceinline__ int notify(int* ctr, int n) {
    __threadfence();
    return atom_add_acq_rel(ctr, n) + n;
}

// bounded mbarrier wait (parity); false on timeout/abort.  A phase that is
// already complete is seen inline; the bounded spin is out of line.
static __device__ __noinline__ bool mbar_wait_spin(uint64_t* b, uint32_t parity, Ctl* ctl, uint64_t timeout_ns,
                                                   int where) {
    uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(b, parity)) return true;
        if ((it & 15) == 0) {
            if (aborted(ctl)) return false;
            if (globaltimer() - t0 > timeout_ns || it > kMaxSpinIters) {
                fail(ctl, ET_ERR_TIMEOUT, where, (int)parity, 0, 0);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, Ctl* ctl, uint64_t timeout_ns, int where) {
    if (mbar_try_wait(b, parity)) return true;
    return mbar_wait_spin(b, parity, ctl, timeout_ns, where);
}

// A phase that one thread of a group has already seen complete, observed by
// every other thread of the group (acquire per thread).  It cannot advance
// again before the whole group moves on, so this ends at once; the loop is
// still bounded, and a bound that runs out is recorded as ET_ERR_TIMEOUT
// (the caller carries on; the run then aborts at its next check).
__device__ __forceinline__ void mbar_observe(uint64_t* b, uint32_t parity, Ctl* ctl, int where) {
    for (uint32_t it = 0; !mbar_try_wait(b, parity); ++it)
        if (it > (1u << 20)) {
            fail(ctl, ET_ERR_TIMEOUT, where, (int)parity, -1, 0);
            return;
        }
}

// ---------------------------------------------------------------- trace ----

__device__ __forceinline__ uint32_t take_ticket(Ctl* ctl) { return atomicAdd(&ctl->ticket, 1u); }

__device__ __forceinline__ void trace_write(Ctl* ctl, TraceRec* buf, int cap, const TraceRec& r) {
    int i = atomicAdd(&ctl->n_trace, 1);
    if (i < cap) buf[i] = r;
}

// pseudo-random delay (debug): 0 .. ~20 us
static __device__ __noinline__ void debug_delay(uint32_t key) {
    uint32_t h = key * 2654435761u;
    h ^= h >> 15;
    h *= 2246822519u;
    h ^= h >> 13;
    uint64_t ns = (uint64_t)(h % 20000u);
    uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < ns) __nanosleep(256);
}

// ---------------------------------------------------------------- queue ----
// Task words: op (6 bits) | a (16 bits) | b (10 bits).
__device__ __forceinline__ uint32_t task_word(int op, int a, int b) {
    return ((uint32_t)op << 26) | ((uint32_t)(a & 0xFFFF) << 10) | (uint32_t)(b & 0x3FF);
}
__device__ __forceinline__ int task_op(uint32_t w) { return (int)(w >> 26); }
__device__ __forceinline__ int task_a(uint32_t w) { return (int)((w >> 10) & 0xFFFF); }
__device__ __forceinline__ int task_b(uint32_t w) { return (int)(w & 0x3FF); }

struct Queue {
    unsigned long long* slots;  // capacity entries, (epoch << 32) | task word
    int cap;
    Ctl* ctl;                   // error reporting (a push past the capacity)
    int* head;                  // next slot to claim
    int* tail;                  // next slot to fill
    int* total;                 // total tasks this run + 1 (0 = not known yet)
    uint32_t epoch;
    int n_init;                 // slots [0, n_init) hold the initial tasks implicitly
    int total_static;           // > 0: the run's task count is known at launch
};

// reserve n slots after the implicit initial ones; returns the first index
__device__ __forceinline__ int q_reserve(const Queue& q, int n) { return q.n_init + atom_add_relaxed(q.tail, n); }

// The ring never wraps within a run: its capacity covers every task of the
// largest run plus one over-claimed batch per CTA, so a slot index is never
// shared by two tasks of one run.  A push past the capacity would lose its
// task: it is recorded as ET_ERR_INTERNAL (and the run aborts) instead.
static __device__ __noinline__ void q_overflow(const Queue& q, int idx) {
    fail(q.ctl, ET_ERR_INTERNAL, 903, idx, q.cap, (int)q.epoch);
}
__device__ __forceinline__ void q_publish(const Queue& q, int idx, uint32_t word) {
    if (idx < q.cap) st_release_u64(&q.slots[idx], ((unsigned long long)q.epoch << 32) | word);
    else q_overflow(q, idx);
}
// Publish after the caller issued one release fence for the whole batch.
__device__ __forceinline__ void q_publish_after_fence(const Queue& q, int idx, uint32_t word) {
    if (idx < q.cap)
        asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(&q.slots[idx]),
                     "l"(((unsigned long long)q.epoch << 32) | word)
                     : "memory");
    else
        q_overflow(q, idx);
}

// Resolve slot `idx`: 1 = task in *word, 0 = no more tasks (idx beyond the
// run's total), -1 = timeout/abort.
template <class InitFn>
__device__ __forceinline__ int q_resolve(const Queue& q, int idx, uint32_t* word, InitFn init_task, Ctl* ctl,
                                         uint64_t timeout_ns) {
    if (idx < q.n_init) {
        *word = init_task(idx);
        return 1;
    }
    if (idx >= q.cap) return 0;  // beyond any run's last task
    const unsigned long long* s = &q.slots[idx];
    uint64_t t0 = 0;
    Backoff bo(256);
    for (uint32_t it = 0;; ++it) {
        unsigned long long v = ld_relaxed_u64(s);
        if ((uint32_t)(v >> 32) == q.epoch) {
            fence_acquire();
            *word = (uint32_t)v;
            return 1;
        }
        int tot = q.total_static > 0 ? q.total_static + 1 : ld_relaxed(q.total);
        if (tot > 0 && idx >= tot - 1) return 0;
        if (it == 0) t0 = globaltimer();
        bo.pause();
        if ((it & 31) == 31) {
            if (aborted(ctl)) return -1;
            if (globaltimer() - t0 > timeout_ns || it > kMaxSpinIters) {
                fail(ctl, ET_ERR_TIMEOUT, 900, idx, tot, 0);
                return -1;
            }
        }
    }
}

}  // namespace et
