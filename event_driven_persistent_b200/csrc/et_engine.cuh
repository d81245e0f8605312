// The persistent megakernel skeleton shared by the three workloads.
//
// One CTA per SM runs until its task source is exhausted ("Event Tensor：用
// “事件张量”编译动态 Megakernel", §Minimal runtime: dispatch, wait, notify
// and push/pop are compiled into the kernel; the only mutable run-time state
// is the event counters and the queue).  Roles inside a CTA:
//
//   warp 0, lane 0  task source + TMA producer.  Static: walks this CTA's
//                   task list.  Dynamic: pops the ready queue in batches.
//                   For a tensor-core task it issues the weight (A) tiles of
//                   the first pipeline stages BEFORE waiting on the task's
//                   input event (weights never depend on activations, so
//                   they stream while the producer tasks finish), then
//                   waits, then loads the activation (B) tiles.
//   warp 1, lane 0  tcgen05.mma issuer: D[tmem] += A[smem] * B[smem]^T,
//                   bf16 in, fp32 accumulate, two TMEM accumulators so the
//                   epilogue of one task overlaps the main loop of the next.
//   warps 2..5      epilogues (tcgen05.ld of the accumulator, fused
//                   element-wise math, stores, notify/push) and all CUDA-core
//                   tasks (norm, reductions, top-k, grouping, combine).
//   warp 6          (workloads with gathered B rows only) the cp.async row
//                   copies of gathered stages, so that warp 0's weight
//                   stream never waits on them.
//
// Tasks flow from warp 0 to the others through a 2-deep ring in shared
// memory guarded by mbarriers.
#pragma once
#include "et_device.cuh"

namespace et {

constexpr uint32_t kExitWord = 0xFFFFFFFFu;

struct TaskDesc {
    uint32_t word;   // task word, kExitWord = stop
    int valid;       // 0 = a static slot with nothing to do at this size
    uint32_t start;  // trace ticket taken after the task's wait
    int gemm;        // 1 = tensor-core task
    int gather;      // 1 = B rows gathered through W::gather_row (cp.async, gather warp), else B by TMA
    uint64_t t_fetch, t_ready, t_acc;  // trace timestamps (ns)
    int a_map, a_row0, a_row1;  // A: tensor map id, rows of the two 64-row boxes
    int b_map, b_row0;          // B: tensor map id, first row
    int n;                      // MMA N (multiple of 16, <= kMaxN)
    int k0, nk;                 // first K element, number of 128-wide K stages (stream: stages)
    int stream;                 // 1 = stream task: warp 0 copies nk byte blocks into arena stages,
                                //     the exec group consumes them (no tensor-core work)
    uint32_t sbytes;            // stream: bytes reserved per stage (1 KB multiple)
    uint32_t st0, off0;         // stream: global index and arena offset of the task's first stage
    int attn;                   // stream task whose stages also run two tensor-core products per
                                //     stage (the attention protocol: S = K Q^T, then O = V^T P^T)
    int p[6];                   // workload-specific
};


struct SmemCtl {
    uint64_t full[kSlots];
    uint64_t empty[kSlots];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t ring_full[kRing];
    uint64_t ring_empty[kRing];
    uint64_t drain;
    uint64_t s_full[2], p_full[2], o_full[2];  // attention stages k: buffers k & 1 of S, P and O
    uint64_t gready[kSlots];  // gathered stage reserved and its weight tile issued (warp 0 -> gather warp)
    uint32_t tmem_base;
    int start_status;
    int bcast[8];
    uint64_t bcast64[2];
    TaskDesc ring[kRing];
    TaskDesc pd;  // warp 0: the task lane 0 fetched, for the other lanes
    int pr, pbrk, pok;
    uint32_t pslot, poff;
    uint32_t r_off[kSlots], r_end[kSlots];  // arena range of the last kSlots stages
};

// Everything a role needs besides the workload parameters.
struct Ctx {
    Ctl* ctl;
    uint64_t timeout_ns;
    int* ctr;            // this run's counter set
    Queue q;
    int dynamic;         // 1 = ready queue, 0 = static lists
    int debug;           // ET_DEBUG_* bits
    TraceRec* trace;
    int trace_cap;
    uint8_t* arena;      // pipeline stages, 1024-aligned
    float* epi;          // gate/up exchange staging
    uint8_t* simt;       // CUDA-core task scratch
    SmemCtl* sc;
    int tid;             // exec-group thread index 0..127 (exec warps only)
    // attention stream tasks (exec group): this task's TMEM accumulator (this
    // warp's lane quadrant), its release barrier, and the attention stages
    // consumed so far (the phase of s_full / p_full / o_full)
    uint32_t taddr;
    uint64_t* acc_empty;
    uint32_t na;
};

// Defaults of the workload interface for what a workload does not use.
struct WorkloadBase {
    // engine paths a workload uses (the others are compiled out: a smaller
    // megakernel has less code to fetch cold)
    static constexpr bool kStream = false;  // stream / attention tasks
    static constexpr bool kGather = false;  // tensor-core tasks with gathered B rows
    // stream tasks: stages that may be copied before the task's input wait,
    // the bytes stage s delivers, and the copies of stage s into `dst`
    // (completing on `bar`); `late` = issued after the input wait, so the
    // copies that depend on the task's inputs are included
    template <class P>
    __device__ static int stream_prefetch(const P&, const TaskDesc&) { return 0; }
    template <class P>
    __device__ static uint32_t stream_bytes(const P&, const TaskDesc&, int) { return 0; }
    template <class P>
    __device__ static void stream_copy(const P&, const TaskDesc&, int, uint8_t*, uint64_t*, uint64_t, bool) {}
    // the input-dependent copies of stage s, which was copied before the
    // wait (its expected bytes counted them)
    template <class P>
    __device__ static void stream_late(const P&, const TaskDesc&, int, uint8_t*, uint64_t*, uint64_t) {}
    template <class P>
    __device__ static bool stream_exec(const P&, Ctx&, TaskDesc&) { return false; }
    // B operand map with a 64-row box (the same tensor as b_map), for the
    // 64-row chunks of wide token tiles: one copy instead of four; null = none
    template <class P>
    __device__ static const CUtensorMap* b_map_wide(const P&, int) { return nullptr; }
};

__device__ __forceinline__ void exec_bar() { named_bar_sync(1, kExecThreads); }

// Push n consumer tasks from the exec group (all 128 threads call; n uniform).
template <class Gen>
__device__ __forceinline__ void group_push(Ctx& x, int n, Gen gen) {
    if (n <= 0) return;
    if (x.tid == 0) x.sc->bcast[0] = q_reserve(x.q, n);
    exec_bar();
    int base = x.sc->bcast[0];
    if (x.tid < n) __threadfence();  // release: this task's writes before its pushes
    for (int i = x.tid; i < n; i += kExecThreads) q_publish_after_fence(x.q, base + i, gen(i));
    exec_bar();
}

// Push n tasks from a single thread.
template <class Gen>
__device__ __forceinline__ void thread_push(Ctx& x, int n, Gen gen) {
    if (n <= 0) return;
    int base = q_reserve(x.q, n);
    __threadfence();
    for (int i = 0; i < n; ++i) q_publish_after_fence(x.q, base + i, gen(i));
}

// Trace record of a finished task (debug; out of line, off the hot path).
static __device__ __noinline__ void trace_task(Ctl* ctl, TraceRec* buf, int cap, uint32_t word, uint32_t start,
                                               uint64_t t_fetch, uint64_t t_ready, uint64_t t_acc,
                                               uint32_t end_ticket, uint64_t t_end) {
    TraceRec r;
    r.end = end_ticket;
    r.t_end = t_end;
    r.op = task_op(word);
    r.a = task_a(word);
    r.b = task_b(word);
    r.sm = (int)smid();
    r.start = start;
    r.t_fetch = t_fetch;
    r.t_ready = t_ready;
    r.t_acc = t_acc;
    trace_write(ctl, buf, cap, r);
}

// End of a task in the exec group: every thread has written its outputs.
// Thread 0 records the trace and adds `n` to one event counter; returns (to
// all threads) whether this notify completed the event (counter == target).
// With trace_if_fired false, a notify that completes the event writes no
// trace record (the task goes on with more work and records at its end).
__device__ __forceinline__ bool group_finish_notify(Ctx& x, const TaskDesc& d, int* ctr, int n, int target,
                                                    bool trace_if_fired = true) {
    exec_bar();
    if (x.tid == 0) {
        int fired = 0;
        const bool tr = (x.debug & ET_DEBUG_TRACE) != 0;
        uint32_t tk = 0;
        uint64_t te = 0;
        if (tr) {
            tk = take_ticket(x.ctl);
            te = globaltimer();
        }
        if (ctr) fired = notify(ctr, n) == target;
        if (tr && (trace_if_fired || !fired))
            trace_task(x.ctl, x.trace, x.trace_cap, d.word, d.start, d.t_fetch, d.t_ready, d.t_acc, tk, te);
        x.sc->bcast[1] = fired;
    }
    exec_bar();
    return x.sc->bcast[1] != 0;
}

// Exec-group wait on an event (SIMT tasks).  Returns false on timeout/abort.
__device__ __forceinline__ bool group_wait(Ctx& x, TaskDesc& d, const int* ctr, int target, int where) {
    if (x.tid == 0) {
        bool ok = ctr == nullptr || wait_geq(ctr, target, x.ctl, x.timeout_ns, where, task_word(0, 0, 0) ^ d.word);
        if (ok && (x.debug & ET_DEBUG_TRACE)) {
            d.start = take_ticket(x.ctl);
            d.t_ready = globaltimer();
        }
        x.sc->bcast[2] = ok;
        x.sc->bcast[3] = (int)d.start;
        x.sc->bcast64[0] = d.t_ready;
    }
    exec_bar();
    bool ok = x.sc->bcast[2] != 0;
    d.start = (uint32_t)x.sc->bcast[3];
    d.t_ready = x.sc->bcast64[0];
    exec_bar();
    return ok;
}

// Bytes of one pipeline stage: the weight tile, then N activation rows
// (1 KB multiples keep every tile on the 128-byte swizzle atom).
// (per K atom: 128 weight rows, then N activation rows; n is a multiple of 16)
__device__ __forceinline__ uint32_t stage_bytes(int n) { return kAStageBytes + 2u * (uint32_t)n * 128u; }


// Stream tasks, exec group: wait for stage s of the task (all 128 threads
// call; false on timeout/abort) and return its arena offset in *off.
__device__ __forceinline__ bool stream_stage_wait(Ctx& x, const TaskDesc& d, int s, StageAlloc& a, uint32_t* off) {
    const uint32_t g = d.st0 + (uint32_t)s;
    const uint32_t slot = g % kSlots, par = (g / kSlots) & 1;
    *off = a.next(d.sbytes);
    if (x.tid == 0) x.sc->bcast[5] = mbar_wait(&x.sc->full[slot], par, x.ctl, x.timeout_ns, 925);
    exec_bar();
    const bool ok = x.sc->bcast[5] != 0;
    if (ok) mbar_observe(&x.sc->full[slot], par, x.ctl, 926);
    return ok;
}
// ... and hand stage s back to the producer once every thread is done with it.
__device__ __forceinline__ void stream_stage_release(Ctx& x, const TaskDesc& d, int s) {
    exec_bar();
    if (x.tid == 0) mbar_arrive(&x.sc->empty[(d.st0 + (uint32_t)s) % kSlots]);
}
// Exec group: wait for phase `parity` of an mbarrier that another role
// completes (all 128 threads call; false on timeout/abort).  Thread 0 waits
// with the bound and broadcasts through bcast[slot]; then every thread
// observes the phase itself.  A slot is written again only after another
// exec-group barrier, so no thread can read a later call's result.
__device__ __forceinline__ bool exec_mbar_wait(Ctx& x, uint64_t* bar, uint32_t parity, int where, int slot) {
    if (x.tid == 0) x.sc->bcast[slot] = mbar_wait(bar, parity, x.ctl, x.timeout_ns, where);
    exec_bar();
    const bool ok = x.sc->bcast[slot] != 0;
    if (ok) mbar_observe(bar, parity, x.ctl, where + 1000);
    return ok;
}
__device__ __forceinline__ StageAlloc stream_alloc(const TaskDesc& d) {
    StageAlloc a;
    a.head = d.off0;
    return a;
}

// B rows of one stage for tiles of more than 32 rows (all 32 lanes of the
// gather warp call): eight lanes per row, so one copy instruction covers
// the 128-byte K atom of four rows (four whole lines); lane l holds the
// addresses of rows l, l + 32, l + 64 and l + 96 (null past the task's
// rows) and hands them to the lanes that copy them.  The 32-row blocks are
// a rolled loop: the code stays small.
__device__ __forceinline__ void gather_rows_wide(uint8_t* bdst, uint32_t atom, int n, int kx, int lane,
                                                 const uint16_t* const (&rows)[4]) {
    const int sub = lane >> 3, cc = lane & 7;
#pragma unroll 1
    for (int i = 0; 32 * i < n; ++i) {
        const uint16_t* r = i == 0 ? rows[0] : i == 1 ? rows[1] : i == 2 ? rows[2] : rows[3];
        const unsigned long long mine = reinterpret_cast<unsigned long long>(r);
        const uint16_t* src[8];  // all eight hand-offs first: independent
#pragma unroll
        for (int g = 0; g < 8; ++g)
            src[g] = reinterpret_cast<const uint16_t*>(__shfl_sync(0xffffffffu, mine, 4 * g + sub));
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            const int rr = 32 * i + 4 * g + sub;
            if (src[g] && rr < n) {
                uint8_t* dr = bdst + rr * 128 + ((cc ^ (rr & 7)) << 4);
                cp_async16(dr, src[g] + kx + cc * 8);
                cp_async16(dr + atom, src[g] + kx + kAtomK + cc * 8);
            }
        }
    }
}

// Megakernel body.  W supplies the task semantics:
//   W::fetch_init(p, idx)              initial dynamic task word for slot idx
//   W::derive(p, x, word, d)           fill a TaskDesc (warp 0; may wait in
//                                      static mode); false = abort
//   W::gemm_wait(p, x, d)              the GEMM task's input wait (warp 0)
//   W::gather_row(p, d, r)             B row r of a gather task (d.gather)
//   W::a_map(p, id), W::b_map(p, id)   tensor maps
//   W::epilogue(p, x, d, acc_taddr)    exec group, after the accumulator is ready
//   W::simt(p, x, d)                   exec group, a CUDA-core task
//   W::stream_prefetch / stream_copy   (stream tasks) warp 0, see WorkloadBase
//   W::stream_exec(p, x, d)            exec group, a stream task (stream_stage_wait/release)
// Task sources: static (this CTA's list), dynamic (the ready queue), or
// hybrid: this CTA's list part A, then the ready queue until it is
// exhausted, then its list part B.
template <class W>
__device__ __forceinline__ void megakernel_body(const typename W::Params& p, const RunArgs& ra) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* arena = base;
    uint8_t* scratch = arena + ((W::kGemm || W::kStream) ? kArenaBytes : 0);
    float* epi = reinterpret_cast<float*>(scratch);
    uint8_t* simt = scratch + kEpiBytes;
    SmemCtl* sc = reinterpret_cast<SmemCtl*>(scratch + kScratchBytes);
    static_assert(sizeof(SmemCtl) <= kCtlBytes, "control block does not fit");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Ctl* ctl = ra.ctl;
    const bool cta_times = (ra.debug & (ET_DEBUG_TRACE | ET_DEBUG_CTA_TIMES)) == (ET_DEBUG_TRACE | ET_DEBUG_CTA_TIMES);
    uint64_t t_enter = 0, t_setup = 0;
    if (cta_times && threadIdx.x == 0) t_enter = globaltimer();

    // zero the other parity's counter set for the next run
    {
        int* other = ra.ctr_next;
        for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < ra.n_ctr; i += gridDim.x * blockDim.x) other[i] = 0;
    }
    if (threadIdx.x == 0) {
        sc->start_status = ld_volatile(&ctl->status);
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(&sc->full[s], 1);
            mbar_init(&sc->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sc->acc_full[b], 1);
            mbar_init(&sc->acc_empty[b], kExecThreads / 32);
        }
        for (int r = 0; r < kRing; ++r) {
            mbar_init(&sc->ring_full[r], 1);
            mbar_init(&sc->ring_empty[r], W::kGather ? 3 : 2);  // MMA warp + exec group (+ gather warp)
        }
        mbar_init(&sc->drain, 1);
        for (int s = 0; s < kSlots; ++s) mbar_init(&sc->gready[s], 1);
        mbar_init(&sc->s_full[0], 1);
        mbar_init(&sc->s_full[1], 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sc->p_full[b], 1);
            mbar_init(&sc->o_full[b], 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    if (warp == 1 && W::kGemm) {
        tmem_alloc(&sc->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool skip = sc->start_status != 0;  // an earlier run failed: do nothing until the host resets
    if (cta_times && threadIdx.x == 0) t_setup = globaltimer();

    Ctx x;
    x.ctl = ctl;
    x.timeout_ns = ra.timeout_ns;
    x.ctr = ra.ctr;
    x.q.slots = ra.qslots;
    x.q.cap = ra.qcap;
    x.q.ctl = ctl;
    x.q.head = ra.ctr + 0;
    x.q.tail = ra.ctr + 1;
    x.q.total = ra.ctr + 2;
    x.q.epoch = ra.epoch;
    x.q.n_init = ra.n_init;
    x.q.total_static = ra.total_static;
    x.dynamic = ra.dynamic;
    x.debug = ra.debug;
    x.trace = ra.trace;
    x.trace_cap = ra.trace_cap;
    x.arena = arena;
    x.epi = epi;
    x.simt = simt;
    x.sc = sc;
    x.tid = threadIdx.x - kExecWarp0 * 32;
    x.taddr = 0;
    x.acc_empty = nullptr;
    x.na = 0;


    if (!skip && warp == 0) {
        // ---------------------------------------------------- task source + loads
        // Lane 0 leads (task fetch, waits, TMA, ring); the other lanes follow
        // (the B rows of gathered tasks are copied by the gather warp).
        const uint64_t pol_w = policy_evict_first();
        const uint64_t pol_a = policy_evict_last();
        // phase 0: list part A; 1: ready queue; 2: list part B
        int lpos = 0, lend = 0, phase = x.dynamic && !ra.hybrid ? 1 : 0;
        if (phase == 0) {
            lpos = ra.lists.off[blockIdx.x];
            lend = ra.lists.off[blockIdx.x + 1];
        }
        int qn = 0, qe = 0;
        // lane 0: stage bookkeeping (global stage count, arena ranges of the
        // last kSlots stages, arms per slot for the exit drain)
        uint32_t nst = 0, tail = 0;  // stages reserved so far; oldest stage not yet seen consumed
        StageAlloc alloc;
        uint32_t armed[kSlots];
        for (int s2 = 0; s2 < kSlots; ++s2) armed[s2] = 0;
        // Reserve the next stage: consume (wait for) stages in order, oldest
        // first, while the new stage is blocked (stage_blocked).
        auto reserve = [&](uint32_t size, uint32_t* slot_out, uint32_t* off_out) -> bool {
            const uint32_t off = alloc.next(size);
            while (tail < nst && stage_blocked(off, size, tail, nst, sc->r_off, sc->r_end)) {
                const uint32_t ts = tail % kSlots;
                if (!mbar_wait(&sc->empty[ts], (tail / kSlots) & 1, ctl, x.timeout_ns, 902)) return false;
                ++tail;
            }
            const uint32_t slot2 = nst % kSlots;
            sc->r_off[slot2] = off;
            sc->r_end[slot2] = off + size;
            ++nst;
            *slot_out = slot2;
            *off_out = off;
            return true;
        };
        auto issue_b = [&](uint32_t slot2, uint32_t off, const CUtensorMap* bm2, const TaskDesc& dd, int stage,
                           uint64_t pol) {
            uint8_t* bdst = arena + off + kAStageBytes;
            const uint32_t atom = (uint32_t)dd.n * 128u;
            const int kx = dd.k0 + stage * kTileK;
            const CUtensorMap* bw = W::b_map_wide(p, dd.b_map);
            for (int rb = 0; rb < dd.n;) {
                const bool wide = bw != nullptr && rb + 64 <= dd.n;  // a 64-row box where one fits
#pragma unroll
                for (int at = 0; at < 2; ++at)
                    tma_load_2d(bdst + at * atom + rb * 128, wide ? bw : bm2, &sc->full[slot2], kx + at * kAtomK,
                                dd.b_row0 + rb, pol);
                rb += wide ? 64 : 16;
            }
        };
        auto issue_a = [&](uint32_t slot2, uint32_t off, const CUtensorMap* am2, const TaskDesc& dd, int stage,
                           uint32_t tx, uint64_t pol, bool arrive = true) {
            if (arrive)
                mbar_arrive_expect_tx(&sc->full[slot2], tx);
            else
                mbar_expect_tx(&sc->full[slot2], tx);
            ++armed[slot2];
            uint8_t* dst = arena + off;
            const int kx = dd.k0 + stage * kTileK;
#pragma unroll
            for (int at = 0; at < 2; ++at) {
                tma_load_2d(dst + at * kAAtomBytes, am2, &sc->full[slot2], kx + at * kAtomK, dd.a_row0, pol);
                tma_load_2d(dst + at * kAAtomBytes + 64 * 128, am2, &sc->full[slot2], kx + at * kAtomK, dd.a_row1, pol);
            }
        };
        for (uint32_t it = 0;; ++it) {
            const uint32_t slot = it % kRing;
            if (lane == 0) {
                TaskDesc d;
                d.word = kExitWord;
                d.valid = 0;
                d.gemm = 0;
                d.gather = 0;
                d.stream = 0;
                d.attn = 0;
                d.start = 0;
                d.t_fetch = d.t_ready = d.t_acc = 0;
                int r = 0;
                for (;;) {
                    if (phase != 1) {
                        const uint32_t* words = phase == 0 ? ra.lists.words : ra.lists.words_b;
                        r = lpos < lend ? 1 : 0;
                        if (r) {
                            d.word = words[lpos++];
                            break;
                        }
                        if (phase == 0 && ra.hybrid) {
                            phase = 1;
                            continue;
                        }
                        break;
                    }
                    if (qn == qe) {
                        qn = atom_add_relaxed(x.q.head, ra.fetch_batch);
                        qe = qn + ra.fetch_batch;
                    }
                    uint32_t w;
                    r = q_resolve(x.q, qn, &w, [&](int i) { return W::fetch_init(p, i); }, ctl, x.timeout_ns);
                    ++qn;
                    if (r == 1) d.word = w;
                    if (r == 0 && ra.hybrid && ra.lists.off_b) {
                        phase = 2;
                        lpos = ra.lists.off_b[blockIdx.x];
                        lend = ra.lists.off_b[blockIdx.x + 1];
                        continue;
                    }
                    break;
                }
                bool brk = r < 0;
                if (!brk && (x.debug & ET_DEBUG_TRACE)) d.t_fetch = globaltimer();
                if (!brk && r == 1 && !W::derive(p, x, d)) brk = true;
                if (!brk && !mbar_wait(&sc->ring_empty[slot], ((it / kRing) & 1) ^ 1, ctl, x.timeout_ns, 901))
                    brk = true;
                sc->pd = d;
                sc->pr = r;
                sc->pbrk = brk;
            }
            __syncwarp();
            const bool brk = sc->pbrk;
            const int r = sc->pr;
            TaskDesc d = sc->pd;
            __syncwarp();
            if (brk) break;
            if (W::kStream && r == 1 && d.valid && d.stream) {
                // stream task: stages that do not depend on the task's input
                // events first, then the wait, then the rest
                bool ok = true;
                if (lane == 0) {
                    const int fit = kArenaBytes / (int)d.sbytes - 1;
                    int npre = W::stream_prefetch(p, d);
                    npre = npre < fit ? npre : fit;
                    npre = npre < kSlots - 1 ? npre : kSlots - 1;
                    npre = npre < d.nk ? npre : d.nk;
                    d.st0 = nst;
                    {
                        StageAlloc probe = alloc;  // where the first stage will land
                        d.off0 = probe.head;
                    }
                    uint32_t pre_sl[kSlots], pre_of[kSlots];  // the stages copied before the wait
                    auto issue_s = [&](int st, bool late) -> bool {
                        uint32_t sl, of;
                        if (!reserve(d.sbytes, &sl, &of)) return false;
                        if (!late) {
                            pre_sl[st] = sl;
                            pre_of[st] = of;
                        }
                        mbar_arrive_expect_tx(&sc->full[sl], W::stream_bytes(p, d, st));
                        ++armed[sl];
                        W::stream_copy(p, d, st, arena + of, &sc->full[sl], pol_w, late);
                        return true;
                    };
                    int s2 = 0;
                    for (; s2 < npre && ok; ++s2) ok = issue_s(s2, false);
                    if (ok) ok = W::gemm_wait(p, x, d);  // the task's input events
                    if (ok) fence_proxy_async_global();  // inputs written this run -> the copies below
                    if (ok && (x.debug & ET_DEBUG_TRACE)) {
                        d.start = take_ticket(ctl);
                        d.t_ready = globaltimer();
                    }
                    sc->ring[slot] = d;
                    mbar_arrive(&sc->ring_full[slot]);
                    for (int i = 0; ok && i < s2; ++i) W::stream_late(p, d, i, arena + pre_of[i], &sc->full[pre_sl[i]], pol_a);
                    for (; ok && s2 < d.nk; ++s2) ok = issue_s(s2, true);
                    sc->pok = ok;
                }
                __syncwarp();
                ok = sc->pok;
                __syncwarp();
                if (!ok) break;
            } else if (W::kGemm && r == 1 && d.valid && d.gemm) {
                const CUtensorMap* am = W::a_map(p, d.a_map);
                const uint32_t bbytes = 2u * (uint32_t)d.n * 128u;  // both K atoms
                bool ok = true;
                if (!(W::kGather && d.gather)) {
                    if (lane == 0) {
                        const CUtensorMap* bm = W::b_map(p, d.b_map);
                        // 1. weight tiles of the first stages, before the input
                        //    wait (as many as fit without waiting on themselves)
                        const int fit = kArenaBytes / (int)stage_bytes(d.n) - 1;
                        int npre = d.nk < fit ? d.nk : fit;
                        npre = npre < kSlots - 1 ? npre : kSlots - 1;
                        uint32_t pslot[kSlots], poff[kSlots];
                        int s = 0;
                        for (; s < npre && ok; ++s) {
                            ok = reserve(stage_bytes(d.n), &pslot[s], &poff[s]);
                            if (ok) issue_a(pslot[s], poff[s], am, d, s, kAStageBytes + bbytes, pol_w);
                        }
                        if (ok) ok = W::gemm_wait(p, x, d);  // the task's input event
                        if (ok && (x.debug & ET_DEBUG_TRACE)) {
                            d.start = take_ticket(ctl);
                            d.t_ready = globaltimer();
                        }
                        if (ok) fence_proxy_async_global();
                        sc->ring[slot] = d;
                        mbar_arrive(&sc->ring_full[slot]);
                        // 2. activation tiles of the prefetched stages
                        for (int i = 0; ok && i < npre; ++i) {
                            issue_b(pslot[i], poff[i], bm, d, i, pol_a);
                        }
                        // 3. the remaining stages, weights and activations together
                        for (; ok && s < d.nk; ++s) {
                            uint32_t sl, of;
                            ok = reserve(stage_bytes(d.n), &sl, &of);
                            if (!ok) break;
                            issue_a(sl, of, am, d, s, kAStageBytes + bbytes, pol_w);
                            issue_b(sl, of, bm, d, s, pol_a);
                        }
                        sc->pok = ok;
                    }
                    __syncwarp();
                    ok = sc->pok;
                    __syncwarp();
                } else {
                    // B rows gathered through an index list: the gather warp
                    // copies them.  Per stage this warp reserves the stage,
                    // raises its expected bytes by the weight tile's without
                    // arriving, issues the weight tile and signals gready; the
                    // gather warp's arrival (after its row copies) completes
                    // the phase.  The weight stream never waits on the rows.
                    // (A gathered task's inputs are complete when it is
                    // derived: derive waits for them, or the queue holds the
                    // task only once they are.)
                    if (lane == 0) {
                        ok = W::gemm_wait(p, x, d);
                        if (ok && (x.debug & ET_DEBUG_TRACE)) {
                            d.start = take_ticket(ctl);
                            d.t_ready = globaltimer();
                        }
                        d.st0 = nst;  // the task's first stage: the gather warp follows from it
                        sc->ring[slot] = d;
                        mbar_arrive(&sc->ring_full[slot]);
                        for (int s = 0; ok && s < d.nk; ++s) {
                            uint32_t sl = 0, of = 0;
                            ok = reserve(stage_bytes(d.n), &sl, &of);
                            if (!ok) break;
                            issue_a(sl, of, am, d, s, kAStageBytes, pol_w, false);
                            mbar_arrive(&sc->gready[sl]);
                        }
                        sc->pok = ok;
                    }
                    __syncwarp();
                    ok = sc->pok;
                    __syncwarp();
                }
                if (!ok) break;
            } else {
                if (lane == 0) {
                    sc->ring[slot] = d;
                    mbar_arrive(&sc->ring_full[slot]);
                }
            }
            if (r == 0) break;
        }
        // drain: every armed stage's copies must land before the CTA exits
        if (lane == 0)
            for (int s = 0; s < kSlots; ++s)
                if (armed[s]) {
                    uint64_t t1 = globaltimer();
                    while (!mbar_try_wait(&sc->full[s], (armed[s] - 1) & 1) && globaltimer() - t1 < 200000000ull) {
                    }
                }
        __syncwarp();
    } else if (!skip && warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------ MMA issuer
            uint32_t nst = 0, g = 0, na = 0;
            StageAlloc alloc;
            bool issued_any = false;
            for (uint32_t it = 0;; ++it) {
                const uint32_t slot = it % kRing;
                if (!mbar_wait(&sc->ring_full[slot], (it / kRing) & 1, ctl, x.timeout_ns, 910)) break;
                TaskDesc d = sc->ring[slot];
                mbar_arrive(&sc->ring_empty[slot]);
                if (d.word == kExitWord) break;
                if (W::kStream && d.valid && d.stream && !d.attn) {  // stages consumed by the exec group: keep the sequence
                    for (int s = 0; s < d.nk; ++s, ++nst) alloc.next(d.sbytes);
                    continue;
                }
                if (W::kStream && d.valid && d.stream) {
                    // attention stages (k = the run's count of attention stages
                    // so far; buffer j = k & 1 of S, P and O): S_k = K Q^T into
                    // TMEM columns [16 j, +16) (keys x query heads), O_k =
                    // V^T P_k^T into columns [32 + 16 j, +16) (head dims x
                    // query heads) once the exec group has read S_k and written
                    // P_k (query heads x keys, bf16) to scratch + 4 KB * j.
                    // S_{k+1} is issued before waiting for P_k, and the exec
                    // group writes P_{k+1} while O_k runs; the stage is free
                    // after O_k.
                    const uint32_t buf = g & 1;
                    if (!mbar_wait(&sc->acc_empty[buf], ((g >> 1) & 1) ^ 1, ctl, x.timeout_ns, 913)) break;
                    tc_fence_after();
                    const uint32_t dT = sc->tmem_base + buf * kMaxN;
                    const uint32_t idesc = idesc_bf16_f32(128, 16);
                    const uint32_t pa = smem_u32(epi);
                    const uint32_t nst0 = nst, na0 = na;
                    auto issue_s = [&](int s, uint32_t off) -> bool {
                        const uint32_t gs = nst0 + (uint32_t)s, k = na0 + (uint32_t)s;
                        if (!mbar_wait(&sc->full[gs % kSlots], (gs / kSlots) & 1, ctl, x.timeout_ns, 914)) return false;
                        tc_fence_after();
                        const uint32_t ka = smem_u32(arena + off), qa = ka + kAttnQOff;
#pragma unroll
                        for (int at = 0; at < 2; ++at) {
                            const uint64_t ad = sdesc_k128(ka + at * kAAtomBytes);
                            const uint64_t bd = sdesc_k128(qa + at * 16u * 128u);
#pragma unroll
                            for (int kk = 0; kk < kAtomK / 16; ++kk)
                                tc_mma_bf16(dT + 16u * (k & 1), ad + 2 * kk, bd + 2 * kk, idesc, (at | kk) ? 1u : 0u);
                        }
                        tc_commit(&sc->s_full[k & 1]);
                        issued_any = true;
                        return true;
                    };
                    bool ok = true;
                    uint32_t off_cur = alloc.next(d.sbytes);
                    ok = issue_s(0, off_cur);
                    for (int s = 0; ok && s < d.nk; ++s) {
                        uint32_t off_next = 0;
                        if (s + 1 < d.nk) {
                            off_next = alloc.next(d.sbytes);
                            if (!(ok = issue_s(s + 1, off_next))) break;
                        }
                        const uint32_t k = na0 + (uint32_t)s, j = k & 1;
                        if (!mbar_wait(&sc->p_full[j], (k >> 1) & 1, ctl, x.timeout_ns, 915)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t va = smem_u32(arena + off_cur) + kAttnVOff;
#pragma unroll
                        for (int at = 0; at < 2; ++at) {
                            const uint64_t ad = sdesc_k128(va + at * kAAtomBytes);
                            const uint64_t bd = sdesc_k128(pa + 4096u * j + at * 16u * 128u);
#pragma unroll
                            for (int kk = 0; kk < kAtomK / 16; ++kk)
                                tc_mma_bf16(dT + 32u + 16u * j, ad + 2 * kk, bd + 2 * kk, idesc, (at | kk) ? 1u : 0u);
                        }
                        tc_commit(&sc->o_full[j]);
                        tc_commit(&sc->empty[(nst0 + (uint32_t)s) % kSlots]);
                        off_cur = off_next;
                    }
                    if (!ok) break;
                    nst += (uint32_t)d.nk;
                    na += (uint32_t)d.nk;
                    // one acc_full phase per use of an accumulator, attention
                    // tasks included: the epilogues' parity counts on it
                    tc_commit(&sc->acc_full[buf]);
                    ++g;
                    continue;
                }
                if (!(W::kGemm && d.valid && d.gemm)) continue;
                const uint32_t buf = g & 1;
                if (!mbar_wait(&sc->acc_empty[buf], ((g >> 1) & 1) ^ 1, ctl, x.timeout_ns, 911)) break;
                tc_fence_after();
                const uint32_t dt = sc->tmem_base + buf * kMaxN;
                const uint32_t idesc = idesc_bf16_f32(128, d.n);
                const uint32_t size = stage_bytes(d.n);
                bool ok = true;
                for (int s = 0; s < d.nk; ++s, ++nst) {
                    const uint32_t ss = nst % kSlots;
                    const uint32_t off = alloc.next(size);
                    if (!mbar_wait(&sc->full[ss], (nst / kSlots) & 1, ctl, x.timeout_ns, 912)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (W::kGather && d.gather) fence_proxy_async_smem();  // rows copied by cp.async (generic proxy) -> tensor core
                    const uint32_t a0 = smem_u32(arena + off);
#pragma unroll
                    for (int at = 0; at < 2; ++at) {
                        const uint64_t ad = sdesc_k128(a0 + at * kAAtomBytes);
                        const uint64_t bd = sdesc_k128(a0 + kAStageBytes + at * (uint32_t)d.n * 128u);
#pragma unroll
                        for (int kk = 0; kk < kAtomK / 16; ++kk)
                            tc_mma_bf16(dt, ad + 2 * kk, bd + 2 * kk, idesc, (s | at | kk) ? 1u : 0u);
                    }
                    tc_commit(&sc->empty[ss]);
                    issued_any = true;
                }
                if (!ok) break;
                tc_commit(&sc->acc_full[buf]);
                ++g;
            }
            if (issued_any) {  // every MMA must finish before TMEM is released
                tc_commit(&sc->drain);
                uint64_t t0 = globaltimer();
                while (!mbar_try_wait(&sc->drain, 0) && globaltimer() - t0 < 200000000ull) {
                }
            }
        }
        __syncwarp();
    } else if (!skip && W::kGather && warp == kGatherWarp) {
        // ------------------------------------------------------ row gather
        // Follows the task ring.  For each gathered task, the B rows of every
        // stage once warp 0 has reserved it and issued its weight tile
        // (gready; warp 0 cannot reuse a slot before this warp's arrival on
        // it, so one parity bit per slot tracks the phases): cp.async into
        // the 128-byte swizzled layout, a lane per row for tiles of up to 32
        // rows, else eight lanes per row; the last arrival completes the
        // stage's full phase.
        uint32_t gpar = 0;
        for (uint32_t it = 0;; ++it) {
            const uint32_t slot = it % kRing;
            int okw = 1;
            if (lane == 0) okw = mbar_wait(&sc->ring_full[slot], (it / kRing) & 1, ctl, x.timeout_ns, 930);
            okw = __shfl_sync(0xffffffffu, okw, 0);
            __syncwarp();  // lane 0's acquire orders the other lanes' reads of the entry
            if (!okw) break;
            const TaskDesc d = sc->ring[slot];
            __syncwarp();  // every lane has the entry before lane 0 frees it
            if (lane == 0) mbar_arrive(&sc->ring_empty[slot]);
            if (d.word == kExitWord) break;
            if (!(d.valid && d.gemm && d.gather)) continue;
            const uint16_t* rows[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) rows[i] = W::gather_row(p, d, lane + 32 * i);
            const uint32_t atom = (uint32_t)d.n * 128u;
            bool ok = true;
            for (int s = 0; s < d.nk; ++s) {
                const uint32_t sl = (d.st0 + (uint32_t)s) % kSlots;
                uint32_t of = 0;
                int okg = 1;
                if (lane == 0) {
                    okg = mbar_wait(&sc->gready[sl], (gpar >> sl) & 1u, ctl, x.timeout_ns, 931);
                    of = sc->r_off[sl];
                }
                if (!__shfl_sync(0xffffffffu, okg, 0)) {
                    ok = false;
                    break;
                }
                of = __shfl_sync(0xffffffffu, of, 0);
                gpar ^= 1u << sl;
                const int kx = d.k0 + s * kTileK;
                uint8_t* bdst = arena + of + kAStageBytes;
                if (d.n <= 32) {
                    if (rows[0]) {
                        const uint16_t* src = rows[0] + kx;
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            cp_async16(bdst + (c >> 3) * atom + lane * 128 + (((c & 7) ^ (lane & 7)) << 4), src + c * 8);
                    }
                } else {
                    gather_rows_wide(bdst, atom, d.n, kx, lane, rows);
                }
                cp_async_mbar_arrive(&sc->full[sl]);
                __syncwarp();
                if (lane == 0) mbar_arrive(&sc->full[sl]);
            }
            if (!ok) break;
        }
        cp_async_wait_all();  // every copy landed before the CTA exits
        __syncwarp();
    } else if (!skip && warp >= kExecWarp0 && warp < kExecWarp0 + kExecThreads / 32) {
        // ------------------------------------------------- epilogue / CUDA-core
        // Every decision that can end the loop is taken by exec thread 0 and
        // broadcast, so the four warps never split around a named barrier.
        uint32_t g = 0;
        for (uint32_t it = 0;; ++it) {
            const uint32_t slot = it % kRing;
            if (x.tid == 0) sc->bcast[4] = mbar_wait(&sc->ring_full[slot], (it / kRing) & 1, ctl, x.timeout_ns, 920);
            exec_bar();
            if (!sc->bcast[4]) break;
            TaskDesc d = sc->ring[slot];
            exec_bar();
            if (x.tid == 0) mbar_arrive(&sc->ring_empty[slot]);
            if (d.word == kExitWord) break;
            if (!d.valid) continue;
            if (x.debug & ET_DEBUG_DELAY) debug_delay(d.word ^ (ra.epoch * 977u));
            if (W::kStream && d.stream) {
                if (d.attn) {
                    const uint32_t buf = g & 1;
                    x.taddr = sc->tmem_base + buf * kMaxN + ((uint32_t)((warp & 3) * 32) << 16);
                    x.acc_empty = &sc->acc_empty[buf];
                    ++g;
                }
                if (!W::stream_exec(p, x, d)) break;
            } else if (W::kGemm && d.gemm) {
                const uint32_t buf = g & 1;
                const uint32_t par = (g >> 1) & 1;
                if (x.tid == 0) sc->bcast[5] = mbar_wait(&sc->acc_full[buf], par, ctl, x.timeout_ns, 921);
                exec_bar();
                if (!sc->bcast[5]) break;
                mbar_observe(&sc->acc_full[buf], par, ctl, 922);
                if (x.debug & ET_DEBUG_TRACE) d.t_acc = globaltimer();
                tc_fence_after();
                const uint32_t taddr = sc->tmem_base + buf * kMaxN + ((uint32_t)((warp & 3) * 32) << 16);
                if (!W::epilogue(p, x, d, taddr, &sc->acc_empty[buf])) break;
                ++g;
            } else {
                if (!W::simt(p, x, d)) break;
            }
            if (x.tid == 0) sc->bcast[6] = aborted(ctl);
            exec_bar();
            if (sc->bcast[6]) break;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1 && W::kGemm) {
        tc_fence_after();
        tmem_dealloc(sc->tmem_base, kTmemCols);
    }
    if (cta_times && threadIdx.x == 0)
        trace_task(ctl, ra.trace, ra.trace_cap, task_word(ET_OP_CTA, blockIdx.x, 0), 0, t_enter, t_setup, 0, 0,
                   globaltimer());
}

// Epilogue helper: read this warp's 32 lanes x 16 columns [c0, c0+16) of
// the accumulator into v (thread = lane).
__device__ __forceinline__ void acc_load16(uint32_t taddr, int c0, float (&v)[16]) {
    __syncwarp();  // tcgen05.ld is .sync.aligned: the warp must be converged
    tmem_ld16_wait(taddr + (uint32_t)c0, v);
}

// Release the accumulator after this warp's last tcgen05.ld.
__device__ __forceinline__ void acc_release(uint64_t* acc_empty) {
    tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(acc_empty);
}


}  // namespace et
