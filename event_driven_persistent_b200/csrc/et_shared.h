// Types shared by the host and device halves of libet (not part of the C ABI).
#pragma once
#include <stdint.h>

#include "../../include/et.h"

namespace et {

typedef et_trace_record TraceRec;

// Launch shape of every megakernel: warp 0 fetches tasks and drives TMA,
// warp 1 issues tcgen05 MMAs, warps 2..5 run epilogues and CUDA-core tasks;
// workloads with gathered B rows add warp 6, which copies those rows.
constexpr int kThreads = 192;
constexpr int kGatherWarp = 6;
constexpr int kThreadsGather = kThreads + 32;
constexpr int kExecThreads = 128;
constexpr int kExecWarp0 = 2;
constexpr int kRing = 2;           // task ring depth (warp 0 runs one task ahead)
constexpr int kTileK = 128;        // K elements per stage: two 128-byte swizzle atoms along K
constexpr int kAtomK = 64;         // K elements per swizzle atom (one 128-byte row)
// Pipeline stages live in a circular smem arena: a stage holds the weight
// tile (A, 16 KB) followed by the activation tile (B, N x 128 B rounded up to
// 1 KB), so tasks with few token rows keep more weight bytes in flight
// (11 stages at N = 16, 6 at N = 128).  kSlots mbarrier pairs track stages.
constexpr int kSlots = 12;

constexpr int kArenaBytes = 208 * 1024;
constexpr int kAAtomBytes = 128 * 128;   // weight tile of one atom: 128 rows x 128 B
constexpr int kAStageBytes = 2 * kAAtomBytes;
constexpr int kBStageBytes = 128 * 128;  // up to 128 rows x 128 B
constexpr int kMaxN = 128;         // largest MMA N (token rows per tile)
constexpr int kTmemCols = 256;     // two accumulators of kMaxN fp32 columns
constexpr int kScratchBytes = 16384;     // epilogue staging and CUDA-core task scratch
// Attention stream stages: K tile (128 keys x 128 dims), V^T tile (128 dims
// x 128 keys), Q tile (16 rows x 128 dims), each in the 128-byte swizzled
// K-major layout of a tensor-core operand.
constexpr uint32_t kAttnVOff = 32768, kAttnQOff = 65536, kAttnStage = 65536 + 4096;
constexpr int kEpiBytes = 64 * 33 * 4;   // gate/up exchange staging (start of the scratch)
constexpr int kCtlBytes = 2048;          // mbarriers, task ring, broadcast words
constexpr int kSmemBytes = 1024 /*align slack*/ + kArenaBytes + kScratchBytes + kCtlBytes;
// a workload with neither tensor-core nor stream tasks has no stage arena and
// asks only for its scratch and control block
constexpr int kSmemNoArenaBytes = 1024 + kScratchBytes + kCtlBytes;
static_assert(kSmemBytes <= 232448, "dynamic shared memory above the sm_100 per-block limit");

// Per-bucket static task lists: CSR over CTAs.  Hybrid schedules have a
// second list per CTA (part B), run after the ready queue is exhausted.
struct StaticLists {
    const int* off;    // [n_ctas + 1]
    const uint32_t* words;
    const int* off_b;  // [n_ctas + 1] or null
    const uint32_t* words_b;
};

// Device control block of a graph (lives in its workspace).
struct Ctl {
    int status;       // sticky error code (0 = ok), cleared by the host
    int abort;        // raised with status; every spin checks it
    int diag[8];      // where the first error happened
    unsigned ticket;  // trace ticket counter
    int n_trace;      // trace records written
    int* host_status; // device address of a mapped host word that mirrors status (or null)
    int pad[2];
};

// Per-run arguments common to every megakernel.
struct RunArgs {
    Ctl* ctl;
    int* ctr;                  // this run's counter set (zero at entry)
    int* ctr_next;             // the other set, zeroed during this run
    int n_ctr;
    unsigned long long* qslots;
    int qcap;
    uint32_t epoch;            // run number, >= 1
    int n_init;                // dynamic: initial tasks (implicit slots)
    int total_static;          // dynamic: task count when known at launch (else 0)
    int dynamic;               // 1 = ready queue (alone, or between the list parts when hybrid)
    int hybrid;                // 1 = list part A, then the queue, then list part B
    int fetch_batch;
    int debug;
    TraceRec* trace;
    int trace_cap;
    StaticLists lists;         // static / unfused: this size bucket's lists
    unsigned long long timeout_ns;
};

// Counter-set slots every workload reserves at the front.
constexpr int kCtrHead = 0, kCtrTail = 1, kCtrTotal = 2, kCtrFirstEvent = 4;

#ifdef __CUDACC__
#define ET_HD __host__ __device__ __forceinline__
#else
#define ET_HD inline
#endif

// Circular allocation of pipeline stages in the smem arena; the producer and
// the MMA issuer replay the same sequence, so both know every stage's
// address.  A stage that does not fit before the end of the arena starts
// again at offset 0.
struct StageAlloc {
    uint32_t head = 0;
    ET_HD uint32_t next(uint32_t size) {
        if (head + size > (uint32_t)kArenaBytes) head = 0;
        const uint32_t o = head;
        head += size;
        return o;
    }
};

// May the stage [off, off + size) be written while stages tail .. nst-1 are
// still in flight (stage u occupies [r_off[u % kSlots], r_end[u % kSlots]))?
// Not while its mbarrier slot is still held by stage nst - kSlots, nor while
// an in-flight stage shares a byte with it.  Consecutive stages are adjacent
// unless an allocation wrapped to offset 0, and a second wrap cannot happen
// while stages of the first are in flight (the wrapping stage would overlap
// them), so the stages in flight cover exactly [lo, hi) -- lo the oldest
// stage's start, hi the newest stage's end -- or, wrapped, [lo, arena end)
// and [0, hi).  O(1); the producer waits for the oldest stage (stages are
// consumed in order) while this is true.
ET_HD bool stage_blocked(uint32_t off, uint32_t size, uint32_t tail, uint32_t nst, const uint32_t* r_off,
                         const uint32_t* r_end) {
    if (tail == nst) return false;
    if (nst - tail >= (uint32_t)kSlots) return true;
    const uint32_t lo = r_off[tail % kSlots], hi = r_end[(nst - 1) % kSlots];
    if (lo < hi) return off < hi && lo < off + size;
    return off < hi || lo < off + size;
}

}  // namespace et
