// Host half of libet: the C ABI (include/et.h), the graph builder (static
// per-SM task lists per size bucket, workspace), tensor-map encoding and the
// launches.  No torch types cross this boundary.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <functional>
#include <queue>
#include <vector>

#include "et_params.h"

namespace et {
cudaError_t splitk_setup(int* max_blocks_per_sm);
cudaError_t launch_splitk(const SplitKParams& p, const RunArgs& ra, int n_ctas, cudaStream_t s);
cudaError_t launch_splitk_two(const float* A, int rows, int cols, int chunk, float* Bp, float* C, cudaStream_t s);
cudaError_t mlp_setup(int* max_blocks_per_sm);
cudaError_t launch_mlp(const MlpParams& p, const RunArgs& ra, int n_ctas, cudaStream_t s);
cudaError_t moe_setup(int* max_blocks_per_sm);
cudaError_t launch_moe(const MoeParams& p, const RunArgs& ra, int n_ctas, cudaStream_t s);
cudaError_t moe_mlp_setup(int* max_blocks_per_sm);
cudaError_t launch_moe_mlp(const MoeMlpParams& p, const RunArgs& ra, int n_ctas, cudaStream_t s);
cudaError_t decode_setup(int* max_blocks_per_sm);
cudaError_t launch_decode(const DecodeParams& p, const RunArgs& ra, int n_ctas, cudaStream_t s);
}  // namespace et

using namespace et;

namespace {

inline int cdiv(int a, int b) { return (a + b - 1) / b; }
inline int next_pow2(int v) {
    int b = 1;
    while (b < v) b <<= 1;
    return b;
}

// -------------------------------------------------------- tensor maps ----
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool load_encode() {
    if (g_encode) return true;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return false;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return true;
}

// bf16 [rows, cols] row-major, 128-byte swizzle, box = box_rows x 64 columns.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    if (!load_encode()) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

struct MapCache {
    const void* ptr = nullptr;
    uint64_t rows = 0, cols = 0;
    uint32_t box = 0;
    CUtensorMap map;
    bool get(CUtensorMap* out, const void* p, uint64_t r, uint64_t c, uint32_t b) {
        if (p != ptr || r != rows || c != cols || b != box) {
            if (!make_map(&map, p, r, c, b)) return false;
            ptr = p;
            rows = r;
            cols = c;
            box = b;
        }
        *out = map;
        return true;
    }
};

// ------------------------------------------------------- static lists ----
struct Slot {
    uint32_t word;
    float cost;
    int part = 0;  // hybrid schedules: 0 = list part A (before the queue), 1 = part B (after it)
};

inline uint32_t tw(int op, int a, int b) {
    return ((uint32_t)op << 26) | ((uint32_t)(a & 0xFFFF) << 10) | (uint32_t)(b & 0x3FF);
}

// Assign level-ordered slots to CTAs: each slot goes to the CTA with the
// least accumulated cost (ties -> lower CTA), so every CTA's list stays in
// level order (a task only waits on lower levels: no deadlock when all CTAs
// are resident).
void assign(const std::vector<Slot>& slots, int n_ctas, std::vector<int>& off, std::vector<uint32_t>& words) {
    std::vector<std::vector<uint32_t>> per(n_ctas);
    typedef std::pair<double, int> E;
    std::priority_queue<E, std::vector<E>, std::greater<E>> pq;
    for (int c = 0; c < n_ctas; ++c) pq.push(E(0.0, c));
    for (const Slot& s : slots) {
        E e = pq.top();
        pq.pop();
        per[e.second].push_back(s.word);
        pq.push(E(e.first + s.cost, e.second));
    }
    off.assign(n_ctas + 1, 0);
    words.clear();
    for (int c = 0; c < n_ctas; ++c) {
        off[c] = (int)words.size();
        words.insert(words.end(), per[c].begin(), per[c].end());
    }
    off[n_ctas] = (int)words.size();
}

}  // namespace

// ---------------------------------------------------------------- graph ----
struct et_graph {
    et_graph_desc d;
    et_graph_info info;
    int dev = 0, n_sm = 0, n_ctas = 0;
    Ctl* ctl = nullptr;
    int* host_status = nullptr;      // mapped host word the kernel mirrors its error status into
    int* host_status_dev = nullptr;  // its device address
    int* ctr[2] = {nullptr, nullptr};
    int n_ctr = 0;
    unsigned long long* qslots = nullptr;
    int qcap = 0;
    TraceRec* trace = nullptr;
    int trace_cap = 0;
    uint32_t epoch = 0;
    // static lists: one CSR per bucket (and list part), concatenated
    std::vector<int> bucket_T;
    std::vector<size_t> off_at, words_at, off_b_at, words_b_at;
    int* lists_off = nullptr;
    uint32_t* lists_words = nullptr;
    bool hybrid = false;  // the run uses list part A, the queue, then list part B
    std::vector<void*> allocs;
    // the last launched run (event-count introspection)
    int last_T = 0;
    SplitKParams last_sk;
    MlpParams last_mlp;
    MoeParams last_moe;
    DecodeParams last_dec;
    MlpParams last_moe_mlp;  // the MLP half of the last MoE -> MLP run
    // workload state
    SplitKParams sk;
    MlpParams mlp;
    MoeParams moe;
    DecodeParams dec;
    MapCache mc[6];
    int bucket_of(int T) const {
        for (size_t i = 0; i < bucket_T.size(); ++i)
            if (bucket_T[i] >= T) return (int)i;
        return (int)bucket_T.size() - 1;
    }
};

namespace {

et_status cuda_fail(cudaError_t e) {
    if (e == cudaErrorMemoryAllocation) return ET_ERR_OOM;
    return ET_ERR_CUDA;
}

#define ET_CU(call)                                   \
    do {                                              \
        cudaError_t e_ = (call);                      \
        if (e_ != cudaSuccess) return cuda_fail(e_);  \
    } while (0)

template <class T>
et_status galloc(et_graph* g, T** p, size_t n) {
    void* q = nullptr;
    if (n == 0) n = 1;
    cudaError_t e = cudaMalloc(&q, n * sizeof(T));
    if (e != cudaSuccess) return cuda_fail(e);
    g->allocs.push_back(q);
    e = cudaMemset(q, 0, n * sizeof(T));
    if (e != cudaSuccess) return cuda_fail(e);
    *p = static_cast<T*>(q);
    return ET_OK;
}

#define ET_TRY(x)                      \
    do {                               \
        et_status s_ = (x);            \
        if (s_ != ET_OK) return s_;    \
    } while (0)

bool aligned16(const void* p) { return p && ((uintptr_t)p & 15) == 0; }

// Build every bucket's lists with `gen(T_b, slots)`, upload them.  Hybrid
// graphs keep a slot's part (A before the queue, B after it) as two lists
// per CTA; the other schedules list every slot in one list, in order.
et_status build_lists(et_graph* g, const std::function<void(int, std::vector<Slot>&)>& gen) {
    std::vector<int> all_off;
    std::vector<uint32_t> all_words;
    for (int T = 1;; T <<= 1) {
        int Tb = std::min(T, g->d.max_T);
        std::vector<Slot> slots, part_a, part_b;
        gen(Tb, slots);
        for (const Slot& sl : slots) (g->hybrid && sl.part == 1 ? part_b : part_a).push_back(sl);
        g->bucket_T.push_back(Tb);
        for (int part = 0; part < 2; ++part) {
            std::vector<int> off;
            std::vector<uint32_t> words;
            assign(part == 0 ? part_a : part_b, g->n_ctas, off, words);
            (part == 0 ? g->off_at : g->off_b_at).push_back(all_off.size());
            (part == 0 ? g->words_at : g->words_b_at).push_back(all_words.size());
            for (int o : off) all_off.push_back(o);
            all_words.insert(all_words.end(), words.begin(), words.end());
        }
        if (Tb >= g->d.max_T) break;
    }
    ET_TRY(galloc(g, &g->lists_off, all_off.size()));
    ET_TRY(galloc(g, &g->lists_words, all_words.size()));
    ET_CU(cudaMemcpy(g->lists_off, all_off.data(), all_off.size() * sizeof(int), cudaMemcpyHostToDevice));
    ET_CU(cudaMemcpy(g->lists_words, all_words.data(), all_words.size() * sizeof(uint32_t), cudaMemcpyHostToDevice));
    return ET_OK;
}

// Arguments of the graph's next run.  The run number (epoch) selects the
// counter set and tags the queue slots; it is committed by commit_run only
// once the launch succeeded, so a launch that failed leaves the counter sets
// as they were (the set the next run uses is still the zeroed one).
RunArgs run_args(et_graph* g, int T, int n_init, int total_static) {
    RunArgs ra;
    memset(&ra, 0, sizeof(ra));
    const uint32_t ep = g->epoch + 1;
    ra.ctl = g->ctl;
    ra.ctr = g->ctr[ep & 1];
    ra.ctr_next = g->ctr[(ep + 1) & 1];
    ra.n_ctr = g->n_ctr;
    ra.qslots = g->qslots;
    ra.qcap = g->qcap;
    ra.epoch = ep;
    ra.n_init = n_init;
    ra.total_static = total_static;
    ra.dynamic = g->d.sched == ET_SCHED_DYNAMIC || g->hybrid;
    ra.hybrid = g->hybrid;
    ra.fetch_batch = g->d.fetch_batch;
    ra.debug = g->d.debug_flags;
    ra.trace = g->trace;
    ra.trace_cap = g->trace_cap;
    int b = g->bucket_of(T);
    ra.lists.off = g->lists_off + g->off_at[b];
    ra.lists.words = g->lists_words + g->words_at[b];
    if (g->hybrid) {
        ra.lists.off_b = g->lists_off + g->off_b_at[b];
        ra.lists.words_b = g->lists_words + g->words_b_at[b];
    }
    ra.timeout_ns = (unsigned long long)((double)g->d.timeout_ms * 1e6);
    return ra;
}

et_status launched(et_graph* g, cudaError_t e) {
    if (e != cudaSuccess) return cuda_fail(e);
    ++g->epoch;
    return ET_OK;
}

// A device error of an earlier run that the host can already see (the
// failing kernel mirrored it into mapped host memory) and that
// et_sync_status has not collected yet.
bool pending(const et_graph* g) { return *reinterpret_cast<volatile const int*>(g->host_status) != 0; }

// Upload a clean control block (status 0, the host mirror's device address).
et_status reset_ctl(et_graph* g) {
    Ctl h;
    memset(&h, 0, sizeof(h));
    h.host_status = g->host_status_dev;
    ET_CU(cudaMemcpy(g->ctl, &h, sizeof(Ctl), cudaMemcpyHostToDevice));
    *reinterpret_cast<volatile int*>(g->host_status) = 0;
    return ET_OK;
}

et_status pre_run(et_graph* g, cudaStream_t s) {
    if (pending(g)) return ET_ERR_PENDING;
    if (g->d.debug_flags & ET_DEBUG_TRACE) {
        // the trace of one run: clear the record counter and tickets
        ET_CU(cudaMemsetAsync(&g->ctl->ticket, 0, 2 * sizeof(int), s));
    }
    return ET_OK;
}

// ------------------------------------------------------------- split-K ----
et_status build_splitk(et_graph* g) {
    et_graph_desc& d = g->d;
    if (d.splitk_cols <= 0) d.splitk_cols = 128;
    if (d.splitk_chunk <= 0) d.splitk_chunk = 32;
    if (d.splitk_tile_rows <= 0) d.splitk_tile_rows = 32;
    if (d.fetch_batch <= 0) d.fetch_batch = 1;
    const int nt_max = cdiv(d.max_T, d.splitk_tile_rows);
    const int nch = cdiv(d.splitk_cols, d.splitk_chunk);
    if (nt_max > 0xFFFF || nch > 0x3FF) return ET_ERR_UNSUPPORTED;
    SplitKParams& p = g->sk;
    memset(&p, 0, sizeof(p));
    p.cols = d.splitk_cols;
    p.chunk = d.splitk_chunk;
    p.tile_rows = d.splitk_tile_rows;
    p.n_chunks = nch;
    p.ev_base = kCtrFirstEvent;
    p.ev_all = kCtrFirstEvent + nt_max;
    p.unfused = d.sched == ET_SCHED_UNFUSED;
    p.bad_count = (d.debug_flags & ET_DEBUG_BAD_COUNT) ? 1 : 0;
    g->n_ctr = p.ev_all + 1;
    g->qcap = nt_max * nch + nt_max + g->n_ctas * d.fetch_batch + 64;
    int mb = 0;
    ET_CU(splitk_setup(&mb));
    if (mb < 1) return ET_ERR_UNSUPPORTED;
    return build_lists(g, [&](int Tb, std::vector<Slot>& s) {
        int nt = cdiv(Tb, d.splitk_tile_rows);
        for (int i = 0; i < nt; ++i)
            for (int j = 0; j < nch; ++j) s.push_back({tw(ET_OP_SK_PARTIAL, i, j), 1.0f});
        if (!g->hybrid)  // hybrid: a final task is queued by the partial that completes its event
            for (int i = 0; i < nt; ++i) s.push_back({tw(ET_OP_SK_FINAL, i, 0), 0.5f});
    });
}

// ----------------------------------------------------------------- MLP ----
// MLP part of a graph: dims, events from ev0 (*ev_end = the next free
// one), workspace; the slots of its static lists (with or without the norm
// tasks; `part` = hybrid list part).
et_status setup_mlp(et_graph* g, MlpParams& p, int hidden, int inter, int maxB, float eps, int ev0, int* ev_end) {
    if (maxB > kMaxN) return ET_ERR_UNSUPPORTED;  // one token tile
    if (hidden % 128 || inter % 128) return ET_ERR_UNSUPPORTED;
    memset(&p, 0, sizeof(p));
    p.hidden = hidden;
    p.inter = inter;
    p.maxB = maxB;
    p.eps = eps;
    p.gu_tile = 64;
    p.down_tile = 128;
    p.kchunk = inter % 1024 == 0 ? 1024 : (inter % 256 == 0 ? 256 : 128);
    p.n_gu = inter / p.gu_tile;
    p.n_m = hidden / p.down_tile;
    p.n_c = inter / p.kchunk;
    p.gu_per_chunk = p.kchunk / p.gu_tile;
    if (p.n_gu > 0xFFFF || p.n_c > 0x3FF) return ET_ERR_UNSUPPORTED;
    p.ev_norm = ev0;
    p.ev_h = p.ev_norm + 1;
    p.ev_y = p.ev_h + p.n_c;
    p.ev_gu_all = p.ev_y + p.n_m;
    p.ev_down_all = p.ev_gu_all + 1;
    *ev_end = p.ev_down_all + 1;
    p.unfused = g->d.sched == ET_SCHED_UNFUSED;
    p.push = g->d.sched == ET_SCHED_DYNAMIC;
    p.bad_count = (g->d.debug_flags & ET_DEBUG_BAD_COUNT) ? 1 : 0;
    const size_t rows = (size_t)std::max(maxB, 16);  // at least one 16-row TMA box
    ET_TRY(galloc(g, &p.xn, rows * p.hidden));
    ET_TRY(galloc(g, &p.h, rows * p.inter));
    ET_TRY(galloc(g, &p.yacc, (size_t)p.maxB * p.hidden));
    if (!make_map(&p.tm_xn, p.xn, rows, p.hidden, 16)) return ET_ERR_CUDA;
    if (!make_map(&p.tm_h, p.h, rows, p.inter, 16)) return ET_ERR_CUDA;
    p.wide_b = rows >= 64;
    if (p.wide_b && (!make_map(&p.tm_xn64, p.xn, rows, p.hidden, 64) || !make_map(&p.tm_h64, p.h, rows, p.inter, 64)))
        return ET_ERR_CUDA;
    return ET_OK;
}
int mlp_queue_tasks(const MlpParams& p) { return p.maxB + p.n_gu + p.n_m * p.n_c + p.n_m; }
void mlp_slots(const MlpParams& p, int Tb, std::vector<Slot>& s, bool with_norm, int part) {
    // cost ~ bytes streamed per task (KB)
    const float c_gu = 2.f * p.gu_tile * p.hidden * 2 / 1024.f, c_dn = (float)p.down_tile * p.kchunk * 2 / 1024.f;
    if (with_norm)
        for (int b = 0; b < Tb; ++b) s.push_back({tw(ET_OP_MLP_NORM, b, 0), 1.f, part});
    for (int n = 0; n < p.n_gu; ++n) s.push_back({tw(ET_OP_MLP_GATEUP, n, 0), c_gu, part});
    for (int c = 0; c < p.n_c; ++c)
        for (int m = 0; m < p.n_m; ++m) s.push_back({tw(ET_OP_MLP_DOWN, m, c), c_dn, part});
    for (int m = 0; m < p.n_m; ++m) s.push_back({tw(ET_OP_MLP_REDUCE, m, 0), 2.f, part});
}

et_status build_mlp(et_graph* g) {
    et_graph_desc& d = g->d;
    if (d.hidden <= 0) d.hidden = 4096;
    if (d.inter <= 0) d.inter = 14336;
    if (d.rms_eps <= 0.f) d.rms_eps = 1e-5f;
    if (d.fetch_batch <= 0) d.fetch_batch = 1;
    MlpParams& p = g->mlp;
    int ev_end = 0;
    ET_TRY(setup_mlp(g, p, d.hidden, d.inter, d.max_T, d.rms_eps, kCtrFirstEvent, &ev_end));
    g->n_ctr = ev_end;
    g->qcap = mlp_queue_tasks(p) + g->n_ctas * d.fetch_batch + 64;
    int mb = 0;
    ET_CU(mlp_setup(&mb));
    if (mb < 1) return ET_ERR_UNSUPPORTED;
    return build_lists(g, [&](int Tb, std::vector<Slot>& s) { mlp_slots(p, Tb, s, true, 0); });
}

// ----------------------------------------------------------------- MoE ----
struct MoeShape {
    int n_tt, n_tk, n_kc, cb, n_cb, f_max;
};

// Tokens per combine task: one while the layer is small (the combine is the
// layer's tail, so it is spread over as many SMs as there are tokens), eight
// beyond 256 tokens (fewer, larger tasks once there are more tokens than SMs).
constexpr int kCbOneMaxT = 256;
inline int moe_cb_for(int T) { return T <= kCbOneMaxT ? 1 : 8; }

MoeShape moe_shape(const et_graph* g, const MoeParams& p, int T) {
    MoeShape m;
    m.n_tt = cdiv(T, p.tt);
    m.n_tk = cdiv(T, p.tkt);
    // router K split: up to 8 chunks while the (token block, chunk) tasks fit
    // in a quarter of the SMs, so that a small batch streams Wr on many SMs
    int kc = 1;
    while (kc < 8 && m.n_tk * kc * 2 * 4 <= g->n_ctas && (p.hidden / (kc * 2)) % kTileK == 0) kc *= 2;
    m.n_kc = kc;
    m.cb = moe_cb_for(T);
    m.n_cb = cdiv(T, m.cb);
    const int pairs = p.k * T;
    m.f_max = std::min(pairs, std::min(p.E, pairs) + cdiv(pairs, p.bm));
    return m;
}

// MoE part of a graph: dims, events from ev0 (*ev_end = the next free
// one), queue slots it may need (*qtasks), workspace; and its list slots.
// Default of et_graph_desc.moe_xp_min_T: never.  Staged rows paid off while
// the producer warp gathered stage-1 rows itself (T = 4096: 1294 -> 1198 us);
// with the gather warp, gathering is faster at every T (T = 2048: 728 -> 592
// us, T = 4096: 1190 -> 987 us without them).
constexpr int kMoeXpMinT = -1;

et_status setup_moe(et_graph* g, int ev0, int* ev_end, int* qtasks) {
    et_graph_desc& d = g->d;
    if (d.hidden <= 0) d.hidden = 2048;
    if (d.inter <= 0) d.inter = 768;
    if (d.n_experts <= 0) d.n_experts = 128;
    if (d.top_k <= 0) d.top_k = 8;
    if (d.fetch_batch <= 0) d.fetch_batch = 1;
    if (d.n_experts > 128 || d.n_experts % 8 || d.top_k > 8 || d.top_k > d.n_experts) return ET_ERR_UNSUPPORTED;
    if (d.hidden % 128 || d.inter % 128) return ET_ERR_UNSUPPORTED;
    MoeParams& p = g->moe;
    memset(&p, 0, sizeof(p));
    p.hidden = d.hidden;
    p.inter = d.inter;
    p.E = d.n_experts;
    p.k = d.top_k;
    p.maxT = d.max_T;
    p.tt = 128;
    p.tkt = 16;
    p.bm = 128;
    p.n1_tile = 64;
    p.n_n1 = p.inter / p.n1_tile;
    p.n2_tile = 128;
    p.n_n2 = p.hidden / p.n2_tile;
    p.cb = moe_cb_for(d.max_T);
    p.sched = d.sched;
    p.early_max = 2 * g->n_ctas;
    p.bad_count = (d.debug_flags & ET_DEBUG_BAD_COUNT) ? 1 : 0;
    const MoeShape mx = moe_shape(g, p, d.max_T);
    if (mx.f_max > 0xFFFF || mx.n_tt > 0xFFFF || p.n_n1 > 0x3FF || p.n_n2 > 0x3FF) return ET_ERR_UNSUPPORTED;
    int ev = ev0;
    p.ev_tk = ev++;
    p.ev_rt = ev;
    ev += mx.n_tk;
    p.ev_sc = ev++;
    p.ev_grp = ev++;
    p.ev_s1_all = ev++;
    p.ev_s2_all = ev++;
    p.ev_exp = ev;
    ev += p.E;
    p.ev_s1 = ev;
    ev += mx.f_max;
    p.ev_cb = ev;
    const int n_cb_max = std::max(mx.n_cb, std::min(d.max_T, kCbOneMaxT));  // over every size bucket
    ev += n_cb_max;
    p.ev_gcnt = ev;
    ev += mx.n_tt * p.E;
    *ev_end = ev;
    *qtasks = mx.n_tk * 8 + mx.n_tt + 1 + mx.f_max * (p.n_n1 + p.n_n2) + n_cb_max;
    const size_t pairs = (size_t)p.maxT * p.k;
    ET_TRY(galloc(g, &p.lacc, (size_t)p.maxT * p.E));
    ET_TRY(galloc(g, &p.topk, pairs));
    ET_TRY(galloc(g, &p.topw, pairs));
    ET_TRY(galloc(g, &p.goff, (size_t)mx.n_tt * p.E));
    ET_TRY(galloc(g, &p.counts, (size_t)p.E));
    ET_TRY(galloc(g, &p.indptr, (size_t)p.E + 1));
    ET_TRY(galloc(g, &p.tindptr, (size_t)p.E + 1));
    ET_TRY(galloc(g, &p.mt_desc, (size_t)mx.f_max));
    ET_TRY(galloc(g, &p.perm, pairs));
    ET_TRY(galloc(g, &p.pos, pairs));
    ET_TRY(galloc(g, &p.scal, 8));
    ET_TRY(galloc(g, &p.Hm, pairs * p.inter));
    ET_TRY(galloc(g, &p.Yacc, (size_t)p.maxT * p.hidden));
    if (!make_map(&p.tm_hm, p.Hm, pairs, p.inter, 16)) return ET_ERR_CUDA;
    if (!make_map(&p.tm_hm64, p.Hm, pairs, p.inter, 64)) return ET_ERR_CUDA;
    if (d.moe_xp_min_T == 0) d.moe_xp_min_T = kMoeXpMinT;
    p.Xp = nullptr;
    if (d.moe_xp_min_T > 0 && p.maxT > p.tt && p.maxT >= d.moe_xp_min_T && p.hidden <= 2048) {  // row copy: <= 8 x 16 B per lane
        ET_TRY(galloc(g, &p.Xp, pairs * p.hidden));
        if (!make_map(&p.tm_xp, p.Xp, pairs, p.hidden, 16)) return ET_ERR_CUDA;
    }
    return ET_OK;
}
void moe_slots(et_graph* g, const MoeParams& p, int Tb, std::vector<Slot>& s) {
    const float c_s1 = 2.f * p.n1_tile * p.hidden * 2 / 1024.f, c_s2 = (float)p.n2_tile * p.inter * 2 / 1024.f;
    MoeShape m = moe_shape(g, p, Tb);
    const float c_rt = (float)p.E * p.hidden * 2 / m.n_kc / 1024.f;
    for (int j = 0; j < m.n_tk; ++j)
        for (int c = 0; c < m.n_kc; ++c) s.push_back({tw(ET_OP_MOE_ROUTER, j, c), c_rt});
    if (g->hybrid) return;  // grouping, expert stages and combine go through the queue
    s.push_back({tw(ET_OP_MOE_SCAN, 0, 0), 8.f});
    if (m.n_tt > 1)
        for (int t = 0; t < m.n_tt; ++t) s.push_back({tw(ET_OP_MOE_GROUP, t, 0), 8.f});
    for (int f = 0; f < m.f_max; ++f)
        for (int n = 0; n < p.n_n1; ++n) s.push_back({tw(ET_OP_MOE_S1, f, n), c_s1});
    for (int f = 0; f < m.f_max; ++f)
        for (int n = 0; n < p.n_n2; ++n) s.push_back({tw(ET_OP_MOE_S2, f, n), c_s2});
    for (int b = 0; b < m.n_cb; ++b) s.push_back({tw(ET_OP_MOE_COMBINE, b, 0), 2.f});
}

void moe_defaults(et_graph_desc& d) {
    if (d.hidden <= 0) d.hidden = 2048;
    if (d.inter <= 0) d.inter = 768;
    if (d.n_experts <= 0) d.n_experts = 128;
    if (d.top_k <= 0) d.top_k = 8;
    if (d.fetch_batch <= 0) d.fetch_batch = 1;
}

et_status build_moe(et_graph* g) {
    moe_defaults(g->d);
    int ev_end = 0, qt = 0;
    ET_TRY(setup_moe(g, kCtrFirstEvent, &ev_end, &qt));
    g->n_ctr = ev_end;
    g->qcap = qt + g->n_ctas * g->d.fetch_batch + 64;
    int mb = 0;
    ET_CU(moe_setup(&mb));
    if (mb < 1) return ET_ERR_UNSUPPORTED;
    return build_lists(g, [&](int Tb, std::vector<Slot>& s) { moe_slots(g, g->moe, Tb, s); });
}

// The MoE layer followed by a dense SwiGLU MLP (hidden -> mlp_inter ->
// hidden) on its output, one launch; T <= 128 (the MLP's one token tile).
et_status build_moe_mlp(et_graph* g) {
    et_graph_desc& d = g->d;
    moe_defaults(d);
    if (d.mlp_inter <= 0) d.mlp_inter = 6144;
    if (d.rms_eps <= 0.f) d.rms_eps = 1e-5f;
    if (d.max_T > kMaxN) return ET_ERR_UNSUPPORTED;
    int ev1 = 0, qt = 0, ev2 = 0;
    ET_TRY(setup_moe(g, kCtrFirstEvent, &ev1, &qt));
    ET_TRY(setup_mlp(g, g->mlp, d.hidden, d.mlp_inter, d.max_T, d.rms_eps, ev1, &ev2));
    MoeParams& p = g->moe;
    const MlpParams& m = g->mlp;
    p.mlp_xn = m.xn;
    p.mlp_eps = d.rms_eps;
    p.mlp_ev_norm = m.ev_norm;
    p.mlp_n_gu = m.push ? m.n_gu : 0;
    p.extra_tasks = m.push ? m.n_gu + m.n_m * m.n_c + m.n_m : 0;
    g->n_ctr = ev2;
    g->qcap = qt + mlp_queue_tasks(m) + g->n_ctas * d.fetch_batch + 64;
    int mb = 0;
    ET_CU(moe_mlp_setup(&mb));
    if (mb < 1) return ET_ERR_UNSUPPORTED;
    return build_lists(g, [&](int Tb, std::vector<Slot>& s) {
        moe_slots(g, g->moe, Tb, s);
        if (!(g->d.sched == ET_SCHED_DYNAMIC)) mlp_slots(g->mlp, Tb, s, false, 1);  // after the queue when hybrid
    });
}

// --------------------------------------------------------- decode layer ----
constexpr int kDecSplit = 512;  // keys per attention split task (four 128-key stages)

// Keys per attention split task for a run of B requests.  Queued splits
// (dynamic and hybrid schedules) get longer as B grows: with enough splits
// to fill the SMs, each split's start (its first stage's load, the hand-off
// to the next task) is paid fewer times — measured on the Llama-3-8B-shaped
// layer: B = 1 best at 512 keys, B = 16 at 1024, B = 64 at 2048 (-12 %).
// Static lists keep the graph's split (their balance assumes it).
int dec_split_for(const et_graph* g, int B) {
    const int base = kDecSplit;  // the graph's split (its partials and lists are sized for it)
    if (g->d.sched != ET_SCHED_DYNAMIC && !g->hybrid) return base;
    return B < 8 ? base : (B < 32 ? 2 * base : 4 * base);
}

et_status build_decode(et_graph* g) {
    et_graph_desc& d = g->d;
    if (d.hidden <= 0) d.hidden = 4096;
    if (d.inter <= 0) d.inter = 14336;
    if (d.n_heads <= 0) d.n_heads = 32;
    if (d.n_kv_heads <= 0) d.n_kv_heads = 8;
    if (d.head_dim <= 0) d.head_dim = 128;
    if (d.max_ctx <= 0) d.max_ctx = 4104;
    if (d.rope_base <= 0.f) d.rope_base = 500000.f;
    if (d.rms_eps <= 0.f) d.rms_eps = 1e-5f;
    if (d.fetch_batch <= 0) d.fetch_batch = 1;
    if (d.max_T > kMaxN) return ET_ERR_UNSUPPORTED;  // one token tile
    if (d.head_dim != 128 || d.n_heads % d.n_kv_heads || d.n_heads / d.n_kv_heads > 4) return ET_ERR_UNSUPPORTED;
    if (d.max_ctx % 8) return ET_ERR_INVALID;  // V^T cache rows are read by TMA: 16-byte multiples
    if (d.hidden % 1024 || d.hidden > 4096 || d.inter % 128) return ET_ERR_UNSUPPORTED;
    DecodeParams& p = g->dec;
    memset(&p, 0, sizeof(p));
    p.maxB = d.max_T;
    p.hidden = d.hidden;
    p.inter = d.inter;
    p.nq = d.n_heads;
    p.nkv = d.n_kv_heads;
    p.hd = d.head_dim;
    p.grp = p.nq / p.nkv;
    p.max_ctx = d.max_ctx;
    p.split = kDecSplit;
    p.s_max = cdiv(d.max_ctx, kDecSplit);
    p.eps = d.rms_eps;
    p.rope_base = (double)d.rope_base;
    p.n_heads = p.nq + 2 * p.nkv;
    const int kt = p.hidden / kTileK;
    // QKV K chunks: as many as keep every (head tile, chunk) task in one wave
    // over the CTAs (chunks of kt / n_kc stages, rounded: 10 or 11 of the 32
    // stages for 48 head tiles on 148 SMs), so no CTA streams two tasks
    p.n_kc = std::max(1, std::min(kt, g->n_ctas / p.n_heads));
    p.o_kc = p.grp * p.hd;
    p.gu_tile = 64;
    p.kchunk = d.inter % 1024 == 0 ? 1024 : (d.inter % 256 == 0 ? 256 : 128);
    p.n_gu = d.inter / p.gu_tile;
    p.n_m = d.hidden / 128;
    p.n_c = d.inter / p.kchunk;
    p.gu_per_chunk = p.kchunk / p.gu_tile;
    p.sched = d.sched;
    p.bad_count = (d.debug_flags & ET_DEBUG_BAD_COUNT) ? 1 : 0;
    const int nq_rows = p.maxB * p.nkv;
    if (nq_rows > 0xFFFF || p.s_max > 0x3FF || p.n_heads > 0xFFFF || p.n_c > 0x3FF || p.nkv > 0x3FF)
        return ET_ERR_UNSUPPORTED;
    if (p.s_max * p.grp > 1024) return ET_ERR_UNSUPPORTED;  // the merge keeps every split's (max, sum) in smem
    int ev = kCtrFirstEvent;
    p.ev_n1 = ev++;
    p.ev_qkv = ev;
    ev += p.n_heads;
    p.ev_g = ev;
    ev += p.nkv;
    p.ev_att = ev;
    ev += p.maxB * p.nkv;
    p.ev_ag = ev;
    ev += p.nkv;
    p.ev_o = ev++;
    p.ev_n2 = ev++;
    p.ev_h = ev;
    ev += p.n_c;
    p.ev_y = ev;
    ev += p.n_m;
    p.ev_branch_all = ev++;
    p.ev_merge_all = ev++;
    p.ev_gu_all = ev++;
    p.ev_down_all = ev++;
    g->n_ctr = ev;
    g->qcap = p.n_heads * p.n_kc + p.nkv * p.maxB * p.s_max + p.n_m * p.nkv + p.maxB + p.n_gu + p.n_m * p.n_c +
              p.n_m + g->n_ctas * d.fetch_batch + 64;
    const size_t rows = (size_t)std::max(p.maxB, 16);  // at least one 16-row TMA box
    ET_TRY(galloc(g, &p.xn, rows * p.hidden));
    ET_TRY(galloc(g, &p.qkvacc, (size_t)p.maxB * p.n_heads * p.hd));
    ET_TRY(galloc(g, &p.q, (size_t)p.maxB * p.nq * p.hd));
    ET_TRY(galloc(g, &p.rope, (size_t)p.maxB * (p.hd / 2)));
    ET_TRY(galloc(g, &p.part, (size_t)p.maxB * p.nkv * p.s_max * p.grp * (p.hd + 2)));
    ET_TRY(galloc(g, &p.attn, rows * p.nq * p.hd));
    ET_TRY(galloc(g, &p.h1acc, (size_t)p.maxB * p.hidden));
    ET_TRY(galloc(g, &p.h1, (size_t)p.maxB * p.hidden));
    ET_TRY(galloc(g, &p.xn2, rows * p.hidden));
    ET_TRY(galloc(g, &p.hm, rows * p.inter));
    ET_TRY(galloc(g, &p.yacc, (size_t)p.maxB * p.hidden));
    if (!make_map(&p.tm_xn, p.xn, rows, p.hidden, 16)) return ET_ERR_CUDA;
    if (!make_map(&p.tm_attn, p.attn, rows, (uint64_t)p.nq * p.hd, 16)) return ET_ERR_CUDA;
    if (!make_map(&p.tm_xn2, p.xn2, rows, p.hidden, 16)) return ET_ERR_CUDA;
    if (!make_map(&p.tm_hm, p.hm, rows, p.inter, 16)) return ET_ERR_CUDA;
    if (!make_map(&p.tm_q, p.q, (uint64_t)p.maxB * p.nq, p.hd, 16)) return ET_ERR_CUDA;
    p.wide_b = rows >= 64;
    if (p.wide_b && (!make_map(&p.tm_xn64, p.xn, rows, p.hidden, 64) ||
                     !make_map(&p.tm_attn64, p.attn, rows, (uint64_t)p.nq * p.hd, 64) ||
                     !make_map(&p.tm_xn2_64, p.xn2, rows, p.hidden, 64) || !make_map(&p.tm_hm64, p.hm, rows, p.inter, 64)))
        return ET_ERR_CUDA;
    int mb = 0;
    ET_CU(decode_setup(&mb));
    if (mb < 1) return ET_ERR_UNSUPPORTED;
    // cost ~ KB a task streams
    const float c_qkv = 128.f * p.hidden / p.n_kc * 2 / 1024.f, c_att = 2.f * kDecSplit * 256 / 1024.f,
                c_o = 128.f * p.o_kc * 2 / 1024.f, c_gu = 2.f * p.gu_tile * p.hidden * 2 / 1024.f,
                c_dn = 128.f * p.kchunk * 2 / 1024.f;
    return build_lists(g, [&](int Tb, std::vector<Slot>& s) {
        for (int b = 0; b < Tb; ++b) s.push_back({tw(ET_OP_DEC_NORM1, b, 0), 1.f, 0});
        for (int n = 0; n < p.n_heads; ++n)
            for (int c = 0; c < p.n_kc; ++c) s.push_back({tw(ET_OP_DEC_QKV, n, c), c_qkv, 0});
        if (!g->hybrid)  // hybrid: the splits are queued once their group's branches are done
            for (int s2 = 0; s2 < p.s_max; ++s2)
                for (int b = 0; b < Tb; ++b)
                    for (int gg = 0; gg < p.nkv; ++gg) s.push_back({tw(ET_OP_DEC_ATTN, b * p.nkv + gg, s2), c_att, 0});
        for (int c = 0; c < p.nkv; ++c)
            for (int m = 0; m < p.n_m; ++m) s.push_back({tw(ET_OP_DEC_OPROJ, m, c), c_o, 1});
        for (int b = 0; b < Tb; ++b) s.push_back({tw(ET_OP_DEC_NORM2, b, 0), 1.f, 1});
        for (int n = 0; n < p.n_gu; ++n) s.push_back({tw(ET_OP_DEC_GATEUP, n, 0), c_gu, 1});
        for (int c = 0; c < p.n_c; ++c)
            for (int m = 0; m < p.n_m; ++m) s.push_back({tw(ET_OP_DEC_DOWN, m, c), c_dn, 1});
        for (int m = 0; m < p.n_m; ++m) s.push_back({tw(ET_OP_DEC_RED, m, 0), 2.f, 1});
    });
}

}  // namespace

// ===================================================================== ABI
extern "C" {

const char* et_status_str(et_status s) {
    switch (s) {
        case ET_OK: return "ok";
        case ET_ERR_INVALID: return "invalid argument";
        case ET_ERR_CUDA: return "CUDA error";
        case ET_ERR_TIMEOUT: return "device wait timed out";
        case ET_ERR_OOM: return "out of device memory";
        case ET_ERR_UNSUPPORTED: return "unsupported device or dims";
        case ET_ERR_PENDING: return "an earlier run failed and its error was not collected";
        case ET_ERR_INTERNAL: return "device-side capacity check failed";
    }
    return "unknown status";
}



et_status et_build_graph(const et_graph_desc* desc, et_graph** out) {
    if (!desc || !out) return ET_ERR_INVALID;
    *out = nullptr;
    if (desc->max_T < 1 || desc->kind < 0 || desc->kind > 4 || desc->sched < 0 || desc->sched > 3)
        return ET_ERR_INVALID;
    et_graph* g = new et_graph();
    g->d = *desc;
    if (g->d.timeout_ms <= 0) g->d.timeout_ms = 1000.f;
    auto fail = [&](et_status s) {
        et_destroy_graph(g);
        return s;
    };
    if (cudaSetDevice(desc->device) != cudaSuccess) return fail(ET_ERR_CUDA);
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, desc->device) != cudaSuccess) return fail(ET_ERR_CUDA);
    if (prop.major != 10) return fail(ET_ERR_UNSUPPORTED);
    g->dev = desc->device;
    g->n_sm = prop.multiProcessorCount;
    g->n_ctas = desc->n_ctas > 0 ? std::min(desc->n_ctas, g->n_sm) : g->n_sm;
    // the decode MLP has no irregular operator: its hybrid schedule is the static one
    g->hybrid = desc->sched == ET_SCHED_HYBRID && desc->kind != ET_GRAPH_MLP;
    et_status st = ET_ERR_INVALID;
    if (desc->kind == ET_GRAPH_SPLITK) st = build_splitk(g);
    else if (desc->kind == ET_GRAPH_MLP) st = build_mlp(g);
    else if (desc->kind == ET_GRAPH_MOE) st = build_moe(g);
    else if (desc->kind == ET_GRAPH_MOE_MLP) st = build_moe_mlp(g);
    else st = build_decode(g);
    if (st != ET_OK) return fail(st);
    // common workspace
    if ((st = galloc(g, &g->ctl, 1)) != ET_OK) return fail(st);
    {
        void* hp = nullptr;
        if (cudaHostAlloc(&hp, sizeof(int), cudaHostAllocMapped) != cudaSuccess) return fail(ET_ERR_OOM);
        g->host_status = static_cast<int*>(hp);
        void* dp = nullptr;
        if (cudaHostGetDevicePointer(&dp, hp, 0) != cudaSuccess) return fail(ET_ERR_CUDA);
        g->host_status_dev = static_cast<int*>(dp);
        if ((st = reset_ctl(g)) != ET_OK) return fail(st);
    }
    if ((st = galloc(g, &g->ctr[0], g->n_ctr)) != ET_OK) return fail(st);
    if ((st = galloc(g, &g->ctr[1], g->n_ctr)) != ET_OK) return fail(st);
    if ((st = galloc(g, &g->qslots, g->qcap)) != ET_OK) return fail(st);
    g->trace_cap = (g->d.debug_flags & ET_DEBUG_TRACE) ? g->qcap + 1024 + 256 : 1;  // + one record per CTA (ET_DEBUG_CTA_TIMES)
    if ((st = galloc(g, &g->trace, g->trace_cap)) != ET_OK) return fail(st);
    if (cudaDeviceSynchronize() != cudaSuccess) return fail(ET_ERR_CUDA);
    // info
    et_graph_info& in = g->info;
    memset(&in, 0, sizeof(in));
    in.kind = g->d.kind;
    in.sched = g->d.sched;
    in.max_T = g->d.max_T;
    in.n_ctas = g->n_ctas;
    in.threads = (desc->kind == ET_GRAPH_MOE || desc->kind == ET_GRAPH_MOE_MLP) ? kThreadsGather : kThreads;
    in.smem_bytes = g->d.kind == ET_GRAPH_SPLITK ? kSmemNoArenaBytes : kSmemBytes;
    in.fetch_batch = g->d.fetch_batch;
    in.hidden = g->d.hidden;
    in.inter = g->d.inter;
    in.n_experts = g->d.n_experts;
    in.top_k = g->d.top_k;
    in.splitk_cols = g->d.splitk_cols;
    in.splitk_chunk = g->d.splitk_chunk;
    in.splitk_tile_rows = g->d.splitk_tile_rows;
    if (desc->kind == ET_GRAPH_MLP) {
        in.mlp_gu_tile = g->mlp.gu_tile;
        in.mlp_down_tile = g->mlp.down_tile;
        in.mlp_kchunk = g->mlp.kchunk;
    }
    if (desc->kind == ET_GRAPH_MOE_MLP) {
        in.mlp_gu_tile = g->mlp.gu_tile;
        in.mlp_down_tile = g->mlp.down_tile;
        in.mlp_kchunk = g->mlp.kchunk;
    }
    if (desc->kind == ET_GRAPH_MOE || desc->kind == ET_GRAPH_MOE_MLP) {
        in.moe_tt = g->moe.tt;
        in.moe_gt = g->moe.tt;
        in.moe_tkt = g->moe.tkt;
        in.moe_bm = g->moe.bm;
        in.moe_n1_tile = g->moe.n1_tile;
        in.moe_n2_tile = g->moe.n2_tile;
        in.moe_cb = moe_cb_for(g->d.max_T);
    }
    if (desc->kind == ET_GRAPH_DECODE) {
        in.dec_split = g->dec.split;
        in.dec_qkv_kc = g->dec.n_kc;
        in.dec_o_kc = g->dec.o_kc;
        in.mlp_gu_tile = g->dec.gu_tile;
        in.mlp_down_tile = 128;
        in.mlp_kchunk = g->dec.kchunk;
    }
    *out = g;
    return ET_OK;
}

void et_destroy_graph(et_graph* g) {
    if (!g) return;
    cudaSetDevice(g->dev);
    cudaDeviceSynchronize();
    for (void* p : g->allocs) cudaFree(p);
    if (g->host_status) cudaFreeHost(g->host_status);
    delete g;
}

et_status et_get_info(const et_graph* g, et_graph_info* info) {
    if (!g || !info) return ET_ERR_INVALID;
    *info = g->info;
    return ET_OK;
}

et_status et_run_splitk(et_graph* g, const float* A, int n_rows, float* Bpart, float* C, void* stream) {
    if (!g || g->d.kind != ET_GRAPH_SPLITK) return ET_ERR_INVALID;
    if (n_rows < 0 || n_rows > g->d.max_T) return ET_ERR_INVALID;
    if (n_rows == 0) return ET_OK;
    if (!aligned16(A) || !aligned16(Bpart) || !aligned16(C)) return ET_ERR_INVALID;
    cudaStream_t s = (cudaStream_t)stream;
    ET_CU(cudaSetDevice(g->dev));
    SplitKParams p = g->sk;
    p.A = A;
    p.Bp = Bpart;
    p.C = C;
    p.rows = n_rows;
    p.n_tiles = cdiv(n_rows, p.tile_rows);
    ET_TRY(pre_run(g, s));
    const int n_init = g->hybrid ? 0 : p.n_tiles * p.n_chunks;  // hybrid: partials are listed
    RunArgs ra = run_args(g, n_rows, n_init, n_init + p.n_tiles);
    ET_TRY(launched(g, launch_splitk(p, ra, g->n_ctas, s)));
    g->last_T = n_rows;
    g->last_sk = p;
    return ET_OK;
}

et_status et_run_splitk_two_launch(const float* A, int n_rows, int cols, int chunk, float* Bpart, float* C,
                                   void* stream) {
    if (n_rows < 0 || cols < 1 || chunk < 1) return ET_ERR_INVALID;
    if (n_rows == 0) return ET_OK;
    if (!aligned16(A) || !aligned16(Bpart) || !aligned16(C)) return ET_ERR_INVALID;
    ET_CU(launch_splitk_two(A, n_rows, cols, chunk, Bpart, C, (cudaStream_t)stream));
    return ET_OK;
}

et_status et_run_mlp(et_graph* g, int B, const uint16_t* X, const uint16_t* gamma, const uint16_t* Wgu,
                     const uint16_t* Wd, uint16_t* Y, void* stream) {
    if (!g || g->d.kind != ET_GRAPH_MLP) return ET_ERR_INVALID;
    if (B < 1 || B > g->d.max_T) return ET_ERR_INVALID;
    if (!aligned16(X) || !aligned16(gamma) || !aligned16(Wgu) || !aligned16(Wd) || !aligned16(Y))
        return ET_ERR_INVALID;
    cudaStream_t s = (cudaStream_t)stream;
    ET_CU(cudaSetDevice(g->dev));
    MlpParams& p = g->mlp;
    if (!g->mc[0].get(&p.tm_wgu, Wgu, 2ull * p.inter, p.hidden, 64)) return ET_ERR_CUDA;
    if (!g->mc[1].get(&p.tm_wd, Wd, p.hidden, p.inter, 64)) return ET_ERR_CUDA;
    p.X = X;
    p.gamma = gamma;
    p.Y = Y;
    p.B = B;
    ET_TRY(pre_run(g, s));
    const int total = B + p.n_gu + p.n_m * p.n_c + p.n_m;
    RunArgs ra = run_args(g, B, B, total);
    ET_TRY(launched(g, launch_mlp(p, ra, g->n_ctas, s)));
    g->last_T = B;
    g->last_mlp = p;
    return ET_OK;
}

// Fill the MoE half's per-run fields (shared by et_run_moe and et_run_moe_mlp).
et_status moe_run_params(et_graph* g, int T, const uint16_t* X, const uint16_t* Wr, const float* bias,
                         const uint16_t* W1, const uint16_t* W2, uint16_t* Y) {
    MoeParams& p = g->moe;
    if (!g->mc[0].get(&p.tm_wr, Wr, p.E, p.hidden, 64)) return ET_ERR_CUDA;
    if (!g->mc[1].get(&p.tm_w1, W1, (uint64_t)p.E * 2 * p.inter, p.hidden, 64)) return ET_ERR_CUDA;
    if (!g->mc[2].get(&p.tm_w2, W2, (uint64_t)p.E * p.hidden, p.inter, 64)) return ET_ERR_CUDA;
    if (!g->mc[3].get(&p.tm_x, X, T, p.hidden, 16)) return ET_ERR_CUDA;
    p.X = X;
    p.bias = bias;
    p.Y = Y;
    p.out_topk = nullptr;
    p.out_w = nullptr;
    p.out_indptr = nullptr;
    p.out_perm = nullptr;
    p.out_logits = nullptr;
    p.T = T;
    const int b = g->bucket_of(T);
    const MoeShape mb = moe_shape(g, p, g->bucket_T[b]);
    const MoeShape mt = moe_shape(g, p, T);
    p.n_tt = mt.n_tt;
    p.n_tk = mt.n_tk;
    p.n_kc = mb.n_kc;  // the size bucket fixes the router split and the combine block
    p.cb = mb.cb;      // (static lists and dynamic alike)
    p.n_cb = cdiv(T, p.cb);
    p.f_max = mb.f_max;
    p.use_xp = p.Xp != nullptr && p.n_tt > 1 && T >= g->d.moe_xp_min_T;
    return ET_OK;
}

et_status et_run_moe(et_graph* g, int T, const uint16_t* X, const uint16_t* Wr, const float* bias,
                     const uint16_t* W1, const uint16_t* W2, uint16_t* Y, int32_t* topk, float* topk_w,
                     int32_t* indptr, int32_t* perm, float* logits, void* stream) {
    if (!g || g->d.kind != ET_GRAPH_MOE) return ET_ERR_INVALID;
    if (T < 1 || T > g->d.max_T) return ET_ERR_INVALID;
    if (!aligned16(X) || !aligned16(Wr) || !bias || !aligned16(W1) || !aligned16(W2) || !aligned16(Y))
        return ET_ERR_INVALID;
    cudaStream_t s = (cudaStream_t)stream;
    ET_CU(cudaSetDevice(g->dev));
    ET_TRY(moe_run_params(g, T, X, Wr, bias, W1, W2, Y));
    MoeParams& p = g->moe;
    p.out_topk = topk;
    p.out_w = topk_w;
    p.out_indptr = indptr;
    p.out_perm = perm;
    p.out_logits = logits;
    ET_TRY(pre_run(g, s));
    RunArgs ra = run_args(g, T, g->hybrid ? 0 : p.n_tk * p.n_kc, 0);  // hybrid: router tasks are listed
    ET_TRY(launched(g, launch_moe(p, ra, g->n_ctas, s)));
    g->last_T = T;
    g->last_moe = p;
    return ET_OK;
}

et_status et_run_decode(et_graph* g, int B, const uint16_t* X, const int32_t* pos, const et_decode_weights* w,
                        uint16_t* Kc, uint16_t* Vc, uint16_t* Y, uint16_t* h1, void* stream) {
    if (!g || g->d.kind != ET_GRAPH_DECODE || !w) return ET_ERR_INVALID;
    if (B < 1 || B > g->d.max_T) return ET_ERR_INVALID;
    if (!aligned16(X) || !aligned16(pos) || !aligned16(w->g1) || !aligned16(w->Wqkv) || !aligned16(w->gq) ||
        !aligned16(w->gk) || !aligned16(w->Wo) || !aligned16(w->g2) || !aligned16(w->Wgu) || !aligned16(w->Wd) ||
        !aligned16(Kc) || !aligned16(Vc) || !aligned16(Y) || (h1 && !aligned16(h1)))
        return ET_ERR_INVALID;
    cudaStream_t s = (cudaStream_t)stream;
    ET_CU(cudaSetDevice(g->dev));
    DecodeParams& p = g->dec;
    if (!g->mc[0].get(&p.tm_wqkv, w->Wqkv, (uint64_t)p.n_heads * p.hd, p.hidden, 64)) return ET_ERR_CUDA;
    if (!g->mc[1].get(&p.tm_wo, w->Wo, p.hidden, (uint64_t)p.nq * p.hd, 64)) return ET_ERR_CUDA;
    if (!g->mc[2].get(&p.tm_wgu, w->Wgu, 2ull * p.inter, p.hidden, 64)) return ET_ERR_CUDA;
    if (!g->mc[3].get(&p.tm_wd, w->Wd, p.hidden, p.inter, 64)) return ET_ERR_CUDA;
    const uint64_t cache_rows = (uint64_t)B * p.nkv;
    if (!g->mc[4].get(&p.tm_kc, Kc, cache_rows * p.max_ctx, p.hd, 128)) return ET_ERR_CUDA;
    if (!g->mc[5].get(&p.tm_vt, Vc, cache_rows * p.hd, p.max_ctx, 128)) return ET_ERR_CUDA;
    p.X = X;
    p.pos = pos;
    p.g1 = w->g1;
    p.gq = w->gq;
    p.gk = w->gk;
    p.g2 = w->g2;
    p.Kc = Kc;
    p.Vc = Vc;
    p.Y = Y;
    p.out_h1 = h1;
    p.out_q = nullptr;
    p.B = B;
    p.split = dec_split_for(g, B);
    ET_TRY(pre_run(g, s));
    RunArgs ra = run_args(g, B, g->d.sched == ET_SCHED_DYNAMIC ? B : 0, 0);
    ET_TRY(launched(g, launch_decode(p, ra, g->n_ctas, s)));
    g->last_T = B;
    g->last_dec = p;
    g->info.dec_split = p.split;  // the info reports the last run's split
    return ET_OK;
}

et_status et_run_moe_mlp(et_graph* g, int T, const uint16_t* X, const uint16_t* Wr, const float* bias,
                         const uint16_t* W1, const uint16_t* W2, const uint16_t* gamma, const uint16_t* Wgu,
                         const uint16_t* Wd, uint16_t* Y1, uint16_t* Y2, void* stream) {
    if (!g || g->d.kind != ET_GRAPH_MOE_MLP) return ET_ERR_INVALID;
    if (T < 1 || T > g->d.max_T) return ET_ERR_INVALID;
    if (!aligned16(X) || !aligned16(Wr) || !bias || !aligned16(W1) || !aligned16(W2) || !aligned16(gamma) ||
        !aligned16(Wgu) || !aligned16(Wd) || !aligned16(Y1) || !aligned16(Y2))
        return ET_ERR_INVALID;
    cudaStream_t s = (cudaStream_t)stream;
    ET_CU(cudaSetDevice(g->dev));
    ET_TRY(moe_run_params(g, T, X, Wr, bias, W1, W2, Y1));
    MlpParams& m = g->mlp;
    if (!g->mc[4].get(&m.tm_wgu, Wgu, 2ull * m.inter, m.hidden, 64)) return ET_ERR_CUDA;
    if (!g->mc[5].get(&m.tm_wd, Wd, m.hidden, m.inter, 64)) return ET_ERR_CUDA;
    m.gamma = gamma;
    m.Y = Y2;
    m.B = T;
    g->moe.mlp_gamma = gamma;
    ET_TRY(pre_run(g, s));
    MoeMlpParams pp;
    pp.moe = g->moe;
    pp.mlp = m;
    RunArgs ra = run_args(g, T, g->hybrid ? 0 : g->moe.n_tk * g->moe.n_kc, 0);
    ET_TRY(launched(g, launch_moe_mlp(pp, ra, g->n_ctas, s)));
    g->last_T = T;
    g->last_moe = g->moe;
    g->last_moe_mlp = m;
    return ET_OK;
}

et_status et_sync_status(et_graph* g, void* stream) {
    if (!g) return ET_ERR_INVALID;
    ET_CU(cudaSetDevice(g->dev));
    ET_CU(cudaStreamSynchronize((cudaStream_t)stream));
    Ctl h;
    ET_CU(cudaMemcpy(&h, g->ctl, sizeof(Ctl), cudaMemcpyDeviceToHost));
    if (h.status == 0) return ET_OK;
    // reset: status, abort flag, host mirror, counters, scratch that must start at zero
    ET_CU(cudaDeviceSynchronize());
    ET_TRY(reset_ctl(g));
    ET_CU(cudaMemset(g->ctr[0], 0, g->n_ctr * sizeof(int)));
    ET_CU(cudaMemset(g->ctr[1], 0, g->n_ctr * sizeof(int)));
    if (g->d.kind == ET_GRAPH_MLP || g->d.kind == ET_GRAPH_MOE_MLP)  // sums kept zero between runs
        ET_CU(cudaMemset(g->mlp.yacc, 0, (size_t)g->mlp.maxB * g->mlp.hidden * sizeof(float)));
    if (g->d.kind == ET_GRAPH_DECODE) {
        const DecodeParams& p = g->dec;
        ET_CU(cudaMemset(p.qkvacc, 0, (size_t)p.maxB * p.n_heads * p.hd * sizeof(float)));
        ET_CU(cudaMemset(p.h1acc, 0, (size_t)p.maxB * p.hidden * sizeof(float)));
        ET_CU(cudaMemset(p.yacc, 0, (size_t)p.maxB * p.hidden * sizeof(float)));
    }
    if ((g->d.kind == ET_GRAPH_MOE || g->d.kind == ET_GRAPH_MOE_MLP) && g->moe.Yacc) {
        ET_CU(cudaMemset(g->moe.Yacc, 0, (size_t)g->moe.maxT * g->moe.hidden * sizeof(float)));
        ET_CU(cudaMemset(g->moe.lacc, 0, (size_t)g->moe.maxT * g->moe.E * sizeof(float)));
    }
    ET_CU(cudaDeviceSynchronize());
    // keep the diagnostic words readable through et_get_diag
    ET_CU(cudaMemcpy(g->ctl->diag, h.diag, sizeof(h.diag), cudaMemcpyHostToDevice));
    return (et_status)h.status;
}

et_status et_get_trace(et_graph* g, void* host_buf, size_t bytes, int* n_records) {
    if (!g || !n_records) return ET_ERR_INVALID;
    ET_CU(cudaSetDevice(g->dev));
    ET_CU(cudaDeviceSynchronize());
    Ctl h;
    ET_CU(cudaMemcpy(&h, g->ctl, sizeof(Ctl), cudaMemcpyDeviceToHost));
    int n = std::min(h.n_trace, g->trace_cap);
    *n_records = n;
    size_t want = std::min((size_t)n * sizeof(TraceRec), bytes);
    if (host_buf && want) ET_CU(cudaMemcpy(host_buf, g->trace, want, cudaMemcpyDeviceToHost));
    return ET_OK;
}

et_status et_get_event_counts(et_graph* g, et_event_count* buf, int cap, int* n_events) {
    if (!g || !n_events || cap < 0 || (cap > 0 && !buf)) return ET_ERR_INVALID;
    if (g->last_T == 0) return ET_ERR_INVALID;
    ET_CU(cudaSetDevice(g->dev));
    ET_CU(cudaDeviceSynchronize());
    std::vector<int> c(g->n_ctr);
    ET_CU(cudaMemcpy(c.data(), g->ctr[g->epoch & 1], g->n_ctr * sizeof(int), cudaMemcpyDeviceToHost));
    std::vector<et_event_count> v;
    auto add = [&](int kind, int idx, int ctr_index) { v.push_back({kind, idx, c[ctr_index]}); };
    if (g->d.kind == ET_GRAPH_SPLITK) {
        const SplitKParams& p = g->last_sk;
        for (int i = 0; i < p.n_tiles; ++i) add(ET_EV_SK_TILE, i, p.ev_base + i);
        add(ET_EV_SK_ALL, 0, p.ev_all);
    } else if (g->d.kind == ET_GRAPH_MLP) {
        const MlpParams& p = g->last_mlp;
        add(ET_EV_MLP_NORM, 0, p.ev_norm);
        for (int i = 0; i < p.n_c; ++i) add(ET_EV_MLP_H, i, p.ev_h + i);
        for (int i = 0; i < p.n_m; ++i) add(ET_EV_MLP_Y, i, p.ev_y + i);
        add(ET_EV_MLP_GU_ALL, 0, p.ev_gu_all);
        add(ET_EV_MLP_DOWN_ALL, 0, p.ev_down_all);
    } else if (g->d.kind == ET_GRAPH_DECODE) {
        const DecodeParams& p = g->last_dec;
        add(ET_EV_DEC_N1, 0, p.ev_n1);
        for (int n = 0; n < p.n_heads; ++n) add(ET_EV_DEC_QKV, n, p.ev_qkv + n);
        for (int gg = 0; gg < p.nkv; ++gg) add(ET_EV_DEC_G, gg, p.ev_g + gg);
        for (int i = 0; i < p.B * p.nkv; ++i) add(ET_EV_DEC_ATT, i, p.ev_att + i);
        for (int gg = 0; gg < p.nkv; ++gg) add(ET_EV_DEC_AG, gg, p.ev_ag + gg);
        add(ET_EV_DEC_O, 0, p.ev_o);
        add(ET_EV_DEC_N2, 0, p.ev_n2);
        for (int c = 0; c < p.n_c; ++c) add(ET_EV_DEC_H, c, p.ev_h + c);
        for (int m = 0; m < p.n_m; ++m) add(ET_EV_DEC_Y, m, p.ev_y + m);
        add(ET_EV_DEC_BRANCH_ALL, 0, p.ev_branch_all);
        add(ET_EV_DEC_MERGE_ALL, 0, p.ev_merge_all);
        add(ET_EV_DEC_GU_ALL, 0, p.ev_gu_all);
        add(ET_EV_DEC_DOWN_ALL, 0, p.ev_down_all);
    } else {
        const MoeParams& p = g->last_moe;
        for (int j = 0; j < p.n_tk; ++j) add(ET_EV_MOE_RT, j, p.ev_rt + j);
        add(ET_EV_MOE_TK, 0, p.ev_tk);
        add(ET_EV_MOE_SC, 0, p.ev_sc);
        add(ET_EV_MOE_GRP, 0, p.ev_grp);
        for (int e = 0; e < p.E; ++e) add(ET_EV_MOE_EXP, e, p.ev_exp + e);
        for (int f = 0; f < p.f_max; ++f) add(ET_EV_MOE_S1, f, p.ev_s1 + f);
        for (int b = 0; b < p.n_cb; ++b) add(ET_EV_MOE_CB, b, p.ev_cb + b);
        add(ET_EV_MOE_S1_ALL, 0, p.ev_s1_all);
        add(ET_EV_MOE_S2_ALL, 0, p.ev_s2_all);
        if (g->d.kind == ET_GRAPH_MOE_MLP) {
            const MlpParams& m = g->last_moe_mlp;
            add(ET_EV_MLP_NORM, 0, m.ev_norm);
            for (int i = 0; i < m.n_c; ++i) add(ET_EV_MLP_H, i, m.ev_h + i);
            for (int i = 0; i < m.n_m; ++i) add(ET_EV_MLP_Y, i, m.ev_y + i);
            add(ET_EV_MLP_GU_ALL, 0, m.ev_gu_all);
            add(ET_EV_MLP_DOWN_ALL, 0, m.ev_down_all);
        }
    }
    *n_events = (int)v.size();
    for (int i = 0; i < cap && i < (int)v.size(); ++i) buf[i] = v[i];
    return ET_OK;
}

et_status et_get_diag(et_graph* g, int32_t* out8) {
    if (!g || !out8) return ET_ERR_INVALID;
    ET_CU(cudaSetDevice(g->dev));
    ET_CU(cudaDeviceSynchronize());
    ET_CU(cudaMemcpy(out8, g->ctl->diag, 8 * sizeof(int32_t), cudaMemcpyDeviceToHost));
    return ET_OK;
}

}  // extern "C"
