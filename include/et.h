/*
 * et.h -- C ABI of the event-tensor megakernel library (libet.so).
 *
 * One persistent kernel launch runs every tiled task of a small operator
 * graph.  Tasks are ordered by event tensors: arrays of counters with a
 * symbolic shape; a producer task notifies an event, a consumer task runs
 * once the event has received its wait count of notifications.  Sources,
 * cited by page title and section:
 *   [ETN] "Event Tensor：用“事件张量”编译动态 Megakernel" (reading notes on
 *         "Event Tensor: A Unified Abstraction for Compiling Dynamic
 *         Megakernel", MLSys 2026)
 *   [ETS] hyper.ai summary of the same paper, §方法
 *   [WV]  "MoE Kernel动态SM调度：从静态分配到任务池，4卡H100加速2.89×"
 *         (batched atomic pops, §2.2)
 *
 * Conventions for every entry point:
 *  - Tensor pointers are DEVICE pointers owned by the caller, row-major and
 *    contiguous, 16-byte aligned.  bf16 tensors are passed as uint16_t bit
 *    patterns.  The library never frees or retains them past the call.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Runs are
 *    asynchronous: et_run_* returns after the launch; device-side errors
 *    (a wait that timed out) are reported by et_sync_status.
 *  - A device error is sticky per graph until et_sync_status collects it.
 *    The failing kernel also mirrors its status into a word of mapped
 *    host memory, so once the error has happened every et_run_* on the
 *    graph returns ET_ERR_PENDING without launching.  A run that was
 *    already launched (or issued before the error happened) finds the error
 *    when it starts, does no work and leaves its outputs untouched; its
 *    et_run_* returned ET_OK, and et_sync_status reports the error.
 *  - The token / batch count T (or B, or the split-K row count) is a plain
 *    run-time int: the same graph and binary serve every value up to
 *    max_T with no recompile and no graph capture ([ETN] §Shape dynamism).
 *  - A graph owns its workspace (event counters, ready queue, static task
 *    lists, scratch tensors, status word, trace buffer).  Runs of one graph
 *    must be issued on one stream, one after another; the library is not
 *    re-entrant per graph.  Different graphs are independent.
 *  - Errors: every function returns an et_status; ET_OK = 0.
 */
#ifndef ET_H_
#define ET_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ET_OK = 0,
    ET_ERR_INVALID = 1,     /* bad argument: null/misaligned pointer, T out of range, wrong graph kind */
    ET_ERR_CUDA = 2,        /* a CUDA runtime/driver call failed */
    ET_ERR_TIMEOUT = 3,     /* a device-side wait exceeded its time limit (see et_sync_status) */
    ET_ERR_OOM = 4,         /* workspace allocation failed */
    ET_ERR_UNSUPPORTED = 5, /* device is not sm_100, or dims outside what the kernels tile */
    ET_ERR_PENDING = 6,     /* an earlier run of this graph failed on the device and the error was
                               not yet collected by et_sync_status: nothing was launched */
    ET_ERR_INTERNAL = 7     /* a device-side capacity check failed (a ready-queue push past its
                               capacity); the run aborted instead of losing the task */
} et_status;

/* How tasks are ordered on the SMs ([ETN] §静态调度, §动态调度, §静态与动态调度的消融). */
typedef enum {
    ET_SCHED_STATIC = 0,  /* per-SM task lists fixed at build time (one set per power-of-two
                             size bucket); consumers spin-wait on their events */
    ET_SCHED_DYNAMIC = 1, /* a device-side ready queue: a producer that brings an event to its
                             wait count pushes the consumers; SMs pop in batches */
    ET_SCHED_UNFUSED = 2, /* control: the static lists with one barrier event between
                             consecutive operators (the "unfused megakernel" baseline) */
    ET_SCHED_HYBRID = 3   /* per operator: regular operators from static per-SM lists, irregular
                             (data-dependent) ones through the ready queue, in one launch.  Each
                             CTA runs its list part A, pops the queue until it is exhausted, then
                             runs its list part B.  split-K: partials static, finals queued;
                             MoE: router static, grouping, expert stages and combine queued;
                             decode layer: QKV static (part A), attention splits queued,
                             o-proj and MLP static (part B); decode MLP: all static */
} et_sched;

typedef enum {
    ET_GRAPH_SPLITK = 0,
    ET_GRAPH_MLP = 1,
    ET_GRAPH_MOE = 2,
    ET_GRAPH_DECODE = 3,
    ET_GRAPH_MOE_MLP = 4  /* the MoE layer followed by a dense SwiGLU MLP on its output */
} et_graph_kind;

/* debug_flags bits */
#define ET_DEBUG_TRACE 1      /* record one et_trace_record per task (tickets from one global counter) */
#define ET_DEBUG_DELAY 2      /* each task first spins a pseudo-random 0..~20 us, to perturb the order */
#define ET_DEBUG_BAD_COUNT 4  /* raise one event's wait count by one: a run must then end in
                                 ET_ERR_TIMEOUT (used to test the timeout path) */
#define ET_DEBUG_CTA_TIMES 8  /* with ET_DEBUG_TRACE: also one ET_OP_CTA record per CTA (a = CTA):
                                 t_fetch = kernel entry, t_ready = set-up done, t_end = roles done */

typedef struct {
    int kind;            /* et_graph_kind */
    int sched;           /* et_sched */
    int max_T;           /* largest T (MoE tokens), B (MLP batch) or split-K row count */
    /* dims; 0 = the default in brackets */
    int hidden;          /* MLP [4096] / MoE [2048] model width */
    int inter;           /* MLP [14336] / MoE [768] intermediate width */
    int n_experts;       /* MoE [128] */
    int top_k;           /* MoE [8] */
    int splitk_cols;     /* split-K columns [128] */
    int splitk_chunk;    /* split-K K-chunk [32] */
    int splitk_tile_rows;/* split-K rows per task [32] */
    float rms_eps;       /* MLP RMSNorm epsilon [1e-5] */
    int fetch_batch;     /* dynamic: tasks claimed per atomic pop [1] */
    int debug_flags;     /* ET_DEBUG_* */
    int device;          /* CUDA device ordinal */
    int n_ctas;          /* persistent CTAs [0 = one per SM] */
    float timeout_ms;    /* per-wait device time limit [1000] */
    /* decode layer (ET_GRAPH_DECODE); hidden/inter above default to 4096 / 14336 */
    int n_heads;         /* query heads [32] */
    int n_kv_heads;      /* key/value heads [8]; n_heads / n_kv_heads <= 4 */
    int head_dim;        /* [128]; only 128 is supported */
    int max_ctx;         /* cache positions per request [4104]: a multiple of 8, at most
                            1024 * dec_split / (n_heads / n_kv_heads); a run's positions must be < max_ctx */
    float rope_base;     /* rotary embedding base [500000] */
    /* MoE -> dense MLP (ET_GRAPH_MOE_MLP); the MoE dims above, the MLP's width = hidden */
    int mlp_inter;       /* dense MLP intermediate width [6144] */
    /* MoE: from this T on (when several 128-token grouping tiles exist) each grouping task
       also copies its tokens' rows of X into a permuted copy in grouped order, and stage 1
       loads its token rows from there by TMA instead of gathering them from X for every
       column tile [0 = the default: never; -1 = never] */
    int moe_xp_min_T;
} et_graph_desc;

typedef struct et_graph et_graph; /* opaque, library-owned */

/* Tile parameters of a built graph (what the task coordinates mean). */
typedef struct {
    int kind, sched, max_T, n_ctas;
    int threads;         /* per CTA: 192 (224 in the MoE graphs, which add a warp that copies
                            gathered token rows) */
    int smem_bytes, fetch_batch;
    int hidden, inter, n_experts, top_k;
    int splitk_cols, splitk_chunk, splitk_tile_rows;
    int mlp_gu_tile;     /* intermediate columns per gate/up task */
    int mlp_down_tile;   /* output columns per down task */
    int mlp_kchunk;      /* K (intermediate) columns per down task */
    int moe_tt;          /* tokens per grouping tile (pair counts are kept per tile) */
    int moe_gt;          /* tokens per grouping task (= moe_tt) */
    int moe_tkt;         /* tokens per router block (router GEMM, then top-k + softmax) */
    int moe_bm;          /* rows (token, slot pairs) per expert m-tile */
    int moe_n1_tile;     /* intermediate columns per stage-1 task */
    int moe_n2_tile;     /* output columns per stage-2 task */
    int moe_cb;          /* tokens per combine task at this graph's max_T; a run whose size
                            bucket (the power of two >= T, capped at max_T) is <= 256 uses 1 */
    int dec_split;       /* decode: keys per attention split task of the last run (before any run:
                            the graph's, 512); the dynamic and hybrid schedules double it from
                            B = 8 and quadruple it from B = 32, static lists keep the graph's */
    int dec_qkv_kc;      /* decode: K chunks of a QKV head tile (as many as keep every QKV task in
                            one wave over the CTAs; chunk c = stages [c kt / n, (c + 1) kt / n)) */
    int dec_o_kc;        /* decode: K columns per o-proj task (the heads of one KV group) */
} et_graph_info;

/* Trace record (ET_DEBUG_TRACE): one per executed task. */
typedef struct {
    int32_t op, a, b, sm;
    uint32_t start;   /* ticket taken after the task's wait succeeded */
    uint32_t end;     /* ticket taken after its outputs were written, before its notify */
    uint64_t t_fetch; /* %globaltimer (ns): task taken from the static list / ready queue */
    uint64_t t_ready; /* %globaltimer: input event complete */
    uint64_t t_acc;   /* %globaltimer: tensor-core accumulator ready (GEMM tasks), else 0 */
    uint64_t t_end;   /* %globaltimer: outputs written */
} et_trace_record;

/* trace op codes */
#define ET_OP_SK_PARTIAL 1
#define ET_OP_SK_FINAL 2
#define ET_OP_MLP_NORM 10
#define ET_OP_MLP_GATEUP 11
#define ET_OP_MLP_DOWN 12
#define ET_OP_MLP_REDUCE 13
#define ET_OP_MOE_ROUTER 20 /* a = 16-token block, b = K chunk (up to 8 at small T); the chunk
                               that completes the block also takes its top-k and softmax */
#define ET_OP_MOE_SCAN 22
#define ET_OP_MOE_GROUP 23
#define ET_OP_MOE_S1 24
#define ET_OP_MOE_S2 25
#define ET_OP_MOE_COMBINE 26
#define ET_OP_DEC_NORM1 30    /* a = request */
#define ET_OP_DEC_QKV 31      /* a = head tile (query heads, then key heads, then value heads), b = K chunk */
#define ET_OP_DEC_QBR 32      /* inline: Q branch (norm + RoPE) of head a, run by the QKV task completing it */
#define ET_OP_DEC_KBR 33      /* inline: K branch (norm + RoPE + cache append) of head tile a */
#define ET_OP_DEC_VBR 34      /* inline: V cache append of head tile a */
#define ET_OP_DEC_ATTN 35     /* a = request * n_kv_heads + KV head, b = split */
#define ET_OP_DEC_MERGE 36    /* inline: merge of the splits of (request, KV head) a */
#define ET_OP_DEC_OPROJ 37    /* a = output tile, b = K chunk (= KV head group) */
#define ET_OP_DEC_NORM2 38    /* a = request */
#define ET_OP_DEC_GATEUP 39   /* a = intermediate tile */
#define ET_OP_DEC_DOWN 40     /* a = output tile, b = K chunk */
#define ET_OP_DEC_RED 41      /* a = output tile */
#define ET_OP_CTA 60          /* ET_DEBUG_CTA_TIMES: a = CTA index (not a task) */

/* Event kinds of et_event_count records; index = the event's coordinate. */
#define ET_EV_SK_TILE 1       /* split-K E[i]: partial tasks of row tile i done (count = #chunks) */
#define ET_EV_SK_ALL 2        /* split-K, unfused control: every partial task done */
#define ET_EV_MLP_NORM 10     /* E_norm: normalised rows (count = B) */
#define ET_EV_MLP_H 11        /* E_h[c]: gate/up tiles of down K-chunk c */
#define ET_EV_MLP_Y 12        /* E_y[m]: down partials of output tile m (count = #K chunks) */
#define ET_EV_MLP_GU_ALL 13   /* unfused control: every gate/up tile */
#define ET_EV_MLP_DOWN_ALL 14 /* unfused control: every down tile */
#define ET_EV_MOE_RT 20       /* E_rt[j]: K chunks of router block j (kept only when the K is split) */
#define ET_EV_MOE_TK 21       /* E_tk: router blocks routed (top-k taken) */
#define ET_EV_MOE_SC 22       /* E_sc: the scan (runs with several grouping tiles) */
#define ET_EV_MOE_GRP 23      /* E_grp: the coarse grouping event (static and unfused schedules) */
#define ET_EV_MOE_EXP 24      /* E_exp[e]: pairs of expert e placed (dynamic, several grouping tiles;
                                 one tile is grouped by the scan, which then triggers directly) */
#define ET_EV_MOE_S1 25       /* E_s1[f]: stage-1 tiles of m-tile f */
#define ET_EV_MOE_CB 26       /* E_cb[b]: stage-2 row contributions to combine block b */
#define ET_EV_MOE_S1_ALL 27   /* unfused control: every stage-1 tile */
#define ET_EV_MOE_S2_ALL 28   /* unfused control: every stage-2 tile */
#define ET_EV_DEC_N1 40        /* E_n1: normalised rows (count B) */
#define ET_EV_DEC_QKV 41       /* E_qkv[n]: K chunks of head tile n */
#define ET_EV_DEC_G 42         /* E_g[g]: branches of KV group g done (its query heads, K and V) */
#define ET_EV_DEC_ATT 43       /* E_att[b * n_kv + g]: attention splits of (request b, KV head g);
                                  wait count = the request's split count (data-dependent) */
#define ET_EV_DEC_AG 44        /* E_ag[g]: attention output of KV group g merged for every request */
#define ET_EV_DEC_O 45         /* E_o: o-proj tiles */
#define ET_EV_DEC_N2 46        /* E_n2: residual + norm rows */
#define ET_EV_DEC_H 47         /* E_h[c]: gate/up tiles of down K-chunk c */
#define ET_EV_DEC_Y 48         /* E_y[m]: down tiles of output tile m */
#define ET_EV_DEC_BRANCH_ALL 49 /* unfused control: every head branch */
#define ET_EV_DEC_MERGE_ALL 50 /* unfused control: every merge */
#define ET_EV_DEC_GU_ALL 51    /* unfused control: every gate/up tile */
#define ET_EV_DEC_DOWN_ALL 52  /* unfused control: every down tile */

/* Notifications one event received in the last run (debug introspection). */
typedef struct {
    int32_t kind;   /* ET_EV_* */
    int32_t index;  /* coordinate of the event in its event tensor */
    int32_t count;  /* notifications received (the pages' wait count minus the remaining count) */
} et_event_count;

/* Build a graph: validate dims, allocate its workspace for max_T, build the
 * static per-SM task lists for every power-of-two bucket up to max_T
 * ([ETN] §静态调度: "per-SM task queue" materialised at build time; an
 * unsampled size reuses the next larger bucket).  Host-side, once.
 * Errors: ET_ERR_INVALID (bad desc), ET_ERR_UNSUPPORTED (not sm_100 or dims
 * the tiles do not cover), ET_ERR_OOM, ET_ERR_CUDA. */
et_status et_build_graph(const et_graph_desc* desc, et_graph** out);

/* Two-stage split-K reduction ([ETN] §Split-K reduction 示例):
 *   Bpart[i,j] = sum_{k=chunk*j}^{chunk*j+chunk-1} A[i,k]   (j < ceil(cols/chunk))
 *   C[i]       = sum_j Bpart[i,j]
 * One task per (row tile i, chunk j) notifies E[i] ("ij->i"); the final
 * task of row tile i waits for E[i] ("i->i"), wait count = #chunks.
 * A: fp32 [n_rows, cols]; Bpart: fp32 [n_rows, nchunk]; C: fp32 [n_rows].
 * 0 <= n_rows <= max_T (n_rows = 0 launches nothing). */
et_status et_run_splitk(et_graph* g, const float* A, int n_rows, float* Bpart, float* C,
                        void* stream);

/* Measurement control, not part of the event-tensor runtime: the same
 * split-K reduction as two plain kernel launches on `stream` (all partials,
 * then all finals), i.e. kernel-per-operator execution, the baseline the
 * megakernel removes ([ETN] §背景: a launch costs several microseconds while
 * a small kernel runs about two).  A fp32 [n_rows, cols]; Bpart fp32
 * [n_rows, ceil(cols/chunk)]; C fp32 [n_rows].  Asynchronous; allocates
 * nothing.  ET_ERR_INVALID on bad sizes or null/misaligned pointers. */
et_status et_run_splitk_two_launch(const float* A, int n_rows, int cols, int chunk, float* Bpart, float* C,
                                   void* stream);

/* Fused decode MLP (RMSNorm -> gate/up GEMM -> SiLU*mul -> down GEMM) of
 * [ETN] §端到端低 batch serving ("Norm, MLP" of the decoding pipeline,
 * weights prefetched before activations arrive):
 *   xn = bf16(x * rsqrt(mean(x^2) + eps) * gamma)
 *   h  = bf16(silu(xn Wg^T) * (xn Wu^T))
 *   Y  = bf16(h Wd^T)                 (fp32 accumulation throughout)
 * X bf16 [B, hidden]; gamma bf16 [hidden]; Wgu bf16 [2*inter, hidden]
 * (gate rows first, then up rows); Wd bf16 [hidden, inter]; Y bf16
 * [B, hidden].  1 <= B <= max_T <= 128. */
et_status et_run_mlp(et_graph* g, int B, const uint16_t* X, const uint16_t* gamma,
                     const uint16_t* Wgu, const uint16_t* Wd, uint16_t* Y, void* stream);

/* MoE layer ([ETN] §Data-dependent event update, §Data-dependent task
 * triggering, §完整 MoE layer): router -> top-k -> token grouping ->
 * stage-1 grouped GEMM + SiLU*mul -> stage-2 grouped GEMM -> weighted
 * combine, in one launch.
 *   logits[t,e] = x_t . Wr_e + bias[e]           (fp32)
 *   topk[t,:]   = the top_k experts by logit, ties -> lower index, in order
 *   w[t,:]      = softmax of the selected logits  (fp32)
 *   h           = bf16(silu(x W1g_e^T) * (x W1u_e^T)),  o = h W2_e^T
 *   Y[t]        = bf16(sum_s w[t,s] * o[t,s])
 * X bf16 [T, hidden]; Wr bf16 [E, hidden]; bias fp32 [E]; W1 bf16
 * [E, 2*inter, hidden] (gate rows first); W2 bf16 [E, hidden, inter];
 * Y bf16 [T, hidden].  Optional outputs (NULL to skip): topk int32 [T,k],
 * topk_w fp32 [T,k], indptr int32 [E+1] (pairs per expert, CSR), perm int32
 * [T*k] (pairs t*k+s grouped by expert, ascending t), logits fp32 [T,E].
 * 1 <= T <= max_T. */
et_status et_run_moe(et_graph* g, int T, const uint16_t* X, const uint16_t* Wr, const float* bias,
                     const uint16_t* W1, const uint16_t* W2, uint16_t* Y, int32_t* topk,
                     float* topk_w, int32_t* indptr, int32_t* perm, float* logits, void* stream);

/* The MoE layer followed by a dense SwiGLU MLP on its output, in one launch
 * ([ETN] §端到端低 batch serving: the MoE GroupGEMM and the dense MLP GEMM
 * pipelined across stages; weights of the next stage prefetched before
 * its activations arrive).  Each combine task of the MoE also takes the
 * MLP's RMSNorm of its tokens, and the MLP's gate/up tasks stream their
 * weights while the MoE finishes:
 *   Y1 = the MoE layer of et_run_moe on X
 *   Y2 = bf16(h Wd^T),  h = bf16(silu(xn Wg^T) * (xn Wu^T)),  xn = bf16(rmsnorm(Y1) gamma)
 * MoE tensors as for et_run_moe; gamma bf16 [hidden]; Wgu bf16 [2 * mlp_inter,
 * hidden] (gate rows first); Wd bf16 [hidden, mlp_inter]; Y1, Y2 bf16 [T, hidden].
 * 1 <= T <= max_T <= 128. */
et_status et_run_moe_mlp(et_graph* g, int T, const uint16_t* X, const uint16_t* Wr, const float* bias,
                         const uint16_t* W1, const uint16_t* W2, const uint16_t* gamma, const uint16_t* Wgu,
                         const uint16_t* Wd, uint16_t* Y1, uint16_t* Y2, void* stream);

/* Weights of the decode layer (bf16 bits, device memory, row-major). */
typedef struct {
    const uint16_t* g1;    /* [hidden] attention rmsnorm weight */
    const uint16_t* Wqkv;  /* [(n_heads + 2 n_kv_heads) * head_dim, hidden]: query heads, key heads,
                              value heads */
    const uint16_t* gq;    /* [head_dim] per-head query rmsnorm weight */
    const uint16_t* gk;    /* [head_dim] per-head key rmsnorm weight */
    const uint16_t* Wo;    /* [hidden, n_heads * head_dim] */
    const uint16_t* g2;    /* [hidden] MLP rmsnorm weight */
    const uint16_t* Wgu;   /* [2 * inter, hidden]: gate rows, then up rows */
    const uint16_t* Wd;    /* [hidden, inter] */
} et_decode_weights;

/* One decode step of a transformer layer for B requests, each adding one
 * token ([ETN] §端到端低 batch serving: Attention, RoPE, KV-cache, Norm and
 * MLP in one megakernel; the Q branch (norm + RoPE) and the K branch
 * (norm + RoPE + cache append) run in parallel; weights of the next stage
 * are prefetched before its activations arrive; §Data-dependent task
 * triggering: request b's attention runs as ceil((pos[b] + 1) / dec_split)
 * split tasks, a run-time count).  Per request b at position p = pos[b]:
 *   xn  = bf16(rmsnorm(x) g1);  qkv = bf16(xn Wqkv^T)
 *   q_h = bf16(rope(rmsnorm(q_h) gq, p)),  k_g = bf16(rope(rmsnorm(k_g) gk, p))
 *   Kc[b,g,p,:] = k_g, Vc[b,g,:,p] = v_g      (written in place)
 *   o_h = softmax over j <= p of (q_h . Kc[b,g,j,:] / sqrt(head_dim)) . Vc[b,g,:,j],
 *         g = h / (n_heads / n_kv_heads)
 *   h1  = bf16(x + bf16(o) Wo^T)
 *   Y   = bf16(h1 + (bf16(silu(xn2 Wg^T) * (xn2 Wu^T))) Wd^T),  xn2 = bf16(rmsnorm(h1) g2)
 * RoPE pairs element i with element i + head_dim/2 at angle p * base^(-2i/head_dim).
 * X bf16 [B, hidden]; pos int32 [B] (device), 0 <= pos[b] < max_ctx, else the
 * run ends with ET_ERR_INVALID from et_sync_status; Kc bf16 [B, n_kv_heads,
 * max_ctx, head_dim] and Vc bf16 [B, n_kv_heads, head_dim, max_ctx] (V stored
 * transposed, positions contiguous: both attention products then read their
 * operands K-major on the tensor cores) (device, updated in place at pos[b]);
 * Y bf16 [B, hidden]; h1 (optional, NULL to skip) bf16 [B, hidden].
 * 1 <= B <= max_T <= 128. */
et_status et_run_decode(et_graph* g, int B, const uint16_t* X, const int32_t* pos, const et_decode_weights* w,
                        uint16_t* Kc, uint16_t* Vc, uint16_t* Y, uint16_t* h1, void* stream);

/* Split-K reduction without any device allocation.  (No counterpart in the
 * paper: this is an interface addition of this library.)
 *
 * Some callers cannot call cudaMalloc: a plugin running inside a host
 * framework that owns every device allocation and gives the plugin no
 * allocator, or a latency-critical path that cannot afford cudaMalloc's
 * implicit device synchronisation.  They cannot build an et_graph (its
 * workspace is allocated), so this entry point runs the same split-K
 * megakernel with its whole workspace -- event counters, ready queue and
 * control block -- in one file-scope device array of 108,032 bytes that
 * every GPU loading libet.so holds until the process exits.  It calls no
 * cudaMalloc, cudaFree or allocating library routine.
 *   - Same computation and arguments as et_run_splitk (A fp32 [n_rows, 128],
 *     chunk 32, Bpart fp32 [n_rows, 4], C fp32 [n_rows]), dynamic schedule.
 *   - 0 <= n_rows <= 65536; larger n_rows returns ET_ERR_INVALID before any
 *     CUDA call.  Null or misaligned pointers: ET_ERR_INVALID.
 *   - The first call on a device does a one-time set-up there (it resolves
 *     the array's device address and clears it with cudaMemsetAsync on
 *     `stream`); make that first call before any stream capture.
 *   - Synchronous: it waits for `stream`, then returns the device status of
 *     this call (ET_ERR_TIMEOUT if a wait gave up, after which the workspace
 *     is cleared again).
 *   - Every call on a device shares the one array, which keeps the last
 *     call's contents; calls that overlap on the GPU (other streams, other
 *     host threads) race on it and must not be issued. */
et_status et_run_splitk_noalloc(const float* A, int n_rows, float* Bpart, float* C, void* stream);

/* Synchronise `stream`, then read and clear the graph's sticky device
 * status.  Returns ET_OK, or the device error of a run since the last call:
 * ET_ERR_TIMEOUT if a wait gave up, ET_ERR_INTERNAL if a capacity check
 * failed (every CTA then drained and exited; no trap).  After a device
 * error the workspace (counters, scratch, the host mirror of the status)
 * is reset here, so the next run starts clean; until then et_run_* returns
 * ET_ERR_PENDING. */
et_status et_sync_status(et_graph* g, void* stream);

/* Copy the trace of the last run (ET_DEBUG_TRACE) to host memory.
 * Synchronises the device.  *n_records receives the record count; at most
 * bytes / sizeof(et_trace_record) records are copied. */
et_status et_get_trace(et_graph* g, void* host_buf, size_t bytes, int* n_records);

/* Every event of the last run's graph (for that run's T) with the number of
 * notifications it received ("Event Tensor：用“事件张量”编译动态 Megakernel",
 * §Event Tensor: a consumer runs once its event received its wait count).
 * Synchronises the device; call it after the run and before the next run of
 * the graph (which clears these counters).  At most `cap` records are
 * written to `buf` (host memory); *n_events receives the total number.
 * ET_ERR_INVALID if the graph has not run yet. */
et_status et_get_event_counts(et_graph* g, et_event_count* buf, int cap, int* n_events);

/* Tile parameters of a built graph. */
et_status et_get_info(const et_graph* g, et_graph_info* info);

/* Diagnostic words of the last device error (which wait, which task);
 * 8 ints.  Synchronises the device. */
et_status et_get_diag(et_graph* g, int32_t* out8);

void et_destroy_graph(et_graph* g);
const char* et_status_str(et_status s);

#ifdef __cplusplus
}
#endif
#endif /* ET_H_ */
