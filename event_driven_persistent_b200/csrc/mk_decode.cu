// Decode-layer megakernel: one decode step of a transformer layer for B
// requests (one new token each), in one launch, B at run time.
//
// "Event Tensor：用“事件张量”编译动态 Megakernel", §端到端低 batch serving:
// the decoding pipeline fuses Attention, RoPE, KV-cache, Norm and MLP; the
// Q branch (Norm + RoPE) and the K branch (Norm + RoPE + cache append) run
// in parallel; weights of the next stage are prefetched before its
// activations arrive.  §Data-dependent task triggering: the attention of
// request b is split into tasks[split_indptr[b] : split_indptr[b+1]], the
// split count following the request's run-time context length.
// §静态与动态调度的消融: regular dense stages favour the static schedule,
// irregular ones the dynamic schedule -- the hybrid schedule runs the dense
// GEMMs from static per-SM lists and the attention splits from the queue.
//
// Task graph (event counts in brackets):
//   N1(b)        x_b -> xn_b = bf16(rmsnorm(x_b) g1)                  -> E_n1 [B]
//   QKV(n, c)    head tile n (128 rows of Wqkv), K chunk c: partial sums
//                added at L2                                           -> E_qkv[n] [n_kc]
//                the chunk completing head n runs its branch inline:
//                  Q head:  bf16 -> per-head rmsnorm gq -> RoPE -> q
//                  K head:  bf16 -> per-head rmsnorm gk -> RoPE -> cache[b, g, pos_b]
//                  V head:  bf16 -> cache[b, g, pos_b]                 -> E_g[g] [grp + 2]
//   ATTN(b, g, s) keys [S s, S s + S) of request b (S = the split, 512 keys), KV head g, all grp
//                query heads, in stages of 128 keys on the tensor cores:
//                S = K Q^T (keys x heads), online softmax on the exec group,
//                O += V^T P^T (head dims x heads); partial (o, m, l)     -> E_att[b, g] [#splits(b)]
//                the split completing (b, g) merges the partials inline  -> E_ag[g] [B]
//   OPROJ(m, c)  output tile m, K chunk = the heads of KV group c, sums
//                added at L2                                           -> E_o [n_m * nkv]
//   N2(b)        h1 = bf16(x + o-proj), xn2 = bf16(rmsnorm(h1) g2)     -> E_n2 [B]
//   GU(n)        SwiGLU gate/up tile n (SiLU*mul epilogue)            -> E_h[c] [kchunk / 64]
//   DOWN(m, c)   output tile m, K chunk c, sums added at L2           -> E_y[m] [#chunks]
//   RED(m)       Y = bf16(h1 + down) for tile m
#include "et_math.cuh"
#include "et_params.h"

namespace et {

constexpr int kKeysPerStage = 128;  // keys of one attention stage (the M of S = K Q^T)

struct Decode : WorkloadBase {
    using Params = DecodeParams;
    static constexpr bool kGemm = true;
    static constexpr bool kStream = true;

    __device__ static bool unfused(const Params& p) { return p.sched == ET_SCHED_UNFUSED; }
    __device__ static bool push_all(const Params& p) { return p.sched == ET_SCHED_DYNAMIC; }
    __device__ static bool push_attn(const Params& p) {
        return p.sched == ET_SCHED_DYNAMIC || p.sched == ET_SCHED_HYBRID;
    }
    __device__ static int n_split(const Params& p, int pos) { return (pos + 1 + p.split - 1) / p.split; }
    __device__ static int tok_n(const Params& p) { return (p.B + 15) & ~15; }

    __device__ static uint32_t fetch_init(const Params&, int idx) { return task_word(ET_OP_DEC_NORM1, idx, 0); }

    __device__ static bool derive(const Params& p, Ctx& x, TaskDesc& d) {
        const int op = task_op(d.word), a = task_a(d.word), b = task_b(d.word);
        d.valid = 1;
        d.gemm = 0;
        if (op == ET_OP_DEC_NORM1 || op == ET_OP_DEC_NORM2) {
            d.valid = a < p.B;
        } else if (op == ET_OP_DEC_QKV) {
            d.gemm = 1;
            d.a_map = DEC_MAP_WQKV;
            d.a_row0 = a * p.hd;
            d.a_row1 = a * p.hd + 64;
            d.b_map = DEC_MAP_XN;
            d.b_row0 = 0;
            d.n = tok_n(p);
            // K chunk b: stages [b kt / n_kc, (b + 1) kt / n_kc) of the kt
            const int kt = p.hidden / kTileK, s0 = b * kt / p.n_kc;
            d.k0 = s0 * kTileK;
            d.nk = (b + 1) * kt / p.n_kc - s0;
        } else if (op == ET_OP_DEC_ATTN) {
            const int bb = a / p.nkv, g = a % p.nkv, s = b;
            d.valid = 0;
            if (bb >= p.B) return true;
            const int pos = __ldg(p.pos + bb);
            if (pos < 0 || pos >= p.max_ctx) return true;  // N1 reports the bad position
            if (s >= n_split(p, pos)) return true;
            const int key0 = s * p.split, nkeys = min(p.split, pos + 1 - key0);
            d.valid = 1;
            d.stream = 1;
            d.attn = 1;
            d.sbytes = kAttnStage;
            d.nk = (nkeys + kKeysPerStage - 1) / kKeysPerStage;
            d.p[0] = bb;
            d.p[1] = g;
            d.p[2] = s;
            d.p[3] = pos;
            d.p[4] = key0;
            d.p[5] = nkeys;
        } else if (op == ET_OP_DEC_OPROJ) {
            d.gemm = 1;
            d.a_map = DEC_MAP_WO;
            d.a_row0 = a * 128;
            d.a_row1 = a * 128 + 64;
            d.b_map = DEC_MAP_ATTN;
            d.b_row0 = 0;
            d.n = tok_n(p);
            d.k0 = b * p.o_kc;
            d.nk = p.o_kc / kTileK;
        } else if (op == ET_OP_DEC_GATEUP) {
            d.gemm = 1;
            d.a_map = DEC_MAP_WGU;
            d.a_row0 = a * p.gu_tile;
            d.a_row1 = p.inter + a * p.gu_tile;
            d.b_map = DEC_MAP_XN2;
            d.b_row0 = 0;
            d.n = tok_n(p);
            d.k0 = 0;
            d.nk = p.hidden / kTileK;
        } else if (op == ET_OP_DEC_DOWN) {
            d.gemm = 1;
            d.a_map = DEC_MAP_WD;
            d.a_row0 = a * 128;
            d.a_row1 = a * 128 + 64;
            d.b_map = DEC_MAP_HM;
            d.b_row0 = 0;
            d.n = tok_n(p);
            d.k0 = b * p.kchunk;
            d.nk = p.kchunk / kTileK;
        }
        return true;
    }

    __device__ static const uint16_t* gather_row(const Params&, const TaskDesc&, int) { return nullptr; }

    // The input wait of a tensor-core or stream task (warp 0, after its
    // weight / cached-key prefetch).
    __device__ static bool gemm_wait(const Params& p, Ctx& x, TaskDesc& d) {
        const int op = task_op(d.word), a = task_a(d.word), b = task_b(d.word);
        if (op == ET_OP_DEC_QKV) return wait_geq(x.ctr + p.ev_n1, p.B + p.bad_count, x.ctl, x.timeout_ns, 300, 0);
        if (op == ET_OP_DEC_ATTN) {
            if (unfused(p)) return wait_geq(x.ctr + p.ev_branch_all, p.n_heads, x.ctl, x.timeout_ns, 301, 0);
            const int g = a % p.nkv;
            return wait_geq(x.ctr + p.ev_g + g, p.grp + 2, x.ctl, x.timeout_ns, 302, g);
        }
        if (op == ET_OP_DEC_OPROJ) {
            if (unfused(p)) return wait_geq(x.ctr + p.ev_merge_all, p.B * p.nkv, x.ctl, x.timeout_ns, 303, 0);
            return wait_geq(x.ctr + p.ev_ag + b, p.B, x.ctl, x.timeout_ns, 304, b);
        }
        if (op == ET_OP_DEC_GATEUP) return wait_geq(x.ctr + p.ev_n2, p.B, x.ctl, x.timeout_ns, 305, 0);
        // DOWN
        if (unfused(p)) return wait_geq(x.ctr + p.ev_gu_all, p.n_gu, x.ctl, x.timeout_ns, 306, 0);
        return wait_geq(x.ctr + p.ev_h + b, p.gu_per_chunk, x.ctl, x.timeout_ns, 307, b);
    }

    __device__ static const CUtensorMap* a_map(const Params& p, int id) {
        return id == DEC_MAP_WQKV ? &p.tm_wqkv : (id == DEC_MAP_WO ? &p.tm_wo : (id == DEC_MAP_WGU ? &p.tm_wgu : &p.tm_wd));
    }
    __device__ static const CUtensorMap* b_map(const Params& p, int id) {
        return id == DEC_MAP_XN ? &p.tm_xn : (id == DEC_MAP_ATTN ? &p.tm_attn : (id == DEC_MAP_XN2 ? &p.tm_xn2 : &p.tm_hm));
    }
    __device__ static const CUtensorMap* b_map_wide(const Params& p, int id) {
        if (!p.wide_b) return nullptr;
        return id == DEC_MAP_XN ? &p.tm_xn64
                                : (id == DEC_MAP_ATTN ? &p.tm_attn64 : (id == DEC_MAP_XN2 ? &p.tm_xn2_64 : &p.tm_hm64));
    }

    // ------------------------------------------------------------ stream
    // Stages of an attention split whose keys were cached before this step
    // (all but the stage holding the new token) are copied before the wait.
    __device__ static int stream_prefetch(const Params&, const TaskDesc& d) {
        const int pos = d.p[3], key0 = d.p[4], nkeys = d.p[5];
        if (key0 + nkeys <= pos) return d.nk;  // the new key is in a later split
        return (pos - key0) / kKeysPerStage;   // stages before the one holding key `pos`
    }
    __device__ static int stage_keys(const TaskDesc& d, int st) { return min(kKeysPerStage, d.p[5] - st * kKeysPerStage); }
    // A stage: K rows [key, key + 128) of (b, g) (cache rows beyond the
    // request's keys are masked), the V^T columns of the same keys (columns
    // beyond them are zeroed in smem before use), and the grp query rows of
    // (b, g) (16-row box: rows past grp only feed unused S columns).  Full
    // boxes always land (out-of-range rows and columns are filled with 0).
    __device__ static uint32_t stream_bytes(const Params&, const TaskDesc&, int) { return kAttnStage; }
    __device__ static void stream_copy(const Params& p, const TaskDesc& d, int st, uint8_t* dst, uint64_t* bar,
                                       uint64_t pol, bool late) {
        const int bb = d.p[0], g = d.p[1], key = d.p[4] + st * kKeysPerStage;
        const int krow = (bb * p.nkv + g) * p.max_ctx + key, vrow = (bb * p.nkv + g) * p.hd;
#pragma unroll
        for (int at = 0; at < 2; ++at) {
            tma_load_2d(dst + at * kAAtomBytes, &p.tm_kc, bar, at * kAtomK, krow, pol);
            tma_load_2d(dst + kAttnVOff + at * kAAtomBytes, &p.tm_vt, bar, key + at * kAtomK, vrow, pol);
        }
        if (late) stream_late(p, d, st, dst, bar, pol);
    }
    __device__ static void stream_late(const Params& p, const TaskDesc& d, int, uint8_t* dst, uint64_t* bar,
                                       uint64_t pol) {
        const int qrow = d.p[0] * p.nq + d.p[1] * p.grp;
#pragma unroll
        for (int at = 0; at < 2; ++at) tma_load_2d(dst + kAttnQOff + at * 16 * 128, &p.tm_q, bar, at * kAtomK, qrow, pol);
    }

    // One attention split (exec group; the MMA warp runs the products).
    // Per stage of 128 keys: thread r (its warp's TMEM lane) reads the scores
    // of key r for every query head from S, the group takes the stage max and
    // the online-softmax rescale; then it folds the previous stage's O (head
    // dim r of every head) while the next stage's S is computed, writes P =
    // bf16(exp(s - max)) (query heads x keys, the 128-byte swizzled K-major
    // layout of a tensor-core B operand) and, on a partial stage, zeroes the
    // V^T columns of the missing keys.  The normaliser sums the bf16
    // probabilities the product used.
    __device__ static bool stream_exec(const Params& p, Ctx& x, TaskDesc& d) {
        const int bb = d.p[0], g = d.p[1], s = d.p[2];
        const int w = x.tid >> 5, lane = x.tid & 31;
        const int r = ((w + kExecWarp0) & 3) * 32 + lane;
        const int grp = p.grp;
        uint8_t* P0 = reinterpret_cast<uint8_t*>(x.epi);  // 2 x [2 key atoms][16 rows][128 B]
        float* red = x.epi + 2048;                           // [max: 4 warps x 4 heads][sum: same]
        for (int i = x.tid; i < 2048; i += kExecThreads)    // query-head rows grp..15 of both P stay 0
            if (((i >> 5) & 15) >= grp) reinterpret_cast<uint32_t*>(P0)[i] = 0u;
        const float scale = 0.08838834764831845f;  // 1 / sqrt(128)
        float m[4], l[4], o[4], alpha_prev[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            m[h] = -INFINITY;
            l[h] = 0.f;
            o[h] = 0.f;
            alpha_prev[h] = 0.f;
        }
        // fold O of attention stage k into o with that stage's rescale
        // (broadcast slot 3 inside the loop; 5 for the last fold, which follows
        // the loop's last fold with no exec-group barrier in between)
        auto fold = [&](uint32_t k, int slot) -> bool {
            if (!exec_mbar_wait(x, &x.sc->o_full[k & 1], (k >> 1) & 1, 317, slot)) return false;
            tc_fence_after();
            float ov[4];
            __syncwarp();
            tmem_ld4_wait(x.taddr + 32u + 16u * (k & 1), ov);
#pragma unroll
            for (int h = 0; h < 4; ++h) o[h] = o[h] * alpha_prev[h] + ov[h];
            return true;
        };
        StageAlloc al = stream_alloc(d);
        for (int st = 0; st < d.nk; ++st) {
            const uint32_t off = al.next(d.sbytes), k = x.na + (uint32_t)st;
            const int nks = stage_keys(d, st);
            uint8_t* P = P0 + 4096 * (k & 1);
            if (!exec_mbar_wait(x, &x.sc->s_full[k & 1], (k >> 1) & 1, 316, 2)) return false;
            tc_fence_after();
            float sv[4];
            __syncwarp();
            tmem_ld4_wait(x.taddr + 16u * (k & 1), sv);
            const bool valid = r < nks;
            float mx[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                sv[h] = (valid && h < grp) ? sv[h] * scale : -INFINITY;
                mx[h] = sv[h];
#pragma unroll
                for (int o2 = 16; o2 > 0; o2 >>= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o2));
            }
            if (lane == 0)
#pragma unroll
                for (int h = 0; h < 4; ++h) red[w * 4 + h] = mx[h];
            exec_bar();
            float alpha[4], ps[4];
            uint16_t pb[4] = {0, 0, 0, 0};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                float pv = 0.f;
                alpha[h] = 1.f;
                if (h < grp) {
                    const float mn = fmaxf(m[h], fmaxf(fmaxf(red[h], red[4 + h]), fmaxf(red[8 + h], red[12 + h])));
                    alpha[h] = expf(m[h] - mn);  // 0 on the first stage (m = -inf)
                    m[h] = mn;
                    if (valid) {
                        pb[h] = bf16_bits(expf(sv[h] - mn));
                        pv = bf16_val(pb[h]);
                    }
                }
                ps[h] = pv;
#pragma unroll
                for (int o2 = 16; o2 > 0; o2 >>= 1) ps[h] += __shfl_xor_sync(0xffffffffu, ps[h], o2);
            }
#pragma unroll
            for (int h = 0; h < 4; ++h)
                if (h < grp)
                    *reinterpret_cast<uint16_t*>(P + (r >> 6) * 2048 + h * 128 + ((((r & 63) >> 3) ^ (h & 7)) << 4) +
                                                 (r & 7) * 2) = pb[h];
            if (nks < kKeysPerStage) {
                // V^T row r (head dim r): the columns of keys nks..127 to 0,
                // after the stage's copies landed (that phase is already
                // complete: the MMA warp waited on it before S)
                const uint32_t gs = d.st0 + (uint32_t)st;
                if (!exec_mbar_wait(x, &x.sc->full[gs % kSlots], (gs / kSlots) & 1, 318, 5)) return false;
                uint8_t* vr = x.arena + off + kAttnVOff + r * 128;
                for (int kk = nks; kk < kKeysPerStage; ++kk)
                    *reinterpret_cast<uint16_t*>(vr + (kk >> 6) * kAAtomBytes + ((((kk & 63) >> 3) ^ (r & 7)) << 4) +
                                                 (kk & 7) * 2) = 0;
            }
            if (lane == 0)
#pragma unroll
                for (int h = 0; h < 4; ++h) red[16 + w * 4 + h] = ps[h];
            fence_proxy_async_smem();  // P and the zeroed V^T columns are read by the tensor core
            tc_fence_before();
            exec_bar();
            if (x.tid == 0) mbar_arrive(&x.sc->p_full[k & 1]);
            // the previous stage's O, while this stage's product runs (its
            // P buffer is then free for the stage after)
            if (st > 0 && !fold(k - 1, 3)) return false;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                l[h] = l[h] * alpha[h] + red[16 + h] + red[20 + h] + red[24 + h] + red[28 + h];
                alpha_prev[h] = alpha[h];
            }
        }
        if (!fold(x.na + (uint32_t)d.nk - 1, 5)) return false;
        x.na += (uint32_t)d.nk;
        acc_release(x.acc_empty);
        const int tid = r;  // head dim of this thread
        // partial of this split: o (unnormalised), running max m, sum l
        const int stride = p.hd + 2;
        float* pp = p.part + ((size_t)(bb * p.nkv + g) * p.s_max + s) * grp * stride;
#pragma unroll
        for (int h = 0; h < 4; ++h)
            if (h < grp) {
                pp[h * stride + tid] = o[h];
                if (tid == 0) {
                    pp[h * stride + p.hd] = m[h];
                    pp[h * stride + p.hd + 1] = l[h];
                }
            }
        const int ns = n_split(p, d.p[3]);
        if (!group_finish_notify(x, d, x.ctr + p.ev_att + bb * p.nkv + g, 1, ns)) return true;
        return merge(p, x, d, bb, g, ns);
    }

    // MERGE(b, g), run by the split that completed E_att[b, g]: combine the
    // splits' partials into the attention output of the group's heads.
    __device__ static bool merge(const Params& p, Ctx& x, const TaskDesc& d0, int bb, int g, int ns) {
        TaskDesc d = d0;
        d.word = task_word(ET_OP_DEC_MERGE, bb * p.nkv + g, 0);
        d.t_fetch = d.t_acc = 0;
        if (x.debug & ET_DEBUG_TRACE) d.t_fetch = globaltimer();
        if (!group_wait(x, d, nullptr, 0, 310)) return false;
        const int tid = x.tid, stride = p.hd + 2;
        const float* base = p.part + (size_t)(bb * p.nkv + g) * p.s_max * p.grp * stride;
        // every split's (max, sum) of every head at once into smem: wgt[s][h]
        // = exp(m_s - m*) and the normaliser 1 / sum_s wgt l_s
        float* ml = x.epi;                 // [s_max * grp][2]
        float* wgt = x.epi + 2 * 1024;     // [s_max * grp]
        float* inv = wgt + 1024;           // [grp]
        const int nsh = ns * p.grp;
        for (int i = tid; i < nsh; i += kExecThreads) {
            const float* q = base + (size_t)i * stride + p.hd;  // i = s * grp + h
            ml[2 * i] = __ldcg(q);
            ml[2 * i + 1] = __ldcg(q + 1);
        }
        exec_bar();
        if (tid < p.grp) {
            float ms = -INFINITY;
            for (int s = 0; s < ns; ++s) ms = fmaxf(ms, ml[2 * (s * p.grp + tid)]);
            float ls = 0.f;
            for (int s = 0; s < ns; ++s) {
                const float w8 = expf(ml[2 * (s * p.grp + tid)] - ms);
                wgt[s * p.grp + tid] = w8;
                ls = fmaf(w8, ml[2 * (s * p.grp + tid) + 1], ls);
            }
            inv[tid] = 1.0f / ls;
        }
        exec_bar();
        // thread t = dim t: the splits' partial outputs of every head, eight
        // splits' loads issued together before their sums
        float os[4] = {0.f, 0.f, 0.f, 0.f};
        for (int s0 = 0; s0 < ns; s0 += 8) {
            float v[8][4];
#pragma unroll
            for (int s = 0; s < 8; ++s)
#pragma unroll
                for (int h = 0; h < 4; ++h)
                    v[s][h] = (s0 + s < ns && h < p.grp) ? __ldcg(base + ((size_t)(s0 + s) * p.grp + h) * stride + tid)
                                                         : 0.f;
#pragma unroll
            for (int s = 0; s < 8; ++s)
#pragma unroll
                for (int h = 0; h < 4; ++h)
                    if (s0 + s < ns && h < p.grp) os[h] = fmaf(wgt[(s0 + s) * p.grp + h], v[s][h], os[h]);
        }
#pragma unroll
        for (int h = 0; h < 4; ++h)
            if (h < p.grp) p.attn[(size_t)bb * p.nq * p.hd + (size_t)(g * p.grp + h) * p.hd + tid] = bf16_bits(os[h] * inv[h]);
        fence_proxy_async_global();  // attn is read by TMA in the o-proj tasks
        int* ev = x.ctr + (unfused(p) ? p.ev_merge_all : p.ev_ag + g);
        const int tgt = unfused(p) ? p.B * p.nkv : p.B;
        if (group_finish_notify(x, d, ev, 1, tgt) && push_all(p))
            group_push(x, p.n_m, [&](int m) { return task_word(ET_OP_DEC_OPROJ, m, g); });
        return true;
    }

    // ------------------------------------------------------------ branches
    // Q head n, K head (n - nq) or V head (n - nq - nkv), all B tokens, from
    // the head's K-chunk sums.  Run by the QKV task that completed E_qkv[n].
    // Warp w takes tokens w, w + 4, ...; lane l holds dims 4l..4l+3, so the
    // per-head RMSNorm is a warp reduction and the rotate-half partner of
    // dim i (i + 64) sits in lane l ^ 16: no exec-group barrier.
    __device__ static bool branch(const Params& p, Ctx& x, const TaskDesc& d0, int n) {
        const int kind = n < p.nq ? 0 : (n < p.nq + p.nkv ? 1 : 2);
        const int g = kind == 0 ? n / p.grp : (kind == 1 ? n - p.nq : n - p.nq - p.nkv);
        TaskDesc d = d0;
        d.word = task_word(kind == 0 ? ET_OP_DEC_QBR : (kind == 1 ? ET_OP_DEC_KBR : ET_OP_DEC_VBR), n, 0);
        d.t_fetch = d.t_acc = 0;
        if (x.debug & ET_DEBUG_TRACE) d.t_fetch = globaltimer();
        if (!group_wait(x, d, nullptr, 0, 311)) return false;
        const int w = x.tid >> 5, lane = x.tid & 31, d4 = lane * 4;
        const size_t stride = (size_t)p.n_heads * p.hd;
        float gam[4] = {1.f, 1.f, 1.f, 1.f};
        if (kind < 2) bf16x4(*reinterpret_cast<const uint2*>((kind == 0 ? p.gq : p.gk) + d4), gam);
        for (int b = w; b < p.B; b += kExecThreads / 32) {
            float* acc = p.qkvacc + (size_t)b * stride + (size_t)n * p.hd + d4;
            const float4 a4 = __ldcg(reinterpret_cast<const float4*>(acc));
            __stcg(reinterpret_cast<float4*>(acc), make_float4(0.f, 0.f, 0.f, 0.f));
            float y[4] = {bf16_val(bf16_bits(a4.x)), bf16_val(bf16_bits(a4.y)), bf16_val(bf16_bits(a4.z)),
                          bf16_val(bf16_bits(a4.w))};  // the qkv tensor is bf16
            const int pos = __ldg(p.pos + b);
            if (pos < 0 || pos >= p.max_ctx) continue;  // N1 reports the bad position
            if (kind == 2) {  // V^T cache: [b][g][dim][position]
                uint16_t* vc = p.Vc + (((size_t)b * p.nkv + g) * p.hd + d4) * p.max_ctx + pos;
#pragma unroll
                for (int e = 0; e < 4; ++e) vc[(size_t)e * p.max_ctx] = bf16_bits(y[e]);
                continue;
            }
            float ss = y[0] * y[0] + y[1] * y[1] + y[2] * y[2] + y[3] * y[3];
#pragma unroll
            for (int o2 = 16; o2 > 0; o2 >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o2);
            const float inv = 1.0f / sqrtf(ss / (float)p.hd + p.eps);
            float other[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                y[e] = y[e] * inv * gam[e];
                other[e] = __shfl_xor_sync(0xffffffffu, y[e], 16);
            }
            // (cos, sin) of frequencies (d4 & 63) .. +3 at this position
            const float4* cs = reinterpret_cast<const float4*>(p.rope + (size_t)b * (p.hd / 2) + (d4 & 63));
            const float4 c01 = __ldcg(cs), c23 = __ldcg(cs + 1);
            const float cv[4] = {c01.x, c01.z, c23.x, c23.z}, sv[4] = {c01.y, c01.w, c23.y, c23.w};
            ushort4 o;
            uint16_t* oo = reinterpret_cast<uint16_t*>(&o);
#pragma unroll
            for (int e = 0; e < 4; ++e)
                oo[e] = bf16_bits(lane < 16 ? y[e] * cv[e] - other[e] * sv[e] : y[e] * cv[e] + other[e] * sv[e]);
            if (kind == 0) {
                const size_t qi = ((size_t)b * p.nq + n) * p.hd + d4;
                *reinterpret_cast<ushort4*>(p.q + qi) = o;
                if (p.out_q) *reinterpret_cast<ushort4*>(p.out_q + qi) = o;
            } else {
                *reinterpret_cast<ushort4*>(p.Kc + (((size_t)b * p.nkv + g) * p.max_ctx + pos) * p.hd + d4) = o;
            }
        }
        fence_proxy_async_global();  // the caches and q are read by TMA in the attention tasks
        int* ev = x.ctr + (unfused(p) ? p.ev_branch_all : p.ev_g + g);
        const int tgt = unfused(p) ? p.n_heads : p.grp + 2;
        if (group_finish_notify(x, d, ev, 1, tgt) && push_attn(p) && !unfused(p)) push_splits(p, x, g);
        return true;
    }

    // Queue the attention splits of KV head g: tasks[split_indptr[b] :
    // split_indptr[b+1]] for every request b (the split counts follow the
    // run-time positions), and publish the queue's total.
    __device__ static void push_splits(const Params& p, Ctx& x, int g) {
        int* tmp = reinterpret_cast<int*>(x.simt);
        const int b = x.tid;
        int ns = 0;
        if (b < p.B) {
            const int pos = __ldg(p.pos + b);
            ns = (pos >= 0 && pos < p.max_ctx) ? n_split(p, pos) : 0;
        }
        int tot;
        const int off = exec_scan(ns, x.tid, tmp, &tot);
        if (x.tid == 0) x.sc->bcast[0] = q_reserve(x.q, tot);
        exec_bar();
        const int base = x.sc->bcast[0];
        __threadfence();
        for (int s = 0; s < ns; ++s) q_publish_after_fence(x.q, base + off + s, task_word(ET_OP_DEC_ATTN, b * p.nkv + g, s));
        if (x.tid == 0) {
            // every group pushes the same number of splits
            int total = p.nkv * tot;
            if (push_all(p))
                total += p.B + p.n_heads * p.n_kc + p.n_m * p.nkv + p.B + p.n_gu + p.n_m * p.n_c + p.n_m;
            atomicExch(x.ctr + kCtrTotal, total + 1);
        }
        exec_bar();
    }

    // --------------------------------------------------------- epilogues
    __device__ static bool epilogue(const Params& p, Ctx& x, TaskDesc& d, uint32_t taddr, uint64_t* acc_empty) {
        const int op = task_op(d.word), a = task_a(d.word), c = task_b(d.word);
        const int w = x.tid >> 5, lane = x.tid & 31;
        const int q = (w + kExecWarp0) & 3;
        const int r = q * 32 + lane;
        if (op == ET_OP_DEC_QKV || op == ET_OP_DEC_OPROJ || op == ET_OP_DEC_DOWN) {
            // add the partial tile at L2: row r of the weight tile = column of the output
            float* dst;
            size_t stride;
            if (op == ET_OP_DEC_QKV) {
                dst = p.qkvacc + (size_t)a * p.hd + r;
                stride = (size_t)p.n_heads * p.hd;
            } else {
                dst = (op == ET_OP_DEC_OPROJ ? p.h1acc : p.yacc) + (size_t)a * 128 + r;
                stride = p.hidden;
            }
            for (int c0 = 0; c0 < d.n; c0 += 16) {
                float v[16];
                acc_load16(taddr, c0, v);
                if (c0 + 16 >= d.n) acc_release(acc_empty);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (c0 + i < p.B) red_add(dst + (size_t)(c0 + i) * stride, v[i]);
            }
            if (op == ET_OP_DEC_QKV) {
                if (!group_finish_notify(x, d, x.ctr + p.ev_qkv + a, 1, p.n_kc)) return true;
                return branch(p, x, d, a);
            }
            if (op == ET_OP_DEC_OPROJ) {
                const int tgt = p.n_m * p.nkv;
                if (group_finish_notify(x, d, x.ctr + p.ev_o, 1, tgt) && push_all(p))
                    group_push(x, p.B, [&](int b) { return task_word(ET_OP_DEC_NORM2, b, 0); });
                return true;
            }
            int* ev = x.ctr + (unfused(p) ? p.ev_down_all : p.ev_y + a);
            const int tgt = unfused(p) ? p.n_m * p.n_c : p.n_c;
            if (group_finish_notify(x, d, ev, 1, tgt) && push_all(p))
                group_push(x, 1, [&](int) { return task_word(ET_OP_DEC_RED, a, 0); });
            return true;
        }
        // GU: rows 0..63 gate, 64..127 up, of intermediate columns a*64 + (r & 63)
        for (int c0 = 0; c0 < d.n; c0 += 16)
            swiglu_tokens16(x, taddr, c0, d.n, acc_empty, p.hm + (size_t)c0 * p.inter + a * p.gu_tile, p.inter,
                            p.B - c0);
        fence_proxy_async_global();  // hm is read by TMA in the down tasks
        const int cc = (a * p.gu_tile) / p.kchunk;
        int* ev = x.ctr + (unfused(p) ? p.ev_gu_all : p.ev_h + cc);
        const int tgt = unfused(p) ? p.n_gu : p.gu_per_chunk;
        if (group_finish_notify(x, d, ev, 1, tgt) && push_all(p))
            group_push(x, p.n_m, [&](int m) { return task_word(ET_OP_DEC_DOWN, m, cc); });
        return true;
    }

    // ---------------------------------------------------------- CUDA-core
    __device__ static bool simt(const Params& p, Ctx& x, TaskDesc& d) {
        const int op = task_op(d.word), a = task_a(d.word);
        if (op == ET_OP_DEC_NORM1) return norm1(p, x, d, a);
        if (op == ET_OP_DEC_NORM2) return norm2(p, x, d, a);
        return reduce(p, x, d, a);
    }

    // rmsnorm of a bf16 row held as 32 fp32 values per thread (hidden <= 4096)
    __device__ static float row_inv_rms(const Params& p, Ctx& x, const float* v, int nv) {
        float* red = reinterpret_cast<float*>(x.simt);
        float ss = 0.f;
        for (int i = 0; i < nv; ++i) ss += v[i] * v[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if ((x.tid & 31) == 0) red[x.tid >> 5] = ss;
        exec_bar();
        const float tot = red[0] + red[1] + red[2] + red[3];
        exec_bar();
        return 1.0f / sqrtf(tot / (float)p.hidden + p.eps);
    }

    __device__ static bool norm1(const Params& p, Ctx& x, TaskDesc& d, int b) {
        if (!group_wait(x, d, nullptr, 0, 312)) return false;
        {
            // the request's rotary (cos, sin) per frequency, for the Q and K
            // branches: angle pos * base^(-2i / head_dim), in double
            const int pos = __ldg(p.pos + b);
            if (pos < 0 || pos >= p.max_ctx) {
                if (x.tid == 0) fail(x.ctl, ET_ERR_INVALID, 313, b, pos, p.max_ctx);
            } else if (x.tid < p.hd / 2) {
                const double inv_freq = exp(-2.0 * (double)x.tid / (double)p.hd * log(p.rope_base));
                double sn, cs;
                sincos((double)pos * inv_freq, &sn, &cs);
                p.rope[(size_t)b * (p.hd / 2) + x.tid] = make_float2((float)cs, (float)sn);
            }
        }
        const uint16_t* xr = p.X + (size_t)b * p.hidden;
        float v[32];
        const int nv = p.hidden / kExecThreads;  // <= 32
        for (int i = 0; i < nv; i += 8) bf16x8(*reinterpret_cast<const uint4*>(xr + x.tid * nv + i), v + i);
        const float inv = row_inv_rms(p, x, v, nv);
        uint16_t* out = p.xn + (size_t)b * p.hidden + x.tid * nv;
        for (int i = 0; i < nv; i += 8) {
            uint4 gm = *reinterpret_cast<const uint4*>(p.g1 + x.tid * nv + i);
            float gg[8];
            bf16x8(gm, gg);
            uint4 o;
            uint16_t* oo = reinterpret_cast<uint16_t*>(&o);
#pragma unroll
            for (int t = 0; t < 8; ++t) oo[t] = bf16_bits(v[i + t] * inv * gg[t]);
            *reinterpret_cast<uint4*>(out + i) = o;
        }
        fence_proxy_async_global();  // xn is read by TMA in the QKV tasks
        if (group_finish_notify(x, d, x.ctr + p.ev_n1, 1, p.B) && push_all(p))
            group_push(x, p.n_heads * p.n_kc,
                       [&](int i) { return task_word(ET_OP_DEC_QKV, i / p.n_kc, i % p.n_kc); });
        return true;
    }

    // N2(b): h1 = bf16(x + o-proj) (the attention block's residual output),
    // xn2 = bf16(rmsnorm(h1) g2); the o-proj sums of row b back to zero.
    __device__ static bool norm2(const Params& p, Ctx& x, TaskDesc& d, int b) {
        const int tgt = p.n_m * p.nkv;
        if (!group_wait(x, d, x.ctr + p.ev_o, tgt, 314)) return false;
        // thread t holds elements (j * 128 + t) * 8 .. +7, j < hidden / 1024:
        // every load issued before the stores
        const int nv = p.hidden / kExecThreads, n8 = nv / 8;  // n8 <= 4
        const size_t row = (size_t)b * p.hidden;
        float4 a[8];
        uint4 xv[4];
        float v[32];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (j < n8) {
                const size_t e = row + (size_t)(j * kExecThreads + x.tid) * 8;
                a[2 * j] = __ldcg(reinterpret_cast<const float4*>(p.h1acc + e));
                a[2 * j + 1] = __ldcg(reinterpret_cast<const float4*>(p.h1acc + e + 4));
                xv[j] = *reinterpret_cast<const uint4*>(p.X + e);
            }
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (j < n8) {
                const size_t e = row + (size_t)(j * kExecThreads + x.tid) * 8;
                __stcg(reinterpret_cast<float4*>(p.h1acc + e), make_float4(0.f, 0.f, 0.f, 0.f));
                __stcg(reinterpret_cast<float4*>(p.h1acc + e + 4), make_float4(0.f, 0.f, 0.f, 0.f));
                float xf[8];
                bf16x8(xv[j], xf);
                const float av[8] = {a[2 * j].x, a[2 * j].y, a[2 * j].z, a[2 * j].w,
                                     a[2 * j + 1].x, a[2 * j + 1].y, a[2 * j + 1].z, a[2 * j + 1].w};
                uint4 o;
                uint16_t* oo = reinterpret_cast<uint16_t*>(&o);
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    oo[t] = bf16_bits(xf[t] + av[t]);
                    v[j * 8 + t] = bf16_val(oo[t]);
                }
                *reinterpret_cast<uint4*>(p.h1 + e) = o;
                if (p.out_h1) *reinterpret_cast<uint4*>(p.out_h1 + e) = o;
            }
        const float inv = row_inv_rms(p, x, v, nv);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (j < n8) {
                const size_t c = (size_t)(j * kExecThreads + x.tid) * 8;
                float gg[8];
                bf16x8(*reinterpret_cast<const uint4*>(p.g2 + c), gg);
                uint4 o;
                uint16_t* oo = reinterpret_cast<uint16_t*>(&o);
#pragma unroll
                for (int t = 0; t < 8; ++t) oo[t] = bf16_bits(v[j * 8 + t] * inv * gg[t]);
                *reinterpret_cast<uint4*>(p.xn2 + row + c) = o;
            }
        fence_proxy_async_global();  // xn2 is read by TMA in the gate/up tasks
        if (group_finish_notify(x, d, x.ctr + p.ev_n2, 1, p.B) && push_all(p))
            group_push(x, p.n_gu, [&](int n) { return task_word(ET_OP_DEC_GATEUP, n, 0); });
        return true;
    }

    // RED(m): Y = bf16(h1 + down) for output columns [128 m, 128 m + 128).
    __device__ static bool reduce(const Params& p, Ctx& x, TaskDesc& d, int m) {
        int* ev = x.ctr + (unfused(p) ? p.ev_down_all : p.ev_y + m);
        const int tgt = unfused(p) ? p.n_m * p.n_c : p.n_c;
        if (!group_wait(x, d, ev, tgt, 315)) return false;
        // B tokens x 128 columns as float4: eight loads in flight per thread
        // before its stores
        const int nv = 128 / 4, total = p.B * nv;
        for (int base = x.tid; base < total; base += kExecThreads * 8) {
            float4 v[8];
            uint2 hv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = base + u * kExecThreads;
                if (i < total) {
                    const size_t off = (size_t)(i / nv) * p.hidden + m * 128 + (i % nv) * 4;
                    v[u] = __ldcg(reinterpret_cast<const float4*>(p.yacc + off));
                    hv[u] = __ldcg(reinterpret_cast<const uint2*>(p.h1 + off));
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = base + u * kExecThreads;
                if (i < total) {
                    const size_t off = (size_t)(i / nv) * p.hidden + m * 128 + (i % nv) * 4;
                    __stcg(reinterpret_cast<float4*>(p.yacc + off), make_float4(0.f, 0.f, 0.f, 0.f));
                    const uint16_t* h = reinterpret_cast<const uint16_t*>(&hv[u]);
                    ushort4 o;
                    o.x = bf16_bits(bf16_val(h[0]) + v[u].x);
                    o.y = bf16_bits(bf16_val(h[1]) + v[u].y);
                    o.z = bf16_bits(bf16_val(h[2]) + v[u].z);
                    o.w = bf16_bits(bf16_val(h[3]) + v[u].w);
                    *reinterpret_cast<ushort4*>(p.Y + off) = o;
                }
            }
        }
        group_finish_notify(x, d, nullptr, 0, 0);
        return true;
    }
};

__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p, const RunArgs ra) {
    megakernel_body<Decode>(p, ra);
}

cudaError_t decode_setup(int* max_blocks_per_sm) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(max_blocks_per_sm, decode_kernel, kThreads, kSmemBytes);
}

cudaError_t launch_decode(const DecodeParams& p, const RunArgs& ra, int n_ctas, cudaStream_t s) {
    // the launch's own status (not an unrelated error left pending earlier)
    void* args[] = {const_cast<DecodeParams*>(&p), const_cast<RunArgs*>(&ra)};
    return cudaLaunchKernel(reinterpret_cast<const void*>(decode_kernel), dim3(n_ctas), dim3(kThreads), args, kSmemBytes,
                            s);
}

}  // namespace et
