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
//                query heads: streamed through the stage arena (K and V
//                blocks of 128 keys), online softmax; partial (o, m, l)  -> E_att[b, g] [#splits(b)]
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

namespace {
// contiguous global -> shared copy completing on an mbarrier (no multicast)
__device__ __forceinline__ void bulk_copy(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}
constexpr int kKeysPerStage = 128;
constexpr uint32_t kAttnStageBytes = 2u * kKeysPerStage * 256u;  // K block then V block (head dim 128)
}  // namespace

struct Decode : WorkloadBase {
    using Params = DecodeParams;
    static constexpr bool kGemm = true;

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
            d.k0 = b * (p.hidden / p.n_kc);
            d.nk = p.hidden / p.n_kc / kTileK;
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
            d.sbytes = kAttnStageBytes;
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

    // ------------------------------------------------------------ stream
    // Stages of an attention split whose keys were cached before this step
    // (all but the stage holding the new token) are copied before the wait.
    __device__ static int stream_prefetch(const Params&, const TaskDesc& d) {
        const int pos = d.p[3], key0 = d.p[4], nkeys = d.p[5];
        if (key0 + nkeys <= pos) return d.nk;  // the new key is in a later split
        return (pos - key0) / kKeysPerStage;   // stages before the one holding key `pos`
    }
    __device__ static int stage_keys(const TaskDesc& d, int st) { return min(kKeysPerStage, d.p[5] - st * kKeysPerStage); }
    __device__ static uint32_t stream_bytes(const Params&, const TaskDesc& d, int st) {
        return 2u * (uint32_t)stage_keys(d, st) * 256u;
    }
    __device__ static void stream_copy(const Params& p, const TaskDesc& d, int st, uint8_t* dst, uint64_t* bar,
                                       uint64_t pol) {
        const int bb = d.p[0], g = d.p[1];
        const size_t row = ((size_t)(bb * p.nkv + g) * p.max_ctx + d.p[4] + st * kKeysPerStage) * p.hd;
        const uint32_t bytes = (uint32_t)stage_keys(d, st) * 256u;
        bulk_copy(dst, p.Kc + row, bytes, bar, pol);
        bulk_copy(dst + kKeysPerStage * 256, p.Vc + row, bytes, bar, pol);
    }

    // One attention split: grp query heads against the split's keys, online
    // softmax across its stages.  Scores: 8 threads per key, thread j of a
    // key holding dims [8j, 8j+8) and [64+8j, 64+8j+8) of every query head
    // (16 x grp floats in registers) -- a warp reads four whole 256-byte key
    // rows per instruction.  Values: thread t owns dim t of every head.
    __device__ static bool stream_exec(const Params& p, Ctx& x, TaskDesc& d) {
        const int bb = d.p[0], g = d.p[1], s = d.p[2];
        const int tid = x.tid, j8 = tid & 7, kg = tid >> 3, w = tid >> 5, lane = tid & 31;
        const int grp = p.grp;
        float qv[4][16];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            if (h < grp) {
                const uint16_t* qr = p.q + ((size_t)bb * p.nq + g * grp + h) * p.hd;
                // (written during the run by another SM's branch: read through L2)
                bf16x8(__ldcg(reinterpret_cast<const uint4*>(qr + 8 * j8)), qv[h]);
                bf16x8(__ldcg(reinterpret_cast<const uint4*>(qr + 64 + 8 * j8)), qv[h] + 8);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) qv[h][i] = 0.f;
            }
        }
        float* sc = x.epi;                                     // [4][128] scaled scores
        float4* pk = reinterpret_cast<float4*>(x.epi + 512);  // [128] probabilities, one float4 per key
        float* red = x.epi + 1024;                             // [4 warps][4 heads] x 2
        const float scale = 0.08838834764831845f;              // 1 / sqrt(128)
        float m[4], l[4], o[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            m[h] = -INFINITY;
            l[h] = 0.f;
            o[h] = 0.f;
        }
        StageAlloc al = stream_alloc(d);
        for (int st = 0; st < d.nk; ++st) {
            uint32_t off;
            if (!stream_stage_wait(x, d, st, al, &off)) return false;
            const uint8_t* Ks = x.arena + off;
            const uint8_t* Vs = Ks + kKeysPerStage * 256;
            const int nks = stage_keys(d, st);
#pragma unroll 2
            for (int pass = 0; pass < kKeysPerStage / 16; ++pass) {
                const int key = pass * 16 + kg;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                if (key < nks) {
                    float kv[16];
                    bf16x8(*reinterpret_cast<const uint4*>(Ks + key * 256 + j8 * 16), kv);
                    bf16x8(*reinterpret_cast<const uint4*>(Ks + key * 256 + 128 + j8 * 16), kv + 8);
                    float acc2[4] = {0.f, 0.f, 0.f, 0.f};  // two chains per head (latency, not work)
#pragma unroll
                    for (int h = 0; h < 4; ++h)
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            acc[h] = fmaf(qv[h][i], kv[i], acc[h]);
                            acc2[h] = fmaf(qv[h][8 + i], kv[8 + i], acc2[h]);
                        }
#pragma unroll
                    for (int h = 0; h < 4; ++h) acc[h] += acc2[h];
                }
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], 1);
                    acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], 2);
                    acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], 4);
                }
                if (j8 == 0 && key < nks)
#pragma unroll
                    for (int h = 0; h < 4; ++h) sc[h * 128 + key] = acc[h] * scale;
            }
            exec_bar();
            // stage maximum per head, then probabilities and their sums
            float mx[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                mx[h] = tid < nks ? sc[h * 128 + tid] : -INFINITY;
#pragma unroll
                for (int o2 = 16; o2 > 0; o2 >>= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o2));
            }
            if (lane == 0)
#pragma unroll
                for (int h = 0; h < 4; ++h) red[w * 4 + h] = mx[h];
            exec_bar();
            float alpha[4], pr[4], ps[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float mn = fmaxf(m[h], fmaxf(fmaxf(red[h], red[4 + h]), fmaxf(red[8 + h], red[12 + h])));
                alpha[h] = expf(m[h] - mn);
                m[h] = mn;
                pr[h] = tid < nks ? expf(sc[h * 128 + tid] - mn) : 0.f;
                ps[h] = pr[h];
#pragma unroll
                for (int o2 = 16; o2 > 0; o2 >>= 1) ps[h] += __shfl_xor_sync(0xffffffffu, ps[h], o2);
            }
            pk[tid] = make_float4(pr[0], pr[1], pr[2], pr[3]);
            if (lane == 0)
#pragma unroll
                for (int h = 0; h < 4; ++h) red[16 + w * 4 + h] = ps[h];
            exec_bar();
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                l[h] = l[h] * alpha[h] + red[16 + h] + red[20 + h] + red[24 + h] + red[28 + h];
                o[h] *= alpha[h];
            }
            // two chains per head over even and odd keys (nks is even unless it is the
            // split's last stage; the odd tail key goes to the first chain)
            const uint16_t* vcol = reinterpret_cast<const uint16_t*>(Vs) + tid;
            float o2[4] = {0.f, 0.f, 0.f, 0.f};
            int key = 0;
#pragma unroll 2
            for (; key + 1 < nks; key += 2) {
                const float4 pa = pk[key], pb = pk[key + 1];
                const float va = bf16_val(vcol[key * 128]), vb = bf16_val(vcol[(key + 1) * 128]);
                o[0] = fmaf(pa.x, va, o[0]);
                o[1] = fmaf(pa.y, va, o[1]);
                o[2] = fmaf(pa.z, va, o[2]);
                o[3] = fmaf(pa.w, va, o[3]);
                o2[0] = fmaf(pb.x, vb, o2[0]);
                o2[1] = fmaf(pb.y, vb, o2[1]);
                o2[2] = fmaf(pb.z, vb, o2[2]);
                o2[3] = fmaf(pb.w, vb, o2[3]);
            }
            if (key < nks) {
                const float4 pa = pk[key];
                const float va = bf16_val(vcol[key * 128]);
                o[0] = fmaf(pa.x, va, o[0]);
                o[1] = fmaf(pa.y, va, o[1]);
                o[2] = fmaf(pa.z, va, o[2]);
                o[3] = fmaf(pa.w, va, o[3]);
            }
#pragma unroll
            for (int h = 0; h < 4; ++h) o[h] += o2[h];
            stream_stage_release(x, d, st);
        }
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
        // thread t = dim t: the splits' partial outputs, loads independent of each other
        for (int h = 0; h < p.grp; ++h) {
            float os = 0.f;
#pragma unroll 4
            for (int s = 0; s < ns; ++s) os = fmaf(wgt[s * p.grp + h], __ldcg(base + ((size_t)s * p.grp + h) * stride + tid), os);
            p.attn[(size_t)bb * p.nq * p.hd + (size_t)(g * p.grp + h) * p.hd + tid] = bf16_bits(os * inv[h]);
        }
        fence_proxy_async_global();  // attn is read by TMA in the o-proj tasks
        int* ev = x.ctr + (unfused(p) ? p.ev_merge_all : p.ev_ag + g);
        const int tgt = unfused(p) ? p.B * p.nkv : p.B;
        if (group_finish_notify(x, d, ev, 1, tgt) && push_all(p))
            group_push(x, p.n_m, [&](int m) { return task_word(ET_OP_DEC_OPROJ, m, g); });
        return true;
    }

    // ------------------------------------------------------------ branches
    // Q head n, K head (n - nq) or V head (n - nq - nkv), all B tokens, from
    // the head's K-chunk sums; thread t = dim t.  Run by the QKV task that
    // completed E_qkv[n].
    __device__ static bool branch(const Params& p, Ctx& x, const TaskDesc& d0, int n) {
        const int kind = n < p.nq ? 0 : (n < p.nq + p.nkv ? 1 : 2);
        const int g = kind == 0 ? n / p.grp : (kind == 1 ? n - p.nq : n - p.nq - p.nkv);
        TaskDesc d = d0;
        d.word = task_word(kind == 0 ? ET_OP_DEC_QBR : (kind == 1 ? ET_OP_DEC_KBR : ET_OP_DEC_VBR), n, 0);
        d.t_fetch = d.t_acc = 0;
        if (x.debug & ET_DEBUG_TRACE) d.t_fetch = globaltimer();
        if (!group_wait(x, d, nullptr, 0, 311)) return false;
        const int t = x.tid, w = t >> 5, lane = t & 31;
        const int stride = p.n_heads * p.hd;
        float* acc = p.qkvacc + (size_t)n * p.hd + t;
        float* sy = x.epi;              // [8][128] exchange for the rotation
        float* red = x.epi + 8 * 128;   // [4 warps][8]
        const int ti = t & 63;
        const double inv_freq = exp(-2.0 * (double)ti / (double)p.hd * log(p.rope_base));
        const float gam = kind == 2 ? 1.f : bf16_val(kind == 0 ? p.gq[t] : p.gk[t]);
        for (int b0 = 0; b0 < p.B; b0 += 8) {
            float y[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int b = b0 + j;
                float v = 0.f;
                if (b < p.B) {
                    v = __ldcg(acc + (size_t)b * stride);
                    __stcg(acc + (size_t)b * stride, 0.f);
                }
                y[j] = bf16_val(bf16_bits(v));  // the qkv tensor is bf16
            }
            if (kind == 2) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int b = b0 + j;
                    if (b < p.B) {
                        const int pos = __ldg(p.pos + b);
                        if (pos >= 0 && pos < p.max_ctx)
                            p.Vc[(((size_t)b * p.nkv + g) * p.max_ctx + pos) * p.hd + t] = bf16_bits(y[j]);
                    }
                }
                continue;
            }
            // per-head RMSNorm: sums of squares over the head's 128 dims
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float ss = y[j] * y[j];
#pragma unroll
                for (int o2 = 16; o2 > 0; o2 >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o2);
                if (lane == 0) red[w * 8 + j] = ss;
            }
            exec_bar();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float tot = red[j] + red[8 + j] + red[16 + j] + red[24 + j];
                y[j] = y[j] * (1.0f / sqrtf(tot / (float)p.hd + p.eps)) * gam;
                sy[j * 128 + t] = y[j];
            }
            exec_bar();
            // RoPE, rotate-half pairing: dim i with dim i + hd/2
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int b = b0 + j;
                if (b >= p.B) continue;
                const int pos = __ldg(p.pos + b);
                if (pos < 0 || pos >= p.max_ctx) continue;
                double sn, cs;
                sincos((double)pos * inv_freq, &sn, &cs);
                const float other = sy[j * 128 + (t ^ 64)];
                const float r = t < 64 ? y[j] * (float)cs - other * (float)sn : y[j] * (float)cs + other * (float)sn;
                if (kind == 0) {
                    const size_t qi = ((size_t)b * p.nq + n) * p.hd + t;
                    p.q[qi] = bf16_bits(r);
                    if (p.out_q) p.out_q[qi] = bf16_bits(r);
                } else {
                    p.Kc[(((size_t)b * p.nkv + g) * p.max_ctx + pos) * p.hd + t] = bf16_bits(r);
                }
            }
            exec_bar();  // sy / red are reused by the next 8 tokens
        }
        fence_proxy_async_global();  // the cache is read by bulk copies in the attention tasks
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
        const bool is_up = q >= 2;
        const int j = r & 63;
        float* stage = x.epi;  // [64][33]
        for (int c0 = 0; c0 < d.n; c0 += 32) {
            float va[16], vb[16];
            acc_load16(taddr, c0, va);
            if (c0 + 16 < d.n) acc_load16(taddr, c0 + 16, vb);
            if (c0 + 32 >= d.n) acc_release(acc_empty);
            if (is_up) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    stage[j * 33 + i] = va[i];
                    stage[j * 33 + 16 + i] = vb[i];
                }
            }
            exec_bar();
            if (!is_up) {
                const int col = a * p.gu_tile + j;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int b = c0 + i;
                    const float gv = i < 16 ? va[i] : vb[i - 16];
                    if (b < p.B) p.hm[(size_t)b * p.inter + col] = bf16_bits(silu(gv) * stage[j * 33 + i]);
                }
            }
            exec_bar();
        }
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
        if (x.tid == 0) {
            const int pos = __ldg(p.pos + b);
            if (pos < 0 || pos >= p.max_ctx) fail(x.ctl, ET_ERR_INVALID, 313, b, pos, p.max_ctx);
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
        const int nv = p.hidden / kExecThreads;
        const size_t r0 = (size_t)b * p.hidden + x.tid * nv;
        float v[32];
        for (int i = 0; i < nv; i += 8) {
            float xv[8];
            bf16x8(*reinterpret_cast<const uint4*>(p.X + r0 + i), xv);
            uint4 o;
            uint16_t* oo = reinterpret_cast<uint16_t*>(&o);
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const float a = __ldcg(p.h1acc + r0 + i + t);
                __stcg(p.h1acc + r0 + i + t, 0.f);
                oo[t] = bf16_bits(xv[t] + a);
                v[i + t] = bf16_val(oo[t]);
            }
            *reinterpret_cast<uint4*>(p.h1 + r0 + i) = o;
            if (p.out_h1) *reinterpret_cast<uint4*>(p.out_h1 + r0 + i) = o;
        }
        const float inv = row_inv_rms(p, x, v, nv);
        for (int i = 0; i < nv; i += 8) {
            float gg[8];
            bf16x8(*reinterpret_cast<const uint4*>(p.g2 + x.tid * nv + i), gg);
            uint4 o;
            uint16_t* oo = reinterpret_cast<uint16_t*>(&o);
#pragma unroll
            for (int t = 0; t < 8; ++t) oo[t] = bf16_bits(v[i + t] * inv * gg[t]);
            *reinterpret_cast<uint4*>(p.xn2 + r0 + i) = o;
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
        const int col = m * 128 + x.tid;
        for (int b = 0; b < p.B; ++b) {
            const size_t i = (size_t)b * p.hidden + col;
            const float a = __ldcg(p.yacc + i);
            __stcg(p.yacc + i, 0.f);
            p.Y[i] = bf16_bits(bf16_val(__ldcg(p.h1 + i)) + a);
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
