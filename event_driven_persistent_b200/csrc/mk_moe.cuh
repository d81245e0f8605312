// MoE layer megakernel: router -> top-k -> token grouping -> stage-1
// grouped GEMM + SiLU*mul -> stage-2 grouped GEMM -> weighted combine, in one
// launch, token count T at run time.
//
// "Event Tensor：用“事件张量”编译动态 Megakernel":
//   §Data-dependent event update: grouping_task[i] -> E[topk[i,:]]; the
//     initial count of expert event E[e] is the number of tokens routed to e.
//   §Data-dependent task triggering: E[e] -> tasks[exp_indptr[e] :
//     exp_indptr[e+1]], the CSR range of expert e's GroupGEMM tiles.
//   §完整 MoE layer: grouping and both GroupGEMM stages in one megakernel,
//     with no global barrier between the two stages.
//   §静态调度: data-dependent edges fall back to a coarse event under
//     static scheduling (here: every grouping task -> every stage-1 slot).
//   §动态调度 (appendix, early push): consumers may be queued once their
//     producers are dispatched and wait on the event before running; used
//     for stage 2 when the stage-1 tasks do not fill the SMs, so stage-2
//     weights stream while stage 1 computes.
//
// Task graph (counts in brackets; dynamic schedule; tiles of 128 tokens):
//   RT(j, c)  16 tokens, K chunk c of n_kc: router GEMM (tensor cores); with n_kc > 1
//             the chunk partials are added at L2 (fp32 red.add) -> E_rt[j] [n_kc];
//             the task that completes E_rt[j] (or the only one) adds the bias and
//             takes top-k and softmax, pair counts per 128-token tile -> E_tk [#blocks]
//   SC        expert counts, CSR (indptr, m-tile indptr), tile offsets -> E_sc [1]
//             (run by the task that completes E_tk; with T <= 128 it is also the
//             grouping task -> E_exp[topk[i,:]])
//   GR(t)     grouped row of every pair of token tile t          -> E_exp[topk[i,:]]
//   S1(f, n)  m-tile f (expert e, <= 128 rows gathered from X) x 64 intermediate cols -> E_s1[f] [#n1]
//   S2(f, n)  m-tile f x 128 output cols, weighted red.add into Yacc -> E_cb[t / cb]
//   CB(b)     Y = bf16(Yacc) for a block of cb tokens (1 up to 256 tokens, else 8), Yacc = 0
#pragma once
#include "et_math.cuh"
#include "et_params.h"

namespace et {

struct Moe : WorkloadBase {
    using Params = MoeParams;
    static constexpr bool kGemm = true;
    static constexpr bool kGather = true;

    __device__ static bool is_unfused(const Params& p) { return p.sched == ET_SCHED_UNFUSED; }

    __device__ static uint32_t fetch_init(const Params& p, int idx) {
        return task_word(ET_OP_MOE_ROUTER, idx / p.n_kc, idx % p.n_kc);
    }

    // m-tile f -> (expert, first grouped row, rows): one 16-byte load of the
    // descriptor the scan wrote.  Data written during the run by other SMs
    // (descriptors, perm, routing weights) is read through L2 (ld.global.cg):
    // an L1 line filled earlier may hold entries that were not written yet.
    __device__ static void mtile(const Params& p, int f, int& e, int& row0, int& cnt) {
        const int4 m = __ldcg(p.mt_desc + f);
        e = m.x;
        row0 = m.y;
        cnt = m.z;
    }

    __device__ static bool derive(const Params& p, Ctx& x, TaskDesc& d) {
        const int op = task_op(d.word), a = task_a(d.word), b = task_b(d.word);
        d.valid = 1;
        d.gemm = 0;
        if (op == ET_OP_MOE_ROUTER) {
            // rows = the E experts of Wr, columns = the task's 16 tokens
            d.valid = a < p.n_tk;
            d.gemm = 1;
            d.a_map = MOE_MAP_WR;
            d.a_row0 = 0;
            d.a_row1 = 64;
            d.b_map = MOE_MAP_X;
            d.b_row0 = a * p.tkt;
            d.n = 16;
            d.nk = p.hidden / p.n_kc / kTileK;
            d.k0 = b * (p.hidden / p.n_kc);
        } else if (op == ET_OP_MOE_GROUP) {
            d.valid = p.n_tt > 1 && a < p.n_tt;  // one tile: the scan task groups
        } else if (op == ET_OP_MOE_COMBINE) {
            d.valid = a < p.n_cb;
        } else if (op == ET_OP_MOE_S1 || op == ET_OP_MOE_S2) {
            if (!x.dynamic) {
                // coarse: the whole grouping must be done before any stage slot
                if (!wait_geq(x.ctr + p.ev_grp, p.n_tt, x.ctl, x.timeout_ns, 200, 0)) return false;
                fence_proxy_async_global();
                if (a >= ld_volatile(p.scal)) {
                    d.valid = 0;
                    return true;
                }
            }
            int e, row0, cnt;
            mtile(p, a, e, row0, cnt);
            d.p[0] = e;
            d.p[1] = row0;
            d.p[2] = cnt;
            d.gemm = 1;
            d.n = (cnt + 15) & ~15;
            d.k0 = 0;
            d.b_row0 = row0;
            if (op == ET_OP_MOE_S1) {
                d.a_map = MOE_MAP_W1;
                d.a_row0 = e * 2 * p.inter + b * p.n1_tile;
                d.a_row1 = e * 2 * p.inter + p.inter + b * p.n1_tile;
                if (p.use_xp) {  // token rows staged in grouped order by the grouping tasks
                    d.b_map = MOE_MAP_XP;
                } else {
                    d.gather = 1;  // token rows straight from X through perm
                }
                d.nk = p.hidden / kTileK;
            } else {
                d.a_map = MOE_MAP_W2;
                d.a_row0 = e * p.hidden + b * p.n2_tile;
                d.a_row1 = e * p.hidden + b * p.n2_tile + 64;
                d.b_map = MOE_MAP_HM;
                d.nk = p.inter / kTileK;
            }
        }
        return true;
    }

    // stage-1 B row r of the task: token perm[row0 + r] / k of X
    __device__ static const uint16_t* gather_row(const Params& p, const TaskDesc& d, int r) {
        if (r >= d.p[2]) return nullptr;
        return p.X + (size_t)(__ldcg(p.perm + d.p[1] + r) / p.k) * p.hidden;
    }

    __device__ static bool gemm_wait(const Params& p, Ctx& x, TaskDesc& d) {
        const int op = task_op(d.word), f = task_a(d.word);
        if (op != ET_OP_MOE_S2) return true;  // router: no input; stage 1: waited before derive
        if (is_unfused(p)) {
            const int mt_total = ld_volatile(p.scal);
            return wait_geq(x.ctr + p.ev_s1_all, mt_total * p.n_n1, x.ctl, x.timeout_ns, 201, 0);
        }
        // static, and dynamic with stage 2 pushed early: wait for the m-tile's stage 1
        return wait_geq(x.ctr + p.ev_s1 + f, p.n_n1, x.ctl, x.timeout_ns, 202, f);
    }

    __device__ static const CUtensorMap* a_map(const Params& p, int id) {
        return id == MOE_MAP_WR ? &p.tm_wr : (id == MOE_MAP_W1 ? &p.tm_w1 : &p.tm_w2);
    }
    __device__ static const CUtensorMap* b_map(const Params& p, int id) {
        return id == MOE_MAP_X ? &p.tm_x : (id == MOE_MAP_XP ? &p.tm_xp : &p.tm_hm);
    }
    __device__ static const CUtensorMap* b_map_wide(const Params& p, int id) {
        return id == MOE_MAP_HM ? &p.tm_hm64 : nullptr;
    }

    // Push the stage-1 tasks of m-tiles [f0, f0 + nf) and, when stage 2 goes
    // early, their stage-2 tasks right after (exec group or single thread).
    __device__ static int n_stage_tasks(const Params& p, int nf, bool early) {
        return nf * (p.n_n1 + (early ? p.n_n2 : 0));
    }
    __device__ static uint32_t stage_task(const Params& p, int f0, int nf, int i) {
        const int n1 = nf * p.n_n1;
        if (i < n1) return task_word(ET_OP_MOE_S1, f0 + i / p.n_n1, i % p.n_n1);
        i -= n1;
        return task_word(ET_OP_MOE_S2, f0 + i / p.n_n2, i % p.n_n2);
    }

    __device__ static bool epilogue(const Params& p, Ctx& x, TaskDesc& d, uint32_t taddr, uint64_t* acc_empty) {
        const int op = task_op(d.word), a = task_a(d.word), b = task_b(d.word);
        const int w = x.tid >> 5, lane = x.tid & 31;
        const int q = (w + kExecWarp0) & 3;
        const int r = q * 32 + lane;
        if (op == ET_OP_MOE_ROUTER) {
            // logits of the task's 16 tokens (+ bias), transposed through
            // smem: L[token][expert], rows padded to 132 floats
            const int t0 = a * p.tkt;
            const int ntok = min(p.tkt, p.T - t0);
            float* L = x.epi;
            float v[16];
            acc_load16(taddr, 0, v);
            acc_release(acc_empty);
            if (p.n_kc > 1) {
                // K split: add this chunk's partials into lacc at L2; the chunk
                // task that completes E_rt[a] reads the sums and re-zeroes lacc
                float* acc = p.lacc + (size_t)t0 * p.E + r;
                if (r < p.E) {
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        if (c < ntok) red_add(acc + (size_t)c * p.E, v[c]);
                }
                if (!group_finish_notify(x, d, x.ctr + p.ev_rt + a, 1, p.n_kc, false)) return true;
                if (r < p.E) {
#pragma unroll
                    for (int c = 0; c < 16; ++c) v[c] = c < ntok ? __ldcg(acc + (size_t)c * p.E) : 0.f;
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        if (c < ntok) __stcg(acc + (size_t)c * p.E, 0.f);
                }
            }
            if (r < p.E) {
                const float bb = p.bias[r];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float lg = v[c] + bb;
                    L[c * 132 + r] = lg;
                    if (p.out_logits && c < ntok) p.out_logits[(size_t)(t0 + c) * p.E + r] = lg;
                }
            }
            exec_bar();
            return route_topk(p, x, d, a, L);
        } else if (op == ET_OP_MOE_S1) {
            const int row0 = d.p[1], cnt = d.p[2];
            for (int c0 = 0; c0 < d.n; c0 += 16)
                swiglu_tokens16(x, taddr, c0, d.n, acc_empty, p.Hm + (size_t)(row0 + c0) * p.inter + b * p.n1_tile,
                                p.inter, cnt - c0);
            fence_proxy_async_global();  // Hm is read by TMA in stage 2
            int* ev = x.ctr + (is_unfused(p) ? p.ev_s1_all : p.ev_s1 + a);
            const int tgt = is_unfused(p) ? ld_volatile(p.scal) * p.n_n1 : p.n_n1;
            const bool fired = group_finish_notify(x, d, ev, 1, tgt);
            if (fired && x.dynamic && !ld_volatile(p.scal + 1))
                group_push(x, p.n_n2, [&](int n2) { return task_word(ET_OP_MOE_S2, a, n2); });
        } else {  // S2
            const int row0 = d.p[1], cnt = d.p[2];
            int* s_tok = reinterpret_cast<int*>(x.simt);  // [128] token of each row
            float* s_w = reinterpret_cast<float*>(s_tok + 128);
            if (x.tid < cnt) {
                const int pp = __ldcg(p.perm + row0 + x.tid);
                s_tok[x.tid] = pp / p.k;
                s_w[x.tid] = __ldcg(p.topw + pp);
            }
            exec_bar();
            // weighted rows into Yacc: each warp turns its 32 columns x 16
            // tokens around through smem so a lane adds 4 consecutive columns
            // of one token with one vector reduction
            float* tr = x.epi + w * 512;  // [16 tokens][32 columns] per warp
            const int j4 = (lane & 7) * 4;
            float* ybase = p.Yacc + b * p.n2_tile + q * 32 + j4;
            for (int c0 = 0; c0 < d.n; c0 += 16) {
                float v[16];
                acc_load16(taddr, c0, v);
                if (c0 + 16 >= d.n) acc_release(acc_empty);
#pragma unroll
                for (int i = 0; i < 16; ++i) tr[i * 32 + lane] = s_w[c0 + i] * v[i];
                __syncwarp();
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int ci = (lane >> 3) + 4 * u, c = c0 + ci;
                    if (c < cnt)
                        red_add4(ybase + (size_t)s_tok[c] * p.hidden, *reinterpret_cast<const float4*>(tr + ci * 32 + j4));
                }
                __syncwarp();
            }
            if (is_unfused(p)) {
                group_finish_notify(x, d, x.ctr + p.ev_s2_all, 1, -1);
            } else {
                group_finish_notify(x, d, nullptr, 0, 0);
                // One notify per run of rows in the same combine block.  Under
                // the dynamic schedule the first block this task completes is
                // converted here and the others are queued.
                int* fired = reinterpret_cast<int*>(s_w + 128);  // [128] completed blocks
                if (x.tid == 0) x.sc->bcast[7] = 0;
                exec_bar();
                if (x.tid < cnt) {
                    const int c = x.tid;
                    const int blk = s_tok[c] / p.cb;
                    const bool head = c == 0 || s_tok[c - 1] / p.cb != blk;
                    if (head) {
                        int len = 1;
                        while (c + len < cnt && s_tok[c + len] / p.cb == blk) ++len;
                        const int ntok = min(p.cb, p.T - blk * p.cb);
                        const int tgt = p.k * p.n_n2 * ntok;
                        if (notify(x.ctr + p.ev_cb + blk, len) == tgt && x.dynamic)
                            fired[atomicAdd(&x.sc->bcast[7], 1)] = blk;
                    }
                }
                exec_bar();
                const int nf = x.sc->bcast[7];
                if (nf > 0) {
                    // the run's task total counts every combine block, so the
                    // block converted here is queued as an empty placeholder
                    // (block index n_cb, which derive marks invalid)
                    group_push(x, nf, [&](int i) { return task_word(ET_OP_MOE_COMBINE, i == 0 ? p.n_cb : fired[i], 0); });
                    TaskDesc cd = d;
                    cd.word = task_word(ET_OP_MOE_COMBINE, fired[0], 0);
                    cd.t_fetch = cd.t_acc = 0;
                    if (x.debug & ET_DEBUG_TRACE) cd.t_fetch = globaltimer();
                    if (!combine_task(p, x, cd)) return false;
                }
                exec_bar();  // s_tok is reused by the next task
            }
        }
        return true;
    }

    __device__ static bool simt(const Params& p, Ctx& x, TaskDesc& d) {
        const int op = task_op(d.word), a = task_a(d.word);
        if (op == ET_OP_MOE_SCAN) return scan_task(p, x, d);
        if (op == ET_OP_MOE_GROUP) return group_task(p, x, d, a);
        return combine_task(p, x, d);
    }


    // CB(b): Y = bf16(Yacc) for tokens [cb*b, cb*b + cb), and Yacc back to 0.
    __device__ static bool combine_task(const Params& p, Ctx& x, TaskDesc& d) {
        const int a = task_a(d.word);
        const int t0 = a * p.cb;
        const int ntok = min(p.cb, p.T - t0);
        if (is_unfused(p)) {
            if (!group_wait(x, d, x.ctr + p.ev_grp, p.n_tt, 210)) return false;
            const int mt_total = ld_volatile(p.scal);
            if (!group_wait(x, d, x.ctr + p.ev_s2_all, mt_total * p.n_n2, 211)) return false;
        } else {
            if (!group_wait(x, d, x.ctr + p.ev_cb + a, p.k * p.n_n2 * ntok, 212)) return false;
        }
        // eight float4 loads in flight per thread, then zero + convert + store
        const int nv = p.hidden / 4, total = ntok * nv;
        for (int base = x.tid; base < total; base += kExecThreads * 8) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = base + u * kExecThreads;
                if (i < total) v[u] = __ldcg(reinterpret_cast<const float4*>(p.Yacc + (size_t)(t0 + i / nv) * p.hidden) + i % nv);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = base + u * kExecThreads;
                if (i < total) {
                    const size_t off = (size_t)(t0 + i / nv) * p.hidden + (i % nv) * 4;
                    __stcg(reinterpret_cast<float4*>(p.Yacc + off), make_float4(0.f, 0.f, 0.f, 0.f));
                    ushort4 o;
                    o.x = bf16_bits(v[u].x);
                    o.y = bf16_bits(v[u].y);
                    o.z = bf16_bits(v[u].z);
                    o.w = bf16_bits(v[u].w);
                    *reinterpret_cast<ushort4*>(p.Y + off) = o;
                }
            }
        }
        if (p.mlp_xn) return mlp_norm(p, x, d, t0, ntok);
        group_finish_notify(x, d, nullptr, 0, 0);
        return true;
    }

    // Fused dense MLP after the layer: the MLP's RMSNorm of the block's tokens
    // from the bf16 outputs just written (same CTA), then E_norm of the MLP.
    __device__ static bool mlp_norm(const Params& p, Ctx& x, TaskDesc& d, int t0, int ntok) {
        exec_bar();  // the block's Y rows are written
        // sums of squares of the bf16 outputs: per token, each warp's part
        // reduced by shuffles into ssw[warp][token], then summed
        const int n8 = p.hidden / 8, total = ntok * n8;
        float* ssw = reinterpret_cast<float*>(x.simt) + 512;  // [4 warps][cb]
        for (int t = 0; t < ntok; ++t) {
            float sq = 0.f;
            for (int c = x.tid; c < n8; c += kExecThreads) {
                float y[8];
                bf16x8(*reinterpret_cast<const uint4*>(p.Y + (size_t)(t0 + t) * p.hidden + c * 8), y);
#pragma unroll
                for (int j = 0; j < 8; ++j) sq = fmaf(y[j], y[j], sq);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
            if ((x.tid & 31) == 0) ssw[(x.tid >> 5) * p.cb + t] = sq;
        }
        exec_bar();
        for (int i = x.tid; i < total; i += kExecThreads) {
            const int t = i / n8, c = (i % n8) * 8;
            const size_t off = (size_t)(t0 + t) * p.hidden + c;
            float y[8], gm[8];
            bf16x8(*reinterpret_cast<const uint4*>(p.Y + off), y);
            bf16x8(__ldg(reinterpret_cast<const uint4*>(p.mlp_gamma + c)), gm);
            const float sst = ssw[t] + ssw[p.cb + t] + ssw[2 * p.cb + t] + ssw[3 * p.cb + t];
            const float inv = 1.0f / sqrtf(sst / (float)p.hidden + p.mlp_eps);
            uint4 o;
            uint16_t* oo = reinterpret_cast<uint16_t*>(&o);
#pragma unroll
            for (int j = 0; j < 8; ++j) oo[j] = bf16_bits(y[j] * inv * gm[j]);
            *reinterpret_cast<uint4*>(p.mlp_xn + off) = o;
        }
        fence_proxy_async_global();  // the MLP's gate/up tasks read xn by TMA
        if (group_finish_notify(x, d, x.ctr + p.mlp_ev_norm, ntok, p.T) && p.mlp_n_gu > 0)
            group_push(x, p.mlp_n_gu, [&](int n) { return task_word(ET_OP_MLP_GATEUP, n, 0); });
        return true;
    }

    // Exec-group scratch of the routing tasks (x.epi and x.simt, which are
    // contiguous and free while the exec group runs a routing task), after
    // the router's logits L [16][132] fp32 at x.epi:
    //   tk    [128 * k] int   selected experts of a 128-token tile, pair order
    //   emask [128][4]  u32   per expert: bit t = token t of the tile picked it
    //   base  [128] int       first grouped row per expert (placement)
    //   hist  [128] int       pairs per expert of a top-k task
    //   misc  [8] int
    struct RouteSmem {
        int* tk;
        uint32_t* emask;
        int* base;
        int* hist;
        int* misc;
    };
    __device__ static RouteSmem route_smem(Ctx& x) {
        RouteSmem s;
        s.tk = reinterpret_cast<int*>(x.epi + 16 * 132);  // after the router's logits L
        s.emask = reinterpret_cast<uint32_t*>(s.tk + 128 * 8);
        s.base = reinterpret_cast<int*>(s.emask + 128 * 4);
        s.hist = s.base + 128;
        s.misc = s.hist + 128;
        return s;
    }

    // Top-k of router task j (tokens [16j, 16j+16)) from its logits L
    // [16][132] in smem: top-k by (logit desc, index asc), softmax of the
    // selected logits, pair counts per expert of the token's 128-token tile.
    // Thread (g, q) = (tid / 8, tid % 8) holds experts 16q .. 16q+15 of token
    // g as 64-bit keys (order-preserving logit bits, then the complemented
    // index, so a larger key is a better candidate); the eight threads of a
    // token take the k best keys in k arg-max rounds, and thread q owns
    // slot q of the token's top-k.  The task that completes E_tk runs the
    // scan itself (dynamic schedule), with no trip through the queue.
    __device__ static uint64_t tk_key(float v, int e) {
        uint32_t b = __float_as_uint(v + 0.0f);  // -0 -> +0: equal logits tie on the index
        b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
        return ((uint64_t)b << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)e);
    }
    __device__ static float tk_val(uint64_t k) {
        const uint32_t h = (uint32_t)(k >> 32);
        return __uint_as_float((h & 0x80000000u) ? (h & 0x7FFFFFFFu) : ~h);
    }
    __device__ static int tk_idx(uint64_t k) { return (int)(0xFFFFFFFFu - (uint32_t)k); }

    __device__ static bool route_topk(const Params& p, Ctx& x, TaskDesc& d, int j, const float* L) {
        RouteSmem sm = route_smem(x);
        const int tile = j * p.tkt / p.tt;
        const int g = x.tid >> 3, q = x.tid & 7;
        const int t0 = j * p.tkt;
        const int ntok = min(p.tkt, p.T - t0);
        const int t = t0 + g;
        const int e0 = q * 16;
        // experts of this thread: 16, 8 (the last group when E % 16 == 8) or none
        const int ne = g < ntok ? max(0, min(16, p.E - e0)) : 0;
        float l[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) l[i] = i < ne ? L[g * 132 + e0 + i] : 0.f;
        if (x.tid < 128) sm.hist[x.tid] = 0;
        uint64_t key[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) key[i] = i < ne ? tk_key(l[i], e0 + i) : 0ull;
        // k rounds of an arg-max over the token's 8 threads: each thread's best
        // key not taken yet, then the max over the eight by xor shuffles; the
        // owner marks it taken (keys are unique: they hold the index).  Thread
        // q keeps the key of round q.  A rolled loop: this code runs once per
        // task and must stay small in the instruction cache.
        uint32_t taken = 0;
        uint64_t kq = 0, k0 = 0;
#pragma unroll 1
        for (int s = 0; s < p.k; ++s) {
            uint64_t best = 0;
            int bi = 16;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const bool ok = !((taken >> i) & 1u) && key[i] > best;
                best = ok ? key[i] : best;
                bi = ok ? i : bi;
            }
            uint64_t w = best;
#pragma unroll
            for (int m = 1; m < 8; m <<= 1) {
                const uint64_t o = __shfl_xor_sync(0xffffffffu, w, m);
                w = o > w ? o : w;
            }
            if (bi < 16 && best == w) taken |= 1u << bi;
            k0 = s == 0 ? w : k0;
            kq = q == s ? w : kq;
        }
        const bool mine = g < ntok && q < p.k;
        float ex = mine ? expf(tk_val(kq) - tk_val(k0)) : 0.f;
        float z = ex;
#pragma unroll
        for (int m = 1; m < 8; m <<= 1) z += __shfl_xor_sync(0xffffffffu, z, m);
        exec_bar();  // hist zeroed
        if (mine) {
            const int e = tk_idx(kq);
            const size_t pi = (size_t)t * p.k + q;
            const float wt = ex / z;
            p.topk[pi] = e;
            p.topw[pi] = wt;
            if (p.out_topk) p.out_topk[pi] = e;
            if (p.out_w) p.out_w[pi] = wt;
            atomicAdd(&sm.hist[e], 1);
        }
        exec_bar();
        // per-tile pair counts (several grouping tiles only: with one tile the
        // scan counts the pairs from the picks it loads anyway)
        if (p.n_tt > 1 && x.tid < p.E && sm.hist[x.tid] > 0)
            atomicAdd(x.ctr + p.ev_gcnt + tile * p.E + x.tid, sm.hist[x.tid]);
        const bool fired = group_finish_notify(x, d, x.ctr + p.ev_tk, 1, p.n_tk);
        if (fired && x.dynamic) {
            // this task completed E_tk: run the scan task here
            TaskDesc sd = d;
            sd.word = task_word(ET_OP_MOE_SCAN, 0, 0);
            sd.t_fetch = sd.t_acc = 0;
            if (x.debug & ET_DEBUG_TRACE) sd.t_fetch = globaltimer();
            return scan_task(p, x, sd);
        }
        return true;
    }

    // Dynamic schedule: the run's queued-task total (CTAs whose next queue
    // slot lies past it stop).  Published after the scan's own pushes, so it
    // stays off the path to the first stage tasks.
    __device__ static void publish_total(Ctx& x, const RouteSmem& sm) {
        if (x.tid == 0) atomicExch(x.ctr + kCtrTotal, sm.misc[6] + 1);
    }

    __device__ static int tile_count(const RouteSmem& sm, int e) {
        return __popc(sm.emask[e * 4]) + __popc(sm.emask[e * 4 + 1]) + __popc(sm.emask[e * 4 + 2]) +
               __popc(sm.emask[e * 4 + 3]);
    }

    // Expert counts -> CSR of pairs (indptr), CSR of m-tiles (tindptr), the
    // m-tile -> expert map, the run's task total and the early-push choice.
    // Exec group; thread e owns expert e.  Returns the number of m-tiles.
    __device__ static int build_csr(const Params& p, Ctx& x, RouteSmem& sm, int cnt, int* ex_out) {
        const int e = x.tid;
        int tot, ttot;
        const int ex = exec_scan(cnt, x.tid, sm.misc, &tot);
        const int nt = (cnt + p.bm - 1) / p.bm;
        const int tex = exec_scan(nt, x.tid, sm.misc, &ttot);
        if (e < p.E) {
            p.counts[e] = cnt;
            p.indptr[e] = ex;
            p.tindptr[e] = tex;
            if (p.out_indptr) p.out_indptr[e] = ex;
            for (int m = 0; m < nt; ++m) p.mt_desc[tex + m] = make_int4(e, ex + m * p.bm, min(p.bm, cnt - m * p.bm), 0);
        }
        if (x.tid == 0) {
            p.indptr[p.E] = tot;
            p.tindptr[p.E] = ttot;
            if (p.out_indptr) p.out_indptr[p.E] = tot;
            p.scal[0] = ttot;
            // early push: with one grouping tile the scan queues every stage-1
            // task before any stage-2 task, so a stage-2 task never holds an
            // SM while stage-1 work waits behind it; with several tiles the
            // experts' batches interleave and it only pays when stage 1 is small
            const bool early = x.dynamic && (p.n_tt == 1 || n_stage_tasks(p, ttot, false) <= p.early_max);
            p.scal[1] = early;
            // queued tasks of the run: router chunks, group (several tiles),
            // stage 1 and 2, combine (the scan runs inline); published once
            // the scan has queued its successors (publish_total)
            // (router tasks are queue slots only when they are the queue's initial tasks)
            sm.misc[6] = (x.q.n_init > 0 ? p.n_tk * p.n_kc : 0) + (p.n_tt > 1 ? p.n_tt : 0) +
                         ttot * (p.n_n1 + p.n_n2) + p.n_cb + p.extra_tasks;
            sm.misc[4] = ttot;
            sm.misc[5] = early;
        }
        exec_bar();
        *ex_out = ex;
        return sm.misc[4];
    }

    // Load a 128-token tile's picks (pair order) into sm.tk and build the
    // per-expert token masks.  Exec group.
    __device__ static void load_tile_picks(const Params& p, Ctx& x, RouteSmem& sm, int t0, int ntok) {
        for (int i = x.tid; i < 128 * 4; i += kExecThreads) sm.emask[i] = 0;
        exec_bar();
        const int tl = x.tid;  // token of the tile; its k picks are loaded together
        if (tl < ntok) {
            int ee[8];
#pragma unroll
            for (int s = 0; s < 8; ++s) ee[s] = s < p.k ? __ldcg(p.topk + (size_t)(t0 + tl) * p.k + s) : 0;
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                if (s < p.k) {
                    sm.tk[tl * p.k + s] = ee[s];
                    atomicOr(&sm.emask[ee[s] * 4 + (tl >> 5)], 1u << (tl & 31));
                }
            }
        }
        exec_bar();
    }

    // Stable placement of one tile's pairs: thread t owns token t of the tile;
    // the grouped row of (t, s) with expert e is base[e] + the number of the
    // tile's tokens before t that picked e (a popcount of e's token mask).
    __device__ static void place_pairs(const Params& p, Ctx& x, RouteSmem& sm, int t0, int ntok) {
        const int t = x.tid;
        if (t >= ntok) return;
        const int wd = t >> 5;
        const uint32_t below = (1u << (t & 31)) - 1u;
        for (int s = 0; s < p.k; ++s) {
            const int e = sm.tk[t * p.k + s];
            const uint32_t* m = sm.emask + e * 4;
            int rank = __popc(m[wd] & below);
            for (int j = 0; j < wd; ++j) rank += __popc(m[j]);
            const int pair = (t0 + t) * p.k + s, row = sm.base[e] + rank;
            p.perm[row] = pair;
            p.pos[pair] = row;
            if (p.out_perm) p.out_perm[row] = pair;
            sm.tk[t * p.k + s] = row;  // the expert is no longer needed: keep the row for the X copy
        }
    }

    // Xp rows of a grouping tile's pairs: each token's X row (read once) to the
    // grouped row of each of its k picks.  Warp w takes tokens w, w + 4, ...;
    // lanes cover the row in 16-byte pieces.  Exec group, after place_pairs.
    __device__ static void stage_rows(const Params& p, Ctx& x, const RouteSmem& sm, int t0, int ntok) {
        exec_bar();  // the rows placed by every thread
        const int w = x.tid >> 5, lane = x.tid & 31, nv = p.hidden / 8;
        for (int t = w; t < ntok; t += kExecThreads / 32) {
            const uint4* src = reinterpret_cast<const uint4*>(p.X + (size_t)(t0 + t) * p.hidden);
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (lane + 32 * u < nv) v[u] = __ldg(src + lane + 32 * u);
            for (int s = 0; s < p.k; ++s) {
                uint4* dst = reinterpret_cast<uint4*>(p.Xp + (size_t)sm.tk[t * p.k + s] * p.hidden);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (lane + 32 * u < nv) dst[lane + 32 * u] = v[u];
            }
        }
        fence_proxy_async_global();  // Xp is read by TMA in stage 1
    }

    // SC: expert counts from the per-tile pair counts, the CSRs and each
    // tile's first grouped row per expert.  With one 128-token tile it is
    // also the grouping task (placement, then the stage tasks / E_grp).
    __device__ static bool scan_task(const Params& p, Ctx& x, TaskDesc& d) {
        if (!group_wait(x, d, x.ctr + p.ev_tk, p.n_tk + p.bad_count, 230)) return false;
        RouteSmem sm = route_smem(x);
        const int e = x.tid;
        if (p.n_tt == 1) {
            // one grouping tile (T <= 128): the picks give the counts (popcounts
            // of the per-expert token masks), the CSRs, then the placement
            load_tile_picks(p, x, sm, 0, p.T);
            int ex;
            const int ttot = build_csr(p, x, sm, e < p.E ? tile_count(sm, e) : 0, &ex);
            if (x.debug & ET_DEBUG_TRACE) d.t_acc = globaltimer();
            if (e < p.E) sm.base[e] = ex;
            exec_bar();
            place_pairs(p, x, sm, 0, p.T);
            if (!x.dynamic) {
                group_finish_notify(x, d, x.ctr + p.ev_grp, 1, p.n_tt);
                return true;
            }
            group_finish_notify(x, d, nullptr, 0, 0);
            const bool early = sm.misc[5] != 0;
            group_push(x, n_stage_tasks(p, ttot, early), [&](int i) { return stage_task(p, 0, ttot, i); });
            publish_total(x, sm);
            return true;
        }
        int cnt = 0;
        // (plain L2 loads after the acquiring wait, sixteen tiles at a time)
#pragma unroll 1
        for (int g0 = 0; g0 < p.n_tt; g0 += 16) {
            int v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                v[i] = (e < p.E && g0 + i < p.n_tt) ? __ldcg(x.ctr + p.ev_gcnt + (g0 + i) * p.E + e) : 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) cnt += v[i];
        }
        int ex;
        build_csr(p, x, sm, cnt, &ex);
        if (x.debug & ET_DEBUG_TRACE) d.t_acc = globaltimer();
        if (e < p.E) {
            int run = ex;
#pragma unroll 1
            for (int g0 = 0; g0 < p.n_tt; g0 += 16) {
                int v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = g0 + i < p.n_tt ? __ldcg(x.ctr + p.ev_gcnt + (g0 + i) * p.E + e) : 0;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    if (g0 + i < p.n_tt) p.goff[(size_t)(g0 + i) * p.E + e] = run;
                    run += v[i];
                }
            }
        }
        const bool fired = group_finish_notify(x, d, x.ctr + p.ev_sc, 1, 1);
        if (fired && x.dynamic) {
            group_push(x, p.n_tt, [&](int g) { return task_word(ET_OP_MOE_GROUP, g, 0); });
            publish_total(x, sm);
        }
        return true;
    }

    // GR(g) (several tiles): grouped rows of 128-token tile g's pairs, then
    // the expert events (grouping_task[g] -> E[topk[i,:]], one add of the
    // tile's pair count per expert it touches).
    __device__ static bool group_task(const Params& p, Ctx& x, TaskDesc& d, int g) {
        if (!group_wait(x, d, x.ctr + p.ev_sc, 1, 240)) return false;
        RouteSmem sm = route_smem(x);
        const int t0 = g * p.tt;
        const int ntok = min(p.tt, p.T - t0);
        const int e = x.tid;
        if (e < p.E) sm.base[e] = __ldcg(p.goff + (size_t)g * p.E + e);
        load_tile_picks(p, x, sm, t0, ntok);
        place_pairs(p, x, sm, t0, ntok);
        if (p.use_xp) stage_rows(p, x, sm, t0, ntok);
        const int cnt = e < p.E ? tile_count(sm, e) : 0;
        if (!x.dynamic) {
            group_finish_notify(x, d, x.ctr + p.ev_grp, 1, p.n_tt);
            return true;
        }
        group_finish_notify(x, d, nullptr, 0, 0);
        if (cnt > 0 && notify(x.ctr + p.ev_exp + e, cnt) == __ldcg(p.counts + e)) {
            const int f0 = __ldcg(p.tindptr + e), nf = __ldcg(p.tindptr + e + 1) - f0;
            const bool early = ld_volatile(p.scal + 1) != 0;
            thread_push(x, n_stage_tasks(p, nf, early), [&](int i) { return stage_task(p, f0, nf, i); });
        }
        return true;
    }
};

}  // namespace et
