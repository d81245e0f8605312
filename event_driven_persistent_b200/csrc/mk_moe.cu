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
//
// Task graph (counts in brackets; dynamic schedule):
//   RT(t, c)  router partial logits of token tile t, K chunk c   -> E_rt[t] [#chunks]
//   TK(t)     sum partials + bias, top-k, softmax, tile histograms -> E_tk [#tiles]
//   SC        expert counts, CSR (indptr, m-tile indptr), E_exp counts -> E_sc [1]
//   GR(g)     place the pairs of token group g, copy their rows   -> E_exp[topk[i,:]]
//   S1(f, n)  m-tile f (expert e, up to 128 rows) x 64 intermediate cols -> E_s1[f] [#n1]
//   S2(f, n)  m-tile f x 128 output cols, weighted red.add into Yacc -> E_cb[t / cb]
//   CB(b)     Y = bf16(Yacc) for a block of cb tokens, Yacc = 0
#include <cuda_bf16.h>

#include "et_engine.cuh"
#include "et_params.h"

namespace et {

namespace {
__device__ __forceinline__ uint16_t bf16_bits(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }
__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }
__device__ __forceinline__ void red_add(float* p, float v) {
    asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}
// (value desc, index asc) total order
__device__ __forceinline__ bool better(float v, int i, float w, int j) { return v > w || (v == w && i < j); }
}  // namespace

struct Moe {
    using Params = MoeParams;
    static constexpr bool kGemm = true;

    __device__ static bool is_static(const Params& p) { return p.sched == ET_SCHED_STATIC; }
    __device__ static bool is_unfused(const Params& p) { return p.sched == ET_SCHED_UNFUSED; }

    __device__ static uint32_t fetch_init(const Params& p, int idx) {
        return task_word(ET_OP_MOE_ROUTER, idx / p.n_kc, idx % p.n_kc);
    }

    // m-tile f -> (expert, first grouped row, rows); needs the scan's outputs
    __device__ static void mtile(const Params& p, int f, int& e, int& row0, int& cnt) {
        e = p.mt_expert[f];
        const int mt = f - p.tindptr[e];
        row0 = p.indptr[e] + mt * p.bm;
        cnt = min(p.bm, p.counts[e] - mt * p.bm);
    }

    __device__ static bool derive(const Params& p, Ctx& x, TaskDesc& d) {
        const int op = task_op(d.word), a = task_a(d.word), b = task_b(d.word);
        d.valid = 1;
        d.gemm = 0;
        if (op == ET_OP_MOE_ROUTER) {
            d.valid = a < p.n_tt;
            const int cnt = min(p.tt, p.T - a * p.tt);
            d.gemm = 1;
            d.a_map = MOE_MAP_WR;
            d.a_row0 = 0;
            d.a_row1 = 64;
            d.b_map = MOE_MAP_X;
            d.b_row0 = a * p.tt;
            d.n = (cnt + 15) & ~15;
            d.nk = p.hidden / p.n_kc / kTileK;
            d.k0 = b * (p.hidden / p.n_kc);
        } else if (op == ET_OP_MOE_TOPK) {
            d.valid = a < p.n_tt;
        } else if (op == ET_OP_MOE_GROUP) {
            d.valid = a < p.n_g;
        } else if (op == ET_OP_MOE_COMBINE) {
            d.valid = a < p.n_cb;
        } else if (op == ET_OP_MOE_S1 || op == ET_OP_MOE_S2) {
            if (!x.dynamic) {
                // coarse: the whole grouping must be done before any stage slot
                if (!wait_geq(x.ctr + p.ev_grp, p.n_g, x.ctl, x.timeout_ns, 200, 0)) return false;
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
                d.b_map = MOE_MAP_XP;
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

    __device__ static bool gemm_wait(const Params& p, Ctx& x, TaskDesc& d) {
        const int op = task_op(d.word), f = task_a(d.word);
        if (op != ET_OP_MOE_S2 || x.dynamic) return true;  // router: no input; S1 waited in derive
        if (is_unfused(p)) {
            const int mt_total = ld_volatile(p.scal);
            return wait_geq(x.ctr + p.ev_s1_all, mt_total * p.n_n1, x.ctl, x.timeout_ns, 201, 0);
        }
        return wait_geq(x.ctr + p.ev_s1 + f, p.n_n1, x.ctl, x.timeout_ns, 202, f);
    }

    __device__ static const CUtensorMap* a_map(const Params& p, int id) {
        return id == MOE_MAP_WR ? &p.tm_wr : (id == MOE_MAP_W1 ? &p.tm_w1 : &p.tm_w2);
    }
    __device__ static const CUtensorMap* b_map(const Params& p, int id) {
        return id == MOE_MAP_X ? &p.tm_x : (id == MOE_MAP_XP ? &p.tm_xp : &p.tm_hm);
    }

    __device__ static bool epilogue(const Params& p, Ctx& x, TaskDesc& d, uint32_t taddr, uint64_t* acc_empty) {
        const int op = task_op(d.word), a = task_a(d.word), b = task_b(d.word);
        const int w = x.tid >> 5, lane = x.tid & 31;
        const int q = (w + kExecWarp0) & 3;
        const int r = q * 32 + lane;
        if (op == ET_OP_MOE_ROUTER) {
            // rows = experts, columns = tokens of tile a; partial logits of K chunk b
            const int t0 = a * p.tt;
            const int cnt = min(p.tt, p.T - t0);
            float* lp = p.lpart + (size_t)b * p.maxT * p.E;
            for (int c0 = 0; c0 < d.n; c0 += 16) {
                float v[16];
                acc_load16(taddr, c0, v);
                if (c0 + 16 >= d.n) acc_release(acc_empty);
                if (r < p.E) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c0 + i < cnt) lp[(size_t)(t0 + c0 + i) * p.E + r] = v[i];
                }
            }
            int* ev = x.ctr + (is_unfused(p) ? p.ev_rt_all : p.ev_rt + a);
            const int tgt = is_unfused(p) ? p.n_tt * p.n_kc : p.n_kc;
            const bool fired = group_finish_notify(x, d, ev, 1, tgt);
            if (fired && x.dynamic) group_push(x, 1, [&](int) { return task_word(ET_OP_MOE_TOPK, a, 0); });
        } else if (op == ET_OP_MOE_S1) {
            const int row0 = d.p[1], cnt = d.p[2];
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
                    const int col = b * p.n1_tile + j;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int c = c0 + i;
                        const float g = i < 16 ? va[i] : vb[i - 16];
                        if (c < cnt) p.Hm[(size_t)(row0 + c) * p.inter + col] = bf16_bits(silu(g) * stage[j * 33 + i]);
                    }
                }
                exec_bar();
            }
            fence_proxy_async_global();  // Hm is read by TMA in stage 2
            int* ev = x.ctr + (is_unfused(p) ? p.ev_s1_all : p.ev_s1 + a);
            const int tgt = is_unfused(p) ? ld_volatile(p.scal) * p.n_n1 : p.n_n1;
            const bool fired = group_finish_notify(x, d, ev, 1, tgt);
            if (fired && x.dynamic)
                group_push(x, p.n_n2, [&](int n2) { return task_word(ET_OP_MOE_S2, a, n2); });
        } else {  // S2
            const int row0 = d.p[1], cnt = d.p[2];
            const int col = b * p.n2_tile + r;
            for (int c0 = 0; c0 < d.n; c0 += 16) {
                float v[16];
                acc_load16(taddr, c0, v);
                if (c0 + 16 >= d.n) acc_release(acc_empty);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int c = c0 + i;
                    if (c < cnt) {
                        const int pp = p.perm[row0 + c];
                        const int t = pp / p.k;
                        red_add(p.Yacc + (size_t)t * p.hidden + col, p.topw[pp] * v[i]);
                    }
                }
            }
            if (is_unfused(p)) {
                group_finish_notify(x, d, x.ctr + p.ev_s2_all, 1, -1);
            } else {
                group_finish_notify(x, d, nullptr, 0, 0);
                // one notify per run of rows in the same combine block
                if (x.tid < cnt) {
                    const int c = x.tid;
                    const int blk = (p.perm[row0 + c] / p.k) / p.cb;
                    const bool head = c == 0 || (p.perm[row0 + c - 1] / p.k) / p.cb != blk;
                    if (head) {
                        int len = 1;
                        while (c + len < cnt && (p.perm[row0 + c + len] / p.k) / p.cb == blk) ++len;
                        const int ntok = min(p.cb, p.T - blk * p.cb);
                        const int tgt = p.k * p.n_n2 * ntok;
                        if (notify(x.ctr + p.ev_cb + blk, len) == tgt && x.dynamic)
                            thread_push(x, 1, [&](int) { return task_word(ET_OP_MOE_COMBINE, blk, 0); });
                    }
                }
            }
        }
        return true;
    }

    __device__ static bool simt(const Params& p, Ctx& x, TaskDesc& d) {
        const int op = task_op(d.word), a = task_a(d.word);
        const int w = x.tid >> 5, lane = x.tid & 31;
        if (op == ET_OP_MOE_TOPK) return topk_task(p, x, d, a, w, lane);
        if (op == ET_OP_MOE_SCAN) return scan_task(p, x, d);
        if (op == ET_OP_MOE_GROUP) return group_task(p, x, d, a);
        // COMBINE
        const int t0 = a * p.cb;
        const int ntok = min(p.cb, p.T - t0);
        if (is_unfused(p)) {
            if (!group_wait(x, d, x.ctr + p.ev_grp, p.n_g, 210)) return false;
            const int mt_total = ld_volatile(p.scal);
            if (!group_wait(x, d, x.ctr + p.ev_s2_all, mt_total * p.n_n2, 211)) return false;
        } else {
            if (!group_wait(x, d, x.ctr + p.ev_cb + a, p.k * p.n_n2 * ntok, 212)) return false;
        }
        const int nv = p.hidden / 4;
        for (int i = x.tid; i < ntok * nv; i += kExecThreads) {
            const int t = t0 + i / nv, j = (i % nv) * 4;
            float4* src = reinterpret_cast<float4*>(p.Yacc + (size_t)t * p.hidden + j);
            float4 v = __ldcg(src);
            __stcg(src, make_float4(0.f, 0.f, 0.f, 0.f));
            ushort4 o;
            o.x = bf16_bits(v.x);
            o.y = bf16_bits(v.y);
            o.z = bf16_bits(v.z);
            o.w = bf16_bits(v.w);
            *reinterpret_cast<ushort4*>(p.Y + (size_t)t * p.hidden + j) = o;
        }
        group_finish_notify(x, d, nullptr, 0, 0);
        return true;
    }

    // TK(tt): logits = sum of the K-chunk partials (chunk order) + bias; top-k
    // by (value desc, index asc); softmax of the selected logits; per-group
    // tile histograms of the routed experts.
    __device__ static bool topk_task(const Params& p, Ctx& x, TaskDesc& d, int tt, int w, int lane) {
        const int* ev = x.ctr + (is_unfused(p) ? p.ev_rt_all : p.ev_rt + tt);
        const int tgt = is_unfused(p) ? p.n_tt * p.n_kc : p.n_kc;
        if (!group_wait(x, d, ev, tgt, 220)) return false;
        const int t0 = tt * p.tt;
        const int ntok = min(p.tt, p.T - t0);
        const int g0 = t0 / p.gt;
        const int ng = (ntok + p.gt - 1) / p.gt;
        int* hist = reinterpret_cast<int*>(x.simt);  // [ng][E]
        for (int i = x.tid; i < ng * p.E; i += kExecThreads) hist[i] = 0;
        exec_bar();
        for (int lt = w; lt < ntok; lt += kExecThreads / 32) {
            const int t = t0 + lt;
            float v[4];
            bool taken[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int e = lane + 32 * i;
                taken[i] = e >= p.E;
                float s = -INFINITY;
                if (e < p.E) {
                    s = 0.f;
                    for (int c = 0; c < p.n_kc; ++c) s += p.lpart[((size_t)c * p.maxT + t) * p.E + e];
                    s += p.bias[e];
                    p.logits[(size_t)t * p.E + e] = s;
                    if (p.out_logits) p.out_logits[(size_t)t * p.E + e] = s;
                }
                v[i] = s;
            }
            int seli = 0;
            float m0 = 0.f;
            float z = 0.f;
            float my_ex = 0.f;
            for (int s = 0; s < p.k; ++s) {
                float bv = -INFINITY;
                int bi = 0x7fffffff;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (!taken[i] && better(v[i], lane + 32 * i, bv, bi)) {
                        bv = v[i];
                        bi = lane + 32 * i;
                    }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                    if (better(ov, oi, bv, bi)) {
                        bv = ov;
                        bi = oi;
                    }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (bi == lane + 32 * i) taken[i] = true;
                if (s == 0) m0 = bv;
                const float ex = expf(bv - m0);
                z += ex;
                if (lane == s) {
                    seli = bi;
                    my_ex = ex;
                }
            }
            if (lane < p.k) {
                const float wt = my_ex / z;
                p.topk[(size_t)t * p.k + lane] = seli;
                p.topw[(size_t)t * p.k + lane] = wt;
                if (p.out_topk) p.out_topk[(size_t)t * p.k + lane] = seli;
                if (p.out_w) p.out_w[(size_t)t * p.k + lane] = wt;
                atomicAdd(&hist[(lt / p.gt) * p.E + seli], 1);
            }
        }
        exec_bar();
        for (int i = x.tid; i < ng * p.E; i += kExecThreads) p.gcnt[(size_t)g0 * p.E + i] = hist[i];
        const bool fired = group_finish_notify(x, d, x.ctr + p.ev_tk, 1, p.n_tt);
        if (fired && x.dynamic) group_push(x, 1, [&](int) { return task_word(ET_OP_MOE_SCAN, 0, 0); });
        return true;
    }

    // SC: counts, pair CSR (indptr), per-group offsets, m-tile CSR and the
    // m-tile -> expert map; the data-dependent counts of the expert events.
    __device__ static bool scan_task(const Params& p, Ctx& x, TaskDesc& d) {
        if (!group_wait(x, d, x.ctr + p.ev_tk, p.n_tt + p.bad_count, 230)) return false;
        int* s_cnt = reinterpret_cast<int*>(x.simt);  // [E]
        int* s_ptr = s_cnt + 128;                      // [E+1]
        int* s_tptr = s_ptr + 132;                     // [E+1]
        const int e = x.tid;
        int cnt = 0;
        if (e < p.E)
            for (int g = 0; g < p.n_g; ++g) cnt += p.gcnt[(size_t)g * p.E + e];
        if (e < p.E) s_cnt[e] = cnt;
        exec_bar();
        if (x.tid == 0) {
            int acc = 0, tacc = 0;
            for (int i = 0; i < p.E; ++i) {
                s_ptr[i] = acc;
                s_tptr[i] = tacc;
                acc += s_cnt[i];
                tacc += (s_cnt[i] + p.bm - 1) / p.bm;
            }
            s_ptr[p.E] = acc;
            s_tptr[p.E] = tacc;
            p.indptr[p.E] = acc;
            p.tindptr[p.E] = tacc;
            if (p.out_indptr) p.out_indptr[p.E] = acc;
            p.scal[0] = tacc;
            if (x.dynamic) {
                const int total = p.n_tt * p.n_kc + p.n_tt + 1 + p.n_g + tacc * (p.n_n1 + p.n_n2) + p.n_cb;
                __threadfence();
                atomicExch(x.ctr + kCtrTotal, total + 1);
            }
        }
        exec_bar();
        if (e < p.E) {
            p.counts[e] = cnt;
            p.indptr[e] = s_ptr[e];
            p.tindptr[e] = s_tptr[e];
            if (p.out_indptr) p.out_indptr[e] = s_ptr[e];
            for (int f = s_tptr[e]; f < s_tptr[e + 1]; ++f) p.mt_expert[f] = e;
            int run = s_ptr[e];
            for (int g = 0; g < p.n_g; ++g) {
                p.goff[(size_t)g * p.E + e] = run;
                run += p.gcnt[(size_t)g * p.E + e];
            }
        }
        const bool fired = group_finish_notify(x, d, x.ctr + p.ev_sc, 1, 1);
        if (fired && x.dynamic) group_push(x, p.n_g, [&](int g) { return task_word(ET_OP_MOE_GROUP, g, 0); });
        return true;
    }

    // GR(g): grouped row of each (token, slot) pair of group g (stable:
    // ascending token inside an expert), perm/pos, and the token rows copied
    // to their grouped positions; then the expert events.
    __device__ static bool group_task(const Params& p, Ctx& x, TaskDesc& d, int g) {
        if (!group_wait(x, d, x.ctr + p.ev_sc, 1, 240)) return false;
        const int t0 = g * p.gt;
        const int ntok = min(p.gt, p.T - t0);
        const int np = ntok * p.k;
        int* s_e = reinterpret_cast<int*>(x.simt);  // [128] expert of pair i
        int* s_row = s_e + 128;                      // [128] grouped row of pair i
        if (x.tid < np) s_e[x.tid] = p.topk[(size_t)t0 * p.k + x.tid];
        exec_bar();
        if (x.tid < np) {
            const int i = x.tid, e = s_e[i];
            int rank = 0;
            for (int j = 0; j < i; ++j) rank += s_e[j] == e;
            const int row = p.goff[(size_t)g * p.E + e] + rank;
            s_row[i] = row;
            const int pair = t0 * p.k + i;
            p.perm[row] = pair;
            p.pos[pair] = row;
            if (p.out_perm) p.out_perm[row] = pair;
        }
        exec_bar();
        const int nv = p.hidden / 8;  // uint4 per row
        for (int i = x.tid; i < np * nv; i += kExecThreads) {
            const int pi = i / nv, j = i % nv;
            const int t = t0 + pi / p.k;
            const uint4 v = *reinterpret_cast<const uint4*>(p.X + (size_t)t * p.hidden + j * 8);
            *reinterpret_cast<uint4*>(p.Xp + (size_t)s_row[pi] * p.hidden + j * 8) = v;
        }
        fence_proxy_async_global();  // Xp is read by TMA in stage 1
        if (!x.dynamic) {
            group_finish_notify(x, d, x.ctr + p.ev_grp, 1, p.n_g);
            return true;
        }
        group_finish_notify(x, d, nullptr, 0, 0);
        // grouping_task[g] -> E[topk[i,:]] for the tokens i of group g: one add
        // of the group's pair count per expert it touches
        if (x.tid < p.E) {
            const int e = x.tid;
            const int c = p.gcnt[(size_t)g * p.E + e];
            if (c > 0 && notify(x.ctr + p.ev_exp + e, c) == p.counts[e]) {
                const int f0 = p.tindptr[e], nf = p.tindptr[e + 1] - f0;
                thread_push(x, nf * p.n_n1, [&](int i) { return task_word(ET_OP_MOE_S1, f0 + i / p.n_n1, i % p.n_n1); });
            }
        }
        return true;
    }
};

__global__ void __launch_bounds__(kThreads, 1) moe_kernel(const __grid_constant__ MoeParams p, const RunArgs ra) {
    megakernel_body<Moe>(p, ra);
}

cudaError_t moe_setup(int* max_blocks_per_sm) {
    cudaError_t e = cudaFuncSetAttribute(moe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(max_blocks_per_sm, moe_kernel, kThreads, kSmemBytes);
}

cudaError_t launch_moe(const MoeParams& p, const RunArgs& ra, int n_ctas, cudaStream_t s) {
    moe_kernel<<<n_ctas, kThreads, kSmemBytes, s>>>(p, ra);
    return cudaGetLastError();
}

}  // namespace et
