// Fused decode MLP megakernel: RMSNorm -> gate/up GEMM + SiLU*mul -> down
// GEMM split along K -> final reduce, one launch, batch B at run time.
//
// "Event Tensor：用“事件张量”编译动态 Megakernel", §端到端低 batch serving
// (the decoding pipeline fuses Norm and MLP; weights of the next stage are
// prefetched before its activations arrive) and §Split-K reduction 示例
// (the down GEMM's K-split partials and their final reduce).
//
// Task graph (event counts in brackets):
//   NORM b          --"b->"-->   E_norm [B]          (a symbolic-shape count)
//   E_norm          --"->n"-->   GU n                (64 gate + 64 up rows)
//   GU n            --"n->c"-->  E_h[c] [kchunk/64]  (c = 64n / kchunk)
//   E_h[c]          --"mc->c"--> DOWN (m, c)         (128 output rows, K chunk c)
//   DOWN (m, c)     --"mc->m"--> E_y[m] [#chunks]   (partial sums added at L2 into yacc)
//   E_y[m]          --"m->m"-->  RED m               (Y = bf16(yacc), yacc back to zero)
// GEMMs run on tcgen05 with swap-AB: the weight rows are the M = 128 side,
// the B tokens (rounded up to 16) are N, so one tile shape serves every B.
#pragma once
#include "et_math.cuh"
#include "et_params.h"

namespace et {

struct Mlp : WorkloadBase {
    using Params = MlpParams;
    static constexpr bool kGemm = true;

    __device__ static uint32_t fetch_init(const Params&, int idx) { return task_word(ET_OP_MLP_NORM, idx, 0); }

    __device__ static bool derive(const Params& p, Ctx&, TaskDesc& d) {
        const int op = task_op(d.word), a = task_a(d.word), b = task_b(d.word);
        d.valid = 1;
        d.gemm = 0;
        const int n = (p.B + 15) & ~15;
        if (op == ET_OP_MLP_NORM) {
            d.valid = a < p.B;
        } else if (op == ET_OP_MLP_GATEUP) {
            d.gemm = 1;
            d.a_map = MLP_MAP_WGU;
            d.a_row0 = a * p.gu_tile;
            d.a_row1 = p.inter + a * p.gu_tile;
            d.b_map = MLP_MAP_XN;
            d.b_row0 = 0;
            d.n = n;
            d.k0 = 0;
            d.nk = p.hidden / kTileK;
        } else if (op == ET_OP_MLP_DOWN) {
            d.gemm = 1;
            d.a_map = MLP_MAP_WD;
            d.a_row0 = a * p.down_tile;
            d.a_row1 = a * p.down_tile + 64;
            d.b_map = MLP_MAP_H;
            d.b_row0 = 0;
            d.n = n;
            d.k0 = b * p.kchunk;
            d.nk = p.kchunk / kTileK;
        }
        return true;
    }

    __device__ static const uint16_t* gather_row(const Params&, const TaskDesc&, int) { return nullptr; }
    __device__ static bool gemm_wait(const Params& p, Ctx& x, TaskDesc& d) {
        const int op = task_op(d.word);
        if (op == ET_OP_MLP_GATEUP)
            return wait_geq(x.ctr + p.ev_norm, p.B + p.bad_count, x.ctl, x.timeout_ns, 100, 0);
        const int c = task_b(d.word);
        if (p.unfused) return wait_geq(x.ctr + p.ev_gu_all, p.n_gu, x.ctl, x.timeout_ns, 101, 0);
        return wait_geq(x.ctr + p.ev_h + c, p.gu_per_chunk, x.ctl, x.timeout_ns, 102, c);
    }

    __device__ static const CUtensorMap* a_map(const Params& p, int id) {
        return id == MLP_MAP_WGU ? &p.tm_wgu : &p.tm_wd;
    }
    __device__ static const CUtensorMap* b_map(const Params& p, int id) {
        return id == MLP_MAP_XN ? &p.tm_xn : &p.tm_h;
    }
    __device__ static const CUtensorMap* b_map_wide(const Params& p, int id) {
        return !p.wide_b ? nullptr : (id == MLP_MAP_XN ? &p.tm_xn64 : &p.tm_h64);
    }

    __device__ static bool epilogue(const Params& p, Ctx& x, TaskDesc& d, uint32_t taddr, uint64_t* acc_empty) {
        const int op = task_op(d.word), a = task_a(d.word), c = task_b(d.word);
        const int w = x.tid >> 5, lane = x.tid & 31;
        const int q = (w + kExecWarp0) & 3;  // TMEM lane quadrant of this warp
        const int r = q * 32 + lane;          // accumulator row (lane) held by this thread
        if (op == ET_OP_MLP_GATEUP) {
            // rows 0..63 = gate, 64..127 = up, of intermediate columns a*64 + (r & 63)
            for (int c0 = 0; c0 < d.n; c0 += 16)
                swiglu_tokens16(x, taddr, c0, d.n, acc_empty, p.h + (size_t)c0 * p.inter + a * p.gu_tile, p.inter,
                                p.B - c0);
            fence_proxy_async_global();  // h is read by TMA in the down tasks
            int* ev = x.ctr + (p.unfused ? p.ev_gu_all : p.ev_h + (a * p.gu_tile) / p.kchunk);
            const int tgt = p.unfused ? p.n_gu : p.gu_per_chunk;
            const bool fired = group_finish_notify(x, d, ev, 1, tgt);
            if (fired && p.push) {
                const int cc = (a * p.gu_tile) / p.kchunk;
                group_push(x, p.n_m, [&](int m) { return task_word(ET_OP_MLP_DOWN, m, cc); });
            }
        } else {
            // DOWN: row r = output column a*128 + r; columns = tokens.  The
            // K chunk's partial sums are added at L2 (a warp adds 32
            // consecutive columns of one token per instruction).
            const int col = a * p.down_tile + r;
            for (int c0 = 0; c0 < d.n; c0 += 16) {
                float v[16];
                acc_load16(taddr, c0, v);
                if (c0 + 16 >= d.n) acc_release(acc_empty);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int b = c0 + i;
                    if (b < p.B) red_add(p.yacc + (size_t)b * p.hidden + col, v[i]);
                }
            }
            int* ev = x.ctr + (p.unfused ? p.ev_down_all : p.ev_y + a);
            const int tgt = p.unfused ? p.n_m * p.n_c : p.n_c;
            const bool fired = group_finish_notify(x, d, ev, 1, tgt);
            if (fired && p.push) group_push(x, 1, [&](int) { return task_word(ET_OP_MLP_REDUCE, a, 0); });
        }
        return true;
    }

    __device__ static bool simt(const Params& p, Ctx& x, TaskDesc& d) {
        const int op = task_op(d.word), a = task_a(d.word);
        if (op == ET_OP_MLP_NORM) {
            if (!group_wait(x, d, nullptr, 0, 103)) return false;
            const uint16_t* xr = p.X + (size_t)a * p.hidden;
            float* red = reinterpret_cast<float*>(x.simt);
            float ss = 0.f;
            for (int i = x.tid * 8; i < p.hidden; i += kExecThreads * 8) {
                uint4 u = *reinterpret_cast<const uint4*>(xr + i);
                const uint16_t* e = reinterpret_cast<const uint16_t*>(&u);
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    float f = bf16_val(e[t]);
                    ss += f * f;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if ((x.tid & 31) == 0) red[x.tid >> 5] = ss;
            exec_bar();
            float tot = 0.f;
            for (int i = 0; i < kExecThreads / 32; ++i) tot += red[i];
            const float inv = 1.0f / sqrtf(tot / (float)p.hidden + p.eps);
            uint16_t* out = p.xn + (size_t)a * p.hidden;
            for (int i = x.tid * 8; i < p.hidden; i += kExecThreads * 8) {
                uint4 u = *reinterpret_cast<const uint4*>(xr + i);
                uint4 gm = *reinterpret_cast<const uint4*>(p.gamma + i);
                const uint16_t* e = reinterpret_cast<const uint16_t*>(&u);
                const uint16_t* gg = reinterpret_cast<const uint16_t*>(&gm);
                uint4 o;
                uint16_t* oo = reinterpret_cast<uint16_t*>(&o);
#pragma unroll
                for (int t = 0; t < 8; ++t) oo[t] = bf16_bits(bf16_val(e[t]) * inv * bf16_val(gg[t]));
                *reinterpret_cast<uint4*>(out + i) = o;
            }
            fence_proxy_async_global();  // xn is read by TMA in the gate/up tasks
            const bool fired = group_finish_notify(x, d, x.ctr + p.ev_norm, 1, p.B);
            if (fired && p.push)
                group_push(x, p.n_gu, [&](int n) { return task_word(ET_OP_MLP_GATEUP, n, 0); });
        } else {  // RED
            const int* ev = x.ctr + (p.unfused ? p.ev_down_all : p.ev_y + a);
            const int tgt = p.unfused ? p.n_m * p.n_c : p.n_c;
            if (!group_wait(x, d, ev, tgt, 104)) return false;
            // B tokens x down_tile columns as float4: eight loads in flight
            // per thread before its stores
            const int nv = p.down_tile / 4, total = p.B * nv;
            for (int base = x.tid; base < total; base += kExecThreads * 8) {
                float4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = base + u * kExecThreads;
                    if (i < total)
                        v[u] = __ldcg(reinterpret_cast<const float4*>(p.yacc + (size_t)(i / nv) * p.hidden +
                                                                      a * p.down_tile) + i % nv);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = base + u * kExecThreads;
                    if (i < total) {
                        const size_t off = (size_t)(i / nv) * p.hidden + a * p.down_tile + (i % nv) * 4;
                        __stcg(reinterpret_cast<float4*>(p.yacc + off), make_float4(0.f, 0.f, 0.f, 0.f));
                        ushort4 o;
                        o.x = bf16_bits(v[u].x);
                        o.y = bf16_bits(v[u].y);
                        o.z = bf16_bits(v[u].z);
                        o.w = bf16_bits(v[u].w);
                        *reinterpret_cast<ushort4*>(p.Y + off) = o;
                    }
                }
            }
            group_finish_notify(x, d, nullptr, 0, 0);
        }
        return true;
    }
};

}  // namespace et
