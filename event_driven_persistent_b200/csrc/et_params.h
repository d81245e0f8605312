// Kernel parameter blocks of the three megakernels (host and device).
#pragma once
#include <cuda.h>
#include <stdint.h>

#include "et_shared.h"

namespace et {

// ------------------------------------------------------------------ split-K
// Tasks: P(i, j) partial of row tile i, K-chunk j; F(i) final of row tile i.
// Events (counter-set index): E[i] = ev_base + i; unfused barrier = ev_all.
struct SplitKParams {
    const float* A;
    float* Bp;
    float* C;
    int rows, cols, chunk, tile_rows;
    int n_tiles, n_chunks;
    int ev_base, ev_all;
    int unfused;
    int bad_count;
};

// ---------------------------------------------------------------------- MLP
// Tasks: NORM(b), GU(n) gate/up tile n, DOWN(m, c), RED(m).
// Events: E_norm (count B), E_h[c] (count gu_per_chunk), E_y[m] (count
// n_chunks); unfused: E_gu_all (count n_gu), E_down_all (count n_m*n_c).
enum { MLP_MAP_WGU = 0, MLP_MAP_WD = 1, MLP_MAP_XN = 2, MLP_MAP_H = 3 };
struct MlpParams {
    CUtensorMap tm_wgu;  // Wgu [2I, H], box 64 x 64
    CUtensorMap tm_wd;   // Wd  [H, I], box 64 x 64
    CUtensorMap tm_xn;   // xn  [maxB, H] (workspace), box 64 x 16
    CUtensorMap tm_h;    // h   [maxB, I] (workspace), box 64 x 16
    CUtensorMap tm_xn64, tm_h64;  // the same, box 64 x 64 (wide_b)
    int wide_b;          // 1 = the workspaces hold 64 rows or more: 64-row boxes for wide token tiles
    const uint16_t* X;
    const uint16_t* gamma;
    uint16_t* xn;
    uint16_t* h;
    float* yacc;         // [maxB, H] fp32 sums of the down GEMM's K chunks (zero between runs)
    uint16_t* Y;
    int B, hidden, inter, maxB;
    float eps;
    int gu_tile, down_tile, kchunk;
    int n_gu, n_m, n_c, gu_per_chunk;
    int ev_norm, ev_h, ev_y, ev_gu_all, ev_down_all;
    int unfused;
    int push;            // 1 = a task that completes an event queues its consumers (dynamic schedule)
    int bad_count;
};

// ---------------------------------------------------------------------- MoE
// Tasks: RT(tt, kc) router partial (tensor core), TK(tt) top-k (and, when
// one token tile covers T, the whole grouping), SC scan, GR(g) grouping,
// S1(f, n) stage-1 tile (token rows gathered from X), S2(f, n) stage-2
// tile, CB(b) combine.
enum { MOE_MAP_WR = 0, MOE_MAP_W1 = 1, MOE_MAP_W2 = 2, MOE_MAP_X = 3, MOE_MAP_HM = 4, MOE_MAP_XP = 5 };
struct MoeParams {
    CUtensorMap tm_wr;  // Wr [E, H], box 64 x 64
    CUtensorMap tm_w1;  // W1 [E*2I, H], box 64 x 64
    CUtensorMap tm_w2;  // W2 [E*H, I], box 64 x 64
    CUtensorMap tm_x;   // X  [T, H], box 64 x 16
    CUtensorMap tm_hm;  // Hm [maxT*k, I] (workspace), box 64 x 16
    CUtensorMap tm_hm64;  // Hm, box 64 x 64 (stage-2 token tiles of 64 rows and more)
    CUtensorMap tm_xp;  // Xp [maxT*k, H] (workspace), box 64 x 16
    const uint16_t* X;
    const float* bias;
    uint16_t* Y;
    // optional exports
    int32_t* out_topk;
    float* out_w;
    int32_t* out_indptr;
    int32_t* out_perm;
    float* out_logits;
    // workspace
    float* lacc;        // [maxT, E] router logits without bias when the router's K is split:
                        // the chunk tasks add their partials (fp32 red.add), the last one
                        // reads and re-zeroes them, so it is zero between runs
    int32_t* topk;      // [maxT, k]
    float* topw;        // [maxT, k]
    int32_t* goff;      // [n_tt, E] first grouped row of tile g's pairs of expert e
    int32_t* counts;    // [E]
    int32_t* indptr;    // [E+1]
    int32_t* tindptr;   // [E+1] m-tile CSR
    int4* mt_desc;      // [F_max] flat m-tile f: (expert, first grouped row, rows, 0)
    int32_t* perm;      // [maxT*k]
    int32_t* pos;       // [maxT*k]
    int32_t* scal;      // [8]: 0 = total m-tiles, 1 = stage-2 tasks were pushed early
    uint16_t* Hm;       // [maxT*k, I] stage-1 output, grouped order
    uint16_t* Xp;       // [maxT*k, H] X rows in grouped order (null when the graph never stages them)
    int use_xp;         // this run: grouping tasks write Xp, stage 1 reads it by TMA
    float* Yacc;        // [maxT, H] fp32 combine accumulator (kept zero between runs)
    int T, hidden, inter, E, k, maxT;
    int tt, n_tt, n_kc, tkt, n_tk, bm, n1_tile, n_n1, n2_tile, n_n2, cb, n_cb;
    int f_max;          // static: m-tile slots of this bucket
    int early_max;      // dynamic: push stage-2 tasks with stage 1 when #stage-1 tasks <= this
    // events
    int ev_rt, ev_tk, ev_sc, ev_grp, ev_exp, ev_s1, ev_cb, ev_s1_all, ev_s2_all;
    int ev_gcnt;        // counter-set block [n_tt, E]: pairs of 128-token tile g per expert
    int sched;          // et_sched
    int bad_count;
    // a dense MLP after the layer (the MoE -> MLP graph; mlp_xn null otherwise):
    // each combine task also normalises its tokens' outputs for the MLP
    uint16_t* mlp_xn;          // [maxT, hidden] MLP input rows, bf16(rmsnorm(y) gamma)
    const uint16_t* mlp_gamma;
    float mlp_eps;
    int mlp_ev_norm;           // the MLP's E_norm (count T)
    int mlp_n_gu;              // gate/up tasks queued by the combine completing E_norm (0 = none)
    int extra_tasks;           // tasks of the MLP in the queue's total (dynamic schedule)
};

// ------------------------------------------------------------ decode layer
// One decode step of a transformer layer (B requests, one new token each).
// Tasks: N1(b) norm; QKV(n, c) head tile n, K chunk c (the chunk completing
// a head runs its branch: Q norm + RoPE, K norm + RoPE + cache append, V
// cache append); ATTN(b*nkv + g, s) split s of request b, KV head g (a
// stream task; the split completing (b, g) merges the splits); OPROJ(m, c)
// output tile m, K chunk = KV group c; N2(b) residual + norm; GU(n);
// DOWN(m, c); RED(m) residual + output.
enum { DEC_MAP_WQKV = 0, DEC_MAP_WO = 1, DEC_MAP_WGU = 2, DEC_MAP_WD = 3,
       DEC_MAP_XN = 4, DEC_MAP_ATTN = 5, DEC_MAP_XN2 = 6, DEC_MAP_HM = 7 };
struct DecodeParams {
    CUtensorMap tm_wqkv, tm_wo, tm_wgu, tm_wd;   // weights, box 64 x 64
    CUtensorMap tm_xn, tm_attn, tm_xn2, tm_hm;   // workspace activations, box 64 x 16
    CUtensorMap tm_kc;   // K cache as [B nkv max_ctx, hd], box 64 x 128 (this run's Kc)
    CUtensorMap tm_vt;   // V^T cache as [B nkv hd, max_ctx], box 64 x 128 (this run's Vc)
    CUtensorMap tm_q;    // q as [maxB nq, hd], box 64 x 16
    CUtensorMap tm_xn64, tm_attn64, tm_xn2_64, tm_hm64;  // workspace activations, box 64 x 64 (wide_b)
    int wide_b;          // 1 = the workspaces hold 64 rows or more: 64-row boxes for wide token tiles
    // inputs / outputs
    const uint16_t* X;
    const int32_t* pos;        // [B] tokens already cached per request (= the new token's position)
    const uint16_t *g1, *gq, *gk, *g2;
    uint16_t *Kc, *Vc;         // K cache [B, nkv, max_ctx, hd], V^T cache [B, nkv, hd, max_ctx] (appended in place)
    uint16_t* Y;
    uint16_t* out_h1;          // optional [B, H] attention-block output (residual stream)
    uint16_t* out_q;           // optional [B, nq*hd] rotated queries
    // workspace
    uint16_t* xn;              // [maxB, H]
    float* qkvacc;             // [maxB, nqkv*hd] K-chunk sums (zero between runs)
    uint16_t* q;               // [maxB, nq, hd] rotated queries
    float2* rope;              // [maxB, hd/2] (cos, sin) of each request's position, per frequency
    float* part;               // [maxB*nkv, S_max, grp, hd + 2] split partials (o, m, l)
    uint16_t* attn;            // [maxB, nq*hd] attention output (o-proj B operand)
    float* h1acc;              // [maxB, H] o-proj sums (zero between runs)
    uint16_t* h1;              // [maxB, H]
    uint16_t* xn2;             // [maxB, H]
    uint16_t* hm;              // [maxB, I]
    float* yacc;               // [maxB, H] down-projection sums (zero between runs)
    int B, maxB, hidden, inter, nq, nkv, hd, grp, max_ctx, split, s_max;
    float eps;
    double rope_base;
    int n_kc, n_heads;         // QKV K chunks, head tiles (nq + 2 nkv)
    int gu_tile, kchunk, n_gu, n_m, n_c, gu_per_chunk, o_kc;  // MLP tiles; o-proj K chunk (grp*hd)
    // events
    int ev_n1, ev_qkv, ev_g, ev_att, ev_ag, ev_o, ev_n2, ev_h, ev_y;
    int ev_branch_all, ev_merge_all, ev_gu_all, ev_down_all;
    int sched;
    int bad_count;
};

// ------------------------------------------------------ MoE -> dense MLP
// The MoE layer followed by a dense SwiGLU MLP on its output, in one launch
// (the MLP's gate/up, down and reduce tasks; its norm is run by the MoE's
// combine tasks).
struct MoeMlpParams {
    MoeParams moe;
    MlpParams mlp;
};

}  // namespace et
