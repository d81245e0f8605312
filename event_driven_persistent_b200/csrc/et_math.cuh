// Element-wise helpers shared by the workload task code (device only).
#pragma once
#include <cuda_bf16.h>

#include "et_engine.cuh"

namespace et {

// fp32 -> bf16 bits, round to nearest even
__device__ __forceinline__ uint16_t bf16_bits(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }
__device__ __forceinline__ float bf16_val(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }
// eight bf16 values (one 16-byte load) -> fp32
__device__ __forceinline__ void bf16x8(uint4 u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}
// 4 bf16 (8 bytes) -> fp32
__device__ __forceinline__ void bf16x4(uint2 u, float* f) {
    const uint16_t* e = reinterpret_cast<const uint16_t*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = bf16_val(e[i]);
}
__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }
// fp32 add at L2 (fire and forget)
__device__ __forceinline__ void red_add(float* p, float v) {
    asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}
// Four consecutive fp32 sums at L2 in one request (p 16-byte aligned).
__device__ __forceinline__ void red_add4(float* p, float4 v) {
    asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
                 : "memory");
}

// Exclusive prefix sum over the 128 exec threads (value v of thread tid);
// returns the prefix, *total gets the sum.  `tmp` holds 4 ints of smem.
__device__ __forceinline__ int exec_scan(int v, int tid, int* tmp, int* total) {
    const int lane = tid & 31, w = tid >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) tmp[w] = inc;
    exec_bar();
    int base = 0, tot = 0;
#pragma unroll
    for (int i = 0; i < kExecThreads / 32; ++i) {
        base += i < w ? tmp[i] : 0;
        tot += tmp[i];
    }
    exec_bar();
    *total = tot;
    return base + inc - v;
}

// SwiGLU epilogue of a 128-row gate/up tile (rows 0..63 gate, 64..127 up,
// of 64 consecutive output columns) for accumulator columns (tokens)
// [c0, c0 + 16): h[t][col] = bf16(silu(gate) * up) for the first `nt`
// of those tokens, stored at out + t * ld + col.  Gate and up go through
// smem ([64][17] each, at the exec scratch); then thread (token, 8-column
// group) stores 16 bytes.  Releases the accumulator after the last chunk
// (c0 + 16 >= n).  `out` points at the chunk's first token row.  All 128
// exec threads call.
__device__ __forceinline__ void swiglu_tokens16(Ctx& x, uint32_t taddr, int c0, int n, uint64_t* acc_empty,
                                                uint16_t* out, int ld, int nt) {
    const int w = x.tid >> 5, lane = x.tid & 31;
    const int r = ((w + kExecWarp0) & 3) * 32 + lane;
    float v[16];
    acc_load16(taddr, c0, v);
    if (c0 + 16 >= n) acc_release(acc_empty);
    float* st = x.epi + (r >> 6) * (64 * 17) + (r & 63) * 17;  // gate rows, then up rows
#pragma unroll
    for (int i = 0; i < 16; ++i) st[i] = v[i];
    exec_bar();
    const int t = x.tid >> 3, cg = (x.tid & 7) * 8;
    if (t < nt) {
        const float* sg = x.epi + cg * 17 + t;
        const float* su = sg + 64 * 17;
        uint4 o;
        uint16_t* oo = reinterpret_cast<uint16_t*>(&o);
#pragma unroll
        for (int e = 0; e < 8; ++e) oo[e] = bf16_bits(silu(sg[e * 17]) * su[e * 17]);
        *reinterpret_cast<uint4*>(out + (size_t)t * ld + cg) = o;
    }
    exec_bar();
}

}  // namespace et
