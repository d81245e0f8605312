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

}  // namespace et
