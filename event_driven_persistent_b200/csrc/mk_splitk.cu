// Split-K two-stage reduction megakernel.
//
// "Event Tensor：用“事件张量”编译动态 Megakernel", §Split-K reduction 示例:
//   B[i,j] = sum_{k=32j}^{32j+31} A[i,k],   C[i] = sum_j B[i,j]
// One event per 32-row tile, E = ETensor((n,), wait_count=#chunks); the
// partial task (i, j) notifies E[i] ("ij->i"), the final task i waits on
// E[i] ("i->i") and can run as soon as its own row tile is done, without
// waiting for the other rows.  n follows the run-time row count.
#include "et_engine.cuh"
#include "et_params.h"

namespace et {

struct SplitK : WorkloadBase {
    using Params = SplitKParams;
    static constexpr bool kGemm = false;

    __device__ static int target(const Params& p, int i) { return p.n_chunks + (p.bad_count && i == 0 ? 1 : 0); }

    __device__ static uint32_t fetch_init(const Params& p, int idx) {
        return task_word(ET_OP_SK_PARTIAL, idx / p.n_chunks, idx % p.n_chunks);
    }

    __device__ static bool derive(const Params& p, Ctx& x, TaskDesc& d) {
        d.valid = task_a(d.word) < p.n_tiles;  // static slots beyond this run's rows do nothing
        d.gemm = 0;
        return true;
    }
    __device__ static const uint16_t* gather_row(const Params&, const TaskDesc&, int) { return nullptr; }
    __device__ static bool gemm_wait(const Params&, Ctx&, TaskDesc&) { return true; }
    __device__ static const CUtensorMap* a_map(const Params&, int) { return nullptr; }
    __device__ static const CUtensorMap* b_map(const Params&, int) { return nullptr; }
    __device__ static bool epilogue(const Params&, Ctx&, TaskDesc&, uint32_t, uint64_t*) { return false; }

    __device__ static bool simt(const Params& p, Ctx& x, TaskDesc& d) {
        const int op = task_op(d.word), i = task_a(d.word);
        const int r0 = i * p.tile_rows;
        const int nr = min(p.tile_rows, p.rows - r0);
        const int warp = x.tid >> 5, lane = x.tid & 31;
        if (op == ET_OP_SK_PARTIAL) {
            const int j = task_b(d.word);
            if (!group_wait(x, d, nullptr, 0, 0)) return false;  // no input event
            const int c0 = j * p.chunk;
            const int nc = min(p.chunk, p.cols - c0);
            // four threads per row, each summing columns q*8 .. q*8+7 of every
            // 32-column block of the chunk (independent loads), then two shuffles
            const int q = lane & 3;
            for (int rb = 0; rb < nr; rb += kExecThreads / 4) {
                const int r = rb + (x.tid >> 2);
                float s = 0.f;
                if (r < nr) {
                    const float* row = p.A + (size_t)(r0 + r) * p.cols + c0;
                    for (int cb = 0; cb < nc; cb += 32) {
                        float v[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int c = cb + q * 8 + e;
                            v[e] = c < nc ? row[c] : 0.f;
                        }
#pragma unroll
                        for (int e = 0; e < 8; ++e) s += v[e];
                    }
                }
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                s += __shfl_xor_sync(0xffffffffu, s, 2);
                if (r < nr && q == 0) p.Bp[(size_t)(r0 + r) * p.n_chunks + j] = s;
            }
            int* ev = x.ctr + (p.unfused ? p.ev_all : p.ev_base + i);
            const int tgt = p.unfused ? p.n_tiles * p.n_chunks : target(p, i);
            const bool fired = group_finish_notify(x, d, ev, 1, tgt);
            if (fired && x.dynamic) group_push(x, 1, [&](int) { return task_word(ET_OP_SK_FINAL, i, 0); });
        } else {
            const int* ev = x.ctr + (p.unfused ? p.ev_all : p.ev_base + i);
            const int tgt = p.unfused ? p.n_tiles * p.n_chunks : target(p, i);
            if (!group_wait(x, d, ev, tgt, 1)) return false;
            for (int r = x.tid; r < nr; r += kExecThreads) {
                const float* b = p.Bp + (size_t)(r0 + r) * p.n_chunks;
                float s = 0.f;
                for (int j = 0; j < p.n_chunks; ++j) s += __ldcg(b + j);  // partials of other SMs: via L2
                p.C[r0 + r] = s;
            }
            group_finish_notify(x, d, nullptr, 0, 0);
        }
        return true;
    }
};

__global__ void __launch_bounds__(kThreads, 1) splitk_kernel(const __grid_constant__ SplitKParams p, const RunArgs ra) {
    megakernel_body<SplitK>(p, ra);
}

// Called once per graph on its device: opt in to the shared-memory size.
cudaError_t splitk_setup(int* max_blocks_per_sm) {
    cudaError_t e = cudaFuncSetAttribute(splitk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemNoArenaBytes);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(max_blocks_per_sm, splitk_kernel, kThreads, kSmemNoArenaBytes);
}

// The two-launch control: the same two operators as plain kernels, one
// launch each, ordered only by the stream (kernel-per-operator execution).
// Partial kernel: one warp per (row, chunk); final kernel: one thread per row.
__global__ void splitk_partial_kernel(const float* A, int rows, int cols, int chunk, int nch, float* Bp) {
    const int gw = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
    if (gw >= rows * nch) return;
    const int r = gw / nch, j = gw % nch, c0 = j * chunk, nc = min(chunk, cols - c0);
    const float* row = A + (size_t)r * cols + c0;
    float s = 0.f;
    for (int c = lane; c < nc; c += 32) s += row[c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) Bp[(size_t)r * nch + j] = s;
}
__global__ void splitk_final_kernel(const float* Bp, int rows, int nch, float* C) {
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    float s = 0.f;
    for (int j = 0; j < nch; ++j) s += Bp[(size_t)r * nch + j];
    C[r] = s;
}
cudaError_t launch_splitk_two(const float* A, int rows, int cols, int chunk, float* Bp, float* C, cudaStream_t s) {
    const int nch = (cols + chunk - 1) / chunk;
    const long warps = (long)rows * nch;
    (void)cudaGetLastError();  // an earlier, unrelated non-sticky error is not this launch's
    splitk_partial_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, s>>>(A, rows, cols, chunk, nch, Bp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    splitk_final_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(Bp, rows, nch, C);
    return cudaGetLastError();
}

cudaError_t launch_splitk(const SplitKParams& p, const RunArgs& ra, int n_ctas, cudaStream_t s) {
    // the launch's own status (not an unrelated error left pending earlier)
    void* args[] = {const_cast<SplitKParams*>(&p), const_cast<RunArgs*>(&ra)};
    return cudaLaunchKernel(reinterpret_cast<const void*>(splitk_kernel), dim3(n_ctas), dim3(kThreads), args, kSmemNoArenaBytes, s);
}

}  // namespace et
