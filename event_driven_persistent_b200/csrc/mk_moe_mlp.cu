// MoE layer -> dense MLP megakernel: the MoE layer (router, grouping, two
// grouped GEMMs, combine) followed by a dense SwiGLU MLP on its output, in
// one launch, T at run time.
//
// "Event Tensor：用“事件张量”编译动态 Megakernel", §端到端低 batch serving:
// the MoE GroupGEMM and the dense MLP GEMM are pipelined across stages, and
// the next stage's weights are prefetched before its activations arrive.
// Here each combine task of the MoE (block b of tokens) also takes the
// MLP's RMSNorm of its tokens and notifies the MLP's E_norm (count T); the
// MLP's gate/up tasks stream their first weight stages before waiting on
// E_norm, so the dense weights move while the MoE's last expert tiles and
// combines finish:
//   MoE ... -> CB(b) [+ MLP norm of block b] -> E_norm [T] -> GU(n) -> E_h[c]
//           -> DOWN(m, c) -> E_y[m] -> RED(m)
#include "mk_mlp.cuh"
#include "mk_moe.cuh"

namespace et {

struct MoeMlp : WorkloadBase {
    using Params = MoeMlpParams;
    static constexpr bool kGemm = true;
    static constexpr bool kGather = true;
    static constexpr int kMlpMaps = 8;  // MLP tensor-map ids are offset by this

    __device__ static bool is_mlp(uint32_t word) {
        const int op = task_op(word);
        return op >= ET_OP_MLP_NORM && op <= ET_OP_MLP_REDUCE;
    }
    __device__ static uint32_t fetch_init(const Params& p, int idx) { return Moe::fetch_init(p.moe, idx); }
    __device__ static bool derive(const Params& p, Ctx& x, TaskDesc& d) {
        if (!is_mlp(d.word)) return Moe::derive(p.moe, x, d);
        const bool ok = Mlp::derive(p.mlp, x, d);
        d.a_map += kMlpMaps;
        d.b_map += kMlpMaps;
        return ok;
    }
    __device__ static const uint16_t* gather_row(const Params& p, const TaskDesc& d, int r) {
        return Moe::gather_row(p.moe, d, r);
    }
    __device__ static bool gemm_wait(const Params& p, Ctx& x, TaskDesc& d) {
        return is_mlp(d.word) ? Mlp::gemm_wait(p.mlp, x, d) : Moe::gemm_wait(p.moe, x, d);
    }
    __device__ static const CUtensorMap* a_map(const Params& p, int id) {
        return id >= kMlpMaps ? Mlp::a_map(p.mlp, id - kMlpMaps) : Moe::a_map(p.moe, id);
    }
    __device__ static const CUtensorMap* b_map_wide(const Params& p, int id) {
        return id >= kMlpMaps ? Mlp::b_map_wide(p.mlp, id - kMlpMaps) : Moe::b_map_wide(p.moe, id);
    }
    __device__ static const CUtensorMap* b_map(const Params& p, int id) {
        return id >= kMlpMaps ? Mlp::b_map(p.mlp, id - kMlpMaps) : Moe::b_map(p.moe, id);
    }
    __device__ static bool epilogue(const Params& p, Ctx& x, TaskDesc& d, uint32_t taddr, uint64_t* acc_empty) {
        return is_mlp(d.word) ? Mlp::epilogue(p.mlp, x, d, taddr, acc_empty)
                              : Moe::epilogue(p.moe, x, d, taddr, acc_empty);
    }
    __device__ static bool simt(const Params& p, Ctx& x, TaskDesc& d) {
        return is_mlp(d.word) ? Mlp::simt(p.mlp, x, d) : Moe::simt(p.moe, x, d);
    }
};

__global__ void __launch_bounds__(kThreadsGather, 1) moe_mlp_kernel(const __grid_constant__ MoeMlpParams p, const RunArgs ra) {
    megakernel_body<MoeMlp>(p, ra);
}

cudaError_t moe_mlp_setup(int* max_blocks_per_sm) {
    cudaError_t e = cudaFuncSetAttribute(moe_mlp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(max_blocks_per_sm, moe_mlp_kernel, kThreadsGather, kSmemBytes);
}

cudaError_t launch_moe_mlp(const MoeMlpParams& p, const RunArgs& ra, int n_ctas, cudaStream_t s) {
    // the launch's own status (not an unrelated error left pending earlier)
    void* args[] = {const_cast<MoeMlpParams*>(&p), const_cast<RunArgs*>(&ra)};
    return cudaLaunchKernel(reinterpret_cast<const void*>(moe_mlp_kernel), dim3(n_ctas), dim3(kThreadsGather), args,
                            kSmemBytes, s);
}

}  // namespace et
