// MoE layer megakernel (task code in mk_moe.cuh).
#include "mk_moe.cuh"

namespace et {

__global__ void __launch_bounds__(kThreadsGather, 1) moe_kernel(const __grid_constant__ MoeParams p, const RunArgs ra) {
    megakernel_body<Moe>(p, ra);
}

cudaError_t moe_setup(int* max_blocks_per_sm) {
    cudaError_t e = cudaFuncSetAttribute(moe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(max_blocks_per_sm, moe_kernel, kThreadsGather, kSmemBytes);
}

cudaError_t launch_moe(const MoeParams& p, const RunArgs& ra, int n_ctas, cudaStream_t s) {
    // the launch's own status (not an unrelated error left pending earlier)
    void* args[] = {const_cast<MoeParams*>(&p), const_cast<RunArgs*>(&ra)};
    return cudaLaunchKernel(reinterpret_cast<const void*>(moe_kernel), dim3(n_ctas), dim3(kThreadsGather), args, kSmemBytes, s);
}

}  // namespace et
