// Fused decode MLP megakernel (task code in mk_mlp.cuh).
#include "mk_mlp.cuh"

namespace et {

__global__ void __launch_bounds__(kThreads, 1) mlp_kernel(const __grid_constant__ MlpParams p, const RunArgs ra) {
    megakernel_body<Mlp>(p, ra);
}

cudaError_t mlp_setup(int* max_blocks_per_sm) {
    cudaError_t e = cudaFuncSetAttribute(mlp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(max_blocks_per_sm, mlp_kernel, kThreads, kSmemBytes);
}

cudaError_t launch_mlp(const MlpParams& p, const RunArgs& ra, int n_ctas, cudaStream_t s) {
    // the launch's own status (not an unrelated error left pending earlier)
    void* args[] = {const_cast<MlpParams*>(&p), const_cast<RunArgs*>(&ra)};
    return cudaLaunchKernel(reinterpret_cast<const void*>(mlp_kernel), dim3(n_ctas), dim3(kThreads), args, kSmemBytes, s);
}

}  // namespace et
