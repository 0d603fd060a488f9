// gemm.cu -- tensor-core grouped GEMM path of the NVFP4 MoE layer (tcgen05, sm_100a).
#include "moe.cuh"

namespace nvfp4 {

int gemm_tile_n() { return 128; }

int launch_gemm_gateup(const MoeArgs &, cudaStream_t) { return NVFP4_EINVAL; }
int launch_gemm_down(const MoeArgs &, cudaStream_t) { return NVFP4_EINVAL; }

}  // namespace nvfp4
