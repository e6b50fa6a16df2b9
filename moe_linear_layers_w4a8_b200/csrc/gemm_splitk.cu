// Instantiations of the W4A8 GEMM kernel for the splitk output mode.
#include "gemm_launch.cuh"

namespace w4a8 {

int launch_gemm_splitk(bool dbg, int bn, int group, const GemmMaps& maps, const GemmParams& p, int grid,
                      cudaStream_t stream) {
    return dbg ? launch_gemm_mode<kModeSplitK, true>(bn, group, maps, p, grid, stream)
               : launch_gemm_mode<kModeSplitK, false>(bn, group, maps, p, grid, stream);
}

}  // namespace w4a8
