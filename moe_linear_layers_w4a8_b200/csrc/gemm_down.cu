// Instantiations of the W4A8 GEMM kernel for the down output mode.
#include "gemm_launch.cuh"

namespace w4a8 {

int launch_gemm_down(bool dbg, int bn, int group, const GemmMaps& maps, const GemmParams& p, int grid,
                      cudaStream_t stream) {
    return dbg ? launch_gemm_mode<kModeDown, true>(bn, group, maps, p, grid, stream)
               : launch_gemm_mode<kModeDown, false>(bn, group, maps, p, grid, stream);
}

}  // namespace w4a8
