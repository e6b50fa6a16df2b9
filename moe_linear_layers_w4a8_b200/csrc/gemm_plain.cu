// Instantiations of the W4A8 GEMM kernel for the plain output mode.
#include "gemm_launch.cuh"

namespace w4a8 {

int launch_gemm_plain(bool dbg, int bn, int group, const GemmMaps& maps, const GemmParams& p, int grid,
                      cudaStream_t stream) {
    return dbg ? launch_gemm_mode<kModePlain, true>(bn, group, maps, p, grid, stream)
               : launch_gemm_mode<kModePlain, false>(bn, group, maps, p, grid, stream);
}

}  // namespace w4a8
