// Launch helpers of the W4A8 GEMM kernel: ring depths per tile shape and
// the per-mode entry points (each defined in its own translation unit,
// gemm_<mode>.cu, so the instantiations compile in parallel).
#pragma once

#include <atomic>
#include <cuda_runtime.h>

#include "gemm_tc.cuh"

namespace w4a8 {

// Tensor maps of one GEMM launch: activations (3-D: k within group, row,
// group), group scales and zero-points (2-D: column, expert*G + group).
struct GemmMaps {
    CUtensorMap act, sw, z;
};

template <int BN, int GROUP, int MODE, bool DBG>
int launch_gemm_t(const GemmMaps& maps, const GemmParams& p, int grid, cudaStream_t stream) {
    using C = GemmCfg<BN, GROUP, MODE>;
    auto kern = w4a8_gemm_tc_kernel<BN, GROUP, MODE, DBG>;
    static std::atomic<uint64_t> attr_done{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_done.load() & bit)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
            return 6;
        attr_done.fetch_or(bit);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.pdl ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, kern, maps.act, maps.sw, maps.z, p) != cudaSuccess) return 6;
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

template <int MODE, bool DBG>
int launch_gemm_mode(int bn, int group, const GemmMaps& maps, const GemmParams& p, int grid,
                     cudaStream_t stream) {
    if (group == 128) {
        switch (bn) {
            case 16: return launch_gemm_t<16, 128, MODE, DBG>(maps, p, grid, stream);
            case 32: return launch_gemm_t<32, 128, MODE, DBG>(maps, p, grid, stream);
            case 64: return launch_gemm_t<64, 128, MODE, DBG>(maps, p, grid, stream);
            case 128: return launch_gemm_t<128, 128, MODE, DBG>(maps, p, grid, stream);
        }
    } else if (group == 64) {
        switch (bn) {
            case 16: return launch_gemm_t<16, 64, MODE, DBG>(maps, p, grid, stream);
            case 32: return launch_gemm_t<32, 64, MODE, DBG>(maps, p, grid, stream);
            case 64: return launch_gemm_t<64, 64, MODE, DBG>(maps, p, grid, stream);
            case 128: return launch_gemm_t<128, 64, MODE, DBG>(maps, p, grid, stream);
        }
    }
    return 2;  // W4A8_ERR_UNSUPPORTED_SHAPE
}

// Groups per request of the activation and scale / zero-point streams (the
// host encodes the tensor-map boxes with these).
inline int chunk_act(int bn, int group, int mode) {
    const int tile = bn * group;
    const int r = 32768 / tile;
    (void)mode;
    return r < 1 ? 1 : (r > 8 ? 8 : r);
}
inline int chunk_packed(int group) { return group == 128 ? 4 : 8; }
constexpr int kChunkScales = 8;

// Status codes as in w4a8.h (0 ok, 2 unsupported shape, 6 CUDA error).
int launch_gemm_plain(bool dbg, int bn, int group, const GemmMaps& maps, const GemmParams& p, int grid,
                      cudaStream_t stream);
int launch_gemm_splitk(bool dbg, int bn, int group, const GemmMaps& maps, const GemmParams& p, int grid,
                       cudaStream_t stream);
int launch_gemm_gateup(bool dbg, int bn, int group, const GemmMaps& maps, const GemmParams& p, int grid,
                       cudaStream_t stream);
int launch_gemm_down(bool dbg, int bn, int group, const GemmMaps& maps, const GemmParams& p, int grid,
                     cudaStream_t stream);

}  // namespace w4a8
