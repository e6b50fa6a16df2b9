// Instantiations and launch of the W8A8 GEMM kernel.
#include <atomic>
#include <cuda_runtime.h>

#include "gemm_w8a8.cuh"

namespace w4a8 {

template <int BN, bool SPLIT>
static int launch_w8a8_t(const CUtensorMap& tmap_w, const CUtensorMap& tmap_x, const W8Params& p, int grid,
                         cudaStream_t stream) {
    using C = W8Cfg<BN>;
    auto kern = w8a8_gemm_kernel<BN, SPLIT>;
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
    cfg.blockDim = dim3(kW8Threads);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tmap_w, tmap_x, p) != cudaSuccess) return 6;
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

int launch_w8a8(int bn, bool split, const CUtensorMap& tmap_w, const CUtensorMap& tmap_x, const W8Params& p,
                int grid, cudaStream_t stream) {
#define W4A8_W8(B)                                                                          \
    case B:                                                                                 \
        return split ? launch_w8a8_t<B, true>(tmap_w, tmap_x, p, grid, stream)              \
                     : launch_w8a8_t<B, false>(tmap_w, tmap_x, p, grid, stream);
    switch (bn) {
        W4A8_W8(16) W4A8_W8(32) W4A8_W8(64) W4A8_W8(128) W4A8_W8(256)
    }
#undef W4A8_W8
    return 2;
}

}  // namespace w4a8
