// Instantiations and launch of the W4A16 GEMM kernel.
#include <atomic>
#include <cuda_runtime.h>

#include "gemm_w4a16.cuh"

namespace w4a8 {

template <int BN, bool SPLIT, bool SYM>
static int launch_w4a16_t(const CUtensorMap& tmap_x, const CUtensorMap& tmap_s, const CUtensorMap& tmap_z,
                          const W16Params& p, int grid, cudaStream_t stream) {
    using C = W16Cfg<BN>;
    auto kern = w4a16_gemm_kernel<BN, SPLIT, SYM>;
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
    cfg.blockDim = dim3(kW16Threads);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tmap_x, tmap_s, tmap_z, p) != cudaSuccess) return 6;
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

template <int BN>
static int launch_w4a16_bn(bool split, bool sym, const CUtensorMap& tx, const CUtensorMap& ts, const CUtensorMap& tz,
                           const W16Params& p, int grid, cudaStream_t stream) {
    if (split) return sym ? launch_w4a16_t<BN, true, true>(tx, ts, tz, p, grid, stream)
                          : launch_w4a16_t<BN, true, false>(tx, ts, tz, p, grid, stream);
    return sym ? launch_w4a16_t<BN, false, true>(tx, ts, tz, p, grid, stream)
               : launch_w4a16_t<BN, false, false>(tx, ts, tz, p, grid, stream);
}

int launch_w4a16(int bn, bool split, bool sym, const CUtensorMap& tx, const CUtensorMap& ts, const CUtensorMap& tz,
                 const W16Params& p, int grid, cudaStream_t stream) {
    switch (bn) {
        case 16: return launch_w4a16_bn<16>(split, sym, tx, ts, tz, p, grid, stream);
        case 32: return launch_w4a16_bn<32>(split, sym, tx, ts, tz, p, grid, stream);
        case 64: return launch_w4a16_bn<64>(split, sym, tx, ts, tz, p, grid, stream);
        case 128: return launch_w4a16_bn<128>(split, sym, tx, ts, tz, p, grid, stream);
        case 256: return launch_w4a16_bn<256>(split, sym, tx, ts, tz, p, grid, stream);
    }
    return 2;
}

}  // namespace w4a8
