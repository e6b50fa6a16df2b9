// Launch helpers of the W4A8 GEMM kernel: ring depths per tile shape and
// the per-mode entry points (each defined in its own translation unit,
// gemm_<mode>.cu, so the instantiations compile in parallel).
#pragma once

#include <atomic>
#include <cuda_runtime.h>

#include "gemm_tc.cuh"

namespace w4a8 {

// Ring depths: SP packed-code stages (shared memory), SA activation +
// unpacked-weight stages (shared memory + TMEM), NACC TMEM partial buffers.
// TMEM columns used: NACC * BN + SA * GROUP / 4 <= 512.
template <int BN, int GROUP>
struct Stages;
template <> struct Stages<16, 128> { static constexpr int SP = 20, SA = 8, NACC = 8; };
template <> struct Stages<32, 128> { static constexpr int SP = 16, SA = 8, NACC = 8; };
template <> struct Stages<64, 128> { static constexpr int SP = 12, SA = 8, NACC = 4; };
template <> struct Stages<128, 128> { static constexpr int SP = 12, SA = 4, NACC = 3; };
template <> struct Stages<16, 64> { static constexpr int SP = 32, SA = 8, NACC = 8; };
template <> struct Stages<32, 64> { static constexpr int SP = 24, SA = 8, NACC = 8; };
template <> struct Stages<64, 64> { static constexpr int SP = 24, SA = 8, NACC = 6; };
template <> struct Stages<128, 64> { static constexpr int SP = 16, SA = 8, NACC = 3; };

template <int BN, int GROUP, int MODE, bool DBG>
int launch_gemm_t(const CUtensorMap& tmap, const GemmParams& p, int grid, cudaStream_t stream) {
    constexpr int SP = Stages<BN, GROUP>::SP, SA = Stages<BN, GROUP>::SA, NACC = Stages<BN, GROUP>::NACC;
    using C = GemmCfg<BN, GROUP, SP, SA, NACC>;
    auto kern = w4a8_gemm_tc_kernel<BN, GROUP, SP, SA, NACC, MODE, DBG>;
    static std::atomic<uint64_t> attr_done{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_done.load() & bit)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
            return 6;
        attr_done.fetch_or(bit);
    }
    kern<<<grid, kGemmThreads, C::SMEM, stream>>>(tmap, p);
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

template <int MODE, bool DBG>
int launch_gemm_mode(int bn, int group, const CUtensorMap& tmap, const GemmParams& p, int grid,
                     cudaStream_t stream) {
    if (group == 128) {
        switch (bn) {
            case 16: return launch_gemm_t<16, 128, MODE, DBG>(tmap, p, grid, stream);
            case 32: return launch_gemm_t<32, 128, MODE, DBG>(tmap, p, grid, stream);
            case 64: return launch_gemm_t<64, 128, MODE, DBG>(tmap, p, grid, stream);
            case 128: return launch_gemm_t<128, 128, MODE, DBG>(tmap, p, grid, stream);
        }
    } else if (group == 64) {
        switch (bn) {
            case 16: return launch_gemm_t<16, 64, MODE, DBG>(tmap, p, grid, stream);
            case 32: return launch_gemm_t<32, 64, MODE, DBG>(tmap, p, grid, stream);
            case 64: return launch_gemm_t<64, 64, MODE, DBG>(tmap, p, grid, stream);
            case 128: return launch_gemm_t<128, 64, MODE, DBG>(tmap, p, grid, stream);
        }
    }
    return 2;  // W4A8_ERR_UNSUPPORTED_SHAPE
}

// Status codes as in w4a8.h (0 ok, 2 unsupported shape, 6 CUDA error).
int launch_gemm_plain(bool dbg, int bn, int group, const CUtensorMap& tmap, const GemmParams& p, int grid,
                      cudaStream_t stream);
int launch_gemm_splitk(bool dbg, int bn, int group, const CUtensorMap& tmap, const GemmParams& p, int grid,
                       cudaStream_t stream);
int launch_gemm_gateup(int bn, int group, const CUtensorMap& tmap, const GemmParams& p, int grid,
                       cudaStream_t stream);
int launch_gemm_down(int bn, int group, const CUtensorMap& tmap, const GemmParams& p, int grid,
                     cudaStream_t stream);

}  // namespace w4a8
