// W8A8 GEMM on the sm_100a tensor cores: INT8 weights with one scale per
// output channel, INT8 activations with one scale per token
// ("Inference Quantization ch.1" §4 ideal path and §8.3):
//   acc[m,n] = sum_k q_x[m,k] q_w[k,n]        exact int32 over all of K
//   y[m,n]   = s_x[m] * (s_w[n] * acc[m,n])   fp32, one bf16 rounding
//
// Compared with the W4A8 kernel there is nothing to unpack and no per-group
// rescale: both operands go from HBM to shared memory by TMA exactly as the
// MMA reads them, the int32 accumulator stays in TMEM for the whole K range,
// and the epilogue runs once per tile.
//   * Swap-AB like the W4A8 kernel: the 128 MMA rows are weight output
//     columns (A = q_w, stored [N][K] so a tile is one 2-D TMA box), the MMA N
//     dimension is BN tokens (B = q_x [M][K]).  Each epilogue thread owns one
//     weight column, so s_w[n] is a per-thread scalar.
//   * Warp 0 streams k-blocks of 128 (a weight box and an activation box per
//     stage), one lane of warp 1 issues four MMAs per k-block (the first MMA of
//     a tile range starts the accumulator), warps 2-5 drain the accumulator.
//     Two TMEM accumulators alternate, so a range's epilogue overlaps the
//     next range's MMAs.
//   * Persistent ranges of (tile, k-block) units as in the W4A8 kernel; when
//     ranges split a tile, contributors store their int32 partial tiles with
//     an epoch flag and the CTA holding the tile's first k-blocks adds them
//     (integer sums: exact in any order).  The same bounded waits and
//     abort/drain paths as the W4A8 kernel.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace w4a8 {

struct W8Params {
    int N, K, M;
    int n_tiles, m_tiles, KB;    // KB = K / 128 k-blocks
    long long units_per_cta;     // Q
    const float* s_w;            // [N]
    const float* s_x;            // [M]
    uint16_t* Y;
    int ldy;
    int vec16;                   // Y and ldy allow 16-byte row stores
    int32_t* partial;            // split: int32 partial tiles [tiles][slots][BN][128]
    int slots;
    unsigned long long* flags;   // split: [tiles][slots]
    unsigned long long epoch;
    int32_t* status;
    unsigned long long wait_ns;
};

constexpr int kW8Threads = 192;  // producer, MMA, 4 epilogue warps
constexpr int kW8EpiWarp0 = 2;

template <int BN>
struct W8Cfg {
    static constexpr int A_STAGE = 128 * 128;              // weight box: 128 columns x 128 k
    static constexpr int B_STAGE = BN * 128;                // activation box: BN tokens x 128 k
    static constexpr int STAGE = A_STAGE + B_STAGE;
    static constexpr int NST_RAW = (196 * 1024) / STAGE;
    static constexpr int NST = NST_RAW > 8 ? 8 : NST_RAW;  // pipeline stages
    static constexpr int ACC_COLS = 2 * BN;                 // two accumulators
    static constexpr uint32_t TMEM_COLS = ACC_COLS <= 32 ? 32 : ACC_COLS <= 64 ? 64 : ACC_COLS <= 128 ? 128
                                          : ACC_COLS <= 256 ? 256 : 512;
    static constexpr int YB = 32 * 128 * 2;                 // output staging: up to 32 tokens x 128 columns bf16
    static constexpr int OFF_Y = NST * STAGE;
    static constexpr int OFF_BAR = OFF_Y + YB;
    static constexpr int NUM_BARS = 2 * NST + 5;
    static constexpr int LB = BN < 32 ? BN : 32;           // accumulator columns per epilogue batch
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    static constexpr uint32_t IDESC = idesc_i8(BN);
    static_assert(BN == 16 || BN == 32 || BN == 64 || BN == 128 || BN == 256, "BN");
    static_assert(NST >= 3, "stages");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

template <int BN, bool SPLIT>
__global__ void __launch_bounds__(kW8Threads, 1)
    w8a8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                     const W8Params p) {
    using C = W8Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint16_t* sY = reinterpret_cast<uint16_t*>(smem + C::OFF_Y);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bars;                  // [NST] weight + activation boxes landed
    uint64_t* empty = full + C::NST;        // [NST] their MMAs completed
    uint64_t* acc_full = empty + C::NST;    // [2] accumulator's MMAs completed
    uint64_t* acc_empty = acc_full + 2;     // [2] drained by the 4 epilogue warps
    uint64_t* drain = acc_empty + 2;        // [1] every MMA of the CTA completed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        pdl_launch_dependents();
        for (int i = 0; i < C::NST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_x);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const WaitCtx wc{abort_flag, p.status, wait_cycles_for_ns(p.wait_ns)};

    const long long KB = p.KB;
    const long long tiles = (long long)p.m_tiles * p.n_tiles;
    const long long U = tiles * KB;
    // split-K: contiguous unit ranges; otherwise whole tiles round-robin
    const RoundRobin rrt(tiles, KB);
    const long long Q = SPLIT ? p.units_per_cta : rrt.waves * KB;
    const long long u0 = SPLIT ? min((long long)blockIdx.x * Q, U) : rrt.u0;
    const long long u1 = SPLIT ? min(u0 + Q, U) : rrt.u1;

    if (warp == 0) {
        // ------------------------------------------------------- producer --
        if (lane == 0) {
            Ring rs;
            long long issued = 0;
            bool ok = true;
            bool waited = false;
            // unit positions advance by increments (no division per unit)
            UnitPos up = SPLIT ? UnitPos(u0, KB, p.n_tiles)
                               : UnitPos(u0, KB, p.n_tiles, rrt.v0, blockIdx.x, gridDim.x);
            for (long long u = u0; u < u1 && ok; ++u, up.next(KB, p.n_tiles)) {
                const int kb = up.kb, mt = up.mt, nt = up.nt;
                if (!wait_bounded(&empty[rs.idx], rs.phase ^ 1u, wc)) { ok = false; break; }
                mbar_arrive_expect_tx(&full[rs.idx], C::STAGE);
                uint8_t* st = smem + rs.idx * C::STAGE;
                tma_load_2d(st, &tmap_w, &full[rs.idx], kb * 128, nt * 128);
                // activations may come from the kernel launched just before
                if (!waited) {
                    pdl_wait_prerequisites();
                    waited = true;
                }
                tma_load_2d(st + C::A_STAGE, &tmap_x, &full[rs.idx], kb * 128, mt * BN);
                rs.next(C::NST);
                ++issued;
            }
            WaitCtx wd = wc;
            volatile int no_abort = 0;
            wd.abort = &no_abort;
            Ring d = rs;
            for (long long k = 0; k < issued && k < C::NST; ++k) {
                ring_back(d, C::NST);
                (void)wait_bounded(&full[d.idx], d.phase, wd);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issue --
        if (lane == 0) {
            Ring rs, ra;
            bool ok = true;
            long long u = u0;
            while (u < u1 && ok) {
                const long long t = u / KB;
                const long long seg_end = min(u1, (t + 1) * KB);
                if (!wait_bounded(&acc_empty[ra.idx], ra.phase ^ 1u, wc)) { ok = false; break; }
                const uint32_t d_tmem = tmem_base + ra.idx * BN;
                for (long long v = u; v < seg_end; ++v) {
                    if (!wait_bounded(&full[rs.idx], rs.phase, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + rs.idx * C::STAGE);
                    const uint64_t adesc = umma_desc_kmajor(a_addr, 128);
                    const uint64_t bdesc = umma_desc_kmajor(a_addr + C::A_STAGE, 128);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_i8(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, C::IDESC, (v > u || kk > 0) ? 1u : 0u);
                    tc_commit(&empty[rs.idx]);
                    rs.next(C::NST);
                }
                if (!ok) break;
                tc_commit(&acc_full[ra.idx]);
                ra.next(2);
                u = seg_end;
            }
            // drain: every MMA issued above completes before TMEM is freed
            tc_commit(drain);
            WaitCtx wd = wc;
            volatile int no_abort = 0;
            wd.abort = &no_abort;
            (void)wait_bounded(drain, 0, wd);
        }
    } else {
        // ------------------------------------------------------- epilogue --
        const int q = warp & 3;                 // TMEM lane quadrant
        const int r = q * 32 + lane;            // weight row within the tile
        const int et = (warp - kW8EpiWarp0) * 32 + lane;  // 0..127
        const uint32_t lane_addr = ((uint32_t)(q * 32)) << 16;
        pdl_wait_prerequisites();
        Ring ra;
        bool ok = true;
        long long u = u0;
        while (u < u1) {
            const long long t = u / KB;
            const int kb0 = (int)(u % KB);
            const long long seg_end = min(u1, (t + 1) * KB);
            const int kb1 = (int)(seg_end - t * KB);
            const long long ta = SPLIT ? t : rrt.tile(t);
            const int mt = (int)(ta / p.n_tiles), nt = (int)(ta % p.n_tiles);
            const int n = nt * 128 + r;
            const int row0 = mt * BN;
            const int rows_valid = min(BN, p.M - row0);
            const int ncols = min(128, p.N - nt * 128);
            const bool n_valid = r < ncols;
            const float sw = n_valid ? __ldg(p.s_w + n) : 0.0f;
            ok = warp_wait_bounded(&acc_full[ra.idx], ra.phase, wc);
            if (named_bar_or(2, 128, !ok)) break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + lane_addr + ra.idx * BN;
            const bool full_tile = (kb0 == 0 && kb1 == p.KB);
            int slot = 0, nsl = 1;
            int32_t* tile_part = nullptr;
            unsigned long long* flags = nullptr;
            if constexpr (SPLIT) {
                if (!full_tile) {
                    const long long c_first = (t * KB) / Q;
                    nsl = (int)((t * KB + KB - 1) / Q - c_first) + 1;
                    slot = (int)((long long)blockIdx.x - c_first);
                    tile_part = p.partial + (t * p.slots) * (BN * 128);
                    flags = p.flags + t * p.slots;
                }
            }
            if (SPLIT && !full_tile && slot != 0) {
                // contributor: the int32 partial tile, then the flag
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    uint32_t v[16];
                    tmem_ld32<16>(tacc + c0, v);
                    tmem_wait_ld();
                    int32_t* dst = tile_part + (long long)slot * (BN * 128) + c0 * 128 + r;
#pragma unroll
                    for (int j = 0; j < 16; ++j) dst[j * 128] = (int32_t)v[j];
                }
                tc_fence_before();
                named_bar_sync(3, 128);
                if (et == 0) st_release_gpu_u64(flags + slot, p.epoch);
            } else {
                if (SPLIT && !full_tile) {
                    // summing CTA: every contributor's flag first
                    if (et < 32) {
                        bool got = true;
                        for (int f = 1 + lane; f < nsl && got; f += 32) {
                            got = spin_until_equal_u64(flags + f, p.epoch, wc);
                            if (got) st_release_gpu_u64(flags + f, 0ull);  // consumed
                        }
                        if (!__all_sync(0xFFFFFFFFu, got) && lane == 0) *wc.abort = 1;
                    }
                    named_bar_sync(3, 128);
                }
                const bool reduce = !*wc.abort;
                constexpr int LB = C::LB;
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += LB) {
                    uint32_t v[LB];
                    tmem_ld32<LB>(tacc + c0, v);
                    tmem_wait_ld();
                    if (SPLIT && !full_tile && reduce) {
                        for (int c = 1; c < nsl; ++c) {
                            const int32_t* src = tile_part + (long long)c * (BN * 128) + c0 * 128 + r;
#pragma unroll
                            for (int j = 0; j < LB; ++j) v[j] += (uint32_t)__ldcg(src + j * 128);
                        }
                    }
                    named_bar_sync(4, 128);  // the previous batch's copy-out is done with sY
#pragma unroll
                    for (int j = 0; j < LB; ++j) {
                        const int col = c0 + j;
                        const float sx = __ldg(p.s_x + row0 + min(col, rows_valid - 1));
                        sY[j * 128 + r] = f32_to_bf16_bits(sx * (sw * (float)(int32_t)v[j]));
                    }
                    named_bar_sync(4, 128);
                    if (reduce) {
                        // rows c0 .. c0+LB-1 of the tile, 16-byte segments
#pragma unroll
                        for (int c = et; c < LB * 16; c += 128) {
                            const int jr = c >> 4, seg = c & 15;
                            if (c0 + jr < rows_valid && seg * 8 < ncols) {
                                const uint4 val = *reinterpret_cast<const uint4*>(sY + jr * 128 + seg * 8);
                                uint16_t* dst = p.Y + (long long)(row0 + c0 + jr) * p.ldy + nt * 128 + seg * 8;
                                if (p.vec16) {
                                    *reinterpret_cast<uint4*>(dst) = val;
                                } else {
                                    const uint32_t w4[4] = {val.x, val.y, val.z, val.w};
#pragma unroll
                                    for (int k = 0; k < 4; ++k) {
                                        dst[2 * k] = (uint16_t)(w4[k] & 0xFFFFu);
                                        dst[2 * k + 1] = (uint16_t)(w4[k] >> 16);
                                    }
                                }
                            }
                        }
                    }
                }
                tc_fence_before();
            }
            // the accumulator is free for the MMA's next range
            named_bar_sync(4, 128);
            if (lane == 0) mbar_arrive(&acc_empty[ra.idx]);
            ra.next(2);
            u = seg_end;
        }
    }

    // ----------------------------------------------------------- teardown --
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace w4a8

namespace w4a8 {

// Launches the W8A8 kernel for a tile width BN in {16, 32, 64, 128, 256}
// (defined in gemm_w8a8.cu).  Status codes as in w4a8.h.
int launch_w8a8(int bn, bool split, const CUtensorMap& tmap_w, const CUtensorMap& tmap_x, const W8Params& p,
                int grid, cudaStream_t stream);

}  // namespace w4a8
