// W4A8 GEMM on the sm_100a tensor cores (tcgen05, kind::i8, TMEM accumulate).
//
// What one launch computes (see w4a8.h): for every output tile,
//   P[m,g,n] = sum_{k in g} q_x[m,k] (q_w[k,n] - z[g,n])   exact int32 per group
//   acc[m,n] = sum_g s_w[g,n] * P[m,g,n]                      fp32
//   y[m,n]   = s_x[m] * acc[m,n]                              epilogue
// following "Inference Quantization ch.1" §4 (INT8 GEMM, int32 accumulate,
// scales in the epilogue) and §11 ("good path": low-bit tile -> unpack inside
// the matmul tile -> fused epilogue), and "Kimi 2.7 MoE, 4-bit storage to
// INT8" §4.4 step 4 (fused 4-bit unpack + INT8 matmul).
//
// Design (B200):
//   * Swap-AB: the 128 MMA rows (M) are weight output columns n, the MMA N
//     dimension (BN = 16..128) is tokens.  A 128 x 128 x 128 int8 MMA block
//     then needs only 16 KB of unpacked weights, each epilogue thread owns
//     one weight column (so s_w[g,n] is a per-thread scalar), and decode-size
//     M runs on the same kernel with BN = 16.
//   * Warp roles (448 threads): warp 0 issues TMA / bulk copies; warp 1
//     allocates TMEM and one lane issues tcgen05.mma; warps 2-5 unpack the
//     4-bit codes (minus the zero-point) into the swizzled int8 A tile;
//     warps 6-13 drain TMEM per group and accumulate in fp32 registers.
//   * TMEM holds two int32 partial buffers (double-buffered across groups).
//     Each buffer is pre-filled with 0x4B400000 before a group's MMAs, so
//     after them it holds the bits of the float 12582912 + P (|P| < 2^22):
//     one FADD turns it into P exactly, one FFMA applies s_w.
//   * K is walked one quantization group per pipeline stage (64 or 128
//     bytes of K per row = one 64B / 128B swizzle atom row).
//   * Persistent: each CTA owns a contiguous range of (tile, group) units.
//     Ranges that split a tile (split-K) write fp32 partial tiles that a
//     second kernel sums in a fixed order.
//   * Every mbarrier wait is bounded (globaltimer); on expiry the CTA
//     records W4A8_ERR_TIMEOUT, drains its in-flight copies and MMAs, frees
//     TMEM and exits.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "kernels_misc.cuh"
#include "ptx.cuh"

namespace w4a8 {

enum GemmMode : int { kModePlain = 0, kModeSplitK = 1, kModeGateUp = 2, kModeDown = 3 };

struct GemmParams {
    const uint8_t* packed;       // tiled 4-bit codes (expert 0)
    const float* s_w;            // [G][N] (expert 0)
    const uint8_t* z;            // [G][N] or null (symmetric)
    long long packed_estride;    // bytes between experts
    long long sw_estride;        // elements between experts (s_w and z)
    int N, K, G, symmetric;
    const float* s_x;            // per activation row
    int M;                       // plain / split-K: activation rows
    int mode;
    uint16_t* Y;                 // plain: Y; gate_up: h; down: expert outputs
    int ldy;
    float* partial;              // split-K partial tiles
    int slots;                   // split-K slots per tile
    int32_t* dbgP;               // optional [M][G][N] int32 partials (plain / split-K)
    int n_tiles;
    int m_tiles;                 // plain / split-K
    long long units_per_cta;     // plain / split-K (MoE derives it on device)
    const int32_t* expert_off;   // MoE: [E+1] row offsets (dispatch order)
    const int32_t* mtile_off;    // MoE: [E+1] prefix of m-tiles
    int E;
    int I;                       // gate_up: intermediate size
    int32_t* status;
    unsigned long long wait_ns;
};

constexpr int kGemmThreads = 448;
constexpr int kNumEpiWarps = 8;
constexpr uint32_t kMagicBits = 0x4B400000u;  // float 12582912 = 1.5 * 2^23
constexpr float kMagicF = 12582912.0f;

template <int BN, int GROUP, int S, int SA>
struct GemmCfg {
    static constexpr int A_STAGE = 128 * GROUP;
    static constexpr int ACT_STAGE = BN * GROUP;
    static constexpr int PK_HALF = 32 * GROUP;  // one 64-column block of one group
    static constexpr int PK_STAGE = 2 * PK_HALF;
    static constexpr int Z_STAGE = 128;
    static constexpr int XBUF = 64 * BN * 4;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_ACT = OFF_A + SA * A_STAGE;
    static constexpr int OFF_PK = OFF_ACT + S * ACT_STAGE;
    static constexpr int OFF_Z = OFF_PK + S * PK_STAGE;
    static constexpr int OFF_X = OFF_Z + S * Z_STAGE;
    static constexpr int OFF_BAR = OFF_X + XBUF;
    static constexpr int NUM_BARS = 2 * S + 2 * SA + 4 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int SMEM = BYTES + 1024;  // slack for 1024-byte alignment
    static constexpr int CH = BN / 2;          // accumulator columns per epilogue thread
    static constexpr uint32_t TMEM_COLS = (2 * BN < 32) ? 32 : 2 * BN;
    static constexpr uint32_t IDESC = idesc_i8(BN);
    static_assert(BN == 16 || BN == 32 || BN == 64 || BN == 128, "BN");
    static_assert(GROUP == 64 || GROUP == 128, "GROUP");
    static_assert(A_STAGE % 1024 == 0 && ACT_STAGE % 1024 == 0, "swizzle atoms need 1024-byte stages");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct Ring {
    uint32_t idx = 0, phase = 0;
    __device__ __forceinline__ void next(uint32_t n) {
        if (++idx == n) {
            idx = 0;
            phase ^= 1u;
        }
    }
};

struct TileInfo {
    int e, mt, nt;
    int row0;        // first activation row of the tile
    int rows_valid;  // activation rows of this tile that exist
};

template <int BN>
__device__ __forceinline__ TileInfo decode_tile(const GemmParams& p, long long t) {
    TileInfo ti;
    const int gm = (int)(t / p.n_tiles);
    ti.nt = (int)(t % p.n_tiles);
    if (p.mode == kModeGateUp || p.mode == kModeDown) {
        int lo = 0, hi = p.E - 1;  // last expert whose m-tile prefix is <= gm
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (__ldg(p.mtile_off + mid) <= gm) lo = mid; else hi = mid - 1;
        }
        ti.e = lo;
        ti.mt = gm - __ldg(p.mtile_off + lo);
        const int r0 = __ldg(p.expert_off + lo);
        const int r1 = __ldg(p.expert_off + lo + 1);
        ti.row0 = r0 + ti.mt * BN;
        ti.rows_valid = min(BN, r1 - ti.row0);
    } else {
        ti.e = 0;
        ti.mt = gm;
        ti.row0 = gm * BN;
        ti.rows_valid = min(BN, p.M - ti.row0);
    }
    return ti;
}

// 64-column weight blocks that form the 128 A rows of a tile: rows 0..63
// come from block nb0 and rows 64..127 from block nb1 (nb1 < 0: absent).
__device__ __forceinline__ void tile_blocks(const GemmParams& p, int nt, int& nb0, int& nb1) {
    if (p.mode == kModeGateUp) {
        nb0 = nt;                  // gate columns [64 nt, 64 nt + 64)
        nb1 = (p.I >> 6) + nt;     // matching up columns I + [64 nt, ...)
    } else {
        nb0 = 2 * nt;
        nb1 = (2 * nt + 1 < (p.N >> 6)) ? 2 * nt + 1 : -1;
    }
}

// Work range of this CTA in (tile, group) units.
__device__ __forceinline__ void cta_units(const GemmParams& p, long long& u0, long long& u1, long long& Q) {
    long long U;
    if (p.mode == kModeGateUp || p.mode == kModeDown) {
        const long long tiles = (long long)__ldg(p.mtile_off + p.E) * p.n_tiles;
        U = tiles * p.G;
        Q = (long long)p.G * ((tiles + gridDim.x - 1) / gridDim.x);
    } else {
        U = (long long)p.m_tiles * p.n_tiles * p.G;
        Q = p.units_per_cta;
    }
    u0 = (long long)blockIdx.x * Q;
    u1 = min(u0 + Q, U);
    if (u0 > U) u0 = U;
}

template <int BN, int GROUP, int S, int SA>
__global__ void __launch_bounds__(kGemmThreads, 1)
    w4a8_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_act, const GemmParams p) {
    using C = GemmCfg<BN, GROUP, S, SA>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem + C::OFF_A;
    uint8_t* sAct = smem + C::OFF_ACT;
    uint8_t* sPk = smem + C::OFF_PK;
    uint8_t* sZ = smem + C::OFF_Z;
    float* sX = reinterpret_cast<float*>(smem + C::OFF_X);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bars;                 // [S]  TMA landed (packed + z + act)
    uint64_t* empty = bars + S;            // [S]  unpack warps + MMA done with stage
    uint64_t* a_full = bars + 2 * S;       // [SA] A tile unpacked
    uint64_t* a_empty = a_full + SA;       // [SA] MMA done with A tile
    uint64_t* acc_full = a_empty + SA;     // [2]  partial buffer ready
    uint64_t* acc_empty = acc_full + 2;    // [2]  partial buffer drained + re-filled
    uint64_t* drain = acc_empty + 2;       // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 4 + 1);
        }
        for (int i = 0; i < SA; ++i) {
            mbar_init(&a_full[i], 4);
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], kNumEpiWarps);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
        prefetch_tmap(&tmap_act);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const WaitCtx wc{abort_flag, p.status, p.wait_ns};

    long long u0, u1, Q;
    cta_units(p, u0, u1, Q);
    const int G = p.G;

    if (warp == 0) {
        // ------------------------------------------------------ producer --
        if (lane == 0) {
            Ring st;
            long long issued = 0;
            bool ok = true;
            for (long long u = u0; u < u1 && ok;) {
                const long long t = u / G;
                const int gb = (int)(u % G);
                const int ge = (int)min((long long)G, gb + (u1 - u));
                const TileInfo ti = decode_tile<BN>(p, t);
                int nb0, nb1;
                tile_blocks(p, ti.nt, nb0, nb1);
                const uint8_t* wbase = p.packed + (long long)ti.e * p.packed_estride;
                const uint8_t* zrow_base = p.symmetric ? nullptr : p.z + (long long)ti.e * p.sw_estride;
                for (int gi = gb; gi < ge; ++gi) {
                    if (!wait_bounded(&empty[st.idx], st.phase ^ 1u, wc)) { ok = false; break; }
                    uint32_t bytes = C::PK_HALF + C::ACT_STAGE;
                    if (nb1 >= 0) bytes += C::PK_HALF;
                    if (!p.symmetric) bytes += (nb1 >= 0) ? 128 : 64;
                    mbar_arrive_expect_tx(&full[st.idx], bytes);
                    uint8_t* pk = sPk + st.idx * C::PK_STAGE;
                    bulk_load(pk, wbase + ((long long)nb0 * G + gi) * C::PK_HALF, C::PK_HALF, &full[st.idx]);
                    if (nb1 >= 0)
                        bulk_load(pk + C::PK_HALF, wbase + ((long long)nb1 * G + gi) * C::PK_HALF, C::PK_HALF,
                                  &full[st.idx]);
                    if (!p.symmetric) {
                        const uint8_t* zr = zrow_base + (long long)gi * p.N;
                        bulk_load(sZ + st.idx * C::Z_STAGE, zr + 64 * nb0, 64, &full[st.idx]);
                        if (nb1 >= 0) bulk_load(sZ + st.idx * C::Z_STAGE + 64, zr + 64 * nb1, 64, &full[st.idx]);
                    }
                    tma_load_2d(sAct + st.idx * C::ACT_STAGE, &tmap_act, &full[st.idx], gi * GROUP, ti.row0);
                    ++issued;
                    st.next(S);
                }
                u += ge - gb;
            }
            // Drain: wait for the last issue of every stage, so no copy is in
            // flight into this CTA's shared memory when it exits.
            Ring d = st;
            const long long n_drain = issued < S ? issued : S;
            for (long long i = 0; i < n_drain; ++i) {
                // step back one stage
                if (d.idx == 0) { d.idx = S - 1; d.phase ^= 1u; } else { --d.idx; }
                WaitCtx wd{abort_flag, p.status, p.wait_ns};
                volatile int no_abort = 0;
                wd.abort = &no_abort;  // drain even after an abort
                (void)wait_bounded(&full[d.idx], d.phase, wd);
            }
        }
    } else if (warp == 1) {
        // ----------------------------------------------------- MMA issue --
        if (lane == 0) {
            Ring st, sa, ac;
            bool ok = true;
            const uint32_t a_base = smem_u32(sA);
            const uint32_t b_base = smem_u32(sAct);
            for (long long u = u0; u < u1 && ok;) {
                const int gb = (int)(u % G);
                const int ge = (int)min((long long)G, gb + (u1 - u));
                for (int gi = gb; gi < ge; ++gi) {
                    if (!wait_bounded(&full[st.idx], st.phase, wc)) { ok = false; break; }
                    if (!wait_bounded(&a_full[sa.idx], sa.phase, wc)) { ok = false; break; }
                    if (!wait_bounded(&acc_empty[ac.idx], ac.phase, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc = umma_desc_kmajor(a_base + sa.idx * C::A_STAGE, GROUP);
                    const uint64_t bdesc = umma_desc_kmajor(b_base + st.idx * C::ACT_STAGE, GROUP);
                    const uint32_t d_tmem = tmem_base + ac.idx * BN;
#pragma unroll
                    for (int kk = 0; kk < GROUP / 32; ++kk)
                        mma_i8(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, C::IDESC, 1u);
                    tc_commit(&empty[st.idx]);
                    tc_commit(&a_empty[sa.idx]);
                    tc_commit(&acc_full[ac.idx]);
                    st.next(S);
                    sa.next(SA);
                    ac.next(2);
                }
                u += ge - gb;
            }
            // Drain: every MMA issued above completes before TMEM is freed.
            tc_commit(drain);
            WaitCtx wd{abort_flag, p.status, p.wait_ns};
            volatile int no_abort = 0;
            wd.abort = &no_abort;
            (void)wait_bounded(drain, 0, wd);
        }
    } else if (warp < 6) {
        // ---------------------------------------------------------- unpack --
        const int r = threadIdx.x - 64;  // A row 0..127
        const int half = r >> 6, rr = r & 63;
        Ring st, sa;
        bool ok = true;
        for (long long u = u0; u < u1 && ok;) {
            const long long t = u / G;
            const int gb = (int)(u % G);
            const int ge = (int)min((long long)G, gb + (u1 - u));
            const TileInfo ti = decode_tile<BN>(p, t);
            int nb0, nb1;
            tile_blocks(p, ti.nt, nb0, nb1);
            const bool row_valid = (half == 0) || (nb1 >= 0);
            // Each byte: 0x80 | code (sym: code ^ 8 = q + 8), minus z (sym: 8),
            // then ^ 0x80: the two's complement int8 of (q - z) in [-15, 15].
            const uint32_t k1 = p.symmetric ? 0x88888888u : 0x80808080u;
            for (int gi = gb; gi < ge; ++gi) {
                if (!warp_wait_bounded(&full[st.idx], st.phase, wc)) { ok = false; break; }
                uint4 w[GROUP / 32];
                uint32_t zz = 0x08080808u;
                if (row_valid) {
                    const uint8_t* pk = sPk + st.idx * C::PK_STAGE + half * C::PK_HALF;
#pragma unroll
                    for (int c = 0; c < GROUP / 32; ++c)
                        w[c] = *reinterpret_cast<const uint4*>(pk + (c * 64 + rr) * 16);
                    if (!p.symmetric) zz = 0x01010101u * (uint32_t)sZ[st.idx * C::Z_STAGE + half * 64 + rr];
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st.idx]);
                if (!warp_wait_bounded(&a_empty[sa.idx], sa.phase ^ 1u, wc)) { ok = false; break; }
                uint8_t* arow = sA + sa.idx * C::A_STAGE + r * GROUP;
#pragma unroll
                for (int c = 0; c < GROUP / 32; ++c) {
                    uint4 lo4 = make_uint4(0, 0, 0, 0), hi4 = make_uint4(0, 0, 0, 0);
                    if (row_valid) {
                        const uint32_t ws[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
                        uint32_t lo[4], hi[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            lo[i] = (((ws[i] & 0x0F0F0F0Fu) ^ k1) - zz) ^ 0x80808080u;
                            hi[i] = ((((ws[i] >> 4) & 0x0F0F0F0Fu) ^ k1) - zz) ^ 0x80808080u;
                        }
                        lo4 = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                        hi4 = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    }
                    // logical 16-byte chunks 2c (k = 32c..32c+15) and 2c+1
                    int p0, p1;
                    if (GROUP == 128) {
                        p0 = (2 * c) ^ (r & 7);
                        p1 = (2 * c + 1) ^ (r & 7);
                    } else {
                        p0 = (2 * c) ^ ((r >> 1) & 3);
                        p1 = (2 * c + 1) ^ ((r >> 1) & 3);
                    }
                    *reinterpret_cast<uint4*>(arow + p0 * 16) = lo4;
                    *reinterpret_cast<uint4*>(arow + p1 * 16) = hi4;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&a_full[sa.idx]);
                st.next(S);
                sa.next(SA);
            }
            u += ge - gb;
        }
    } else {
        // -------------------------------------------------------- epilogue --
        const int ew = warp - 6;           // 0..7
        const int q = warp & 3;            // TMEM lane quadrant this warp may access
        const int hcol = ew >> 2;          // column half
        const int r = q * 32 + lane;       // A row = weight column within the tile
        constexpr int CH = C::CH;
        const uint32_t lane_addr = ((uint32_t)(q * 32)) << 16;

        // Pre-fill both partial buffers, then hand them to the MMA warp.
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            const uint32_t ta = tmem_base + lane_addr + b * BN + hcol * CH;
            if constexpr (CH >= 32) {
#pragma unroll
                for (int c0 = 0; c0 < CH; c0 += 32) tmem_fill32<32>(ta + c0, kMagicBits);
            } else {
                tmem_fill32<CH>(ta, kMagicBits);
            }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&acc_empty[0]);
            mbar_arrive(&acc_empty[1]);
        }

        Ring ac;
        bool ok = true;
        for (long long u = u0; u < u1 && ok;) {
            const long long t = u / G;
            const int gb = (int)(u % G);
            const int ge = (int)min((long long)G, gb + (u1 - u));
            const TileInfo ti = decode_tile<BN>(p, t);
            int nb0, nb1;
            tile_blocks(p, ti.nt, nb0, nb1);
            const int half = r >> 6;
            const bool n_valid = (half == 0) || (nb1 >= 0);
            const int n = (half == 0 ? nb0 : nb1) * 64 + (r & 63);  // weight column
            const float* swp = p.s_w + (long long)ti.e * p.sw_estride + n;

            float acc[CH];
#pragma unroll
            for (int j = 0; j < CH; ++j) acc[j] = 0.0f;
            float sw_next = n_valid ? __ldg(swp + (long long)gb * p.N) : 0.0f;

            for (int gi = gb; gi < ge; ++gi) {
                const float sw = sw_next;
                if (gi + 1 < ge) sw_next = n_valid ? __ldg(swp + (long long)(gi + 1) * p.N) : 0.0f;
                if (!warp_wait_bounded(&acc_full[ac.idx], ac.phase, wc)) { ok = false; break; }
                tc_fence_after();
                const uint32_t ta = tmem_base + lane_addr + ac.idx * BN + hcol * CH;
                constexpr int CW = CH < 16 ? CH : 16;  // columns per TMEM load
#pragma unroll
                for (int c0 = 0; c0 < CH; c0 += CW) {
                    uint32_t v[CW];
                    tmem_ld32<CW>(ta + c0, v);
                    tmem_wait_ld();
                    tmem_fill32<CW>(ta + c0, kMagicBits);  // re-arm for the next group
#pragma unroll
                    for (int j = 0; j < CW; ++j)
                        acc[c0 + j] = fmaf(sw, __uint_as_float(v[j]) - kMagicF, acc[c0 + j]);
                    if (p.dbgP != nullptr && n_valid) {
#pragma unroll
                        for (int j = 0; j < CW; ++j) {
                            const int col = hcol * CH + c0 + j;
                            if (col < ti.rows_valid) {
                                const long long m = ti.row0 + col;
                                p.dbgP[(m * G + gi) * p.N + n] = (int32_t)(v[j] - kMagicBits);
                            }
                        }
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[ac.idx]);
                ac.next(2);
            }
            if (p.mode == kModeGateUp) {
                // The exchange below uses named barriers: decide together
                // whether any epilogue warp gave up, so none waits alone.
                if (named_bar_or(2, kNumEpiWarps * 32, !ok)) break;
            } else if (!ok) {
                break;
            }

            // ---------------------------------------------- tile output --
            const bool full_tile = (gb == 0 && ge == G);
            if (p.mode == kModeSplitK) {
                const long long c_first = (t * G) / Q;
                const long long slot = (long long)blockIdx.x - c_first;
                float* dst = p.partial + ((t * p.slots + slot) * BN) * 128 + r;
#pragma unroll
                for (int j = 0; j < CH; ++j) dst[(long long)(hcol * CH + j) * 128] = acc[j];
            } else if (p.mode == kModeGateUp) {
                // rows 64..127 hold "up", rows 0..63 the matching "gate"
                if (half == 1) {
#pragma unroll
                    for (int j = 0; j < CH; ++j) {
                        const int col = hcol * CH + j;
                        const float sx = (col < ti.rows_valid) ? __ldg(p.s_x + ti.row0 + col) : 0.0f;
                        sX[col * 64 + (r - 64)] = sx * acc[j];
                    }
                }
                named_bar_sync(1, kNumEpiWarps * 32);
                if (half == 0) {
                    const int i = ti.nt * 64 + r;
#pragma unroll
                    for (int j = 0; j < CH; ++j) {
                        const int col = hcol * CH + j;
                        if (col < ti.rows_valid) {
                            const long long m = ti.row0 + col;
                            const float gte = __ldg(p.s_x + m) * acc[j];
                            const float up = sX[col * 64 + r];
                            const float hv = (gte / (1.0f + expf(-gte))) * up;
                            p.Y[m * p.ldy + i] = f32_to_bf16_bits(hv);
                        }
                    }
                }
                named_bar_sync(1, kNumEpiWarps * 32);
            } else if (full_tile && n_valid) {
#pragma unroll
                for (int j = 0; j < CH; ++j) {
                    const int col = hcol * CH + j;
                    if (col < ti.rows_valid) {
                        const long long m = ti.row0 + col;
                        p.Y[m * p.ldy + n] = f32_to_bf16_bits(__ldg(p.s_x + m) * acc[j]);
                    }
                }
            }
            u += ge - gb;
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
