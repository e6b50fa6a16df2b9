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
//     dimension (BN = 16..128) is tokens.  Each epilogue thread owns one
//     weight column (so s_w[g,n] is a per-thread scalar), and decode-size M
//     runs on the same kernel with BN = 16.
//   * The unpacked int8 weight tile lives in TMEM (tcgen05.mma with A from
//     TMEM): each unpack thread turns one row of packed codes into int8 in
//     registers and writes the whole row of the group with one tcgen05.st,
//     so the only shared-memory traffic per step is the packed codes and the
//     activation tile.
//   * Warp roles (512 threads): warps 0-3 unpack (warp q owns TMEM lanes /
//     weight rows 32q..32q+31), warps 4-11 drain the partial sums, warp 12
//     brings packed codes (TMA bulk copies, deep ring), warp 13 brings
//     activation tiles (tiled TMA), one lane of warp 14 issues the MMAs.
//   * TMEM holds NACC int32 partial buffers.  Each is pre-filled with
//     0x4B400000 before a group's MMAs, so afterwards it holds the bits of
//     the float 12582912 + P (|P| < 2^22): one FADD turns it into P exactly,
//     one FFMA applies s_w.
//   * K is walked one quantization group per MMA step, but every TMA request
//     brings several consecutive groups ("chunks"): the packed codes of up to
//     4 (g=128) / 8 (g=64) groups per 64-column half, the activation tiles of
//     up to 8 groups through a 3-D tensor map (k within group, row, group),
//     and the scales / zero-points of 8 groups through 2-D tensor maps.  An
//     SM's TMA unit spends a roughly fixed time per request, so few large
//     requests keep it off the critical path.
//   * Persistent: each CTA owns a contiguous range of (tile, group) units.
//     Ranges that split a tile (split-K) write fp32 partial tiles that a
//     second kernel sums in a fixed order.
//   * Every mbarrier wait is bounded; on expiry the CTA records
//     W4A8_ERR_TIMEOUT, drains its in-flight copies and MMAs, frees TMEM and
//     exits.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

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

constexpr int kGemmThreads = 512;  // 4 unpack, 8 epilogue, 2 producer, 1 MMA, 1 spare warp
constexpr int kNumEpiWarps = 8;
constexpr uint32_t kMagicBits = 0x4B400000u;  // float 12582912 = 1.5 * 2^23
constexpr float kMagicF = 12582912.0f;

// Ring geometry of one kernel instantiation.
template <int BN, int GROUP, int MODE>
struct GemmCfg {
    static constexpr int GW = GROUP / 4;                 // TMEM columns of one unpacked group
    static constexpr int ACT_TILE = BN * GROUP;          // one group's activation tile
    static constexpr int PK_HALF = 32 * GROUP;           // one group of one 64-column block
    // groups per request (chunk) of each stream
    static constexpr int SGP = GROUP == 128 ? 4 : 8;     // packed codes + zero-points
    static constexpr int SGA_RAW = 32768 / ACT_TILE;
    static constexpr int SGA = SGA_RAW < 1 ? 1 : (SGA_RAW > 8 ? 8 : SGA_RAW);  // activation tiles
    static constexpr int SGW = 8;                        // group scales
    // ring depths (in chunks) and the TMEM rings (in groups)
    static constexpr int SPC = (BN == 16) ? 4 : (BN == 128 ? 2 : 3);
    static constexpr int SAC = (SGA * ACT_TILE <= 16384) ? 3 : (BN == 128 ? 3 : 2);
    static constexpr int SWC = 4;
    static constexpr int NACC = BN == 16 ? 8 : BN == 32 ? 8 : BN == 64 ? (GROUP == 128 ? 4 : 6) : 3;
    static constexpr int SA = BN == 128 && GROUP == 128 ? 4 : 8;
    static constexpr int A_COL0 = NACC * BN;             // first TMEM column of the A ring
    static constexpr int TMEM_USED = A_COL0 + SA * GW;
    static constexpr uint32_t TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128
                                          : TMEM_USED <= 256 ? 256 : 512;
    // shared memory
    static constexpr int ACT_STAGE = SGA * ACT_TILE;
    static constexpr int PK_STAGE = 2 * SGP * PK_HALF;   // [half][group][...]
    static constexpr int Z_STAGE = 2 * SGP * 64;         // [half][group][64 columns]
    static constexpr int SW_STAGE = 2 * SGW * 64 * 4;    // [half][group][64 columns] fp32
    static constexpr int XBUF = MODE == kModeGateUp ? 64 * BN * 4 : 0;
    static constexpr int OFF_ACT = 0;
    static constexpr int OFF_PK = OFF_ACT + SAC * ACT_STAGE;
    static constexpr int OFF_Z = OFF_PK + SPC * PK_STAGE;
    static constexpr int OFF_SW = OFF_Z + SPC * Z_STAGE;
    static constexpr int OFF_X = OFF_SW + SWC * SW_STAGE;
    static constexpr int OFF_BAR = OFF_X + XBUF;
    static constexpr int NUM_BARS = 2 * SPC + 2 * SAC + 2 * SWC + 2 * SA + 2 * NACC + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int SMEM = BYTES + 1024;            // slack for 1024-byte alignment
    static constexpr int CH = BN / 2;                    // accumulator columns per epilogue thread
    static constexpr uint32_t IDESC = idesc_i8(BN);
    static_assert(BN == 16 || BN == 32 || BN == 64 || BN == 128, "BN");
    static_assert(GROUP == 64 || GROUP == 128, "GROUP");
    static_assert(ACT_TILE % 1024 == 0, "swizzle atoms need 1024-byte tiles");
    static_assert(TMEM_USED <= 512, "TMEM columns");
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

template <int BN, int MODE>
__device__ __forceinline__ TileInfo decode_tile(const GemmParams& p, long long t) {
    TileInfo ti;
    const int gm = (int)(t / p.n_tiles);
    ti.nt = (int)(t % p.n_tiles);
    if constexpr (MODE == kModeGateUp || MODE == kModeDown) {
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
template <int MODE>
__device__ __forceinline__ void tile_blocks(const GemmParams& p, int nt, int& nb0, int& nb1) {
    if constexpr (MODE == kModeGateUp) {
        nb0 = nt;                  // gate columns [64 nt, 64 nt + 64)
        nb1 = (p.I >> 6) + nt;     // matching up columns I + [64 nt, ...)
    } else {
        nb0 = 2 * nt;
        nb1 = (2 * nt + 1 < (p.N >> 6)) ? 2 * nt + 1 : -1;
    }
}

// Work range of this CTA in (tile, group) units.
template <int MODE>
__device__ __forceinline__ void cta_units(const GemmParams& p, long long& u0, long long& u1, long long& Q) {
    long long U;
    if constexpr (MODE == kModeGateUp || MODE == kModeDown) {
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

constexpr int kUnpackWarps = 4;
constexpr int kWarpPack = 12, kWarpAct = 13, kWarpMma = 14;

// One tile's run of groups [gb, ge) in this CTA's range.
struct Segment {
    long long t;
    int gb, ge;
};

__device__ __forceinline__ Segment segment_at(long long u, long long u1, int G) {
    Segment sg;
    sg.t = u / G;
    sg.gb = (int)(u % G);
    sg.ge = (int)min((long long)G, sg.gb + (u1 - u));
    return sg;
}

// Steps back `n` uses of a ring (for the exit drains).
__device__ __forceinline__ void ring_back(Ring& r, int n) {
    if (r.idx == 0) {
        r.idx = n - 1;
        r.phase ^= 1u;
    } else {
        --r.idx;
    }
}

// MODE (GemmMode) and DBG (write the int32 group partials) are compile-time,
// so each launched kernel carries only its own epilogue.
template <int BN, int GROUP, int MODE, bool DBG>
__global__ void __launch_bounds__(kGemmThreads, 1)
    w4a8_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_act, const __grid_constant__ CUtensorMap tmap_sw,
                        const __grid_constant__ CUtensorMap tmap_z, const GemmParams p) {
    using C = GemmCfg<BN, GROUP, MODE>;
    constexpr int NACC = C::NACC, SA = C::SA;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sAct = smem + C::OFF_ACT;
    uint8_t* sPk = smem + C::OFF_PK;
    uint8_t* sZ = smem + C::OFF_Z;
    float* sSW = reinterpret_cast<float*>(smem + C::OFF_SW);
    float* sX = reinterpret_cast<float*>(smem + C::OFF_X);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* p_full = bars;                     // [SPC] packed codes (+ z) of a chunk landed
    uint64_t* p_empty = p_full + C::SPC;         // [SPC] the 4 unpack warps read them
    uint64_t* act_full = p_empty + C::SPC;       // [SAC] activation tiles of a chunk landed
    uint64_t* act_empty = act_full + C::SAC;     // [SAC] MMA done with them
    uint64_t* sw_full = act_empty + C::SAC;      // [SWC] group scales of a chunk landed
    uint64_t* sw_empty = sw_full + C::SWC;       // [SWC] the 8 epilogue warps read them
    uint64_t* a_full = sw_empty + C::SWC;        // [SA] weight tile of a group unpacked into TMEM
    uint64_t* a_empty = a_full + SA;             // [SA] MMA done with it
    uint64_t* acc_full = a_empty + SA;           // [NACC] partial buffer ready
    uint64_t* acc_empty = acc_full + NACC;       // [NACC] partial buffer drained + re-armed
    uint64_t* drain = acc_empty + NACC;          // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::SPC; ++i) {
            mbar_init(&p_full[i], 1);
            mbar_init(&p_empty[i], kUnpackWarps);
        }
        for (int i = 0; i < C::SAC; ++i) {
            mbar_init(&act_full[i], 1);
            mbar_init(&act_empty[i], 1);
        }
        for (int i = 0; i < C::SWC; ++i) {
            mbar_init(&sw_full[i], 1);
            mbar_init(&sw_empty[i], kNumEpiWarps);
        }
        for (int i = 0; i < SA; ++i) {
            mbar_init(&a_full[i], kUnpackWarps);
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < NACC; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], kNumEpiWarps);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
        prefetch_tmap(&tmap_act);
        prefetch_tmap(&tmap_sw);
        if (!p.symmetric) prefetch_tmap(&tmap_z);
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const WaitCtx wc{abort_flag, p.status, wait_cycles_for_ns(p.wait_ns)};

    long long u0, u1, Q;
    cta_units<MODE>(p, u0, u1, Q);
    const int G = p.G;

    if (warp == kWarpPack) {
        // ------------------------------------- producer: packed codes (+ z) --
        if (lane == 0) {
            Ring rp;
            long long issued = 0;
            bool ok = true;
            for (long long u = u0; u < u1 && ok;) {
                const Segment sg = segment_at(u, u1, G);
                const TileInfo ti = decode_tile<BN, MODE>(p, sg.t);
                int nb0, nb1;
                tile_blocks<MODE>(p, ti.nt, nb0, nb1);
                const uint8_t* wbase = p.packed + (long long)ti.e * p.packed_estride;
                const int zrow = ti.e * G;
                for (int g0 = sg.gb; g0 < sg.ge; g0 += C::SGP) {
                    const int clen = min(C::SGP, sg.ge - g0);
                    if (!wait_bounded(&p_empty[rp.idx], rp.phase ^ 1u, wc)) { ok = false; break; }
                    const int halves = nb1 >= 0 ? 2 : 1;
                    uint32_t bytes = halves * clen * C::PK_HALF;
                    if (!p.symmetric) bytes += halves * C::SGP * 64;
                    mbar_arrive_expect_tx(&p_full[rp.idx], bytes);
                    uint8_t* pk = sPk + rp.idx * C::PK_STAGE;
                    bulk_load(pk, wbase + ((long long)nb0 * G + g0) * C::PK_HALF, clen * C::PK_HALF, &p_full[rp.idx]);
                    if (nb1 >= 0)
                        bulk_load(pk + C::SGP * C::PK_HALF, wbase + ((long long)nb1 * G + g0) * C::PK_HALF,
                                  clen * C::PK_HALF, &p_full[rp.idx]);
                    if (!p.symmetric) {
                        uint8_t* zs = sZ + rp.idx * C::Z_STAGE;
                        tma_load_2d(zs, &tmap_z, &p_full[rp.idx], 64 * nb0, zrow + g0);
                        if (nb1 >= 0) tma_load_2d(zs + C::SGP * 64, &tmap_z, &p_full[rp.idx], 64 * nb1, zrow + g0);
                    }
                    rp.next(C::SPC);
                    ++issued;
                }
                u += sg.ge - sg.gb;
            }
            // Drain: the last copy of every stage lands before the CTA exits.
            WaitCtx wd{abort_flag, p.status, wait_cycles_for_ns(p.wait_ns)};
            volatile int no_abort = 0;
            wd.abort = &no_abort;
            Ring d = rp;
            for (long long k = 0; k < issued && k < C::SPC; ++k) {
                ring_back(d, C::SPC);
                (void)wait_bounded(&p_full[d.idx], d.phase, wd);
            }
        }
    } else if (warp == kWarpAct) {
        // ------------------------- producer: activation tiles, group scales --
        if (lane == 0) {
            Ring ra, rw;
            long long na = 0, nw = 0;
            bool ok = true;
            for (long long u = u0; u < u1 && ok;) {
                const Segment sg = segment_at(u, u1, G);
                const TileInfo ti = decode_tile<BN, MODE>(p, sg.t);
                int nb0, nb1;
                tile_blocks<MODE>(p, ti.nt, nb0, nb1);
                const int wrow = ti.e * G;
                for (int g = sg.gb; g < sg.ge; ++g) {
                    const int j = g - sg.gb;
                    if (j % C::SGW == 0) {
                        if (!wait_bounded(&sw_empty[rw.idx], rw.phase ^ 1u, wc)) { ok = false; break; }
                        mbar_arrive_expect_tx(&sw_full[rw.idx], (nb1 >= 0 ? 2 : 1) * C::SGW * 256);
                        float* ws = sSW + rw.idx * (C::SW_STAGE / 4);
                        tma_load_2d(ws, &tmap_sw, &sw_full[rw.idx], 64 * nb0, wrow + g);
                        if (nb1 >= 0) tma_load_2d(ws + C::SGW * 64, &tmap_sw, &sw_full[rw.idx], 64 * nb1, wrow + g);
                        rw.next(C::SWC);
                        ++nw;
                    }
                    if (j % C::SGA == 0) {
                        if (!wait_bounded(&act_empty[ra.idx], ra.phase ^ 1u, wc)) { ok = false; break; }
                        mbar_arrive_expect_tx(&act_full[ra.idx], C::ACT_STAGE);
                        tma_load_3d(sAct + ra.idx * C::ACT_STAGE, &tmap_act, &act_full[ra.idx], 0, ti.row0, g);
                        ra.next(C::SAC);
                        ++na;
                    }
                }
                u += sg.ge - sg.gb;
            }
            WaitCtx wd{abort_flag, p.status, wait_cycles_for_ns(p.wait_ns)};
            volatile int no_abort = 0;
            wd.abort = &no_abort;
            Ring d = ra;
            for (long long k = 0; k < na && k < C::SAC; ++k) {
                ring_back(d, C::SAC);
                (void)wait_bounded(&act_full[d.idx], d.phase, wd);
            }
            Ring dw = rw;
            for (long long k = 0; k < nw && k < C::SWC; ++k) {
                ring_back(dw, C::SWC);
                (void)wait_bounded(&sw_full[dw.idx], dw.phase, wd);
            }
        }
    } else if (warp == kWarpMma) {
        // ----------------------------------------------------- MMA issue --
        if (lane == 0) {
            const uint32_t b_base = smem_u32(sAct);
            Ring ra, rt, rc;
            bool ok = true;
            for (long long u = u0; u < u1 && ok;) {
                const Segment sg = segment_at(u, u1, G);
                for (int g = sg.gb; g < sg.ge; ++g) {
                    const int j = (g - sg.gb) % C::SGA;
                    const int cend = min(C::SGA, sg.ge - (g - j)) - 1;
                    if (j == 0 && !wait_bounded(&act_full[ra.idx], ra.phase, wc)) { ok = false; break; }
                    if (!wait_bounded(&a_full[rt.idx], rt.phase, wc)) { ok = false; break; }
                    if (!wait_bounded(&acc_empty[rc.idx], rc.phase, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t bdesc =
                        umma_desc_kmajor(b_base + ra.idx * C::ACT_STAGE + j * C::ACT_TILE, GROUP);
                    const uint32_t a_tmem = tmem_base + C::A_COL0 + rt.idx * C::GW;
                    const uint32_t d_tmem = tmem_base + rc.idx * BN;
#pragma unroll
                    for (int kk = 0; kk < GROUP / 32; ++kk)
                        mma_i8_tmem_a(d_tmem, a_tmem + 8 * kk, bdesc + 2 * kk, C::IDESC, 1u);
                    tc_commit(&a_empty[rt.idx]);
                    tc_commit(&acc_full[rc.idx]);
                    if (j == cend) {
                        tc_commit(&act_empty[ra.idx]);
                        ra.next(C::SAC);
                    }
                    rt.next(SA);
                    rc.next(NACC);
                }
                u += sg.ge - sg.gb;
            }
            // Drain: every MMA issued above completes before TMEM is freed.
            tc_commit(drain);
            WaitCtx wd{abort_flag, p.status, wait_cycles_for_ns(p.wait_ns)};
            volatile int no_abort = 0;
            wd.abort = &no_abort;
            (void)wait_bounded(drain, 0, wd);
        }
    } else if (warp < kUnpackWarps) {
        // ---------------------------------------------------------- unpack --
        // Warp q turns rows 32q..32q+31 of every group's weight tile into int8
        // and stores them in TMEM lanes 32q..32q+31 (row = lane).
        const int r = warp * 32 + lane;
        const int half = r >> 6, rr = r & 63;
        const uint32_t lane_addr = ((uint32_t)(warp * 32)) << 16;
        // Each byte: 0x80 | code (sym: code ^ 8 = q + 8), minus z (sym: 8),
        // then ^ 0x80: the two's complement int8 of (q - z) in [-15, 15].
        const uint32_t k1 = p.symmetric ? 0x88888888u : 0x80808080u;
        Ring rp, ra;
        bool ok = true;
        for (long long u = u0; u < u1 && ok;) {
            const Segment sg = segment_at(u, u1, G);
            const TileInfo ti = decode_tile<BN, MODE>(p, sg.t);
            int nb0, nb1;
            tile_blocks<MODE>(p, ti.nt, nb0, nb1);
            const bool row_valid = (half == 0) || (nb1 >= 0);
            for (int g = sg.gb; g < sg.ge; ++g) {
                const int j = (g - sg.gb) % C::SGP;
                const int cend = min(C::SGP, sg.ge - (g - j)) - 1;
                if (j == 0 && !warp_wait_bounded(&p_full[rp.idx], rp.phase, wc)) { ok = false; break; }
                uint4 w[GROUP / 32];
                uint32_t zz = 0x08080808u;
                const uint8_t* pk = sPk + rp.idx * C::PK_STAGE + (half * C::SGP + j) * C::PK_HALF;
#pragma unroll
                for (int c = 0; c < GROUP / 32; ++c)
                    w[c] = row_valid ? *reinterpret_cast<const uint4*>(pk + (c * 64 + rr) * 16)
                                     : make_uint4(0, 0, 0, 0);
                if (!p.symmetric)
                    zz = 0x01010101u * (uint32_t)sZ[rp.idx * C::Z_STAGE + (half * C::SGP + j) * 64 + rr];
                if (j == cend) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&p_empty[rp.idx]);
                    rp.next(C::SPC);
                }
                // TMEM column 8c + i holds k = 32c + 4i .. 32c + 4i + 3
                uint32_t out[C::GW];
#pragma unroll
                for (int c = 0; c < GROUP / 32; ++c) {
                    const uint32_t ws[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t lo = (((ws[i] & 0x0F0F0F0Fu) ^ k1) - zz) ^ 0x80808080u;
                        const uint32_t hi = ((((ws[i] >> 4) & 0x0F0F0F0Fu) ^ k1) - zz) ^ 0x80808080u;
                        out[8 * c + i] = row_valid ? lo : 0u;
                        out[8 * c + 4 + i] = row_valid ? hi : 0u;
                    }
                }
                if (!warp_wait_bounded(&a_empty[ra.idx], ra.phase ^ 1u, wc)) { ok = false; break; }
                tc_fence_after();
                tmem_st32<C::GW>(tmem_base + lane_addr + C::A_COL0 + ra.idx * C::GW, out);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&a_full[ra.idx]);
                ra.next(SA);
            }
            u += sg.ge - sg.gb;
        }
    } else if (warp < kUnpackWarps + kNumEpiWarps) {
        // -------------------------------------------------------- epilogue --
        const int ew = warp - kUnpackWarps;  // 0..7
        const int q = warp & 3;              // TMEM lane quadrant this warp may access
        const int hcol = ew >> 2;            // column half
        const int r = q * 32 + lane;         // weight row within the tile
        const int half = r >> 6;
        constexpr int CH = C::CH;
        const uint32_t lane_addr = ((uint32_t)(q * 32)) << 16;

        // Arm every partial buffer, then hand them to the MMA warp.
#pragma unroll
        for (int b = 0; b < NACC; ++b) {
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
        if (lane == 0)
            for (int b = 0; b < NACC; ++b) mbar_arrive(&acc_empty[b]);

        bool ok = true;
        Ring rw, rc;
        for (long long u = u0; u < u1 && ok;) {
            const Segment sg = segment_at(u, u1, G);
            const long long t = sg.t;
            const int gb = sg.gb, ge = sg.ge;
            const TileInfo ti = decode_tile<BN, MODE>(p, t);
            int nb0, nb1;
            tile_blocks<MODE>(p, ti.nt, nb0, nb1);
            const bool n_valid = (half == 0) || (nb1 >= 0);
            const int n = (half == 0 ? nb0 : nb1) * 64 + (r & 63);  // weight column

            float acc[CH];
#pragma unroll
            for (int jj = 0; jj < CH; ++jj) acc[jj] = 0.0f;

            for (int gi = gb; gi < ge; ++gi) {
                const int j = (gi - gb) % C::SGW;
                const int cend = min(C::SGW, ge - (gi - j)) - 1;
                if (j == 0 && !warp_wait_bounded(&sw_full[rw.idx], rw.phase, wc)) { ok = false; break; }
                const float sw = n_valid ? sSW[rw.idx * (C::SW_STAGE / 4) + (half * C::SGW + j) * 64 + (r & 63)]
                                         : 0.0f;
                if (j == cend) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sw_empty[rw.idx]);
                    rw.next(C::SWC);
                }
                const uint32_t ab = rc.idx;
                if (!warp_wait_bounded(&acc_full[ab], rc.phase, wc)) { ok = false; break; }
                tc_fence_after();
                const uint32_t ta = tmem_base + lane_addr + ab * BN + hcol * CH;
                constexpr int CW = CH < 16 ? CH : 16;  // columns per TMEM load
#pragma unroll
                for (int c0 = 0; c0 < CH; c0 += CW) {
                    uint32_t v[CW];
                    tmem_ld32<CW>(ta + c0, v);
                    tmem_wait_ld();
                    tmem_fill32<CW>(ta + c0, kMagicBits);  // re-arm for the next group
#pragma unroll
                    for (int jj = 0; jj < CW; ++jj)
                        acc[c0 + jj] = fmaf(sw, __uint_as_float(v[jj]) - kMagicF, acc[c0 + jj]);
                    if (DBG && n_valid) {
#pragma unroll
                        for (int jj = 0; jj < CW; ++jj) {
                            const int col = hcol * CH + c0 + jj;
                            if (col < ti.rows_valid) {
                                const long long m = ti.row0 + col;
                                p.dbgP[(m * G + gi) * p.N + n] = (int32_t)(v[jj] - kMagicBits);
                            }
                        }
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[ab]);
                rc.next(NACC);
            }
            if constexpr (MODE == kModeGateUp) {
                // The exchange below uses named barriers: decide together
                // whether any epilogue warp gave up, so none waits alone.
                if (named_bar_or(2, kNumEpiWarps * 32, !ok)) break;
            } else if (!ok) {
                break;
            }

            // ---------------------------------------------- tile output --
            const bool full_tile = (gb == 0 && ge == G);
            if constexpr (MODE == kModeSplitK) {
                const long long c_first = (t * G) / Q;
                const long long slot = (long long)blockIdx.x - c_first;
                float* dst = p.partial + ((t * p.slots + slot) * BN) * 128 + r;
#pragma unroll
                for (int jj = 0; jj < CH; ++jj) dst[(long long)(hcol * CH + jj) * 128] = acc[jj];
            } else if constexpr (MODE == kModeGateUp) {
                // rows 64..127 hold "up", rows 0..63 the matching "gate"
                if (half == 1) {
#pragma unroll
                    for (int jj = 0; jj < CH; ++jj) {
                        const int col = hcol * CH + jj;
                        const float sx = (col < ti.rows_valid) ? __ldg(p.s_x + ti.row0 + col) : 0.0f;
                        sX[col * 64 + (r - 64)] = sx * acc[jj];
                    }
                }
                named_bar_sync(1, kNumEpiWarps * 32);
                if (half == 0) {
                    const int ii = ti.nt * 64 + r;
#pragma unroll
                    for (int jj = 0; jj < CH; ++jj) {
                        const int col = hcol * CH + jj;
                        if (col < ti.rows_valid) {
                            const long long m = ti.row0 + col;
                            const float gte = __ldg(p.s_x + m) * acc[jj];
                            const float up = sX[col * 64 + r];
                            const float hv = (gte / (1.0f + expf(-gte))) * up;
                            p.Y[m * p.ldy + ii] = f32_to_bf16_bits(hv);
                        }
                    }
                }
                named_bar_sync(1, kNumEpiWarps * 32);
            } else {
                if (full_tile && n_valid) {
#pragma unroll
                    for (int jj = 0; jj < CH; ++jj) {
                        const int col = hcol * CH + jj;
                        if (col < ti.rows_valid) {
                            const long long m = ti.row0 + col;
                            p.Y[m * p.ldy + n] = f32_to_bf16_bits(__ldg(p.s_x + m) * acc[jj]);
                        }
                    }
                }
            }
            u += ge - gb;
        }
    }

    // ----------------------------------------------------------- teardown --
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace w4a8
