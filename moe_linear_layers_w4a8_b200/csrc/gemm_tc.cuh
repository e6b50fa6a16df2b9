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
//     so the only shared-memory traffic per group is the packed codes and the
//     activation tile.
//   * Warp roles (512 threads): warps 0-3 unpack (warp q owns TMEM lanes /
//     weight rows 32q..32q+31), warps 4-11 drain the partial sums, warp 12
//     brings packed codes (TMA bulk copies), warp 13 brings activation tiles
//     (tiled TMA) and scales, one lane of warp 14 issues the MMAs.
//   * The pipeline advances in steps of S consecutive K-groups of one tile
//     (S = 4 for BN <= 32, 2 for 64, 1 for 128).  A step owns one TMEM
//     "slot": S unpacked weight tiles and S int32 partial buffers.  Three
//     barriers per slot-use and one MMA commit per step: the MMA thread waits
//     once (`ready`: all 4 unpack warps wrote the weight tiles and all 8
//     epilogue warps drained the buffers' previous use), issues S x GROUP/32
//     MMAs and commits once (`done`: weight tiles free, partials ready).
//     Every fixed per-step cost (barrier waits, commits, fences) is paid once
//     per S groups.
//   * Each partial buffer is pre-filled with 0x4B400000 before its MMAs, so
//     afterwards it holds the bits of the float 12582912 + P (|P| < 2^22):
//     one FADD turns it into P exactly, one FFMA applies s_w.
//   * Every TMA request brings several consecutive groups ("chunks"): the
//     packed codes of up to 4 (g=128) / 8 (g=64) groups per 64-column half,
//     the activation tiles of up to 8 groups through a 3-D tensor map (k
//     within group, row, group), and the scales / zero-points of 8 groups
//     through 2-D tensor maps.
//   * Persistent: each CTA owns a contiguous range of (tile, group) units.
//     When ranges split a tile (split-K), the CTA holding the tile's first
//     groups sums it: the other contributors (later CTAs, whose ranges start
//     inside the tile) store fp32 partial tiles plus a flag set to the
//     launch's epoch; the summing CTA waits (bounded) for those flags, clears
//     them, adds the partials in slot order and writes the output.  It only
//     waits on CTAs with higher indices, which never wait on it, so no cycle
//     of waits exists; a flag left by another launch holds another epoch.
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
    float* partial;              // split-K partial tiles [tiles][slots][BN][128]
    int slots;                   // split-K slots per tile
    unsigned long long* flags;   // split-K: [tiles][slots] "partial stored" flags (epoch values)
    unsigned long long epoch;    // this launch's epoch (nonzero)
    int32_t* dbgP;               // optional int32 partials [rows][G][N] (test hook)
    const int32_t* dbg_map;      // grouped modes: slot of each (token, k) pair in dbgP, or -1
    const int32_t* dbg_perm;     // grouped modes: dispatch row -> (token, k) pair
    int n_tiles;
    int m_tiles;                 // plain / split-K
    long long units_per_cta;     // plain / split-K (MoE derives it on device)
    const int32_t* expert_off;   // MoE: [E+1] row offsets (dispatch order)
    const int32_t* mtile_off;    // MoE: [E+1] prefix of m-tiles
    int E;
    int I;                       // gate_up: intermediate size
    int32_t* status;
    unsigned long long wait_ns;
    int vec16;                   // Y and ldy allow 16-byte row stores
    int pdl;                     // launched with programmatic stream serialization
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
    // pipeline steps: S groups per step, NS TMEM slots of S (weight tile + partial buffer)
    static constexpr int S = BN <= 32 ? 4 : (BN == 64 ? 2 : 1);
    static constexpr int SLOT_COLS = S * (GW + BN);
    static constexpr int NS_RAW = 512 / SLOT_COLS;
    static constexpr int NS = NS_RAW > 4 ? 4 : NS_RAW;
    // ring depths of the shared-memory streams (in chunks)
    static constexpr int SPC = (BN <= 32) ? 4 : (BN == 128 ? 2 : 3);
    static constexpr int SAC = (SGA * ACT_TILE <= 16384) ? 3 : (BN == 128 ? 3 : 2);
    static constexpr int SWC = 4;
    static constexpr int A_COL0 = NS * S * BN;           // first TMEM column of the weight tiles
    static constexpr int TMEM_USED = NS * SLOT_COLS;
    static constexpr uint32_t TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128
                                          : TMEM_USED <= 256 ? 256 : 512;
    // shared memory
    static constexpr int ACT_STAGE = SGA * ACT_TILE;
    static constexpr int PK_STAGE = 2 * SGP * PK_HALF;   // [half][group][...]
    static constexpr int Z_STAGE = 2 * SGP * 64;         // [half][group][64 columns]
    static constexpr int SW_STAGE = 2 * SGW * 64 * 4;    // [half][group][64 columns] fp32
    static constexpr int XBUF = MODE == kModeGateUp ? 64 * BN * 4 : 0;
    static constexpr int YBUF = MODE == kModeGateUp ? 0 : BN * 128 * 2;   // bf16 output tile staging
    static constexpr int OFF_ACT = 0;
    static constexpr int OFF_PK = OFF_ACT + SAC * ACT_STAGE;
    static constexpr int OFF_Z = OFF_PK + SPC * PK_STAGE;
    static constexpr int OFF_SW = OFF_Z + SPC * Z_STAGE;
    static constexpr int OFF_X = OFF_SW + SWC * SW_STAGE;
    static constexpr int OFF_Y = OFF_X + XBUF;
    static constexpr int OFF_BAR = OFF_Y + YBUF;
    static constexpr int NUM_BARS = 2 * SPC + 2 * SAC + 2 * SWC + 2 * NS + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int SMEM = BYTES + 1024;            // slack for 1024-byte alignment
    static constexpr int CH = BN / 2;                    // accumulator columns per epilogue thread
    static constexpr uint32_t IDESC = idesc_i8(BN);
    static_assert(BN == 16 || BN == 32 || BN == 64 || BN == 128, "BN");
    static_assert(GROUP == 64 || GROUP == 128, "GROUP");
    static_assert(ACT_TILE % 1024 == 0, "swizzle atoms need 1024-byte tiles");
    static_assert(SGP % S == 0 && SGA % S == 0 && SGW % S == 0, "a step never straddles a chunk");
    static_assert(NS >= 1 && TMEM_USED <= 512, "TMEM columns");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct TileInfo {
    int e, mt, nt;
    int row0;        // first activation row of the tile
    int rows_valid;  // activation rows of this tile that exist
};

template <int BN, int MODE>
__device__ __forceinline__ TileInfo decode_tile(const GemmParams& p, long long t) {
    TileInfo ti;
    if constexpr (MODE == kModeGateUp) {
        // Tiles are ordered (expert, m-tile, n-tile): the n-tiles of an m-tile
        // run back to back, so the m-tiles whose last n-tile finishes in a CTA
        // (and which that CTA then quantizes) are spread evenly over the CTAs.
        const int gm = (int)(t / p.n_tiles);
        ti.nt = (int)(t % p.n_tiles);
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
    } else if constexpr (MODE == kModeDown) {
        // Tiles are ordered (expert, n-tile, m-tile): the m-tiles that share
        // one weight tile of an expert are consecutive units, so they run back
        // to back in one CTA and the repeated weight reads hit L2.
        int lo = 0, hi = p.E - 1;  // last expert whose first tile index is <= t
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if ((long long)__ldg(p.mtile_off + mid) * p.n_tiles <= t) lo = mid; else hi = mid - 1;
        }
        const int m0 = __ldg(p.mtile_off + lo);
        const int mte = __ldg(p.mtile_off + lo + 1) - m0;
        const long long local = t - (long long)m0 * p.n_tiles;
        ti.e = lo;
        ti.nt = (int)(local / mte);
        ti.mt = (int)(local % mte);
        const int r0 = __ldg(p.expert_off + lo);
        const int r1 = __ldg(p.expert_off + lo + 1);
        ti.row0 = r0 + ti.mt * BN;
        ti.rows_valid = min(BN, r1 - ti.row0);
    } else {
        const int gm = (int)(t / p.n_tiles);
        ti.nt = (int)(t % p.n_tiles);
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

// Work range of this CTA in (tile, group) units.  SplitK: a contiguous run
// of units (a tile may be shared by several CTAs).  The other modes hand out
// whole tiles round-robin: the CTA's i-th tile is blockIdx.x + i * gridDim.x,
// so the CTAs running at the same time work on neighbouring tiles (the same
// token block and the same expert's weights), and a tile's operands are
// fetched from HBM about once and shared through L2.  The range stays
// contiguous in a virtual numbering (the CTA's i-th tile is virtual tile
// blockIdx.x * waves + i); tile_of() maps a virtual tile to the real one.
template <int MODE>
__device__ __forceinline__ void cta_units(const GemmParams& p, long long& u0, long long& u1, long long& Q) {
    if constexpr (MODE == kModeSplitK) {
        const long long U = (long long)p.m_tiles * p.n_tiles * p.G;
        Q = p.units_per_cta;
        u0 = (long long)blockIdx.x * Q;
        u1 = min(u0 + Q, U);
        if (u0 > U) u0 = U;
    } else {
        long long tiles;
        if constexpr (MODE == kModeGateUp || MODE == kModeDown)
            tiles = (long long)__ldg(p.mtile_off + p.E) * p.n_tiles;
        else
            tiles = (long long)p.m_tiles * p.n_tiles;
        const long long grid = gridDim.x;
        const long long waves = (tiles + grid - 1) / grid;
        const long long mine = (long long)blockIdx.x < tiles ? (tiles - 1 - blockIdx.x) / grid + 1 : 0;
        Q = (long long)p.G * waves;
        u0 = (long long)blockIdx.x * Q;
        u1 = u0 + mine * p.G;
    }
}

template <int MODE>
__device__ __forceinline__ long long tile_of(long long t_virtual, long long Q, int G) {
    if constexpr (MODE == kModeSplitK) {
        return t_virtual;
    } else {
        const long long waves = Q / G;
        return (long long)blockIdx.x + (t_virtual - (long long)blockIdx.x * waves) * gridDim.x;
    }
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


// s_x of the tile's activation rows col0 .. col0 + JW - 1, all loads issued
// back to back (indices clamped into the tile's valid rows; the values of
// clamped columns are never stored).
template <int JW>
__device__ __forceinline__ void load_sx(const float* s_x, const TileInfo& ti, int col0, float* sx) {
#pragma unroll
    for (int jj = 0; jj < JW; ++jj) sx[jj] = __ldg(s_x + ti.row0 + min(col0 + jj, ti.rows_valid - 1));
}

// Copies a bf16 output tile staged in shared memory ([BN rows][128 columns])
// to Y: 16-byte row segments, one per thread and iteration (256 epilogue
// threads), skipping rows past the tile's valid rows and columns past ncols.
template <int BN>
__device__ __forceinline__ void store_staged_tile(const uint16_t* sY, const GemmParams& p, const TileInfo& ti,
                                                  int n0, int ncols, int et) {
#pragma unroll
    for (int c = et; c < BN * 16; c += kNumEpiWarps * 32) {
        const int row = c >> 4, seg = c & 15;
        if (row < ti.rows_valid && seg * 8 < ncols) {
            const uint4 v = *reinterpret_cast<const uint4*>(sY + row * 128 + seg * 8);
            uint16_t* dst = p.Y + (long long)(ti.row0 + row) * p.ldy + n0 + seg * 8;
            if (p.vec16) {
                *reinterpret_cast<uint4*>(dst) = v;
            } else {
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    dst[2 * k] = (uint16_t)(w[k] & 0xFFFFu);
                    dst[2 * k + 1] = (uint16_t)(w[k] >> 16);
                }
            }
        }
    }
}

// MODE (GemmMode) and DBG (write the int32 group partials) are compile-time,
// so each launched kernel carries only its own epilogue.
template <int BN, int GROUP, int MODE, bool DBG>
__global__ void __launch_bounds__(kGemmThreads, 1)
    w4a8_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_act, const __grid_constant__ CUtensorMap tmap_sw,
                        const __grid_constant__ CUtensorMap tmap_z, const GemmParams p) {
    using C = GemmCfg<BN, GROUP, MODE>;
    constexpr int S = C::S, NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sAct = smem + C::OFF_ACT;
    uint8_t* sPk = smem + C::OFF_PK;
    uint8_t* sZ = smem + C::OFF_Z;
    float* sSW = reinterpret_cast<float*>(smem + C::OFF_SW);
    float* sX = reinterpret_cast<float*>(smem + C::OFF_X);
    uint16_t* sY = reinterpret_cast<uint16_t*>(smem + C::OFF_Y);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* p_full = bars;                     // [SPC] packed codes (+ z) of a chunk landed
    uint64_t* p_empty = p_full + C::SPC;         // [SPC] the 4 unpack warps read them
    uint64_t* act_full = p_empty + C::SPC;       // [SAC] activation tiles of a chunk landed
    uint64_t* act_empty = act_full + C::SAC;     // [SAC] MMA done with them
    uint64_t* sw_full = act_empty + C::SAC;      // [SWC] group scales of a chunk landed
    uint64_t* sw_empty = sw_full + C::SWC;       // [SWC] the 8 epilogue warps read them
    uint64_t* ready = sw_empty + C::SWC;         // [NS] slot's weight tiles written + partial buffers re-armed
    uint64_t* done = ready + NS;                 // [NS] slot's MMAs complete
    uint64_t* drain = done + NS;                 // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Start-up: the packed-code producer initialises every barrier and starts
    // streaming weights at once; it only arrives on the start barrier, while
    // the other warps wait there (for the barriers and the TMEM allocation).
    if (warp == kWarpPack) {
        if (lane == 0) {
            // A kernel launched after this one with programmatic stream
            // serialization may be scheduled on SMs this grid frees; it waits
            // for this grid's completion before touching anything it writes.
            pdl_launch_dependents();
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
            for (int i = 0; i < NS; ++i) {
                mbar_init(&ready[i], kUnpackWarps + kNumEpiWarps);
                mbar_init(&done[i], 1);
            }
            mbar_init(drain, 1);
            *abort_flag = 0;
            fence_mbar_init();
            fence_proxy_async_smem();
            prefetch_tmap(&tmap_act);
            prefetch_tmap(&tmap_sw);
            if (!p.symmetric) prefetch_tmap(&tmap_z);
        }
        __syncwarp();
        named_bar_arrive(5, kGemmThreads);
    } else {
        if (warp == kWarpMma) {
            tmem_alloc(tmem_slot, C::TMEM_COLS);
            tmem_relinquish();
        }
        tc_fence_before();
        named_bar_sync(5, kGemmThreads);
        tc_fence_after();
    }
    const uint32_t tmem_base = (warp == kWarpPack) ? 0u : *tmem_slot;  // the producer never touches TMEM
    const WaitCtx wc{abort_flag, p.status, wait_cycles_for_ns(p.wait_ns)};
    // Launched right behind the kernel that produces the activations
    // (programmatic dependent launch): only the packed weights, scales and
    // zero-points may be read before griddepcontrol.wait.  The grouped MoE
    // modes need the dispatch offsets to plan their ranges, so all threads
    // wait; the dense modes wait in the activation producer and epilogue.
    if constexpr (MODE == kModeGateUp || MODE == kModeDown) pdl_wait_prerequisites();

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
                const TileInfo ti = decode_tile<BN, MODE>(p, tile_of<MODE>(sg.t, Q, G));
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
            if constexpr (MODE == kModePlain || MODE == kModeSplitK) pdl_wait_prerequisites();
            Ring ra, rw;
            long long na = 0, nw = 0;
            bool ok = true;
            for (long long u = u0; u < u1 && ok;) {
                const Segment sg = segment_at(u, u1, G);
                const TileInfo ti = decode_tile<BN, MODE>(p, tile_of<MODE>(sg.t, Q, G));
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
            Ring ra, rs;
            bool ok = true;
            for (long long u = u0; u < u1 && ok;) {
                const Segment sg = segment_at(u, u1, G);
                for (int g0 = sg.gb; g0 < sg.ge; g0 += S) {
                    const int ns = min(S, sg.ge - g0);
                    const int j = (g0 - sg.gb) % C::SGA;            // position in the activation chunk
                    const int clen = min(C::SGA, sg.ge - (g0 - j));  // groups in that chunk
                    if (j == 0 && !wait_bounded(&act_full[ra.idx], ra.phase, wc)) { ok = false; break; }
                    if (!wait_bounded(&ready[rs.idx], rs.phase, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t b0 = b_base + ra.idx * C::ACT_STAGE + j * C::ACT_TILE;
                    const uint32_t slot0 = rs.idx * S;
#pragma unroll
                    for (int i = 0; i < S; ++i) {
                        if (i < ns) {
                            const uint64_t bdesc = umma_desc_kmajor(b0 + i * C::ACT_TILE, GROUP);
                            const uint32_t a_tmem = tmem_base + C::A_COL0 + (slot0 + i) * C::GW;
                            const uint32_t d_tmem = tmem_base + (slot0 + i) * BN;
#pragma unroll
                            for (int kk = 0; kk < GROUP / 32; ++kk)
                                mma_i8_tmem_a(d_tmem, a_tmem + 8 * kk, bdesc + 2 * kk, C::IDESC, 1u);
                        }
                    }
                    tc_commit(&done[rs.idx]);
                    if (j + ns == clen) {
                        tc_commit(&act_empty[ra.idx]);
                        ra.next(C::SAC);
                    }
                    rs.next(NS);
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
        // and stores them in TMEM lanes 32q..32q+31 (row = lane).  Rows of an
        // absent 64-column half are unpacked from whatever the stage holds:
        // their partials are never read.
        const int r = warp * 32 + lane;
        const int half = r >> 6, rr = r & 63;
        const uint32_t lane_addr = ((uint32_t)(warp * 32)) << 16;
        Ring rp, rs;
        bool ok = true;
        for (long long u = u0; u < u1 && ok;) {
            const Segment sg = segment_at(u, u1, G);
            for (int g0 = sg.gb; g0 < sg.ge; g0 += S) {
                const int ns = min(S, sg.ge - g0);
                const int jp = (g0 - sg.gb) % C::SGP;             // position in the packed chunk
                const int plen = min(C::SGP, sg.ge - (g0 - jp));  // groups in that chunk
                if (jp == 0 && !warp_wait_bounded(&p_full[rp.idx], rp.phase, wc)) { ok = false; break; }
                // the slot's weight tiles are free once its previous MMAs completed
                if (!warp_wait_bounded(&done[rs.idx], rs.phase ^ 1u, wc)) { ok = false; break; }
                tc_fence_after();
                const uint8_t* pk = sPk + rp.idx * C::PK_STAGE + (half * C::SGP + jp) * C::PK_HALF + rr * 16;
                const uint8_t* zp = sZ + rp.idx * C::Z_STAGE + (half * C::SGP + jp) * 64 + rr;
                const uint32_t a0 = tmem_base + lane_addr + C::A_COL0 + rs.idx * S * C::GW;
                // packed words of group i + 1 are loaded while group i is unpacked
                uint4 wb[2][GROUP / 32];
#pragma unroll
                for (int c = 0; c < GROUP / 32; ++c) wb[0][c] = *reinterpret_cast<const uint4*>(pk + c * 1024);
#pragma unroll
                for (int i = 0; i < S; ++i) {
                    if (i < ns) {
                        if (i + 1 < ns) {
#pragma unroll
                            for (int c = 0; c < GROUP / 32; ++c)
                                wb[(i + 1) & 1][c] =
                                    *reinterpret_cast<const uint4*>(pk + (i + 1) * C::PK_HALF + c * 1024);
                        }
                        // TMEM column 8c + q holds k = 32c + 4q .. 32c + 4q + 3
                        uint32_t out[C::GW];
                        if (p.symmetric) {
                            // A 4-bit two's complement code moved to the top of
                            // its byte is the int8 16 q: the tile holds 16 q_w
                            // and the MMA yields 16 P exactly (|16 P| < 2^21).
#pragma unroll
                            for (int c = 0; c < GROUP / 32; ++c) {
                                const uint4 w = wb[i & 1][c];
                                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    out[8 * c + q] = (ws[q] << 4) & 0xF0F0F0F0u;
                                    out[8 * c + 4 + q] = ws[q] & 0xF0F0F0F0u;
                                }
                            }
                        } else {
                            // Each byte: 0x80 | u, minus z, then ^ 0x80: the int8 u - z.
                            const uint32_t zz = 0x01010101u * (uint32_t)zp[i * 64];
#pragma unroll
                            for (int c = 0; c < GROUP / 32; ++c) {
                                const uint4 w = wb[i & 1][c];
                                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    out[8 * c + q] = (((ws[q] & 0x0F0F0F0Fu) | 0x80808080u) - zz) ^ 0x80808080u;
                                    out[8 * c + 4 + q] = ((((ws[q] >> 4) & 0x0F0F0F0Fu) | 0x80808080u) - zz) ^ 0x80808080u;
                                }
                            }
                        }
                        tmem_st32<C::GW>(a0 + i * C::GW, out);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (jp + ns == plen) mbar_arrive(&p_empty[rp.idx]);
                    mbar_arrive(&ready[rs.idx]);
                }
                if (jp + ns == plen) rp.next(C::SPC);
                rs.next(NS);
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
        // A step's partials are read in batches of BC columns (all groups of
        // the step when they fit in 32 registers), one TMEM wait per batch.
        constexpr int LDW = CH < 16 ? CH : 16;                              // columns per tcgen05.ld
        constexpr int BC = CH >= 64 ? 16 : (S * CH < 32 ? S * CH : 32);    // columns per batch (register budget)
        constexpr int NBAT = S * CH / BC;
        static_assert(BC % LDW == 0 && (BC % CH == 0 || CH % BC == 0), "batches");
        const uint32_t lane_addr = ((uint32_t)(q * 32)) << 16;

        // Arm every partial buffer of every slot, then release the slots.
#pragma unroll
        for (int b = 0; b < NS * S; ++b) {
            const uint32_t ta = tmem_base + lane_addr + b * BN + hcol * CH;
#pragma unroll
            for (int c0 = 0; c0 < CH; c0 += LDW) tmem_fill32<LDW>(ta + c0, kMagicBits);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            for (int b = 0; b < NS; ++b) mbar_arrive(&ready[b]);
        // s_x, Y and the split-K workspace are touched only after this
        if constexpr (MODE == kModePlain || MODE == kModeSplitK) pdl_wait_prerequisites();

        bool ok = true;
        Ring rw, rs;
        for (long long u = u0; u < u1;) {
            const Segment sg = segment_at(u, u1, G);
            const long long t = sg.t;
            const int gb = sg.gb, ge = sg.ge;
            const TileInfo ti = decode_tile<BN, MODE>(p, tile_of<MODE>(t, Q, G));
            int nb0, nb1;
            tile_blocks<MODE>(p, ti.nt, nb0, nb1);
            const bool n_valid = (half == 0) || (nb1 >= 0);
            const int n = (half == 0 ? nb0 : nb1) * 64 + (r & 63);  // weight column

            // fp32 sums of the group partials, as pairs of adjacent columns
            uint64_t acc2[CH / 2];
#pragma unroll
            for (int jj = 0; jj < CH / 2; ++jj) acc2[jj] = 0ull;
            const uint64_t neg_magic = f2_splat(-kMagicF);
            const float psc = p.symmetric ? 0.0625f : 1.0f;
            const int pshift = p.symmetric ? 4 : 0;

            for (int g0 = gb; g0 < ge && ok; g0 += S) {
                const int ns = min(S, ge - g0);
                // scales of the step's groups
                uint64_t sw2[S];
#pragma unroll
                for (int i = 0; i < S; ++i) {
                    sw2[i] = 0ull;
                    if (i < ns) {
                        const int gi = g0 + i;
                        const int jw = (gi - gb) % C::SGW;
                        const int wlen = min(C::SGW, ge - (gi - jw));
                        if (jw == 0 && !warp_wait_bounded(&sw_full[rw.idx], rw.phase, wc)) { ok = false; break; }
                        // symmetric tiles hold 16 P: s_w / 16 is exact, so s_w/16 * 16P rounds like s_w * P
                        sw2[i] = f2_splat(
                            n_valid ? sSW[rw.idx * (C::SW_STAGE / 4) + (half * C::SGW + jw) * 64 + (r & 63)] * psc
                                    : 0.0f);
                        if (jw == wlen - 1) {
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&sw_empty[rw.idx]);
                            rw.next(C::SWC);
                        }
                    }
                }
                if (!ok) break;
                if (!warp_wait_bounded(&done[rs.idx], rs.phase, wc)) { ok = false; break; }
                tc_fence_after();
                const uint32_t tslot = tmem_base + lane_addr + rs.idx * S * BN + hcol * CH;
                const int last_b = (ns * CH + BC - 1) / BC - 1;  // last batch holding groups of this step
#pragma unroll
                for (int b = 0; b < NBAT; ++b) {
                    if (b <= last_b) {
                        uint32_t v[BC];
#pragma unroll
                        for (int x = 0; x < BC; x += LDW) {
                            const int f = b * BC + x, i = f / CH, c = f % CH;
                            if (i < ns) tmem_ld32<LDW>(tslot + i * BN + c, v + x);
                        }
                        tmem_wait_ld();
#pragma unroll
                        for (int x = 0; x < BC; x += LDW) {  // re-arm for the slot's next use
                            const int f = b * BC + x, i = f / CH, c = f % CH;
                            if (i < ns) tmem_fill32<LDW>(tslot + i * BN + c, kMagicBits);
                        }
#pragma unroll
                        for (int x = 0; x < BC; x += 2) {
                            const int f = b * BC + x, i = f / CH, c = f % CH;
                            // (12582912 + P) - 12582912 = P exactly; acc += s_w P
                            if (i < ns)
                                acc2[c / 2] = f2_fma(sw2[i], f2_add(f2_from_bits(v[x], v[x + 1]), neg_magic), acc2[c / 2]);
                        }
                        if (DBG && n_valid) {
#pragma unroll
                            for (int x = 0; x < BC; ++x) {
                                const int f = b * BC + x, i = f / CH, c = f % CH;
                                const int col = hcol * CH + c;
                                if (i < ns && col < ti.rows_valid) {
                                    long long m = ti.row0 + col;
                                    if constexpr (MODE == kModeGateUp || MODE == kModeDown)
                                        m = p.dbg_map ? __ldg(p.dbg_map + __ldg(p.dbg_perm + m)) : -1;
                                    if (m >= 0)
                                        p.dbgP[(m * G + g0 + i) * p.N + n] = ((int32_t)(v[x] - kMagicBits)) >> pshift;
                                }
                            }
                        }
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ready[rs.idx]);
                rs.next(NS);
            }
            float acc[CH];
#pragma unroll
            for (int jj = 0; jj < CH / 2; ++jj) f2_split(acc2[jj], acc[2 * jj], acc[2 * jj + 1]);
            // The output below uses named barriers: decide together whether
            // any epilogue warp gave up, so none waits alone.
            if (named_bar_or(2, kNumEpiWarps * 32, !ok)) break;
            const int et = ew * 32 + lane;  // 0..255
            const int n0 = nb0 * 64, ncols = nb1 >= 0 ? 128 : 64;

            // ---------------------------------------------- tile output --
            if constexpr (MODE == kModeSplitK) {
                const bool full_tile = (gb == 0 && ge == G);
                if (full_tile) {
                    named_bar_sync(4, kNumEpiWarps * 32);  // the previous tile's copy-out is done with sY
                    constexpr int JW = CH < 16 ? CH : 16;
#pragma unroll
                    for (int j0 = 0; j0 < CH; j0 += JW) {
                        float sx[JW];
                        load_sx<JW>(p.s_x, ti, hcol * CH + j0, sx);
#pragma unroll
                        for (int jj = 0; jj < JW; ++jj)
                            sY[(hcol * CH + j0 + jj) * 128 + r] = f32_to_bf16_bits(sx[jj] * acc[j0 + jj]);
                    }
                    named_bar_sync(4, kNumEpiWarps * 32);
                    store_staged_tile<BN>(sY, p, ti, n0, ncols, et);
                } else {
                    // Split tile.  The CTA holding the tile's first groups
                    // (slot 0) sums it; every other contributor stores its
                    // fp32 partial tile and then its flag (the launch's epoch).
                    // A contributor's range starts inside the tile, so its
                    // partial is stored early in its run, while slot 0 reaches
                    // the tile at the end of its own run.
                    const long long c_first = (t * G) / Q;
                    const int nsl = (int)((t * G + G - 1) / Q - c_first) + 1;
                    const int slot = (int)((long long)blockIdx.x - c_first);
                    float* tile_part = p.partial + (t * p.slots) * (BN * 128);
                    unsigned long long* flags = p.flags + t * p.slots;
                    if (slot != 0) {
                        float* dst = tile_part + (long long)slot * (BN * 128) + r;
#pragma unroll
                        for (int jj = 0; jj < CH; ++jj) dst[(hcol * CH + jj) * 128] = acc[jj];
                        // Every epilogue thread's stores precede the barrier; the one
                        // gpu-scope release store after it publishes them all.
                        named_bar_sync(3, kNumEpiWarps * 32);
                        if (ew == 0 && lane == 0) st_release_gpu_u64(flags + slot, p.epoch);
                    } else {
                        if (ew == 0) {
                            // slots 1 .. nsl-1, 32 at a time (nsl exceeds 32 for
                            // narrow N with long K)
                            bool got = true;
                            for (int f = 1 + lane; f < nsl && got; f += 32) {
                                got = spin_until_equal_u64(flags + f, p.epoch, wc);
                                if (got) st_release_gpu_u64(flags + f, 0ull);  // consumed
                            }
                            if (!__all_sync(0xFFFFFFFFu, got) && lane == 0) *wc.abort = 1;
                        }
                        named_bar_sync(3, kNumEpiWarps * 32);
                        const bool reduce = !*wc.abort;
                        if (reduce) {
                            // the flags were read with acquire before the barrier
                            // slot order: own partial first, then slots 1, 2, ...
                            constexpr int JW = CH < 16 ? CH : 16;
#pragma unroll
                            for (int j0 = 0; j0 < CH; j0 += JW) {
                                float tot[JW];
#pragma unroll
                                for (int jj = 0; jj < JW; ++jj) tot[jj] = acc[j0 + jj];
                                for (int c = 1; c < nsl; ++c) {
                                    const float* src =
                                        tile_part + (long long)c * (BN * 128) + (hcol * CH + j0) * 128 + r;
                                    float v[JW];
#pragma unroll
                                    for (int jj = 0; jj < JW; ++jj) v[jj] = __ldcg(src + jj * 128);
#pragma unroll
                                    for (int jj = 0; jj < JW; ++jj) tot[jj] += v[jj];
                                }
                                float sx[JW];
                                load_sx<JW>(p.s_x, ti, hcol * CH + j0, sx);
#pragma unroll
                                for (int jj = 0; jj < JW; ++jj)
                                    sY[(hcol * CH + j0 + jj) * 128 + r] = f32_to_bf16_bits(sx[jj] * tot[jj]);
                            }
                        }
                        named_bar_sync(4, kNumEpiWarps * 32);
                        if (reduce) store_staged_tile<BN>(sY, p, ti, n0, ncols, et);
                        named_bar_sync(4, kNumEpiWarps * 32);  // sY is free again
                    }
                }
            } else if constexpr (MODE == kModeGateUp) {
                // rows 64..127 hold "up", rows 0..63 the matching "gate"
                constexpr int JW = CH < 16 ? CH : 16;
                if (half == 1) {
#pragma unroll
                    for (int j0 = 0; j0 < CH; j0 += JW) {
                        float sx[JW];
                        load_sx<JW>(p.s_x, ti, hcol * CH + j0, sx);
#pragma unroll
                        for (int jj = 0; jj < JW; ++jj) sX[(hcol * CH + j0 + jj) * 64 + (r - 64)] = sx[jj] * acc[j0 + jj];
                    }
                }
                named_bar_sync(1, kNumEpiWarps * 32);
                if (half == 0) {
                    const int ii = ti.nt * 64 + r;
#pragma unroll
                    for (int j0 = 0; j0 < CH; j0 += JW) {
                        float sx[JW];
                        load_sx<JW>(p.s_x, ti, hcol * CH + j0, sx);
#pragma unroll
                        for (int jj = 0; jj < JW; ++jj) {
                            const int col = hcol * CH + j0 + jj;
                            if (col < ti.rows_valid) {
                                const float gte = sx[jj] * acc[j0 + jj];
                                const float up = sX[col * 64 + r];
                                const float hv = (gte / (1.0f + expf(-gte))) * up;
                                p.Y[(long long)(ti.row0 + col) * p.ldy + ii] = f32_to_bf16_bits(hv);
                            }
                        }
                    }
                }
                named_bar_sync(1, kNumEpiWarps * 32);
            } else {
                // plain / down: every range holds whole tiles
                named_bar_sync(4, kNumEpiWarps * 32);  // the previous tile's copy-out is done with sY
                constexpr int JW = CH < 16 ? CH : 16;
#pragma unroll
                for (int j0 = 0; j0 < CH; j0 += JW) {
                    float sx[JW];
                    load_sx<JW>(p.s_x, ti, hcol * CH + j0, sx);
#pragma unroll
                    for (int jj = 0; jj < JW; ++jj)
                        sY[(hcol * CH + j0 + jj) * 128 + r] = f32_to_bf16_bits(sx[jj] * acc[j0 + jj]);
                }
                named_bar_sync(4, kNumEpiWarps * 32);
                store_staged_tile<BN>(sY, p, ti, n0, ncols, et);
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
