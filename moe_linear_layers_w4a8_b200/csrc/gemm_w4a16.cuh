// W4A16 weight-only GEMM on the sm_100a tensor cores: packed 4-bit group
// weights are dequantized to bf16 inside the tile and multiplied with bf16
// activations ("Inference Quantization ch.1" §2-§3.2: the weight-only path
// with the dequantization fused into the GEMM, never written back to HBM):
//   w_hat[k,n] = bf16( fp32( s_w[g,n] * (q[k,n] - z[g,n]) ) )   g = k / group
//   y[m,n]     = bf16( sum_k x[m,k] * w_hat[k,n] )             fp32 accumulation
//
// The weight format is the W4A8 one (same packed codes, fp32 group scales,
// uint8 zero-points), so one packed weight serves both paths.
//   * Swap-AB: the 128 MMA rows are weight output columns, the MMA N
//     dimension is BN tokens.  A = the dequantized bf16 weight tile (written to
//     shared memory by the dequant warps in the MMA's 128-byte swizzled K-major
//     layout), B = the bf16 activation tile (TMA, same swizzle).
//   * Pipeline unit = one k-block of 64 (128 bytes of bf16 per row).  Two
//     producer warps fill two rings with few, large copies (issuing a copy
//     costs the issuing thread about 0.1 us, so copies are sized in tens of
//     KB): warp 0 the weight ring, one stage = up to 8 k-blocks of one tile
//     (the two 64-column halves of packed codes, one contiguous 16 KB copy
//     each, plus one 2-D TMA each for the group scales and zero-points);
//     warp 14 the activation ring (one 3-D TMA of up to 8 k-blocks x BN
//     rows, about 16 KB).
//   * Warps 6-13 dequantize into an A ring whose stages hold 2 k-blocks: per
//     stage each thread loads its two 16-byte code chunks together, writes 4
//     x 16 bytes of bf16 per chunk, and the stage is handed over with one
//     fence and one arrive.  One lane of warp 1 waits once per A stage and
//     issues four K=16 MMAs per k-block into an fp32 accumulator that stays in
//     TMEM for the tile's whole K range; warps 2-5 drain it (two accumulators
//     alternate so a drain overlaps the next range's MMAs).
//   * Stages of every ring start at the first k-block of the CTA's range in a
//     tile and every KS k-blocks after it, cut at the tile's (or range's)
//     end, so producer and consumers agree on them without a table.
//   * Loop positions advance by increments: one 64-bit division per k-block
//     in a producer loop was, measured, the bottleneck of the whole pipeline.
//   * Dequantization, exactly: a code c (offset binary: q + 8 for symmetric
//     codes, q for asymmetric ones) at nibble position p of a 32-bit word,
//     masked into the mantissa of 2^23, is the float 2^23 + c 16^p; minus
//     2^23 + zc 16^p (zc = 8 or z) that is (q - z) 16^p with no rounding, and
//     times s 16^-p it is the single fp32 rounding of s (q - z) (scaling by a
//     power of two commutes with rounding while s 16^-4 stays normal, i.e.
//     s >= 2^-110).  Nibbles at bits 0-19 are used in place; the word's top
//     three nibbles after one shift.  The products are rounded to bf16 in
//     pairs (cvt.rn.bf16x2).
//   * Persistent ranges of (tile, k-block) units as in the W8A8 kernel; when
//     ranges split a tile, contributors store fp32 partial tiles with an epoch
//     flag and the CTA holding the tile's first k-blocks adds them in slot
//     order (deterministic).  The same bounded waits and abort/drain paths.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace w4a8 {

struct W16Params {
    int N, K, M, G, group;
    int n_tiles, m_tiles, KB;    // KB = K / 64 k-blocks
    long long units_per_cta;     // Q
    const uint8_t* packed;       // W4A8 packed layout
    const float* s_w;            // [G][N]
    const uint8_t* z;            // [G][N] or null (symmetric)
    int sg_rows;                 // rows (groups) of the scale / zero-point boxes
    uint16_t* Y;
    int ldy;
    int vec16;                   // Y and ldy allow 16-byte row stores
    float* partial;              // split: fp32 partial tiles [tiles][slots][BN][128]
    int slots;
    unsigned long long* flags;   // split: [tiles][slots]
    unsigned long long epoch;
    int32_t* status;
    unsigned long long wait_ns;
};

constexpr int kW16Threads = 480;     // 2 producers, MMA, 4 epilogue warps, 8 dequant warps
constexpr int kW16EpiWarp0 = 2;
constexpr int kW16DqWarp0 = 6;
constexpr int kW16DqWarps = 8;
constexpr int kW16XWarp = 14;        // activation producer
constexpr int kW16KSW = 8;           // k-blocks per weight stage
constexpr int kW16SGMax = 8;         // scale / zero-point rows per weight stage

// Instruction descriptor: kind::f16, D fp32, A and B bf16, both K-major,
// M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 x bf16 -> fp32, K = 16.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <int BN>
struct W16Cfg {
    static constexpr int XB = BN * 128;                    // one k-block of activations: BN rows x 64 k bf16
    static constexpr int KX_RAW = 16384 / XB;
    static constexpr int KX = KX_RAW < 1 ? 1 : (KX_RAW > 8 ? 8 : KX_RAW);  // k-blocks per activation stage
    static constexpr int X_STAGE = KX * XB;
    static constexpr int NX = 2;                           // activation stages
    static constexpr int A_BYTES = 128 * 128;              // bf16 weight tile: 128 columns x 64 k
    static constexpr int KA = 2;                           // k-blocks per A stage
    static constexpr int A_STAGE = KA * A_BYTES;
    static constexpr int NA = 2;                           // A ring stages
    static constexpr int PK_HALF = kW16KSW * 2048;         // codes of one 64-column half
    static constexpr int W_S = 2 * PK_HALF;                // fp32 scales [kW16SGMax][128]
    static constexpr int W_Z = W_S + kW16SGMax * 512;      // uint8 zero-points [kW16SGMax][128]
    static constexpr int W_STAGE = W_Z + kW16SGMax * 128;
    static constexpr int NW = BN == 256 ? 2 : 3;           // weight stages
    static constexpr int YB = 32 * 128 * 2;                // output staging
    static constexpr int OFF_X = 0;
    static constexpr int OFF_A = OFF_X + NX * X_STAGE;
    static constexpr int OFF_W = OFF_A + NA * A_STAGE;
    static constexpr int OFF_Y = OFF_W + NW * W_STAGE;
    static constexpr int OFF_BAR = OFF_Y + YB;
    static constexpr int NUM_BARS = 2 * NW + 2 * NX + 2 * NA + 5;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    static constexpr int ACC_COLS = 2 * BN;
    static constexpr uint32_t TMEM_COLS = ACC_COLS <= 32 ? 32 : ACC_COLS <= 64 ? 64 : ACC_COLS <= 128 ? 128
                                          : ACC_COLS <= 256 ? 256 : 512;
    static constexpr int LB = BN < 32 ? BN : 32;
    static constexpr uint32_t IDESC = idesc_bf16(BN);
    static_assert(BN == 16 || BN == 32 || BN == 64 || BN == 128 || BN == 256, "BN");
    static_assert(X_STAGE % 1024 == 0 && W_STAGE % 1024 == 0, "1024-byte aligned stages");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

// (w & mask) ^ flip, with the exponent bits of 2^23 set: lop3 with the table
// of  b ? (a ^ c) : c  (mask in b, flip | 0x4B000000 in c).
__device__ __forceinline__ uint32_t magic_nibble(uint32_t w, uint32_t mask, uint32_t fc) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(w), "r"(mask), "r"(fc));
    return d;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// One 16-byte chunk of packed codes (32 codes of one column: byte b holds
// k = b in its low nibble and k = 16 + b in its high nibble) -> 32 bf16
// weights in k order, as four 16-byte runs out[0..3] (k 0-7, 8-15, 16-23,
// 24-31).  A[p], S[p] (p = 0..4): paired 2^23 + zc 16^p and s 16^-p.
template <bool SYM>
__device__ __forceinline__ void dequant_chunk(const uint4 c, const uint64_t* A, const uint64_t* S, uint4* out) {
    const uint32_t flip = SYM ? 0x88888888u : 0u;
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    // word pair (w[2h], w[2h+1]) covers bytes 8h .. 8h+7
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t a = w[2 * h], b = w[2 * h + 1];
        const uint32_t ta = a >> 20, tb = b >> 20;
        // value of nibble at in-place position p of a and b (paired)
        auto nib = [&](uint32_t xa, uint32_t xb, int p) -> uint64_t {
            const uint32_t m = 0xFu << (4 * p);
            const uint32_t fc = (flip & m) | 0x4B000000u;
            const uint64_t f = f2_from_bits(magic_nibble(xa, m, fc), magic_nibble(xb, m, fc));
            return f2_mul(f2_add(f, A[p]), S[p]);
        };
        // low nibbles: byte 0 (p0), byte 1 (p2), byte 2 (p4), byte 3 (t: p1)
        const uint64_t l0 = nib(a, b, 0), l1 = nib(a, b, 2), l2 = nib(a, b, 4), l3 = nib(ta, tb, 1);
        // high nibbles: byte 0 (p1), byte 1 (p3), byte 2 (t: p0), byte 3 (t: p2)
        const uint64_t h0 = nib(a, b, 1), h1 = nib(a, b, 3), h2 = nib(ta, tb, 0), h3 = nib(ta, tb, 2);
        float l0a, l0b, l1a, l1b, l2a, l2b, l3a, l3b, h0a, h0b, h1a, h1b, h2a, h2b, h3a, h3b;
        f2_split(l0, l0a, l0b);
        f2_split(l1, l1a, l1b);
        f2_split(l2, l2a, l2b);
        f2_split(l3, l3a, l3b);
        f2_split(h0, h0a, h0b);
        f2_split(h1, h1a, h1b);
        f2_split(h2, h2a, h2b);
        f2_split(h3, h3a, h3b);
        // word a = bytes 8h..8h+3 -> k 8h..8h+3; word b -> k 8h+4..8h+7
        out[h] = make_uint4(pack_bf16x2(l0a, l1a), pack_bf16x2(l2a, l3a), pack_bf16x2(l0b, l1b),
                            pack_bf16x2(l2b, l3b));
        out[2 + h] = make_uint4(pack_bf16x2(h0a, h1a), pack_bf16x2(h2a, h3a), pack_bf16x2(h0b, h1b),
                                pack_bf16x2(h2b, h3b));
    }
}

template <int BN, bool SPLIT, bool SYM>
__global__ void __launch_bounds__(kW16Threads, 1)
    w4a16_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_s,
                      const __grid_constant__ CUtensorMap tmap_z, const W16Params p) {
    using C = W16Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint16_t* sY = reinterpret_cast<uint16_t*>(smem + C::OFF_Y);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* w_full = bars;                   // [NW] codes, scales, zero-points landed
    uint64_t* w_empty = w_full + C::NW;        // [NW] the 8 dequant warps read them
    uint64_t* x_full = w_empty + C::NW;        // [NX] activation box landed
    uint64_t* x_empty = x_full + C::NX;        // [NX] its MMAs completed
    uint64_t* a_full = x_empty + C::NX;        // [NA] bf16 weight tile written
    uint64_t* a_empty = a_full + C::NA;        // [NA] its MMAs completed
    uint64_t* acc_full = a_empty + C::NA;      // [2]
    uint64_t* acc_empty = acc_full + 2;        // [2]
    uint64_t* drain = acc_empty + 2;           // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        pdl_launch_dependents();
        for (int i = 0; i < C::NW; ++i) {
            mbar_init(&w_full[i], 1);
            mbar_init(&w_empty[i], kW16DqWarps);
        }
        for (int i = 0; i < C::NX; ++i) {
            mbar_init(&x_full[i], 1);
            mbar_init(&x_empty[i], 1);
        }
        for (int i = 0; i < C::NA; ++i) {
            mbar_init(&a_full[i], kW16DqWarps);
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
        prefetch_tmap(&tmap_x);
        prefetch_tmap(&tmap_s);
        if (!SYM) prefetch_tmap(&tmap_z);
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
    const int KBi = p.KB;
    const long long tiles = (long long)p.m_tiles * p.n_tiles;
    const long long U = tiles * KB;
    // split-K: contiguous unit ranges; otherwise whole tiles round-robin
    const RoundRobin rrt(tiles, KB);
    const long long Q = SPLIT ? p.units_per_cta : rrt.waves * KB;
    const long long u0 = SPLIT ? min((long long)blockIdx.x * Q, U) : rrt.u0;
    const long long u1 = SPLIT ? min(u0 + Q, U) : rrt.u1;
    const int kb_shift = p.group == 128 ? 1 : 0;   // k-blocks of 64 per group: 1 << kb_shift

    if (warp == 0) {
        // ------------------------------------------ producer: weight ring --
        if (lane == 0) {
            Ring rw;
            long long issued = 0;
            bool ok = true;
            // positions advance by increments: one 64-bit division per unit
            // would cost more than the copies it schedules
            UnitPos up = SPLIT ? UnitPos(u0, KB, p.n_tiles)
                               : UnitPos(u0, KB, p.n_tiles, rrt.v0, blockIdx.x, gridDim.x);
            for (long long u = u0; u < u1 && ok;) {
                const int kb = up.kb, nt = up.nt;
                const int len = (int)min((long long)min(kW16KSW, KBi - kb), u1 - u);
                const int halves = min(128, p.N - nt * 128) / 64;
                if (!wait_bounded(&w_empty[rw.idx], rw.phase ^ 1u, wc)) { ok = false; break; }
                uint32_t bytes = halves * len * 2048 + p.sg_rows * 512;
                if (!SYM) bytes += p.sg_rows * 128;
                mbar_arrive_expect_tx(&w_full[rw.idx], bytes);
                uint8_t* st = smem + C::OFF_W + rw.idx * C::W_STAGE;
                const int g0 = kb >> kb_shift;
                const int c0 = (kb & kb_shift) * 2;           // first 32-k chunk in group g0
                for (int hf = 0; hf < halves; ++hf) {
                    const long long nb = (long long)nt * 2 + hf;
                    const uint8_t* src = p.packed + (nb * p.G + g0) * (32LL * p.group) + c0 * 1024;
                    bulk_load(st + hf * C::PK_HALF, src, len * 2048, &w_full[rw.idx]);
                }
                tma_load_2d(st + C::W_S, &tmap_s, &w_full[rw.idx], nt * 128, g0);
                if (!SYM) tma_load_2d(st + C::W_Z, &tmap_z, &w_full[rw.idx], nt * 128, g0);
                rw.next(C::NW);
                ++issued;
                for (int i = 0; i < len; ++i) up.next(KB, p.n_tiles);
                u += len;
            }
            WaitCtx wd = wc;
            volatile int no_abort = 0;
            wd.abort = &no_abort;
            Ring d = rw;
            for (long long k = 0; k < issued && k < C::NW; ++k) {
                ring_back(d, C::NW);
                (void)wait_bounded(&w_full[d.idx], d.phase, wd);
            }
        }
    } else if (warp == kW16XWarp) {
        // -------------------------------------- producer: activation ring --
        if (lane == 0) {
            Ring rx;
            long long issued = 0;
            bool ok = true;
            UnitPos up = SPLIT ? UnitPos(u0, KB, p.n_tiles)
                               : UnitPos(u0, KB, p.n_tiles, rrt.v0, blockIdx.x, gridDim.x);
            // activations may come from the kernel launched just before
            pdl_wait_prerequisites();
            for (long long u = u0; u < u1 && ok;) {
                const int kb = up.kb, mt = up.mt;
                const int len = (int)min((long long)min(C::KX, KBi - kb), u1 - u);
                if (!wait_bounded(&x_empty[rx.idx], rx.phase ^ 1u, wc)) { ok = false; break; }
                mbar_arrive_expect_tx(&x_full[rx.idx], C::X_STAGE);
                tma_load_3d(smem + C::OFF_X + rx.idx * C::X_STAGE, &tmap_x, &x_full[rx.idx], 0, mt * BN, kb);
                rx.next(C::NX);
                ++issued;
                for (int i = 0; i < len; ++i) up.next(KB, p.n_tiles);
                u += len;
            }
            WaitCtx wd = wc;
            volatile int no_abort = 0;
            wd.abort = &no_abort;
            Ring d = rx;
            for (long long k = 0; k < issued && k < C::NX; ++k) {
                ring_back(d, C::NX);
                (void)wait_bounded(&x_full[d.idx], d.phase, wd);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issue --
        // One iteration per A stage (up to KA k-blocks): one wait and one
        // commit of the A handshake, then four K=16 MMAs per k-block.
        if (lane == 0) {
            Ring rx, ra, rc;
            int xo = 0;   // offset of the next k-block in its activation stage
            bool ok = true;
            long long u = u0;
            while (u < u1 && ok) {
                const long long t = u / KB;
                const long long tile_u = t * KB;
                const long long seg_end = min(u1, tile_u + KB);
                if (!wait_bounded(&acc_empty[rc.idx], rc.phase ^ 1u, wc)) { ok = false; break; }
                const uint32_t d_tmem = tmem_base + rc.idx * BN;
                for (long long v = u; v < seg_end && ok;) {
                    const int len = (int)min((long long)C::KA, seg_end - v);
                    if (!wait_bounded(&a_full[ra.idx], ra.phase, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc0 = umma_desc_kmajor(smem_u32(smem + C::OFF_A + ra.idx * C::A_STAGE), 128);
#pragma unroll
                    for (int j = 0; j < C::KA; ++j) {
                        if (j < len) {
                            if (xo == 0) {
                                if (!wait_bounded(&x_full[rx.idx], rx.phase, wc)) { ok = false; break; }
                                tc_fence_after();
                            }
                            const uint64_t adesc = adesc0 + (uint64_t)(j * (C::A_BYTES >> 4));
                            const uint64_t bdesc =
                                umma_desc_kmajor(smem_u32(smem + C::OFF_X + rx.idx * C::X_STAGE + xo * C::XB), 128);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_bf16(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, C::IDESC,
                                         (v > u || j > 0 || kk > 0) ? 1u : 0u);
                            // activation stages: KX k-blocks from the segment start, cut at its end
                            if (xo + 1 == C::KX || v + j + 1 == seg_end) {
                                tc_commit(&x_empty[rx.idx]);
                                rx.next(C::NX);
                                xo = 0;
                            } else {
                                ++xo;
                            }
                        }
                    }
                    if (!ok) break;
                    tc_commit(&a_empty[ra.idx]);
                    ra.next(C::NA);
                    v += len;
                }
                if (!ok) break;
                tc_commit(&acc_full[rc.idx]);
                rc.next(2);
                u = seg_end;
            }
            tc_commit(drain);
            WaitCtx wd = wc;
            volatile int no_abort = 0;
            wd.abort = &no_abort;
            (void)wait_bounded(drain, 0, wd);
        }
    } else if (warp >= kW16DqWarp0 && warp < kW16DqWarp0 + kW16DqWarps) {
        // ----------------------------------------------------- dequantize --
        // One iteration per A stage: the codes of its KA k-blocks are loaded
        // together (independent dequant chains), stored, and handed to the
        // MMA with one fence and one arrive.
        const int dt = threadIdx.x - kW16DqWarp0 * 32;  // 0..255
        const int r = dt & 127;                          // weight column within the tile = A row
        const int cc = dt >> 7;                          // 32-k chunk of the k-block
        const int hf = r >> 6;
        const uint32_t row_addr = smem_u32(smem + C::OFF_A) + r * 128;
        Ring rw, ra;
        int wo = 0;      // offset of the next k-block in its weight stage
        int g0 = 0, g_prev = -1;
        uint64_t A[5], S[5];
        bool ok = true;
        UnitPos up = SPLIT ? UnitPos(u0, KB, p.n_tiles)
                               : UnitPos(u0, KB, p.n_tiles, rrt.v0, blockIdx.x, gridDim.x);
        for (long long u = u0; u < u1;) {
            const int kb = up.kb;
            const int len = (int)min((long long)min(C::KA, KBi - kb), u1 - u);
            const bool valid = hf * 64 < min(128, p.N - up.nt * 128);
            if (wo == 0) {
                ok = warp_wait_bounded(&w_full[rw.idx], rw.phase, wc);
                g0 = kb >> kb_shift;
                g_prev = -1;   // a weight stage may start a new tile
            }
            if (ok) ok = warp_wait_bounded(&a_empty[ra.idx], ra.phase ^ 1u, wc);
            if (!ok) break;
            const uint8_t* st = smem + C::OFF_W + rw.idx * C::W_STAGE;
            uint4 c[C::KA];
#pragma unroll
            for (int j = 0; j < C::KA; ++j)
                c[j] = (valid && j < len)
                           ? *reinterpret_cast<const uint4*>(st + hf * C::PK_HALF + (wo + j) * 2048 + cc * 1024 +
                                                             (r & 63) * 16)
                           : make_uint4(0u, 0u, 0u, 0u);
            uint4 out[C::KA][4];
#pragma unroll
            for (int j = 0; j < C::KA; ++j) {
                if (valid && j < len) {
                    const int g = (kb + j) >> kb_shift;
                    if (g != g_prev) {
                        const float sv = reinterpret_cast<const float*>(st + C::W_S)[(g - g0) * 128 + r];
                        const float zc = SYM ? 8.0f : (float)st[C::W_Z + (g - g0) * 128 + r];
#pragma unroll
                        for (int q = 0; q < 5; ++q) {
                            const float sc = (float)(1 << (4 * q));
                            A[q] = f2_splat(-(8388608.0f + zc * sc));
                            S[q] = f2_splat(sv * (1.0f / sc));
                        }
                        g_prev = g;
                    }
                    dequant_chunk<SYM>(c[j], A, S, out[j]);
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i) out[j][i] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            // weight stages: KSW k-blocks from the segment start, cut at its end
            if (wo + len == kW16KSW || kb + len == KBi || u + len == u1) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&w_empty[rw.idx]);
                rw.next(C::NW);
                wo = 0;
            } else {
                wo += len;
            }
            const uint32_t a_row = row_addr + ra.idx * C::A_STAGE;
#pragma unroll
            for (int j = 0; j < C::KA; ++j) {
                if (j < len) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int jj = cc * 4 + i;
                        const uint32_t addr = a_row + j * C::A_BYTES + ((jj ^ (r & 7)) << 4);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(out[j][i].x),
                                     "r"(out[j][i].y), "r"(out[j][i].z), "r"(out[j][i].w)
                                     : "memory");
                    }
                }
            }
            fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[ra.idx]);
            ra.next(C::NA);
            u += len;
            for (int j = 0; j < len; ++j) up.next(KB, p.n_tiles);
        }
    } else if (warp >= kW16EpiWarp0 && warp < kW16EpiWarp0 + 4) {
        // ------------------------------------------------------- epilogue --
        const int q = warp & 3;                 // TMEM lane quadrant
        const int r = q * 32 + lane;            // weight column within the tile
        const int et = (warp - kW16EpiWarp0) * 32 + lane;  // 0..127
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
            const int row0 = mt * BN;
            const int rows_valid = min(BN, p.M - row0);
            const int ncols = min(128, p.N - nt * 128);
            ok = warp_wait_bounded(&acc_full[ra.idx], ra.phase, wc);
            if (named_bar_or(2, 128, !ok)) break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + lane_addr + ra.idx * BN;
            const bool full_tile = (kb0 == 0 && kb1 == p.KB);
            int slot = 0, nsl = 1;
            float* tile_part = nullptr;
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
                // contributor: the fp32 partial tile, then the flag
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    uint32_t v[16];
                    tmem_ld32<16>(tacc + c0, v);
                    tmem_wait_ld();
                    float* dst = tile_part + (long long)slot * (BN * 128) + c0 * 128 + r;
#pragma unroll
                    for (int j = 0; j < 16; ++j) dst[j * 128] = __uint_as_float(v[j]);
                }
                tc_fence_before();
                named_bar_sync(3, 128);
                if (et == 0) st_release_gpu_u64(flags + slot, p.epoch);
            } else {
                if (SPLIT && !full_tile) {
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
                    float acc[LB];
#pragma unroll
                    for (int j = 0; j < LB; ++j) acc[j] = __uint_as_float(v[j]);
                    if (SPLIT && !full_tile && reduce) {
                        for (int c = 1; c < nsl; ++c) {
                            const float* src = tile_part + (long long)c * (BN * 128) + c0 * 128 + r;
#pragma unroll
                            for (int j = 0; j < LB; ++j) acc[j] += __ldcg(src + j * 128);
                        }
                    }
                    named_bar_sync(4, 128);  // the previous batch's copy-out is done with sY
#pragma unroll
                    for (int j = 0; j < LB; ++j) sY[j * 128 + r] = f32_to_bf16_bits(acc[j]);
                    named_bar_sync(4, 128);
                    if (reduce) {
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

// Launches the W4A16 kernel for a tile width BN in {16, 32, 64, 128, 256}
// (defined in gemm_w4a16.cu).  Status codes as in w4a8.h.
int launch_w4a16(int bn, bool split, bool sym, const CUtensorMap& tmap_x, const CUtensorMap& tmap_s,
                 const CUtensorMap& tmap_z, const W16Params& p, int grid, cudaStream_t stream);

}  // namespace w4a8
