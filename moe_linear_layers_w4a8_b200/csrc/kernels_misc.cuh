// Memory-bound kernels around the W4A8 GEMM: per-token INT8 quantization,
// offline 4-bit group packing, MoE routing / dispatch / combine, and the
// fixed-order split-K reduction.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace w4a8 {

constexpr int kStatusNonfinite = 4;

// Per-half maximum of the bf16 magnitudes in w and acc (bf16 bits in each
// 16-bit half).  Unsigned order of the magnitude bits is the order of the
// magnitudes, and every Inf / NaN pattern (>= 0x7F80) sorts above every
// finite value, so the row maximum also tells whether the row is finite.
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t acc, uint32_t w) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(acc), "r"(w & 0x7FFF7FFFu));
    return d;
}

// The INT8 codes of one 16-byte chunk (8 bf16 values x, k order) for the
// divisor d (r = the correctly rounded 1 / d), four codes per output word,
// with the decisions of rne_quotient: the code is RNE(x * r) unless x * r lies
// within 2^-14 of a half-integer (or is not finite), where the correctly
// rounded quotient x / d decides.  RNE(x * r) comes from one addition of
// 1.5 * 2^23: the float grid there is the integers, so the sum is
// 1.5 * 2^23 + RNE(x * r) exactly and its low byte is the code in two's
// complement (|x| <= max|x| keeps the code within [-127, 127]).  The
// distance to the nearest integer, x * r - RNE(x * r), is exact.
// csum (may be null) receives the sum of the eight codes.
__device__ __forceinline__ void quant_chunk8(const uint4 raw, float d, float r, uint32_t& q0, uint32_t& q1,
                                             int32_t* csum) {
    constexpr float kM = 12582912.0f;  // 1.5 * 2^23
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    const uint64_t r2 = f2_splat(r), m2 = f2_splat(kM);
    uint32_t a[8];
    bool slow = false;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const uint64_t x2 = f2_from_bits(w[h] << 16, w[h] & 0xFFFF0000u);  // (k even, k odd)
        const uint64_t t2 = f2_mul(x2, r2);
        const uint64_t a2 = f2_add(t2, m2);
        const uint64_t e2 = f2_sub(t2, f2_sub(a2, m2));
        float e0, e1;
        f2_split(e2, e0, e1);
        slow |= !(fabsf(e0) < 0.49993896484375f) | !(fabsf(e1) < 0.49993896484375f);  // 0.5 - 2^-14
        float f0, f1;
        f2_split(a2, f0, f1);
        a[2 * h] = __float_as_uint(f0);
        a[2 * h + 1] = __float_as_uint(f1);
    }
    q0 = __byte_perm(__byte_perm(a[0], a[1], 0x0040), __byte_perm(a[2], a[3], 0x0040), 0x5410);
    q1 = __byte_perm(__byte_perm(a[4], a[5], 0x0040), __byte_perm(a[6], a[7], 0x0040), 0x5410);
    if (slow) {
        uint32_t packed[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t bits = (e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xFFFFu);
            float t = rne_quotient(bf16_bits_to_f32(bits), d, r);
            t = fminf(fmaxf(t, -127.0f), 127.0f);
            packed[e >> 2] |= ((uint32_t)((int)t & 0xFF)) << (8 * (e & 3));
        }
        q0 = packed[0];
        q1 = packed[1];
    }
    if (csum) *csum = __dp4a((int)q0, 0x01010101, __dp4a((int)q1, 0x01010101, 0));
}

// ---------------------------------------------------------------------------
// Per-token INT8 activation quantization ("Inference Quantization ch.1" §9.2;
// "Kimi 2.7 MoE, 4-bit storage to INT8" §3.3):
//   s = max|x| / 127 (correctly rounded), q = clamp(rne(x / s), -127, 127),
//   s == 0 -> divisor 1.
// One CTA per source row; each thread holds CPT chunks of 8 bf16 in registers
// (one 16-byte load each), so the row is read from HBM once.  With `dest`,
// row m is written to the `dest_k` rows dest[m*dest_k + j] (the MoE dispatch
// order) instead of row m.
// ---------------------------------------------------------------------------
constexpr int kQuantThreads = 256;

template <int CPT>
__global__ void __launch_bounds__(kQuantThreads) quant_act_kernel(
    const uint16_t* __restrict__ X, int K, int ldx, int8_t* __restrict__ q, float* __restrict__ s_x,
    int32_t* __restrict__ rowsum, int group, const int32_t* __restrict__ dest, int dest_k,
    int32_t* status) {
    // A GEMM launched after this kernel with programmatic stream serialization
    // may start its prologue and weight streaming now (it reads only packed
    // weights and scales before it waits for this grid's completion).
    // Launched the same way itself, this kernel may start while the preceding
    // kernel is still running: X and the outputs are touched only after that
    // kernel completed.
    pdl_launch_dependents();
    pdl_wait_prerequisites();
    const int m = blockIdx.x;
    const int tid = threadIdx.x;
    const int nchunk = K >> 3;
    const uint4* xr = reinterpret_cast<const uint4*>(X + (size_t)m * ldx);

    uint4 raw[CPT];
    uint32_t am2 = 0;  // per-half maxima of the bf16 magnitudes
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = i * kQuantThreads + tid;
        raw[i] = make_uint4(0, 0, 0, 0);
        if (c < nchunk) raw[i] = __ldg(xr + c);
        am2 = absmax_bf16x2(am2, raw[i].x);
        am2 = absmax_bf16x2(am2, raw[i].y);
        am2 = absmax_bf16x2(am2, raw[i].z);
        am2 = absmax_bf16x2(am2, raw[i].w);
    }
    // block-wide maximum of the magnitude bits
    __shared__ uint32_t red_max[kQuantThreads / 32];
    uint32_t am = __reduce_max_sync(0xFFFFFFFFu, max(am2 & 0xFFFFu, am2 >> 16));
    if ((tid & 31) == 0) red_max[tid >> 5] = am;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kQuantThreads / 32; ++i) am = max(am, red_max[i]);
    const bool bad = am >= 0x7F80u;  // an Inf or NaN in the row
    const float amax = bf16_bits_to_f32(am);
    const float s = __fdiv_rn(amax, 127.0f);
    const float d = (s > 0.0f) ? s : 1.0f;
    const float r_d = __frcp_rn(d);  // for the exact quotient rounding (rne_quotient)

    const int nrows_out = dest ? dest_k : 1;
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = i * kQuantThreads + tid;
        const bool live = c < nchunk;
        uint32_t packed[2];
        int32_t csum = 0;
        quant_chunk8(raw[i], d, r_d, packed[0], packed[1], rowsum ? &csum : nullptr);
        if (live) {
            for (int j = 0; j < nrows_out; ++j) {
                const int row = dest ? dest[(size_t)m * dest_k + j] : m;
                *reinterpret_cast<uint2*>(q + (size_t)row * K + (size_t)c * 8) = make_uint2(packed[0], packed[1]);
            }
        }
        if (rowsum) {
            // group/8 consecutive chunks (8 or 16 lanes of one warp) form a
            // group; chunks past the row end hold zeros.  All lanes shuffle.
            const int lanes = group >> 3;
            for (int off = lanes >> 1; off > 0; off >>= 1) csum += __shfl_xor_sync(0xFFFFFFFFu, csum, off);
            if (live && (c % lanes) == 0) {
                const int G = K / group;
                for (int j = 0; j < nrows_out; ++j) {
                    const int row = dest ? dest[(size_t)m * dest_k + j] : m;
                    rowsum[(size_t)row * G + c / lanes] = csum;
                }
            }
        }
    }
    if (tid == 0) {
        for (int j = 0; j < nrows_out; ++j) {
            const int row = dest ? dest[(size_t)m * dest_k + j] : m;
            s_x[row] = s;
        }
        if (bad) report_status(status, kStatusNonfinite);
    }
}

// The same quantization for rows longer than quant_act_kernel holds in
// registers (K > 8192): one CTA per row reads the row twice, first for the
// absmax, then for the codes (the second pass mostly from L2).  Every value is
// computed by the same operations, so codes, scales and code sums are those of
// quant_act_kernel.
__global__ void __launch_bounds__(kQuantThreads) quant_act_long_kernel(
    const uint16_t* __restrict__ X, int K, int ldx, int8_t* __restrict__ q, float* __restrict__ s_x,
    int32_t* __restrict__ rowsum, int group, int32_t* status) {
    pdl_launch_dependents();
    pdl_wait_prerequisites();
    const int m = blockIdx.x;
    const int tid = threadIdx.x;
    const int nchunk = K >> 3;
    const uint4* xr = reinterpret_cast<const uint4*>(X + (size_t)m * ldx);

    uint32_t am2 = 0;  // per-half maxima of the bf16 magnitudes
    for (int c = tid; c < nchunk; c += kQuantThreads) {
        const uint4 raw = __ldg(xr + c);
        am2 = absmax_bf16x2(am2, raw.x);
        am2 = absmax_bf16x2(am2, raw.y);
        am2 = absmax_bf16x2(am2, raw.z);
        am2 = absmax_bf16x2(am2, raw.w);
    }
    __shared__ uint32_t red_max[kQuantThreads / 32];
    uint32_t am = __reduce_max_sync(0xFFFFFFFFu, max(am2 & 0xFFFFu, am2 >> 16));
    if ((tid & 31) == 0) red_max[tid >> 5] = am;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kQuantThreads / 32; ++i) am = max(am, red_max[i]);
    const bool bad = am >= 0x7F80u;  // an Inf or NaN in the row
    const float amax = bf16_bits_to_f32(am);
    const float s = __fdiv_rn(amax, 127.0f);
    const float d = (s > 0.0f) ? s : 1.0f;
    const float r_d = __frcp_rn(d);  // for the exact quotient rounding (rne_quotient)

    // all threads run the same number of iterations (the code-sum shuffles
    // need every lane); chunks past the row end hold zeros
    for (int c0 = 0; c0 < nchunk; c0 += kQuantThreads) {
        const int c = c0 + tid;
        const bool live = c < nchunk;
        const uint4 raw = live ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
        uint32_t packed[2];
        int32_t csum = 0;
        quant_chunk8(raw, d, r_d, packed[0], packed[1], rowsum ? &csum : nullptr);
        if (live) *reinterpret_cast<uint2*>(q + (size_t)m * K + (size_t)c * 8) = make_uint2(packed[0], packed[1]);
        if (rowsum) {
            const int lanes = group >> 3;
            for (int off = lanes >> 1; off > 0; off >>= 1) csum += __shfl_xor_sync(0xFFFFFFFFu, csum, off);
            if (live && (c % lanes) == 0) rowsum[(size_t)m * (K / group) + c / lanes] = csum;
        }
    }
    if (tid == 0) {
        s_x[m] = s;
        if (bad) report_status(status, kStatusNonfinite);
    }
}

// The same quantization with one warp per row (8 rows per CTA): no block-wide
// reduction, and many more rows in flight per SM, for launches with many rows
// of at most 4096 elements.  Lane l holds chunks l, l + 32, ... of its row, so
// the per-group code sums are segmented shuffles over 8 or 16 lanes exactly
// as above; every value is computed by the same operations.
constexpr int kQuantRowsPerCta = 8;

template <int CPL>
__global__ void __launch_bounds__(32 * kQuantRowsPerCta) quant_act_rows_kernel(
    const uint16_t* __restrict__ X, int rows, int K, int ldx, int8_t* __restrict__ q, float* __restrict__ s_x,
    int32_t* __restrict__ rowsum, int group, const int32_t* __restrict__ dest, int dest_k, int32_t* status) {
    pdl_launch_dependents();
    pdl_wait_prerequisites();
    const int lane = threadIdx.x & 31;
    const int m = blockIdx.x * kQuantRowsPerCta + (threadIdx.x >> 5);
    if (m >= rows) return;  // warp-uniform
    const int nchunk = K >> 3;
    const uint4* xr = reinterpret_cast<const uint4*>(X + (size_t)m * ldx);

    uint4 raw[CPL];
    uint32_t am2 = 0;  // per-half maxima of the bf16 magnitudes
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const int c = i * 32 + lane;
        raw[i] = make_uint4(0, 0, 0, 0);
        if (c < nchunk) raw[i] = __ldg(xr + c);
    }
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        am2 = absmax_bf16x2(am2, raw[i].x);
        am2 = absmax_bf16x2(am2, raw[i].y);
        am2 = absmax_bf16x2(am2, raw[i].z);
        am2 = absmax_bf16x2(am2, raw[i].w);
    }
    const uint32_t am = __reduce_max_sync(0xFFFFFFFFu, max(am2 & 0xFFFFu, am2 >> 16));
    const bool bad = am >= 0x7F80u;  // an Inf or NaN in the row
    const float amax = bf16_bits_to_f32(am);
    const float s = __fdiv_rn(amax, 127.0f);
    const float d = (s > 0.0f) ? s : 1.0f;
    const float r_d = __frcp_rn(d);  // for the exact quotient rounding (rne_quotient)

    const int nrows_out = dest ? dest_k : 1;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const int c = i * 32 + lane;
        const bool live = c < nchunk;
        uint32_t packed[2];
        int32_t csum = 0;
        quant_chunk8(raw[i], d, r_d, packed[0], packed[1], rowsum ? &csum : nullptr);
        if (live) {
            for (int j = 0; j < nrows_out; ++j) {
                const int row = dest ? dest[(size_t)m * dest_k + j] : m;
                *reinterpret_cast<uint2*>(q + (size_t)row * K + (size_t)c * 8) = make_uint2(packed[0], packed[1]);
            }
        }
        if (rowsum) {
            const int lanes = group >> 3;
            for (int off = lanes >> 1; off > 0; off >>= 1) csum += __shfl_xor_sync(0xFFFFFFFFu, csum, off);
            if (live && (c % lanes) == 0) {
                const int G = K / group;
                for (int j = 0; j < nrows_out; ++j) {
                    const int row = dest ? dest[(size_t)m * dest_k + j] : m;
                    rowsum[(size_t)row * G + c / lanes] = csum;
                }
            }
        }
    }
    if (lane == 0) {
        for (int j = 0; j < nrows_out; ++j) {
            const int row = dest ? dest[(size_t)m * dest_k + j] : m;
            s_x[row] = s;
        }
        if (bad) report_status(status, kStatusNonfinite);
    }
}

// ---------------------------------------------------------------------------
// Offline group-wise 4-bit quantization and packing ("Quantization: formats,
// error and the real execution path", sections "Basic mapping" and
// "Symmetric group-wise reference"; "Inference Quantization ch.1" §6).
// One thread per (output column n, group g); columns are consecutive across
// the warp so every W load is coalesced.  Output layout: see w4a8.h.
// ---------------------------------------------------------------------------
template <int GROUP>
__global__ void __launch_bounds__(128) pack_weights_kernel(const float* __restrict__ W, int K, int N,
                                                           int symmetric, uint8_t* __restrict__ packed,
                                                           float* __restrict__ s_w, uint8_t* __restrict__ z,
                                                           int32_t* status) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int gi = blockIdx.y;
    if (n >= N) return;
    const int G = K / GROUP;
    const float* col = W + (size_t)gi * GROUP * N + n;

    float amax = 0.0f, lo = 0.0f, hi = 0.0f;
    bool bad = false;
    for (int k = 0; k < GROUP; ++k) {
        const float w = __ldg(col + (size_t)k * N);
        bad |= !isfinite(w);
        amax = fmaxf(amax, fabsf(w));
        lo = fminf(lo, w);
        hi = fmaxf(hi, w);
    }
    float s, zf = 0.0f;
    if (symmetric) {
        s = __fdiv_rn(amax, 7.0f);
    } else {
        s = __fdiv_rn(__fsub_rn(hi, lo), 15.0f);
    }
    const float d = (s > 0.0f) ? s : 1.0f;
    if (!symmetric) {
        zf = rintf(__fdiv_rn(-lo, d));
        zf = fminf(fmaxf(zf, 0.0f), 15.0f);
    }

    uint8_t* blk = packed + ((size_t)(n >> 6) * G + gi) * 32u * GROUP;
    const int r = n & 63;
#pragma unroll 1
    for (int c = 0; c < GROUP / 32; ++c) {
        uint32_t words[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int b = 0; b < 16; ++b) {
            uint32_t nib2 = 0;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int k = 32 * c + 16 * half + b;
                const float w = __ldg(col + (size_t)k * N);
                float t = rintf(__fdiv_rn(w, d));
                uint32_t code;
                if (symmetric) {
                    t = fminf(fmaxf(t, -7.0f), 7.0f);
                    code = ((uint32_t)(int)t) & 0xFu;
                } else {
                    t = fminf(fmaxf(__fadd_rn(t, zf), 0.0f), 15.0f);
                    code = (uint32_t)(int)t;
                }
                nib2 |= code << (4 * half);
            }
            words[b >> 2] |= nib2 << (8 * (b & 3));
        }
        *reinterpret_cast<uint4*>(blk + ((size_t)c * 64 + r) * 16) =
            make_uint4(words[0], words[1], words[2], words[3]);
    }
    s_w[(size_t)gi * N + n] = s;
    if (z) z[(size_t)gi * N + n] = (uint8_t)(int)zf;
    if (bad) report_status(status, kStatusNonfinite);
}

// ---------------------------------------------------------------------------
// MoE routing ("Kimi 2.7 MoE, 4-bit storage to INT8" §4.1, §4.4 step 1): the
// router output stays fp32; top-k by logit (ties to the lower expert index);
// weight = softmax over all E experts.  One warp per token; lane l holds
// experts l, l+32, ...; the exp-sum uses a fixed reduction tree.
// ---------------------------------------------------------------------------
template <int EPL>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits, int T, int E,
                                                         int topk, int32_t* __restrict__ idx,
                                                         float* __restrict__ p, int32_t* status) {
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= T) return;
    const float* l = logits + (size_t)t * E;
    float v[EPL];
    bool bad = false;
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = i * 32 + lane;
        v[i] = (e < E) ? __ldg(l + e) : -INFINITY;
        if (e < E) {
            bad |= !isfinite(v[i]);
            mx = fmaxf(mx, v[i]);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    float sum = 0.0f;
#pragma unroll
    for (int i = 0; i < EPL; ++i)
        if (i * 32 + lane < E) sum += expf(v[i] - mx);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);

    uint32_t taken = 0;
    for (int j = 0; j < topk; ++j) {
        float bv = 0.0f;
        int be = 0x7FFFFFFF;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = i * 32 + lane;
            if (e < E && !((taken >> i) & 1u) && (be == 0x7FFFFFFF || v[i] > bv)) {
                bv = v[i];
                be = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
            const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, off);
            if (oe != 0x7FFFFFFF && (be == 0x7FFFFFFF || ov > bv || (ov == bv && oe < be))) {
                bv = ov;
                be = oe;
            }
        }
        if (be != 0x7FFFFFFF && lane == (be & 31)) taken |= 1u << (be >> 5);
        if (lane == 0) {
            idx[(size_t)t * topk + j] = (be == 0x7FFFFFFF) ? 0 : be;
            p[(size_t)t * topk + j] = expf(bv - mx) / sum;
        }
    }
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) report_status(status, kStatusNonfinite);
}

// ---------------------------------------------------------------------------
// Dispatch ("Kimi 2.7 MoE, 4-bit storage to INT8" §4.4 step 3;
// "Choosing a weight-quantization scheme", MoE grouped-GEMM path): count per
// expert, exclusive prefix sum, then the stable (expert, token, slot) order.
// Single CTA of 256 threads, deterministic (no order-dependent atomics):
// tokens are walked in chunks of 256; inside a chunk, a per-(warp, expert)
// lane bitmask gives each pair its rank among earlier tokens.  Also writes
// the prefix over experts of ceil(count / BN) m-tiles for the grouped GEMMs.
// ---------------------------------------------------------------------------
constexpr int kDispatchThreads = 256;
constexpr int kMaxExperts = 512;

__global__ void __launch_bounds__(kDispatchThreads) dispatch_kernel(const int32_t* __restrict__ idx, int T,
                                                                    int E, int topk, int bn,
                                                                    int32_t* __restrict__ offsets,
                                                                    int32_t* __restrict__ mtile_off,
                                                                    int32_t* __restrict__ perm,
                                                                    int32_t* __restrict__ inv) {
    __shared__ int32_t cnt[kMaxExperts];
    __shared__ int32_t base[kMaxExperts];
    __shared__ uint32_t bits[kDispatchThreads / 32][kMaxExperts];
    __shared__ int32_t wpre[kDispatchThreads / 32][kMaxExperts];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < E; e += kDispatchThreads) cnt[e] = 0;
    __syncthreads();
    const int pairs = T * topk;
    for (int i = tid; i < pairs; i += kDispatchThreads) atomicAdd(&cnt[idx[i]], 1);
    __syncthreads();
    if (tid == 0) {
        int32_t run = 0, tiles = 0;
        for (int e = 0; e < E; ++e) {
            offsets[e] = run;
            mtile_off[e] = tiles;
            base[e] = run;
            run += cnt[e];
            tiles += (cnt[e] + bn - 1) / bn;
        }
        offsets[E] = run;
        mtile_off[E] = tiles;
    }
    __syncthreads();
    for (int t0 = 0; t0 < T; t0 += kDispatchThreads) {
        for (int e = lane; e < E; e += 32) bits[warp][e] = 0u;
        __syncthreads();
        const int t = t0 + tid;
        if (t < T)
            for (int j = 0; j < topk; ++j) atomicOr(&bits[warp][idx[(size_t)t * topk + j]], 1u << lane);
        __syncthreads();
        for (int e = tid; e < E; e += kDispatchThreads) {
            int32_t run = 0;
            for (int w = 0; w < kDispatchThreads / 32; ++w) {
                wpre[w][e] = run;
                run += __popc(bits[w][e]);
            }
            cnt[e] = run;  // chunk total for this expert
        }
        __syncthreads();
        if (t < T) {
            const uint32_t lt = (1u << lane) - 1u;
            for (int j = 0; j < topk; ++j) {
                const int e = idx[(size_t)t * topk + j];
                const int32_t pos = base[e] + wpre[warp][e] + __popc(bits[warp][e] & lt);
                inv[(size_t)t * topk + j] = pos;
                perm[pos] = t * topk + j;
            }
        }
        __syncthreads();
        for (int e = tid; e < E; e += kDispatchThreads) base[e] += cnt[e];
        __syncthreads();
    }
}

// The same dispatch spread over many CTAs, for many tokens: each CTA owns a
// contiguous run of `tpc` tokens.  (1) every CTA counts its pairs per
// expert; (2) one CTA turns the counts into the expert offsets, the m-tile
// prefix and every CTA's first position per expert (written over the
// counts); (3) every CTA places its pairs exactly as dispatch_kernel does,
// chunk by chunk from its own first positions.  Positions stay ordered by
// (expert, token, slot), so the output equals dispatch_kernel's.
__global__ void __launch_bounds__(kDispatchThreads) dispatch_count_kernel(const int32_t* __restrict__ idx, int T,
                                                                          int E, int topk, int tpc,
                                                                          int32_t* __restrict__ cnt_g) {
    __shared__ int32_t cnt[kMaxExperts];
    const int c = blockIdx.x, tid = threadIdx.x;
    for (int e = tid; e < E; e += kDispatchThreads) cnt[e] = 0;
    __syncthreads();
    const long long p0 = (long long)c * tpc * topk;
    const long long p1 = (long long)min((long long)(c + 1) * tpc, (long long)T) * topk;
    for (long long i = p0 + tid; i < p1; i += kDispatchThreads) atomicAdd(&cnt[idx[i]], 1);
    __syncthreads();
    for (int e = tid; e < E; e += kDispatchThreads) cnt_g[(size_t)c * E + e] = cnt[e];
}

constexpr int kDispatchScanThreads = kMaxExperts;  // one thread per expert

__global__ void __launch_bounds__(kDispatchScanThreads) dispatch_scan_kernel(int32_t* __restrict__ cnt_g, int C,
                                                                            int E, int bn,
                                                                            int32_t* __restrict__ offsets,
                                                                            int32_t* __restrict__ mtile_off) {
    __shared__ int32_t tot[kMaxExperts], til[kMaxExperts];
    const int e = threadIdx.x;
    int32_t total = 0;
    if (e < E)
        for (int c = 0; c < C; ++c) total += cnt_g[(size_t)c * E + e];
    const int32_t tiles = (total + bn - 1) / bn;
    tot[e] = total;  // zero for e >= E
    til[e] = tiles;
    __syncthreads();
    for (int off = 1; off < kMaxExperts; off <<= 1) {  // inclusive scans over the experts
        const int32_t a = (e >= off) ? tot[e - off] : 0;
        const int32_t b = (e >= off) ? til[e - off] : 0;
        __syncthreads();
        tot[e] += a;
        til[e] += b;
        __syncthreads();
    }
    if (e < E) {
        const int32_t first = tot[e] - total;
        offsets[e] = first;
        mtile_off[e] = til[e] - tiles;
        int32_t run = first;
        for (int c = 0; c < C; ++c) {
            const int32_t v = cnt_g[(size_t)c * E + e];
            cnt_g[(size_t)c * E + e] = run;  // the CTA's first position for this expert
            run += v;
        }
        if (e == E - 1) {
            offsets[E] = tot[e];
            mtile_off[E] = til[e];
        }
    }
}

__global__ void __launch_bounds__(kDispatchThreads) dispatch_scatter_kernel(const int32_t* __restrict__ idx, int T,
                                                                            int E, int topk, int tpc,
                                                                            const int32_t* __restrict__ base_g,
                                                                            int32_t* __restrict__ perm,
                                                                            int32_t* __restrict__ inv) {
    __shared__ int32_t cnt[kMaxExperts];
    __shared__ int32_t base[kMaxExperts];
    __shared__ uint32_t bits[kDispatchThreads / 32][kMaxExperts];
    __shared__ int32_t wpre[kDispatchThreads / 32][kMaxExperts];
    const int c = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < E; e += kDispatchThreads) base[e] = base_g[(size_t)c * E + e];
    __syncthreads();
    const int t_end = (int)min((long long)(c + 1) * tpc, (long long)T);
    for (int t0 = c * tpc; t0 < t_end; t0 += kDispatchThreads) {
        for (int e = lane; e < E; e += 32) bits[warp][e] = 0u;
        __syncthreads();
        const int t = t0 + tid;
        if (t < t_end)
            for (int j = 0; j < topk; ++j) atomicOr(&bits[warp][idx[(size_t)t * topk + j]], 1u << lane);
        __syncthreads();
        for (int e = tid; e < E; e += kDispatchThreads) {
            int32_t run = 0;
            for (int w = 0; w < kDispatchThreads / 32; ++w) {
                wpre[w][e] = run;
                run += __popc(bits[w][e]);
            }
            cnt[e] = run;
        }
        __syncthreads();
        if (t < t_end) {
            const uint32_t lt = (1u << lane) - 1u;
            for (int j = 0; j < topk; ++j) {
                const int e = idx[(size_t)t * topk + j];
                const int32_t pos = base[e] + wpre[warp][e] + __popc(bits[warp][e] & lt);
                inv[(size_t)t * topk + j] = pos;
                perm[pos] = t * topk + j;
            }
        }
        __syncthreads();
        for (int e = tid; e < E; e += kDispatchThreads) base[e] += cnt[e];
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Weighted combine ("Kimi 2.7 MoE, 4-bit storage to INT8" §4.3-4.4 step 5):
// out[t] = sum_j p[t,j] * y[inv(t,j)], fp32 in slot order, one bf16 rounding.
// One thread per (token, 8 consecutive columns): 16-byte loads and stores.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ Yd,
                                                      const float* __restrict__ p,
                                                      const int32_t* __restrict__ inv, int T, int topk, int H,
                                                      uint16_t* __restrict__ out) {
    const int cpr = H >> 3;
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (long long)T * cpr) return;
    const int t = (int)(gid / cpr), c = (int)(gid % cpr);
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
    for (int j = 0; j < topk; ++j) {
        // inv == null: the rows are already in (token, slot) order
        const int r = inv ? __ldg(inv + (size_t)t * topk + j) : t * topk + j;
        const float w = __ldg(p + (size_t)t * topk + j);
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(Yd + (size_t)r * H) + c);
        const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t bits = (e & 1) ? (ws[e >> 1] >> 16) : (ws[e >> 1] & 0xFFFFu);
            acc[e] = fmaf(w, bf16_bits_to_f32(bits), acc[e]);
        }
    }
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
        o[e] = (uint32_t)f32_to_bf16_bits(acc[2 * e]) | ((uint32_t)f32_to_bf16_bits(acc[2 * e + 1]) << 16);
    *reinterpret_cast<uint4*>(out + (size_t)t * H + (size_t)c * 8) = make_uint4(o[0], o[1], o[2], o[3]);
}

// ---------------------------------------------------------------------------
// Offline per-channel INT8 weight quantization for the W8A8 path
// ("Inference Quantization ch.1" §2 worked example and §8.2 per-channel
// scales): s_w[n] = max_k |W[k,n]| / 127, q = clamp(rne(W / s_w), -127, 127),
// s_w == 0 -> divisor 1.  Output q_w[n][k] (k contiguous: the GEMM's weight
// tile is one 2-D TMA box).  One thread per output column n (coalesced reads
// of W across the warp); each thread writes its row 16 codes at a time.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) pack_w8_kernel(const float* __restrict__ W, int K, int N,
                                                      int8_t* __restrict__ q_w, float* __restrict__ s_w,
                                                      int32_t* status) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    float amax = 0.0f;
    bool bad = false;
    for (int k = 0; k < K; ++k) {
        const float w = __ldg(W + (size_t)k * N + n);
        bad |= !isfinite(w);
        amax = fmaxf(amax, fabsf(w));
    }
    const float s = __fdiv_rn(amax, 127.0f);
    const float d = (s > 0.0f) ? s : 1.0f;
    int8_t* row = q_w + (size_t)n * K;
    for (int k0 = 0; k0 < K; k0 += 16) {
        uint32_t words[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int b = 0; b < 16; ++b) {
            float t = rintf(__fdiv_rn(__ldg(W + (size_t)(k0 + b) * N + n), d));
            t = fminf(fmaxf(t, -127.0f), 127.0f);
            words[b >> 2] |= ((uint32_t)((int)t & 0xFF)) << (8 * (b & 3));
        }
        *reinterpret_cast<uint4*>(row + k0) = make_uint4(words[0], words[1], words[2], words[3]);
    }
    s_w[n] = s;
    if (bad) report_status(status, kStatusNonfinite);
}

// Pre-routed expert rows (expert parallelism: the routing ran on another
// rank): copies the expert id of every row into the routing output with
// weight 1, so the layer's dispatch / expert GEMMs / combine run unchanged
// and the combine returns each row's expert output as is.  An id outside
// [0, E) is reported (W4A8_ERR_INVALID_ARG) and replaced by 0, so every later
// index stays in bounds.
__global__ void __launch_bounds__(256) preroute_kernel(const int32_t* __restrict__ ids, int R, int E,
                                                       int32_t* __restrict__ idx, float* __restrict__ w,
                                                       int32_t* status) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= R) return;
    int e = __ldg(ids + i);
    if (e < 0 || e >= E) {
        report_status(status, 1);
        e = 0;
    }
    idx[i] = e;
    w[i] = 1.0f;
}

// Test hook: one warp waits on a barrier nobody arrives on.
__global__ void bounded_wait_selftest_kernel(int32_t* status, unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    WaitCtx w{&abort_flag, status, wait_cycles_for_ns(limit_ns)};
    if (threadIdx.x == 0) (void)wait_bounded(&bar, 0, w);
    __syncthreads();
}

}  // namespace w4a8
