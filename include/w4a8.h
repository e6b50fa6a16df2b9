/*
 * w4a8.h — C ABI of libw4a8.so, the W4A8 quantized Linear / MoE-expert path
 * for NVIDIA B200 (sm_100a).
 *
 * What is computed (notation of "Inference Quantization ch.1 (the Linear
 * layer)", §1: X [M,K], W [K,N], Y = X W):
 *
 *   s_x[m]   = max_k |X[m,k]| / 127                       (fp32, IEEE division)
 *   q_x[m,k] = clamp(rne(X[m,k] / s_x[m]), -127, 127)     (int8)
 *   W is stored offline as 4-bit codes q_w with one scale s_w[g,n] (and, for
 *   asymmetric weights, one zero-point z[g,n]) per group g of `group` (64 or
 *   128) consecutive k of one output column n;
 *   P[m,g,n] = sum_{k in g} q_x[m,k] * (q_w[k,n] - z[g,n])  (exact int32)
 *   Y[m,n]   = s_x[m] * sum_g s_w[g,n] * P[m,g,n]          (fp32 across groups)
 *
 * Sources: "Inference Quantization ch.1" §4 (INT8 x INT8 -> int32, scales in
 * the epilogue), §7 (zero-point term), §8.3-8.4 (per-token / group-wise
 * scales), §9.2 (dynamic per-token scale); "Quantization: formats, error and
 * the real execution path", sections "Basic mapping", "Symmetric group-wise
 * reference" and "Correctness contract"; "Kimi 2.7 MoE, 4-bit storage to
 * INT8" §3.3 (per-token INT8), §4.1-4.4 (MoE flow), §5.2 (two codes per byte);
 * "Kimi 2.7 MoE W4A8 deployment in practice" §2.1-2.2.
 *
 * Conventions for every call:
 *   - Pointers named as device pointers must be device memory owned by the
 *     caller; the library never allocates and never frees.  Scratch memory is
 *     the caller's `workspace` (size from the *_workspace_size queries).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call only enqueues work on it and returns at once.
 *   - Argument, shape and format checks run on the host before anything is
 *     launched and return a status; nothing is thrown across the ABI.
 *   - Device-detected failures (non-finite inputs, a bounded wait that ran
 *     out) are written to `dev_status`, a device int32 owned by the caller
 *     that must hold 0 beforehand: the first failing kernel stores its
 *     w4a8_status code there.  NULL skips device-side reporting.  Read it with
 *     w4a8_get_device_status.  On such a failure output contents are
 *     unspecified.
 *   - There is no fallback path: an unsupported shape returns
 *     W4A8_ERR_UNSUPPORTED_SHAPE and launches nothing.
 *   - bf16 tensors are passed as raw 16-bit patterns (uint16_t).
 */
#ifndef W4A8_H
#define W4A8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Only the calls below are exported from libw4a8.so. */
#if defined(__GNUC__)
#define W4A8_API __attribute__((visibility("default")))
#else
#define W4A8_API
#endif

#define W4A8_ABI_VERSION 1
#define W4A8_LAYOUT_VERSION 1

typedef enum {
    W4A8_OK = 0,
    W4A8_ERR_INVALID_ARG = 1,       /* null pointer, negative size, K % group != 0, ... */
    W4A8_ERR_UNSUPPORTED_SHAPE = 2, /* valid but outside what the kernels cover */
    W4A8_ERR_FORMAT_MISMATCH = 3,   /* descriptor does not match the call */
    W4A8_ERR_NONFINITE = 4,         /* NaN/Inf in an input (device-detected) */
    W4A8_ERR_TIMEOUT = 5,           /* a bounded device wait ran out */
    W4A8_ERR_CUDA = 6,              /* a CUDA runtime/driver call failed */
    W4A8_ERR_WORKSPACE = 7          /* workspace missing or too small */
} w4a8_status;

/* Weight-format descriptor, filled by w4a8_pack_weights and checked by every
 * call that reads packed weights ("Quantization: formats, error and the real
 * execution path", "Correctness contract": no call may read weights under
 * another quantization schema). */
typedef struct {
    int32_t bits;           /* always 4 */
    int32_t symmetric;      /* 1: codes in [-7,7], z = 0;  0: uint4 codes + z */
    int32_t group;          /* 64 or 128, along K */
    int32_t K;
    int32_t N;
    int32_t layout_version; /* W4A8_LAYOUT_VERSION */
} w4a8_wdesc;

/*
 * Packed weight layout (layout_version 1).  N must be a multiple of 64 and K
 * a multiple of `group`; G = K / group.  The packed buffer holds N*K/2 bytes:
 *   - blocks of 64 output columns x one K-group: block (nb, g) starts at byte
 *     (nb * G + g) * 32 * group, for nb in [0, N/64);
 *   - inside a block, the 16-byte chunk (c, r) starts at (c * 64 + r) * 16,
 *     c in [0, group/32), r in [0, 64), output column n = 64 * nb + r;
 *   - byte b (0..15) of chunk c holds the code of k = g*group + 32*c + b in its
 *     low nibble and the code of k + 16 in its high nibble;
 *   - a symmetric code q in [-7,7] is stored as its 4-bit two's complement
 *     (q & 0xF); an asymmetric code is the uint4 q in [0,15].
 * s_w is fp32 [G][N] row-major; z is uint8 [G][N] row-major (values 0..15).
 * (Why this order: a warp's 32 lanes read 32 consecutive 16-byte chunks of
 * consecutive columns, and each chunk unpacks to two 16-byte runs of
 * consecutive k without byte shuffles.)
 */

/* ---------------------------------------------------------------- sizes -- */

/* Bytes of the packed buffer for a K x N weight (N*K/2). */
W4A8_API size_t w4a8_packed_bytes(int K, int N);

/* Workspace bytes w4a8_gemm needs for M rows (0 when it needs none). */
W4A8_API size_t w4a8_gemm_workspace_size(int M, const w4a8_wdesc* w);

/* Workspace bytes w4a8_moe_grouped_gemm needs. */
W4A8_API size_t w4a8_moe_workspace_size(int T, int E, int topk,
                               const w4a8_wdesc* w1, const w4a8_wdesc* w2);

/* ---------------------------------------------------------------- calls -- */

/*
 * w4a8_pack_weights — offline group-wise 4-bit quantization + packing.
 * Follows "Quantization: formats, error and the real execution path",
 * sections "Basic mapping" and "Symmetric group-wise reference", and
 * "Inference Quantization ch.1" §6 (scale / zero-point).  Per (g, n):
 *   symmetric:  s = max|w| / 7;  q = clamp(rne(w / s), -7, 7)
 *   asymmetric: lo = min(min w, 0), hi = max(max w, 0), s = (hi - lo) / 15,
 *               z = clamp(rne(-lo / s), 0, 15), q = clamp(rne(w / s) + z, 0, 15)
 *   s == 0 (all-zero group): divisor 1, codes 0, z 0, stored s 0.
 * W       device fp32 [K][N] row-major (ldw = N).
 * packed  device, w4a8_packed_bytes(K, N) bytes, layout above.
 * s_w     device fp32 [G][N].
 * z       device uint8 [G][N] for asymmetric; must be NULL when symmetric.
 * out     host descriptor, filled on success (may be NULL).
 * Errors: INVALID_ARG (null pointers, K % group, group not 64/128, N % 64),
 *         NONFINITE via dev_status (a NaN/Inf weight).
 */
W4A8_API w4a8_status w4a8_pack_weights(const float* W, int K, int N, int group, int symmetric,
                              uint8_t* packed, float* s_w, uint8_t* z,
                              w4a8_wdesc* out, int32_t* dev_status, void* stream);

/*
 * w4a8_quant_act — fused per-token absmax reduce + INT8 quantization.
 * "Inference Quantization ch.1" §9.2 and "Kimi 2.7 MoE, 4-bit storage to
 * INT8" §3.3: s_x[m] = max_k|X[m,k]| / 127 (fp32, correctly rounded),
 * q = clamp(rne(X / s_x), -127, 127) with the correctly rounded fp32 quotient;
 * a zero row gives s_x = 0 and codes 0.
 * X        device bf16 [M][ldx] (rows of K used); X and ldx 16-byte aligned
 *          (ldx % 8 == 0).
 * qx       device int8 [M][K];  s_x device fp32 [M].
 * rowsum   device int32 [M][K/group_for_rowsum] = per-group sum of codes
 *          ("Inference Quantization ch.1" §7, the term that multiplies a
 *          weight zero-point), or NULL with group_for_rowsum = 0.
 * Requires K % 8 == 0 and K <= 2^24 (rows longer than 8192 are read twice:
 * once for the absmax, once for the codes).
 */
W4A8_API w4a8_status w4a8_quant_act(const uint16_t* X, int M, int K, int ldx, int group_for_rowsum,
                           int8_t* qx, float* s_x, int32_t* rowsum,
                           int32_t* dev_status, void* stream);

/*
 * w4a8_gemm — Y = W4A8(q_x, packed W): the fused kernel.  Weight codes are
 * unpacked int4 -> int8 inside the tile (the zero-point is subtracted there,
 * in the integer domain), multiplied on the tcgen05 INT8 tensor cores into
 * TMEM one K-group at a time, and each group's exact int32 partial is scaled
 * by s_w and summed in fp32; s_x and the bf16 cast happen in the epilogue
 * ("Inference Quantization ch.1" §4 ideal path and §11 "good path";
 * "Kimi 2.7 MoE, 4-bit storage to INT8" §4.4 step 4).  Small M uses a
 * split-K schedule whose fp32 partials go through `workspace` and are summed
 * in a fixed order (deterministic).
 * qx      device int8 [M][K] (row pitch K, 16-byte aligned).
 * s_x     device fp32 [M].
 * packed, s_w, z: as produced by w4a8_pack_weights (z NULL iff symmetric).
 * w       host descriptor of the packed weight.
 * Y       device bf16 [M][ldy], ldy >= N.
 * workspace / ws_bytes: device scratch of at least
 *         w4a8_gemm_workspace_size(M, w) bytes (may be NULL when that is 0).
 *         Split-K keeps fp32 partial tiles and per-tile flags there.  The
 *         flags carry a per-launch epoch, so the workspace needs no
 *         initialisation and may be reused freely; the one exception: after a
 *         launch that ended with W4A8_ERR_TIMEOUT, zero the workspace before
 *         replaying a captured graph of that launch (a replay repeats the
 *         epoch).  Calls that can overlap on the GPU need separate workspaces.
 * Co-residency: the split-K schedule launches at most one CTA per SM and the
 *         CTA that sums a tile waits for flags set by later CTAs of the same
 *         grid, so it assumes the whole grid is resident at once.  When other
 *         work holds SMs for longer than the wait limit (4 s) the call ends
 *         with W4A8_ERR_TIMEOUT in dev_status instead of a result (no hang).
 *         The same holds for the split-K schedules of w8a8_gemm and
 *         w4a16_gemm.
 * Errors: INVALID_ARG, FORMAT_MISMATCH (bad descriptor), WORKSPACE,
 *         UNSUPPORTED_SHAPE; TIMEOUT via dev_status.
 */
W4A8_API w4a8_status w4a8_gemm(const int8_t* qx, const float* s_x,
                      const uint8_t* packed, const float* s_w, const uint8_t* z,
                      const w4a8_wdesc* w, int M, uint16_t* Y, int ldy,
                      void* workspace, size_t ws_bytes,
                      int32_t* dev_status, void* stream);

/* Workspace bytes w4a8_linear needs for M rows. */
W4A8_API size_t w4a8_linear_workspace_size(int M, const w4a8_wdesc* w);

/*
 * w4a8_linear — the quantized Linear layer Y = X W in one call: per-token
 * INT8 quantization of X (as w4a8_quant_act) followed by the W4A8 GEMM (as
 * w4a8_gemm), "Inference Quantization ch.1" §9.2 then §4.  The GEMM is
 * launched so that its prologue and weight streaming overlap the
 * quantization kernel (programmatic dependent launch); it reads q_x and s_x
 * only after the quantization kernel completed.  Results are identical to
 * w4a8_quant_act followed by w4a8_gemm.
 * X         device bf16 [M][ldx] (rows of K = w->K used), 16-byte aligned,
 *           ldx % 8 == 0, K <= 2^24.
 * packed, s_w, z, w: as for w4a8_gemm.
 * Y         device bf16 [M][ldy], ldy >= N.
 * workspace device scratch of at least w4a8_linear_workspace_size(M, w)
 *           bytes, 16-byte aligned: holds q_x, s_x and the GEMM's split-K
 *           partials.
 * Errors: as w4a8_quant_act and w4a8_gemm.
 */
W4A8_API w4a8_status w4a8_linear(const uint16_t* X, int M, int ldx, const uint8_t* packed, const float* s_w,
                        const uint8_t* z, const w4a8_wdesc* w, uint16_t* Y, int ldy, void* workspace,
                        size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * w4a8_gemm_debug_partials — test-only variant of w4a8_gemm that also writes
 * every exact int32 group partial P[m][g][n] (device int32 [M][G][N]) as the
 * tensor core produced it, so partials can be compared bit for bit.
 */
W4A8_API w4a8_status w4a8_gemm_debug_partials(const int8_t* qx, const float* s_x,
                                     const uint8_t* packed, const float* s_w, const uint8_t* z,
                                     const w4a8_wdesc* w, int M, uint16_t* Y, int ldy,
                                     int32_t* P, void* workspace, size_t ws_bytes,
                                     int32_t* dev_status, void* stream);

/*
 * w4a8_gemm_static_scratch — w4a8_gemm for callers that cannot allocate.
 * The pages have no counterpart of this call: it is a library-integration
 * entry point, not a step of the method.  It computes exactly what w4a8_gemm
 * computes, with the same kernels.
 *
 * Who needs it: callers with no device allocator at the call site, or that
 * must not use one there — a plain C host that links libw4a8.so without a
 * framework and owns no scratch buffer; code running while a caching
 * allocator's pool is capped or frozen; decode loops where cudaMalloc /
 * cudaFree would synchronize the device or can fail under memory pressure.
 * Instead of the caller's workspace, the split-K partials go to one fixed
 * buffer of W4A8_STATIC_SCRATCH_BYTES per device, compiled into the library
 * (a static __device__ array).  This call allocates and frees nothing.
 *
 * Set-up: the first call on each device looks up the buffer's device address
 * with that device current (cudaGetSymbolAddress; this may load the
 * library's device code).  Make that first call before any stream capture.
 * Sharing: every call on a device uses the same buffer.  Two calls whose
 * kernels can overlap on the GPU (different streams without an ordering
 * between them, or concurrent host threads) race on it and give wrong
 * results: issue them on one stream or order them.
 * Nothing in the buffer has to start at zero: each call writes every partial
 * it later reads.
 * Limit: a call whose plan needs more than W4A8_STATIC_SCRATCH_BYTES (i.e.
 * w4a8_gemm_workspace_size(M, w) > W4A8_STATIC_SCRATCH_BYTES; for instance
 * M = 64 with K = 4096, N = 14336) returns W4A8_ERR_WORKSPACE and launches
 * nothing; use w4a8_gemm with a workspace then.  Shapes that need no scratch
 * (large M) run as in w4a8_gemm.
 * Arguments and other errors: as w4a8_gemm, without workspace / ws_bytes;
 * W4A8_ERR_CUDA if the address lookup fails.
 */
#define W4A8_STATIC_SCRATCH_BYTES ((size_t)8 << 20)
W4A8_API w4a8_status w4a8_gemm_static_scratch(const int8_t* qx, const float* s_x,
                                     const uint8_t* packed, const float* s_w, const uint8_t* z,
                                     const w4a8_wdesc* w, int M, uint16_t* Y, int ldy,
                                     int32_t* dev_status, void* stream);

/* ------------------------------------------------------------- W8A8 ---- */

/*
 * The W8A8 variant of the Linear layer ("Inference Quantization ch.1" §4, the
 * INT8 ideal path, with §8.2 per-channel weight scales and §8.3 per-token
 * activation scales):
 *   s_w[n]   = max_k |W[k,n]| / 127,  q_w = clamp(rne(W / s_w), -127, 127)
 *   acc[m,n] = sum_k q_x[m,k] q_w[k,n]                   (exact int32)
 *   Y[m,n]   = s_x[m] * (s_w[n] * acc[m,n])              (fp32, bf16 output)
 * q_x / s_x are w4a8_quant_act's.  Same kernel structure as w4a8_gemm without
 * the 4-bit unpack and without per-group rescaling: the int32 accumulator
 * spans all of K and the epilogue runs once per tile.
 * Descriptor: bits = 8, symmetric = 1, group = K (one scale per column),
 * layout_version = W4A8_LAYOUT_VERSION; the w4a8_* calls reject it.
 * Weight layout: q_w int8 [N][K] row-major (k contiguous), s_w fp32 [N].
 * Limits: K % 128 == 0, K <= 2^17 (so |acc| < 2^31), N % 16 == 0.
 */

/* w8a8_pack_weights — offline per-channel INT8 quantization of W fp32 [K][N]
 * (device, row-major) into q_w / s_w as above; a zero column gives s_w = 0 and
 * codes 0.  out (host) is filled on success.  Errors: INVALID_ARG (null
 * pointers, K % 128, N % 16, q_w not 16-byte aligned); NONFINITE via
 * dev_status. */
W4A8_API w4a8_status w8a8_pack_weights(const float* W, int K, int N, int8_t* q_w, float* s_w, w4a8_wdesc* out,
                                       int32_t* dev_status, void* stream);

/* Workspace bytes w8a8_gemm needs for M rows (split-K int32 partial tiles and
 * their flags; 0 when none). */
W4A8_API size_t w8a8_gemm_workspace_size(int M, const w4a8_wdesc* w);

/* w8a8_gemm — Y = W8A8(q_x, q_w).  qx int8 [M][K] and q_w 16-byte aligned;
 * Y bf16 [M][ldy].  Workspace rules as for w4a8_gemm (split-K partials are
 * int32, so their sum is exact in any order).  Errors as w4a8_gemm. */
W4A8_API w4a8_status w8a8_gemm(const int8_t* qx, const float* s_x, const int8_t* q_w, const float* s_w,
                               const w4a8_wdesc* w, int M, uint16_t* Y, int ldy, void* workspace, size_t ws_bytes,
                               int32_t* dev_status, void* stream);

/* Workspace bytes w8a8_linear needs for M rows (q_x, s_x, the GEMM's). */
W4A8_API size_t w8a8_linear_workspace_size(int M, const w4a8_wdesc* w);

/* w8a8_linear — per-token INT8 quantization of X bf16 [M][ldx] followed by
 * w8a8_gemm, in one call (results identical to the two calls). */
W4A8_API w4a8_status w8a8_linear(const uint16_t* X, int M, int ldx, const int8_t* q_w, const float* s_w,
                                 const w4a8_wdesc* w, uint16_t* Y, int ldy, void* workspace, size_t ws_bytes,
                                 int32_t* dev_status, void* stream);

/* ------------------------------------------------------------ W4A16 ---- */

/*
 * The weight-only W4A16 variant ("Inference Quantization ch.1" §2 and §3.2:
 * the activations stay bf16, the low-bit weights are dequantized inside the
 * GEMM kernel and never written back as a full-precision tensor):
 *   w_hat[k,n] = bf16( fp32( s_w[g,n] * (q[k,n] - z[g,n]) ) ),  g = k / group
 *               (z = 0 for symmetric weights; one fp32 product, one bf16
 *               rounding: the bf16 operand of the tensor-core MMA)
 *   Y[m,n]     = bf16( sum_k X[m,k] * w_hat[k,n] )   fp32 accumulation
 * Reads the W4A8 packed weights as they are (w4a8_pack_weights' packed, s_w,
 * z and descriptor), so one packed copy serves both paths.
 * The dequantization is exact for s_w >= 2^-110 (every scale of a weight
 * group whose largest magnitude exceeds about 1e-32).
 */

/* Workspace bytes w4a16_gemm needs for M rows (split-K fp32 partial tiles and
 * their flags; 0 when none). */
W4A8_API size_t w4a16_gemm_workspace_size(int M, const w4a8_wdesc* w);

/* w4a16_gemm — Y = X · dequant(packed W).
 * X        device bf16 [M][ldx] row-major, 16-byte aligned, ldx % 8 == 0,
 *          ldx >= K (read by TMA).
 * packed, s_w, z, w: as produced by w4a8_pack_weights (z NULL iff
 *          symmetric); packed, s_w and z 16-byte aligned.
 * Y        device bf16 [M][ldy], ldy >= N.
 * workspace / ws_bytes: at least w4a16_gemm_workspace_size(M, w) bytes of
 *          device memory when that is > 0 (caller-owned, reused freely
 *          between calls on one stream).  Split-K partial tiles are summed in
 *          a fixed order, so results are deterministic.
 * Errors: INVALID_ARG (null pointers, alignment, ldx/ldy), FORMAT_MISMATCH
 *         (descriptor, z presence), UNSUPPORTED_SHAPE (K or M > 2^24),
 *         WORKSPACE, CUDA; TIMEOUT via dev_status. */
W4A8_API w4a8_status w4a16_gemm(const uint16_t* X, int M, int ldx, const uint8_t* packed, const float* s_w,
                                const uint8_t* z, const w4a8_wdesc* w, uint16_t* Y, int ldy, void* workspace,
                                size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * w4a8_moe_grouped_gemm — one MoE expert layer, following "Kimi 2.7 MoE,
 * 4-bit storage to INT8" §4.1-4.4:
 *   1. routing in fp32 (the router stays in high precision): topk_idx = the
 *      top-k experts by logit (ties to the lower index), topk_w = their
 *      softmax weights over all E experts (not renormalised);
 *   2. dispatch: count per expert, exclusive prefix sum (expert_offsets),
 *      stable order by (expert, token, slot);
 *   3. per-token INT8 quantization of X, written directly in dispatch order;
 *   4. grouped W4A8 gate_up GEMM over all experts in one persistent launch,
 *      with h = silu(gate) * up fused in its epilogue (gate = columns [0, I),
 *      up = [I, 2I)), h stored as bf16;
 *   5. per-row INT8 quantization of h;
 *   6. grouped W4A8 down GEMM, expert outputs stored as bf16;
 *   7. weighted combine out[t] = sum_j topk_w[t,j] * y[t,j] in fp32, slot order
 *      j = 0..k-1, one bf16 rounding.
 * X       device bf16 [T][H];  logits device fp32 [T][E].
 * Experts are stacked: w1_packed = E consecutive packed [H x 2I] weights
 *         (w4a8_packed_bytes(H, 2I) bytes each), w1_s fp32 [E][G1][2I],
 *         w1_z uint8 [E][G1][2I] (NULL iff symmetric); w2_* likewise for the
 *         [I x H] down weights.  w1 = {K=H, N=2I}, w2 = {K=I, N=H}; both
 *         descriptors must share symmetry and group.
 * out     device bf16 [T][H].
 * topk_idx_out int32 [T][topk], topk_w_out fp32 [T][topk],
 * expert_offsets_out int32 [E+1]: device outputs (all required).
 * Limits: E <= 512, topk <= 16 and topk <= E, H and I multiples of 64,
 *         H and I <= 8192.
 * Errors: as w4a8_gemm; NONFINITE via dev_status for NaN/Inf logits or X.
 */
W4A8_API w4a8_status w4a8_moe_grouped_gemm(const uint16_t* X, const float* logits, int T, int E, int topk,
                                  const uint8_t* w1_packed, const float* w1_s, const uint8_t* w1_z,
                                  const w4a8_wdesc* w1,
                                  const uint8_t* w2_packed, const float* w2_s, const uint8_t* w2_z,
                                  const w4a8_wdesc* w2,
                                  uint16_t* out, int32_t* topk_idx_out, float* topk_w_out,
                                  int32_t* expert_offsets_out,
                                  void* workspace, size_t ws_bytes,
                                  int32_t* dev_status, void* stream);

/* w4a8_moe_grouped_gemm_profiled — the same call, which also records the
 * caller's CUDA events (cudaEvent_t passed as void*; NULL entries skipped)
 * on `stream` at its stage boundaries, for timing: stage_events[0] before
 * routing, [1] before dispatch, [2] before quantizing X, [3] before gate_up,
 * [4] before quantizing h, [5] before down, [6] before the combine, [7] after
 * it.  Events are recorded as external events, so they also work inside a
 * stream capture.  stage_events may be NULL. */
W4A8_API w4a8_status w4a8_moe_grouped_gemm_profiled(
    const uint16_t* X, const float* logits, int T, int E, int topk,
    const uint8_t* w1_packed, const float* w1_s, const uint8_t* w1_z, const w4a8_wdesc* w1,
    const uint8_t* w2_packed, const float* w2_s, const uint8_t* w2_z, const w4a8_wdesc* w2,
    uint16_t* out, int32_t* topk_idx_out, float* topk_w_out, int32_t* expert_offsets_out,
    void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream, void* const* stage_events);

/* Byte offsets of the MoE intermediates inside the workspace, for stage-wise
 * inspection (tests): perm int32 [T*k] (position -> t*k+j), inv int32 [T*k],
 * qx int8 [T*k][H] and sx fp32 [T*k] in dispatch order, h bf16 [T*k][I],
 * qh int8 [T*k][I], sh fp32 [T*k], yd bf16 [T*k][H]. */
typedef struct {
    size_t perm, inv, qx, sx, h, qh, sh, yd, total;
} w4a8_moe_ws_layout;
W4A8_API w4a8_status w4a8_moe_workspace_layout(int T, int E, int topk, const w4a8_wdesc* w1,
                                      const w4a8_wdesc* w2, w4a8_moe_ws_layout* out);

/*
 * w4a8_moe_debug_partials — test-only variant of w4a8_moe_grouped_gemm
 * (same arguments and results) whose grouped GEMMs also write the exact int32
 * group partials of selected (token, slot) pairs as the tensor cores produced
 * them ("Quantization: formats, error and the real execution path",
 * "Correctness contract": partials are compared bit for bit).
 * pair_slot  device int32 [T*topk]: for pair p = t*topk + j, the row of P1 / P2
 *            that receives its partials, or -1 to skip the pair.
 * P1         device int32 [S][H/group][2I]: gate_up partials, S = 1 + the
 *            largest slot in pair_slot; column n < I is gate column n,
 *            n >= I is up column n - I.
 * P2         device int32 [S][I/group][H]: down partials.
 * Rows of skipped pairs and unlisted slots are left untouched.
 */
W4A8_API w4a8_status w4a8_moe_debug_partials(
    const uint16_t* X, const float* logits, int T, int E, int topk,
    const uint8_t* w1_packed, const float* w1_s, const uint8_t* w1_z, const w4a8_wdesc* w1,
    const uint8_t* w2_packed, const float* w2_s, const uint8_t* w2_z, const w4a8_wdesc* w2,
    uint16_t* out, int32_t* topk_idx_out, float* topk_w_out, int32_t* expert_offsets_out,
    void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream,
    const int32_t* pair_slot, int32_t* P1, int32_t* P2);

/* ------------------------------------------- expert-parallel building blocks -- */

/*
 * The three pieces of w4a8_moe_grouped_gemm that an expert-parallel layer
 * ("Kimi 2.7 MoE W4A8 deployment in practice" §5.4: experts spread over
 * GPUs, tokens exchanged all-to-all) runs on different ranks: routing on the
 * rank that holds the tokens, the expert GEMMs on the rank that holds the
 * experts, the weighted combine back on the tokens' rank.  Composed in that
 * order with the rows exchanged in between, they compute exactly what
 * w4a8_moe_grouped_gemm computes (the same kernels, the same rounding).
 */

/* w4a8_moe_route — step 1 alone: topk_idx_out int32 [T][topk], topk_w_out
 * fp32 [T][topk] from logits fp32 [T][E] (device). */
W4A8_API w4a8_status w4a8_moe_route(const float* logits, int T, int E, int topk, int32_t* topk_idx_out,
                                    float* topk_w_out, int32_t* dev_status, void* stream);

/* Workspace bytes w4a8_moe_experts needs for R rows. */
W4A8_API size_t w4a8_moe_experts_workspace_size(int R, int E, const w4a8_wdesc* w1, const w4a8_wdesc* w2);

/* w4a8_moe_experts — steps 2-6 for rows whose expert is already chosen: row
 * r of X bf16 [R][H] goes through expert expert_ids[r] (device int32 [R], in
 * [0, E): the experts stacked in w1_* / w2_* as for w4a8_moe_grouped_gemm);
 * y_out bf16 [R][H] receives each row's expert output, unweighted (bf16, as
 * the layer stores expert outputs before its combine).  An id outside [0, E)
 * is reported as W4A8_ERR_INVALID_ARG through dev_status.  Limits and errors
 * as w4a8_moe_grouped_gemm. */
W4A8_API w4a8_status w4a8_moe_experts(const uint16_t* X, const int32_t* expert_ids, int R, int E,
                                      const uint8_t* w1_packed, const float* w1_s, const uint8_t* w1_z,
                                      const w4a8_wdesc* w1, const uint8_t* w2_packed, const float* w2_s,
                                      const uint8_t* w2_z, const w4a8_wdesc* w2, uint16_t* y_out, void* workspace,
                                      size_t ws_bytes, int32_t* dev_status, void* stream);

/* w4a8_moe_combine — step 7 alone: out[t] = sum_j topk_w[t,j] * y_rows[t*topk
 * + j] in fp32, slot order, one bf16 rounding (y_rows bf16 [T*topk][H] in
 * (token, slot) order; H % 8 == 0; y_rows and out 16-byte aligned). */
W4A8_API w4a8_status w4a8_moe_combine(const uint16_t* y_rows, const float* topk_w, int T, int topk, int H,
                                      uint16_t* out, void* stream);

/* --------------------------------------------------------------- status -- */

/* Synchronizes `stream`, then reads the device status word (0 = W4A8_OK).
 * Returns W4A8_ERR_CUDA if the synchronization or the copy fails. */
W4A8_API w4a8_status w4a8_get_device_status(const int32_t* dev_status, void* stream);

/* Static, human-readable name of a status code. */
W4A8_API const char* w4a8_status_string(w4a8_status s);

/* ABI version (W4A8_ABI_VERSION). */
W4A8_API int w4a8_abi_version(void);

/* Test hook for the failure path of the bounded device waits: launches one
 * tiny kernel that waits on a shared-memory barrier nobody signals, using the
 * same bounded-wait routine as the GEMM kernels, with a limit of `limit_ns`
 * nanoseconds (1e3..1e9).  The kernel gives up, stores W4A8_ERR_TIMEOUT in
 * *dev_status and exits normally. */
W4A8_API w4a8_status w4a8_selftest_bounded_wait(int32_t* dev_status, uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* W4A8_H */
