// libw4a8.so: the C ABI declared in include/w4a8.h.
//
// Host side only: argument / shape / descriptor checks, launch planning
// (tile shape, persistent grid, split-K), TMA descriptor encoding, and the
// launches.  Every call is asynchronous on the caller's stream and never
// allocates; scratch lives in the caller's workspace.
#include <algorithm>
#include <atomic>
#include <chrono>
#include <random>
#include <cstdint>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>
#include <mutex>

#include "w4a8.h"
#include "gemm_launch.cuh"
#include "kernels_misc.cuh"
#include "gemm_w8a8.cuh"
#include "gemm_w4a16.cuh"

using namespace w4a8;

namespace {

constexpr unsigned long long kDefaultWaitNs = 4000000000ull;  // 4 s per wait

// ------------------------------------------------------------ device info --

int sm_count_current() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    static std::atomic<int> cache[64];
    if (dev >= 0 && dev < 64) {
        int v = cache[dev].load();
        if (v > 0) return v;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < 64) cache[dev].store(n);
    return n;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Tensor map over the int8 activations [rows][K] seen as 3-D
// (k within group, row, group), box = group x bn x (groups per request);
// swizzle = group bytes (64B or 128B), matching the MMA's K-major layout.
bool make_act_tmap(CUtensorMap* map, const void* base, int rows, int K, int group, int bn, int chunk) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)group, (cuuint64_t)rows, (cuuint64_t)(K / group)};
    cuuint64_t strides[2] = {(cuuint64_t)K, (cuuint64_t)group};
    cuuint32_t box[3] = {(cuuint32_t)group, (cuuint32_t)bn, (cuuint32_t)chunk};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE,
                     group == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Tensor map over a [rows][N] matrix (fp32 scales or uint8 zero-points),
// box = 64 columns x `chunk` rows.
bool make_cols_tmap(CUtensorMap* map, const void* base, long long rows, int N, bool f32, int chunk) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    const int es = f32 ? 4 : 1;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)N * es};
    cuuint32_t box[2] = {64, (cuuint32_t)chunk};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                     const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// All three maps of one GEMM launch.
bool make_gemm_maps(GemmMaps* m, const void* act, int rows, int K, int group, int bn, int mode, const float* s_w,
                    const uint8_t* z, int E, int N) {
    std::memset(m, 0, sizeof(*m));
    const long long wrows = (long long)E * (K / group);
    if (!make_act_tmap(&m->act, act, rows, K, group, bn, chunk_act(bn, group, mode))) return false;
    if (!make_cols_tmap(&m->sw, s_w, wrows, N, true, kChunkScales)) return false;
    if (z && !make_cols_tmap(&m->z, z, wrows, N, false, chunk_packed(group))) return false;
    return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

w4a8_status last_cuda() { return cudaGetLastError() == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA; }

// ---------------------------------------------------------- GEMM configs --

// GEMM launch: per-mode entry points live in gemm_<mode>.cu (see gemm_launch.cuh).
w4a8_status launch_gemm(int mode, bool dbg, int bn, int group, const GemmMaps& maps, const GemmParams& p,
                        int grid, cudaStream_t stream) {
    int r;
    switch (mode) {
        case kModePlain: r = launch_gemm_plain(dbg, bn, group, maps, p, grid, stream); break;
        case kModeSplitK: r = launch_gemm_splitk(dbg, bn, group, maps, p, grid, stream); break;
        case kModeGateUp: r = launch_gemm_gateup(dbg, bn, group, maps, p, grid, stream); break;
        case kModeDown: r = launch_gemm_down(dbg, bn, group, maps, p, grid, stream); break;
        default: r = W4A8_ERR_UNSUPPORTED_SHAPE;
    }
    return static_cast<w4a8_status>(r);
}

int pick_bn(long long rows_per_group) {
    if (rows_per_group <= 16) return 16;
    if (rows_per_group <= 32) return 32;
    if (rows_per_group <= 64) return 64;
    return 128;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Launch plan of the plain (dense) GEMM.
struct GemmPlan {
    int bn, m_tiles, n_tiles, G, grid, slots;
    long long Q;
    bool splitk;
    size_t flags_off;  // split-K: byte offset of the [tiles][slots] flags in the workspace
    size_t ws_bytes;
};

// Launch epochs of split-K GEMMs: nonzero 64-bit values, distinct for every
// launch of this process, starting from a random point so that flags left
// in a reused buffer by another process are unlikely to match.
unsigned long long next_epoch() {
    static std::atomic<unsigned long long> counter{[] {
        std::random_device rd;
        unsigned long long v = ((unsigned long long)rd() << 32) ^ rd();
        v ^= (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count();
        return v;
    }()};
    unsigned long long e = counter.fetch_add(1);
    return e != 0 ? e : counter.fetch_add(1);
}

GemmPlan plan_gemm(int M, int N, int K, int group, int sms) {
    GemmPlan pl{};
    pl.bn = pick_bn(M);
    pl.m_tiles = (M + pl.bn - 1) / pl.bn;
    pl.n_tiles = (N + 127) / 128;
    pl.G = K / group;
    const long long tiles = (long long)pl.m_tiles * pl.n_tiles;
    const long long U = tiles * pl.G;
    if (sms <= 0) sms = 1;
    const long long waves = (tiles + sms - 1) / sms;
    const double eff = (double)tiles / (double)(waves * sms);
    pl.splitk = (eff < 0.85) && pl.G > 1;
    if (pl.splitk) {
        pl.Q = (U + sms - 1) / sms;
        pl.grid = (int)((U + pl.Q - 1) / pl.Q);
        pl.slots = (int)((pl.G + pl.Q - 1) / pl.Q) + 1;
        pl.flags_off = align_up((size_t)tiles * pl.slots * pl.bn * 128 * sizeof(float), 256);
        pl.ws_bytes = pl.flags_off + (size_t)tiles * pl.slots * sizeof(unsigned long long);
    } else {
        pl.Q = (long long)pl.G * waves;
        pl.grid = (int)((tiles + waves - 1) / waves);
        pl.slots = 0;
        pl.ws_bytes = 0;
    }
    return pl;
}

w4a8_status check_wdesc(const w4a8_wdesc* w) {
    if (!w) return W4A8_ERR_INVALID_ARG;
    if (w->bits != 4 || w->layout_version != W4A8_LAYOUT_VERSION) return W4A8_ERR_FORMAT_MISMATCH;
    if (w->group != 64 && w->group != 128) return W4A8_ERR_FORMAT_MISMATCH;
    if (w->symmetric != 0 && w->symmetric != 1) return W4A8_ERR_FORMAT_MISMATCH;
    if (w->K <= 0 || w->N <= 0 || w->K % w->group != 0 || w->N % 64 != 0) return W4A8_ERR_FORMAT_MISMATCH;
    return W4A8_OK;
}

w4a8_status gemm_impl(const int8_t* qx, const float* s_x, const uint8_t* packed, const float* s_w,
                      const uint8_t* z, const w4a8_wdesc* w, int M, uint16_t* Y, int ldy, int32_t* P,
                      void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream) {
    w4a8_status st = check_wdesc(w);
    if (st != W4A8_OK) return st;
    if (M < 0 || !Y || ldy < w->N) return W4A8_ERR_INVALID_ARG;
    if (M == 0) return W4A8_OK;
    if (!qx || !s_x || !packed || !s_w) return W4A8_ERR_INVALID_ARG;
    if (w->symmetric ? (z != nullptr) : (z == nullptr)) return W4A8_ERR_FORMAT_MISMATCH;
    if (!aligned16(qx) || !aligned16(packed) || (z && !aligned16(z))) return W4A8_ERR_INVALID_ARG;
    if (w->K % 16 != 0 || w->K > (1 << 24) || M > (1 << 24)) return W4A8_ERR_UNSUPPORTED_SHAPE;
    const GemmPlan pl = plan_gemm(M, w->N, w->K, w->group, sm_count_current());
    if (pl.ws_bytes > 0 && (!workspace || ws_bytes < pl.ws_bytes)) return W4A8_ERR_WORKSPACE;

    const int mode = pl.splitk ? kModeSplitK : kModePlain;
    GemmMaps maps;
    if (!make_gemm_maps(&maps, qx, M, w->K, w->group, pl.bn, mode, s_w, z, 1, w->N)) return W4A8_ERR_CUDA;
    GemmParams p{};
    p.packed = packed;
    p.s_w = s_w;
    p.z = z;
    p.N = w->N;
    p.K = w->K;
    p.G = pl.G;
    p.symmetric = w->symmetric;
    p.s_x = s_x;
    p.M = M;
    p.mode = pl.splitk ? kModeSplitK : kModePlain;
    p.Y = Y;
    p.ldy = ldy;
    p.vec16 = (aligned16(Y) && ldy % 8 == 0) ? 1 : 0;
    // Launched with programmatic stream serialization: the prologue and the
    // weight stream may overlap the preceding kernel; activations, scales of
    // the activations, Y and the workspace are touched only after it ended.
    p.pdl = 1;
    p.partial = static_cast<float*>(workspace);
    p.slots = pl.slots;
    if (pl.splitk) {
        p.flags = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(workspace) + pl.flags_off);
        p.epoch = next_epoch();
    }
    p.dbgP = P;
    p.n_tiles = pl.n_tiles;
    p.m_tiles = pl.m_tiles;
    p.units_per_cta = pl.Q;
    p.status = dev_status;
    p.wait_ns = kDefaultWaitNs;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return launch_gemm(p.mode, P != nullptr, pl.bn, w->group, maps, p, pl.grid, s);
}

// Launches `kern` on `s`, with programmatic stream serialization when `pdl`
// (the kernel may then start before the preceding kernel of the stream ends;
// the quantization kernels wait for it before touching memory).
template <typename... KArgs, typename... Args>
w4a8_status launch_maybe_pdl(void (*kern)(KArgs...), unsigned grid, unsigned block, cudaStream_t s, bool pdl,
                             Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...) != cudaSuccess) return W4A8_ERR_CUDA;
    return W4A8_OK;
}

w4a8_status launch_quant(const uint16_t* X, int rows, int K, int ldx, int8_t* q, float* s_x, int32_t* rowsum,
                         int group, const int32_t* dest, int dest_k, int32_t* status, cudaStream_t s,
                         bool pdl = false) {
    if (rows == 0) return W4A8_OK;
    if (rows >= 8192 && K <= 1536) {
        // very many short rows (measured on B200: 24576 x 1408 80 -> 57 us;
        // slower for fewer or longer rows, e.g. 65536 x 2048): one warp per
        // row, chunks per lane rounded up to a built size
        const int need = (K / 8 + 31) / 32;
        const int cpl = need <= 1 ? 1 : need <= 2 ? 2 : need <= 4 ? 4 : need <= 6 ? 6 : need <= 8 ? 8 : need <= 12 ? 12 : 16;
        const unsigned blocks = (unsigned)((rows + kQuantRowsPerCta - 1) / kQuantRowsPerCta);
        const unsigned threads = 32 * kQuantRowsPerCta;
        w4a8_status st = W4A8_ERR_UNSUPPORTED_SHAPE;
        switch (cpl) {
#define W4A8_QROWS(n) case n: st = launch_maybe_pdl(quant_act_rows_kernel<n>, blocks, threads, s, pdl, X, rows, K, ldx, q, s_x, rowsum, group, dest, dest_k, status); break;
            W4A8_QROWS(1) W4A8_QROWS(2) W4A8_QROWS(4) W4A8_QROWS(6) W4A8_QROWS(8) W4A8_QROWS(12) W4A8_QROWS(16)
#undef W4A8_QROWS
        }
        return st != W4A8_OK ? st : last_cuda();
    }
    const int cpt = (K / 8 + kQuantThreads - 1) / kQuantThreads;
    if (cpt > 4) {
        // rows longer than 8192: two passes over the row (scatter form unused here)
        if (dest) return W4A8_ERR_UNSUPPORTED_SHAPE;
        const w4a8_status st = launch_maybe_pdl(quant_act_long_kernel, (unsigned)rows, kQuantThreads, s, pdl, X, K,
                                                ldx, q, s_x, rowsum, group, status);
        return st != W4A8_OK ? st : last_cuda();
    }
    w4a8_status st = W4A8_ERR_UNSUPPORTED_SHAPE;
    switch (cpt) {
#define W4A8_QCTA(n) case n: st = launch_maybe_pdl(quant_act_kernel<n>, (unsigned)rows, kQuantThreads, s, pdl, X, K, ldx, q, s_x, rowsum, group, dest, dest_k, status); break;
        W4A8_QCTA(1) W4A8_QCTA(2) W4A8_QCTA(3) W4A8_QCTA(4)
#undef W4A8_QCTA
        default: return W4A8_ERR_UNSUPPORTED_SHAPE;
    }
    return st != W4A8_OK ? st : last_cuda();
}

// ------------------------------------------------------------ MoE layout --


struct MoeLayout {
    size_t mtile_off, perm, inv, qx, sx, h, qh, sh, yd, dcnt, total;
};

// Dispatch over several CTAs: tokens per CTA (a multiple of 256, at most 1024 CTAs).
int dispatch_tokens_per_cta(int T) {
    const int chunks = (T + kDispatchThreads - 1) / kDispatchThreads;
    return kDispatchThreads * ((chunks + 1023) / 1024);
}
int dispatch_ctas(int T) {
    const int tpc = dispatch_tokens_per_cta(T);
    return (T + tpc - 1) / tpc;
}

MoeLayout moe_layout(int T, int E, int topk, int H, int I) {
    MoeLayout L{};
    const size_t R = (size_t)T * topk;
    size_t o = 0;
    L.mtile_off = o; o = align_up(o + sizeof(int32_t) * (E + 1), 256);
    L.perm = o;      o = align_up(o + sizeof(int32_t) * R, 256);
    L.inv = o;       o = align_up(o + sizeof(int32_t) * R, 256);
    L.qx = o;        o = align_up(o + R * H, 256);
    L.sx = o;        o = align_up(o + sizeof(float) * R, 256);
    L.h = o;         o = align_up(o + 2 * R * I, 256);
    L.qh = o;        o = align_up(o + R * I, 256);
    L.sh = o;        o = align_up(o + sizeof(float) * R, 256);
    L.yd = o;        o = align_up(o + 2 * R * H, 256);
    L.dcnt = o;      o = align_up(o + sizeof(int32_t) * (size_t)dispatch_ctas(T) * E, 256);
    L.total = o;
    return L;
}

w4a8_status check_moe(int T, int E, int topk, const w4a8_wdesc* w1, const w4a8_wdesc* w2) {
    w4a8_status st = check_wdesc(w1);
    if (st != W4A8_OK) return st;
    st = check_wdesc(w2);
    if (st != W4A8_OK) return st;
    if (T < 0 || E <= 0 || topk <= 0 || topk > E) return W4A8_ERR_INVALID_ARG;
    if (w1->symmetric != w2->symmetric || w1->group != w2->group) return W4A8_ERR_FORMAT_MISMATCH;
    const int H = w1->K, I2 = w1->N;
    if (I2 % 2 != 0 || w2->K != I2 / 2 || w2->N != H) return W4A8_ERR_FORMAT_MISMATCH;
    const int I = I2 / 2;
    if (E > kMaxExperts || topk > 16) return W4A8_ERR_UNSUPPORTED_SHAPE;
    if (H % 64 != 0 || I % 64 != 0 || H > 8192 || I > 8192) return W4A8_ERR_UNSUPPORTED_SHAPE;
    if ((long long)T * topk > (1ll << 26)) return W4A8_ERR_UNSUPPORTED_SHAPE;
    return W4A8_OK;
}

// ------------------------------------------------------------------ W8A8 --

// A W8A8 weight descriptor: bits 8, one group spanning K (per-channel scale).
w4a8_status check_w8desc(const w4a8_wdesc* w) {
    if (!w) return W4A8_ERR_INVALID_ARG;
    if (w->bits != 8 || w->layout_version != W4A8_LAYOUT_VERSION || w->symmetric != 1 || w->group != w->K)
        return W4A8_ERR_FORMAT_MISMATCH;
    if (w->K <= 0 || w->N <= 0 || w->K % 128 != 0 || w->N % 16 != 0) return W4A8_ERR_FORMAT_MISMATCH;
    return W4A8_OK;
}

// Launch plan of the W8A8 GEMM: (tile, k-block of 128) units over a
// persistent grid, split-K when the tiles do not fill the SMs.
struct W8Plan {
    int bn, m_tiles, n_tiles, KB, grid, slots;
    long long Q;
    bool split;
    size_t flags_off, ws_bytes;
};

W8Plan plan_w8(int M, int N, int K, int sms, int kblock = 128) {
    W8Plan pl{};
    pl.bn = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256;
    pl.m_tiles = (M + pl.bn - 1) / pl.bn;
    pl.n_tiles = (N + 127) / 128;
    pl.KB = K / kblock;
    const long long tiles = (long long)pl.m_tiles * pl.n_tiles;
    const long long U = tiles * pl.KB;
    if (sms <= 0) sms = 1;
    const long long waves = (tiles + sms - 1) / sms;
    const double eff = (double)tiles / (double)(waves * sms);
    pl.split = (eff < 0.85) && pl.KB > 1;
    if (pl.split) {
        pl.Q = (U + sms - 1) / sms;
        pl.grid = (int)((U + pl.Q - 1) / pl.Q);
        pl.slots = (int)((pl.KB + pl.Q - 1) / pl.Q) + 1;
        pl.flags_off = align_up((size_t)tiles * pl.slots * pl.bn * 128 * sizeof(int32_t), 256);
        pl.ws_bytes = pl.flags_off + (size_t)tiles * pl.slots * sizeof(unsigned long long);
    } else {
        pl.Q = (long long)pl.KB * waves;
        pl.grid = (int)((tiles + waves - 1) / waves);
        pl.slots = 0;
        pl.ws_bytes = 0;
    }
    return pl;
}

// 2-D tensor map over an int8 [rows][K] matrix, box 128 k x box_rows rows,
// 128-byte swizzle (the MMA's K-major operand layout).
bool make_k128_tmap(CUtensorMap* map, const void* base, long long rows, int K, int box_rows) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K};
    cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

w4a8_status w8_gemm_impl(const int8_t* qx, const float* s_x, const int8_t* q_w, const float* s_w,
                         const w4a8_wdesc* w, int M, uint16_t* Y, int ldy, void* workspace, size_t ws_bytes,
                         int32_t* dev_status, void* stream) {
    w4a8_status st = check_w8desc(w);
    if (st != W4A8_OK) return st;
    if (M < 0 || !Y || ldy < w->N) return W4A8_ERR_INVALID_ARG;
    if (M == 0) return W4A8_OK;
    if (!qx || !s_x || !q_w || !s_w) return W4A8_ERR_INVALID_ARG;
    if (!aligned16(qx) || !aligned16(q_w)) return W4A8_ERR_INVALID_ARG;
    if (w->K > (1 << 17) || M > (1 << 24)) return W4A8_ERR_UNSUPPORTED_SHAPE;  // |acc| < 2^31
    const W8Plan pl = plan_w8(M, w->N, w->K, sm_count_current());
    if (pl.ws_bytes > 0 && (!workspace || ws_bytes < pl.ws_bytes)) return W4A8_ERR_WORKSPACE;
    CUtensorMap tw, tx;
    if (!make_k128_tmap(&tw, q_w, w->N, w->K, 128) || !make_k128_tmap(&tx, qx, M, w->K, pl.bn)) return W4A8_ERR_CUDA;
    W8Params p{};
    p.N = w->N;
    p.K = w->K;
    p.M = M;
    p.n_tiles = pl.n_tiles;
    p.m_tiles = pl.m_tiles;
    p.KB = pl.KB;
    p.units_per_cta = pl.Q;
    p.s_w = s_w;
    p.s_x = s_x;
    p.Y = Y;
    p.ldy = ldy;
    p.vec16 = (aligned16(Y) && ldy % 8 == 0) ? 1 : 0;
    p.partial = static_cast<int32_t*>(workspace);
    p.slots = pl.slots;
    if (pl.split) {
        p.flags = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(workspace) + pl.flags_off);
        p.epoch = next_epoch();
    }
    p.status = dev_status;
    p.wait_ns = kDefaultWaitNs;
    return static_cast<w4a8_status>(
        launch_w8a8(pl.bn, pl.split, tw, tx, p, pl.grid, static_cast<cudaStream_t>(stream)));
}

// W4A16: (tile, k-block of 64) units; the fp32 partial tiles of a split have
// the int32 ones' size.
W8Plan plan_w16(int M, int N, int K, int sms) { return plan_w8(M, N, K, sms, 64); }

// 3-D tensor map over bf16 activations [rows][K] (row stride ldx elements)
// seen as (64 k, row, k-block): box 64 k x box_rows rows x box_kb k-blocks,
// 128-byte swizzle (the MMA's K-major layout, one 1024-byte-aligned sub-tile
// per k-block).
bool make_bf16_k64_tmap(CUtensorMap* map, const void* base, long long rows, int K, int ldx, int box_rows,
                        int box_kb) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)(K / 64)};
    cuuint64_t strides[2] = {(cuuint64_t)ldx * 2, 128};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, (cuuint32_t)box_kb};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D tensor map over a [G][N] matrix of group scales (fp32) or zero-points
// (uint8), box 128 columns x box_rows groups.
bool make_group_tmap(CUtensorMap* map, const void* base, int G, int N, bool f32, int box_rows) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    const int es = f32 ? 4 : 1;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)G};
    cuuint64_t strides[1] = {(cuuint64_t)N * es};
    cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                     const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// k-blocks of 64 per activation box of the W4A16 kernel (about 16 KB).
int w16_box_kb(int bn) {
    const int k = 16384 / (bn * 128);
    return k < 1 ? 1 : (k > 8 ? 8 : k);
}

w4a8_status w16_gemm_impl(const uint16_t* X, int M, int ldx, const uint8_t* packed, const float* s_w,
                          const uint8_t* z, const w4a8_wdesc* w, uint16_t* Y, int ldy, void* workspace,
                          size_t ws_bytes, int32_t* dev_status, void* stream) {
    w4a8_status st = check_wdesc(w);
    if (st != W4A8_OK) return st;
    if (M < 0 || !Y || ldy < w->N) return W4A8_ERR_INVALID_ARG;
    if (M == 0) return W4A8_OK;
    if (!X || !packed || !s_w || ldx < w->K) return W4A8_ERR_INVALID_ARG;
    if (w->symmetric ? (z != nullptr) : (z == nullptr)) return W4A8_ERR_FORMAT_MISMATCH;
    if (!aligned16(X) || ldx % 8 != 0 || !aligned16(packed) || !aligned16(s_w) || (z && !aligned16(z)))
        return W4A8_ERR_INVALID_ARG;
    if (w->K > (1 << 24) || M > (1 << 24)) return W4A8_ERR_UNSUPPORTED_SHAPE;
    const W8Plan pl = plan_w16(M, w->N, w->K, sm_count_current());
    if (pl.ws_bytes > 0 && (!workspace || ws_bytes < pl.ws_bytes)) return W4A8_ERR_WORKSPACE;
    // scale / zero-point rows of one weight stage of 8 k-blocks: 8 groups of
    // 64, or up to 5 groups of 128 when the stage starts inside a group
    const int sg_rows = w->group == 64 ? 8 : 5;
    CUtensorMap tx, ts, tz;
    if (!make_bf16_k64_tmap(&tx, X, M, w->K, ldx, pl.bn, w16_box_kb(pl.bn)) ||
        !make_group_tmap(&ts, s_w, w->K / w->group, w->N, true, sg_rows))
        return W4A8_ERR_CUDA;
    if (z) {
        if (!make_group_tmap(&tz, z, w->K / w->group, w->N, false, sg_rows)) return W4A8_ERR_CUDA;
    } else {
        tz = ts;  // never read by the symmetric kernels
    }
    W16Params p{};
    p.sg_rows = sg_rows;
    p.N = w->N;
    p.K = w->K;
    p.M = M;
    p.G = w->K / w->group;
    p.group = w->group;
    p.n_tiles = pl.n_tiles;
    p.m_tiles = pl.m_tiles;
    p.KB = pl.KB;
    p.units_per_cta = pl.Q;
    p.packed = packed;
    p.s_w = s_w;
    p.z = z;
    p.Y = Y;
    p.ldy = ldy;
    p.vec16 = (aligned16(Y) && ldy % 8 == 0) ? 1 : 0;
    p.partial = static_cast<float*>(workspace);
    p.slots = pl.slots;
    if (pl.split) {
        p.flags = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(workspace) + pl.flags_off);
        p.epoch = next_epoch();
    }
    p.status = dev_status;
    p.wait_ns = kDefaultWaitNs;
    return static_cast<w4a8_status>(launch_w4a16(pl.bn, pl.split, w->symmetric != 0, tx, ts, tz, p, pl.grid,
                                                 static_cast<cudaStream_t>(stream)));
}

}  // namespace

// ===================================================================== ABI ==

// Workspace of w4a8_linear: q_x [M][K] int8, s_x [M] fp32, then the GEMM's own.
struct LinearLayout {
    size_t qx, sx, gemm, total;
};

LinearLayout linear_layout(int M, const w4a8_wdesc* w) {
    LinearLayout L{};
    L.qx = 0;
    L.sx = align_up((size_t)M * w->K, 256);
    L.gemm = align_up(L.sx + sizeof(float) * (size_t)M, 256);
    L.total = L.gemm + plan_gemm(M, w->N, w->K, w->group, sm_count_current()).ws_bytes;
    return L;
}

extern "C" {

int w4a8_abi_version(void) { return W4A8_ABI_VERSION; }

const char* w4a8_status_string(w4a8_status s) {
    switch (s) {
        case W4A8_OK: return "W4A8_OK";
        case W4A8_ERR_INVALID_ARG: return "W4A8_ERR_INVALID_ARG";
        case W4A8_ERR_UNSUPPORTED_SHAPE: return "W4A8_ERR_UNSUPPORTED_SHAPE";
        case W4A8_ERR_FORMAT_MISMATCH: return "W4A8_ERR_FORMAT_MISMATCH";
        case W4A8_ERR_NONFINITE: return "W4A8_ERR_NONFINITE";
        case W4A8_ERR_TIMEOUT: return "W4A8_ERR_TIMEOUT";
        case W4A8_ERR_CUDA: return "W4A8_ERR_CUDA";
        case W4A8_ERR_WORKSPACE: return "W4A8_ERR_WORKSPACE";
    }
    return "W4A8_ERR_UNKNOWN";
}

size_t w4a8_packed_bytes(int K, int N) {
    if (K <= 0 || N <= 0) return 0;
    return (size_t)K * (size_t)N / 2;
}

size_t w4a8_gemm_workspace_size(int M, const w4a8_wdesc* w) {
    if (M <= 0 || check_wdesc(w) != W4A8_OK) return 0;
    return plan_gemm(M, w->N, w->K, w->group, sm_count_current()).ws_bytes;
}

size_t w4a8_linear_workspace_size(int M, const w4a8_wdesc* w) {
    if (M <= 0 || check_wdesc(w) != W4A8_OK) return 0;
    return linear_layout(M, w).total;
}

size_t w4a8_moe_workspace_size(int T, int E, int topk, const w4a8_wdesc* w1, const w4a8_wdesc* w2) {
    if (check_moe(T, E, topk, w1, w2) != W4A8_OK) return 0;
    return moe_layout(T, E, topk, w1->K, w1->N / 2).total;
}

w4a8_status w4a8_moe_workspace_layout(int T, int E, int topk, const w4a8_wdesc* w1, const w4a8_wdesc* w2,
                                      w4a8_moe_ws_layout* out) {
    w4a8_status st = check_moe(T, E, topk, w1, w2);
    if (st != W4A8_OK) return st;
    if (!out) return W4A8_ERR_INVALID_ARG;
    const MoeLayout L = moe_layout(T, E, topk, w1->K, w1->N / 2);
    out->perm = L.perm;
    out->inv = L.inv;
    out->qx = L.qx;
    out->sx = L.sx;
    out->h = L.h;
    out->qh = L.qh;
    out->sh = L.sh;
    out->yd = L.yd;
    out->total = L.total;
    return W4A8_OK;
}

w4a8_status w4a8_pack_weights(const float* W, int K, int N, int group, int symmetric, uint8_t* packed,
                              float* s_w, uint8_t* z, w4a8_wdesc* out, int32_t* dev_status, void* stream) {
    if (!W || !packed || !s_w) return W4A8_ERR_INVALID_ARG;
    if (group != 64 && group != 128) return W4A8_ERR_INVALID_ARG;
    if (symmetric != 0 && symmetric != 1) return W4A8_ERR_INVALID_ARG;
    if (K <= 0 || N <= 0 || K % group != 0 || N % 64 != 0) return W4A8_ERR_INVALID_ARG;
    if (symmetric ? (z != nullptr) : (z == nullptr)) return W4A8_ERR_INVALID_ARG;
    if (!aligned16(packed)) return W4A8_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    dim3 grid((N + 127) / 128, K / group);
    if (group == 128)
        pack_weights_kernel<128><<<grid, 128, 0, s>>>(W, K, N, symmetric, packed, s_w, z, dev_status);
    else
        pack_weights_kernel<64><<<grid, 128, 0, s>>>(W, K, N, symmetric, packed, s_w, z, dev_status);
    w4a8_status st = last_cuda();
    if (st == W4A8_OK && out) {
        out->bits = 4;
        out->symmetric = symmetric;
        out->group = group;
        out->K = K;
        out->N = N;
        out->layout_version = W4A8_LAYOUT_VERSION;
    }
    return st;
}

w4a8_status w4a8_quant_act(const uint16_t* X, int M, int K, int ldx, int group_for_rowsum, int8_t* qx,
                           float* s_x, int32_t* rowsum, int32_t* dev_status, void* stream) {
    if (M < 0 || K <= 0 || ldx < K) return W4A8_ERR_INVALID_ARG;
    if (M == 0) return W4A8_OK;
    if (!X || !qx || !s_x) return W4A8_ERR_INVALID_ARG;
    if (K % 8 != 0 || ldx % 8 != 0 || !aligned16(X)) return W4A8_ERR_UNSUPPORTED_SHAPE;
    if (K > (1 << 24)) return W4A8_ERR_UNSUPPORTED_SHAPE;
    if (rowsum) {
        if (group_for_rowsum != 64 && group_for_rowsum != 128) return W4A8_ERR_INVALID_ARG;
        if (K % group_for_rowsum != 0) return W4A8_ERR_INVALID_ARG;
    } else if (group_for_rowsum != 0) {
        return W4A8_ERR_INVALID_ARG;
    }
    if ((reinterpret_cast<uintptr_t>(qx) & 7u) != 0 || K % 8 != 0) return W4A8_ERR_UNSUPPORTED_SHAPE;
    return launch_quant(X, M, K, ldx, qx, s_x, rowsum, group_for_rowsum, nullptr, 0, dev_status,
                        static_cast<cudaStream_t>(stream));
}

w4a8_status w4a8_gemm(const int8_t* qx, const float* s_x, const uint8_t* packed, const float* s_w, const uint8_t* z,
                      const w4a8_wdesc* w, int M, uint16_t* Y, int ldy, void* workspace, size_t ws_bytes,
                      int32_t* dev_status, void* stream) {
    return gemm_impl(qx, s_x, packed, s_w, z, w, M, Y, ldy, nullptr, workspace, ws_bytes, dev_status, stream);
}

w4a8_status w4a8_linear(const uint16_t* X, int M, int ldx, const uint8_t* packed, const float* s_w,
                        const uint8_t* z, const w4a8_wdesc* w, uint16_t* Y, int ldy, void* workspace,
                        size_t ws_bytes, int32_t* dev_status, void* stream) {
    w4a8_status st = check_wdesc(w);
    if (st != W4A8_OK) return st;
    if (M < 0 || !Y || ldy < w->N) return W4A8_ERR_INVALID_ARG;
    if (M == 0) return W4A8_OK;
    if (!X || ldx < w->K) return W4A8_ERR_INVALID_ARG;
    if (w->K % 8 != 0 || ldx % 8 != 0 || !aligned16(X) || w->K > (1 << 24)) return W4A8_ERR_UNSUPPORTED_SHAPE;
    const LinearLayout L = linear_layout(M, w);
    if (!workspace || ws_bytes < L.total || !aligned16(workspace)) return W4A8_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int8_t* qx = reinterpret_cast<int8_t*>(ws + L.qx);
    float* sx = reinterpret_cast<float*>(ws + L.sx);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = launch_quant(X, M, w->K, ldx, qx, sx, nullptr, 0, nullptr, 0, dev_status, s);
    if (st != W4A8_OK) return st;
    // The GEMM follows our quantization kernel, which triggers its dependents
    // at entry: launched with programmatic stream serialization, its prologue
    // and weight streaming overlap the quantization.
    return gemm_impl(qx, sx, packed, s_w, z, w, M, Y, ldy, nullptr, ws + L.gemm, ws_bytes - L.gemm, dev_status,
                     stream);
}

w4a8_status w4a8_gemm_debug_partials(const int8_t* qx, const float* s_x, const uint8_t* packed, const float* s_w,
                                     const uint8_t* z, const w4a8_wdesc* w, int M, uint16_t* Y, int ldy, int32_t* P,
                                     void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream) {
    if (!P) return W4A8_ERR_INVALID_ARG;
    return gemm_impl(qx, s_x, packed, s_w, z, w, M, Y, ldy, P, workspace, ws_bytes, dev_status, stream);
}

}  // extern "C"

namespace {

// The MoE layer; with dbg_map, the grouped GEMMs also write the int32 group
// partials of the flagged (token, k) pairs to P1 / P2 (test hook).
w4a8_status moe_impl(const uint16_t* X, const float* logits, int T, int E, int topk, const uint8_t* w1_packed,
                     const float* w1_s, const uint8_t* w1_z, const w4a8_wdesc* w1, const uint8_t* w2_packed,
                     const float* w2_s, const uint8_t* w2_z, const w4a8_wdesc* w2, uint16_t* out,
                     int32_t* topk_idx_out, float* topk_w_out, int32_t* expert_offsets_out, void* workspace,
                     size_t ws_bytes, int32_t* dev_status, void* stream, void* const* stage_events,
                     const int32_t* dbg_map, int32_t* P1, int32_t* P2, const int32_t* pre_ids = nullptr) {
    w4a8_status st = check_moe(T, E, topk, w1, w2);
    if (st != W4A8_OK) return st;
    if (T == 0) return W4A8_OK;
    if (pre_ids && topk != 1) return W4A8_ERR_INVALID_ARG;
    if (!X || !(logits || pre_ids) || !w1_packed || !w1_s || !w2_packed || !w2_s || !out || !topk_idx_out || !topk_w_out ||
        !expert_offsets_out)
        return W4A8_ERR_INVALID_ARG;
    const bool sym = w1->symmetric != 0;
    if (sym ? (w1_z || w2_z) : (!w1_z || !w2_z)) return W4A8_ERR_FORMAT_MISMATCH;
    if (!aligned16(X) || !aligned16(out) || !aligned16(w1_packed) || !aligned16(w2_packed) ||
        (w1_z && !aligned16(w1_z)) || (w2_z && !aligned16(w2_z)))
        return W4A8_ERR_INVALID_ARG;
    const int H = w1->K, I = w1->N / 2, group = w1->group;
    const MoeLayout L = moe_layout(T, E, topk, H, I);
    if (!workspace || ws_bytes < L.total || !aligned16(workspace)) return W4A8_ERR_WORKSPACE;
    const int sms = sm_count_current();
    if (sms <= 0) return W4A8_ERR_CUDA;

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* mtile_off = reinterpret_cast<int32_t*>(ws + L.mtile_off);
    int32_t* perm = reinterpret_cast<int32_t*>(ws + L.perm);
    int32_t* inv = reinterpret_cast<int32_t*>(ws + L.inv);
    int8_t* qx = reinterpret_cast<int8_t*>(ws + L.qx);
    float* sx = reinterpret_cast<float*>(ws + L.sx);
    uint16_t* h = reinterpret_cast<uint16_t*>(ws + L.h);
    int8_t* qh = reinterpret_cast<int8_t*>(ws + L.qh);
    float* sh = reinterpret_cast<float*>(ws + L.sh);
    uint16_t* yd = reinterpret_cast<uint16_t*>(ws + L.yd);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int R = T * topk;
    // Token tile width from the mean rows per expert (measured on the T=64,
    // E=256 top-8 layer: BN = 16 with several m-tiles for the hot experts is
    // faster than one BN = 64 tile per expert, 0.45 vs 0.62 ms for gate_up).
    const int bn = pick_bn(((long long)R + E - 1) / E);
    auto mark = [&](int i) -> bool {
        if (!stage_events || !stage_events[i]) return true;
        return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(stage_events[i]), s, cudaEventRecordExternal) ==
               cudaSuccess;
    };

    // 1. routing (or the given expert of each row)
    if (!mark(0)) return W4A8_ERR_CUDA;
    if (pre_ids) {
        preroute_kernel<<<(unsigned)((T + 255) / 256), 256, 0, s>>>(pre_ids, T, E, topk_idx_out, topk_w_out,
                                                                    dev_status);
        if ((st = last_cuda()) != W4A8_OK) return st;
    } else {
        const int epl = (E + 31) / 32;
        const unsigned blocks = (unsigned)(((long long)T * 32 + 255) / 256);
        switch (epl) {
#define W4A8_ROUTE(n) case n: route_topk_kernel<n><<<blocks, 256, 0, s>>>(logits, T, E, topk, topk_idx_out, topk_w_out, dev_status); break;
            W4A8_ROUTE(1) W4A8_ROUTE(2) W4A8_ROUTE(3) W4A8_ROUTE(4) W4A8_ROUTE(5) W4A8_ROUTE(6) W4A8_ROUTE(7)
            W4A8_ROUTE(8) W4A8_ROUTE(9) W4A8_ROUTE(10) W4A8_ROUTE(11) W4A8_ROUTE(12) W4A8_ROUTE(13)
            W4A8_ROUTE(14) W4A8_ROUTE(15) W4A8_ROUTE(16)
#undef W4A8_ROUTE
            default: return W4A8_ERR_UNSUPPORTED_SHAPE;
        }
        if ((st = last_cuda()) != W4A8_OK) return st;
    }
    // 2. dispatch
    if (!mark(1)) return W4A8_ERR_CUDA;
    if (T <= kDispatchThreads) {
        dispatch_kernel<<<1, kDispatchThreads, 0, s>>>(topk_idx_out, T, E, topk, bn, expert_offsets_out, mtile_off,
                                                       perm, inv);
    } else {
        const int tpc = dispatch_tokens_per_cta(T), C = dispatch_ctas(T);
        int32_t* dcnt = reinterpret_cast<int32_t*>(ws + L.dcnt);
        dispatch_count_kernel<<<C, kDispatchThreads, 0, s>>>(topk_idx_out, T, E, topk, tpc, dcnt);
        if ((st = last_cuda()) != W4A8_OK) return st;
        dispatch_scan_kernel<<<1, kDispatchScanThreads, 0, s>>>(dcnt, C, E, bn, expert_offsets_out, mtile_off);
        if ((st = last_cuda()) != W4A8_OK) return st;
        dispatch_scatter_kernel<<<C, kDispatchThreads, 0, s>>>(topk_idx_out, T, E, topk, tpc, dcnt, perm, inv);
    }
    if ((st = last_cuda()) != W4A8_OK) return st;
    // 3. quantize X straight into dispatch order
    if (!mark(2)) return W4A8_ERR_CUDA;
    if ((st = launch_quant(X, T, H, H, qx, sx, nullptr, 0, inv, topk, dev_status, s)) != W4A8_OK) return st;
    // 4. gate_up + SiLU * up
    if (!mark(3)) return W4A8_ERR_CUDA;
    {
        GemmMaps maps;
        if (!make_gemm_maps(&maps, qx, R, H, group, bn, kModeGateUp, w1_s, w1_z, E, w1->N)) return W4A8_ERR_CUDA;
        GemmParams p{};
        p.packed = w1_packed;
        p.s_w = w1_s;
        p.z = w1_z;
        p.N = w1->N;
        p.K = H;
        p.G = H / group;
        p.packed_estride = (long long)w1->N * H / 2;
        p.sw_estride = (long long)p.G * w1->N;
        p.symmetric = w1->symmetric;
        p.s_x = sx;
        p.mode = kModeGateUp;
        p.Y = h;
        p.ldy = I;
        p.vec16 = 1;
        p.n_tiles = I / 64;
        p.expert_off = expert_offsets_out;
        p.mtile_off = mtile_off;
        p.E = E;
        p.I = I;
        p.status = dev_status;
        p.wait_ns = kDefaultWaitNs;
        p.dbgP = P1;
        p.dbg_map = dbg_map;
        p.dbg_perm = perm;
        if ((st = launch_gemm(kModeGateUp, dbg_map != nullptr, bn, group, maps, p, sms, s)) != W4A8_OK) return st;
    }
    // 5. quantize h per (token, expert) row
    if (!mark(4)) return W4A8_ERR_CUDA;
    if ((st = launch_quant(h, R, I, I, qh, sh, nullptr, 0, nullptr, 0, dev_status, s)) != W4A8_OK) return st;
    // 6. down
    if (!mark(5)) return W4A8_ERR_CUDA;
    {
        GemmMaps maps;
        if (!make_gemm_maps(&maps, qh, R, I, group, bn, kModeDown, w2_s, w2_z, E, H)) return W4A8_ERR_CUDA;
        GemmParams p{};
        p.packed = w2_packed;
        p.s_w = w2_s;
        p.z = w2_z;
        p.N = H;
        p.K = I;
        p.G = I / group;
        p.packed_estride = (long long)H * I / 2;
        p.sw_estride = (long long)p.G * H;
        p.symmetric = w2->symmetric;
        p.s_x = sh;
        p.mode = kModeDown;
        p.Y = yd;
        p.ldy = H;
        p.vec16 = 1;
        p.n_tiles = (H + 127) / 128;
        p.expert_off = expert_offsets_out;
        p.mtile_off = mtile_off;
        p.E = E;
        p.status = dev_status;
        p.wait_ns = kDefaultWaitNs;
        p.dbgP = P2;
        p.dbg_map = dbg_map;
        p.dbg_perm = perm;
        if ((st = launch_gemm(kModeDown, dbg_map != nullptr, bn, group, maps, p, sms, s)) != W4A8_OK) return st;
    }
    // 7. weighted combine
    if (!mark(6)) return W4A8_ERR_CUDA;
    {
        const long long n = (long long)T * (H / 8);
        combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(yd, topk_w_out, inv, T, topk, H, out);
        if ((st = last_cuda()) != W4A8_OK) return st;
    }
    if (!mark(7)) return W4A8_ERR_CUDA;
    return W4A8_OK;
}

}  // namespace

extern "C" {

w4a8_status w4a8_moe_grouped_gemm_profiled(const uint16_t* X, const float* logits, int T, int E, int topk,
                                           const uint8_t* w1_packed, const float* w1_s, const uint8_t* w1_z,
                                           const w4a8_wdesc* w1, const uint8_t* w2_packed, const float* w2_s,
                                           const uint8_t* w2_z, const w4a8_wdesc* w2, uint16_t* out,
                                           int32_t* topk_idx_out, float* topk_w_out, int32_t* expert_offsets_out,
                                           void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream,
                                           void* const* stage_events) {
    return moe_impl(X, logits, T, E, topk, w1_packed, w1_s, w1_z, w1, w2_packed, w2_s, w2_z, w2, out, topk_idx_out,
                    topk_w_out, expert_offsets_out, workspace, ws_bytes, dev_status, stream, stage_events, nullptr,
                    nullptr, nullptr);
}

w4a8_status w4a8_moe_debug_partials(const uint16_t* X, const float* logits, int T, int E, int topk,
                                    const uint8_t* w1_packed, const float* w1_s, const uint8_t* w1_z,
                                    const w4a8_wdesc* w1, const uint8_t* w2_packed, const float* w2_s,
                                    const uint8_t* w2_z, const w4a8_wdesc* w2, uint16_t* out, int32_t* topk_idx_out,
                                    float* topk_w_out, int32_t* expert_offsets_out, void* workspace,
                                    size_t ws_bytes, int32_t* dev_status, void* stream, const int32_t* pair_slot,
                                    int32_t* P1, int32_t* P2) {
    if (!pair_slot || !P1 || !P2) return W4A8_ERR_INVALID_ARG;
    return moe_impl(X, logits, T, E, topk, w1_packed, w1_s, w1_z, w1, w2_packed, w2_s, w2_z, w2, out, topk_idx_out,
                    topk_w_out, expert_offsets_out, workspace, ws_bytes, dev_status, stream, nullptr, pair_slot, P1,
                    P2);
}

w4a8_status w4a8_moe_grouped_gemm(const uint16_t* X, const float* logits, int T, int E, int topk,
                                  const uint8_t* w1_packed, const float* w1_s, const uint8_t* w1_z,
                                  const w4a8_wdesc* w1, const uint8_t* w2_packed, const float* w2_s,
                                  const uint8_t* w2_z, const w4a8_wdesc* w2, uint16_t* out,
                                  int32_t* topk_idx_out, float* topk_w_out, int32_t* expert_offsets_out,
                                  void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream) {
    return w4a8_moe_grouped_gemm_profiled(X, logits, T, E, topk, w1_packed, w1_s, w1_z, w1, w2_packed, w2_s, w2_z,
                                          w2, out, topk_idx_out, topk_w_out, expert_offsets_out, workspace,
                                          ws_bytes, dev_status, stream, nullptr);
}

w4a8_status w4a8_moe_route(const float* logits, int T, int E, int topk, int32_t* topk_idx_out, float* topk_w_out,
                           int32_t* dev_status, void* stream) {
    if (T < 0 || E <= 0 || topk <= 0 || topk > E || E > kMaxExperts || topk > 16) return W4A8_ERR_INVALID_ARG;
    if (T == 0) return W4A8_OK;
    if (!logits || !topk_idx_out || !topk_w_out) return W4A8_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int epl = (E + 31) / 32;
    const unsigned blocks = (unsigned)(((long long)T * 32 + 255) / 256);
    switch (epl) {
#define W4A8_ROUTE(n) case n: route_topk_kernel<n><<<blocks, 256, 0, s>>>(logits, T, E, topk, topk_idx_out, topk_w_out, dev_status); break;
        W4A8_ROUTE(1) W4A8_ROUTE(2) W4A8_ROUTE(3) W4A8_ROUTE(4) W4A8_ROUTE(5) W4A8_ROUTE(6) W4A8_ROUTE(7)
        W4A8_ROUTE(8) W4A8_ROUTE(9) W4A8_ROUTE(10) W4A8_ROUTE(11) W4A8_ROUTE(12) W4A8_ROUTE(13)
        W4A8_ROUTE(14) W4A8_ROUTE(15) W4A8_ROUTE(16)
#undef W4A8_ROUTE
        default: return W4A8_ERR_UNSUPPORTED_SHAPE;
    }
    return last_cuda();
}

size_t w4a8_moe_experts_workspace_size(int R, int E, const w4a8_wdesc* w1, const w4a8_wdesc* w2) {
    if (check_moe(R, E, 1, w1, w2) != W4A8_OK) return 0;
    return moe_layout(R, E, 1, w1->K, w1->N / 2).total + align_up(sizeof(int32_t) * (size_t)(2 * R + E + 1), 256);
}

w4a8_status w4a8_moe_experts(const uint16_t* X, const int32_t* expert_ids, int R, int E, const uint8_t* w1_packed,
                             const float* w1_s, const uint8_t* w1_z, const w4a8_wdesc* w1, const uint8_t* w2_packed,
                             const float* w2_s, const uint8_t* w2_z, const w4a8_wdesc* w2, uint16_t* y_out,
                             void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream) {
    w4a8_status st = check_moe(R, E, 1, w1, w2);
    if (st != W4A8_OK) return st;
    if (R == 0) return W4A8_OK;
    if (!expert_ids) return W4A8_ERR_INVALID_ARG;
    const size_t base = moe_layout(R, E, 1, w1->K, w1->N / 2).total;
    if (!workspace || ws_bytes < w4a8_moe_experts_workspace_size(R, E, w1, w2)) return W4A8_ERR_WORKSPACE;
    // the routing outputs of the layer (expert id, weight 1, offsets) live past the layer's own workspace
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* idx = reinterpret_cast<int32_t*>(ws + base);
    float* wts = reinterpret_cast<float*>(idx + R);
    int32_t* offs = reinterpret_cast<int32_t*>(wts + R);
    return moe_impl(X, nullptr, R, E, 1, w1_packed, w1_s, w1_z, w1, w2_packed, w2_s, w2_z, w2, y_out, idx, wts, offs,
                    workspace, base, dev_status, stream, nullptr, nullptr, nullptr, nullptr, expert_ids);
}

w4a8_status w4a8_moe_combine(const uint16_t* y_rows, const float* topk_w, int T, int topk, int H, uint16_t* out,
                             void* stream) {
    if (T < 0 || topk <= 0 || H <= 0 || H % 8 != 0) return W4A8_ERR_INVALID_ARG;
    if (T == 0) return W4A8_OK;
    if (!y_rows || !topk_w || !out || !aligned16(y_rows) || !aligned16(out)) return W4A8_ERR_INVALID_ARG;
    const long long n = (long long)T * (H / 8);
    combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        y_rows, topk_w, nullptr, T, topk, H, out);
    return last_cuda();
}

w4a8_status w4a8_get_device_status(const int32_t* dev_status, void* stream) {
    if (!dev_status) return W4A8_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return W4A8_ERR_CUDA;
    int32_t v = 0;
    if (cudaMemcpy(&v, dev_status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return W4A8_ERR_CUDA;
    return static_cast<w4a8_status>(v);
}

w4a8_status w8a8_pack_weights(const float* W, int K, int N, int8_t* q_w, float* s_w, w4a8_wdesc* out,
                              int32_t* dev_status, void* stream) {
    if (!W || !q_w || !s_w) return W4A8_ERR_INVALID_ARG;
    if (K <= 0 || N <= 0 || K % 128 != 0 || N % 16 != 0) return W4A8_ERR_INVALID_ARG;
    if (!aligned16(q_w)) return W4A8_ERR_INVALID_ARG;
    pack_w8_kernel<<<(unsigned)((N + 127) / 128), 128, 0, static_cast<cudaStream_t>(stream)>>>(W, K, N, q_w, s_w,
                                                                                              dev_status);
    w4a8_status st = last_cuda();
    if (st == W4A8_OK && out) {
        out->bits = 8;
        out->symmetric = 1;
        out->group = K;
        out->K = K;
        out->N = N;
        out->layout_version = W4A8_LAYOUT_VERSION;
    }
    return st;
}

size_t w8a8_gemm_workspace_size(int M, const w4a8_wdesc* w) {
    if (M <= 0 || check_w8desc(w) != W4A8_OK) return 0;
    return plan_w8(M, w->N, w->K, sm_count_current()).ws_bytes;
}

size_t w4a16_gemm_workspace_size(int M, const w4a8_wdesc* w) {
    if (M <= 0 || check_wdesc(w) != W4A8_OK) return 0;
    return plan_w16(M, w->N, w->K, sm_count_current()).ws_bytes;
}

w4a8_status w4a16_gemm(const uint16_t* X, int M, int ldx, const uint8_t* packed, const float* s_w, const uint8_t* z,
                       const w4a8_wdesc* w, uint16_t* Y, int ldy, void* workspace, size_t ws_bytes,
                       int32_t* dev_status, void* stream) {
    return w16_gemm_impl(X, M, ldx, packed, s_w, z, w, Y, ldy, workspace, ws_bytes, dev_status, stream);
}

w4a8_status w8a8_gemm(const int8_t* qx, const float* s_x, const int8_t* q_w, const float* s_w, const w4a8_wdesc* w,
                      int M, uint16_t* Y, int ldy, void* workspace, size_t ws_bytes, int32_t* dev_status,
                      void* stream) {
    return w8_gemm_impl(qx, s_x, q_w, s_w, w, M, Y, ldy, workspace, ws_bytes, dev_status, stream);
}

size_t w8a8_linear_workspace_size(int M, const w4a8_wdesc* w) {
    if (M <= 0 || check_w8desc(w) != W4A8_OK) return 0;
    const size_t sx = align_up((size_t)M * w->K, 256);
    const size_t g = align_up(sx + sizeof(float) * (size_t)M, 256);
    return g + plan_w8(M, w->N, w->K, sm_count_current()).ws_bytes;
}

w4a8_status w8a8_linear(const uint16_t* X, int M, int ldx, const int8_t* q_w, const float* s_w, const w4a8_wdesc* w,
                        uint16_t* Y, int ldy, void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream) {
    w4a8_status st = check_w8desc(w);
    if (st != W4A8_OK) return st;
    if (M < 0 || !Y || ldy < w->N) return W4A8_ERR_INVALID_ARG;
    if (M == 0) return W4A8_OK;
    if (!X || ldx < w->K) return W4A8_ERR_INVALID_ARG;
    if (ldx % 8 != 0 || !aligned16(X)) return W4A8_ERR_UNSUPPORTED_SHAPE;
    const size_t need = w8a8_linear_workspace_size(M, w);
    if (!workspace || ws_bytes < need || !aligned16(workspace)) return W4A8_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const size_t sxo = align_up((size_t)M * w->K, 256);
    const size_t go = align_up(sxo + sizeof(float) * (size_t)M, 256);
    int8_t* qx = reinterpret_cast<int8_t*>(ws);
    float* sx = reinterpret_cast<float*>(ws + sxo);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = launch_quant(X, M, w->K, ldx, qx, sx, nullptr, 0, nullptr, 0, dev_status, s);
    if (st != W4A8_OK) return st;
    return w8_gemm_impl(qx, sx, q_w, s_w, w, M, Y, ldy, ws + go, ws_bytes - go, dev_status, stream);
}

w4a8_status w4a8_selftest_bounded_wait(int32_t* dev_status, uint64_t limit_ns, void* stream) {
    if (!dev_status || limit_ns < 1000ull || limit_ns > 1000000000ull) return W4A8_ERR_INVALID_ARG;
    bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev_status, limit_ns);
    return last_cuda();
}

}  // extern "C"

// ------------------------------------------------ static-scratch GEMM entry --
//
// w4a8_gemm_static_scratch: w4a8_gemm for callers that cannot allocate (see
// include/w4a8.h).  The split-K partials live in the fixed buffer below
// instead of a caller workspace.  `g_static_scratch` names the buffer on the
// host side only; it is not a device address.  The device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[W4A8_STATIC_SCRATCH_BYTES];

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxScratchDevices] = {};

// Device address of g_static_scratch on the current device, or null.
void* static_scratch_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxScratchDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = ptr;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" w4a8_status w4a8_gemm_static_scratch(const int8_t* qx, const float* s_x, const uint8_t* packed,
                                                const float* s_w, const uint8_t* z, const w4a8_wdesc* w, int M,
                                                uint16_t* Y, int ldy, int32_t* dev_status, void* stream) {
    w4a8_status st = check_wdesc(w);
    if (st != W4A8_OK) return st;
    if (M < 0) return W4A8_ERR_INVALID_ARG;
    const size_t need = M > 0 ? plan_gemm(M, w->N, w->K, w->group, sm_count_current()).ws_bytes : 0;
    if (need > W4A8_STATIC_SCRATCH_BYTES) return W4A8_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need > 0) {
        scratch = static_scratch_current_device();
        if (!scratch) return W4A8_ERR_CUDA;
    }
    return gemm_impl(qx, s_x, packed, s_w, z, w, M, Y, ldy, nullptr, scratch, need > 0 ? W4A8_STATIC_SCRATCH_BYTES : 0,
                     dev_status, stream);
}
