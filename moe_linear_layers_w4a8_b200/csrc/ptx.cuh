// Thin inline-PTX wrappers for the sm_100a features the kernels use:
// mbarriers, TMA (tiled 2-D and plain bulk copies), tcgen05 (TMEM alloc,
// MMA kind::i8, commit, TMEM load/store, fences), and a bounded wait.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace w4a8 {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h16) { return __uint_as_float(h16 << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&b);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------ mbarrier --

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Like mbar_try_wait, but a thread whose phase is not complete yet sleeps
// (until the phase completes, or at most about `hint_ns`) instead of
// returning at once, so waiting warps do not take issue slots from the
// warps doing work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Shared context of the bounded waits of one CTA.  `abort` lives in shared
// memory: once any wait gives up, every other wait of the CTA returns false
// promptly so that all roles reach the common exit.
struct WaitCtx {
    volatile int* abort;
    int32_t* status;        // device status word of the call (may be null)
    long long limit_cycles; // per-wait limit in SM clock cycles
};

__device__ __forceinline__ void report_status(int32_t* status, int code) {
    if (status) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

// SM cycles that cover `ns` nanoseconds at any SM clock up to 2 GHz.
__host__ __device__ constexpr long long wait_cycles_for_ns(unsigned long long ns) {
    return (long long)(ns * 2ull);
}

// Slow path of wait_bounded: sleep-polls until the phase completes, the CTA
// aborts or the limit runs out.
__device__ __forceinline__ bool wait_bounded_slow(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;  // sleeps <= ~0.1 ms
        if (*w.abort) return false;
        if (clock64() - t0 > w.limit_cycles) {
            *w.abort = 1;
            report_status(w.status, 5);
            return false;
        }
    }
}

// Waits for the phase of `bar` with the given parity to complete.  Returns
// false (after recording W4A8_ERR_TIMEOUT = 5) once `limit_cycles` SM cycles
// have passed, or when another wait of the CTA already gave up.  The SM
// cycle counter is cheap to read, so the common path costs one try_wait.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bounded_slow(bar, parity, w);
}

// Round-half-to-even of the correctly rounded fp32 quotient x / d (the code
// decision of the INT8 quantization), given r = the correctly rounded 1/d.
// x * r is within 2^-22 |x/d| of the exact quotient, and so is the correctly
// rounded quotient; for |x/d| <= 128 both lie on the same side of every
// half-integer unless x * r is within 2^-15 of one.  Only then (about one
// value in 10^4) is the quotient divided out exactly.
__device__ __forceinline__ float rne_quotient(float x, float d, float r) {
    const float t = x * r;
    const float dist = fabsf(t - (floorf(t) + 0.5f));
    return dist > 0x1p-14f ? rintf(t) : rintf(__fdiv_rn(x, d));
}

// Paired fp32 arithmetic (two independent IEEE round-to-nearest results per
// instruction, as the scalar FADD / FFMA would give).
__device__ __forceinline__ uint64_t f2_from_bits(uint32_t lo, uint32_t hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}
__device__ __forceinline__ uint64_t f2_splat(float a) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(a));
    return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Programmatic dependent launch.  launch_dependents: the next kernel of the
// stream (launched with programmatic stream serialization) may start now.
// wait_prerequisites: block until the preceding kernel has completed and its
// memory operations are visible; a kernel launched without the attribute
// returns at once.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_prerequisites() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Global-memory flags between CTAs (split-K partial tiles).
__device__ __forceinline__ void st_release_gpu_u64(unsigned long long* ptr, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(ptr), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned long long ld_acquire_gpu_u64(const unsigned long long* ptr) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(ptr) : "memory");
    return v;
}

// Waits until *ptr == v, bounded like wait_bounded; false on abort / timeout.
__device__ __forceinline__ bool spin_until_equal_u64(const unsigned long long* ptr, unsigned long long v,
                                                     const WaitCtx& w) {
    if (ld_acquire_gpu_u64(ptr) == v) return true;
    const long long t0 = clock64();
    while (true) {
        __nanosleep(200);
        if (ld_acquire_gpu_u64(ptr) == v) return true;
        if (*w.abort) return false;
        if (clock64() - t0 > w.limit_cycles) {
            *w.abort = 1;
            report_status(w.status, 5);
            return false;
        }
    }
}

// ----------------------------------------------------------------- TMA --

// 2-D tiled tensor load into shared memory, completion counted on `bar`.
// Callers keep the innermost coordinate a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// 3-D tiled tensor load (coordinates innermost first).
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int32_t x,
                                            int32_t y, int32_t z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// Plain (untiled) bulk copy global -> shared; addresses 16-byte aligned and
// size a multiple of 16.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// L2 eviction-priority policies for the cache-hinted copies below.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// tma_load_3d / bulk_load with an L2 cache-eviction policy.
__device__ __forceinline__ void tma_load_3d_hint(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int32_t x,
                                                 int32_t y, int32_t z, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void bulk_load_hint(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar,
                                               uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// 16-byte global store marked streaming (evict first): output written once.
__device__ __forceinline__ void st_global_cs_v4(void* ptr, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(ptr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------- tcgen05 --

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_slot)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrives once on `bar` when every tcgen05 operation issued so far by this
// thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, signed int8 x signed int8 -> int32.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, signed int8 x signed int8 -> int32; the
// A tile sits in TMEM (lane = row, 4 consecutive k per 32-bit column).
__device__ __forceinline__ void mma_i8_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile whose rows are
// `row_bytes` (64 or 128) long and swizzled with the matching 64B / 128B
// pattern (8-row atoms, atom stride 8 * row_bytes).
__device__ __forceinline__ uint64_t umma_desc_kmajor(uint32_t smem_addr, uint32_t row_bytes) {
    const uint64_t start = (smem_addr >> 4) & 0x3FFFu;
    const uint64_t lbo = 1;                               // unused for swizzled K-major
    const uint64_t sbo = ((8u * row_bytes) >> 4) & 0x3FFFu;
    const uint64_t layout = (row_bytes == 128u) ? 2u : 4u;  // SWIZZLE_128B : SWIZZLE_64B
    return start | (lbo << 16) | (sbo << 32) | (1ull << 46) | (layout << 61);
}

// Instruction descriptor: kind::i8, D int32, A and B signed int8, both
// K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_i8(int n) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// TMEM -> registers, 32 lanes x N consecutive 32-bit columns (one lane per
// thread of the warp).  `r` must be indexable at compile time after inlining.
template <int N>
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r);

template <>
__device__ __forceinline__ void tmem_ld32<8>(uint32_t taddr, uint32_t* r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7])
                 : "r"(taddr));
}

template <>
__device__ __forceinline__ void tmem_ld32<16>(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, "
        "[%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

template <>
__device__ __forceinline__ void tmem_ld32<32>(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// Registers -> TMEM, 32 lanes x N consecutive 32-bit columns.  These read
// registers only, so they carry no memory clobber (ordinary loads may be
// scheduled across them); being volatile, they stay in order with the other
// tcgen05 statements (fences, waits, MMAs).
template <int N>
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r);

template <>
__device__ __forceinline__ void tmem_st32<8>(uint32_t taddr, const uint32_t* r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]));
}

template <>
__device__ __forceinline__ void tmem_st32<16>(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]));
}

template <>
__device__ __forceinline__ void tmem_st32<32>(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Fill 32 lanes x N columns of TMEM with the same 32-bit value.
template <int N>
__device__ __forceinline__ void tmem_fill32(uint32_t taddr, uint32_t v);

template <>
__device__ __forceinline__ void tmem_fill32<8>(uint32_t taddr, uint32_t v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr), "r"(v));
}

template <>
__device__ __forceinline__ void tmem_fill32<16>(uint32_t taddr, uint32_t v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(
            taddr),
        "r"(v));
}

template <>
__device__ __forceinline__ void tmem_fill32<32>(uint32_t taddr, uint32_t v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,"
        "%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
        "r"(v));
}

// Per-warpgroup register budget (all 128 threads of the warpgroup execute
// it): .dec hands registers back to the CTA's pool, .inc takes them (waiting
// until enough are free).  N is a multiple of 8 in [24, 256].
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Counts the calling threads on named barrier `id` without waiting.
__device__ __forceinline__ void named_bar_arrive(int id, int nthreads) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier that also ORs a predicate over all participating threads;
// every thread gets the same result.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// Bounded wait taken by every lane of a warp, with one decision for the
// whole warp (a lane that gives up makes all lanes give up), so that the
// warp stays converged for the .sync.aligned operations that follow.
__device__ __forceinline__ bool warp_wait_bounded(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
    const bool ok = wait_bounded(bar, parity, w);
    return __all_sync(0xFFFFFFFFu, ok) != 0;
}

// Position of a unit: k-block kb of the virtual tile t, which is the real
// tile ta = base + (t - v0) * stride (stride 1, base = v0 = 0 for a
// contiguous range; stride = the grid size for tiles handed out round-robin),
// ta = mt * n_tiles + nt.  Advanced one unit at a time: no division per
// unit, one per tile when tiles are strided.
struct UnitPos {
    long long t, ta, stride;
    int kb, mt, nt;
    __device__ __forceinline__ UnitPos(long long u, long long KB, int n_tiles, long long v0 = 0, long long base = 0,
                                       long long stride_ = 1) {
        t = u / KB;
        kb = (int)(u - t * KB);
        stride = stride_;
        ta = base + (t - v0) * stride;
        mt = (int)(ta / n_tiles);
        nt = (int)(ta - (long long)mt * n_tiles);
    }
    __device__ __forceinline__ void next(long long KB, int n_tiles) {
        if (++kb == KB) {
            kb = 0;
            ++t;
            ta += stride;
            if (stride == 1) {
                if (++nt == n_tiles) {
                    nt = 0;
                    ++mt;
                }
            } else {
                mt = (int)(ta / n_tiles);
                nt = (int)(ta - (long long)mt * n_tiles);
            }
        }
    }
};

// Whole tiles handed out round-robin (the CTA's i-th tile is blockIdx.x + i *
// gridDim.x), kept as a contiguous range of units in a virtual tile numbering
// (the CTA's i-th tile is virtual tile blockIdx.x * waves + i): CTAs running
// at the same time then work on neighbouring tiles and share their operands
// through L2.
struct RoundRobin {
    long long waves, v0, u0, u1;
    __device__ __forceinline__ RoundRobin(long long tiles, long long KB) {
        const long long grid = gridDim.x, c = blockIdx.x;
        waves = (tiles + grid - 1) / grid;
        const long long mine = c < tiles ? (tiles - 1 - c) / grid + 1 : 0;
        v0 = c * waves;
        u0 = v0 * KB;
        u1 = u0 + mine * KB;
    }
    // real tile of virtual tile t
    __device__ __forceinline__ long long tile(long long t) const {
        return (long long)blockIdx.x + (t - v0) * (long long)gridDim.x;
    }
};

// Position in a ring of n stages and the parity of its current pass.
struct Ring {
    uint32_t idx = 0, phase = 0;
    __device__ __forceinline__ void next(uint32_t n) {
        if (++idx == n) {
            idx = 0;
            phase ^= 1u;
        }
    }
};

// Steps back `n` uses of a ring (for the exit drains).
__device__ __forceinline__ void ring_back(Ring& r, int n) {
    if (r.idx == 0) {
        r.idx = n - 1;
        r.phase ^= 1u;
    } else {
        --r.idx;
    }
}

}  // namespace w4a8
