// Thin inline-PTX wrappers for the sm_100a features the M²RNN kernels use:
// mbarriers, bulk (TMA) copies, async-proxy fences and the tcgen05 tensor-core
// instructions (TMEM allocation, MMA, commit, tensor-memory loads).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace m2rnn {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbarrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-suspending probe of an mbarrier phase.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Named barrier over `count` threads (a multiple of 32); id 0 is __syncthreads.
__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Generic-proxy writes to shared memory become visible to the async proxy
// (tensor-core operand reads, bulk copies).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- bulk copy
// One-dimensional bulk copy global -> shared, completing on an mbarrier.
// dst/src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// ---------------------------------------------------------------- L2 policies
// Cache policy for accesses with .L2::cache_hint: lines of data that is
// re-read soon are evicted last.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void st_global_v4_hint(float* dst, float a, float b, float c, float d, uint64_t policy) {
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(dst), "f"(a), "f"(b), "f"(c),
                 "f"(d), "l"(policy)
                 : "memory");
}
// 32-byte (256-bit) global accesses, sm_100: half the instructions of two
// 16-byte ones.  dst / src 32-byte aligned.
__device__ __forceinline__ void st_global_v8_hint(float* dst, const float* v, uint64_t policy) {
    asm volatile("st.global.L2::cache_hint.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8}, %9;" ::"l"(dst), "f"(v[0]),
                 "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "l"(policy)
                 : "memory");
}
__device__ __forceinline__ void ld_global_v8(const float* src, float* v) {
    asm volatile("ld.global.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
                 : "l"(src));
}
// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
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
// D[tmem] (+)= A[smem desc] · B[smem desc], kind::f16 (bf16 inputs, fp32 accumulator).
__device__ __forceinline__ void tc_mma_f16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive (once) on an mbarrier when all previously issued MMAs of this thread complete.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Ties registers written by an earlier tcgen05.ld to a point after
// tc_wait_ld(), so that no use of them is scheduled before the wait.
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// Tensor-memory loads.  32x32b.xN: thread i of the warp reads lane (base+i),
// N consecutive 32-bit columns.  16x32bx2.xN: threads 0-15 read lanes
// base..base+15 at columns [c, c+N); threads 16-31 read the same lanes at
// columns [c+SPLIT, c+SPLIT+N).
#define M2RNN_R4(a) "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
#define M2RNN_R8(a) M2RNN_R4(a), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7])
#define M2RNN_R8o(a, o) "=r"(a[o + 0]), "=r"(a[o + 1]), "=r"(a[o + 2]), "=r"(a[o + 3]), "=r"(a[o + 4]), \
                         "=r"(a[o + 5]), "=r"(a[o + 6]), "=r"(a[o + 7])

template <int N>
__device__ __forceinline__ void tmem_ld_32x32b(uint32_t taddr, uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void tmem_ld_32x32b<4>(uint32_t taddr, uint32_t (&r)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];" : M2RNN_R4(r) : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_32x32b<8>(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : M2RNN_R8(r)
                 : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_32x32b<16>(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : M2RNN_R8o(r, 0), M2RNN_R8o(r, 8)
        : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_32x32b<32>(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : M2RNN_R8o(r, 0), M2RNN_R8o(r, 8), M2RNN_R8o(r, 16), M2RNN_R8o(r, 24)
        : "r"(taddr));
}

// Tensor-memory stores, 32x32b.xN: thread i of the warp writes lane (base+i),
// N consecutive 32-bit columns.  Asynchronous: tc_wait_st() orders them
// before a later tcgen05.ld of the same thread.
#define M2RNN_W4(a) "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3])
template <int N>
__device__ __forceinline__ void tmem_st_32x32b(uint32_t taddr, const uint32_t (&r)[N]) {
    static_assert(N == 4 || N == 8, "tmem_st_32x32b width");
    if constexpr (N == 4) {
        asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), M2RNN_W4(r)
                     : "memory");
    } else {
        asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                     M2RNN_W4(r), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                     : "memory");
    }
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

template <int N, int SPLIT>
__device__ __forceinline__ void tmem_ld_16x32bx2(uint32_t taddr, uint32_t (&r)[N]) {
    static_assert(N == 4 || N == 8 || N == 16 || N == 32, "tmem_ld_16x32bx2 width");
    if constexpr (N == 4) {
        asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x4.b32 {%0,%1,%2,%3}, [%4], %5;"
                     : M2RNN_R4(r)
                     : "r"(taddr), "n"(SPLIT));
    } else if constexpr (N == 8) {
        asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8], %9;"
                     : M2RNN_R8(r)
                     : "r"(taddr), "n"(SPLIT));
    } else if constexpr (N == 16) {
        asm volatile(
            "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
            "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], %17;"
            : M2RNN_R8o(r, 0), M2RNN_R8o(r, 8)
            : "r"(taddr), "n"(SPLIT));
    } else {
        asm volatile(
            "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
            "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
            "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], %33;"
            : M2RNN_R8o(r, 0), M2RNN_R8o(r, 8), M2RNN_R8o(r, 16), M2RNN_R8o(r, 24)
            : "r"(taddr), "n"(SPLIT));
    }
}

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor, no swizzle ("interleaved" canonical layout
// of 8x16-byte core matrices).  lbo/sbo in bytes.  Bits: start address >> 4
// [0,14), leading byte offset >> 4 [16,30), stride byte offset >> 4 [32,46),
// descriptor version 1 [46,48), layout type 0 (no swizzle) [61,64).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    return d;
}

// Instruction descriptor for kind::f16 with bf16 A and B, fp32 D.
// a_mn / b_mn select MN-major operand layouts.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn) {
    return (1u << 4)                       // D format: f32
           | (1u << 7)                     // A format: bf16
           | (1u << 10)                    // B format: bf16
           | ((uint32_t)a_mn << 15)        // A major
           | ((uint32_t)b_mn << 16)        // B major
           | ((uint32_t)(N >> 3) << 17)    // N / 8
           | ((uint32_t)(M >> 4) << 24);   // M / 16
}

// ---------------------------------------------------------------- math
__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// tanh from the identity tanh(x) = 1 - 2 / (1 + e^{2x}), evaluated with the
// exponential and fast-division intrinsics (two SFU operations).  Absolute
// error below ~1e-6 on the whole line (saturates to +-1 for large |x|), about
// three orders of magnitude below tanh.approx.f32, whose ~2^-11 relative error
// the backward's sensitivity over long sequences would amplify.
__device__ __forceinline__ float tanh_exp(float x) {
    const float e = __expf(2.f * x);
    return 1.f - __fdividef(2.f, 1.f + e);
}
// tanh of two values from the identity tanh(x) = 1 - 2 / (1 + 2^{x·2/ln 2}),
// with the hardware base-2 exponential and reciprocal approximations
// (ex2.approx.ftz.f32, rcp.approx.ftz.f32: two SFU operations per value, as
// in tanh_exp) and the surrounding arithmetic on packed fp32 pairs.  For
// large |x| the exponential meets 0 or +inf, and the result is exactly -1 or
// +1.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float2 tanh2_ex2(float2 x) {
    constexpr float kTwoOverLn2 = 2.885390081777927f;   // 2 / ln 2 = 2 log2(e)
    const float2 y = __fmul2_rn(x, make_float2(kTwoOverLn2, kTwoOverLn2));
    const float2 d = __fadd2_rn(make_float2(ex2_approx(y.x), ex2_approx(y.y)), make_float2(1.f, 1.f));
    return __ffma2_rn(make_float2(-2.f, -2.f), make_float2(rcp_approx(d.x), rcp_approx(d.y)), make_float2(1.f, 1.f));
}
// tanh of two values with a small relative error at every argument.  The
// exp form above loses relative accuracy near zero (1 - 2/(1 + e^{2x}) cancels
// to an absolute error of ~2e-7, i.e. 1e-4 of the value at |x| = 1e-3); for
// |x| < 1/8 this takes the odd Taylor series of tanh instead,
//   x - x^3/3 + 2x^5/15 - 17x^7/315,
// whose next term, 62x^9/2835, is below 2e-10 of x there (about one ulp in
// fp32 with the rounding of the evaluation), and the exp form elsewhere
// (relative error at most ~1.6e-6, at |x| = 1/8).
__device__ __forceinline__ float2 tanh2_acc(float2 x) {
    const float2 big = tanh2_ex2(x);
    const float2 s = __fmul2_rn(x, x);
    float2 q = __ffma2_rn(make_float2(-17.f / 315.f, -17.f / 315.f), s, make_float2(2.f / 15.f, 2.f / 15.f));
    q = __ffma2_rn(q, s, make_float2(-1.f / 3.f, -1.f / 3.f));
    const float2 small = __ffma2_rn(__fmul2_rn(x, s), q, x);
    return make_float2(fabsf(x.x) < 0.125f ? small.x : big.x, fabsf(x.y) < 0.125f ? small.y : big.y);
}
__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

}  // namespace m2rnn
