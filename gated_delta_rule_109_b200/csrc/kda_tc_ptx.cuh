// Inline-PTX wrappers and shared-memory tile helpers of libkda's tcgen05 kernels
// (internal header, sm_100a only).
//
// Shared-memory operands use the no-swizzle canonical layout: core matrices of
// 8 rows x 16 bytes (8 bf16).  A tile indexed (outer, inner) puts element
// (outer, inner) at core_off(outer, inner, s_outer, s_inner).  K-major tiles have
// outer = M (or N) and inner = K; MN-major tiles have outer = K and inner = M (or N).
// In the matrix descriptor, LBO is the byte stride between core matrices along K
// and SBO the stride along M/N.
#pragma once

#include <cuda.h>

#include "kda_internal.cuh"

namespace kda {
namespace tcx {

constexpr long long kWaitCycles = 4000000000ll;   // bounded mbarrier waits: ~2 s at 2 GHz

__device__ __forceinline__ uint32_t core_off(int outer, int inner, uint32_t so, uint32_t si)
{
    return (uint32_t)(outer >> 3) * so + (uint32_t)(inner >> 3) * si + (uint32_t)(outer & 7) * 16u +
           (uint32_t)(inner & 7) * 2u;
}

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    // no-swizzle shared-memory matrix descriptor (sm_100 format, version 1)
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}

__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn)
{
    // D fp32, A bf16, B bf16, dense, no negation
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
                 :: "r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t mbar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(mbar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
                   "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr) : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                 :: "r"(taddr), "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
                    "f"(v[7]), "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]),
                    "f"(v[14]), "f"(v[15]) : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Stores of raw 32-bit words (packed bf16 pairs of an A operand held in tensor memory).
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                 :: "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
                    "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]),
                    "r"(v[14]), "r"(v[15]) : "memory");
}
__device__ __forceinline__ void tmem_st8u(uint32_t taddr, const uint32_t (&v)[8])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 :: "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
                    "r"(v[7]) : "memory");
}

// Split two fp32 values into a packed bf16 pair (first value in the low half) and the
// packed pair of their remainders: x = hi + lo to about 16 significant bits.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t &hi, uint32_t &lo)
{
    const __nv_bfloat162 hv = __floats2bfloat162_rn(x0, x1);
    const float2 hf = __bfloat1622float2(hv);
    const __nv_bfloat162 lv = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&hv);
    lo = *reinterpret_cast<const uint32_t *>(&lv);
}

// Packed fp32 pair arithmetic (the f32x2 forms of sm_100): one instruction does the
// operation on both lanes of a pair, each lane rounded as its scalar form.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// split_pair on a packed pair: the bf16 pair widened back by shifts and the two
// remainders taken by one packed subtraction (exact: x - hi has at most 16
// significant bits), so the bits are those of split_pair.
__device__ __forceinline__ void split_pair2(float2 x, uint32_t &hi, uint32_t &lo)
{
    const __nv_bfloat162 hv = __floats2bfloat162_rn(x.x, x.y);
    const uint32_t hb = *reinterpret_cast<const uint32_t *>(&hv);
    const float2 r = sub2(x, make_float2(__uint_as_float(hb << 16), __uint_as_float(hb & 0xffff0000u)));
    const __nv_bfloat162 lv = __floats2bfloat162_rn(r.x, r.y);
    hi = hb;
    lo = *reinterpret_cast<const uint32_t *>(&lv);
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(mbar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t mbar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(mbar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t mbar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(mbar) : "memory");
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t mbar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(dst), "l"(src), "r"(bytes), "r"(mbar) : "memory");
}

// shared -> global bulk copy through the async proxy (16-byte aligned addresses, a
// multiple of 16 bytes), tracked in the issuing thread's bulk group.  The shared
// source must have been written before a fence.proxy.async by its writers.
__device__ __forceinline__ void bulk_s2g(void *dst, uint32_t src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 :: "l"(dst), "r"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until every committed bulk copy of this thread has read its shared source
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// TMA tensor store (and reduce-add) of one 4-D box from shared memory through a tensor
// map passed as a __grid_constant__ kernel parameter; tracked in the issuing thread's
// bulk group like bulk_s2g.  Coordinates are element indices, innermost first.
__device__ __forceinline__ void tma_store_4d(const void *tmap, uint32_t src, int c0, int c1, int c2, int c3)
{
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
                 :: "l"(tmap), "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3) : "memory");
}
__device__ __forceinline__ void tma_store_3d(const void *tmap, uint32_t src, int c0, int c1, int c2)
{
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
                 :: "l"(tmap), "r"(src), "r"(c0), "r"(c1), "r"(c2) : "memory");
}
__device__ __forceinline__ void tma_reduce_add_4d(const void *tmap, uint32_t src, int c0, int c1, int c2, int c3)
{
    asm volatile("cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
                 :: "l"(tmap), "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3) : "memory");
}

// 16-byte global -> shared copy (sm_80 cp.async); src_bytes = 0 zero-fills the
// destination without reading the source.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// 4-byte global -> shared copy (cp.async.ca); src_bytes = 0 zero-fills
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// L2 prefetch of a global range (16-byte aligned, a multiple of 16 bytes); a hint
// that nothing waits for
__device__ __forceinline__ void l2_prefetch(const void *src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// log(sigmoid(x)) without overflow for either sign of x
__device__ __forceinline__ float log_sigmoid(float x)
{
    return x < 0.f ? x - log1pf(expf(x)) : -log1pf(expf(-x));
}

// One try at the phase with the given parity (true if it has completed).
__device__ __forceinline__ bool mbar_try(uint32_t mbar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}\n" : "=r"(ok) : "r"(mbar), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity; false if it never completed
// within `limit` SM cycles.  The first try reads no clock (most waits on a hot path
// find the phase complete or complete while the try suspends the thread).
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity, long long limit = kWaitCycles)
{
    if (mbar_try(mbar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try(mbar, parity)) return true;
        if (clock64() - t0 > limit) return false;
    }
}

// Split 8 fp32 values into bf16 hi / lo parts packed as two 16-byte vectors.
__device__ __forceinline__ void split8(const float (&x)[8], uint4 &hi, uint4 &lo)
{
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) split_pair2(make_float2(x[2 * i], x[2 * i + 1]), h[i], l[i]);
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ void st_split8(uint8_t *smem, uint32_t off_hi, uint32_t off_lo, const float (&x)[8])
{
    uint4 hi, lo;
    split8(x, hi, lo);
    *reinterpret_cast<uint4 *>(smem + off_hi) = hi;
    *reinterpret_cast<uint4 *>(smem + off_lo) = lo;
}

// tcgen05.mma with the A operand in tensor memory: lane = row of A, each 32-bit
// column a pair of consecutive K elements (the first in the low half), a K step of
// 16 taking 8 columns.
__device__ __forceinline__ void umma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n"
                 :: "r"(d_tmem), "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc) : "memory");
}

// D = A B on hi/lo split operands with A (hi and lo) in tensor memory and B in shared
// memory: hi*hi + lo*hi + hi*lo, K in `ksteps` steps of 16.
__device__ __forceinline__ void mma_split_ta(uint32_t d, uint32_t a_hi, uint32_t a_lo, uint32_t b_hi,
                                             uint32_t b_lo, uint32_t b_lbo, uint32_t b_sbo, int ksteps,
                                             uint32_t idesc)
{
    const uint64_t db[2] = {smem_desc(b_hi, b_lbo, b_sbo), smem_desc(b_lo, b_lbo, b_sbo)};
    const uint64_t sb = (2u * b_lbo) >> 4;
    bool acc = false;
#pragma unroll
    for (int tt = 0; tt < 3; ++tt) {
        const uint32_t a = tt == 1 ? a_lo : a_hi;
        uint64_t bd = db[tt == 2 ? 1 : 0];
#pragma unroll
        for (int ks = 0; ks < ksteps; ++ks) {
            umma_bf16_ta(d, a + 8u * (uint32_t)ks, bd, idesc, acc ? 1u : 0u);
            acc = true;
            bd += sb;
        }
    }
}

// The K steps ks0, ks0 + kstride, ... (kcount of them) of mma_split_ta, all three
// terms; `accumulate` false starts D afresh with the first instruction.
__device__ __forceinline__ void mma_split_ta_steps(uint32_t d, uint32_t a_hi, uint32_t a_lo, uint32_t b_hi,
                                                   uint32_t b_lo, uint32_t b_lbo, uint32_t b_sbo, int ks0,
                                                   int kstride, int kcount, uint32_t idesc, bool accumulate)
{
    const uint64_t db[2] = {smem_desc(b_hi, b_lbo, b_sbo), smem_desc(b_lo, b_lbo, b_sbo)};
    const uint64_t sb = (2u * b_lbo) >> 4;
    bool acc = accumulate;
#pragma unroll
    for (int tt = 0; tt < 3; ++tt) {
        const uint32_t a = tt == 1 ? a_lo : a_hi;
        const uint64_t b0 = db[tt == 2 ? 1 : 0];
#pragma unroll
        for (int i = 0; i < kcount; ++i) {
            const int ks = ks0 + i * kstride;
            umma_bf16_ta(d, a + 8u * (uint32_t)ks, b0 + sb * (uint64_t)ks, idesc, acc ? 1u : 0u);
            acc = true;
        }
    }
}

// One product D (+)= A B on bf16 hi/lo split operands: hi*hi, plus lo*hi when A has
// a lo part and hi*lo when B has one (an operand without a lo part is an exact
// bf16 input).  Each term walks K in `ksteps` steps of 16 (two core matrices,
// 2 * LBO bytes).  The descriptors are built once; a K step adds 2 * LBO / 16 to
// their address field (every operand lies below 256 KB, so the 14-bit field
// never carries into the LBO field).
__device__ __forceinline__ void mma_split(uint32_t d, uint32_t a_hi, uint32_t a_lo, uint32_t a_lbo,
                                          uint32_t a_sbo, uint32_t b_hi, uint32_t b_lo, uint32_t b_lbo,
                                          uint32_t b_sbo, int ksteps, uint32_t idesc, bool accumulate,
                                          bool a_has_lo = true, bool b_has_lo = true)
{
    const uint64_t da[2] = {smem_desc(a_hi, a_lbo, a_sbo), smem_desc(a_lo, a_lbo, a_sbo)};
    const uint64_t db[2] = {smem_desc(b_hi, b_lbo, b_sbo), smem_desc(b_lo, b_lbo, b_sbo)};
    const uint64_t sa = (2u * a_lbo) >> 4, sb = (2u * b_lbo) >> 4;
    bool acc = accumulate;
#pragma unroll
    for (int tt = 0; tt < 3; ++tt) {
        if ((tt == 1 && !a_has_lo) || (tt == 2 && !b_has_lo)) continue;
        uint64_t ad = da[tt == 1 ? 1 : 0], bd = db[tt == 2 ? 1 : 0];
#pragma unroll
        for (int ks = 0; ks < ksteps; ++ks) {
            umma_bf16(d, ad, bd, idesc, acc ? 1u : 0u);
            acc = true;
            ad += sa;
            bd += sb;
        }
    }
}

}  // namespace tcx
}  // namespace kda
