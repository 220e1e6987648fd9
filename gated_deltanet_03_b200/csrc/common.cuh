// Shared device helpers for the sm_100a kernels: dtype loads/stores, warp reductions,
// the NVFP4 conversions (hardware cvt), and thin wrappers over the mbarrier, TMA and
// tcgen05 PTX instructions used by the tensor-core kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

#define GDN_DEV __device__ __forceinline__

namespace gdn {

// ---------------------------------------------------------------- dtype access ----

// Eight consecutive values of a bf16 or fp32 row as fp32 (16-byte aligned source).
template <bool BF16>
GDN_DEV void load8(const void *base, size_t idx, float (&x)[8]) {
    if constexpr (BF16) {
        uint4 u = *reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(base) + idx);
        const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(p[i]);
            x[2 * i] = f.x;
            x[2 * i + 1] = f.y;
        }
    } else {
        const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(base) + idx);
        float4 a = p[0], b = p[1];
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
}

template <bool BF16>
GDN_DEV void load4(const void *base, size_t idx, float (&x)[4]) {
    if constexpr (BF16) {
        uint2 u = *reinterpret_cast<const uint2 *>(reinterpret_cast<const __nv_bfloat16 *>(base) + idx);
        const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&u);
        float2 f0 = __bfloat1622float2(p[0]), f1 = __bfloat1622float2(p[1]);
        x[0] = f0.x; x[1] = f0.y; x[2] = f1.x; x[3] = f1.y;
    } else {
        float4 a = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(base) + idx);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    }
}

template <bool BF16>
GDN_DEV float load1(const void *base, size_t idx) {
    if constexpr (BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(base)[idx]);
    else return reinterpret_cast<const float *>(base)[idx];
}

template <bool BF16>
GDN_DEV void store8(void *base, size_t idx, const float (&x)[8]) {
    if constexpr (BF16) {
        uint4 u;
        __nv_bfloat162 *p = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) p[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        *reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(base) + idx) = u;
    } else {
        float4 *p = reinterpret_cast<float4 *>(reinterpret_cast<float *>(base) + idx);
        p[0] = make_float4(x[0], x[1], x[2], x[3]);
        p[1] = make_float4(x[4], x[5], x[6], x[7]);
    }
}

template <bool BF16>
GDN_DEV void store1(void *base, size_t idx, float x) {
    if constexpr (BF16) reinterpret_cast<__nv_bfloat16 *>(base)[idx] = __float2bfloat16_rn(x);
    else reinterpret_cast<float *>(base)[idx] = x;
}

GDN_DEV float round_bf16(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// ----------------------------------------------------------------- reductions ----

// Sum over groups of WIDTH consecutive lanes (WIDTH a power of two <= 32).
template <int WIDTH>
GDN_DEV float group_sum(float v) {
#pragma unroll
    for (int off = WIDTH / 2; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// ---------------------------------------------------------------------- gates ----

// softplus(x) = log(1 + e^x), stable for large x; library expf / log1pf.
GDN_DEV float softplus_f(float x) { return x > 20.0f ? x : log1pf(expf(x)); }
GDN_DEV float sigmoid_f(float x) { return 1.0f / (1.0f + expf(-x)); }
// 2^x with the hardware approximation (relative error about 2^-22; results below the smallest
// normal float are flushed to zero), and e^x through it.
GDN_DEV float exp2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
constexpr float kLog2e = 1.4426950408889634f;
GDN_DEV float exp_approx(float x) { return exp2_approx(x * kLog2e); }

// z * sigmoid(z) with the fast exponential and division intrinsics (a few ulp; the tail's
// tolerance is 1e-5 relative).
GDN_DEV float silu_fast(float z) { return __fdividef(z, 1.0f + exp_approx(-z)); }

// log of the decay gate, g = -exp(A_log) * softplus(a + dt_bias), and the write strength.
GDN_DEV void gdn_gates(float a, float b, float A_log, float dt_bias, float &g, float &beta) {
    g = -expf(A_log) * softplus_f(a + dt_bias);
    beta = sigmoid_f(b);
}

// --------------------------------------------------------------- NVFP4 convert ----

// E4M3 code of s >= 0 (round to nearest even, saturating to 448).
GDN_DEV uint32_t cvt_e4m3(float s) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(s));
    return r & 0xFFu;
}

// fp32 value of a non-negative E4M3 code, from the format's definition (exact):
// exponent field e (bias 7) and mantissa m; e == 0 is subnormal, m * 2^-9.
GDN_DEV float e4m3_to_f32(uint32_t c) {
    uint32_t e = (c >> 3) & 15u, m = c & 7u;
    return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;
}

// Eight E2M1 codes packed in a 32-bit word, value 2j in the low nibble of byte j and
// 2j+1 in the high nibble (round to nearest even, saturating to +-6).
GDN_DEV uint32_t cvt_e2m1x8(const float (&p)[8]) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(p[0]), "f"(p[1]), "f"(p[2]), "f"(p[3]), "f"(p[4]), "f"(p[5]), "f"(p[6]), "f"(p[7]));
    return r;
}

// amax / 6 rounded to nearest even, as __fdiv_rn(amax, 6.0f) gives it: the product with the
// rounded reciprocal corrected by one fused residual step (a division by a constant as in
// Markstein's FMA division schemes). For finite amax >= 2^-125 this equals the correctly rounded
// quotient for every input (checked exhaustively by tests/test_div6_cpu.py); below that, and
// for inf or NaN, the plain division is used.
GDN_DEV float div6_rn(float amax) {
    if (amax >= 0x1p-125f && amax <= 3.4028235e38f) {
        const float c = 1.0f / 6.0f;
        const float q0 = amax * c;
        return fmaf(fmaf(-q0, 6.0f, amax), c, q0);
    }
    return __fdiv_rn(amax, 6.0f);
}

// NVFP4 block scale from the block's largest magnitude and the global encode scale `gs`,
// in this order of fp32 operations: s = (amax / 6) * gs; sb = E4M3(s); r = gs / sb
// (r = 0 when sb == 0). Returns the E4M3 code; *r is the factor that maps values to codes.
GDN_DEV uint32_t nvfp4_block_scale(float amax, float gs, float &r) {
    float s = __fmul_rn(div6_rn(amax), gs);
    uint32_t sb = cvt_e4m3(s);
    r = (sb == 0u) ? 0.0f : __fdiv_rn(gs, e4m3_to_f32(sb));
    return sb;
}

// Eight values of a block, scaled by r and packed as E2M1 codes.
GDN_DEV uint32_t nvfp4_pack8(const float (&x)[8], float r) {
    float p[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) p[j] = __fmul_rn(x[j], r);
    return cvt_e2m1x8(p);
}

GDN_DEV float amax8(const float (&x)[8]) {
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(x[j]));
    return m;
}

// -------------------------------------------------------------- device status ----

// The library's device control block: the status word that bounded waits report into, the
// wait limit in nanoseconds (1 s unless lowered for a test) and test switches that make a
// kernel skip issuing its loads, so that a test can make a wait run out with nothing in flight.
// Kernels receive the address of `status`; the other fields follow it.
struct DeviceCtl {
    int status;
    unsigned int flags;
    unsigned long long wait_limit_ns;
};
constexpr unsigned int kInjectSkipPrepLoads = 1u;   // the chunked prep kernel issues no tile loads
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

GDN_DEV void report_status(int *status, int code) {
    if (status) atomicCAS(status, 0, code);
}
GDN_DEV unsigned long long ctl_wait_limit(const int *status) {
    return status ? reinterpret_cast<const volatile DeviceCtl *>(status)->wait_limit_ns : kWaitLimitNs;
}
GDN_DEV unsigned int ctl_flags(const int *status) {
    return status ? reinterpret_cast<const volatile DeviceCtl *>(status)->flags : 0u;
}

}  // namespace gdn

// ===================================================================================
// Asynchronous-proxy helpers: mbarriers with bounded waits, TMA tile loads, tcgen05.
// ===================================================================================
namespace gdn {

GDN_DEV uint32_t smem_u32(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

GDN_DEV uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

GDN_DEV void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
GDN_DEV void fence_barrier_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
GDN_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

GDN_DEV void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
GDN_DEV void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
GDN_DEV bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
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

// Wait for the phase with the given parity to complete, for at most the control block's wait
// limit (1 s by default) of device time. On expiry records GDN_ERR_TIMEOUT in the status word
// and returns false; callers then stop issuing work, drain what they issued and fall through
// to the kernel's teardown.
GDN_DEV bool mbar_wait(uint64_t *bar, uint32_t parity, int *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    const uint64_t limit = ctl_wait_limit(status);
    for (uint32_t i = 0;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && global_timer_ns() - t0 > limit) {
            report_status(status, GDN_ERR_TIMEOUT);
            return false;
        }
    }
}

// 2-D TMA tile load into shared memory, completing on `bar` (transaction bytes).
GDN_DEV void tma_load_2d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}
GDN_DEV void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- tensor memory ----
GDN_DEV void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
GDN_DEV void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
GDN_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
GDN_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
GDN_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive on `bar` once every tcgen05 operation this thread issued so far has completed.
GDN_DEV void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Shared-memory matrix descriptor (tcgen05): start address, leading / stride byte offsets,
// version 1, layout type (0 none, 2 = 128-byte swizzle, 4 = 64B, 6 = 32B).
GDN_DEV uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes, uint32_t layout) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)(layout & 7u) << 61;
    return d;
}

// 32 lanes x 32 consecutive 32-bit columns of tensor memory into registers (this warp's
// lane quarter), followed by the wait that makes the registers valid.
GDN_DEV void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
GDN_DEV void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
GDN_DEV void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}
// Two fp32 values in one 64-bit register pair (first value in the low half), for the packed
// f32x2 arithmetic of sm_100: one instruction issues both lanes' multiply / add / fma.
typedef unsigned long long f2_t;
GDN_DEV f2_t f2(float a, float b) {
    return (f2_t)__float_as_uint(a) | ((f2_t)__float_as_uint(b) << 32);
}
GDN_DEV float f2lo(f2_t v) { return __uint_as_float((uint32_t)v); }
GDN_DEV float f2hi(f2_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
GDN_DEV f2_t mul2(f2_t a, f2_t b) {
    f2_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
GDN_DEV f2_t add2(f2_t a, f2_t b) {
    f2_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
GDN_DEV f2_t fma2(f2_t a, f2_t b, f2_t c) {
    f2_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
GDN_DEV float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// Asynchronous global -> shared copies (LDGSTS): 16 bytes (both addresses 16-byte aligned) or 4
// bytes (4-byte aligned), completed by cp_async_wait<N> (at most N younger groups pending).
GDN_DEV void cp_async16(void *smem, const void *gmem) {
    const uint32_t sa = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem) : "memory");
}
GDN_DEV void cp_async4(void *smem, const void *gmem) {
    const uint32_t sa = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(sa), "l"(gmem) : "memory");
}
GDN_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
GDN_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// bf16 word pair -> fp32 pair (exact: a bf16 is the high half of its fp32)
GDN_DEV f2_t bf16x2_to_f2(uint32_t w) { return f2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)); }

// Gated RMSNorm of one head row, eight values per thread, LANES threads per row (the row's
// threads are consecutive lanes): y = o (w / rms(o)) z sigma(z), rms over the whole row,
// sigma(z) = 1 / (1 + 2^(-z log2 e)). "Red Lite dev15d - DeltaNet gated tail", Pinned graph
// semantics, steps 1-5. Shared by the standalone tail and the fused scan epilogue so that the
// two agree bit for bit.
// Sum of squares of eight values as the tail's threads form it: pairwise fp32x2 fma over the
// four pairs, then the two lanes added.
GDN_DEV float row_sumsq8(const f2_t (&o2)[4]) {
    f2_t sq = mul2(o2[0], o2[0]);
#pragma unroll
    for (int k = 1; k < 4; ++k) sq = fma2(o2[k], o2[k], sq);
    return f2lo(sq) + f2hi(sq);
}

// y = o (w inv_rms) z sigma(z) for eight values, sigma(z) = 1 / (1 + 2^(-z log2 e)).
GDN_DEV void gated_apply8(const f2_t (&o2)[4], const f2_t (&z2)[4], const f2_t (&w2)[4], float inv_rms, f2_t (&y2)[4]) {
    const f2_t ir2 = f2(inv_rms, inv_rms), nlog2e = f2(-kLog2e, -kLog2e), one2 = f2(1.0f, 1.0f);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const f2_t t = mul2(z2[k], nlog2e);
        const f2_t d = add2(f2(exp2_approx(f2lo(t)), exp2_approx(f2hi(t))), one2);
        const f2_t sl = mul2(z2[k], f2(rcp_approx(f2lo(d)), rcp_approx(f2hi(d))));
        y2[k] = mul2(mul2(o2[k], mul2(w2[k], ir2)), sl);
    }
}

// Gated RMSNorm of one head row, eight values per thread, LANES threads per row (the row's
// threads are consecutive lanes): y = o (w / rms(o)) z sigma(z), rms over the whole row.
// "Red Lite dev15d - DeltaNet gated tail", Pinned graph semantics, steps 1-5. Shared by the
// standalone tail and the fused kernels so that they agree bit for bit.
template <int LANES>
GDN_DEV void gated_row8(const f2_t (&o2)[4], const f2_t (&z2)[4], const f2_t (&w2)[4], float inv_d, float eps,
                        f2_t (&y2)[4]) {
    const float ss = group_sum<LANES>(row_sumsq8(o2));
    gated_apply8(o2, z2, w2, rsqrtf(__fmaf_rn(ss, inv_d, eps)), y2);
}

// NVFP4 encode of eight values of y (half of a 16-value block; the partner lane, lane ^ 1,
// holds the other half): y rounded to bf16 first (the tensor the two-call path hands to the
// encoder), block scale sb = E4M3((amax / 6) gs), codes E2M1(y r) with r = gs / sb (from r_tab
// when given, else by division).
GDN_DEV void nvfp4_encode_row8(f2_t (&y2)[4], float gs, const float *r_tab, uint32_t &packed, uint32_t &sb) {
    float amax = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const __nv_bfloat162 hb = __floats2bfloat162_rn(f2lo(y2[k]), f2hi(y2[k]));
        y2[k] = bf16x2_to_f2(*reinterpret_cast<const uint32_t *>(&hb));
        amax = fmaxf(amax, fmaxf(fabsf(f2lo(y2[k])), fabsf(f2hi(y2[k]))));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    sb = cvt_e4m3(__fmul_rn(div6_rn(amax), gs));
    // r = gs / E4M3(sb) (0 for sb = 0), from the table when one is given
    const float r = r_tab ? r_tab[sb & 127u] : ((sb & 127u) == 0 ? 0.0f : __fdiv_rn(gs, e4m3_to_f32(sb & 127u)));
    const f2_t r2 = f2(r, r);
    float p[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const f2_t q = mul2(y2[k], r2);
        p[2 * k] = f2lo(q);
        p[2 * k + 1] = f2hi(q);
    }
    packed = cvt_e2m1x8(p);
}

// The factor table of nvfp4_encode_row8 for encode scale gs: r_tab[c] = gs / E4M3(c), r_tab[0] = 0
// (thread t < 128 of the block fills entry t; the caller synchronises).
GDN_DEV void nvfp4_fill_r_tab(float *r_tab, float gs, int t) {
    if (t < 128) r_tab[t] = t == 0 ? 0.0f : __fdiv_rn(gs, e4m3_to_f32((uint32_t)t));
}

// Programmatic dependent launch. Every kernel of this library is launched with programmatic
// stream serialization (launch_pdl): it may start while the previous kernel in the stream is
// still running, so it calls pdl_wait() before its first global-memory access (which returns
// once that kernel has finished and its writes are visible), and pdl_launch_dependents() at
// entry so that the next kernel's CTAs can be placed on SMs this grid no longer needs.
GDN_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
GDN_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

GDN_DEV void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Registers into 32 lanes x N consecutive 32-bit columns of tensor memory (this warp's
// lane quarter); tmem_st_wait() makes the stores visible to later tcgen05 operations.
GDN_DEV void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
GDN_DEV void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}
GDN_DEV void tmem_st4(uint32_t taddr, const uint32_t (&r)[4]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
                 "r"(r[2]), "r"(r[3])
                 : "memory");
}
GDN_DEV void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

}  // namespace gdn
