// Token-by-token gated delta rule on CUDA cores: the decode step (one token per sequence,
// state read once and written once, in place) and the recurrent prefill used for head
// sizes the tensor-core chunked kernel does not take.
//
// "Why Gated DeltaNet Survives 4-Bit Quantization" (abstract, mechanisms ii-iii): per
// token, with unit key k and query q,
//     alpha = exp(-exp(A_log) softplus(a + dt_bias)),  beta = sigmoid(b),
//     S <- alpha S (I - beta k k^T) + beta v k^T = alpha S + beta (v - alpha S k) k^T,
//     o = S q.
// The rows of S (value index i) evolve independently, so a CTA owns rows of one (sequence,
// value head) state and keeps them in registers across the sequence; each row is spread over
// a group of lanes, and the two row dot products (S k and S q) are lane-group shuffle
// reductions. Head size 128 has its own layout (below); smaller heads spread a row over D/4
// lanes holding 4 key columns each.
#include "common.cuh"
#include "kernels.h"

namespace gdn {

template <int D>
struct RecurrentShape {
    static constexpr int NT = (D * D / 4) < 128 ? (D * D / 4) : 128;  // threads per CTA
    static constexpr int LANES = D / 4;                                // lanes per row
    static constexpr int RPB = NT / LANES;                             // rows per pass
    static constexpr int R = D >= 128 ? 32 : (D >= 32 ? 16 : D);       // rows per CTA
    static constexpr int PASSES = R / RPB;
    static constexpr int SLICES = D / R;
    static_assert(R % RPB == 0 && PASSES >= 1, "row tiling");
};

GDN_DEV float dot4(const float (&x)[4], const float (&y)[4]) {
    return x[0] * y[0] + x[1] * y[1] + x[2] * y[2] + x[3] * y[3];
}

template <int D, bool IN_BF16, bool OUT_BF16>
__global__ void __launch_bounds__(RecurrentShape<D>::NT)
gdn_recurrent_kernel(const void *__restrict__ q, const void *__restrict__ k,
                     const void *__restrict__ v, const float *__restrict__ a,
                     const float *__restrict__ b, const float *__restrict__ A_log,
                     const float *__restrict__ dt_bias, const int32_t *__restrict__ cu_seqlens,
                     int32_t tokens_per_seq, int32_t Hk, int32_t Hv, float scale, int32_t l2norm,
                     const float *S0, float *S_out, void *__restrict__ o, const int32_t *__restrict__ n_apply) {
    pdl_launch_dependents();
    pdl_wait();
    using Sh = RecurrentShape<D>;
    constexpr int LANES = Sh::LANES, RPB = Sh::RPB, PASSES = Sh::PASSES, R = Sh::R;
    const int slice = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
    const int hk = h / (Hv / Hk);
    const int tid = threadIdx.x;
    const int col = (tid % LANES) * 4;
    const int row0 = slice * R + tid / LANES;

    int t0, t1;
    if (cu_seqlens) {
        t0 = cu_seqlens[n];
        t1 = cu_seqlens[n + 1];
    } else {
        t0 = n * tokens_per_seq;
        t1 = t0 + tokens_per_seq;
    }
    if (n_apply) t1 = t0 + min(max(n_apply[n], 0), t1 - t0);   // only the first n_apply[n] tokens
    const size_t sbase = ((size_t)n * Hv + h) * D * D;

    float s[PASSES][4];
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const size_t off = sbase + (size_t)(row0 + p * RPB) * D + col;
        if (S0) {
            float4 x = __ldcs(reinterpret_cast<const float4 *>(S0 + off));
            s[p][0] = x.x; s[p][1] = x.y; s[p][2] = x.z; s[p][3] = x.w;
        } else {
            s[p][0] = s[p][1] = s[p][2] = s[p][3] = 0.0f;
        }
    }

    const float Al = A_log[h], db = dt_bias[h];
    for (int t = t0; t < t1; ++t) {
        float kk[4], qq[4], vv[PASSES];
        load4<IN_BF16>(k, ((size_t)t * Hk + hk) * D + col, kk);
        load4<IN_BF16>(q, ((size_t)t * Hk + hk) * D + col, qq);
#pragma unroll
        for (int p = 0; p < PASSES; ++p) vv[p] = load1<IN_BF16>(v, ((size_t)t * Hv + h) * D + row0 + p * RPB);
        float g, beta;
        gdn_gates(a[(size_t)t * Hv + h], b[(size_t)t * Hv + h], Al, db, g, beta);
        const float alpha = expf(g);

        float kn = 1.0f, qn = scale;
        if (l2norm) {
            float ks = group_sum<LANES>(dot4(kk, kk));
            float qs = group_sum<LANES>(dot4(qq, qq));
            kn = rsqrtf(ks + 1e-6f);
            qn = rsqrtf(qs + 1e-6f) * scale;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) { kk[c] *= kn; qq[c] *= qn; }

        float sk[PASSES];
#pragma unroll
        for (int p = 0; p < PASSES; ++p) sk[p] = dot4(s[p], kk);
#pragma unroll
        for (int p = 0; p < PASSES; ++p) sk[p] = group_sum<LANES>(sk[p]);
#pragma unroll
        for (int p = 0; p < PASSES; ++p) {
            const float u = beta * (vv[p] - alpha * sk[p]);
#pragma unroll
            for (int c = 0; c < 4; ++c) s[p][c] = alpha * s[p][c] + u * kk[c];
        }
        float op[PASSES];
#pragma unroll
        for (int p = 0; p < PASSES; ++p) op[p] = dot4(s[p], qq);
#pragma unroll
        for (int p = 0; p < PASSES; ++p) op[p] = group_sum<LANES>(op[p]);
        if (o && (tid % LANES) == 0) {
#pragma unroll
            for (int p = 0; p < PASSES; ++p) store1<OUT_BF16>(o, ((size_t)t * Hv + h) * D + row0 + p * RPB, op[p]);
        }
    }

    if (S_out) {
#pragma unroll
        for (int p = 0; p < PASSES; ++p) {
            const size_t off = sbase + (size_t)(row0 + p * RPB) * D + col;
            __stcs(reinterpret_cast<float4 *>(S_out + off), make_float4(s[p][0], s[p][1], s[p][2], s[p][3]));
        }
    }
}

// ---------------------------------------------------------------- d = 128 ----
// A CTA of 128 threads owns 64 rows of one (sequence, value head) state: the 8 consecutive
// lanes of a row group share 4 rows (slice*64 + tid/8 + 16 p, p < 4), and lane c of the group
// holds key columns 32 j + 4 c + e (j, e < 4), so each of its four 16-byte state accesses per
// row is part of one 128-byte run per row group. The arithmetic runs on packed f32 pairs; the
// key norm is folded into the update's scalar (S k^ = kn (S k), and the rank-one write uses
// u kn with the raw k); the gates of 32 tokens are computed once per warp, one per lane, and
// broadcast per token.
constexpr int kR128Threads = 128;
constexpr unsigned kFull = 0xffffffffu;

// Four per-thread values summed over the 8 lanes of a row group: after the exchange, lanes whose
// bits 2 and 1 are (p >> 1, p & 1) hold the total of value p (4 shuffles instead of 12).
GDN_DEV float group8_sum4_t(const float (&x)[4], int l8) {
    const bool b2 = (l8 & 4) != 0, b1 = (l8 & 2) != 0;
    const float r0 = __shfl_xor_sync(kFull, b2 ? x[0] : x[2], 4);
    const float r1 = __shfl_xor_sync(kFull, b2 ? x[1] : x[3], 4);
    const float k0 = (b2 ? x[2] : x[0]) + r0, k1 = (b2 ? x[3] : x[1]) + r1;
    float v = (b1 ? k1 : k0) + __shfl_xor_sync(kFull, b1 ? k0 : k1, 2);
    v += __shfl_xor_sync(kFull, v, 1);
    return v;
}

// The 16 key-index values of lane c (columns 32 j + 4 c + e) of one 128-vector, as 8 pairs.
template <bool BF16>
GDN_DEV void load_cols16(const void *base, size_t row, int l8, f2_t (&x)[8]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const size_t idx = row + 32 * j + 4 * l8;
        if constexpr (BF16) {
            const uint2 u = *reinterpret_cast<const uint2 *>(reinterpret_cast<const __nv_bfloat16 *>(base) + idx);
            x[2 * j] = bf16x2_to_f2(u.x);
            x[2 * j + 1] = bf16x2_to_f2(u.y);
        } else {
            const float4 f = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(base) + idx);
            x[2 * j] = f2(f.x, f.y);
            x[2 * j + 1] = f2(f.z, f.w);
        }
    }
}

GDN_DEV float dot16(const f2_t (&a)[8], const f2_t (&b)[8]) {
    f2_t acc = mul2(a[0], b[0]);
#pragma unroll
    for (int c = 1; c < 8; ++c) acc = fma2(a[c], b[c], acc);
    return f2lo(acc) + f2hi(acc);
}

template <bool IN_BF16, bool OUT_BF16>
__global__ void __launch_bounds__(kR128Threads)
gdn_recurrent128_kernel(const void *__restrict__ q, const void *__restrict__ k, const void *__restrict__ v,
                        const float *__restrict__ a, const float *__restrict__ b, const float *__restrict__ A_log,
                        const float *__restrict__ dt_bias, const int32_t *__restrict__ cu_seqlens,
                        int32_t tokens_per_seq, int32_t Hk, int32_t Hv, float scale, int32_t l2norm,
                        const float *S0, float *S_out, void *__restrict__ o, const int32_t *__restrict__ n_apply) {
    pdl_launch_dependents();
    pdl_wait();
    constexpr int D = 128;
    const int slice = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
    const int hk = h / (Hv / Hk);
    const int tid = threadIdx.x, lane = tid & 31, l8 = tid & 7;
    const int rbase = slice * 64 + (tid >> 3);
    const int gbase = lane & ~7;

    int t0, t1;
    if (cu_seqlens) {
        t0 = cu_seqlens[n];
        t1 = cu_seqlens[n + 1];
    } else {
        t0 = n * tokens_per_seq;
        t1 = t0 + tokens_per_seq;
    }
    if (n_apply) t1 = t0 + min(max(n_apply[n], 0), t1 - t0);   // only the first n_apply[n] tokens
    const size_t sbase = ((size_t)n * Hv + h) * D * D;

    f2_t s[4][8];
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float4 x = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (S0) x = __ldcs(reinterpret_cast<const float4 *>(S0 + sbase + (size_t)(rbase + 16 * p) * D + 32 * j + 4 * l8));
            s[p][2 * j] = f2(x.x, x.y);
            s[p][2 * j + 1] = f2(x.z, x.w);
        }

    const float Al = A_log[h], db = dt_bias[h];
    float g_alpha = 0.0f, g_beta = 0.0f;   // gates of token (t - t0) / 32 * 32 + lane
    for (int t = t0; t < t1; ++t) {
        const int i = (t - t0) & 31;
        if (i == 0) {
            const int tt = t + lane;
            if (tt < t1) {
                float g;
                gdn_gates(a[(size_t)tt * Hv + h], b[(size_t)tt * Hv + h], Al, db, g, g_beta);
                g_alpha = expf(g);
            }
        }
        const float alpha = __shfl_sync(kFull, g_alpha, i), beta = __shfl_sync(kFull, g_beta, i);
        f2_t k2[8], q2[8];
        load_cols16<IN_BF16>(k, ((size_t)t * Hk + hk) * D, l8, k2);
        load_cols16<IN_BF16>(q, ((size_t)t * Hk + hk) * D, l8, q2);
        float vv[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) vv[p] = load1<IN_BF16>(v, ((size_t)t * Hv + h) * D + rbase + 16 * p);

        float kn = 1.0f, qn = scale;
        if (l2norm) {
            const float ks = group_sum<8>(dot16(k2, k2)), qs = group_sum<8>(dot16(q2, q2));
            kn = rsqrtf(ks + 1e-6f);
            qn = rsqrtf(qs + 1e-6f) * scale;
        }
        float part[4], sk[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) part[p] = dot16(s[p], k2);
        const float skt = group8_sum4_t(part, l8);
#pragma unroll
        for (int p = 0; p < 4; ++p) sk[p] = __shfl_sync(kFull, skt, gbase + 4 * (p >> 1) + 2 * (p & 1));
        // S <- alpha S + beta (v - alpha S k^) k^T, k^ = kn k
        const f2_t a2 = f2(alpha, alpha);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float u = beta * (vv[p] - alpha * kn * sk[p]) * kn;
            const f2_t u2 = f2(u, u);
#pragma unroll
            for (int c = 0; c < 8; ++c) s[p][c] = fma2(a2, s[p][c], mul2(u2, k2[c]));
        }
        // o = S q^, q^ = qn q (qn includes scale)
#pragma unroll
        for (int p = 0; p < 4; ++p) part[p] = dot16(s[p], q2);
        const float ot = group8_sum4_t(part, l8);
        if (o && (l8 & 1) == 0) {
            const int p = 2 * ((l8 >> 2) & 1) + ((l8 >> 1) & 1);
            store1<OUT_BF16>(o, ((size_t)t * Hv + h) * D + rbase + 16 * p, ot * qn);
        }
    }

    if (S_out) {
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                __stcs(reinterpret_cast<float4 *>(S_out + sbase + (size_t)(rbase + 16 * p) * D + 32 * j + 4 * l8),
                       make_float4(f2lo(s[p][2 * j]), f2hi(s[p][2 * j]), f2lo(s[p][2 * j + 1]), f2hi(s[p][2 * j + 1])));
    }
}

// Draft verify in the chunk (WY) form: outputs for the T <= 8 draft tokens of each sequence from
// the state S0, which is only read. With unit keys k^_t, queries q^_t (scale included), decay
// gamma_t = alpha_1 ... alpha_t and c_st = gamma_t / gamma_s (a product of alphas), the token-by-token
// rule S_t = alpha_t S_{t-1} + u_t k^_t^T, u_t = beta_t (v_t - alpha_t S_{t-1} k^_t), unrolls to
//     S_{t-1} k^_t = gamma_{t-1} S0 k^_t + sum_{s<t} c_{s,t-1} u_s (k^_s . k^_t),
//     o_t = S_t q^_t = gamma_t S0 q^_t + sum_{s<=t} c_{s,t} u_s (k^_s . q^_t),
// so each state row needs only the 2 T products S0 k_t and S0 q_t (independent of one another,
// no state update) and T x T scalars shared by the CTA (the Gram dots of the tokens' keys and
// queries), instead of T dependent rank-one updates.
//
// The 2 T products are one small matrix product per CTA, [S0 rows] x [k_1..k_T | q_1..q_T], on
// warp-level bf16 MMAs (m16n8k16, fp32 accumulation): each warp owns 16 state rows, the keys and
// the queries are one 8-column tile each. S0 enters as bf16 hi + lo (hi = S0 rounded, lo = the
// rounded remainder: the product misses S0 - hi - lo, at most 2^-17 of |S0| per element); bf16
// keys and queries are exact in bf16, fp32 ones are split the same way and add the hi x lo term.
// Within each 16-wide k-step a thread holds state columns 4c .. 4c + 3 (c = lane % 4) in the
// places the MMA layout gives to columns 2c, 2c + 1, 2c + 8, 2c + 9; the key / query tiles use the
// same column order, so the sums are those of the plain products.
constexpr int kVerifyMaxT = 8;
constexpr int kVerifyPairPitch = 72;   // bf16 pairs per staged row: 64 + 8, so B-fragment loads are conflict-free

// D += A B on one m16n8k16 tile (bf16 inputs, fp32 accumulation)
GDN_DEV void mma_bf16_m16n8k16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// (x, y) as a bf16 pair (x in the low half) and the pair of their rounded remainders
GDN_DEV void split_bf16x2(float x, float y, uint32_t &hi, uint32_t &lo) {
    __nv_bfloat162 p = __floats2bfloat162_rn(x, y);
    hi = *reinterpret_cast<const uint32_t *>(&p);
    const f2_t w = bf16x2_to_f2(hi);
    p = __floats2bfloat162_rn(x - f2lo(w), y - f2hi(w));
    lo = *reinterpret_cast<const uint32_t *>(&p);
}

template <bool IN_BF16, bool OUT_BF16>
__global__ void __launch_bounds__(kR128Threads, 5)
gdn_verify128_kernel(const void *__restrict__ q, const void *__restrict__ k, const void *__restrict__ v,
                     const float *__restrict__ a, const float *__restrict__ b, const float *__restrict__ A_log,
                     const float *__restrict__ dt_bias, int32_t T, int32_t Hk, int32_t Hv, float scale,
                     int32_t l2norm, const float *__restrict__ S0, void *__restrict__ o) {
    pdl_launch_dependents();
    pdl_wait();
    constexpr int D = 128;
    const int slice = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
    const int hk = h / (Hv / Hk);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, tig = lane & 3;         // MMA fragment row group, thread in group
    const int r0 = slice * 64 + warp * 16 + gq;       // this thread's state rows r0 and r0 + 8
    const int t0 = n * T;
    const size_t sbase = ((size_t)n * Hv + h) * D * D;
    __shared__ float s_kk[kVerifyMaxT][kVerifyMaxT], s_kq[kVerifyMaxT][kVerifyMaxT];
    __shared__ float s_qq[kVerifyMaxT], s_alpha[kVerifyMaxT], s_beta[kVerifyMaxT];
    // the tokens' raw key (0) and query (1) rows as bf16 pairs (and for fp32 inputs the pairs of
    // their rounded remainders), the MMAs' operands; rows of unused tokens are zero
    __shared__ __align__(16) uint32_t kq_hi[2][kVerifyMaxT][kVerifyPairPitch];
    __shared__ __align__(16) uint32_t kq_lo[2][kVerifyMaxT][IN_BF16 ? 2 : kVerifyPairPitch];

    // the gate inputs of token `lane` (warp 2), fetched before the state
    float ga_raw = 0.0f, gb_raw = 0.0f;
    if (warp == 2 && lane < T) {
        ga_raw = a[(size_t)(t0 + lane) * Hv + h];
        gb_raw = b[(size_t)(t0 + lane) * Hv + h];
    }
    // stage the keys and queries: 2 x 8 rows of 16 pieces of 8 values, two pieces a thread. bf16
    // rows are their own hi pairs: they are copied in asynchronously, ahead of the state loads.
    if constexpr (IN_BF16) {
#pragma unroll
        for (int e = tid; e < 2 * kVerifyMaxT * (D / 8); e += kR128Threads) {
            const int which = e / (kVerifyMaxT * (D / 8)), rem = e % (kVerifyMaxT * (D / 8));
            const int t = rem / (D / 8), c8 = (rem % (D / 8)) * 8;
            uint32_t *dst = &kq_hi[which][t][c8 / 2];
            if (t < T)
                cp_async16(dst, reinterpret_cast<const __nv_bfloat16 *>(which ? q : k) + ((size_t)(t0 + t) * Hk + hk) * D + c8);
            else
                *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
        cp_async_commit();
    }
    // state rows r0 and r0 + 8, columns 16 ks + 4 tig .. + 3 of each k-step ks (read once)
    float4 sa[8], sb[8];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        sa[ks] = __ldcs(reinterpret_cast<const float4 *>(S0 + sbase + (size_t)r0 * D + 16 * ks + 4 * tig));
        sb[ks] = __ldcs(reinterpret_cast<const float4 *>(S0 + sbase + (size_t)(r0 + 8) * D + 16 * ks + 4 * tig));
    }
    if constexpr (IN_BF16) {
        cp_async_wait<0>();
    } else {
#pragma unroll
        for (int e = tid; e < 2 * kVerifyMaxT * (D / 8); e += kR128Threads) {
            const int which = e / (kVerifyMaxT * (D / 8)), rem = e % (kVerifyMaxT * (D / 8));
            const int t = rem / (D / 8), c8 = (rem % (D / 8)) * 8;
            float x[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
            if (t < T) load8<false>(which ? q : k, ((size_t)(t0 + t) * Hk + hk) * D + c8, x);
            uint4 hi, lo;
            split_bf16x2(x[0], x[1], hi.x, lo.x);
            split_bf16x2(x[2], x[3], hi.y, lo.y);
            split_bf16x2(x[4], x[5], hi.z, lo.z);
            split_bf16x2(x[6], x[7], hi.w, lo.w);
            *reinterpret_cast<uint4 *>(&kq_hi[which][t][c8 / 2]) = hi;
            *reinterpret_cast<uint4 *>(&kq_lo[which][t][c8 / 2]) = lo;
        }
    }
    __syncthreads();

    // Gram dots of the tokens' raw keys and queries, X X^T with X = [k_1 .. k_8; q_1 .. q_8] (rows
    // of unused tokens zero): warp 0 multiplies X by its key tile (n = k_1 .. k_8: k.k and q.k),
    // warp 1 by its query tile (n = q_1 .. q_8: q.q). The A fragments of X are, pair for pair, the
    // B fragments of both tiles. Two accumulators (even and odd k-steps) halve the dependent chain.
    if (warp < 2) {
        float acc[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const int pc = 8 * ks + 2 * tig;
            const uint2 xk = *reinterpret_cast<const uint2 *>(&kq_hi[0][gq][pc]);
            const uint2 xq = *reinterpret_cast<const uint2 *>(&kq_hi[1][gq][pc]);
            const uint2 xn = warp == 0 ? xk : xq;
            const uint32_t ax[4] = {xk.x, xq.x, xk.y, xq.y};
            mma_bf16_m16n8k16(acc[ks & 1], ax, xn.x, xn.y);
            if constexpr (!IN_BF16) {
                const uint2 lk = *reinterpret_cast<const uint2 *>(&kq_lo[0][gq][pc]);
                const uint2 lq = *reinterpret_cast<const uint2 *>(&kq_lo[1][gq][pc]);
                const uint2 ln = warp == 0 ? lk : lq;
                const uint32_t al[4] = {lk.x, lq.x, lk.y, lq.y};
                mma_bf16_m16n8k16(acc[ks & 1], ax, ln.x, ln.y);
                mma_bf16_m16n8k16(acc[ks & 1], al, xn.x, xn.y);
            }
        }
        // rows gq (k_gq) in [0], [1] and gq + 8 (q_gq) in [2], [3]; columns n = 2 tig, 2 tig + 1
        const int n0 = 2 * tig;
        const float g0 = acc[0][0] + acc[1][0], g1 = acc[0][1] + acc[1][1];
        const float g2 = acc[0][2] + acc[1][2], g3 = acc[0][3] + acc[1][3];
        if (warp == 0) {
            s_kk[gq][n0] = g0;
            s_kk[gq][n0 + 1] = g1;
            s_kq[n0][gq] = g2;
            s_kq[n0 + 1][gq] = g3;
        } else {
            if (n0 == gq) s_qq[gq] = g2;
            if (n0 + 1 == gq) s_qq[gq] = g3;
        }
    } else if (warp == 2 && lane < T) {
        float g, beta;
        gdn_gates(ga_raw, gb_raw, A_log[h], dt_bias[h], g, beta);
        s_alpha[lane] = expf(g);
        s_beta[lane] = beta;
    }

    // the row this lane finishes (below: lanes 0, 1 of a group row r0, lanes 2, 3 row r0 + 8) and
    // its v values, loaded ahead of the dependent recurrence
    const int rsel = tig >> 1;
    const int row = r0 + 8 * rsel;
    float vrow[kVerifyMaxT];
#pragma unroll
    for (int t = 0; t < kVerifyMaxT; ++t)
        vrow[t] = t < T ? load1<IN_BF16>(v, ((size_t)(t0 + t) * Hv + h) * D + row) : 0.0f;

    // [S0 k_1 .. S0 k_8] and [S0 q_1 .. S0 q_8] for the warp's 16 rows: the D fragments hold
    // (row r0, tokens 2 tig, 2 tig + 1) in [0], [1] and (row r0 + 8, the same tokens) in [2], [3]
    float dk[4] = {0.0f, 0.0f, 0.0f, 0.0f}, dq[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        uint32_t ahi[4], alo[4];
        split_bf16x2(sa[ks].x, sa[ks].y, ahi[0], alo[0]);
        split_bf16x2(sb[ks].x, sb[ks].y, ahi[1], alo[1]);
        split_bf16x2(sa[ks].z, sa[ks].w, ahi[2], alo[2]);
        split_bf16x2(sb[ks].z, sb[ks].w, ahi[3], alo[3]);
        const int pc = 8 * ks + 2 * tig;
        const uint2 bk = *reinterpret_cast<const uint2 *>(&kq_hi[0][gq][pc]);
        const uint2 bq = *reinterpret_cast<const uint2 *>(&kq_hi[1][gq][pc]);
        mma_bf16_m16n8k16(dk, ahi, bk.x, bk.y);
        mma_bf16_m16n8k16(dk, alo, bk.x, bk.y);
        mma_bf16_m16n8k16(dq, ahi, bq.x, bq.y);
        mma_bf16_m16n8k16(dq, alo, bq.x, bq.y);
        if constexpr (!IN_BF16) {
            const uint2 lk = *reinterpret_cast<const uint2 *>(&kq_lo[0][gq][pc]);
            const uint2 lq = *reinterpret_cast<const uint2 *>(&kq_lo[1][gq][pc]);
            mma_bf16_m16n8k16(dk, ahi, lk.x, lk.y);
            mma_bf16_m16n8k16(dq, ahi, lq.x, lq.y);
        }
    }
    // this lane's row: token t's products sit in lane (group, t / 2), element t % 2 (+ 2 for r0 + 8)
    float xk[kVerifyMaxT], xq[kVerifyMaxT];
#pragma unroll
    for (int t = 0; t < kVerifyMaxT; ++t) {
        xk[t] = 0.0f;
        xq[t] = 0.0f;
        if (t < T) {
            const int src = (lane & ~3) | (t >> 1);
            const float k0 = __shfl_sync(kFull, dk[t & 1], src), k1 = __shfl_sync(kFull, dk[2 + (t & 1)], src);
            const float q0 = __shfl_sync(kFull, dq[t & 1], src), q1 = __shfl_sync(kFull, dq[2 + (t & 1)], src);
            xk[t] = rsel ? k1 : k0;
            xq[t] = rsel ? q1 : q0;
        }
    }
    __syncthreads();

    // per row: the T x T recurrence on the projections (lanes with tig even own one row each)
    float kn[kVerifyMaxT], u[kVerifyMaxT], c[kVerifyMaxT];
#pragma unroll
    for (int t = 0; t < kVerifyMaxT; ++t) {
        if (t >= T) break;
        kn[t] = l2norm ? rsqrtf(s_kk[t][t] + 1e-6f) : 1.0f;
        const float qn = l2norm ? rsqrtf(s_qq[t] + 1e-6f) * scale : scale;
        const float alpha = s_alpha[t], beta = s_beta[t];
        // c[s] = gamma_{t-1} / gamma_s before the update; gamma_{t-1} itself is c_{-1}
        float proj = 0.0f, gam_prev = 1.0f;
#pragma unroll
        for (int r = 0; r < kVerifyMaxT; ++r)
            if (r < t) proj += c[r] * u[r] * (kn[r] * kn[t] * s_kk[r][t]);
#pragma unroll
        for (int r = 0; r < kVerifyMaxT; ++r)
            if (r < t) gam_prev *= s_alpha[r];
        proj += gam_prev * kn[t] * xk[t];
        u[t] = beta * (vrow[t] - alpha * proj);
#pragma unroll
        for (int r = 0; r < kVerifyMaxT; ++r)
            if (r < t) c[r] *= alpha;
        c[t] = 1.0f;
        const float gam = gam_prev * alpha;
        float ot = gam * qn * xq[t];
#pragma unroll
        for (int r = 0; r < kVerifyMaxT; ++r)
            if (r <= t) ot += c[r] * u[r] * (kn[r] * qn * s_kq[r][t]);
        if ((tig & 1) == 0) store1<OUT_BF16>(o, ((size_t)(t0 + t) * Hv + h) * D + row, ot);
    }
}

// Decode step fused with the gated tail: one CTA of 256 threads per (sequence, value head) owns
// all 128 rows of the state (the two 64-row halves of gdn_recurrent128_kernel, same thread layout
// and arithmetic), so the head's o is complete inside the CTA. It is rounded to bf16 (the tensor
// the two-call path hands to the tail), and one warp applies the gated RMSNorm and the NVFP4
// encode with the tail kernel's row functions, so the codes and scales equal the two-call path's
// bit for bit. "Red Lite dev15d - DeltaNet gated tail", Pinned graph semantics, steps 1-5.
constexpr int kFusedDecThreads = 256;

__global__ void __launch_bounds__(kFusedDecThreads, 2)
gdn_decode128_gated_nvfp4_kernel(const void *__restrict__ q, const void *__restrict__ k, const void *__restrict__ v,
                                 const float *__restrict__ a, const float *__restrict__ b,
                                 const float *__restrict__ A_log, const float *__restrict__ dt_bias, int32_t Hk,
                                 int32_t Hv, float scale, int32_t l2norm, float *state, const void *__restrict__ z,
                                 const float *__restrict__ norm_w, float eps, float gs, uint8_t *__restrict__ xq,
                                 uint8_t *__restrict__ xs, void *__restrict__ o) {
    pdl_launch_dependents();
    pdl_wait();
    constexpr int D = 128;
    const int h = blockIdx.x, n = blockIdx.y;          // sequence n decodes token n
    const int hk = h / (Hv / Hk);
    const int tid = threadIdx.x, lane = tid & 31, l8 = tid & 7;
    const int rbase = (tid >> 7) * 64 + ((tid & 127) >> 3);
    const int gbase = lane & ~7;
    __shared__ __align__(16) __nv_bfloat16 o_s[D];
    // the tail's z row and norm weights, copied in asynchronously with the state loads so that
    // neither their DRAM / L2 latency nor registers are spent after the update
    __shared__ __align__(16) __nv_bfloat16 z_s[D];
    __shared__ __align__(16) float w_s[D];
    if (tid < D) cp_async4(w_s + tid, norm_w + tid);
    else if (tid < D + D / 8)
        cp_async16(z_s + (tid - D) * 8, reinterpret_cast<const __nv_bfloat16 *>(z) + ((size_t)n * Hv + h) * D + (tid - D) * 8);
    cp_async_commit();
    const size_t sbase = ((size_t)n * Hv + h) * D * D;

    f2_t s[4][8];
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 x = __ldcs(reinterpret_cast<const float4 *>(state + sbase + (size_t)(rbase + 16 * p) * D + 32 * j + 4 * l8));
            s[p][2 * j] = f2(x.x, x.y);
            s[p][2 * j + 1] = f2(x.z, x.w);
        }
    const int lr = lane & 15, col = lr * 8;
    float g_alpha = 0.0f, g_beta = 0.0f;
    if (lane == 0) {
        float g;
        gdn_gates(a[(size_t)n * Hv + h], b[(size_t)n * Hv + h], A_log[h], dt_bias[h], g, g_beta);
        g_alpha = expf(g);
    }
    const float alpha = __shfl_sync(kFull, g_alpha, 0), beta = __shfl_sync(kFull, g_beta, 0);
    f2_t k2[8], q2[8];
    load_cols16<true>(k, ((size_t)n * Hk + hk) * D, l8, k2);
    load_cols16<true>(q, ((size_t)n * Hk + hk) * D, l8, q2);
    float vv[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) vv[p] = load1<true>(v, ((size_t)n * Hv + h) * D + rbase + 16 * p);

    float kn = 1.0f, qn = scale;
    if (l2norm) {
        const float ks = group_sum<8>(dot16(k2, k2)), qs = group_sum<8>(dot16(q2, q2));
        kn = rsqrtf(ks + 1e-6f);
        qn = rsqrtf(qs + 1e-6f) * scale;
    }
    float part[4], sk[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) part[p] = dot16(s[p], k2);
    const float skt = group8_sum4_t(part, l8);
#pragma unroll
    for (int p = 0; p < 4; ++p) sk[p] = __shfl_sync(kFull, skt, gbase + 4 * (p >> 1) + 2 * (p & 1));
    const f2_t a2 = f2(alpha, alpha);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float u = beta * (vv[p] - alpha * kn * sk[p]) * kn;
        const f2_t u2 = f2(u, u);
#pragma unroll
        for (int c = 0; c < 8; ++c) s[p][c] = fma2(a2, s[p][c], mul2(u2, k2[c]));
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) part[p] = dot16(s[p], q2);
    const float ot = group8_sum4_t(part, l8);
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            __stcs(reinterpret_cast<float4 *>(state + sbase + (size_t)(rbase + 16 * p) * D + 32 * j + 4 * l8),
                   make_float4(f2lo(s[p][2 * j]), f2hi(s[p][2 * j]), f2lo(s[p][2 * j + 1]), f2hi(s[p][2 * j + 1])));
    if ((l8 & 1) == 0) {
        const int p = 2 * ((l8 >> 2) & 1) + ((l8 >> 1) & 1);
        const __nv_bfloat16 ob = __float2bfloat16_rn(ot * qn);
        o_s[rbase + 16 * p] = ob;
        if (o) reinterpret_cast<__nv_bfloat16 *>(o)[((size_t)n * Hv + h) * D + rbase + 16 * p] = ob;
    }
    cp_async_wait<0>();
    __syncthreads();
    if (tid < 32) {
        // the head row: 16 lanes x 8 values (lanes 16-31 repeat them, their results unused)
        const uint4 ou = *reinterpret_cast<const uint4 *>(o_s + col);
        const uint4 zu = *reinterpret_cast<const uint4 *>(z_s + col);
        const f2_t o2[4] = {bf16x2_to_f2(ou.x), bf16x2_to_f2(ou.y), bf16x2_to_f2(ou.z), bf16x2_to_f2(ou.w)};
        const f2_t z2[4] = {bf16x2_to_f2(zu.x), bf16x2_to_f2(zu.y), bf16x2_to_f2(zu.z), bf16x2_to_f2(zu.w)};
        const float4 wa = *reinterpret_cast<const float4 *>(w_s + col), wb = *reinterpret_cast<const float4 *>(w_s + col + 4);
        const f2_t w2[4] = {f2(wa.x, wa.y), f2(wa.z, wa.w), f2(wb.x, wb.y), f2(wb.z, wb.w)};
        f2_t y2[4];
        gated_row8<16>(o2, z2, w2, 1.0f / (float)D, eps, y2);
        uint32_t packed, sb;
        nvfp4_encode_row8(y2, gs, nullptr, packed, sb);
        if (lane < 16) {
            const size_t base = ((size_t)n * Hv + h) * D + col;
            reinterpret_cast<uint32_t *>(xq)[base / 8] = packed;
            if ((lr & 1) == 0) xs[base / 16] = (uint8_t)sb;
        }
    }
}

cudaError_t launch_decode_gated_nvfp4(const DecodeTailArgs &d, cudaStream_t st) {
    if (d.B == 0 || d.Hv == 0) return cudaSuccess;
    return launch_pdl(gdn_decode128_gated_nvfp4_kernel, dim3(d.Hv, d.B), dim3(kFusedDecThreads), 0, st, d.q, d.k, d.v,
                      d.a, d.b, d.A_log, d.dt_bias, d.Hk, d.Hv, d.scale, d.l2norm, d.state, d.z, d.norm_w, d.eps,
                      d.gs, d.xq, d.xs, d.o);
}

template <bool IN_BF16, bool OUT_BF16>
static cudaError_t launch_verify128_t(const RecurrentArgs &r, cudaStream_t st) {
    dim3 grid(2, r.Hv, r.num_seqs);
    return launch_pdl(gdn_verify128_kernel<IN_BF16, OUT_BF16>, grid, dim3(kR128Threads), 0, st, r.q, r.k, r.v, r.a,
                      r.b, r.A_log, r.dt_bias, r.tokens_per_seq, r.Hk, r.Hv, r.scale, r.l2norm, r.S0, r.o);
}

template <bool IN_BF16, bool OUT_BF16>
static cudaError_t launch_recurrent128_t(const RecurrentArgs &r, cudaStream_t st) {
    // outputs only, from a given state, for 2..8 tokens per sequence: the chunk form
    if (!r.cu_seqlens && !r.S_out && r.o && r.S0 && !r.n_apply && r.tokens_per_seq >= 2 &&
        r.tokens_per_seq <= kVerifyMaxT)
        return launch_verify128_t<IN_BF16, OUT_BF16>(r, st);
    dim3 grid(2, r.Hv, r.num_seqs);
    return launch_pdl(gdn_recurrent128_kernel<IN_BF16, OUT_BF16>, grid, dim3(kR128Threads), 0, st, r.q, r.k, r.v,
                      r.a, r.b, r.A_log, r.dt_bias, r.cu_seqlens, r.tokens_per_seq, r.Hk, r.Hv, r.scale, r.l2norm,
                      r.S0, r.S_out, r.o, r.n_apply);
}

template <int D, bool IN_BF16, bool OUT_BF16>
static cudaError_t launch_recurrent_t(const RecurrentArgs &r, cudaStream_t st) {
    using Sh = RecurrentShape<D>;
    dim3 grid(Sh::SLICES, r.Hv, r.num_seqs);
    return launch_pdl(gdn_recurrent_kernel<D, IN_BF16, OUT_BF16>, grid, dim3(Sh::NT), 0, st, r.q, r.k, r.v, r.a, r.b,
                      r.A_log, r.dt_bias, r.cu_seqlens, r.tokens_per_seq, r.Hk, r.Hv, r.scale, r.l2norm, r.S0,
                      r.S_out, r.o, r.n_apply);
}

template <int D>
static cudaError_t launch_recurrent_d(const RecurrentArgs &r, cudaStream_t st) {
    if (r.in_bf16 && r.out_bf16) return launch_recurrent_t<D, true, true>(r, st);
    if (r.in_bf16 && !r.out_bf16) return launch_recurrent_t<D, true, false>(r, st);
    if (!r.in_bf16 && r.out_bf16) return launch_recurrent_t<D, false, true>(r, st);
    return launch_recurrent_t<D, false, false>(r, st);
}

cudaError_t launch_recurrent(const RecurrentArgs &r, cudaStream_t st) {
    if (r.num_seqs == 0 || r.Hv == 0) return cudaSuccess;
    switch (r.D) {
        case 16: return launch_recurrent_d<16>(r, st);
        case 32: return launch_recurrent_d<32>(r, st);
        case 64: return launch_recurrent_d<64>(r, st);
        case 128:
            if (r.in_bf16 && r.out_bf16) return launch_recurrent128_t<true, true>(r, st);
            if (r.in_bf16) return launch_recurrent128_t<true, false>(r, st);
            if (r.out_bf16) return launch_recurrent128_t<false, true>(r, st);
            return launch_recurrent128_t<false, false>(r, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gdn
