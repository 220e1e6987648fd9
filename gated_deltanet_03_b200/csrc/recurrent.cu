// Token-by-token gated delta rule on CUDA cores: the decode step (one token per sequence,
// state read once and written once, in place) and the recurrent prefill used for head
// sizes the tensor-core chunked kernel does not take.
//
// "Why Gated DeltaNet Survives 4-Bit Quantization" (abstract, mechanisms ii-iii): per
// token, with unit key k and query q,
//     alpha = exp(-exp(A_log) softplus(a + dt_bias)),  beta = sigmoid(b),
//     S <- alpha S (I - beta k k^T) + beta v k^T = alpha S + beta (v - alpha S k) k^T,
//     o = S q.
// The rows of S (value index i) evolve independently, so a CTA owns R rows of one
// (sequence, value head) state and keeps them in registers across the sequence; each
// row is spread over D/4 lanes holding 4 key columns each (128-bit loads), and the two
// row dot products (S k and S q) are lane-group shuffle reductions.
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
                     const float *S0, float *S_out, void *__restrict__ o) {
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
        if ((tid % LANES) == 0) {
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

template <int D, bool IN_BF16, bool OUT_BF16>
static cudaError_t launch_recurrent_t(const RecurrentArgs &r, cudaStream_t st) {
    using Sh = RecurrentShape<D>;
    dim3 grid(Sh::SLICES, r.Hv, r.num_seqs);
    return launch_pdl(gdn_recurrent_kernel<D, IN_BF16, OUT_BF16>, grid, dim3(Sh::NT), 0, st, r.q, r.k, r.v, r.a, r.b,
                      r.A_log, r.dt_bias, r.cu_seqlens, r.tokens_per_seq, r.Hk, r.Hv, r.scale, r.l2norm, r.S0,
                      r.S_out, r.o);
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
        case 128: return launch_recurrent_d<128>(r, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gdn
