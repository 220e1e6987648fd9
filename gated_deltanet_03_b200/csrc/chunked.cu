// Chunked gated delta-rule prefill on the fifth-generation tensor cores (tcgen05, TMEM).
//
// "Why Gated DeltaNet Survives 4-Bit Quantization" (abstract, mechanisms ii-iii) describes
// the recurrence; here it is evaluated 64 tokens at a time in the WY / UT form, which is
// exact algebra on the token-by-token rule. Within a chunk with start state S0 (Dv x Dk),
// cumulative log decay G_r = sum_{s<=r} g_s, gamma_r = exp(G_r), unit keys k_r, queries q_r:
//   A_rs = beta_r exp(G_r - G_s) k_r.k_s  (s < r),      T = (I + A)^-1,
//   W = T diag(beta gamma) K,   U~ = T diag(beta) V,     U = U~ - W S0^T,
//   O = diag(gamma) Q S0^T + (Q K^T o Gamma) U,          Gamma_rs = exp(G_r - G_s), s <= r,
//   S_C = gamma_C S0 + U^T diag(gamma_C / gamma) K.
// The L2 norms of q and k never touch an MMA operand: raw bf16 inputs (exact in fp16) feed
// the tensor cores and 1/|k|, scale/|q| enter as diagonal factors of the derived operands.
// Derived operands (T', T'', W, U, P, S0) are staged in fp16 (11-bit significand) with fp32
// accumulation in tensor memory; the state itself stays fp32 in registers.
//
// Everything is computed transposed so that every MMA has M = 128 (the value or key index
// on the tensor-memory lanes):
//   MMA1  D1[128 x 64]  = [K; Q] K^T                      (K K^T rows 0-63, Q K^T rows 64-127)
//   MMA2  D2 = W^T      = K^T T'^T      T' = T diag(beta gamma / |k|)
//   MMA3  D3 = U~^T     = V^T T''^T     T'' = T diag(beta)
//   MMA4  D3 -= S0 W^T                  (D3 becomes U^T)
//   MMA5  D5 = S0 Q^T
//   MMA6  D6 = U^T P^T                  P = Q K^T o Gamma / (|q| |k|) * scale
//   MMA7  D7 = U_S^T K                  U_S = U diag(gamma_C / gamma / |k|)
// then o^T = D5 diag(gamma * scale / |q|) + D6 and S <- gamma_C S + D7.
//
// One CTA (256 threads) owns one (sequence, value head) and walks its chunks in order; the
// next chunk's q/k/v tiles stream in by TMA (3-D maps over [T, heads, 128]) while the
// current one is processed. Tensor memory: 448 of 512 columns.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace gdn {
namespace {

constexpr int C = 64;          // chunk length
constexpr int D = 128;         // head size
constexpr int NT = 256;        // threads

// shared-memory map (bytes); 1024-byte aligned tiles for the 128-byte swizzle
constexpr int TILE = C * 128;                  // 64 rows x 128 B (one half of a 64 x 128 fp16/bf16 tile)
constexpr int OFF_KQ = 0;                      // [K_lo][Q_lo][K_hi][Q_hi] fp16 working tiles
constexpr int OFF_V = OFF_KQ + 4 * TILE;       // [V_lo][V_hi]
constexpr int OFF_STG = OFF_V + 2 * TILE;      // bf16 staging of the next chunk, same 6-tile order
constexpr int OFF_S = OFF_STG + 6 * TILE;      // S0 fp16, [S_lo: 128 rows x 64][S_hi]   (32 KB)
constexpr int OFF_W = OFF_S + 2 * 2 * TILE;    // W as [j: 128 rows][s: 64] fp16        (16 KB)
constexpr int OFF_P = OFF_W + 2 * TILE;        // P [r: 64][s: 64] fp16                 (8 KB)
constexpr int OFF_TP = OFF_P + TILE;           // T'  [s][r] fp16                       (8 KB)
constexpr int OFF_TPP = OFF_TP + TILE;         // T'' [s][r] fp16                       (8 KB)
constexpr int OFF_U = OFF_TPP + TILE;          // U_A, U_S [i: 128][s: 64] fp16          (32 KB)
// fp32 scratch of the (I + A)^-1 step, in areas that are dead while it runs:
constexpr int OFF_AF = OFF_U;                  //   A [64][65] and X [3][256] in the U area
constexpr int OFF_XF = OFF_U + 64 * 65 * 4;
constexpr int OFF_TF = OFF_W;                  //   T [64][64] in the W area
constexpr int OFF_VEC = OFF_U + 4 * TILE;      // per-chunk vectors
constexpr int VEC_FLOATS = 8 * 64;
constexpr int OFF_BAR = OFF_VEC + VEC_FLOATS * 4;
constexpr int SMEM_USED = OFF_BAR + 64;
constexpr int SMEM_BYTES = SMEM_USED + 1024;
static_assert(64 * 65 * 4 + 3 * 256 * 4 <= 4 * TILE, "A and X fit in the U area");
static_assert(64 * 64 * 4 <= 2 * TILE, "T fits in the W area");
static_assert(SMEM_BYTES <= 232448, "shared memory per block");

// tensor-memory columns
constexpr uint32_t TM_D1 = 0, TM_D2 = 64, TM_D3 = 128, TM_D5 = 192, TM_D6 = 256, TM_D7 = 320;

// kind::f16 instruction descriptor: fp16 A/B, fp32 accumulate, M = 128.
__host__ __device__ constexpr uint32_t idesc_f16(int N, bool a_mn, bool b_mn, bool neg_a) {
    return (1u << 4) | ((neg_a ? 1u : 0u) << 13) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

// K-major, 128-byte swizzle: rows of 128 B, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t kdesc(const uint8_t *p) { return smem_desc(smem_u32(p), 16, 1024, 2); }
// MN-major, 128-byte swizzle: 64 MN values per 128-B row, 8 K rows per 1024-B group,
// MN blocks of 64 `mn_stride` bytes apart.
__device__ __forceinline__ uint64_t mndesc(const uint8_t *p, uint32_t mn_stride) {
    return smem_desc(smem_u32(p), mn_stride, 1024, 2);
}

// Byte offset of (row, 16-byte chunk) inside a 128-byte-swizzled tile of 128-byte rows.
__device__ __forceinline__ uint32_t swz(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Eight fp32 values as one 16-byte chunk of fp16.
__device__ __forceinline__ void st_h8(uint8_t *p, const float *v) {
    uint4 u = make_uint4(pack_h2(v[0], v[1]), pack_h2(v[2], v[3]), pack_h2(v[4], v[5]), pack_h2(v[6], v[7]));
    *reinterpret_cast<uint4 *>(p) = u;
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

struct Maps {
    CUtensorMap q, k, v;
};

__global__ void __launch_bounds__(NT, 1)
gdn_chunked_kernel(const __grid_constant__ Maps maps, const float *__restrict__ ga, const float *__restrict__ gb,
                   const float *__restrict__ A_log, const float *__restrict__ dt_bias,
                   const int32_t *__restrict__ cu_seqlens, int32_t T, int32_t Hk, int32_t Hv, float scale,
                   int32_t l2norm, int32_t out_bf16, const float *S0g, float *S_out, void *__restrict__ o,
                   int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *vec = reinterpret_cast<float *>(sm + OFF_VEC);
    float *sG = vec, *sBeta = vec + 64, *sRk = vec + 128, *sRq = vec + 192, *sGam = vec + 256;
    float *sDecS = vec + 320;   // exp(G_last - G_s) / |k_s| for the state update
    float *sSS = vec + 384;     // row sums of squares of [K; Q] (64 + 64)
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *bar_mma = bar_tma + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_tma + 2);
    float *Af = reinterpret_cast<float *>(sm + OFF_AF);   // [64][65]
    float *Tf = reinterpret_cast<float *>(sm + OFF_TF);   // [64][64]
    float *Xf = reinterpret_cast<float *>(sm + OFF_XF);   // 3 x 256

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int h = blockIdx.x, n = blockIdx.y;
    const int hk = h / (Hv / Hk);
    int t_begin = 0, t_end = T;
    if (cu_seqlens) {
        t_begin = cu_seqlens[n];
        t_end = cu_seqlens[n + 1];
    }
    const int nchunks = (t_end - t_begin + C - 1) / C;
    const float Al = A_log[h], db = dt_bias[h];

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint32_t ph_tma = 0, ph_mma = 0;
    bool alive = true;

    auto issue_loads = [&](int t0) {
        mbar_arrive_expect_tx(bar_tma, 6 * TILE);
        uint8_t *stg = sm + OFF_STG;
        tma_load_3d(stg + 0 * TILE, &maps.k, bar_tma, 0, hk, t0);
        tma_load_3d(stg + 1 * TILE, &maps.q, bar_tma, 0, hk, t0);
        tma_load_3d(stg + 2 * TILE, &maps.k, bar_tma, 64, hk, t0);
        tma_load_3d(stg + 3 * TILE, &maps.q, bar_tma, 64, hk, t0);
        tma_load_3d(stg + 4 * TILE, &maps.v, bar_tma, 0, h, t0);
        tma_load_3d(stg + 5 * TILE, &maps.v, bar_tma, 64, h, t0);
    };
    // Wait on an mbarrier phase: one thread polls (bounded), the block learns the outcome
    // at a barrier, so every thread takes the same branch after a timeout.
    auto wait_bar = [&](uint64_t *bar, uint32_t &ph) -> bool {
        int ok = 1;
        if (tid == 0) ok = mbar_wait(bar, ph, status) ? 1 : 0;
        ph ^= 1u;
        return __syncthreads_and(ok) != 0;
    };

    if (tid == 0 && nchunks > 0) issue_loads(t_begin);

    // ---- initial state: thread (lane row i, column half wg) holds S[i][64 wg .. 64 wg + 63]
    const int wg = warp / 4;                 // column half
    const int row = (warp % 4) * 32 + lane;  // tensor-memory lane == value index i
    const uint32_t lane_base = ((uint32_t)((warp % 4) * 32)) << 16;
    float S[64];
    {
        const size_t base = (((size_t)n * Hv + h) * D + row) * D + 64 * wg;
        if (S0g) {
#pragma unroll
            for (int c = 0; c < 64; c += 4) {
                float4 x = *reinterpret_cast<const float4 *>(S0g + base + c);
                S[c] = x.x; S[c + 1] = x.y; S[c + 2] = x.z; S[c + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int c = 0; c < 64; ++c) S[c] = 0.0f;
        }
    }
    auto write_S_smem = [&]() {
        uint8_t *half = sm + OFF_S + wg * 2 * TILE;   // 128 rows x 128 B
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) st_h8(half + swz(row, ch), &S[ch * 8]);
    };
    write_S_smem();

    for (int c = 0; c < nchunks && alive; ++c) {
        const int t0 = t_begin + c * C;
        const int L = min(C, t_end - t0);

        // ---------------------------------------------------------------- stage in
        if (!wait_bar(bar_tma, ph_tma)) { alive = false; break; }
        {
            // [K;Q] rows: thread -> (row rho = tid / 2, half = tid % 2): convert and square-sum
            const int rho = tid >> 1, half = tid & 1;
            const uint32_t off = (uint32_t)(half * 2 * TILE + rho * 128);
            float ss = 0.0f;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint4 u = *reinterpret_cast<const uint4 *>(sm + OFF_STG + off + ch * 16);
                const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
                float f[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float2 x = __bfloat1622float2(b2[e]);
                    f[2 * e] = x.x; f[2 * e + 1] = x.y;
                    ss += x.x * x.x + x.y * x.y;
                }
                st_h8(sm + OFF_KQ + off + ch * 16, f);
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            if (half == 0) sSS[rho] = ss;
            // V: 1024 chunks, 4 per thread
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t o16 = (uint32_t)(4 * TILE + (tid * 4 + e) * 16);
                uint4 u = *reinterpret_cast<const uint4 *>(sm + OFF_STG + o16);
                const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
                float f[8];
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    float2 x = __bfloat1622float2(b2[q2]);
                    f[2 * q2] = x.x; f[2 * q2 + 1] = x.y;
                }
                st_h8(sm + OFF_KQ + o16, f);
            }
        }
        // gates and the in-chunk cumulative log decay (warps 0-1: token r = tid)
        if (tid < 64) {
            const int r = tid;
            float g = 0.0f, beta = 0.0f;
            if (r < L) gdn_gates(ga[(size_t)(t0 + r) * Hv + h], gb[(size_t)(t0 + r) * Hv + h], Al, db, g, beta);
            float x = g;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                float y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            sG[r] = x;       // warp-local inclusive sums; warp 1 adds warp 0's total below
            sBeta[r] = beta;
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            // MMA1: D1 = [K; Q] K^T (M = 128, N = 64, K = 128)
            tc_fence_after();
            const uint32_t id = idesc_f16(64, false, false, false);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint8_t *abase = sm + OFF_KQ + (kk < 4 ? 0 : 2 * TILE) + (kk & 3) * 32;
                mma_f16(tmem + TM_D1, kdesc(abase), kdesc(abase), id, kk > 0 ? 1u : 0u);
            }
            tc_commit(bar_mma);
            // the staging tiles are free: stream in the next chunk
            if (c + 1 < nchunks) {
                fence_proxy_async_smem();
                issue_loads(t0 + C);
            }
        }
        if (tid >= 32 && tid < 64) sG[tid] += sG[31];
        __syncthreads();
        if (tid < 64) {
            const int r = tid;
            const float G = sG[r];
            const bool v = r < L;
            const float rk = v ? (l2norm ? rsqrtf(sSS[r] + 1e-6f) : 1.0f) : 0.0f;
            const float rq = v ? (l2norm ? rsqrtf(sSS[64 + r] + 1e-6f) * scale : scale) : 0.0f;
            sRk[r] = rk;
            sRq[r] = rq;
            sGam[r] = v ? expf(G) : 0.0f;
        }
        __syncthreads();
        const float G_last = sG[L - 1];
        if (tid < 64) sDecS[tid] = tid < L ? expf(G_last - sG[tid]) * sRk[tid] : 0.0f;

        // ---------------------------------------------------- A and P from D1
        if (!wait_bar(bar_mma, ph_mma)) { alive = false; break; }
        tc_fence_after();
        {
            uint32_t r32[32];
            const int col0 = wg * 32;
            tmem_ld32(tmem + TM_D1 + lane_base + col0, r32);
            tmem_ld_wait();
            if (row < 64) {
                const int r = row;
                const float Gr = sG[r], br = sBeta[r], rkr = sRk[r];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int s = col0 + j;
                    float a = 0.0f;
                    if (s < r && r < L) a = br * expf(Gr - sG[s]) * __uint_as_float(r32[j]) * rkr * sRk[s];
                    Af[r * 65 + s] = a;
                }
            } else {
                const int r = row - 64;
                const float Gr = sG[r], rqr = sRq[r];
                float pv[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int s = col0 + j;
                    float p = 0.0f;
                    if (s <= r && r < L) p = __uint_as_float(r32[j]) * rqr * sRk[s] * expf(Gr - sG[s]);
                    pv[j] = p;
                }
                uint8_t *P = sm + OFF_P;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) st_h8(P + swz(r, wg * 4 + ch), &pv[ch * 8]);
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---------------------------------------------------- T = (I + A)^-1, blocked 16 x 16
        if (tid < 64) {
            const int bi = tid / 16, cc = tid % 16, o0 = bi * 16;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = (r == cc) ? 1.0f : 0.0f;
#pragma unroll
                for (int s = 0; s < r; ++s) acc -= Af[(o0 + r) * 65 + o0 + s] * x[s];
                x[r] = acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) Tf[(o0 + r) * 64 + o0 + cc] = x[r];
        }
        __syncthreads();
        for (int lvl = 1; lvl < 4; ++lvl) {
            const int nblk = 4 - lvl;
            const int er = tid / 16, ec = tid % 16;
            // X_ij = sum_{k=j}^{i-1} A_ik T_kj   for (i, j) = (j + lvl, j)
            for (int bj = 0; bj < nblk; ++bj) {
                const int bi = bj + lvl;
                float acc = 0.0f;
                for (int bk = bj; bk < bi; ++bk)
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        acc += Af[(bi * 16 + er) * 65 + bk * 16 + e] * Tf[(bk * 16 + e) * 64 + bj * 16 + ec];
                Xf[bj * 256 + er * 16 + ec] = acc;
            }
            __syncthreads();
            // T_ij = -T_ii X_ij
            for (int bj = 0; bj < nblk; ++bj) {
                const int bi = bj + lvl;
                float acc = 0.0f;
#pragma unroll
                for (int e = 0; e < 16; ++e) acc += Tf[(bi * 16 + er) * 64 + bi * 16 + e] * Xf[bj * 256 + e * 16 + ec];
                Tf[(bi * 16 + er) * 64 + bj * 16 + ec] = -acc;
            }
            __syncthreads();
        }
        // T' = T diag(beta gamma rk), T'' = T diag(beta) as fp16 B operands [s][r] (r <= s)
        {
            const int s = tid / 4, part = tid % 4;   // 16 columns each
            float tp[16], tpp[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int r = part * 16 + e;
                const float t = (r <= s) ? Tf[s * 64 + r] : 0.0f;
                tp[e] = t * sBeta[r] * sGam[r] * sRk[r];
                tpp[e] = t * sBeta[r];
            }
            st_h8(sm + OFF_TP + swz(s, part * 2), tp);
            st_h8(sm + OFF_TP + swz(s, part * 2 + 1), tp + 8);
            st_h8(sm + OFF_TPP + swz(s, part * 2), tpp);
            st_h8(sm + OFF_TPP + swz(s, part * 2 + 1), tpp + 8);
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            // MMA2: D2 = K^T T'^T (A = K, MN-major over the key index; K-extent = token r)
            const uint32_t id_mn = idesc_f16(64, true, false, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + TM_D2, mndesc(sm + OFF_KQ + kk * 2048, 2 * TILE), kdesc(sm + OFF_TP + kk * 32), id_mn,
                        kk > 0);
            // MMA3: D3 = V^T T''^T
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + TM_D3, mndesc(sm + OFF_V + kk * 2048, TILE), kdesc(sm + OFF_TPP + kk * 32), id_mn, kk > 0);
            // MMA5: D5 = S0 Q^T (A = S0 K-major over j, B = Q K-major over j)
            const uint32_t id_kk = idesc_f16(64, false, false, false);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint8_t *a = sm + OFF_S + (kk < 4 ? 0 : 2 * TILE) + (kk & 3) * 32;
                const uint8_t *b = sm + OFF_KQ + TILE + (kk < 4 ? 0 : 2 * TILE) + (kk & 3) * 32;
                mma_f16(tmem + TM_D5, kdesc(a), kdesc(b), id_kk, kk > 0);
            }
            tc_commit(bar_mma);
        }
        if (!wait_bar(bar_mma, ph_mma)) { alive = false; break; }
        tc_fence_after();
        // ---------------------------------------------------- W (fp16, [j][s]) from D2
        {
            uint32_t r32[32];
            tmem_ld32(tmem + TM_D2 + lane_base + wg * 32, r32);
            tmem_ld_wait();
            float w[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) w[j] = __uint_as_float(r32[j]);
            uint8_t *Wt = sm + OFF_W;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) st_h8(Wt + swz(row, wg * 4 + ch), &w[ch * 8]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            // MMA4: D3 -= S0 W^T (B = W, MN-major over the token index s; K-extent = j)
            const uint32_t id = idesc_f16(64, false, true, true);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint8_t *a = sm + OFF_S + (kk < 4 ? 0 : 2 * TILE) + (kk & 3) * 32;
                mma_f16(tmem + TM_D3, kdesc(a), mndesc(sm + OFF_W + kk * 2048, 0), id, 1u);
            }
            tc_commit(bar_mma);
        }
        if (!wait_bar(bar_mma, ph_mma)) { alive = false; break; }
        tc_fence_after();
        // ---------------------------------------------------- U^T rows -> U_A, U_S (fp16 [i][s])
        {
            uint32_t r32[32];
            tmem_ld32(tmem + TM_D3 + lane_base + wg * 32, r32);
            tmem_ld_wait();
            float ua[32], us[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int s = wg * 32 + j;
                const float u = (s < L) ? __uint_as_float(r32[j]) : 0.0f;
                ua[j] = u;
                us[j] = u * sDecS[s];
            }
            uint8_t *UA = sm + OFF_U, *US = sm + OFF_U + 2 * TILE;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                st_h8(UA + swz(row, wg * 4 + ch), &ua[ch * 8]);
                st_h8(US + swz(row, wg * 4 + ch), &us[ch * 8]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            // MMA6: D6 = U^T P^T ; MMA7: D7 = U_S^T K (B = K MN-major over j; K-extent = s)
            const uint32_t id6 = idesc_f16(64, false, false, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + TM_D6, kdesc(sm + OFF_U + kk * 32), kdesc(sm + OFF_P + kk * 32), id6, kk > 0);
            const uint32_t id7 = idesc_f16(128, false, true, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + TM_D7, kdesc(sm + OFF_U + 2 * TILE + kk * 32), mndesc(sm + OFF_KQ + kk * 2048, 2 * TILE),
                        id7, kk > 0);
            tc_commit(bar_mma);
        }
        if (!wait_bar(bar_mma, ph_mma)) { alive = false; break; }
        tc_fence_after();
        // ---------------------------------------------------- outputs and the state update
        {
            uint32_t a5[32], a6[32];
            tmem_ld32(tmem + TM_D5 + lane_base + wg * 32, a5);
            tmem_ld32(tmem + TM_D6 + lane_base + wg * 32, a6);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int r = wg * 32 + j;
                if (r < L) {
                    const float val = __uint_as_float(a5[j]) * sGam[r] * sRq[r] + __uint_as_float(a6[j]);
                    const size_t idx = ((size_t)(t0 + r) * Hv + h) * D + row;
                    if (out_bf16) store1<true>(o, idx, val);
                    else store1<false>(o, idx, val);
                }
            }
            const float gC = sGam[L - 1];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t r7[32];
                tmem_ld32(tmem + TM_D7 + lane_base + wg * 64 + half * 32, r7);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) S[half * 32 + j] = gC * S[half * 32 + j] + __uint_as_float(r7[j]);
            }
            write_S_smem();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    if (alive && S_out) {
        const size_t base = (((size_t)n * Hv + h) * D + row) * D + 64 * wg;
#pragma unroll
        for (int c = 0; c < 64; c += 4)
            *reinterpret_cast<float4 *>(S_out + base + c) = make_float4(S[c], S[c + 1], S[c + 2], S[c + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D bf16 map over [T, heads, 128] (innermost first), box 64 values x 1 head x 64 tokens.
bool make_map3(CUtensorMap *m, const void *ptr, int T, int heads) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)heads, (cuuint64_t)T};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)heads * 128 * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t elem[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, elem,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_chunked(const ChunkedArgs &c, cudaStream_t st) {
    Maps maps;
    if (!make_map3(&maps.q, c.q, c.T, c.Hk) || !make_map3(&maps.k, c.k, c.T, c.Hk) ||
        !make_map3(&maps.v, c.v, c.T, c.Hv))
        return cudaErrorInvalidValue;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(gdn_chunked_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    dim3 grid(c.Hv, c.num_seqs);
    gdn_chunked_kernel<<<grid, NT, SMEM_BYTES, st>>>(maps, c.a, c.b, c.A_log, c.dt_bias, c.cu_seqlens, c.T, c.Hk, c.Hv,
                                                      c.scale, c.l2norm, c.out_bf16 ? 1 : 0, c.S0, c.S_out, c.o,
                                                      c.status);
    return cudaGetLastError();
}

}  // namespace gdn
