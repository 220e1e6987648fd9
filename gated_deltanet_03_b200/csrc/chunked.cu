// Chunked gated delta-rule prefill on the fifth-generation tensor cores (tcgen05, TMEM): a prep
// kernel that is parallel over (chunk, value head), and the state chain, sequential over the
// chunks of each (sequence, value head) and cut into segments (state and transition passes, a
// short combine of the segments' maps, then the output pass from each segment's true start).
//
// "Why Gated DeltaNet Survives 4-Bit Quantization" (abstract, mechanisms ii-iii) describes
// the recurrence; here it is evaluated 64 tokens at a time in the WY / UT form, which is
// exact algebra on the token-by-token rule. Within a chunk with start state S0 (Dv x Dk),
// cumulative log decay G_r = sum_{s<=r} g_s, gamma_r = exp(G_r), unit keys k_r, queries q_r:
//   A_rs = beta_r exp(G_r - G_s) k_r.k_s  (s < r),      T = (I + A)^-1,
//   W = T diag(beta gamma) K,   U~ = T diag(beta) V,     U = U~ - W S0^T,
//   O = diag(gamma) Q S0^T + (Q K^T o Gamma) U,          Gamma_rs = exp(G_r - G_s), s <= r,
//   S_C = gamma_C S0 + U^T diag(gamma_C / gamma) K.
// W, U~, P = (Q K^T o Gamma), the scaled Q and the factors c_r = gamma_C / gamma_r / |k_r| do
// not depend on the state: the prep kernel computes them for every chunk at once into the
// caller's workspace; the chain kernels then run the state-dependent MMAs per chunk.
//
// Precision. The L2 norms of q and k never touch an MMA operand: the raw bf16 inputs feed the
// tensor cores and 1/|k|, scale/|q| enter as diagonal factors. When keys are nearly parallel and
// beta -> 1 (each write replaces the state along a key close to earlier ones), T has O(1)
// entries of alternating sign and W, U are small differences, so a single 11-bit rounding of the
// derived operands costs several 1e-3 of the result. The operands that carry this cancellation
// are therefore kept to about 16 bits: the inverse is fp32, T' and T'' enter MMA2 as bf16 hi + lo
// parts, U~ is stored in fp32, and in the chain U (with P^T) and U diag(c) (with the raw K) enter
// as bf16 hi + lo parts (hi hi + hi lo + lo hi). W, Q' and the state's A-operand copy S0 stay
// fp16, which the result tolerates; the state itself stays fp32 in registers.
//
// Every MMA has M = 128 (value or key index on the TMEM lanes):
//   prep   MMA1  D1 = [K; Q] [K; Q]^T      on the raw bf16 tiles (rows 0-63: K K^T | K Q^T,
//                                          rows 64-127: Q K^T | Q Q^T; the diagonals give the norms)
//          MMA2a D2 = [T'; T''] K          bf16, hi then lo A parts; rows 0-63: W = T' K
//          MMA2b D2 = [T'; T''] V          then, over the same columns, rows 64-127: U~ = T'' V;
//                                          T' = T diag(beta gamma / |k|), T'' = T diag(beta)
//   chain  MMA45 [D4 | D5a] = S0 [W; Q']^T      fp16; Q' = diag(gamma scale / |q|) Q
//          MMA7  D7 = (U diag(c))^T K           bf16 hi / lo A, raw bf16 K
//          MMA5b D5a += U^T P^T                 bf16 hi / lo, P^T[s][r] = k_s.q_r Gamma_rs scale / (|q_r| |k_s|)
//   with U^T = U~^T - D4, S <- gamma_C S + D7, o^T = D5a. In the chain the copies of S0 and of U
//   live in tensor memory as the A operands; the element-wise warps (sixteen in the output pass,
//   beside one copy/MMA warp; eight in the lean pass, one of whose threads issues) hand over to
//   the issuing thread through mbarriers.
//
// Workspace: one 81 KB item per (value head, chunk slot): [W; Q'] (fp16, K-major, 128 rows,
// 128-byte swizzled), P^T hi and lo (bf16, MN-major over r), U~ (fp32 [s][i]), c[64] and
// gamma_C. Chunk c of sequence n uses slot cu_seqlens[n] / 64 + n + c, so slots never collide
// and T / 64 + num_seqs slots per head suffice. The chain reads the raw K tiles itself.
#include <algorithm>
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace gdn {

constexpr int kChunk = 64;
constexpr int kWsItem = 82944;
constexpr int kWsWQ = 0, kWsP = 32768, kWsU = 49152, kWsVec = 81920;

constexpr size_t kSegItemBytes = 196608;

// Chunks per segment of the chain: the state chain of a sequence is split into segments that
// run in parallel (state and transition passes), a short sequential combine, and the output
// pass. Picks the length that minimises a cost model of the three passes - per-chunk costs of
// the output pass (one CTA per SM) and of the state / transition passes (two CTAs per SM) and the
// cost of one combine step - fitted to fused-prefill timings on B200 over 8192 - 32768 tokens
// (segment lengths 4 - 256, powers of two and others), within 1 % of every timing once a constant
// per workload is allowed for the prep kernel. CTA waves above one count halfway between their
// fraction and the next whole wave (a second wave of equal CTAs costs a whole wave, but CTAs
// finish unevenly). A single sequence searches every length; a batch is planned from its mean
// sequence length (the host does not read cu_seqlens) over powers of two only, since one long
// sequence in a skewed batch sets the chain's length whatever the mean says.
int chunked_segment_chunks(int T, int num_seqs, int Hv) {
    const int nseq = num_seqs > 0 ? num_seqs : 1;
    const double nch = (double)T / kChunk / nseq;
    const double c_full = 2.0, c_state = 1.4, c_comb = 3.0, sms = 148.0;
    auto waves = [](double x) { return x <= 1.0 ? 1.0 : 0.5 * (x + std::ceil(x)); };
    int best = 1 << 30;
    double best_cost = 1e30;
    for (int seg = 4; seg <= 4096; seg = nseq == 1 ? seg + 1 : seg * 2) {
        const double nseg = nch / seg > 1.0 ? std::ceil(nch / seg) : 1.0;
        const double ctas = (double)Hv * nseq * nseg;
        double cost = waves(ctas / sms) * std::min((double)seg, nch) * c_full;
        if (nseg > 1.0) {
            const double lean_ctas = 2.0 * Hv * nseq * (nseg - 1.0);
            cost += waves(lean_ctas / (2.0 * sms)) * seg * c_state + (nseg - 2.0) * c_comb;
        }
        if (cost < best_cost) {
            best_cost = cost;
            best = seg;
        }
        if (seg >= nch) break;
    }
    return best;
}

size_t chunked_workspace_bytes(int T, int num_seqs, int Hk, int Hv) {
    (void)Hk;
    const int seg = chunked_segment_chunks(T, num_seqs, Hv);
    return (size_t)Hv * (size_t)(T / kChunk + num_seqs) * kWsItem +
           (size_t)Hv * (size_t)(T / (kChunk * seg) + num_seqs) * kSegItemBytes;
}

namespace {

constexpr int C = kChunk;      // chunk length
constexpr int D = 128;         // head size
constexpr int NT = 256;        // element-wise threads per CTA
constexpr int TILE = C * 128;  // 64 rows x 128 B: one half (64 columns) of a 64 x 128 16-bit tile

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

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

struct Maps {
    CUtensorMap q, k, v;
};

// Chunk location: slot `id` of the workspace belongs to sequence n (the last n whose first
// slot cu[n] / 64 + n is <= id) and is its chunk id - (cu[n] / 64 + n).
__device__ __forceinline__ void locate(int id, const int32_t *cu, int num_seqs, int T, int &n, int &t_begin,
                                       int &t_end) {
    n = 0;
    t_begin = 0;
    t_end = T;
    if (cu) {
        int lo = 0, hi = num_seqs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) / 2;
            if (cu[mid] / C + mid <= id) lo = mid;
            else hi = mid - 1;
        }
        n = lo;
        t_begin = cu[n];
        t_end = cu[n + 1];
    }
}

// Warp-level 16 x 8 x 16 MMA, bf16 inputs, fp32 accumulation (row-major A, column-major B): the
// 16 x 16 blocks of the triangular inverse. Fragments: a = {A[g][2t..], A[g+8][2t..], A[g][2t+8..],
// A[g+8][2t+8..]}, b = {B[2t..][g], B[2t+8..][g]}, c = {C[g][2t], C[g][2t+1], C[g+8][2t], C[g+8][2t+1]}
// with g = lane / 4, t = lane % 4 (pairs in one 32-bit register, the lower index in the low half).
__device__ __forceinline__ void mma_bf16_m16n8k16(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// ===================================================================================
// Prep kernel: one CTA per (chunk slot, value head); three CTAs per SM (68 KB of shared memory,
// 128 tensor-memory columns, at most 80 registers a thread).
// ===================================================================================
// Shared memory (TILE = 8 KB). [K_lo; Q_lo] (tiles 0-1) and [K_hi; Q_hi] (tiles 2-3) are the two
// K-major column blocks of the MMA1 operand [K; Q]; K_lo and K_hi, 2 TILE apart, are also the
// MN-major B operand K of MMA2a. Once MMA1 has completed and the Q' rows are written out, V is
// loaded into the Q tiles (V_lo over Q_lo, V_hi over Q_hi: the B operand of MMA2b, blocks 2 TILE
// apart as well). Tiles 4-6 hold the fp32 A / T array; once T is in registers, tiles 4-7 take
// the bf16 hi (4-5) and lo (6-7) images of [T'; T''], the A operand of MMA2a and MMA2b. P^T, W
// and U~ go from registers straight into the workspace item.
constexpr int P_OFF_KLO = 0, P_OFF_QLO = TILE, P_OFF_KHI = 2 * TILE, P_OFF_QHI = 3 * TILE;
constexpr int P_OFF_VLO = P_OFF_QLO, P_OFF_VHI = P_OFF_QHI;
constexpr int P_AT = 72;                           // fp32 row pitch of the A / T array (8-byte fragment loads
                                                   // of a warp-level MMA without bank conflicts)
constexpr int P_OFF_AT = 4 * TILE;                 // T (strict lower, row-major) and A (strict lower, transposed)
constexpr int P_OFF_AHI = 4 * TILE, P_OFF_ALO = 6 * TILE;   // [T'; T''] hi / lo, after T is read
constexpr int P_OFF_VEC = 8 * TILE;                // G, beta, rk, rq, gamma, c, beta gamma rk, spare (64 each)
constexpr int P_OFF_BAR = P_OFF_VEC + 8 * 64 * 4;
constexpr int P_SMEM = P_OFF_BAR + 64 + 1024;
static_assert(P_OFF_AT + 64 * P_AT * 4 <= P_OFF_VEC, "the A / T array stays clear of the vectors");
static_assert(3 * (P_SMEM + 1024) <= 233472, "three prep CTAs per SM");
// tensor memory (128 columns): D1 = [K; Q] [K; Q]^T, then D2a = [T'; T''] K (rows 0-63: W) and
// D2b = [T'; T''] V (rows 64-127: U~) in turn over it
constexpr uint32_t P_TM_D1 = 0, P_TM_D2 = 0;

// bf16 hi / lo split of two fp32 values, packed as bf16x2 words: hi = bf16(x), lo = bf16(x - hi).
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

__global__ void __launch_bounds__(NT, 3)
gdn_chunk_prep_kernel(const __grid_constant__ Maps maps, const float *__restrict__ ga, const float *__restrict__ gb,
                      const float *__restrict__ A_log, const float *__restrict__ dt_bias,
                      const int32_t *__restrict__ cu_seqlens, int32_t T, int32_t num_seqs, int32_t Hk, int32_t Hv,
                      int32_t slots, float scale, int32_t l2norm, uint8_t *__restrict__ ws, int *status) {
    pdl_launch_dependents();
    pdl_wait();
    // heads fastest: the value heads of a chunk run together, so the gate rows they read and the
    // K and Q tiles that value heads of one key head share come from DRAM once
    const int h = blockIdx.x, id = blockIdx.y;
    int n, t_begin, t_end;
    locate(id, cu_seqlens, num_seqs, T, n, t_begin, t_end);
    const int t0 = t_begin + (id - (t_begin / C + n)) * C;
    if (id < t_begin / C + n || t0 >= t_end) return;   // a slot no chunk uses
    const int L = min(C, t_end - t0);
    const int hk = h / (Hv / Hk);
    uint8_t *item = ws + ((size_t)h * slots + id) * kWsItem;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *vec = reinterpret_cast<float *>(sm + P_OFF_VEC);
    float *sG = vec, *sBeta = vec + 64, *sRk = vec + 128, *sRq = vec + 192, *sGam = vec + 256, *sDec = vec + 320;
    float *sBG = vec + 384;
    float *AT = reinterpret_cast<float *>(sm + P_OFF_AT);
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + P_OFF_BAR);
    uint64_t *bar_mma = bar_tma + 1;
    uint64_t *bar_v = bar_tma + 2;
    uint64_t *bar_drain = bar_tma + 3;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_tma + 4);

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int wg = warp / 4;
    const int x = (warp % 4) * 32 + lane;   // this thread's TMEM lane
    const uint32_t lane_base = ((uint32_t)((warp % 4) * 32)) << 16;
    // what thread 0 has issued, for the drain on the failure path
    bool loads_issued = false, v_issued = false;
    int mmas_issued = 0;
    bool failed = false;

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_drain, 1);
        fence_barrier_init();
        if (!(ctl_flags(status) & kInjectSkipPrepLoads)) {
            // K and Q on one barrier (MMA1 starts when they land); V follows into the Q tiles later
            mbar_arrive_expect_tx(bar_tma, 4 * TILE);
            tma_load_3d(sm + P_OFF_KLO, &maps.k, bar_tma, 0, hk, t0);
            tma_load_3d(sm + P_OFF_QLO, &maps.q, bar_tma, 0, hk, t0);
            tma_load_3d(sm + P_OFF_KHI, &maps.k, bar_tma, 64, hk, t0);
            tma_load_3d(sm + P_OFF_QHI, &maps.q, bar_tma, 64, hk, t0);
            loads_issued = true;
        }
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    // gates and the warp-local part of the cumulative log decay, while the tiles stream in
    if (tid < 64) {
        float g = 0.0f, beta = 0.0f;
        if (tid < L) gdn_gates(ga[(size_t)(t0 + tid) * Hv + h], gb[(size_t)(t0 + tid) * Hv + h], A_log[h], dt_bias[h], g, beta);
        float xs = g;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            float y = __shfl_up_sync(0xffffffffu, xs, off);
            if (lane >= off) xs += y;
        }
        sG[tid] = xs;
        sBeta[tid] = beta;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (tid >= 32 && tid < 64) sG[tid] += sG[31];

    int ok = 1;
    if (tid == 0) {
        ok = mbar_wait(bar_tma, 0, status) ? 1 : 0;
        if (ok) {
            // D1 = [K; Q] [K; Q]^T straight from the raw bf16 tiles: lanes 0-63 hold K K^T | K Q^T,
            // lanes 64-127 Q K^T | Q Q^T (row = token, column = token). The diagonals are the
            // squared norms |k_r|^2 and |q_r|^2 (exact bf16 products, fp32 sums).
            tc_fence_after();
            const uint32_t id1 = idesc_f16(128, false, false, false) | (1u << 7) | (1u << 10);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint8_t *base = sm + (kk < 4 ? P_OFF_KLO : P_OFF_KHI) + (kk & 3) * 32;
                mma_f16(tmem + P_TM_D1, kdesc(base), kdesc(base), id1, kk > 0 ? 1u : 0u);
            }
            tc_commit(bar_mma);
            mmas_issued = 1;
        }
    }
    if (!__syncthreads_and(ok)) { failed = true; goto teardown; }
    // while MMA1 runs: the decay factors
    if (tid < 64) sGam[tid] = tid < L ? expf(sG[tid]) : 0.0f;
    if (tid == 0) ok = mbar_wait(bar_mma, 0, status) ? 1 : 0;
    if (!__syncthreads_and(ok)) { failed = true; goto teardown; }
    tc_fence_after();
    {
        // every warp reads 32 columns (key tokens s) of its 32 lanes; warps 2 and 3 first read the
        // Q Q^T block that holds their lanes' diagonal
        uint32_t r32[32];
        const int quarter = warp % 4;
        if (wg == 0 && quarter >= 2) {
            tmem_ld32(tmem + P_TM_D1 + lane_base + 64 + (quarter - 2) * 32, r32);
            tmem_ld_wait();
            float d = 0.0f;
#pragma unroll
            for (int j = 0; j < 32; ++j) d = (j == lane) ? __uint_as_float(r32[j]) : d;
            const int r = x - 64;
            sRq[r] = r < L ? (l2norm ? rsqrtf(d + 1e-6f) * scale : scale) : 0.0f;
        }
        tmem_ld32(tmem + P_TM_D1 + lane_base + wg * 32, r32);
        tmem_ld_wait();
        if (quarter < 2 && wg == quarter) {
            // lanes 0-63: the K K^T diagonal sits in column x, i.e. this warp's column `lane`
            float d = 0.0f;
#pragma unroll
            for (int j = 0; j < 32; ++j) d = (j == lane) ? __uint_as_float(r32[j]) : d;
            const int r = x;
            const float rk = r < L ? (l2norm ? rsqrtf(d + 1e-6f) : 1.0f) : 0.0f;
            sRk[r] = rk;
            sDec[r] = r < L ? __expf(sG[L - 1] - sG[r]) * rk : 0.0f;
        }
        __syncthreads();
        // this warp's 32 columns (key tokens s), two at a time; the decay and key-norm factors of a
        // column pair come from shared memory (the same address for every lane)
        if (x < 64) {
            // row r of A (fp32): A_rs = beta_r exp(G_r - G_s) k_r.k_s / (|k_r| |k_s|) for s < r < L
            const int r = x;
            const float Gr = sG[r], cr = sBeta[r] * sRk[r];
            const f2_t cr2 = f2(cr, cr);
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                const int s0 = wg * 32 + j;
                const float2 g2 = *reinterpret_cast<const float2 *>(sG + s0);
                const float2 k2 = *reinterpret_cast<const float2 *>(sRk + s0);
                const f2_t v2 = mul2(mul2(f2(exp_approx(Gr - g2.x), exp_approx(Gr - g2.y)),
                                          f2(__uint_as_float(r32[j]), __uint_as_float(r32[j + 1]))),
                                     mul2(f2(k2.x, k2.y), cr2));
                if (s0 < r) AT[s0 * P_AT + r] = f2lo(v2);
                if (s0 + 1 < r) AT[(s0 + 1) * P_AT + r] = f2hi(v2);
            }
        } else {
            // row r of P = (Q K^T o Gamma) scaled, as bf16 hi and lo P^T images [s][r] (MN-major over
            // r, 128-byte swizzled), written straight into the workspace item (zeros above the
            // diagonal, so the images are whole)
            const int r = x - 64;
            const float Gr = sG[r], cr = sRq[r];
            const f2_t cr2 = f2(cr, cr);
            uint8_t *pimg = item + kWsP;
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                const int s0 = wg * 32 + j;
                const float2 g2 = *reinterpret_cast<const float2 *>(sG + s0);
                const float2 k2 = *reinterpret_cast<const float2 *>(sRk + s0);
                const f2_t v2 = mul2(mul2(f2(exp_approx(Gr - g2.x), exp_approx(Gr - g2.y)),
                                          f2(__uint_as_float(r32[j]), __uint_as_float(r32[j + 1]))),
                                     mul2(f2(k2.x, k2.y), cr2));
                const float pv[2] = {s0 <= r ? f2lo(v2) : 0.0f, s0 + 1 <= r ? f2hi(v2) : 0.0f};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const __nv_bfloat16 hb = __float2bfloat16_rn(pv[e]);
                    const __nv_bfloat16 lb = __float2bfloat16_rn(pv[e] - __bfloat162float(hb));
                    const uint32_t off = swz(s0 + e, r >> 3) + (r & 7) * 2;
                    *reinterpret_cast<__nv_bfloat16 *>(pimg + off) = hb;
                    *reinterpret_cast<__nv_bfloat16 *>(pimg + TILE + off) = lb;
                }
            }
        }
    }
    __syncthreads();

    // ---- T = (I + A)^-1 (unit lower triangular) in fp32. A is stored transposed in the strict
    //      upper part of the array (A[r][s] at AT[s][r]), T row-major in the strict lower part.
    //      Two warps solve the 16 x 16 diagonal blocks by forward substitution while the other six
    //      write the Q' rows (64 + r of the [W; Q'] image: the raw bf16 Q tile scaled row by row,
    //      swizzle positions unchanged), the decay vector and the column factors of T'.
    if (tid < 64) {
        const int bi = tid / 16, cc = tid % 16, o0 = bi * 16;
        float xv[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            float acc = (rr == cc) ? 1.0f : 0.0f;
#pragma unroll
            for (int s = 0; s < rr; ++s)
                if (s >= cc) acc -= AT[(o0 + s) * P_AT + o0 + rr] * xv[s];
            xv[rr] = (rr < cc) ? 0.0f : acc;
        }
#pragma unroll
        for (int rr = 0; rr < 16; ++rr)
            if (rr > cc) AT[(o0 + rr) * P_AT + o0 + cc] = xv[rr];
    } else {
        const int t6 = tid - 64;
        // Q' (1024 chunks over 192 threads, loads issued before the stores)
        {
            uint4 hv[6];
            float f[6];
#pragma unroll
            for (int e = 0; e < 6; ++e) {
                const int idx = e * 192 + t6;
                const int w = idx < 1024 ? idx : 0, half = w >> 9, within = w & 511, r = within >> 3;
                hv[e] = *reinterpret_cast<const uint4 *>(sm + (half ? P_OFF_QHI : P_OFF_QLO) + within * 16);
                f[e] = sGam[r] * sRq[r];
            }
#pragma unroll
            for (int e = 0; e < 6; ++e) {
                const int idx = e * 192 + t6;
                if (idx < 1024) {
                    const int half = idx >> 9, within = idx & 511;
                    const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&hv[e]);
                    float xv[8];
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2) {
                        const float2 t = __bfloat1622float2(b2[q2]);
                        xv[2 * q2] = t.x * f[e];
                        xv[2 * q2 + 1] = t.y * f[e];
                    }
                    st_h8(item + kWsWQ + half * 2 * TILE + TILE + within * 16, xv);
                }
            }
        }
        // the per-token factors of the state update, c_r = gamma_C / gamma_r / |k_r|, and gamma_C
        if (t6 < 64) reinterpret_cast<float *>(item + kWsVec)[t6] = sDec[t6];
        if (t6 == 64) reinterpret_cast<float *>(item + kWsVec)[64] = L > 0 ? __expf(sG[L - 1]) : 1.0f;
        // column factors of T' = T diag(beta gamma / |k|)
        if (t6 >= 128) sBG[t6 - 128] = sBeta[t6 - 128] * sGam[t6 - 128] * sRk[t6 - 128];
    }
    __syncthreads();
    // MMA1 has completed and the Q' rows are out: V into the Q tiles (needed by MMA2b)
    if (tid == 0 && loads_issued) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar_v, 2 * TILE);
        tma_load_3d(sm + P_OFF_VLO, &maps.v, bar_v, 0, h, t0);
        tma_load_3d(sm + P_OFF_VHI, &maps.v, bar_v, 64, h, t0);
        v_issued = true;
    }
    // ---- off-diagonal blocks level by level, from T (I + A) = I:
    //      X = sum_{bk = bj+1 .. bi} T_{bi,bk} A_{bk,bj},   T_{bi,bj} = -X T_{bj,bj},
    //      one warp per block on the warp-level tensor-core MMA (m16n8k16) with every operand split
    //      into bf16 hi + lo parts (hi hi + hi lo + lo hi, fp32 accumulation: about 16 significant
    //      bits per product, as the fp32 blocks need); the sum's accumulator fragments are
    //      directly the A fragments of the product with T_jj.
#pragma unroll 1
    for (int lvl = 1; lvl < 4; ++lvl) {
        if (warp < 4 - lvl) {
            const int bj = warp, bi = bj + lvl;
            const int g = lane >> 2, t = lane & 3;
            const int r0 = bi * 16 + g, r1 = r0 + 8;
            float xc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            for (int bk = bj + 1; bk <= bi; ++bk) {
                // A fragment: T[r][k] for r in block bi, k = 16 bk + {2t, 2t+1, 2t+8, 2t+9}
                const int k0 = bk * 16 + 2 * t;
                float2 e00 = *reinterpret_cast<const float2 *>(AT + r0 * P_AT + k0);
                float2 e10 = *reinterpret_cast<const float2 *>(AT + r1 * P_AT + k0);
                float2 e01 = *reinterpret_cast<const float2 *>(AT + r0 * P_AT + k0 + 8);
                float2 e11 = *reinterpret_cast<const float2 *>(AT + r1 * P_AT + k0 + 8);
                if (bk == bi) {   // the diagonal block: 1 on the diagonal, 0 above it
                    auto fix = [](float v, int r, int k) { return k < r ? v : (k == r ? 1.0f : 0.0f); };
                    e00 = make_float2(fix(e00.x, r0, k0), fix(e00.y, r0, k0 + 1));
                    e10 = make_float2(fix(e10.x, r1, k0), fix(e10.y, r1, k0 + 1));
                    e01 = make_float2(fix(e01.x, r0, k0 + 8), fix(e01.y, r0, k0 + 9));
                    e11 = make_float2(fix(e11.x, r1, k0 + 8), fix(e11.y, r1, k0 + 9));
                }
                uint32_t ah[4], al[4];
                split_bf16x2(e00.x, e00.y, ah[0], al[0]);
                split_bf16x2(e10.x, e10.y, ah[1], al[1]);
                split_bf16x2(e01.x, e01.y, ah[2], al[2]);
                split_bf16x2(e11.x, e11.y, ah[3], al[3]);
#pragma unroll
                for (int hn = 0; hn < 2; ++hn) {
                    // B fragment: A[k][c] (stored at AT[c][k]) for k = 16 bk + {2t, 2t+1, 2t+8, 2t+9}
                    const int c = bj * 16 + hn * 8 + g;
                    const float2 b0 = *reinterpret_cast<const float2 *>(AT + c * P_AT + k0);
                    const float2 b1 = *reinterpret_cast<const float2 *>(AT + c * P_AT + k0 + 8);
                    uint32_t bh[2], bl[2];
                    split_bf16x2(b0.x, b0.y, bh[0], bl[0]);
                    split_bf16x2(b1.x, b1.y, bh[1], bl[1]);
                    mma_bf16_m16n8k16(xc[hn], ah, bh);
                    mma_bf16_m16n8k16(xc[hn], ah, bl);
                    mma_bf16_m16n8k16(xc[hn], al, bh);
                }
            }
            uint32_t ah[4], al[4];
            split_bf16x2(xc[0][0], xc[0][1], ah[0], al[0]);
            split_bf16x2(xc[0][2], xc[0][3], ah[1], al[1]);
            split_bf16x2(xc[1][0], xc[1][1], ah[2], al[2]);
            split_bf16x2(xc[1][2], xc[1][3], ah[3], al[3]);
#pragma unroll
            for (int hn = 0; hn < 2; ++hn) {
                // B fragment: T_jj[k][c], k = 16 bj + {2t, 2t+1, 2t+8, 2t+9}, c = 16 bj + 8 hn + g
                const int c = bj * 16 + hn * 8 + g, k0 = bj * 16 + 2 * t;
                float bv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int k = k0 + (e & 1) + (e >> 1) * 8;
                    const float v = AT[k * P_AT + c];
                    bv[e] = k > c ? v : (k == c ? 1.0f : 0.0f);
                }
                uint32_t bh[2], bl[2];
                split_bf16x2(bv[0], bv[1], bh[0], bl[0]);
                split_bf16x2(bv[2], bv[3], bh[1], bl[1]);
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                mma_bf16_m16n8k16(d, ah, bh);
                mma_bf16_m16n8k16(d, ah, bl);
                mma_bf16_m16n8k16(d, al, bh);
                const int col = bj * 16 + hn * 8 + 2 * t;
                *reinterpret_cast<float2 *>(AT + r0 * P_AT + col) = make_float2(-d[0], -d[1]);
                *reinterpret_cast<float2 *>(AT + r1 * P_AT + col) = make_float2(-d[2], -d[3]);
            }
        }
        __syncthreads();
    }
    // ---- the A operand of MMA2a / MMA2b as bf16 hi / lo K-major images (128-byte swizzle):
    //      rows 0-63 T' = T diag(beta gamma / |k|), rows 64-127 T'' = T diag(beta). The images
    //      overwrite the A / T array, so every thread first takes its 16 values of T.
    {
        float tv[2][8];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int idx = e * NT + tid, r = idx >> 3, ch = idx & 7;
            // two 16-byte loads of row r (the eight lanes of a row read 256 contiguous bytes)
            const float4 a0 = *reinterpret_cast<const float4 *>(AT + r * P_AT + ch * 8);
            const float4 a1 = *reinterpret_cast<const float4 *>(AT + r * P_AT + ch * 8 + 4);
            const float raw[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int s0 = ch * 8 + j;
                tv[e][j] = (s0 < r) ? raw[j] : (s0 == r ? 1.0f : 0.0f);
            }
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int idx = e * NT + tid, r = idx >> 3, ch = idx & 7;
            uint32_t h1[4], l1[4], h2[4], l2[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int s0 = ch * 8 + 2 * j;
                split_bf16x2(tv[e][2 * j] * sBG[s0], tv[e][2 * j + 1] * sBG[s0 + 1], h1[j], l1[j]);
                split_bf16x2(tv[e][2 * j] * sBeta[s0], tv[e][2 * j + 1] * sBeta[s0 + 1], h2[j], l2[j]);
            }
            const uint32_t off = swz(r, ch);
            *reinterpret_cast<uint4 *>(sm + P_OFF_AHI + off) = make_uint4(h1[0], h1[1], h1[2], h1[3]);
            *reinterpret_cast<uint4 *>(sm + P_OFF_AHI + TILE + off) = make_uint4(h2[0], h2[1], h2[2], h2[3]);
            *reinterpret_cast<uint4 *>(sm + P_OFF_ALO + off) = make_uint4(l1[0], l1[1], l1[2], l1[3]);
            *reinterpret_cast<uint4 *>(sm + P_OFF_ALO + TILE + off) = make_uint4(l2[0], l2[1], l2[2], l2[3]);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // D2a = [T'; T''] K and then D2b = [T'; T''] V (N = 128 each, the hi and lo parts of the A
    // operand accumulated; K and V are the raw bf16 tiles): lanes 0-63 of D2a hold W = T' K, lanes
    // 64-127 of D2b hold U~ = T'' V. They share the tensor-memory columns, so W is read out between.
    if (tid == 0) {
        const uint32_t id2 = idesc_f16(128, false, true, false) | (1u << 7) | (1u << 10);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            mma_f16(tmem + P_TM_D2, kdesc(sm + (kk < 4 ? P_OFF_AHI : P_OFF_ALO) + (kk & 3) * 32),
                    mndesc(sm + P_OFF_KLO + (kk & 3) * 2048, 2 * TILE), id2, kk > 0 ? 1u : 0u);
        tc_commit(bar_mma);
        mmas_issued = 2;
        ok = mbar_wait(bar_mma, 1, status) ? 1 : 0;
    }
    if (!__syncthreads_and(ok)) { failed = true; goto teardown; }
    tc_fence_after();
    if (x < 64) {
        // W row x (fp16): this warp group's 64 key columns are one half of the K-major swizzled
        // [W; Q'] image
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t v[32];
            tmem_ld32(tmem + P_TM_D2 + lane_base + wg * 64 + hh * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float f8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f8[e] = __uint_as_float(v[c * 8 + e]);
                st_h8(item + kWsWQ + wg * 2 * TILE + swz(x, hh * 4 + c), f8);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        ok = mbar_wait(bar_v, 0, status) ? 1 : 0;
        if (ok) {
            const uint32_t id2 = idesc_f16(128, false, true, false) | (1u << 7) | (1u << 10);
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_f16(tmem + P_TM_D2, kdesc(sm + (kk < 4 ? P_OFF_AHI : P_OFF_ALO) + (kk & 3) * 32),
                        mndesc(sm + P_OFF_VLO + (kk & 3) * 2048, 2 * TILE), id2, kk > 0 ? 1u : 0u);
            tc_commit(bar_mma);
            mmas_issued = 3;
            ok = mbar_wait(bar_mma, 0, status) ? 1 : 0;
        }
    }
    if (!__syncthreads_and(ok)) { failed = true; goto teardown; }
    tc_fence_after();
    if (x >= 64) {
        // U~ row s (fp32 [s][i]): this warp group's 64 value columns
        const int s0 = x - 64;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t v[32];
            tmem_ld32(tmem + P_TM_D2 + lane_base + wg * 64 + hh * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4 *>(item + kWsU + s0 * 512 + (wg * 64 + hh * 32 + c * 4) * 4) =
                    make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        }
    }
teardown:
    if (failed && tid == 0) {
        // a wait ran out: before the tensor memory is freed and the CTA exits, wait (bounded) for
        // what this thread issued - the MMAs through one more commit, the tile loads on their
        // barriers (each armed once, so parity 0 names its only phase)
        if (mmas_issued) {
            tc_commit(bar_drain);
            mbar_wait(bar_drain, 0, status);
        }
        if (loads_issued) mbar_wait(bar_tma, 0, status);
        if (v_issued) mbar_wait(bar_v, 0, status);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// ===================================================================================
// Chain kernel: one CTA per (value head, sequence), chunks in order, double-buffered.
// Warps 0-15: element-wise work; warp 16: bulk copies and MMA issue.
// ===================================================================================
// Output pass: 16 element-wise warps, four per tensor-memory lane quarter, each thread one state
// row and 32 of its columns, plus the copy/MMA warp. The chain's critical path per chunk is
// D4 -> U -> D7 -> S update; each chunk's outputs are finished one chunk later, in two halves
// placed where the chain waits for its MMAs (while D7 of the next chunk runs, and while D4 of the
// chunk after it runs), from o kept in two tensor-memory slots.
constexpr int CH_WARPS = 16;
constexpr int CH_WORKERS = CH_WARPS * 32;
constexpr int CH_COLS = 128 / (CH_WARPS / 4);      // state columns per thread
constexpr int CH_TOK = C / (CH_WARPS / 4);         // chunk tokens per thread in U and o
constexpr int CH_THREADS = CH_WORKERS + 32;
// per-chunk buffer: [W; Q'] image (32 KB), P^T hi and lo images (16 KB), the raw bf16 K tile (16 KB)
constexpr int CB_BUF = 65536, CB_WQ = 0, CB_P = 32768, CB_K = 49152;
constexpr int kVecBytes = 272;                     // c[64] and gamma_C of a chunk
constexpr int CH_OFF_VEC = 0;                      // two 512-byte slots
constexpr int CH_OFF_BUF = 1024;                   // two chunk buffers
constexpr int CH_OFF_U = CH_OFF_BUF + 2 * CB_BUF;  // U~ of the current chunk, fp32 [s][i] (one buffer)
constexpr int CH_OFF_STAGE = CH_OFF_U + 32768;     // o staging, [r][i] (bf16 or fp32)
constexpr int CH_OFF_BAR = CH_OFF_STAGE + 64 * 128 * 4;
constexpr int CH_SMEM = CH_OFF_BAR + 128 + 1024;
static_assert(CH_SMEM <= 232448, "chain shared memory");
// Fused variant (gated RMSNorm + NVFP4 encode of each chunk's o rows): o staged in bf16; z tiles
// of three chunks in flight (a chunk's tile is read while the chain works on the next chunk).
constexpr int CHF_THREADS = CH_THREADS;
constexpr int CHF_STAGE = 64 * 128 * 2;            // one chunk's o rows, bf16 [r][i]
constexpr int CHF_OFF_Z = CH_OFF_STAGE + CHF_STAGE;
constexpr int CHF_ZBYTES = 2 * TILE;               // [z_lo][z_hi], 64 tokens x 64 values each
constexpr int CHF_OFF_RTAB = CHF_OFF_Z + 3 * CHF_ZBYTES;
constexpr int CHF_OFF_BAR = CHF_OFF_RTAB + 128 * 4;
constexpr int CHF_SMEM = CHF_OFF_BAR + 128 + 1024;
static_assert(CHF_SMEM <= 232448, "fused chain shared memory");
static_assert(CHF_OFF_Z % 1024 == 0 && CB_K % 1024 == 0 && CB_BUF % 1024 == 0 && CH_OFF_BUF % 1024 == 0,
              "TMA destination alignment");
static_assert(kWsItem % 1024 == 0 && kWsP % 1024 == 0 && kWsU % 16 == 0 && kWsVec % 16 == 0,
              "1024-byte aligned operand tiles, 16-byte aligned bulk sources");
// tensor memory: D4 (U's state term), o in two slots (chunk c in slot c & 1: MMA5a, then the
// intra-chunk part accumulated onto it), D7 (state update), the fp16 copy of S0, U as bf16 hi /
// lo A operands, U diag(c) as bf16 hi / lo
constexpr uint32_t C_TM_D4 = 0, C_TM_O = 64, C_TM_D7 = 192, C_TM_SA = 320, C_TM_UA = 384, C_TM_UCA = 448;

// kind::f16 instruction descriptor bits for bf16 A and B
constexpr uint32_t kIdescBf16 = (1u << 7) | (1u << 10);

// tcgen05.mma kind::f16 with the A operand in tensor memory (M = 128, K-major rows on lanes).
__device__ __forceinline__ void mma_f16_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

// Barrier among the output pass's element-wise threads only (named barrier 1), with an AND vote.
__device__ __forceinline__ int workers_and(int pred) {
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %1, 0;\n\t"
        "barrier.cta.red.and.pred q, 1, %2, p;\n\tselp.s32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(pred), "n"(CH_WORKERS)
        : "memory");
    return r;
}
__device__ __forceinline__ void workers_sync() { asm volatile("barrier.cta.sync 2, %0;" ::"n"(CH_WORKERS) : "memory"); }

// Chain modes: the full chain with outputs from a segment's true start state; a segment's
// state from S0 (first segment) or zero, with no outputs; a segment's transition matrix,
// the state from the identity with U~ taken as zero (its final state is the map S -> S M).
enum ChainMode { kChainFull = 0, kChainState = 1, kChainTransition = 2 };

struct ChainParams {
    CUtensorMap kmap;      // k [T, Hk, 128] bf16, boxes of 64 values x 64 tokens (the state update's B)
    CUtensorMap zmap;      // fused output pass: z [T, Hv, 128] bf16, boxes of 64 values x 64 tokens
    const int32_t *cu_seqlens;
    int32_t T, num_seqs, Hk, Hv, slots, seg_chunks, seg_slots, mode_base, out_bf16;
    const float *S0g;
    float *S_out;
    void *o;               // may be null in the fused output pass
    const uint8_t *ws;     // per-chunk operand items
    uint8_t *ws_seg;       // per-segment B (fp32), M (fp16 hi/lo operand images), start state (fp32)
    int *status;
    const float *norm_w;   // fused: RMSNorm weight [128], eps, NVFP4 encode scale and outputs
    float eps, gs;
    uint8_t *xq, *xs;
};
constexpr size_t kSegItem = kSegItemBytes;
constexpr size_t kSegB = 0, kSegMhi = 65536, kSegMlo = 98304, kSegS = 131072;
static_assert(kSegMlo == kSegMhi + 32768, "the combine reads M_lo right after M_hi");

// Segment states (B, start states) are stored lane-interleaved: the 16-byte group c4 of the
// 64-column half wg of row i sits at ((wg * 16 + c4) * 128 + i) * 16, so that the thread owning
// (row i, half wg) and its 31 neighbours touch 512 contiguous bytes per access.
__device__ __forceinline__ size_t ilv_off(int row, int wg, int c4) {
    return ((size_t)((wg * 16 + c4) * 128 + row)) * 16;
}
__device__ __forceinline__ void ilv_load(const uint8_t *base, int row, int wg, float (&S)[64]) {
#pragma unroll
    for (int c4 = 0; c4 < 16; ++c4) {
        const float4 x = *reinterpret_cast<const float4 *>(base + ilv_off(row, wg, c4));
        S[4 * c4] = x.x; S[4 * c4 + 1] = x.y; S[4 * c4 + 2] = x.z; S[4 * c4 + 3] = x.w;
    }
}
__device__ __forceinline__ void ilv_store(uint8_t *base, int row, int wg, const float (&S)[64]) {
#pragma unroll
    for (int c4 = 0; c4 < 16; ++c4)
        *reinterpret_cast<float4 *>(base + ilv_off(row, wg, c4)) =
            make_float4(S[4 * c4], S[4 * c4 + 1], S[4 * c4 + 2], S[4 * c4 + 3]);
}
// The 32-column quarter cq of row i (the same layout: 16-byte group cq * 8 + c4).
__device__ __forceinline__ void ilv_load32(const uint8_t *base, int row, int cq, float (&S)[32]) {
#pragma unroll
    for (int c4 = 0; c4 < 8; ++c4) {
        const float4 x = *reinterpret_cast<const float4 *>(base + ((size_t)((cq * 8 + c4) * 128 + row)) * 16);
        S[4 * c4] = x.x; S[4 * c4 + 1] = x.y; S[4 * c4 + 2] = x.z; S[4 * c4 + 3] = x.w;
    }
}
// A row-major 128 x 128 fp32 state through shared memory (rows padded to 528 bytes, so both the
// coalesced side and the row-per-thread side are free of bank conflicts).
constexpr int kStgPitch = 528;

// FUSED: the outputs are the gated RMSNorm of each chunk's o rows, NVFP4-encoded (o itself only
// when P.o is set); otherwise o.
template <bool FUSED>
__global__ void __launch_bounds__(FUSED ? CHF_THREADS : CH_THREADS, 1)
gdn_chunk_chain_kernel(const __grid_constant__ ChainParams P) {
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + (FUSED ? CHF_OFF_BAR : CH_OFF_BAR));
    // full[2]: chunk copies; full_u: U~; bar_u / bar_s: D4 / D7 done; bar_uready / bar_sready: the
    // element-wise warps have stored U / S0; bar_o[2]: a chunk's o complete (per o slot)
    uint64_t *full = bars, *full_u = bars + 2, *bar_u = bars + 3, *bar_s = bars + 4, *bar_uready = bars + 5,
             *bar_sready = bars + 6, *bar_drain = bars + 7, *bar_o = bars + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 10);

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int h = blockIdx.x, id = blockIdx.y;
    const int T = P.T, Hv = P.Hv, SEG = P.seg_chunks;
    const int hk = h / (Hv / P.Hk);
    int n = 0, t_begin = 0, t_end = T;
    if (P.cu_seqlens) {
        int lo = 0, hi = P.num_seqs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) / 2;
            if (P.cu_seqlens[mid] / (C * SEG) + mid <= id) lo = mid;
            else hi = mid - 1;
        }
        n = lo;
        t_begin = P.cu_seqlens[n];
        t_end = P.cu_seqlens[n + 1];
    }
    const int nch_seq = (t_end - t_begin + C - 1) / C;
    const int nseg = (nch_seq + SEG - 1) / SEG;
    const int pseg = id - (t_begin / (C * SEG) + n);
    if (pseg < 0 || pseg >= (nseg > 0 ? nseg : 1)) return;   // a slot no segment uses
    const int c_first = pseg * SEG;
    const int nchunks = max(0, min(nch_seq, c_first + SEG) - c_first);
    const bool last_seg = pseg >= nseg - 1;
    const uint8_t *seg_item = P.ws_seg + ((size_t)h * P.seg_slots + id) * kSegItem;
    const int32_t slots = P.slots;
    const float *S0g = P.S0g;
    const int slot0 = t_begin / C + n + c_first;
    const uint8_t *ws_h = P.ws + (size_t)h * slots * kWsItem;
    int *status = P.status;

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(full_u, 1);
        mbar_init(bar_u, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_uready, CH_WARPS);
        mbar_init(bar_sready, CH_WARPS);
        mbar_init(bar_drain, 1);
        mbar_init(&bar_o[0], 1);
        mbar_init(&bar_o[1], 1);
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

    if (warp == CH_WARPS) {
        // ------------------------------------------------ copy + MMA issue (one thread)
        if (lane == 0) {
            // issued phases per barrier, for the drain on the failure path
            int n_full[2] = {0, 0}, n_u = 0, n_mma = 0;
            bool ok = true;
            auto issue_chunk = [&](int c) {
                const int b = c & 1;
                uint64_t *bar = &full[b];
                uint8_t *buf = sm + CH_OFF_BUF + b * CB_BUF;
                const uint8_t *item = ws_h + (size_t)(slot0 + c) * kWsItem;
                const int t0c = t_begin + (c_first + c) * C;
                mbar_arrive_expect_tx(bar, CB_K + 2 * TILE + kVecBytes + (FUSED ? CHF_ZBYTES : 0));
                bulk_load(buf + CB_WQ, item + kWsWQ, 4 * TILE, bar);
                bulk_load(buf + CB_P, item + kWsP, 2 * TILE, bar);
                bulk_load(sm + CH_OFF_VEC + b * 512, item + kWsVec, kVecBytes, bar);
                tma_load_3d(buf + CB_K, &P.kmap, bar, 0, hk, t0c);
                tma_load_3d(buf + CB_K + TILE, &P.kmap, bar, 64, hk, t0c);
                if constexpr (FUSED) {   // this chunk's z rows, two boxes of 64 values
                    uint8_t *zb = sm + CHF_OFF_Z + (c % 3) * CHF_ZBYTES;
                    tma_load_3d(zb, &P.zmap, bar, 0, h, t0c);
                    tma_load_3d(zb + TILE, &P.zmap, bar, 64, h, t0c);
                }
                ++n_full[b];
            };
            auto issue_u = [&](int c) {
                mbar_arrive_expect_tx(full_u, 4 * TILE);
                bulk_load(sm + CH_OFF_U, ws_h + (size_t)(slot0 + c) * kWsItem + kWsU, 4 * TILE, full_u);
                ++n_u;
            };
            // with a caller's initial state the element-wise warps stage it over buffer 1 and the
            // head of the U~ buffer: the first U~ load waits until they have released it (bar_sready)
            const bool s0_staged = pseg == 0 && S0g;
            if (nchunks > 0) {
                issue_chunk(0);
                if (!s0_staged) issue_u(0);
            }
            const uint32_t id4 = idesc_f16(64, false, false, false);
            const uint32_t id7 = idesc_f16(128, false, true, false) | kIdescBf16;
            const uint32_t id5 = idesc_f16(64, false, true, false) | kIdescBf16;
            for (int c = 0; c < nchunks; ++c) {
                const int b = c & 1;
                const uint8_t *buf = sm + CH_OFF_BUF + b * CB_BUF;
                if (!(ok = mbar_wait(&full[b], (uint32_t)((c >> 1) & 1), status))) break;
                // S0 of chunk c is in tensor memory, and the workers have read chunk c - 2's o
                if (!(ok = mbar_wait(bar_sready, (uint32_t)(c & 1), status))) break;
                if (c == 0 && s0_staged) issue_u(0);
                tc_fence_after();
                // D4 = S0 W^T (fp16; B: the W rows of the [W; Q'] image, K = 128 key columns),
                // committed alone; then o = S0 Q'^T into o slot b (both read the S0 copy before
                // D7's commit, after which the state update rewrites it)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_f16_ts(tmem + C_TM_D4, tmem + C_TM_SA + kk * 8,
                               kdesc(buf + CB_WQ + (kk < 4 ? 0 : 2 * TILE) + (kk & 3) * 32), id4, kk > 0);
                tc_commit(bar_u);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_f16_ts(tmem + C_TM_O + b * 64, tmem + C_TM_SA + kk * 8,
                               kdesc(buf + CB_WQ + (kk < 4 ? TILE : 3 * TILE) + (kk & 3) * 32), id4, kk > 0);
                ++n_mma;
                if (c + 1 < nchunks) {
                    // buffer (c + 1) & 1 was chunk c - 1's: its MMAs are done once its o is, its
                    // readers among the workers (c, gamma_C, the z tile) before they handed on S0
                    if (c > 0 && !(ok = mbar_wait(&bar_o[(c - 1) & 1], (uint32_t)(((c - 1) >> 1) & 1), status))) break;
                    fence_proxy_async_smem();
                    issue_chunk(c + 1);
                }
                if (!(ok = mbar_wait(bar_uready, (uint32_t)(c & 1), status))) break;
                if (c + 1 < nchunks) {   // every worker has read this chunk's U~
                    fence_proxy_async_smem();
                    issue_u(c + 1);
                }
                tc_fence_after();
                // D7 = (U diag(c))^T K with U diag(c) as bf16 hi + lo and the raw bf16 K (MN-major,
                // two blocks of 64 keys), committed alone: the state update waits only for it
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16_ts(tmem + C_TM_D7, tmem + C_TM_UCA + part * 32 + kk * 8,
                                   mndesc(buf + CB_K + kk * 2048, TILE), id7, (part | kk) ? 1u : 0u);
                tc_commit(bar_s);
                // o += U^T P^T with U and P^T as bf16 hi / lo (hi hi + hi lo + lo hi)
#pragma unroll
                for (int part = 0; part < 3; ++part)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16_ts(tmem + C_TM_O + b * 64, tmem + C_TM_UA + (part == 2 ? 32 : 0) + kk * 8,
                                   mndesc(buf + CB_P + (part == 1 ? TILE : 0) + kk * 2048, TILE), id5, 1u);
                tc_commit(&bar_o[b]);
            }
            if (!ok) {
                // a wait ran out: wait (bounded) for this thread's MMAs and for the latest phase of
                // every barrier it armed before the CTA frees its tensor memory and exits
                if (n_mma) {
                    tc_commit(bar_drain);
                    mbar_wait(bar_drain, 0, status);
                }
                for (int b = 0; b < 2; ++b)
                    if (n_full[b]) mbar_wait(&full[b], (uint32_t)((n_full[b] - 1) & 1), status);
                if (n_u) mbar_wait(full_u, (uint32_t)((n_u - 1) & 1), status);
            }
        }
    } else {
        // ------------------------------------------------ element-wise work (16 warps)
        const int cq = warp / 4;                  // column quarter: state columns 32 cq .. 32 cq + 31
        const int row = (warp % 4) * 32 + lane;   // TMEM lane == value index i
        const uint32_t lane_base = ((uint32_t)((warp % 4) * 32)) << 16;
        float S[CH_COLS];   // S[i][32 cq .. 32 cq + 31], fp32
        // fused: this thread's eight RMSNorm weights (16 threads per o row) and the encoder table
        const int lr = tid & 15, ecol = lr * 8;
        f2_t w2[4];
        if constexpr (FUSED) {
#pragma unroll
            for (int k = 0; k < 4; ++k) w2[k] = f2(P.norm_w[ecol + 2 * k], P.norm_w[ecol + 2 * k + 1]);
            nvfp4_fill_r_tab(reinterpret_cast<float *>(sm + CHF_OFF_RTAB), P.gs, tid);
        }
        const int out_bf16 = FUSED ? 1 : P.out_bf16;
        uint8_t *stage = sm + CH_OFF_STAGE;
        // Outputs of chunk cc, first half: its o (done once bar_o has landed) out of tensor memory
        // into the staging area as rows [r][i], then rows 0-31 finished (gated RMSNorm + NVFP4
        // encode, or the o stores); the z values of the second half are kept in registers, so that
        // the z tile is free when this half is done. Returns false if the wait ran out.
        uint4 z_keep = make_uint4(0u, 0u, 0u, 0u);
        auto out_rows = [&](int cc, int pass, const uint4 &zu) {
            const int t0e = t_begin + (c_first + cc) * C;
            const int Le = min(C, t_end - t0e);
            if constexpr (FUSED) {
                const int r = pass * (CH_WORKERS / 16) + (tid >> 4);
                const uint4 ou = *reinterpret_cast<const uint4 *>(stage + r * (D * 2) + ecol * 2);
                const float *r_tab = reinterpret_cast<const float *>(sm + CHF_OFF_RTAB);
                const f2_t o2[4] = {bf16x2_to_f2(ou.x), bf16x2_to_f2(ou.y), bf16x2_to_f2(ou.z), bf16x2_to_f2(ou.w)};
                const f2_t z2[4] = {bf16x2_to_f2(zu.x), bf16x2_to_f2(zu.y), bf16x2_to_f2(zu.z), bf16x2_to_f2(zu.w)};
                f2_t y2[4];
                gated_row8<16>(o2, z2, w2, 1.0f / (float)D, P.eps, y2);
                uint32_t packed, sb;
                nvfp4_encode_row8(y2, P.gs, r_tab, packed, sb);
                if (r < Le) {
                    const size_t base = ((size_t)(t0e + r) * Hv + h) * D + ecol;
                    reinterpret_cast<uint32_t *>(P.xq)[base / 8] = packed;
                    if ((lr & 1) == 0) P.xs[base / 16] = (uint8_t)sb;
                    if (P.o) *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(P.o) + base * 2) = ou;
                }
            } else {
                const int row_bytes = out_bf16 ? D * 2 : D * 4;
                const int per_row = row_bytes / 16;
                uint8_t *ob = static_cast<uint8_t *>(P.o);
                const int r_lo = pass * 32, r_hi = min(Le, r_lo + 32);
                for (int e = r_lo * per_row + tid; e < r_hi * per_row; e += CH_WORKERS) {
                    const int r = e / per_row, chn = e % per_row;
                    const uint4 val = *reinterpret_cast<const uint4 *>(stage + r * row_bytes + chn * 16);
                    *reinterpret_cast<uint4 *>(ob + (((size_t)(t0e + r) * Hv + h) * D) * (row_bytes / D) + chn * 16) = val;
                }
            }
        };
        auto out_first = [&](int cc) -> bool {
            int ok = 1;
            if (tid == 0) ok = mbar_wait(&bar_o[cc & 1], (uint32_t)((cc >> 1) & 1), status) ? 1 : 0;
            if (!workers_and(ok)) return false;
            tc_fence_after();
            uint32_t a5[16];
            tmem_ld16(tmem + C_TM_O + (cc & 1) * 64 + lane_base + cq * CH_TOK, a5);
            tmem_ld_wait();
            if (out_bf16) {
                __nv_bfloat16 *st = reinterpret_cast<__nv_bfloat16 *>(stage);
#pragma unroll
                for (int j = 0; j < CH_TOK; ++j) st[(cq * CH_TOK + j) * D + row] = __float2bfloat16_rn(__uint_as_float(a5[j]));
            } else {
                float *st = reinterpret_cast<float *>(stage);
#pragma unroll
                for (int j = 0; j < CH_TOK; ++j) st[(cq * CH_TOK + j) * D + row] = __uint_as_float(a5[j]);
            }
            workers_sync();
            uint4 zu0 = make_uint4(0u, 0u, 0u, 0u);
            if constexpr (FUSED) {
                const uint8_t *zt = sm + CHF_OFF_Z + (cc % 3) * CHF_ZBYTES;
                const int r0 = tid >> 4, r1 = (CH_WORKERS / 16) + (tid >> 4);
                zu0 = *reinterpret_cast<const uint4 *>(zt + (ecol >> 6) * TILE + swz(r0, (ecol & 63) >> 3));
                z_keep = *reinterpret_cast<const uint4 *>(zt + (ecol >> 6) * TILE + swz(r1, (ecol & 63) >> 3));
            }
            out_rows(cc, 0, zu0);
            return true;
        };
        if (pseg == 0 && S0g) {
            // the caller's row-major initial state, staged over chunk buffer 1 and the head of the
            // U~ buffer (neither is loaded before the workers release S0 through bar_sready)
            const float4 *src = reinterpret_cast<const float4 *>(S0g + ((size_t)n * Hv + h) * D * D);
            uint8_t *stg = sm + CH_OFF_BUF + CB_BUF;
#pragma unroll 4
            for (int e = 0; e < 4096 / CH_WORKERS; ++e) {
                const int f = e * CH_WORKERS + tid;
                *reinterpret_cast<float4 *>(stg + (f >> 5) * kStgPitch + (f & 31) * 16) = src[f];
            }
            workers_sync();
#pragma unroll
            for (int c4 = 0; c4 < CH_COLS / 4; ++c4) {
                const float4 x = *reinterpret_cast<const float4 *>(stg + row * kStgPitch + cq * CH_COLS * 4 + c4 * 16);
                S[4 * c4] = x.x; S[4 * c4 + 1] = x.y; S[4 * c4 + 2] = x.z; S[4 * c4 + 3] = x.w;
            }
            workers_sync();
        } else if (pseg > 0) {
            ilv_load32(seg_item + kSegS, row, cq, S);
        } else {
#pragma unroll
            for (int c = 0; c < CH_COLS; ++c) S[c] = 0.0f;
        }
        // fp16 copy of S as an A operand: row i on lane i, key index j two per column (one slot:
        // the MMAs that read it have completed before the workers rewrite it)
        auto store_S = [&]() {
            uint32_t pk[16];
#pragma unroll
            for (int w = 0; w < 16; ++w) pk[w] = pack_h2(S[2 * w], S[2 * w + 1]);
            tmem_st16(tmem + lane_base + C_TM_SA + cq * 16, pk);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_sready);
        };
        store_S();

        bool alive = true;
        for (int c = 0; c < nchunks; ++c) {
            const int t0 = t_begin + (c_first + c) * C;
            const int L = min(C, t_end - t0);
            const int b = c & 1;
            const float *vecb = reinterpret_cast<const float *>(sm + CH_OFF_VEC + b * 512);
            const uint32_t ph = (uint32_t)(c & 1);

            int ok = 1;
            if (tid == 0)
                ok = (mbar_wait(&full[b], (uint32_t)((c >> 1) & 1), status) && mbar_wait(bar_u, ph, status) &&
                      mbar_wait(full_u, ph, status))
                         ? 1 : 0;
            if (!workers_and(ok)) { alive = false; break; }
            tc_fence_after();
            {
                // U^T = U~^T - D4 (fp32) for tokens 16 cq .. + 15 of this row, then U and U diag(c)
                // as bf16 hi / lo A operands (packed f32x2 arithmetic, eight tokens at a time)
                const float *ut = reinterpret_cast<const float *>(sm + CH_OFF_U);
                const f2_t neg1 = f2(-1.0f, -1.0f);
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const int sb = cq * CH_TOK + part * 8;
                    f2_t u2[4], c2[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const int s0 = sb + 2 * w;
                        u2[w] = f2(s0 < L ? ut[s0 * D + row] : 0.0f, s0 + 1 < L ? ut[(s0 + 1) * D + row] : 0.0f);
                        const float2 cc = *reinterpret_cast<const float2 *>(vecb + s0);
                        c2[w] = f2(cc.x, cc.y);
                    }
                    uint32_t r8[8];
                    tmem_ld8(tmem + C_TM_D4 + lane_base + sb, r8);
                    tmem_ld_wait();
                    uint32_t uh[4], ul[4], ch[4], cl[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const int s0 = sb + 2 * w;
                        f2_t u = fma2(f2(__uint_as_float(r8[2 * w]), __uint_as_float(r8[2 * w + 1])), neg1, u2[w]);
                        if (s0 >= L) u = f2(0.0f, 0.0f);
                        else if (s0 + 1 >= L) u = f2(f2lo(u), 0.0f);
                        const f2_t uc = mul2(u, c2[w]);
                        split_bf16x2(f2lo(u), f2hi(u), uh[w], ul[w]);
                        split_bf16x2(f2lo(uc), f2hi(uc), ch[w], cl[w]);
                    }
                    tmem_st4(tmem + lane_base + C_TM_UA + sb / 2, uh);
                    tmem_st4(tmem + lane_base + C_TM_UA + 32 + sb / 2, ul);
                    tmem_st4(tmem + lane_base + C_TM_UCA + sb / 2, ch);
                    tmem_st4(tmem + lane_base + C_TM_UCA + 32 + sb / 2, cl);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_uready);
            }
            // while D7 runs: the first half of chunk c - 1's outputs
            if (c > 0 && !out_first(c - 1)) { alive = false; break; }
            if (tid == 0) ok = mbar_wait(bar_s, ph, status) ? 1 : 0;
            if (!workers_and(ok)) { alive = false; break; }
            tc_fence_after();
            {
                // S <- gamma_C S + D7 for this quarter, handed on at once
                const float gC = vecb[64];
                const f2_t g2 = f2(gC, gC);
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    uint32_t r7[16];
                    tmem_ld16(tmem + C_TM_D7 + lane_base + cq * CH_COLS + part * 16, r7);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; j += 2) {
                        const int jj = part * 16 + j;
                        const f2_t s2 = fma2(g2, f2(S[jj], S[jj + 1]), f2(__uint_as_float(r7[j]), __uint_as_float(r7[j + 1])));
                        S[jj] = f2lo(s2);
                        S[jj + 1] = f2hi(s2);
                    }
                }
                store_S();   // S0 of chunk c + 1; releases the MMA warp
            }
            // while D4 of chunk c + 1 runs: the second half of chunk c - 1's outputs
            if (c > 0) out_rows(c - 1, 1, z_keep);
        }
        // the last chunk's outputs
        if (alive && nchunks > 0) {
            if (!out_first(nchunks - 1)) alive = false;
            else out_rows(nchunks - 1, 1, z_keep);
        }
        if (alive && last_seg && P.S_out) {
            // every MMA is done (the last o was waited for): the chunk buffers are free for staging
            // the final state
            workers_sync();
            uint8_t *stg = sm + CH_OFF_BUF;
#pragma unroll
            for (int c4 = 0; c4 < CH_COLS / 4; ++c4)
                *reinterpret_cast<float4 *>(stg + row * kStgPitch + cq * CH_COLS * 4 + c4 * 16) =
                    make_float4(S[4 * c4], S[4 * c4 + 1], S[4 * c4 + 2], S[4 * c4 + 3]);
            workers_sync();
            float4 *dst = reinterpret_cast<float4 *>(P.S_out + ((size_t)n * Hv + h) * D * D);
#pragma unroll 4
            for (int e = 0; e < 4096 / CH_WORKERS; ++e) {
                const int f = e * CH_WORKERS + tid;
                dst[f] = *reinterpret_cast<const float4 *>(stg + (f >> 5) * kStgPitch + (f & 31) * 16);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}


// ===================================================================================
// Lean chain kernel for the state and transition passes (no outputs). A buffer holds W, the raw
// K tile and the chunk's c and gamma_C; U~ (state pass only) has one buffer of its own, refilled
// as soon as every thread has read it. 256 threads, thread 0 also issuing the copies and the
// MMAs; 256 tensor-memory columns and at most 128 registers, so that two CTAs share an SM. The
// two passes of a segment are adjacent blocks (blockIdx.x = 2 h + pass) and the two value heads
// of a key head are neighbours too, so W and K reach the four CTAs from L2 after one HBM read.
// ===================================================================================
constexpr int CL_W = 0, CL_K = 2 * TILE, CL_VEC = 4 * TILE;
constexpr int CL_BUF = 4 * TILE + 1024;
constexpr int CL_U = 2 * CL_BUF;
constexpr int CL_OFF_BAR = CL_U + 4 * TILE;
constexpr int CL_SMEM = CL_OFF_BAR + 128 + 1024;
static_assert(2 * (CL_SMEM + 1024) <= 233472, "two lean chain CTAs per SM");
static_assert(CL_BUF % 1024 == 0 && CL_K % 1024 == 0, "TMA destination alignment");
// D4 (64 columns) and D7 (128) share columns: D4 is read out before MMA7 is issued
constexpr uint32_t CL_TM_D4 = 0, CL_TM_D7 = 0, CL_TM_SA = 128, CL_TM_UCA = 192;

__global__ void __launch_bounds__(NT, 2)
gdn_chunk_lean_kernel(const __grid_constant__ ChainParams P) {
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + CL_OFF_BAR);
    // full[2]: chunk copies; full_u: U~; bar45 / bar67: MMA completion; bar_s / bar_u: the eight
    // warps have stored S0 / U into tensor memory (one arrival per warp); bar_drain: failure path
    uint64_t *full = bars, *full_u = bars + 2, *bar45 = bars + 3, *bar67 = bars + 4, *bar_s = bars + 5,
             *bar_u = bars + 6, *bar_drain = bars + 7;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 8);

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int h = blockIdx.x >> 1, id = blockIdx.y, mode = kChainState + (int)(blockIdx.x & 1);
    const int T = P.T, Hv = P.Hv, SEG = P.seg_chunks;
    const int hk = h / (Hv / P.Hk);
    int n = 0, t_begin = 0, t_end = T;
    if (P.cu_seqlens) {
        int lo = 0, hi = P.num_seqs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) / 2;
            if (P.cu_seqlens[mid] / (C * SEG) + mid <= id) lo = mid;
            else hi = mid - 1;
        }
        n = lo;
        t_begin = P.cu_seqlens[n];
        t_end = P.cu_seqlens[n + 1];
    }
    const int nch_seq = (t_end - t_begin + C - 1) / C;
    const int nseg = (nch_seq + SEG - 1) / SEG;
    const int pseg = id - (t_begin / (C * SEG) + n);
    // the last segment has no successor; the transition of the first is never needed
    if (pseg < 0 || pseg >= nseg - 1) return;
    if (mode == kChainTransition && pseg == 0) return;
    const int c_first = pseg * SEG;
    const int nchunks = max(0, min(nch_seq, c_first + SEG) - c_first);
    const uint8_t *seg_item = P.ws_seg + ((size_t)h * P.seg_slots + id) * kSegItem;
    const int slot0 = t_begin / C + n + c_first;
    const uint8_t *ws_h = P.ws + (size_t)h * P.slots * kWsItem;
    int *status = P.status;
    const bool with_u = mode == kChainState;

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(full_u, 1);
        mbar_init(bar45, 1);
        mbar_init(bar67, 1);
        mbar_init(bar_s, 8);
        mbar_init(bar_u, 8);
        mbar_init(bar_drain, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // issued phases per barrier (thread 0), for the drain on the failure path
    int n_full[2] = {0, 0}, n_u = 0, n_mma = 0;
    auto issue_chunk = [&](int c) {
        const int b = c & 1;
        uint64_t *bar = &full[b];
        uint8_t *dst = sm + b * CL_BUF;
        const uint8_t *item = ws_h + (size_t)(slot0 + c) * kWsItem;
        const int t0c = t_begin + (c_first + c) * C;
        mbar_arrive_expect_tx(bar, 4 * TILE + kVecBytes);
        bulk_load(dst + CL_W, item + kWsWQ, TILE, bar);
        bulk_load(dst + CL_W + TILE, item + kWsWQ + 2 * TILE, TILE, bar);
        tma_load_3d(dst + CL_K, &P.kmap, bar, 0, hk, t0c);
        tma_load_3d(dst + CL_K + TILE, &P.kmap, bar, 64, hk, t0c);
        bulk_load(dst + CL_VEC, item + kWsVec, kVecBytes, bar);
        ++n_full[b];
    };
    auto issue_u = [&](int c) {
        mbar_arrive_expect_tx(full_u, 4 * TILE);
        bulk_load(sm + CL_U, ws_h + (size_t)(slot0 + c) * kWsItem + kWsU, 4 * TILE, full_u);
        ++n_u;
    };
    if (tid == 0) {
        if (nchunks > 0) issue_chunk(0);
        if (nchunks > 1) issue_chunk(1);
        if (with_u && nchunks > 0) issue_u(0);
    }

    const int wg = warp / 4;
    const int row = (warp % 4) * 32 + lane;   // TMEM lane == value index i
    const uint32_t lane_base = ((uint32_t)((warp % 4) * 32)) << 16;
    float S[64];   // S[i][64 wg .. 64 wg + 63], fp32
    if (mode == kChainState && pseg == 0 && P.S0g) {
        const float *src = P.S0g + (((size_t)n * Hv + h) * D + row) * D + 64 * wg;
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
            const float4 xv = *reinterpret_cast<const float4 *>(src + c);
            S[c] = xv.x; S[c + 1] = xv.y; S[c + 2] = xv.z; S[c + 3] = xv.w;
        }
    } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) S[c] = (mode == kChainTransition && row == 64 * wg + c) ? 1.0f : 0.0f;
    }
    // fp16 copy of S as the A operand of MMA45: row i on lane i, key index j two per column;
    // each warp signals bar_s once its part is in tensor memory
    auto store_S = [&]() {
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            uint32_t pk[16];
#pragma unroll
            for (int w = 0; w < 16; ++w) pk[w] = pack_h2(S[part * 32 + 2 * w], S[part * 32 + 2 * w + 1]);
            tmem_st16(tmem + lane_base + CL_TM_SA + wg * 32 + part * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_s);
    };
    // Every thread waits on the MMA barriers itself. A wait that runs out marks the thread
    // dead: it records the status, stops waiting and issuing, and still takes every later step,
    // so that no barrier is left short of arrivals.
    bool dead = false;
    auto wait = [&](uint64_t *bar, uint32_t parity) {
        if (!dead && !mbar_wait(bar, parity, status)) dead = true;
    };
    store_S();

    const uint32_t id45 = idesc_f16(64, false, false, false);
    const uint32_t id7 = idesc_f16(128, false, true, false) | kIdescBf16;
    for (int c = 0; c < nchunks; ++c) {
        const int L = min(C, t_end - (t_begin + (c_first + c) * C));
        const int b = c & 1;
        const uint32_t ph = (uint32_t)(c & 1);
        const uint8_t *buf = sm + b * CL_BUF;
        const float *vecb = reinterpret_cast<const float *>(buf + CL_VEC);
        if (tid == 0) {
            wait(bar_s, ph);                                // S0 of this chunk is in tensor memory
            wait(&full[b], (uint32_t)((c >> 1) & 1));
            if (!dead) {
                tc_fence_after();
                // D4 = S0 W^T   (B: W, K-major rows s, K = 128 key columns in two halves)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_f16_ts(tmem + CL_TM_D4, tmem + CL_TM_SA + kk * 8,
                               kdesc(buf + CL_W + (kk < 4 ? 0 : TILE) + (kk & 3) * 32), id45, kk > 0);
                tc_commit(bar45);
                ++n_mma;
            }
        }
        wait(&full[b], (uint32_t)((c >> 1) & 1));           // this chunk's c and gamma_C are visible
        if (with_u) wait(full_u, ph);
        wait(bar45, ph);
        tc_fence_after();
        const float gC = vecb[64];
        {
            // U^T = U~^T - D4 (the transition pass takes U~ = 0), scaled per token by c, as the bf16
            // hi / lo A operands of MMA7, 8 tokens at a time
            const float *ut = reinterpret_cast<const float *>(sm + CL_U);
#pragma unroll
            for (int part = 0; part < 4; ++part) {
                float u8v[8];
#pragma unroll
                for (int w = 0; w < 8; ++w) u8v[w] = with_u ? ut[(wg * 32 + part * 8 + w) * D + row] : 0.0f;
                uint32_t r8[8];
                tmem_ld8(tmem + CL_TM_D4 + lane_base + wg * 32 + part * 8, r8);
                tmem_ld_wait();
                uint32_t uh[4], ul[4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const int s0 = wg * 32 + part * 8 + 2 * w;
                    const float u0 = (s0 < L) ? u8v[2 * w] - __uint_as_float(r8[2 * w]) : 0.0f;
                    const float u1 = (s0 + 1 < L) ? u8v[2 * w + 1] - __uint_as_float(r8[2 * w + 1]) : 0.0f;
                    split_bf16x2(u0 * vecb[s0], u1 * vecb[s0 + 1], uh[w], ul[w]);
                }
                tmem_st4(tmem + lane_base + CL_TM_UCA + wg * 16 + part * 4, uh);
                tmem_st4(tmem + lane_base + CL_TM_UCA + 32 + wg * 16 + part * 4, ul);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_u);
        }
        if (tid == 0) {
            wait(bar_u, ph);                                // U is in tensor memory, D4 and U~ are consumed
            if (!dead) {
                if (with_u && c + 1 < nchunks) {
                    fence_proxy_async_smem();
                    issue_u(c + 1);
                }
                tc_fence_after();
                // D7 = (U diag(c))^T K   (A: bf16 hi then lo; B: the raw K tile, MN-major blocks of
                // 64 keys, K = 64 tokens)
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16_ts(tmem + CL_TM_D7, tmem + CL_TM_UCA + part * 32 + kk * 8,
                                   mndesc(buf + CL_K + kk * 2048, TILE), id7, (part | kk) ? 1u : 0u);
                tc_commit(bar67);
                ++n_mma;
            }
        }
        wait(bar67, ph);
        // this buffer's readers (both MMAs, every thread's c and gamma_C) are done: refill it
        if (tid == 0 && !dead && c + 2 < nchunks) {
            fence_proxy_async_smem();
            issue_chunk(c + 2);
        }
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t r7[16];
            tmem_ld16(tmem + CL_TM_D7 + lane_base + wg * 64 + q * 16, r7);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) S[q * 16 + j] = gC * S[q * 16 + j] + __uint_as_float(r7[j]);
        }
        store_S();
    }
    const bool alive = __syncthreads_and(!dead);
    if (!alive && tid == 0) {
        // a wait ran out somewhere: wait (bounded) for this thread's MMAs and for the latest phase
        // of every barrier it armed before the tensor memory is freed
        if (n_mma) {
            tc_commit(bar_drain);
            mbar_wait(bar_drain, 0, status);
        }
        for (int b = 0; b < 2; ++b)
            if (n_full[b]) mbar_wait(&full[b], (uint32_t)((n_full[b] - 1) & 1), status);
        if (n_u) mbar_wait(full_u, (uint32_t)((n_u - 1) & 1), status);
    }
    if (alive) {
        if (mode == kChainState) {
            ilv_store(const_cast<uint8_t *>(seg_item) + kSegB, row, wg, S);
        } else {
            // the segment's map M (row j = this lane) as fp16 hi / lo B operand images, MN-major
            // over the output column, 128-byte swizzled rows: built in the (free) operand
            // buffers, then copied out in 16-byte chunks
            uint8_t *mhi = sm + wg * 16384, *mlo = sm + 32768 + wg * 16384;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                float hi8[8], lo8[8];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const float2 hf = __half22float2(__floats2half2_rn(S[ch * 8 + e], S[ch * 8 + e + 1]));
                    hi8[e] = hf.x;
                    hi8[e + 1] = hf.y;
                    lo8[e] = S[ch * 8 + e] - hf.x;
                    lo8[e + 1] = S[ch * 8 + e + 1] - hf.y;
                }
                st_h8(mhi + swz(row, ch), hi8);
                st_h8(mlo + swz(row, ch), lo8);
            }
            __syncthreads();
            uint4 *dst = reinterpret_cast<uint4 *>(const_cast<uint8_t *>(seg_item) + kSegMhi);
#pragma unroll 4
            for (int e = 0; e < 16; ++e) dst[e * NT + tid] = reinterpret_cast<const uint4 *>(sm)[e * NT + tid];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}


// ===================================================================================
// Segment combine: per (value head, sequence), S_start(p + 1) = S_start(p) M_p + B_p in order,
// S_start(1) = B_0. The product runs on the tensor cores with S split into fp16 hi + lo and M
// given as fp16 hi + lo operand images (S_hi M_hi + S_lo M_hi + S_hi M_lo, fp32 accumulation).
// Rows of S are independent in S M + B, so four CTAs share a (value head, sequence), each owning
// 32 rows (blockIdx.z): each streams the whole M_p (64 KB) but only its quarter of B_p and of the
// published states, 80 KB per step instead of 128 KB, which is what bounds a step (an SM takes
// about 30 bytes per cycle from L2). Its rows sit in TMEM lanes 0-31, handled by warps 0 and 4;
// the MMA's other 96 lanes carry no data and their results are not read.
// ===================================================================================
constexpr int CB_OFF_BUF = 0;                   // two buffers of [M_hi | M_lo] images, 64 KB each
constexpr int CB_OFF_BAR = 2 * 65536;
constexpr int CB_SMEM = CB_OFF_BAR + 64 + 1024;
constexpr uint32_t CB_TM_SHI = 0, CB_TM_SLO = 64, CB_TM_D = 128;

__global__ void __launch_bounds__(NT, 1)
gdn_segment_combine_kernel(const __grid_constant__ ChainParams P) {
    pdl_launch_dependents();
    pdl_wait();
    const int h = blockIdx.x, n = blockIdx.y, rblk = blockIdx.z;
    const int SEG = P.seg_chunks;
    int t_begin = 0, t_end = P.T;
    if (P.cu_seqlens) {
        t_begin = P.cu_seqlens[n];
        t_end = P.cu_seqlens[n + 1];
    }
    const int nch = (t_end - t_begin + C - 1) / C;
    const int nseg = (nch + SEG - 1) / SEG;
    if (nseg <= 1) return;
    const int base = t_begin / (C * SEG) + n;
    auto seg = [&](int p) { return P.ws_seg + ((size_t)h * P.seg_slots + base + p) * kSegItem; };

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + CB_OFF_BAR);
    uint64_t *bar_mma = full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(full + 3);
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int wg = warp / 4, row = rblk * 32 + lane;
    const bool active = (warp % 4) == 0;   // warps 0 and 4: TMEM lanes 0-31, this CTA's rows
    const uint32_t lane_base = 0;

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(bar_mma, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto issue_m = [&](int p) {
        uint64_t *bar = &full[(p - 1) & 1];
        mbar_arrive_expect_tx(bar, 65536);
        bulk_load(sm + CB_OFF_BUF + ((p - 1) & 1) * 65536, seg(p) + kSegMhi, 65536, bar);
    };
    if (tid == 0 && nseg > 2) issue_m(1);

    float S[64];   // S_start(p), starting from S_start(1) = B_0
    if (active) ilv_load(seg(0) + kSegB, row, wg, S);
    const uint32_t idm = idesc_f16(128, false, true, false);
    const f2_t neg1 = f2(-1.0f, -1.0f);
    for (int p = 1; p + 1 < nseg; ++p) {
        const int b = (p - 1) & 1;
        uint8_t *buf = sm + CB_OFF_BUF + b * 65536;
        // S -> fp16 hi / lo A operands
#pragma unroll
        for (int part = 0; part < 2 && active; ++part) {
            uint32_t hi[16], lo[16];
#pragma unroll
            for (int w = 0; w < 16; ++w) {
                const f2_t x2 = f2(S[part * 32 + 2 * w], S[part * 32 + 2 * w + 1]);
                const __half2 h = __floats2half2_rn(f2lo(x2), f2hi(x2));
                const float2 hf = __half22float2(h);
                const f2_t r2 = fma2(f2(hf.x, hf.y), neg1, x2);
                hi[w] = *reinterpret_cast<const uint32_t *>(&h);
                lo[w] = pack_h2(f2lo(r2), f2hi(r2));
            }
            tmem_st16(tmem + lane_base + CB_TM_SHI + wg * 32 + part * 16, hi);
            tmem_st16(tmem + lane_base + CB_TM_SLO + wg * 32 + part * 16, lo);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncthreads();
        int ok = 1;
        if (tid == 0) {
            if (p + 2 < nseg) {
                fence_proxy_async_smem();
                issue_m(p + 1);
            }
            ok = mbar_wait(&full[b], (uint32_t)(((p - 1) >> 1) & 1), P.status) ? 1 : 0;
            if (ok) {
                tc_fence_after();
                const uint8_t *mhi = buf, *mlo = buf + 32768;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_f16_ts(tmem + CB_TM_D, tmem + CB_TM_SHI + kk * 8, mndesc(mhi + kk * 2048, 16384), idm, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_f16_ts(tmem + CB_TM_D, tmem + CB_TM_SLO + kk * 8, mndesc(mhi + kk * 2048, 16384), idm, 1u);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_f16_ts(tmem + CB_TM_D, tmem + CB_TM_SHI + kk * 8, mndesc(mlo + kk * 2048, 16384), idm, 1u);
                tc_commit(bar_mma);
            }
        }
        // while the MMAs run: publish S_start(p) for the output pass, fetch B_p
        float Bp[64];
        if (active) {
            ilv_store(seg(p) + kSegS, row, wg, S);
            ilv_load(seg(p) + kSegB, row, wg, Bp);
        }
        if (tid == 0 && ok) ok = mbar_wait(bar_mma, (uint32_t)((p - 1) & 1), P.status) ? 1 : 0;
        if (!__syncthreads_and(ok)) break;
        tc_fence_after();
        if (!active) continue;
        uint32_t r32[2][32];
        tmem_ld32(tmem + CB_TM_D + lane_base + wg * 64, r32[0]);
        tmem_ld32(tmem + CB_TM_D + lane_base + wg * 64 + 32, r32[1]);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
            const f2_t s2 = add2(f2(__uint_as_float(r32[j >> 5][j & 31]), __uint_as_float(r32[j >> 5][(j & 31) + 1])),
                                 f2(Bp[j], Bp[j + 1]));
            S[j] = f2lo(s2);
            S[j + 1] = f2hi(s2);
        }
        tc_fence_before();
    }
    if (active) ilv_store(seg(nseg - 1) + kSegS, row, wg, S);   // the last segment's start state
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
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
    static PerDevice<int> attr;
    int unused = 0;
    cudaError_t e = attr.get(
        [](int, int &) {
            cudaError_t r = cudaFuncSetAttribute(gdn_chunk_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM);
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(gdn_chunk_chain_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, CH_SMEM);
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(gdn_chunk_chain_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, CHF_SMEM);
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(gdn_chunk_lean_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, CL_SMEM);
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(gdn_segment_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, CB_SMEM);
            return r;
        },
        &unused);
    if (e != cudaSuccess) return e;
    const int slots = c.T / kChunk + c.num_seqs;
    const int seg = chunked_segment_chunks(c.T, c.num_seqs, c.Hv);
    const int seg_slots = c.T / (kChunk * seg) + c.num_seqs;
    uint8_t *ws = static_cast<uint8_t *>(c.ws);
    if (!chunked_size_ok(c.T, c.num_seqs)) return cudaErrorInvalidValue;
    e = launch_pdl(gdn_chunk_prep_kernel, dim3(c.Hv, slots), dim3(NT), P_SMEM, st, maps, c.a, c.b, c.A_log,
                               c.dt_bias, c.cu_seqlens, c.T, c.num_seqs, c.Hk, c.Hv, slots, c.scale, c.l2norm, ws,
                               c.status);
    if (e != cudaSuccess) return e;
    ChainParams P{};
    const bool fused = c.xq != nullptr;
    if (fused && !make_map3(&P.zmap, c.z, c.T, c.Hv)) return cudaErrorInvalidValue;
    P.kmap = maps.k;
    P.cu_seqlens = c.cu_seqlens;
    P.T = c.T;
    P.num_seqs = c.num_seqs;
    P.Hk = c.Hk;
    P.Hv = c.Hv;
    P.slots = slots;
    P.seg_chunks = seg;
    P.seg_slots = seg_slots;
    P.mode_base = kChainFull;
    P.out_bf16 = c.out_bf16 ? 1 : 0;
    P.S0g = c.S0;
    P.S_out = c.S_out;
    P.o = c.o;
    P.ws = ws;
    P.ws_seg = ws + (size_t)c.Hv * slots * kWsItem;
    P.status = c.status;
    P.norm_w = c.norm_w;
    P.eps = c.eps;
    P.gs = c.gs;
    P.xq = c.xq;
    P.xs = c.xs;
    if (c.T > kChunk * seg) {   // some sequence may span several segments
        P.mode_base = kChainState;   // x = 2 h: segment states (B), x = 2 h + 1: segment transitions (M)
        if ((e = launch_pdl(gdn_chunk_lean_kernel, dim3(2 * c.Hv, seg_slots, 1), dim3(NT), CL_SMEM, st, P)) != cudaSuccess)
            return e;
        if ((e = launch_pdl(gdn_segment_combine_kernel, dim3(c.Hv, c.num_seqs, 4), dim3(NT), CB_SMEM, st, P)) != cudaSuccess)
            return e;
        P.mode_base = kChainFull;
    }
    if (fused) return launch_pdl(gdn_chunk_chain_kernel<true>, dim3(c.Hv, seg_slots, 1), dim3(CHF_THREADS), CHF_SMEM, st, P);
    return launch_pdl(gdn_chunk_chain_kernel<false>, dim3(c.Hv, seg_slots, 1), dim3(CH_THREADS), CH_SMEM, st, P);
}

}  // namespace gdn
