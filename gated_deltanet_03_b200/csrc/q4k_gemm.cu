// Output projection with Q4_K weights (the comparison format of "Red Lite dev15d - DeltaNet gated
// tail + Q4_K output projection", section "Q4_K implementation"): y[m, n] = sum_k a[m, k] w[n, k]
// with a the bf16 activations and w decoded on the fly from 256-value blocks of 144 bytes (f16 d,
// f16 dmin, twelve bytes of 6-bit sub-block scales and mins, 128 bytes of 4-bit quants;
// w = d * scale * q - dmin * min; bit positions of the GGUF K-quant layout, which the page calls
// canonical).
//
// tcgen05 kind::f16 (bf16 A and B, fp32 accumulation in tensor memory), CTA tile 128 x BN, 64
// values of K per stage, two CTAs per SM: BN = 128 with a 3-stage ring (small and medium M, and
// the split-K form below), BN = 256 with a 2-stage ring for large M (each stage's MMA work doubles
// while its shared-memory traffic - the activation tile written by TMA and read by the MMA, the
// weight tile written by the decode warps and read by the MMA - grows by half, and that traffic is
// what bounds the kernel). Warp 0: TMA of the activation tile; warp 1: tensor memory and the MMA
// issue (one thread); warps 4 .. 4 + BN/32 - 1: one output column (weight row) per thread - per
// stage it reads the row's 32 quant bytes for the stage (and the block header at a block's first
// stage), one stage ahead of their use, decodes the 64 weights two at a time in bf16 arithmetic
// (the sub-block factors d scale and dmin min rounded to bf16, one bf16x2 FMA per pair) and writes
// them into the stage's K-major 128-byte-swizzled B tile; at the end the same warps read the
// accumulator (one lane quarter and 128 columns each) and store y. The weights are decoded once
// per output tile; the 4.5 MB
// weight of the 4096 -> 2048 projection stays in L2 across the M tiles.
//
// Split K for small M (the decode shapes, where the output tiles alone would leave most SMs
// idle): a cluster of S CTAs (2, 4 or 8) along grid z shares one output tile, CTA r taking the
// r-th of S equal K ranges. Each CTA writes its fp32 partial tile into its own shared memory
// (over the then idle stage ring), and after a cluster barrier CTA r sums rows
// [r 128/S, (r+1) 128/S) over the S partials in rank order (ld.shared::cluster) and stores them;
// a second cluster barrier keeps every partial in place until all CTAs have read it. The order
// of the sums is fixed, so results do not depend on scheduling.
#include "common.cuh"
#include "kernels.h"

namespace gdn {
namespace {

constexpr int QK_BM = 128, QK_BK = 64;
constexpr int QK_TILE_A = QK_BM * QK_BK * 2;                // 16 KB activation tile per stage
constexpr int QK_BLOCK_BYTES = 144;
constexpr int QK_MAX_SPLIT = 8;
// Two tile widths: N = 128 (three stages, the split-K form for small M) and N = 256 (two stages,
// eight decode warps; half again as much MMA work per byte of shared-memory traffic, for large
// M). Both keep two CTAs per SM.
template <int BN>
struct QkCfg {
    static constexpr int STAGES = BN == 128 ? 3 : 2;
    static constexpr int TILE_B = BN * QK_BK * 2;
    static constexpr int STAGE_BYTES = QK_TILE_A + TILE_B;
    static constexpr int PART_PITCH = BN + 4;                 // fp32 row pitch of a split-K partial tile
    static constexpr int PART_BYTES = BN == 128 ? QK_BM * PART_PITCH * 4 : 0;
    static constexpr int OFF_BAR = STAGES * STAGE_BYTES > PART_BYTES ? STAGES * STAGE_BYTES : PART_BYTES;
    static constexpr int SMEM = OFF_BAR + 128 + 1024;
    static constexpr int DEC_WARPS = BN / 32;                  // one weight row per decode thread
    static constexpr int THREADS = 128 + BN;
};
static_assert(2 * (QkCfg<128>::SMEM + 1024) <= 233472 && 2 * (QkCfg<256>::SMEM + 1024) <= 233472,
              "two Q4_K GEMM CTAs per SM");

__device__ __forceinline__ uint32_t qk_cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void qk_cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// 16 bytes at this CTA's shared address `p` as seen in CTA `rank` of the cluster.
__device__ __forceinline__ float4 qk_ld_cluster(const void *p, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(a)
                 : "memory");
    return v;
}

__device__ __forceinline__ uint32_t qk_swz(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

__device__ __forceinline__ void qk_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

// Scale and min of sub-block j from the twelve packed bytes (sc[0..11]).
__device__ __forceinline__ void q4k_scale_min(const uint8_t (&sc)[12], int j, int &scale, int &mn) {
    if (j < 4) {
        scale = sc[j] & 63;
        mn = sc[j + 4] & 63;
    } else {
        scale = (sc[j + 4] & 15) | ((sc[j - 4] >> 6) << 4);
        mn = (sc[j + 4] >> 4) | ((sc[j] >> 6) << 4);
    }
}


template <bool OUT_BF16, int BN>
__global__ void __launch_bounds__(QkCfg<BN>::THREADS, 2)
q4k_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const uint8_t *__restrict__ w, int M, int N, int K,
                void *__restrict__ y, int split, int *status) {
    using Cfg = QkCfg<BN>;
    constexpr int QK_STAGES = Cfg::STAGES;
    pdl_launch_dependents();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Cfg::OFF_BAR);
    uint64_t *a_full = bars, *b_full = bars + QK_STAGES, *empty = bars + 2 * QK_STAGES;
    uint64_t *acc_full = bars + 3 * QK_STAGES, *drain = bars + 3 * QK_STAGES + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3 * QK_STAGES + 2);
    auto tile_a = [&](int s) { return sm + s * Cfg::STAGE_BYTES; };
    auto tile_b = [&](int s) { return sm + s * Cfg::STAGE_BYTES + QK_TILE_A; };

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int n0 = blockIdx.x * BN, m0 = blockIdx.y * QK_BM;
    const int nb = K / 256;
    // this CTA's K range (all of K without split): k-tiles [kt0, kt0 + num_k)
    const uint32_t crank = split > 1 ? qk_cluster_rank() : 0u;
    const int num_k = K / QK_BK / split, kt0 = (int)crank * num_k;

    if (tid == 0) {
        for (int s = 0; s < QK_STAGES; ++s) {
            mbar_init(&a_full[s], 1);
            mbar_init(&b_full[s], Cfg::DEC_WARPS);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, BN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();

    if (warp == 0) {
        if (lane == 0) {
            for (int i = 0; i < num_k; ++i) {
                const int s = i % QK_STAGES;
                if (!mbar_wait(&empty[s], (uint32_t)(((i / QK_STAGES) & 1) ^ 1), status)) break;
                mbar_arrive_expect_tx(&a_full[s], QK_TILE_A);
                tma_load_2d(tile_a(s), &map_a, &a_full[s], (kt0 + i) * QK_BK, m0);
            }
            // before the CTA may exit: the last load armed on each stage has landed
            for (int s = 0; s < QK_STAGES && s < num_k; ++s) {
                const int last = num_k - 1 - ((num_k - 1 - s) % QK_STAGES);
                mbar_wait(&a_full[s], (uint32_t)((last / QK_STAGES) & 1), status);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // bf16 A and B, fp32 accumulation, both K-major, N = BN, M = 128
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                   ((uint32_t)(QK_BM >> 4) << 24);
            int issued = 0;
            for (int i = 0; i < num_k; ++i) {
                const int s = i % QK_STAGES;
                const uint32_t ph = (uint32_t)((i / QK_STAGES) & 1);
                if (!mbar_wait(&a_full[s], ph, status) || !mbar_wait(&b_full[s], ph, status)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < QK_BK / 16; ++kk)
                    qk_mma(tmem, smem_desc(smem_u32(tile_a(s)) + kk * 32, 16, 1024, 2),
                           smem_desc(smem_u32(tile_b(s)) + kk * 32, 16, 1024, 2), idesc, (i | kk) ? 1u : 0u);
                tc_commit(&empty[s]);
                ++issued;
                if (i == num_k - 1) tc_commit(acc_full);
            }
            // before tensor memory is freed: every MMA issued has completed (bounded)
            if (issued) {
                tc_commit(drain);
                mbar_wait(drain, 0, status);
            }
        }
    } else if (warp >= 4) {
        const int dw = warp - 4;                          // decode warp: weight rows 32 dw ..
        const int quarter = dw & 3, col0 = (dw >> 2) * 128;   // its accumulator lanes and columns
        const int rl = dw * 32 + lane;                    // weight row within the tile
        const int n = n0 + rl;
        const uint8_t *wrow = w + (size_t)n * nb * QK_BLOCK_BYTES;
        bool ok = true;
        float ds[2] = {0.f, 0.f}, dm[2] = {0.f, 0.f};
        // the quant bytes of a stage's 64 values (sub-blocks 2 g and 2 g + 1), loaded one stage
        // ahead of their decode so that the L2 round trip overlaps it; the block's 16-byte header
        // only at the first stage of a block (or of this CTA's range) - each lane reads its own
        // row, so every 16-byte load is a separate L1 wavefront
        auto load_stage = [&](int i, uint4 &q0, uint4 &q1, uint4 &hd) {
            const int kt = kt0 + i, g = kt & 3;
            const uint8_t *blk = wrow + (size_t)(kt >> 2) * QK_BLOCK_BYTES;
            q0 = *reinterpret_cast<const uint4 *>(blk + 16 + 32 * g);
            q1 = *reinterpret_cast<const uint4 *>(blk + 16 + 32 * g + 16);
            if (g == 0 || i == 0) hd = *reinterpret_cast<const uint4 *>(blk);
        };
        uint4 nq0 = make_uint4(0u, 0u, 0u, 0u), nq1 = nq0, nhd = nq0;
        if (num_k > 0) load_stage(0, nq0, nq1, nhd);
        for (int i = 0; i < num_k && ok; ++i) {
            const int kt = kt0 + i;
            const int s = i % QK_STAGES, g = kt & 3;
            const uint4 q0 = nq0, q1 = nq1;
            uint8_t sc[12];
            float d = 0.f, dmin = 0.f;
            {
                const uint4 hd = nhd;
                if (i + 1 < num_k) load_stage(i + 1, nq0, nq1, nhd);
                d = __half2float(__ushort_as_half((unsigned short)(hd.x & 0xFFFFu)));
                dmin = __half2float(__ushort_as_half((unsigned short)(hd.x >> 16)));
                const uint32_t words[3] = {hd.y, hd.z, hd.w};
#pragma unroll
                for (int i = 0; i < 12; ++i) sc[i] = (uint8_t)(words[i >> 2] >> (8 * (i & 3)));
            }
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                int scale, mn;
                q4k_scale_min(sc, 2 * g + h2, scale, mn);
                ds[h2] = d * (float)scale;
                dm[h2] = dmin * (float)mn;
            }
            if (lane == 0) ok = mbar_wait(&empty[s], (uint32_t)(((i / QK_STAGES) & 1) ^ 1), status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            // values 0-31 of the stage: low nibbles (sub-block 2 g); 32-63: high nibbles (2 g + 1).
            // Two quants at a time as bf16 pairs: a byte permute puts the nibbles of two adjacent
            // bytes into the two 16-bit halves, OR-ing in the exponent of 128 makes them the bf16
            // values 128 + q (exact, 7 mantissa bits), a bf16x2 subtraction gives q exactly, and one
            // bf16x2 FMA gives d scale q - dmin min (d scale and dmin min rounded to bf16 first)
            const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
            uint8_t *brow = tile_b(s);
            const __nv_bfloat162 c128 = __floats2bfloat162_rn(128.0f, 128.0f);
            const __nv_bfloat162 ds2[2] = {__floats2bfloat162_rn(ds[0], ds[0]), __floats2bfloat162_rn(ds[1], ds[1])};
            const __nv_bfloat162 nd2[2] = {__floats2bfloat162_rn(-dm[0], -dm[0]), __floats2bfloat162_rn(-dm[1], -dm[1])};
#pragma unroll
            for (int c = 0; c < 8; ++c) {   // 16-byte chunk c: values 8 c .. 8 c + 7
                const int h2 = c >> 2, sh = h2 ? 4 : 0;
                const uint32_t wa = qw[(c & 3) * 2] >> sh, wb = qw[(c & 3) * 2 + 1] >> sh;
                uint32_t packed[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t src = e < 2 ? wa : wb;
                    const uint32_t xb = (__byte_perm(src, 0u, (e & 1) ? 0x4342u : 0x4140u) & 0x000F000Fu) | 0x43004300u;
                    const __nv_bfloat162 q2 = __hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&xb), c128);
                    const __nv_bfloat162 w2 = __hfma2(q2, ds2[h2], nd2[h2]);
                    packed[e] = *reinterpret_cast<const uint32_t *>(&w2);
                }
                *reinterpret_cast<uint4 *>(brow + qk_swz(rl, c)) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&b_full[s]);
        }
        // epilogue: this warp's lane quarter of the 128 x 128 accumulator, one output row per thread
        if (ok) {
            if (lane == 0) ok = mbar_wait(acc_full, 0, status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        if (ok && BN == 128 && split > 1) {
            // the partial tile into this CTA's shared memory (the stage ring is idle: every load
            // was consumed by an MMA that has completed), row = tensor-memory lane
            tc_fence_after();
            const uint32_t lb = ((uint32_t)(quarter * 32)) << 16;
            float *prow = reinterpret_cast<float *>(sm) + (size_t)(quarter * 32 + lane) * Cfg::PART_PITCH;
#pragma unroll 1
            for (int c32 = 0; c32 < 4; ++c32) {
                uint32_t r[32];
                tmem_ld32(tmem + lb + c32 * 32, r);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    *reinterpret_cast<float4 *>(prow + c32 * 32 + 4 * i) =
                        make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                    __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
            }
        } else if (ok) {
            tc_fence_after();
            const int m = m0 + quarter * 32 + lane;
            const uint32_t lb = ((uint32_t)(quarter * 32)) << 16;
#pragma unroll 1
            for (int c32 = 0; c32 < 4; ++c32) {   // this warp's 128 accumulator columns from col0
                uint32_t r[32];
                tmem_ld32(tmem + lb + col0 + c32 * 32, r);
                tmem_ld_wait();
                if (m < M) {
                    if constexpr (OUT_BF16) {
                        __nv_bfloat16 *yr = reinterpret_cast<__nv_bfloat16 *>(y) + (size_t)m * N + n0 + col0 + c32 * 32;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            uint4 u;
                            __nv_bfloat162 *p2 = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                p2[q] = __floats2bfloat162_rn(__uint_as_float(r[8 * i + 2 * q]), __uint_as_float(r[8 * i + 2 * q + 1]));
                            *reinterpret_cast<uint4 *>(yr + 8 * i) = u;
                        }
                    } else {
                        float *yr = reinterpret_cast<float *>(y) + (size_t)m * N + n0 + col0 + c32 * 32;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            *reinterpret_cast<float4 *>(yr + 4 * i) =
                                make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                            __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
                    }
                }
            }
        }
    }
    if (BN == 128 && split > 1) {
        // every CTA of the cluster reaches both barriers, on the failure path too (its partial is
        // then stale and the status word already says so)
        qk_cluster_sync();
        const int rows = QK_BM / split, r0 = (int)crank * rows;
        for (int u = tid; u < rows * (BN / 4); u += Cfg::THREADS) {
            const int rr = r0 + u / (BN / 4), c4 = u % (BN / 4);
            const float *src = reinterpret_cast<const float *>(sm) + (size_t)rr * Cfg::PART_PITCH + 4 * c4;
            float4 acc = qk_ld_cluster(src, 0);
            for (int z = 1; z < split; ++z) {
                const float4 v = qk_ld_cluster(src, (uint32_t)z);
                acc.x += v.x;
                acc.y += v.y;
                acc.z += v.z;
                acc.w += v.w;
            }
            const int m = m0 + rr;
            if (m < M) {
                if constexpr (OUT_BF16) {
                    const __nv_bfloat162 p0 = __floats2bfloat162_rn(acc.x, acc.y);
                    const __nv_bfloat162 p1 = __floats2bfloat162_rn(acc.z, acc.w);
                    uint2 u2;
                    u2.x = *reinterpret_cast<const uint32_t *>(&p0);
                    u2.y = *reinterpret_cast<const uint32_t *>(&p1);
                    *reinterpret_cast<uint2 *>(reinterpret_cast<__nv_bfloat16 *>(y) + (size_t)m * N + n0 + 4 * c4) = u2;
                } else {
                    *reinterpret_cast<float4 *>(reinterpret_cast<float *>(y) + (size_t)m * N + n0 + 4 * c4) = acc;
                }
            }
        }
        qk_cluster_sync();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, BN);
    }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn qk_encode_fn() {
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

}  // namespace

cudaError_t launch_q4k_gemm(const Q4kGemmArgs &g, cudaStream_t st) {
    if (g.M == 0 || g.N == 0) return cudaSuccess;
    EncodeTiledFn fn = qk_encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    CUtensorMap ma;
    cuuint64_t dims[2] = {(cuuint64_t)g.K, (cuuint64_t)g.M};
    cuuint64_t strides[1] = {(cuuint64_t)g.K * 2};
    cuuint32_t box[2] = {QK_BK, QK_BM};
    cuuint32_t elem[2] = {1, 1};
    if (fn(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(g.a), dims, strides, box, elem,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    static PerDevice<int> sm_count;   // the shared-memory attributes are set per device alongside
    int sms = 0;
    cudaError_t e = sm_count.get(
        [](int dev, int &r) {
            cudaError_t x = cudaSuccess;
            if (x == cudaSuccess)
                x = cudaFuncSetAttribute(q4k_gemm_kernel<true, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize, QkCfg<128>::SMEM);
            if (x == cudaSuccess)
                x = cudaFuncSetAttribute(q4k_gemm_kernel<false, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize, QkCfg<128>::SMEM);
            if (x == cudaSuccess)
                x = cudaFuncSetAttribute(q4k_gemm_kernel<true, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize, QkCfg<256>::SMEM);
            if (x == cudaSuccess)
                x = cudaFuncSetAttribute(q4k_gemm_kernel<false, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize, QkCfg<256>::SMEM);
            if (x == cudaSuccess) x = cudaDeviceGetAttribute(&r, cudaDevAttrMultiProcessorCount, dev);
            return x;
        },
        &sms);
    if (e != cudaSuccess) return e;
    const int mt = (g.M + QK_BM - 1) / QK_BM;
    const int tiles = (g.N / 128) * mt;
    const int num_k = g.K / QK_BK;
    int split = 1;   // double while the CTAs still fit at two per SM and every range keeps a whole block
    while (split < QK_MAX_SPLIT && tiles * split * 2 <= 2 * sms && num_k % (2 * split) == 0 &&
           num_k / (2 * split) >= 256 / QK_BK)
        split *= 2;
    // 256-wide tiles when K is not split and they still give every SM slot several tiles
    const bool wide = split == 1 && g.N % 256 == 0 && (g.N / 256) * mt >= 4 * sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(g.N / (wide ? 256 : 128)), (unsigned)mt, (unsigned)split);
    cfg.blockDim = dim3(wide ? QkCfg<256>::THREADS : QkCfg<128>::THREADS);
    cfg.dynamicSmemBytes = wide ? QkCfg<256>::SMEM : QkCfg<128>::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attrs[2];
    attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[0].val.programmaticStreamSerializationAllowed = 1;
    attrs[1].id = cudaLaunchAttributeClusterDimension;
    attrs[1].val.clusterDim.x = 1;
    attrs[1].val.clusterDim.y = 1;
    attrs[1].val.clusterDim.z = (unsigned)split;
    cfg.attrs = attrs;
    cfg.numAttrs = split > 1 ? 2 : 1;
    if (wide) {
        if (g.out_bf16)
            return cudaLaunchKernelEx(&cfg, q4k_gemm_kernel<true, 256>, ma, g.w, g.M, g.N, g.K, g.y, split, g.status);
        return cudaLaunchKernelEx(&cfg, q4k_gemm_kernel<false, 256>, ma, g.w, g.M, g.N, g.K, g.y, split, g.status);
    }
    if (g.out_bf16)
        return cudaLaunchKernelEx(&cfg, q4k_gemm_kernel<true, 128>, ma, g.w, g.M, g.N, g.K, g.y, split, g.status);
    return cudaLaunchKernelEx(&cfg, q4k_gemm_kernel<false, 128>, ma, g.w, g.M, g.N, g.K, g.y, split, g.status);
}

}  // namespace gdn
