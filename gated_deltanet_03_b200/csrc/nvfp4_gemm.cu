// NVFP4 W4A4 GEMM on the block-scaled FP4 tensor cores (tcgen05 kind::mxf4nvf4, 16-value
// E4M3 scale blocks, fp32 accumulation in tensor memory):
//     y[m, n] = alpha * sum_k E2M1(a)[m,k] E4M3(as)[m,k/16] * E2M1(b)[n,k] E4M3(bs)[n,k/16].
// "Why Gated DeltaNet Survives 4-Bit Quantization", abstract: NVFP4 W4A4 on every linear
// layer; "Red Lite dev15d - DeltaNet gated tail", Pinned graph semantics, step 6: the output
// projection (4096 -> 2048 in the 27B-class layer).
//
// SM pairs: a cluster of two CTAs (one per SM) computes 256 x 256 tiles of y with
// tcgen05.mma.cta_group::2. CTA r holds A rows 128 r .. 128 r + 127 of the tile and B rows
// (output columns) 128 r .. 128 r + 127 in its shared memory and accumulates its 128 rows x 256
// columns in its own tensor memory, so each SM reads 38 KB per 256-value k-stage for the work
// that would take 54 KB on one SM with a 128 x 256 tile. Block scales: each CTA's tensor memory
// holds the scales of its own A rows and of all 256 B rows. Only CTA 0 (the leader) issues MMAs;
// its commits arrive on both CTAs' barriers (tcgen05.commit multicast).
//
// Persistent: the pairs walk the tiles (pair p takes tiles p, p + pairs, ...; consecutive
// tiles share their A rows, so concurrent pairs read each A tile from DRAM once). The stage ring
// and its barriers run on one counter across tiles, so the producer fetches the next tile's
// stages while the epilogue drains the current one. Warp roles in each CTA:
//   warp 0     TMA producer: A (128 rows x 128 B) and B (128 rows x 128 B) tiles per stage,
//              128-byte swizzle, into a 5-stage ring, with the stage's row-major [rows, 16 B]
//              E4M3 scales (this CTA's A rows, all 256 B rows) when K % 256 == 0;
//   warp 1     allocates the pair's tensor memory; in the leader, lane 0 issues the MMAs: per
//              stage it waits until both CTAs' scale warps have put the stage's scales into
//              tensor memory (they do so after the stage's TMA data has landed, so that arrival
//              also means "operands ready"), and before a tile's first MMA until both CTAs'
//              epilogues have read the previous accumulator;
//   warps 4-7  per stage each writes the scales into its lane quarter of the stage's
//              tensor-memory scale slot with tcgen05.st (the layout the block-scaled MMA reads:
//              for 32 rows r = 32 c + l, lane l, column 4 kb + c holds the four 16-value block
//              scales of MMA k-step kb; B's 256 rows take 8 columns per k-step; the four lane
//              quarters hold the same copy), read from the TMA-staged tile, or from global memory
//              (zero past K) when the scales cannot be TMA-loaded;
//   warps 8-15 the epilogue, two warps per lane quarter (column halves): tensor memory ->
//              registers (64 columns at a time; after its last read the warp releases the
//              accumulator) -> alpha * acc -> 16-byte stores of the thread's row.
// Cross-CTA arrivals use mapa-mapped barrier addresses. Every barrier wait is bounded (about
// 1 s); an expired wait records GDN_ERR_TIMEOUT and the CTA finishes without issuing more work.
// Before tensor memory is freed the producer waits for the last load it armed on each stage and
// the leader for a final commit of its MMAs (both bounded); then both CTAs meet at a cluster
// barrier.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace gdn {
namespace {

constexpr int BK = 256;                    // FP4 values per stage per row (128 bytes)
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 512;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_ACC = 0;             // accumulator: 128 lanes x 256 columns fp32
constexpr uint32_t TM_SF = 256;            // per stage slot: A scales 4 x 4 columns, B scales 4 x 8
constexpr uint32_t SF_SLOT = 48;
constexpr int A_BYTES = 128 * BK / 2;      // 16 KB
constexpr int B_BYTES = 128 * BK / 2;      // 16 KB: this CTA's half of the 256 output columns
constexpr int SFA_BYTES = 128 * 16;        // 2 KB
constexpr int SFB_BYTES = 256 * 16;        // 4 KB: both halves
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int STAGES = 5;
constexpr int BAR_OFF = STAGES * STAGE_BYTES;
constexpr int SMEM_BYTES = BAR_OFF + 256 + 1024;
static_assert(STAGE_BYTES % 1024 == 0, "stage bases stay 1024-byte aligned");
static_assert(TM_SF + STAGES * SF_SLOT <= TMEM_COLS, "scale slots fit in tensor memory");

// Instruction descriptor, kind::mxf4nvf4 block-scaled: A and B E2M1 (format 1), K-major,
// scales UE4M3, M = 256 (the CTA pair), N = 256, dense K = 64 per instruction.
__host__ __device__ constexpr uint32_t make_idesc() {
    return (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

// 16 scale bytes of one row for the k-range of a stage (zero past K or past the last row).
__device__ __forceinline__ uint4 load_scale_row(const uint8_t *sf, int row, int rows, int kblk16, int nblk16) {
    uint4 r = make_uint4(0, 0, 0, 0);
    if (row >= rows || kblk16 >= nblk16) return r;
    const uint8_t *p = sf + (size_t)row * nblk16 + kblk16;
    if (nblk16 - kblk16 >= 16 && (reinterpret_cast<uintptr_t>(p) & 15u) == 0) {
        return __ldg(reinterpret_cast<const uint4 *>(p));
    }
    uint8_t tmp[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) tmp[j] = (kblk16 + j < nblk16) ? p[j] : (uint8_t)0;
    r.x = tmp[0] | (tmp[1] << 8) | (tmp[2] << 16) | ((uint32_t)tmp[3] << 24);
    r.y = tmp[4] | (tmp[5] << 8) | (tmp[6] << 16) | ((uint32_t)tmp[7] << 24);
    r.z = tmp[8] | (tmp[9] << 8) | (tmp[10] << 16) | ((uint32_t)tmp[11] << 24);
    r.w = tmp[12] | (tmp[13] << 8) | (tmp[14] << 16) | ((uint32_t)tmp[15] << 24);
    return r;
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// The shared::cluster address of this CTA's object `p` in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_rank(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
// Arrival on a barrier of a CTA of the cluster. The pairs' barriers carry no generic-memory data
// (tensor-memory and operand ordering is by the tcgen05 fences around them), so the arrive keeps
// the default CTA-scope semantics and no cluster-wide fence is paid per stage.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
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
// Bounded wait (the control block's limit, 1 s by default) on a barrier that receives arrivals
// from the peer CTA.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, int *status) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    const uint64_t limit = ctl_wait_limit(status);
    for (uint32_t i = 0;; ++i) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if ((i & 255u) == 255u && global_timer_ns() - t0 > limit) {
            report_status(status, GDN_ERR_TIMEOUT);
            return false;
        }
    }
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The MMAs issued so far complete -> one arrival on `bar` in both CTAs of the pair.
__device__ __forceinline__ void tc_commit_pair(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 ::"r"(smem_u32(bar)), "h"((uint16_t)3)
                 : "memory");
}

__global__ void __launch_bounds__(THREADS, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                       const __grid_constant__ CUtensorMap map_sfa, const __grid_constant__ CUtensorMap map_sfb,
                       int sf_tma, const uint8_t *__restrict__ sfa_g, const uint8_t *__restrict__ sfb_g,
                       float alpha, const float *__restrict__ col_alpha, int M, int N, int K, int out_bf16,
                       void *__restrict__ y, int *status) {
    pdl_launch_dependents();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    auto sa = [&](int s) { return base + s * STAGE_BYTES; };
    auto sb = [&](int s) { return base + s * STAGE_BYTES + A_BYTES; };
    auto ssfa = [&](int s) { return base + s * STAGE_BYTES + A_BYTES + B_BYTES; };
    auto ssfb = [&](int s) { return base + s * STAGE_BYTES + A_BYTES + B_BYTES + SFA_BYTES; };
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + BAR_OFF);
    uint64_t *full = bars, *empty = bars + STAGES, *sf_ready = bars + 2 * STAGES;
    uint64_t *acc_full = bars + 3 * STAGES, *acc_empty = bars + 3 * STAGES + 1, *drain = bars + 3 * STAGES + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3 * STAGES + 3);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cluster_rank();
    const int pair = blockIdx.x / 2, npairs = gridDim.x / 2;
    const int tiles_n = (N + 255) / 256;
    const int num_tiles = tiles_n * ((M + 255) / 256);
    const int num_k = (K + BK - 1) / BK;
    const int nblk16 = K / 16;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);      // this CTA's TMA: expect_tx arrive
            mbar_init(&empty[s], 1);     // the leader's commit of the MMAs that read the stage
            mbar_init(&sf_ready[s], 8);  // leader only: four scale warps in each CTA
        }
        mbar_init(acc_full, 1);          // the leader's commit after a tile's last MMA
        mbar_init(acc_empty, 2 * EPI_WARPS);   // leader only: every epilogue warp of both CTAs
        mbar_init(drain, 1);             // the leader's last commit (every MMA of the pair done)
        fence_barrier_init();
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_b);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync_all();   // both CTAs' barriers are initialised and tensor memory is allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();

    if (warp == 0) {
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += npairs) {
                const int tile_m = t / tiles_n, tile_n = t % tiles_n;
                for (int kt = 0; kt < num_k; ++kt, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&empty[s], ph ^ 1, status)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[s], A_BYTES + B_BYTES + (sf_tma ? SFA_BYTES + SFB_BYTES : 0));
                    tma_load_2d(sa(s), &map_a, &full[s], kt * (BK / 2), tile_m * 256 + (int)rank * 128);
                    tma_load_2d(sb(s), &map_b, &full[s], kt * (BK / 2), tile_n * 256 + (int)rank * 128);
                    if (sf_tma) {
                        tma_load_2d(ssfa(s), &map_sfa, &full[s], kt * (BK / 16), tile_m * 256 + (int)rank * 128);
                        tma_load_2d(ssfb(s), &map_sfb, &full[s], kt * (BK / 16), tile_n * 256);
                    }
                }
            }
            // before the CTA may exit: the latest load armed on each stage has landed (bounded; on
            // the normal path every one of them was consumed already)
            for (int s = 0; s < STAGES && s < it; ++s) {
                const int last = it - 1 - ((it - 1 - s) % STAGES);   // the last use of stage s
                mbar_wait(&full[s], (uint32_t)((last / STAGES) & 1), status);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = make_idesc();
            bool ok = true;
            int it = 0, j = 0;
            for (int t = pair; t < num_tiles && ok; t += npairs, ++j) {
                if (j > 0 && !mbar_wait_cluster(acc_empty, (uint32_t)((j - 1) & 1), status)) { ok = false; break; }
                tc_fence_after();
                for (int kt = 0; kt < num_k; ++kt, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait_cluster(&sf_ready[s], ph, status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sf = tmem + TM_SF + s * SF_SLOT;
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        const uint64_t adesc = smem_desc(smem_u32(sa(s)) + kb * 32, 16, 1024, 2);
                        const uint64_t bdesc = smem_desc(smem_u32(sb(s)) + kb * 32, 16, 1024, 2);
                        const uint32_t acc = (kt > 0 || kb > 0) ? 1u : 0u;
                        asm volatile(
                            "{\n\t.reg .pred p;\n\t"
                            "setp.ne.b32 p, %4, 0;\n\t"
                            "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
                            "}" ::"r"(tmem + TM_ACC),
                            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(sf + kb * 4), "r"(sf + 16 + kb * 8));
                    }
                    tc_commit_pair(&empty[s]);
                }
                if (ok) tc_commit_pair(acc_full);
            }
            // before the pair may free tensor memory: every MMA issued has completed (bounded)
            if (it > 0) {
                tc_commit_pair(drain);
                mbar_wait(drain, 0, status);
            }
        }
    } else if (warp >= 4 && warp < 8) {
        const int quarter = warp - 4;
        const uint32_t lane_q = (uint32_t)(quarter * 32) << 16;
        const uint32_t leader_sf_ready = mapa_rank(sf_ready, 0);
        bool ok = true;
        int it = 0;
        for (int t = pair; t < num_tiles && ok; t += npairs) {
            const int tile_m = t / tiles_n, tile_n = t % tiles_n;
            for (int kt = 0; kt < num_k; ++kt, ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                uint32_t ra[16], rb[32];
                // the stage's operands (and scale tiles) have landed in this CTA; the tensor-memory
                // slot is free then too (the producer refilled the stage after the MMAs released it)
                if (lane == 0) ok = mbar_wait(&full[s], ph, status);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (sf_tma) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 v = reinterpret_cast<const uint4 *>(ssfa(s))[c * 32 + lane];
                        ra[c] = v.x; ra[4 + c] = v.y; ra[8 + c] = v.z; ra[12 + c] = v.w;
                    }
#pragma unroll
                    for (int gc = 0; gc < 8; ++gc) {
                        const uint4 v = reinterpret_cast<const uint4 *>(ssfb(s))[gc * 32 + lane];
                        rb[gc] = v.x; rb[8 + gc] = v.y; rb[16 + gc] = v.z; rb[24 + gc] = v.w;
                    }
                } else {
                    const int kb16 = kt * (BK / 16);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 v = load_scale_row(sfa_g, tile_m * 256 + (int)rank * 128 + c * 32 + lane, M, kb16, nblk16);
                        ra[c] = v.x; ra[4 + c] = v.y; ra[8 + c] = v.z; ra[12 + c] = v.w;
                    }
#pragma unroll
                    for (int gc = 0; gc < 8; ++gc) {
                        const uint4 v = load_scale_row(sfb_g, tile_n * 256 + gc * 32 + lane, N, kb16, nblk16);
                        rb[gc] = v.x; rb[8 + gc] = v.y; rb[16 + gc] = v.z; rb[24 + gc] = v.w;
                    }
                }
                const uint32_t sf = tmem + lane_q + TM_SF + s * SF_SLOT;
                tmem_st16(sf, ra);
                tmem_st16(sf + 16, *reinterpret_cast<const uint32_t(*)[16]>(&rb[0]));
                tmem_st16(sf + 32, *reinterpret_cast<const uint32_t(*)[16]>(&rb[16]));
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(leader_sf_ready + (uint32_t)(s * 8));
            }
        }
    } else if (warp >= 8) {
        const int e = warp - 8, quarter = e % 4, half = e / 4;
        const uint32_t lane_q = (uint32_t)(quarter * 32) << 16;
        const uint32_t leader_acc_empty = mapa_rank(acc_empty, 0);
        bool ok = true;
        int j = 0;
        for (int t = pair; t < num_tiles && ok; t += npairs, ++j) {
            const int tile_m = t / tiles_n, tile_n = t % tiles_n;
            if (lane == 0) ok = mbar_wait(acc_full, (uint32_t)(j & 1), status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const int row = tile_m * 256 + (int)rank * 128 + quarter * 32 + lane;
#pragma unroll 1
            for (int pr = 0; pr < 2; ++pr) {
                uint32_t rr[2][32];
                tmem_ld32(tmem + TM_ACC + lane_q + half * 128 + 64 * pr, rr[0]);
                tmem_ld32(tmem + TM_ACC + lane_q + half * 128 + 64 * pr + 32, rr[1]);
                tmem_ld_wait();
                if (pr == 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote(leader_acc_empty);
                }
                if (row >= M) continue;
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    const int c0 = tile_n * 256 + half * 128 + 64 * pr + 32 * q2;
                    if (c0 >= N) break;
                    float v[32];
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const float al = col_alpha ? __ldg(col_alpha + min(c0 + jj, N - 1)) : alpha;
                        v[jj] = __uint_as_float(rr[q2][jj]) * al;
                    }
                    if (out_bf16) {
                        __nv_bfloat16 *yr = reinterpret_cast<__nv_bfloat16 *>(y) + (size_t)row * N + c0;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            if (c0 + 8 * i >= N) break;
                            uint4 u;
                            __nv_bfloat162 *p2 = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                p2[q] = __floats2bfloat162_rn(v[8 * i + 2 * q], v[8 * i + 2 * q + 1]);
                            *reinterpret_cast<uint4 *>(yr + 8 * i) = u;
                        }
                    } else {
                        float *yr = reinterpret_cast<float *>(y) + (size_t)row * N + c0;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            if (c0 + 4 * i >= N) break;
                            *reinterpret_cast<float4 *>(yr + 4 * i) =
                                make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                        }
                    }
                }
            }
        }
    }

    // neither CTA frees tensor memory or exits while the pair's MMAs, reads or remote arrivals
    // may still touch it
    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

// ---------------------------------------------------------------- host side ----

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

// Byte-granular 2-D map over a [rows, row_bytes] matrix, box [box_rows, box_bytes].
bool make_map(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t row_bytes, uint32_t box_rows,
              uint32_t box_bytes = 128, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {row_bytes, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_bytes, box_rows};
    cuuint32_t elem[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(ptr), dims, strides, box, elem,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

namespace {

// One thread per output column: find its module (a short linear search over the module ends)
// and write 1 / (act * scale) with IEEE division.
__global__ void fused_col_alpha_kernel(const __grid_constant__ ColAlphaArgs c, int32_t N) {
    pdl_launch_dependents();
    pdl_wait();
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    int m = 0;
    while (m + 1 < c.n_modules && n >= c.end[m]) ++m;
    c.col_alpha[n] = __fdiv_rn(1.0f, __fmul_rn(c.act, c.scale[m]));
}

}  // namespace

cudaError_t launch_fused_col_alpha(const ColAlphaArgs &c, int32_t N, cudaStream_t st) {
    return launch_pdl(fused_col_alpha_kernel, dim3((unsigned)((N + 255) / 256)), dim3(256), 0, st, c, N);
}

cudaError_t launch_nvfp4_gemm(const GemmArgs &g, cudaStream_t st) {
    CUtensorMap ma, mb, msa, msb;
    if (!make_map(&ma, g.aq, (uint64_t)g.M, (uint64_t)g.K / 2, 128)) return cudaErrorInvalidValue;
    if (!make_map(&mb, g.bq, (uint64_t)g.N, (uint64_t)g.K / 2, 128)) return cudaErrorInvalidValue;
    // scales by TMA when their rows are whole 16-byte multiples per stage and 16-byte aligned
    const bool sf_tma = (g.K % BK == 0) && ((reinterpret_cast<uintptr_t>(g.as) | reinterpret_cast<uintptr_t>(g.bs)) & 15u) == 0;
    if (sf_tma) {
        if (!make_map(&msa, g.as, (uint64_t)g.M, (uint64_t)g.K / 16, 128, 16, CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !make_map(&msb, g.bs, (uint64_t)g.N, (uint64_t)g.K / 16, 256, 16, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    } else {
        msa = ma;   // unused
        msb = mb;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attrs[2];
    attrs[0].id = cudaLaunchAttributeClusterDimension;
    attrs[0].val.clusterDim.x = 2;
    attrs[0].val.clusterDim.y = 1;
    attrs[0].val.clusterDim.z = 1;
    attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = st;
    cfg.attrs = attrs;
    cfg.numAttrs = 2;
    // as many pairs as run at once (one CTA per SM), no more than there are 256 x 256 tiles;
    // the shared-memory attribute and the occupancy query are per device
    static PerDevice<int> max_pairs;
    int pairs = 0;
    const cudaError_t e = max_pairs.get(
        [&cfg](int, int &r) {
            cudaError_t x = cudaFuncSetAttribute(nvfp4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
            if (x != cudaSuccess) return x;
            cudaLaunchConfig_t q = cfg;
            q.gridDim = dim3(2);
            int clusters = 0;
            if ((x = cudaOccupancyMaxActiveClusters(&clusters, nvfp4_gemm_kernel, &q)) != cudaSuccess) return x;
            r = clusters > 0 ? clusters : 1;
            return cudaSuccess;
        },
        &pairs);
    if (e != cudaSuccess) return e;
    const int pair_tiles = ((g.N + 255) / 256) * ((g.M + 255) / 256);
    cfg.gridDim = dim3((unsigned)(2 * (pair_tiles < pairs ? pair_tiles : pairs)));
    return cudaLaunchKernelEx(&cfg, nvfp4_gemm_kernel, ma, mb, msa, msb, sf_tma ? 1 : 0, g.as, g.bs, g.alpha,
                              g.col_alpha, g.M, g.N, g.K, g.out_bf16 ? 1 : 0, g.y, g.status);
}

}  // namespace gdn
