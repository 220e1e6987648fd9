// Causal short convolution + SiLU on the layer's q/k/v channels, before the scan.
//
// "A Node-by-Node White-Box Walkthrough of a Quantized Hybrid Gated DeltaNet Language Model",
// Principais Contribuicoes, item 2 (the short convolutions on the layer's path), read as the
// depthwise causal convolution of width K <= 4 followed by SiLU:
//     y[t, c] = SiLU(sum_{j<K} w[c, j] x[t - (K - 1) + j, c]),
// where the inputs before a sequence's first token come from its carried state (its last K - 1
// inputs, oldest first) or are zero.
//
// HBM-bound work with little arithmetic, so the design is about memory-level parallelism and
// few instructions per element: each thread owns 8 channels (16-byte loads and stores, values
// in packed f32 pairs), keeps the last K - 1 inputs in registers and walks its tokens in order,
// crossing sequence boundaries by cu_seqlens. The output may be split into planes (q, k, v),
// each [T, width] contiguous, so the scan reads them without a copy. A second kernel writes
// every sequence's last K - 1 inputs; decode has one kernel that also shifts the state in place.
#include "common.cuh"
#include "kernels.h"

namespace gdn {
namespace {

constexpr int kConvThreads = 128;
constexpr int kConvTile = 8;       // rows per staged sub-tile
constexpr int kConvStages = 2;     // sub-tiles in the ring: kConvStages - 1 loads in flight
constexpr size_t kConvSmem = kConvStages * kConvTile * kConvThreads * 16 + kConvThreads * 2 * 4 * 16;
constexpr int kDecRows = 4;        // decode: batch rows per thread

__device__ __forceinline__ void seq_bounds(const int32_t *cu, int tokens_per_seq, int n, int &s0, int &s1) {
    if (cu) {
        s0 = cu[n];
        s1 = cu[n + 1];
    } else {
        s0 = n * tokens_per_seq;
        s1 = s0 + tokens_per_seq;
    }
}

// Sequence holding token t: the last n with start(n) <= t (so empty sequences are skipped).
__device__ __forceinline__ int seq_of(const int32_t *cu, int tokens_per_seq, int num_seqs, int t) {
    if (!cu) return t / tokens_per_seq;
    int lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if (cu[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ uint4 ld16(const void *base, size_t idx) {
    return *reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(base) + idx);
}

__device__ __forceinline__ void st16(void *base, size_t idx, uint4 v) {
    *reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(base) + idx) = v;
}

__device__ __forceinline__ void unpack8(uint4 u, f2_t (&x)[4]) {
    x[0] = bf16x2_to_f2(u.x);
    x[1] = bf16x2_to_f2(u.y);
    x[2] = bf16x2_to_f2(u.z);
    x[3] = bf16x2_to_f2(u.w);
}

// Output planes: plane p holds channels [start_p, end_p) as a contiguous [rows, end_p - start_p]
// block at offset rows * start_p.
struct Planes {
    int32_t end[4];
    int32_t n;
};

// Start of this thread's column in its plane (row 0) and the plane's row pitch.
__device__ __forceinline__ __nv_bfloat16 *plane_column(const Planes &pl, void *y, int rows, int c0, int &pitch) {
    int start = 0, width = pl.end[0];
#pragma unroll
    for (int p = 1; p < 4; ++p)
        if (p < pl.n && c0 >= pl.end[p - 1]) {
            start = pl.end[p - 1];
            width = pl.end[p] - start;
        }
    pitch = width;
    return reinterpret_cast<__nv_bfloat16 *>(y) + (size_t)rows * start + (c0 - start);
}

// Tap j of the thread's 8 channels as 4 pairs, from their 8 * K weights (channel-major).
template <int K>
__device__ __forceinline__ void pair_weights(const float (&flat)[8 * K], f2_t (&w2)[K][4]) {
#pragma unroll
    for (int j = 0; j < K; ++j)
#pragma unroll
        for (int p = 0; p < 4; ++p) w2[j][p] = f2(flat[(2 * p) * K + j], flat[(2 * p + 1) * K + j]);
}

// The weights of channel block cb (weight[c, j] at c * K + j: thread t's 8 channels are the
// 2K float4s from t * 2K on). They are read coalesced into shared memory, each thread's 2K
// float4s rotated by its index so that the threads of a quarter-warp hit different banks when
// each reads its own back; a block barrier separates the two. Every thread of the block calls it.
template <int K>
__device__ __forceinline__ void load_weights(const float *w, int cb, int C, float4 *wsm, f2_t (&w2)[K][4]) {
    const int tid = threadIdx.x;
    const float4 *wg = reinterpret_cast<const float4 *>(w) + (size_t)cb * kConvThreads * 2 * K;
    const int nf4 = C * K / 4 - cb * kConvThreads * 2 * K;
#pragma unroll
    for (int jj = 0; jj < 2 * K; ++jj) {
        const int f = tid + kConvThreads * jj;
        if (f < nf4) {
            const int tt = f / (2 * K), q = f % (2 * K);
            wsm[tt * 2 * K + (q + tt) % (2 * K)] = __ldg(wg + f);
        }
    }
    __syncthreads();
    float flat[8 * K];
#pragma unroll
    for (int q = 0; q < 2 * K; ++q) {
        const float4 f = wsm[tid * 2 * K + (q + tid) % (2 * K)];
        flat[4 * q] = f.x;
        flat[4 * q + 1] = f.y;
        flat[4 * q + 2] = f.z;
        flat[4 * q + 3] = f.w;
    }
    pair_weights<K>(flat, w2);
}

// SiLU(sum_{j<K-1} w_j h_j + w_{K-1} x) for 8 channels (h[j] is the input K - 1 - j tokens
// back), as 8 bf16: x / (1 + 2^(-x log2 e)) with the approximate exponential and reciprocal.
template <int K>
__device__ __forceinline__ uint4 conv_silu8(const f2_t (&w2)[K][4], const f2_t (&h2)[K > 1 ? K - 1 : 1][4],
                                            const f2_t (&x2)[4]) {
    const f2_t nlog2e = f2(-kLog2e, -kLog2e), one2 = f2(1.0f, 1.0f);
    uint4 out;
    uint32_t *ow = reinterpret_cast<uint32_t *>(&out);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        f2_t acc = mul2(w2[K - 1][p], x2[p]);
#pragma unroll
        for (int j = 0; j < K - 1; ++j) acc = fma2(w2[j][p], h2[j][p], acc);
        const f2_t t = mul2(acc, nlog2e);
        const f2_t d = add2(f2(exp2_approx(f2lo(t)), exp2_approx(f2hi(t))), one2);
        const f2_t yv = mul2(acc, f2(rcp_approx(f2lo(d)), rcp_approx(f2hi(d))));
        const __nv_bfloat162 hb = __floats2bfloat162_rn(f2lo(yv), f2hi(yv));
        ow[p] = *reinterpret_cast<const uint32_t *>(&hb);
    }
    return out;
}

template <int K>
__device__ __forceinline__ void shift_in(f2_t (&h2)[K > 1 ? K - 1 : 1][4], const f2_t (&x2)[4]) {
#pragma unroll
    for (int i = 0; i + 1 < K - 1; ++i)
#pragma unroll
        for (int p = 0; p < 4; ++p) h2[i][p] = h2[i + 1][p];
    if (K > 1) {
#pragma unroll
        for (int p = 0; p < 4; ++p) h2[K > 1 ? K - 2 : 0][p] = x2[p];
    }
}

// Persistent: block b owns channel block b % n_cblk (128 threads x 8 channels) and an equal
// share of the tokens; it walks them in sub-tiles of kConvTile rows, with the next
// kConvStages - 1 sub-tiles on their way into a ring in shared memory (cp.async, each thread
// its own 16-byte column, so no block barrier is needed) while it computes the current one. The history stays in registers
// across sub-tiles, so only the K - 1 rows before a block's share are read twice.
template <int K>
__global__ void __launch_bounds__(kConvThreads)
short_conv_kernel(const void *__restrict__ x, int64_t ldx, const float *__restrict__ w,
                  const int32_t *__restrict__ cu, int32_t tokens_per_seq, int32_t num_seqs, int32_t T, int32_t C,
                  const void *init_state, void *__restrict__ y, Planes pl, int32_t n_cblk) {
    extern __shared__ uint4 stage[];   // [kConvStages][kConvTile][kConvThreads], then the weights
    pdl_launch_dependents();
    pdl_wait();
    const int tid = threadIdx.x, cb = (int)(blockIdx.x % n_cblk);
    const int c0 = (cb * kConvThreads + tid) * 8;
    const int nj = gridDim.x / n_cblk, j = blockIdx.x / n_cblk;
    const int ra = (int)((int64_t)T * j / nj), rb = (int)((int64_t)T * (j + 1) / nj);
    if (ra >= rb) return;   // the whole block: an empty share
    const bool active = c0 < C;
    auto issue = [&](int ta, int buf) {
        const int tb = min(ta + kConvTile, rb);
        for (int t = ta; t < tb; ++t)
            cp_async16(&stage[(buf * kConvTile + (t - ta)) * kConvThreads + tid],
                       reinterpret_cast<const __nv_bfloat16 *>(x) + (size_t)t * ldx + c0);
        cp_async_commit();
    };
#pragma unroll
    for (int st = 0; st < kConvStages - 1; ++st) {
        if (active && ra + st * kConvTile < rb) issue(ra + st * kConvTile, st);
        else cp_async_commit();   // empty groups keep the group count fixed
    }
    f2_t w2[K][4];
    load_weights<K>(w, cb, C, reinterpret_cast<float4 *>(stage + kConvStages * kConvTile * kConvThreads), w2);
    if (!active) return;

    int n = seq_of(cu, tokens_per_seq, num_seqs, ra), s0, s1;
    seq_bounds(cu, tokens_per_seq, n, s0, s1);
    f2_t h2[K > 1 ? K - 1 : 1][4];
    auto fill_history = [&](int t) {   // the K - 1 inputs before token t of sequence n
#pragma unroll
        for (int i = 0; i < K - 1; ++i) {
            const int tp = t - (K - 1) + i;
            if (tp >= s0) {
                unpack8(ld16(x, (size_t)tp * ldx + c0), h2[i]);
            } else if (init_state) {
                unpack8(ld16(init_state, ((size_t)n * (K - 1) + (tp - s0 + K - 1)) * C + c0), h2[i]);
            } else {
#pragma unroll
                for (int p = 0; p < 4; ++p) h2[i][p] = 0ull;
            }
        }
    };
    fill_history(ra);
    int pitch;
    __nv_bfloat16 *ycol = plane_column(pl, y, T, c0, pitch);
    int buf = 0;
    for (int ta = ra; ta < rb; ta += kConvTile, buf = buf + 1 == kConvStages ? 0 : buf + 1) {
        // the ring slot computed in the previous iteration receives the sub-tile kConvStages - 1 ahead
        const int ahead = ta + (kConvStages - 1) * kConvTile;
        if (ahead < rb) issue(ahead, buf == 0 ? kConvStages - 1 : buf - 1);
        else cp_async_commit();
        cp_async_wait<kConvStages - 1>();   // all but the newest kConvStages - 1 groups: this sub-tile
        const uint4 *rows = &stage[buf * kConvTile * kConvThreads + tid];
        if (ta + kConvTile <= min(rb, s1)) {
            // whole sub-tile inside sequence n: unrolled, the history rotates by renaming
#pragma unroll
            for (int r = 0; r < kConvTile; ++r) {
                f2_t x2[4];
                unpack8(rows[r * kConvThreads], x2);
                *reinterpret_cast<uint4 *>(ycol + (size_t)(ta + r) * pitch) = conv_silu8<K>(w2, h2, x2);
                shift_in<K>(h2, x2);
            }
            continue;
        }
        const int tb = min(ta + kConvTile, rb);
        for (int t = ta; t < tb; ++t) {
            while (t >= s1 && n + 1 < num_seqs) {   // the next non-empty sequence starts at t
                ++n;
                seq_bounds(cu, tokens_per_seq, n, s0, s1);
                if (t >= s0 && t < s1) fill_history(t);
            }
            f2_t x2[4];
            unpack8(rows[(t - ta) * kConvThreads], x2);
            *reinterpret_cast<uint4 *>(ycol + (size_t)t * pitch) = conv_silu8<K>(w2, h2, x2);
            shift_in<K>(h2, x2);
        }
    }
}

// final_state[n][i] = the input K - 1 - i positions before the sequence's end: from x when
// inside the sequence, else from the carried state (entry len + i), else zero. One thread per
// (sequence, 8 channels), entries in ascending order, so final_state may be initial_state.
__global__ void __launch_bounds__(kConvThreads)
short_conv_state_kernel(const void *__restrict__ x, int64_t ldx, const int32_t *__restrict__ cu,
                        int32_t tokens_per_seq, int32_t num_seqs, int32_t C, int32_t K, const void *init_state,
                        void *final_state) {
    pdl_launch_dependents();
    pdl_wait();
    const int c0 = (blockIdx.x * kConvThreads + threadIdx.x) * 8;
    const int n = blockIdx.y;
    if (c0 >= C || n >= num_seqs) return;
    int s0, s1;
    seq_bounds(cu, tokens_per_seq, n, s0, s1);
    const int len = s1 - s0;
    for (int i = 0; i < K - 1; ++i) {
        const int tp = s1 - (K - 1) + i;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (tp >= s0) v = ld16(x, (size_t)tp * ldx + c0);
        else if (init_state) v = ld16(init_state, ((size_t)n * (K - 1) + len + i) * C + c0);
        st16(final_state, ((size_t)n * (K - 1) + i) * C + c0, v);
    }
}

// One token per sequence, kDecRows sequences per thread: y from the carried state and x, then
// the state shifted by one. The inputs are requested before the weights.
template <int K>
__global__ void __launch_bounds__(kConvThreads)
short_conv_decode_kernel(const void *__restrict__ x, int64_t ldx, const float *__restrict__ w, int32_t B,
                         int32_t C, void *state, void *__restrict__ y, Planes pl) {
    __shared__ float4 wsm[kConvThreads * 2 * K];
    pdl_launch_dependents();
    pdl_wait();
    const int tid = threadIdx.x, cb = blockIdx.x;
    const int c0 = (cb * kConvThreads + tid) * 8;
    const int b0 = blockIdx.y * kDecRows;
    const bool active = c0 < C;
    uint4 xr[kDecRows], sr[kDecRows][K > 1 ? K - 1 : 1];
#pragma unroll
    for (int r = 0; r < kDecRows; ++r)
        if (active && b0 + r < B) {
            xr[r] = ld16(x, (size_t)(b0 + r) * ldx + c0);
#pragma unroll
            for (int i = 0; i < K - 1; ++i) sr[r][i] = ld16(state, ((size_t)(b0 + r) * (K - 1) + i) * C + c0);
        }
    f2_t w2[K][4];
    load_weights<K>(w, cb, C, wsm, w2);
    if (!active) return;
    int pitch;
    __nv_bfloat16 *ycol = plane_column(pl, y, B, c0, pitch);
#pragma unroll
    for (int r = 0; r < kDecRows; ++r) {
        const int bi = b0 + r;
        if (bi >= B) break;
        f2_t h2[K > 1 ? K - 1 : 1][4], x2[4];
#pragma unroll
        for (int i = 0; i < K - 1; ++i) unpack8(sr[r][i], h2[i]);
        unpack8(xr[r], x2);
        *reinterpret_cast<uint4 *>(ycol + (size_t)bi * pitch) = conv_silu8<K>(w2, h2, x2);
#pragma unroll
        for (int i = 0; i < K - 1; ++i)
            st16(state, ((size_t)bi * (K - 1) + i) * C + c0, i + 1 < K - 1 ? sr[r][i + 1 < K - 1 ? i + 1 : 0] : xr[r]);
    }
}

Planes make_planes(const ConvArgs &a) {
    Planes pl{{a.C, a.C, a.C, a.C}, 1};
    if (a.n_parts > 1) {
        pl.n = a.n_parts;
        for (int p = 0; p < 4; ++p) pl.end[p] = p < a.n_parts ? a.part_end[p] : a.C;
    }
    return pl;
}

// Grid of the persistent prefill kernel: as many blocks as fit on the device at once, rounded
// down to a whole number of channel blocks, but no more token shares than sub-tiles.
template <int K>
int conv_grid(int n_cblk, int T) {
    struct Occ {
        int per_sm, sms;
    };
    static PerDevice<Occ> occ;
    Occ o{};
    const cudaError_t e = occ.get(
        [](int dev, Occ &r) {
            cudaError_t x = cudaFuncSetAttribute(short_conv_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)kConvSmem);
            int b = 0, m = 0;
            if (x == cudaSuccess)
                x = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, short_conv_kernel<K>, kConvThreads, kConvSmem);
            if (x == cudaSuccess) x = cudaDeviceGetAttribute(&m, cudaDevAttrMultiProcessorCount, dev);
            r.per_sm = b > 0 ? b : 1;
            r.sms = m;
            return x;
        },
        &o);
    if (e != cudaSuccess) return -1;
    const int shares = max(1, min(o.per_sm * o.sms / n_cblk, (T + kConvTile - 1) / kConvTile));
    return shares * n_cblk;
}

template <int K>
cudaError_t launch_conv_k(const ConvArgs &a, cudaStream_t st) {
    const int n_cblk = (a.C / 8 + kConvThreads - 1) / kConvThreads;
    const Planes pl = make_planes(a);
    if (a.decode)
        return launch_pdl(short_conv_decode_kernel<K>,
                          dim3((unsigned)n_cblk, (unsigned)((a.num_seqs + kDecRows - 1) / kDecRows)),
                          dim3(kConvThreads), 0, st, a.x, a.ldx, a.w, a.num_seqs, a.C, a.final_state, a.y, pl);
    if (a.T > 0) {
        const int grid = conv_grid<K>(n_cblk, a.T);
        if (grid < 0) return cudaErrorUnknown;
        const cudaError_t e = launch_pdl(short_conv_kernel<K>, dim3((unsigned)grid), dim3(kConvThreads), kConvSmem,
                                         st, a.x, a.ldx, a.w, a.cu_seqlens, a.tokens_per_seq, a.num_seqs, a.T,
                                         a.C, a.init_state, a.y, pl, (int32_t)n_cblk);
        if (e != cudaSuccess) return e;
    }
    if (a.final_state && K > 1)
        return launch_pdl(short_conv_state_kernel, dim3((unsigned)n_cblk, (unsigned)a.num_seqs), dim3(kConvThreads),
                          0, st, a.x, a.ldx, a.cu_seqlens, a.tokens_per_seq, a.num_seqs, a.C, (int32_t)K,
                          a.init_state, a.final_state);
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_short_conv(const ConvArgs &a, cudaStream_t st) {
    switch (a.K) {
        case 1: return launch_conv_k<1>(a, st);
        case 2: return launch_conv_k<2>(a, st);
        case 3: return launch_conv_k<3>(a, st);
        case 4: return launch_conv_k<4>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gdn
