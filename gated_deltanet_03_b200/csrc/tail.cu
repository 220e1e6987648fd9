// The gated tail before the output projection, and the NVFP4 activation encoder.
//
// "Red Lite dev15d - DeltaNet gated tail + Q4_K output projection", Pinned graph
// semantics, steps 1-5: per value head of D values, RMSNorm with one shared weight,
// times SiLU(z), flattened head-major (which is the identity on the [M, Hv, D] memory).
// "Why Gated DeltaNet Survives 4-Bit Quantization", abstract, mechanism i: NVFP4 with
// 16-element block scales (E4M3) over E2M1 values and an fp32 global scale.
//
// Both kernels are HBM-bound streams: 16-byte loads, D/8 lanes per head row, the mean of
// squares as a lane-group shuffle reduction, and (NVFP4) the block maximum over a pair
// of lanes, then the hardware E4M3 / E2M1 conversions.
#include "common.cuh"
#include "kernels.h"

namespace gdn {

constexpr int kTailThreads = 256;


// Eight consecutive values as loaded (bf16: one 16-byte word; fp32: two), converted on use.
template <bool BF16>
struct Raw8 {
    uint4 a, b;
    __device__ __forceinline__ void load(const void *base, size_t idx) {
        if constexpr (BF16) {
            a = *reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(base) + idx);
        } else {
            const uint4 *p = reinterpret_cast<const uint4 *>(reinterpret_cast<const float *>(base) + idx);
            a = p[0];
            b = p[1];
        }
    }
    __device__ __forceinline__ void get(float (&x)[8]) const {
        f2_t v[4];
        get2(v);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            x[2 * k] = f2lo(v[k]);
            x[2 * k + 1] = f2hi(v[k]);
        }
    }
    __device__ __forceinline__ void get2(f2_t (&v)[4]) const {
        if constexpr (BF16) {
            v[0] = bf16x2_to_f2(a.x); v[1] = bf16x2_to_f2(a.y); v[2] = bf16x2_to_f2(a.z); v[3] = bf16x2_to_f2(a.w);
        } else {
            v[0] = f2(__uint_as_float(a.x), __uint_as_float(a.y)); v[1] = f2(__uint_as_float(a.z), __uint_as_float(a.w));
            v[2] = f2(__uint_as_float(b.x), __uint_as_float(b.y)); v[3] = f2(__uint_as_float(b.z), __uint_as_float(b.w));
        }
    }
};

// Rows handled per thread per pass: all their loads are issued before any is consumed, so
// that enough bytes are in flight to cover the HBM latency.
constexpr int kTailUnroll = 4;

template <int D, bool IN_BF16, bool OUT_BF16, bool NVFP4>
__global__ void __launch_bounds__(kTailThreads)
gated_rmsnorm_kernel(const void *__restrict__ o, const void *__restrict__ z,
                     const float *__restrict__ w, float eps, int64_t rows,
                     void *__restrict__ y, float gs, uint8_t *__restrict__ xq,
                     uint8_t *__restrict__ xs) {
    pdl_launch_dependents();
    pdl_wait();
    constexpr int LANES = D / 8;                 // lanes per head row, 8 values each
    constexpr int RPB = kTailThreads / LANES;    // head rows per block pass
    constexpr int U = kTailUnroll;
    // NVFP4: the per-block factor r = gs / E4M3(sb) for every scale code (sb = 0: r = 0)
    __shared__ float r_tab[128];
    if constexpr (NVFP4) {
        nvfp4_fill_r_tab(r_tab, gs, threadIdx.x);
        __syncthreads();
    }
    const int lane_in_row = threadIdx.x % LANES;
    const int col = lane_in_row * 8;
    f2_t w2[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) w2[k] = f2(w[col + 2 * k], w[col + 2 * k + 1]);
    const float inv_d = 1.0f / (float)D;
    const int64_t stride = (int64_t)gridDim.x * RPB;

    // the loop condition is uniform over the block (the shuffles below need whole warps)
    for (int64_t row0 = (int64_t)blockIdx.x * RPB + threadIdx.x / LANES; row0 - threadIdx.x / LANES < rows;
         row0 += U * stride) {
        Raw8<IN_BF16> ro[U], rz[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = row0 + u * stride;
            const size_t base = (size_t)(row < rows ? row : 0) * D + col;
            ro[u].load(o, base);
            rz[u].load(z, base);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = row0 + u * stride;
            const bool live = row < rows;
            const size_t base = (size_t)(live ? row : 0) * D + col;
            f2_t o2[4], z2[4];
            ro[u].get2(o2);
            rz[u].get2(z2);
            f2_t y2[4];
            gated_row8<LANES>(o2, z2, w2, inv_d, eps, y2);
            if constexpr (!NVFP4) {
                if (live) {
                    if constexpr (OUT_BF16) {
                        uint4 u4;
                        uint32_t *pw = reinterpret_cast<uint32_t *>(&u4);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const __nv_bfloat162 hb = __floats2bfloat162_rn(f2lo(y2[k]), f2hi(y2[k]));
                            pw[k] = *reinterpret_cast<const uint32_t *>(&hb);
                        }
                        *reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(y) + base) = u4;
                    } else {
                        float4 *p = reinterpret_cast<float4 *>(reinterpret_cast<float *>(y) + base);
                        p[0] = make_float4(f2lo(y2[0]), f2hi(y2[0]), f2lo(y2[1]), f2hi(y2[1]));
                        p[1] = make_float4(f2lo(y2[2]), f2hi(y2[2]), f2lo(y2[3]), f2hi(y2[3]));
                    }
                }
            } else {
                uint32_t packed, sb;
                nvfp4_encode_row8(y2, gs, r_tab, packed, sb);
                if (live) {
                    reinterpret_cast<uint32_t *>(xq)[base / 8] = packed;
                    if ((lane_in_row & 1) == 0) xs[base / 16] = (uint8_t)sb;
                }
            }
        }
    }
}

template <int D, bool IN_BF16, bool OUT_BF16, bool NVFP4>
static cudaError_t launch_tail_t(const TailArgs &t, cudaStream_t st) {
    const int64_t rows = (int64_t)t.M * t.Hv;
    if (rows == 0) return cudaSuccess;
    constexpr int RPB = kTailThreads / (D / 8);
    int64_t blocks = (rows + RPB * kTailUnroll - 1) / (RPB * kTailUnroll);
    const int64_t cap = 148 * 8;
    if (blocks > cap) blocks = cap;
    return launch_pdl(gated_rmsnorm_kernel<D, IN_BF16, OUT_BF16, NVFP4>, dim3((unsigned)blocks), dim3(kTailThreads), 0,
                      st, t.o, t.z, t.w, t.eps, rows, t.y, t.gs, t.xq, t.xs);
}

template <bool NVFP4, int D>
static cudaError_t launch_tail_d(const TailArgs &t, cudaStream_t st) {
    if (t.in_bf16) {
        return t.out_bf16 ? launch_tail_t<D, true, true, NVFP4>(t, st) : launch_tail_t<D, true, false, NVFP4>(t, st);
    }
    return t.out_bf16 ? launch_tail_t<D, false, true, NVFP4>(t, st) : launch_tail_t<D, false, false, NVFP4>(t, st);
}

template <bool NVFP4>
static cudaError_t launch_tail(const TailArgs &t, cudaStream_t st) {
    switch (t.D) {
        case 16: return launch_tail_d<NVFP4, 16>(t, st);
        case 32: return launch_tail_d<NVFP4, 32>(t, st);
        case 64: return launch_tail_d<NVFP4, 64>(t, st);
        case 128: return launch_tail_d<NVFP4, 128>(t, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gated_rmsnorm(const TailArgs &t, cudaStream_t st) { return launch_tail<false>(t, st); }
cudaError_t launch_gated_rmsnorm_nvfp4(const TailArgs &t, cudaStream_t st) { return launch_tail<true>(t, st); }

// One thread per 16-value block and pass position: two 16-byte loads (bf16) or four (fp32), one
// 8-byte store of codes and one byte of scale; four blocks per thread per pass, loads first.
template <bool IN_BF16>
__global__ void __launch_bounds__(256)
nvfp4_quantize_kernel(const void *__restrict__ x, int64_t nblocks, float gs,
                      uint8_t *__restrict__ xq, uint8_t *__restrict__ xs) {
    pdl_launch_dependents();
    pdl_wait();
    constexpr int U = 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b0 < nblocks; b0 += U * stride) {
        Raw8<IN_BF16> rlo[U], rhi[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t blk = b0 + u * stride < nblocks ? b0 + u * stride : b0;
            rlo[u].load(x, (size_t)blk * 16);
            rhi[u].load(x, (size_t)blk * 16 + 8);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t blk = b0 + u * stride;
            if (blk >= nblocks) break;
            float lo[8], hi[8];
            rlo[u].get(lo);
            rhi[u].get(hi);
            float r;
            const uint32_t sb = nvfp4_block_scale(fmaxf(amax8(lo), amax8(hi)), gs, r);
            const uint2 packed = make_uint2(nvfp4_pack8(lo, r), nvfp4_pack8(hi, r));
            reinterpret_cast<uint2 *>(xq)[blk] = packed;
            xs[blk] = (uint8_t)sb;
        }
    }
}

// E2M1 and E4M3 values from their bit fields (the formats' definitions: E2M1 = sign, 2-bit
// exponent with bias 1, 1-bit mantissa; E4M3 = sign, 4-bit exponent with bias 7, 3-bit mantissa,
// exponent 0 subnormal, 0x7F / 0xFF NaN).
GDN_DEV float e2m1_value(uint32_t c) {
    const uint32_t e = (c >> 1) & 3u, m = c & 1u;
    const float mag = e == 0 ? 0.5f * (float)m : (1.0f + 0.5f * (float)m) * (float)(1u << (e - 1));
    return (c & 8u) ? -mag : mag;
}
GDN_DEV float e4m3_value(uint32_t b) {
    const uint32_t e = (b >> 3) & 15u, m = b & 7u;
    if (e == 15u && m == 7u) return __int_as_float(0x7fc00000);
    const float mag = e == 0 ? (float)m * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
    return (b & 0x80u) ? -mag : mag;
}

// x_hat = E2M1(code) * E4M3(block scale) / gs: the product is exact in fp32 and the IEEE
// division rounds it once, so each value is the correctly rounded fp32 quotient. One thread per
// 16-value block (8 code bytes, 1 scale byte).
template <bool OUT_BF16>
__global__ void __launch_bounds__(256)
nvfp4_dequantize_kernel(const uint8_t *__restrict__ xq, const uint8_t *__restrict__ xs, int64_t nblocks, float gs,
                        void *__restrict__ y) {
    pdl_launch_dependents();
    pdl_wait();
    for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < nblocks;
         blk += (int64_t)gridDim.x * blockDim.x) {
        const uint2 codes = *reinterpret_cast<const uint2 *>(xq + blk * 8);
        const float sc = e4m3_value(xs[blk]);
        float v[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t byte = ((i < 4 ? codes.x : codes.y) >> (8 * (i & 3))) & 0xFFu;
            v[2 * i] = __fdiv_rn(e2m1_value(byte & 15u) * sc, gs);
            v[2 * i + 1] = __fdiv_rn(e2m1_value(byte >> 4) * sc, gs);
        }
        if constexpr (OUT_BF16) {
            uint4 u[2];
            __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(u);
#pragma unroll
            for (int i = 0; i < 8; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(y) + blk * 16);
            dst[0] = u[0];
            dst[1] = u[1];
        } else {
            float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(y) + blk * 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
    }
}

cudaError_t launch_nvfp4_dequantize(const uint8_t *xq, const uint8_t *xs, int32_t M, int32_t K, float gs,
                                    bool out_bf16, void *y, cudaStream_t st) {
    const int64_t nblocks = (int64_t)M * (K / 16);
    if (nblocks == 0) return cudaSuccess;
    int64_t grid = (nblocks + 255) / 256;
    if (grid > 148 * 8) grid = 148 * 8;
    if (out_bf16) return launch_pdl(nvfp4_dequantize_kernel<true>, dim3((unsigned)grid), dim3(256), 0, st, xq, xs, nblocks, gs, y);
    return launch_pdl(nvfp4_dequantize_kernel<false>, dim3((unsigned)grid), dim3(256), 0, st, xq, xs, nblocks, gs, y);
}

cudaError_t launch_nvfp4_quantize(const void *x, bool in_bf16, int32_t M, int32_t K, float gs,
                                  uint8_t *xq, uint8_t *xs, cudaStream_t st) {
    const int64_t nblocks = (int64_t)M * (K / 16);
    if (nblocks == 0) return cudaSuccess;
    int64_t grid = (nblocks + 1023) / 1024;
    if (grid > 148 * 8) grid = 148 * 8;
    if (in_bf16) return launch_pdl(nvfp4_quantize_kernel<true>, dim3((unsigned)grid), dim3(256), 0, st, x, nblocks, gs, xq, xs);
    return launch_pdl(nvfp4_quantize_kernel<false>, dim3((unsigned)grid), dim3(256), 0, st, x, nblocks, gs, xq, xs);
}

}  // namespace gdn
