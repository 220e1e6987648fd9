// Internal launcher interface between the C entry points (api.cu) and the kernels.
// Every launcher enqueues on the given stream and returns the launch's cudaError_t.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <utility>

namespace gdn {

// Per-device set-up (function attributes, occupancy queries): a kernel attribute such as the
// dynamic shared-memory limit belongs to one device, so each launcher keeps one record per
// device index and fills it under a lock the first time it runs with that device current.
// A failed set-up is not recorded and runs again on the next call.
constexpr int kMaxDevices = 64;
template <typename Rec>
struct PerDevice {
    Rec rec[kMaxDevices] = {};
    bool done[kMaxDevices] = {};
    std::mutex mu;
    // The current device's record, filled by init(dev, rec) on first use.
    template <typename F>
    cudaError_t get(F &&init, Rec *out) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
        std::lock_guard<std::mutex> lock(mu);
        if (!done[dev]) {
            Rec r{};
            if ((e = init(dev, r)) != cudaSuccess) return e;
            rec[dev] = r;
            done[dev] = true;
        }
        *out = rec[dev];
        return cudaSuccess;
    }
};

// Launch with programmatic stream serialization (see pdl_wait in common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

struct RecurrentArgs {
    const void *q, *k, *v;
    const float *a, *b, *A_log, *dt_bias;
    const int32_t *cu_seqlens;   // device [num_seqs + 1], or null: seq n = [n*T1, (n+1)*T1)
    int32_t tokens_per_seq;      // T1 when cu_seqlens is null
    int32_t num_seqs, Hk, Hv, D;
    float scale;
    int32_t l2norm;
    bool in_bf16, out_bf16;
    const float *S0;             // may be null (zero state); may alias S_out
    float *S_out;                // may be null
    void *o;                     // may be null (no outputs)
    const int32_t *n_apply;      // device [num_seqs] or null: sequence n takes only its first n_apply[n] tokens
};
cudaError_t launch_recurrent(const RecurrentArgs &r, cudaStream_t st);

// One decode token per sequence (d = 128, bf16) fused with the gated RMSNorm and the NVFP4 encode.
struct DecodeTailArgs {
    const void *q, *k, *v;       // [B, Hk, 128], [B, Hk, 128], [B, Hv, 128] bf16
    const float *a, *b, *A_log, *dt_bias;
    int32_t B, Hk, Hv;
    float scale;
    int32_t l2norm;
    float *state;                // [B, Hv, 128, 128] fp32, in place
    const void *z;               // [B, Hv, 128] bf16
    const float *norm_w;         // [128]
    float eps, gs;
    uint8_t *xq, *xs;            // [B, Hv * 64], [B, Hv * 8]
    void *o;                     // [B, Hv, 128] bf16 or null
};
cudaError_t launch_decode_gated_nvfp4(const DecodeTailArgs &d, cudaStream_t st);

struct ChunkedArgs {
    const void *q, *k, *v;       // bf16
    const float *a, *b, *A_log, *dt_bias;
    const int32_t *cu_seqlens;   // may be null (one sequence of T tokens)
    int32_t T, num_seqs, Hk, Hv;
    float scale;
    int32_t l2norm;
    bool out_bf16;
    const float *S0;
    float *S_out;
    void *o;
    void *ws;                    // workspace of chunked_workspace_bytes(T, num_seqs, Hk, Hv) bytes
    int *status;
    // fused gated RMSNorm + NVFP4 encode of o (when xq is set; o may then be null):
    const void *z;               // [T, Hv, 128] bf16
    const float *norm_w;         // [128]
    float eps, gs;
    uint8_t *xq, *xs;            // [T, Hv * 64], [T, Hv * 8]
};
size_t chunked_workspace_bytes(int T, int num_seqs, int Hk, int Hv);
// The prep grid's y dimension counts the chunk slots (T / 64 + num_seqs), at most 65535.
inline bool chunked_size_ok(int T, int num_seqs) { return (int64_t)T / 64 + num_seqs <= 65535; }
cudaError_t launch_chunked(const ChunkedArgs &c, cudaStream_t st);

struct TailArgs {
    const void *o, *z;
    const float *w;
    float eps;
    int32_t M, Hv, D;
    bool in_bf16;
    void *y;                     // gated output (plain variant)
    bool out_bf16;
    float gs;                    // NVFP4 variant: encode scale, outputs xq/xs
    uint8_t *xq, *xs;
};
cudaError_t launch_gated_rmsnorm(const TailArgs &t, cudaStream_t st);
cudaError_t launch_gated_rmsnorm_nvfp4(const TailArgs &t, cudaStream_t st);

cudaError_t launch_nvfp4_quantize(const void *x, bool in_bf16, int32_t M, int32_t K, float gs,
                                  uint8_t *xq, uint8_t *xs, cudaStream_t st);
cudaError_t launch_nvfp4_dequantize(const uint8_t *xq, const uint8_t *xs, int32_t M, int32_t K, float gs,
                                    bool out_bf16, void *y, cudaStream_t st);

struct GemmArgs {
    const uint8_t *aq, *as, *bq, *bs;
    float alpha;
    int32_t M, N, K;
    bool out_bf16;
    void *y;
    int *status;
    const float *col_alpha;      // [N] per-column factor, or null: alpha for every column
};
cudaError_t launch_nvfp4_gemm(const GemmArgs &g, cudaStream_t st);

// Per-column factors of a fused-module weight: column n of module m gets 1 / (act * scale[m]).
constexpr int kMaxModules = 64;
struct ColAlphaArgs {
    int32_t end[kMaxModules];    // exclusive end column of each module
    float scale[kMaxModules];
    int32_t n_modules;
    float act;
    float *col_alpha;
};
cudaError_t launch_fused_col_alpha(const ColAlphaArgs &c, int32_t N, cudaStream_t st);

// Output projection with Q4_K weights: y [M, N] = a [M, K] (bf16) times the decoded w [N, K]^T.
struct Q4kGemmArgs {
    const void *a;               // bf16 [M, K]
    const uint8_t *w;            // [N, K / 256 * 144] Q4_K blocks
    int32_t M, N, K;
    bool out_bf16;
    void *y;
    int *status;
};
cudaError_t launch_q4k_gemm(const Q4kGemmArgs &g, cudaStream_t st);

struct ConvArgs {
    const void *x;               // bf16 rows of ldx elements; channels [0, C) are convolved
    int64_t ldx;
    const float *w;              // [C, K]
    const int32_t *cu_seqlens;   // device [num_seqs + 1], or null: num_seqs runs of tokens_per_seq
    int32_t tokens_per_seq, num_seqs, T, C, K;
    const void *init_state;      // bf16 [num_seqs, K - 1, C] or null (zero history)
    void *final_state;           // bf16 [num_seqs, K - 1, C] or null; decode: the state, in place
    void *y;                     // bf16, planes of [T, width] (one plane: [T, C])
    int32_t part_end[4];
    int32_t n_parts;
    bool decode;                 // one token per sequence, state shifted in place
};
cudaError_t launch_short_conv(const ConvArgs &a, cudaStream_t st);

}  // namespace gdn
