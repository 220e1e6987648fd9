// C entry points declared in include/gdn.h: host-side argument checks, kernel variant
// selection and launches on the caller's stream. No device memory is allocated here; the
// only library-owned device object is the control block (status word, wait limit, test switches).
#include <climits>
#include <cmath>
#include <cstdio>

#include "common.cuh"
#include "kernels.h"

namespace {

__device__ gdn::DeviceCtl g_device_ctl = {0, 0u, gdn::kWaitLimitNs};

// Device address of the status word on the current device (looked up once per device, under a
// lock; a device reset between calls is not supported, see gdn.h).
int *status_ptr() {
    static gdn::PerDevice<int *> addr;
    int *p = nullptr;
    if (addr.get(
            [](int, int *&r) {
                void *a = nullptr;
                const cudaError_t e = cudaGetSymbolAddress(&a, g_device_ctl);
                r = static_cast<int *>(a);
                return e;
            },
            &p) != cudaSuccess)
        return nullptr;
    return p;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool head_ok(int32_t d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool dtype_ok(gdn_dtype t) { return t == GDN_BF16 || t == GDN_F32; }

gdn_status launched(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

}  // namespace

extern "C" {

int32_t gdn_version(void) { return 100; }

const char *gdn_status_string(gdn_status s) {
    switch (s) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARG: return "invalid argument";
        case GDN_ERR_UNSUPPORTED: return "unsupported size or dtype";
        case GDN_ERR_CUDA: return "CUDA error";
        case GDN_ERR_TIMEOUT: return "device-side wait timed out";
        case GDN_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

gdn_status gdn_get_device_status(gdn_stream_t stream) {
    int *p = status_ptr();
    if (!p) return GDN_ERR_CUDA;
    int h = 0;
    if (cudaMemcpyAsync(&h, p, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess) return GDN_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GDN_ERR_CUDA;
    if (h != 0) {
        const int zero = 0;
        if (cudaMemcpyAsync(p, &zero, sizeof(int), cudaMemcpyHostToDevice, stream) != cudaSuccess) return GDN_ERR_CUDA;
        if (cudaStreamSynchronize(stream) != cudaSuccess) return GDN_ERR_CUDA;
    }
    return static_cast<gdn_status>(h);
}

gdn_status gdn_debug_set_wait(uint64_t wait_limit_ns, uint32_t inject_flags) {
    int *p = status_ptr();
    if (!p) return GDN_ERR_CUDA;
    if (wait_limit_ns == 0) wait_limit_ns = gdn::kWaitLimitNs;
    if (wait_limit_ns > gdn::kWaitLimitNs || (inject_flags & ~gdn::kInjectSkipPrepLoads) != 0u) return GDN_ERR_INVALID_ARG;
    gdn::DeviceCtl *ctl = reinterpret_cast<gdn::DeviceCtl *>(p);
    const unsigned long long lim = wait_limit_ns;
    const unsigned int fl = inject_flags;
    if (cudaMemcpy(&ctl->wait_limit_ns, &lim, sizeof(lim), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(&ctl->flags, &fl, sizeof(fl), cudaMemcpyHostToDevice) != cudaSuccess)
        return GDN_ERR_CUDA;
    return GDN_OK;
}

size_t gdn_prefill_workspace_bytes(int32_t T, int32_t num_seqs, int32_t Hk, int32_t Hv, int32_t Dk,
                                   int32_t Dv) {
    if (T <= 0 || num_seqs < 1 || Hk < 1 || Hv < 1 || Dk != 128 || Dv != 128) return 0;
    return gdn::chunked_workspace_bytes(T, num_seqs, Hk, Hv);
}

gdn_status gdn_prefill_chunked(const void *q, const void *k, const void *v, const float *a, const float *b,
                               const float *A_log, const float *dt_bias, const int32_t *cu_seqlens,
                               int32_t num_seqs, int32_t T, int32_t Hk, int32_t Hv, int32_t Dk, int32_t Dv,
                               float scale, int32_t qk_l2norm, gdn_dtype in_dtype,
                               const float *initial_state, float *final_state, void *o,
                               gdn_dtype out_dtype, void *workspace, size_t workspace_bytes,
                               gdn_stream_t stream) {
    if (T < 0 || num_seqs < 1 || Hk < 1 || Hv < 1 || Hv % Hk != 0) return GDN_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return GDN_ERR_INVALID_ARG;
    if (!cu_seqlens && num_seqs != 1) return GDN_ERR_INVALID_ARG;
    if (Dk != Dv) return GDN_ERR_UNSUPPORTED;
    if (!head_ok(Dk)) return GDN_ERR_UNSUPPORTED;
    if (T > 0) {
        if (!q || !k || !v || !a || !b || !o) return GDN_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return GDN_ERR_INVALID_ARG;
    }
    if (!A_log || !dt_bias) return GDN_ERR_INVALID_ARG;
    if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
        return GDN_ERR_INVALID_ARG;

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (Dk == 128 && in_dtype == GDN_BF16 && T > 0) {
        if (!gdn::chunked_size_ok(T, num_seqs)) return GDN_ERR_UNSUPPORTED;
        const size_t need = gdn::chunked_workspace_bytes(T, num_seqs, Hk, Hv);
        if (!workspace || workspace_bytes < need || !aligned16(workspace)) return GDN_ERR_WORKSPACE;
        gdn::ChunkedArgs c{q, k, v, a, b, A_log, dt_bias, cu_seqlens, T, num_seqs, Hk, Hv, scale, qk_l2norm,
                           out_dtype == GDN_BF16, initial_state, final_state, o, workspace, status_ptr()};
        cudaError_t e = gdn::launch_chunked(c, st);
        if (e != cudaErrorNotSupported) return launched(e);
    }
    gdn::RecurrentArgs r{q, k, v, a, b, A_log, dt_bias, cu_seqlens, T, num_seqs, Hk, Hv, Dk, scale,
                         qk_l2norm, in_dtype == GDN_BF16, out_dtype == GDN_BF16, initial_state,
                         final_state, o};
    return launched(gdn::launch_recurrent(r, st));
}

gdn_status gdn_prefill_chunked_gated_nvfp4(const void *q, const void *k, const void *v, const float *a,
                                           const float *b, const float *A_log, const float *dt_bias,
                                           const int32_t *cu_seqlens, int32_t num_seqs, int32_t T, int32_t Hk,
                                           int32_t Hv, int32_t Dk, int32_t Dv, float scale, int32_t qk_l2norm,
                                           gdn_dtype in_dtype, const float *initial_state, float *final_state,
                                           void *o, const void *z, const float *norm_weight, float eps,
                                           float global_scale, uint8_t *xq, uint8_t *xs, void *workspace,
                                           size_t workspace_bytes, gdn_stream_t stream) {
    if (T < 0 || num_seqs < 1 || Hk < 1 || Hv < 1 || Hv % Hk != 0) return GDN_ERR_INVALID_ARG;
    if (!cu_seqlens && num_seqs != 1) return GDN_ERR_INVALID_ARG;
    if (Dk != 128 || Dv != 128 || in_dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (!A_log || !dt_bias) return GDN_ERR_INVALID_ARG;
    if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
        return GDN_ERR_INVALID_ARG;
    if (T == 0)   // nothing to encode; the final state is the initial one
        return gdn_prefill_chunked(q, k, v, a, b, A_log, dt_bias, cu_seqlens, num_seqs, T, Hk, Hv, Dk, Dv, scale,
                                   qk_l2norm, in_dtype, initial_state, final_state, o, GDN_BF16, workspace,
                                   workspace_bytes, stream);
    if (!q || !k || !v || !a || !b || !z || !norm_weight || !xq || !xs) return GDN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(z) || (o && !aligned16(o)) ||
        (reinterpret_cast<uintptr_t>(xq) & 3u))
        return GDN_ERR_INVALID_ARG;
    if (!gdn::chunked_size_ok(T, num_seqs)) return GDN_ERR_UNSUPPORTED;
    const size_t need = gdn::chunked_workspace_bytes(T, num_seqs, Hk, Hv);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return GDN_ERR_WORKSPACE;
    gdn::ChunkedArgs c{q, k, v, a, b, A_log, dt_bias, cu_seqlens, T, num_seqs, Hk, Hv, scale, qk_l2norm, true,
                       initial_state, final_state, o, workspace, status_ptr(), z, norm_weight, eps, global_scale,
                       xq, xs};
    return launched(gdn::launch_chunked(c, reinterpret_cast<cudaStream_t>(stream)));
}

gdn_status gdn_decode_step(const void *q, const void *k, const void *v, const float *a, const float *b,
                           const float *A_log, const float *dt_bias, int32_t B, int32_t Hk, int32_t Hv,
                           int32_t Dk, int32_t Dv, float scale, int32_t qk_l2norm, gdn_dtype in_dtype,
                           float *state, void *o, gdn_dtype out_dtype, gdn_stream_t stream) {
    if (B < 0 || Hk < 1 || Hv < 1 || Hv % Hk != 0) return GDN_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return GDN_ERR_INVALID_ARG;
    if (Dk != Dv || !head_ok(Dk)) return GDN_ERR_UNSUPPORTED;
    if (B == 0) return GDN_OK;
    if (!q || !k || !v || !a || !b || !A_log || !dt_bias || !state || !o) return GDN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(state))
        return GDN_ERR_INVALID_ARG;
    gdn::RecurrentArgs r{q, k, v, a, b, A_log, dt_bias, nullptr, 1, B, Hk, Hv, Dk, scale, qk_l2norm,
                         in_dtype == GDN_BF16, out_dtype == GDN_BF16, state, state, o};
    return launched(gdn::launch_recurrent(r, reinterpret_cast<cudaStream_t>(stream)));
}

gdn_status gdn_decode_step_gated_nvfp4(const void *q, const void *k, const void *v, const float *a, const float *b,
                                       const float *A_log, const float *dt_bias, int32_t B, int32_t Hk, int32_t Hv,
                                       int32_t Dk, int32_t Dv, float scale, int32_t qk_l2norm, gdn_dtype in_dtype,
                                       float *state, const void *z, const float *norm_weight, float eps,
                                       float global_scale, uint8_t *xq, uint8_t *xs, void *o, gdn_stream_t stream) {
    if (B < 0 || Hk < 1 || Hv < 1 || Hv % Hk != 0 || !dtype_ok(in_dtype)) return GDN_ERR_INVALID_ARG;
    if (Dk != 128 || Dv != 128 || in_dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (!(eps >= 0.0f) || !(global_scale > 0.0f) || !std::isfinite(global_scale)) return GDN_ERR_INVALID_ARG;
    if (B == 0) return GDN_OK;
    if (!q || !k || !v || !a || !b || !A_log || !dt_bias || !state || !z || !norm_weight || !xq || !xs)
        return GDN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) || !aligned16(z) || !aligned16(xq) ||
        (o && !aligned16(o)))
        return GDN_ERR_INVALID_ARG;
    gdn::DecodeTailArgs d{q, k, v, a, b, A_log, dt_bias, B, Hk, Hv, scale, qk_l2norm, state, z, norm_weight,
                          eps, global_scale, xq, xs, o};
    return launched(gdn::launch_decode_gated_nvfp4(d, reinterpret_cast<cudaStream_t>(stream)));
}

static gdn_status multi_check(const void *q, const void *k, const void *v, const float *a, const float *b,
                              const float *A_log, const float *dt_bias, int32_t B, int32_t T, int32_t Hk, int32_t Hv,
                              int32_t Dk, int32_t Dv, gdn_dtype in_dtype) {
    if (B < 0 || T < 1 || Hk < 1 || Hv < 1 || Hv % Hk != 0 || !dtype_ok(in_dtype)) return GDN_ERR_INVALID_ARG;
    if (Dk != Dv || !head_ok(Dk)) return GDN_ERR_UNSUPPORTED;
    if ((int64_t)B * T > INT32_MAX) return GDN_ERR_UNSUPPORTED;
    if (B == 0) return GDN_OK;
    if (!q || !k || !v || !a || !b || !A_log || !dt_bias) return GDN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

gdn_status gdn_decode_verify(const void *q, const void *k, const void *v, const float *a, const float *b,
                             const float *A_log, const float *dt_bias, int32_t B, int32_t T, int32_t Hk, int32_t Hv,
                             int32_t Dk, int32_t Dv, float scale, int32_t qk_l2norm, gdn_dtype in_dtype,
                             const float *state, float *final_state, void *o, gdn_dtype out_dtype,
                             gdn_stream_t stream) {
    const gdn_status c = multi_check(q, k, v, a, b, A_log, dt_bias, B, T, Hk, Hv, Dk, Dv, in_dtype);
    if (c != GDN_OK || B == 0) return c;
    if (!dtype_ok(out_dtype) || !state || !o || !aligned16(state) || !aligned16(o) ||
        (final_state && !aligned16(final_state)))
        return GDN_ERR_INVALID_ARG;
    gdn::RecurrentArgs r{q, k, v, a, b, A_log, dt_bias, nullptr, T, B, Hk, Hv, Dk, scale, qk_l2norm,
                         in_dtype == GDN_BF16, out_dtype == GDN_BF16, state, final_state, o, nullptr};
    return launched(gdn::launch_recurrent(r, reinterpret_cast<cudaStream_t>(stream)));
}

gdn_status gdn_decode_commit(const void *q, const void *k, const void *v, const float *a, const float *b,
                             const float *A_log, const float *dt_bias, int32_t B, int32_t T, int32_t Hk, int32_t Hv,
                             int32_t Dk, int32_t Dv, float scale, int32_t qk_l2norm, gdn_dtype in_dtype,
                             const int32_t *accepted, float *state, gdn_stream_t stream) {
    const gdn_status c = multi_check(q, k, v, a, b, A_log, dt_bias, B, T, Hk, Hv, Dk, Dv, in_dtype);
    if (c != GDN_OK || B == 0) return c;
    if (!accepted || !state || !aligned16(state)) return GDN_ERR_INVALID_ARG;
    gdn::RecurrentArgs r{q, k, v, a, b, A_log, dt_bias, nullptr, T, B, Hk, Hv, Dk, scale, qk_l2norm,
                         in_dtype == GDN_BF16, true, state, state, nullptr, accepted};
    return launched(gdn::launch_recurrent(r, reinterpret_cast<cudaStream_t>(stream)));
}

static gdn_status tail_check(const void *o, const void *z, const float *weight, float eps, int32_t M,
                             int32_t Hv, int32_t Dv, gdn_dtype in_dtype) {
    if (M < 0 || Hv < 1 || !dtype_ok(in_dtype) || !(eps >= 0.0f)) return GDN_ERR_INVALID_ARG;
    if (!head_ok(Dv)) return GDN_ERR_UNSUPPORTED;
    if (M > 0 && (!o || !z || !weight || !aligned16(o) || !aligned16(z))) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

gdn_status gdn_gated_rmsnorm_silu(const void *o, const void *z, const float *weight, float eps, int32_t M,
                                  int32_t Hv, int32_t Dv, gdn_dtype in_dtype, void *y, gdn_dtype out_dtype,
                                  gdn_stream_t stream) {
    gdn_status s = tail_check(o, z, weight, eps, M, Hv, Dv, in_dtype);
    if (s != GDN_OK) return s;
    if (!dtype_ok(out_dtype)) return GDN_ERR_INVALID_ARG;
    if (M == 0) return GDN_OK;
    if (!y || !aligned16(y)) return GDN_ERR_INVALID_ARG;
    gdn::TailArgs t{o, z, weight, eps, M, Hv, Dv, in_dtype == GDN_BF16, y, out_dtype == GDN_BF16, 0.0f,
                    nullptr, nullptr};
    return launched(gdn::launch_gated_rmsnorm(t, reinterpret_cast<cudaStream_t>(stream)));
}

gdn_status gdn_gated_rmsnorm_silu_nvfp4(const void *o, const void *z, const float *weight, float eps,
                                        int32_t M, int32_t Hv, int32_t Dv, gdn_dtype in_dtype,
                                        float global_scale, uint8_t *xq, uint8_t *xs, gdn_stream_t stream) {
    gdn_status s = tail_check(o, z, weight, eps, M, Hv, Dv, in_dtype);
    if (s != GDN_OK) return s;
    if (!(global_scale > 0.0f) || !(global_scale < 3.0e38f)) return GDN_ERR_INVALID_ARG;
    if ((int64_t)Hv * Dv % 32 != 0) return GDN_ERR_UNSUPPORTED;
    if (M == 0) return GDN_OK;
    if (!xq || !xs || !aligned16(xq)) return GDN_ERR_INVALID_ARG;
    gdn::TailArgs t{o, z, weight, eps, M, Hv, Dv, in_dtype == GDN_BF16, nullptr, true, global_scale, xq, xs};
    return launched(gdn::launch_gated_rmsnorm_nvfp4(t, reinterpret_cast<cudaStream_t>(stream)));
}

gdn_status nvfp4_quantize_act(const void *x, gdn_dtype in_dtype, int32_t M, int32_t K, float global_scale,
                              uint8_t *xq, uint8_t *xs, gdn_stream_t stream) {
    if (M < 0 || K < 0 || !dtype_ok(in_dtype)) return GDN_ERR_INVALID_ARG;
    if (!(global_scale > 0.0f) || !(global_scale < 3.0e38f)) return GDN_ERR_INVALID_ARG;
    if (K % 32 != 0) return GDN_ERR_UNSUPPORTED;
    if (M == 0 || K == 0) return GDN_OK;
    if (!x || !xq || !xs || !aligned16(x) || !aligned16(xq)) return GDN_ERR_INVALID_ARG;
    return launched(gdn::launch_nvfp4_quantize(x, in_dtype == GDN_BF16, M, K, global_scale, xq, xs,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

gdn_status nvfp4_dequantize_act(const uint8_t *xq, const uint8_t *xs, int32_t M, int32_t K, float global_scale,
                                gdn_dtype out_dtype, void *y, gdn_stream_t stream) {
    if (M < 0 || K < 0 || !dtype_ok(out_dtype)) return GDN_ERR_INVALID_ARG;
    if (!(global_scale > 0.0f) || !(global_scale < 3.0e38f)) return GDN_ERR_INVALID_ARG;
    if (K % 16 != 0) return GDN_ERR_UNSUPPORTED;
    if (M == 0 || K == 0) return GDN_OK;
    if (!xq || !xs || !y || (reinterpret_cast<uintptr_t>(xq) & 7u) || !aligned16(y)) return GDN_ERR_INVALID_ARG;
    return launched(gdn::launch_nvfp4_dequantize(xq, xs, M, K, global_scale, out_dtype == GDN_BF16, y,
                                                 reinterpret_cast<cudaStream_t>(stream)));
}

gdn_status nvfp4_gemm(const uint8_t *aq, const uint8_t *as, const uint8_t *bq, const uint8_t *bs, float alpha,
                      int32_t M, int32_t N, int32_t K, gdn_dtype out_dtype, void *y, gdn_stream_t stream) {
    if (M < 0 || N < 0 || K < 0 || !dtype_ok(out_dtype)) return GDN_ERR_INVALID_ARG;
    if (K % 32 != 0 || N % 16 != 0) return GDN_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return GDN_OK;
    if (K == 0) return GDN_ERR_UNSUPPORTED;
    if (!aq || !as || !bq || !bs || !y) return GDN_ERR_INVALID_ARG;
    if (!aligned16(aq) || !aligned16(bq) || !aligned16(y)) return GDN_ERR_INVALID_ARG;
    gdn::GemmArgs g{aq, as, bq, bs, alpha, M, N, K, out_dtype == GDN_BF16, y, status_ptr(), nullptr};
    return launched(gdn::launch_nvfp4_gemm(g, reinterpret_cast<cudaStream_t>(stream)));
}

gdn_status nvfp4_gemm_colscale(const uint8_t *aq, const uint8_t *as, const uint8_t *bq, const uint8_t *bs,
                               const float *col_alpha, int32_t M, int32_t N, int32_t K, gdn_dtype out_dtype,
                               void *y, gdn_stream_t stream) {
    if (M < 0 || N < 0 || K < 0 || !dtype_ok(out_dtype)) return GDN_ERR_INVALID_ARG;
    if (K % 32 != 0 || N % 16 != 0) return GDN_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return GDN_OK;
    if (K == 0) return GDN_ERR_UNSUPPORTED;
    if (!aq || !as || !bq || !bs || !y || !col_alpha) return GDN_ERR_INVALID_ARG;
    if (!aligned16(aq) || !aligned16(bq) || !aligned16(y)) return GDN_ERR_INVALID_ARG;
    gdn::GemmArgs g{aq, as, bq, bs, 1.0f, M, N, K, out_dtype == GDN_BF16, y, status_ptr(), col_alpha};
    return launched(gdn::launch_nvfp4_gemm(g, reinterpret_cast<cudaStream_t>(stream)));
}

gdn_status q4k_gemm(const void *a, const uint8_t *w, int32_t M, int32_t N, int32_t K, gdn_dtype out_dtype, void *y,
                    gdn_stream_t stream) {
    if (M < 0 || N < 0 || K < 0 || !dtype_ok(out_dtype)) return GDN_ERR_INVALID_ARG;
    if (K % 256 != 0 || N % 128 != 0) return GDN_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return GDN_OK;
    if (K == 0) return GDN_ERR_UNSUPPORTED;
    if (!a || !w || !y || !aligned16(a) || !aligned16(w) || !aligned16(y)) return GDN_ERR_INVALID_ARG;
    gdn::Q4kGemmArgs g{a, w, M, N, K, out_dtype == GDN_BF16, y, status_ptr()};
    return launched(gdn::launch_q4k_gemm(g, reinterpret_cast<cudaStream_t>(stream)));
}

gdn_status nvfp4_fused_col_alpha(const int32_t *widths, const float *module_scales, int32_t n_modules,
                                 float act_scale, float *col_alpha, gdn_stream_t stream) {
    if (!widths || !module_scales || !col_alpha || n_modules < 1 || n_modules > gdn::kMaxModules)
        return GDN_ERR_INVALID_ARG;
    gdn::ColAlphaArgs c{};
    int64_t end = 0;
    for (int m = 0; m < n_modules; ++m) {
        const float prod = act_scale * module_scales[m];
        if (widths[m] < 1 || !(prod != 0.0f) || !std::isfinite(prod)) return GDN_ERR_INVALID_ARG;
        end += widths[m];
        if (end > INT32_MAX) return GDN_ERR_INVALID_ARG;
        c.end[m] = (int32_t)end;
        c.scale[m] = module_scales[m];
    }
    c.n_modules = n_modules;
    c.act = act_scale;
    c.col_alpha = col_alpha;
    return launched(gdn::launch_fused_col_alpha(c, (int32_t)end, reinterpret_cast<cudaStream_t>(stream)));
}

namespace {

// Checks and fills the plane layout of a short-convolution output.
bool conv_planes(const int32_t *part_widths, int32_t n_parts, int32_t C, gdn::ConvArgs &a) {
    a.n_parts = 1;
    for (int p = 0; p < 4; ++p) a.part_end[p] = C;
    if (n_parts <= 1) return n_parts >= 0 && (n_parts == 0 || !part_widths || part_widths[0] == C);
    if (n_parts > 4 || !part_widths) return false;
    int64_t end = 0;
    for (int p = 0; p < n_parts; ++p) {
        if (part_widths[p] <= 0 || part_widths[p] % 8 != 0) return false;
        end += part_widths[p];
        a.part_end[p] = (int32_t)(end > C ? C : end);
    }
    a.n_parts = n_parts;
    return end == C;
}

bool conv_common_ok(const void *x, int64_t ldx, const float *weight, int32_t C, int32_t K, const void *y) {
    return K >= 1 && K <= 4 && C > 0 && C % 8 == 0 && ldx >= C && ldx % 8 == 0 && x && weight && y &&
           aligned16(x) && aligned16(weight) && aligned16(y);
}

// [p0, p0 + n0) and [p1, p1 + n1) (bytes) overlap
bool overlaps(const void *p0, size_t n0, const void *p1, size_t n1) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p0), b = reinterpret_cast<uintptr_t>(p1);
    return n0 && n1 && a < b + n1 && b < a + n0;
}

}  // namespace

gdn_status gdn_short_conv1d_silu(const void *x, int64_t ldx, const float *weight, const int32_t *cu_seqlens,
                                 int32_t num_seqs, int32_t T, int32_t C, int32_t K, const void *initial_state,
                                 void *final_state, void *y, const int32_t *part_widths, int32_t n_parts,
                                 gdn_stream_t stream) {
    if (T < 0 || num_seqs < 1 || K < 1 || C < 0) return GDN_ERR_INVALID_ARG;
    if (K > 4) return GDN_ERR_UNSUPPORTED;
    if (!cu_seqlens && T % num_seqs != 0) return GDN_ERR_INVALID_ARG;
    if (C == 0) return GDN_OK;
    if (C % 8 != 0) return GDN_ERR_UNSUPPORTED;
    gdn::ConvArgs a{};
    if (!conv_planes(part_widths, n_parts, C, a)) return GDN_ERR_INVALID_ARG;
    if (T > 0 && !conv_common_ok(x, ldx, weight, C, K, y)) return GDN_ERR_INVALID_ARG;
    if (T == 0 && (ldx < C || !weight)) return GDN_ERR_INVALID_ARG;
    const size_t state_bytes = (size_t)num_seqs * (K - 1) * C * 2;
    if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
        return GDN_ERR_INVALID_ARG;
    if (final_state && (overlaps(final_state, state_bytes, x, (size_t)T * ldx * 2) ||
                        overlaps(final_state, state_bytes, y, (size_t)T * C * 2)))
        return GDN_ERR_INVALID_ARG;
    if (T == 0 && (!final_state || K == 1)) return GDN_OK;
    a.x = x;
    a.ldx = ldx;
    a.w = weight;
    a.cu_seqlens = cu_seqlens;
    a.tokens_per_seq = cu_seqlens ? 0 : T / num_seqs;
    a.num_seqs = num_seqs;
    a.T = T;
    a.C = C;
    a.K = K;
    a.init_state = initial_state;
    a.final_state = K > 1 ? final_state : nullptr;
    a.y = y;
    a.decode = false;
    return launched(gdn::launch_short_conv(a, reinterpret_cast<cudaStream_t>(stream)));
}

gdn_status gdn_short_conv1d_silu_decode(const void *x, int64_t ldx, const float *weight, int32_t B, int32_t C,
                                        int32_t K, void *conv_state, void *y, const int32_t *part_widths,
                                        int32_t n_parts, gdn_stream_t stream) {
    if (B < 0 || K < 1 || C < 0) return GDN_ERR_INVALID_ARG;
    if (K > 4) return GDN_ERR_UNSUPPORTED;
    if (B == 0 || C == 0) return GDN_OK;
    if (C % 8 != 0) return GDN_ERR_UNSUPPORTED;
    gdn::ConvArgs a{};
    if (!conv_planes(part_widths, n_parts, C, a)) return GDN_ERR_INVALID_ARG;
    if (!conv_common_ok(x, ldx, weight, C, K, y)) return GDN_ERR_INVALID_ARG;
    const size_t state_bytes = (size_t)B * (K - 1) * C * 2;
    if (K > 1 && (!conv_state || !aligned16(conv_state))) return GDN_ERR_INVALID_ARG;
    if (K > 1 && (overlaps(conv_state, state_bytes, x, (size_t)B * ldx * 2) ||
                  overlaps(conv_state, state_bytes, y, (size_t)B * C * 2)))
        return GDN_ERR_INVALID_ARG;
    a.x = x;
    a.ldx = ldx;
    a.w = weight;
    a.num_seqs = B;
    a.T = B;
    a.C = C;
    a.K = K;
    a.final_state = conv_state;
    a.y = y;
    a.decode = true;
    return launched(gdn::launch_short_conv(a, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
