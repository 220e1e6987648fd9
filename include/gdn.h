/*
 * gdn.h - C ABI of the Gated DeltaNet token mixer and its NVFP4 gated tail on B200 (sm_100a).
 *
 * The operations (page title, section):
 *   [GDN]  "Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4 W4A4 for the Recurrent
 *          Half of a Hybrid 27B LLM", abstract. A fixed-size recurrent state per head; a
 *          decay gate through softplus and an exponential and a write-strength gate through
 *          a sigmoid (mechanism ii); each write overwrites the state along the current key
 *          (mechanism iii); NVFP4 W4A4 with 16-element block scaling (mechanism i). The
 *          explicit recurrence is the gated delta rule (Yang, Kautz, Hatamizadeh, "Gated
 *          Delta Networks", ICLR 2025):
 *              S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t,
 *              alpha_t = exp(-exp(A_log) * softplus(a_t + dt_bias)),  beta_t = sigmoid(b_t).
 *   [TAIL] "Red Lite dev15d - DeltaNet gated tail + Q4_K output projection", section
 *          "Pinned graph semantics", steps 1-6: per value head of 128, RMSNorm with one
 *          shared F32 weight, times SiLU(z), flattened head-major, then the output
 *          projection (here NVFP4 W4A4 instead of Q4_K).
 *   [WALK] "A Node-by-Node White-Box Walkthrough of a Quantized Hybrid Gated DeltaNet Language
 *          Model", Principais Contribuicoes, items 2 and 3: the short convolutions on the
 *          layer's path and their window. The page gives no formula; the reading here is the
 *          depthwise causal convolution of width K <= 4 without bias, followed by SiLU.
 *
 * Conventions for every entry point:
 *   - All pointers are DEVICE pointers owned by the caller, row-major and contiguous,
 *     16-byte aligned (a misaligned pointer is GDN_ERR_INVALID_ARG). The library never
 *     allocates device memory and keeps no pointer after a call returns.
 *   - Work is enqueued on `stream` and the call returns without synchronising. Arguments
 *     are checked on the host before anything is launched; on any error nothing runs.
 *   - GDN_ERR_CUDA means a launch failed (cudaGetLastError after the launch).
 *   - Kernels that wait on barriers bound every wait; on expiry they record
 *     GDN_ERR_TIMEOUT in a device status word and finish without deadlocking. Read (and
 *     clear) it with gdn_get_device_status().
 *   - Per-device set-up (kernel attributes, the device addresses of the status word and of
 *     the allocation-free scratch array) is done once per device on first use and kept:
 *     resetting a device (cudaDeviceReset) between calls into this library is not supported.
 *   - Multi-head layouts: q, k [T, Hk, Dk]; v, o, z [T, Hv, Dv]; value head h reads key
 *     head h / (Hv / Hk) (contiguous groups). The state is [.., Hv, Dv, Dk] fp32, key index
 *     contiguous, so that o = S q.
 */
#ifndef GDN_B200_H
#define GDN_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *gdn_stream_t; /* the same handle as cudaStream_t */

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or dtype */
    GDN_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. head size) */
    GDN_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed */
    GDN_ERR_TIMEOUT = 4,     /* a bounded device-side wait expired */
    GDN_ERR_WORKSPACE = 5    /* workspace missing or too small */
} gdn_status;

typedef enum { GDN_BF16 = 0, GDN_F32 = 1 } gdn_dtype;

/* ------------------------------------------------------------------ prefill ----
 * [GDN]: the gated delta rule over whole sequences, o_t = S_t q_t for every token.
 *
 * q, k        [T, Hk, Dk] in `in_dtype`;  v [T, Hv, Dv] in `in_dtype`
 * a, b        [T, Hv] fp32 gate pre-activations; A_log, dt_bias [Hv] fp32
 * cu_seqlens  device int32 [num_seqs + 1], cumulative token offsets of the packed
 *             sequences (cu_seqlens[0] = 0, non-decreasing, cu_seqlens[num_seqs] = T); NULL
 *             means one sequence of T tokens (then num_seqs must be 1). Every sequence starts
 *             from its own initial state. The array lives in device memory and is not checked:
 *             entries outside that contract are undefined behaviour.
 * scale       multiplies q after normalisation (1.0 = the formula as written)
 * qk_l2norm   non-zero: q and k are L2-normalised per head inside the path,
 *             x * (sum x^2 + 1e-6)^-1/2, before use (the delta rule wants unit keys)
 * initial_state  [num_seqs, Hv, Dv, Dk] fp32, or NULL for zero states
 * final_state    [num_seqs, Hv, Dv, Dk] fp32 output, or NULL; may alias initial_state
 * o           [T, Hv, Dv] in `out_dtype`
 * workspace   device scratch of at least gdn_prefill_workspace_bytes(...) bytes, 16-byte
 *             aligned, owned by the caller; its contents on entry do not matter and are
 *             overwritten. GDN_ERR_WORKSPACE if it is needed and missing or too small.
 * Supported: Dk == Dv in {16, 32, 64, 128}; Hv % Hk == 0; T >= 0 (T == 0 only writes
 * final_state = initial_state); on the tensor-core path T / 64 + num_seqs <= 65535 (about
 * 4.19 M tokens; GDN_ERR_UNSUPPORTED beyond). Dk == Dv == 128 with bf16 inputs runs the tensor-core
 * chunked path (64-token chunks; a prep kernel parallel over chunks writes the
 * state-independent operands to the workspace; long sequences are cut into segments whose
 * states and transition matrices are computed in parallel and combined in order; a chain
 * kernel then walks the chunks of each segment from its true start state; operands are
 * staged in fp16, so |q|, |k|, |v| and the state must stay below
 * 6.5e4). Other sizes and fp32 inputs run the CUDA-core recurrent kernel (no workspace).
 */
GDN_API gdn_status gdn_prefill_chunked(const void *q, const void *k, const void *v,
                               const float *a, const float *b,
                               const float *A_log, const float *dt_bias,
                               const int32_t *cu_seqlens, int32_t num_seqs,
                               int32_t T, int32_t Hk, int32_t Hv, int32_t Dk, int32_t Dv,
                               float scale, int32_t qk_l2norm, gdn_dtype in_dtype,
                               const float *initial_state, float *final_state,
                               void *o, gdn_dtype out_dtype,
                               void *workspace, size_t workspace_bytes, gdn_stream_t stream);

/* Scratch bytes the tensor-core path of gdn_prefill_chunked needs for these sizes, 0 unless
 * Dk == Dv == 128. It is Hv * (T / 64 + num_seqs) * 74752 (state-independent operands, one
 * item per 64-token chunk slot) plus Hv * (T / (64 * L) + num_seqs) * 196608 (per segment of
 * L chunks: its state, its transition matrix, its start state), where the segment length L
 * (a power of two, 4 <= L <= 4096) is picked on the host from T, num_seqs and Hv; so never
 * more than Hv * (T / 64 + num_seqs) * 74752 + Hv * (T / 256 + num_seqs) * 196608.
 * Host-only, no CUDA call. */
GDN_API size_t gdn_prefill_workspace_bytes(int32_t T, int32_t num_seqs, int32_t Hk, int32_t Hv,
                                   int32_t Dk, int32_t Dv);

/* ------------------------------------------------- prefill + gated tail, fused ----
 * [GDN] + [TAIL] "Pinned graph semantics", steps 1-5, with the NVFP4 activation encode of
 * [GDN] mechanism i: the prefill above, whose output pass also applies the gated RMSNorm to
 * every o row and writes it as NVFP4 activations for the output projection, so that neither o
 * nor the gated y has to round-trip through HBM. The result is bit for bit that of
 *   gdn_prefill_chunked(..., o bf16 ...) followed by gdn_gated_rmsnorm_silu_nvfp4(o, z, ...):
 * the tail reads o rounded to bf16, as the two-call path stores it.
 * Arguments as gdn_prefill_chunked, plus
 * o            [T, Hv, 128] bf16 output, or NULL (o is then not written)
 * z            [T, Hv, 128] bf16 gate input; norm_weight [128] fp32 (one weight for all heads); eps
 * global_scale NVFP4 encode scale gs (block scale E4M3((amax / 6) gs), codes E2M1(y gs / scale))
 * xq           [T, Hv * 64] u8: two E2M1 codes per byte, element 2j in the low nibble of byte j
 * xs           [T, Hv * 8] E4M3 block scales, one per 16 consecutive values
 * Supported: Dk == Dv == 128 and bf16 inputs (the tensor-core path), else GDN_ERR_UNSUPPORTED;
 * the workspace is the one gdn_prefill_workspace_bytes gives. xq must be 4-byte aligned.
 */
GDN_API gdn_status gdn_prefill_chunked_gated_nvfp4(const void *q, const void *k, const void *v,
                                           const float *a, const float *b,
                                           const float *A_log, const float *dt_bias,
                                           const int32_t *cu_seqlens, int32_t num_seqs,
                                           int32_t T, int32_t Hk, int32_t Hv, int32_t Dk, int32_t Dv,
                                           float scale, int32_t qk_l2norm, gdn_dtype in_dtype,
                                           const float *initial_state, float *final_state,
                                           void *o, const void *z, const float *norm_weight,
                                           float eps, float global_scale, uint8_t *xq, uint8_t *xs,
                                           void *workspace, size_t workspace_bytes,
                                           gdn_stream_t stream);

/* ------------------------------------------------------------------- decode ----
 * [GDN]: one token per sequence; the state is read once and written once, in place.
 * q, k [B, Hk, Dk], v [B, Hv, Dv] in `in_dtype`; a, b [B, Hv] fp32; A_log, dt_bias [Hv];
 * state [B, Hv, Dv, Dk] fp32, updated in place; o [B, Hv, Dv] in `out_dtype`.
 * Supported: Dk == Dv in {16, 32, 64, 128}, Hv % Hk == 0, B >= 0.
 */
GDN_API gdn_status gdn_decode_step(const void *q, const void *k, const void *v,
                           const float *a, const float *b,
                           const float *A_log, const float *dt_bias,
                           int32_t B, int32_t Hk, int32_t Hv, int32_t Dk, int32_t Dv,
                           float scale, int32_t qk_l2norm, gdn_dtype in_dtype,
                           float *state, void *o, gdn_dtype out_dtype, gdn_stream_t stream);

/* gdn_decode_step fused with the gated tail and the NVFP4 encode:
 * [GDN] recurrence for one token per sequence, then [TAIL] steps 1-5 on each head's o and the
 * 16-value NVFP4 block encode ([GDN] mechanism i) in the same kernel, so o never goes through
 * HBM. Dk = Dv = 128, bf16 inputs. state [B, Hv, 128, 128] fp32 updated in place; z [B, Hv, 128]
 * bf16; norm_weight [128] fp32; eps and global_scale as gdn_gated_rmsnorm_silu_nvfp4; outputs
 * xq [B, Hv*64] u8 and xs [B, Hv*8] (E4M3), the same bytes as gdn_decode_step (bf16 o) followed by
 * gdn_gated_rmsnorm_silu_nvfp4; o [B, Hv, 128] bf16 is also written when not NULL. */
GDN_API gdn_status gdn_decode_step_gated_nvfp4(const void *q, const void *k, const void *v, const float *a,
                                               const float *b, const float *A_log, const float *dt_bias,
                                               int32_t B, int32_t Hk, int32_t Hv, int32_t Dk, int32_t Dv,
                                               float scale, int32_t qk_l2norm, gdn_dtype in_dtype,
                                               float *state, const void *z, const float *norm_weight,
                                               float eps, float global_scale, uint8_t *xq, uint8_t *xs,
                                               void *o, gdn_stream_t stream);

/* ------------------------------------------------ multi-token decode (verify) ----
 * [GDN]: the same recurrence over T tokens per sequence (a draft of T tokens to check in one
 * pass, e.g. speculative decoding), without changing the state: o for every draft token, the
 * state read once. Sequence b's tokens are rows b*T .. b*T + T - 1 of q, k [B*T, Hk, Dk] and
 * v, a, b, o [B*T, Hv, ...]; state [B, Hv, Dv, Dk] fp32 is read only. final_state: NULL, or
 * [B, Hv, Dv, Dk] fp32 written with the state after all T tokens (may alias state: every
 * CTA reads its rows before it writes them). Sizes and dtypes as gdn_decode_step; T >= 1.
 * Equal to gdn_prefill_chunked over B sequences of T tokens from `state`. */
GDN_API gdn_status gdn_decode_verify(const void *q, const void *k, const void *v, const float *a,
                                     const float *b, const float *A_log, const float *dt_bias,
                                     int32_t B, int32_t T, int32_t Hk, int32_t Hv, int32_t Dk,
                                     int32_t Dv, float scale, int32_t qk_l2norm, gdn_dtype in_dtype,
                                     const float *state, float *final_state, void *o,
                                     gdn_dtype out_dtype, gdn_stream_t stream);

/* After gdn_decode_verify: advances each sequence's state, in place, by the first
 * accepted[b] of its T draft tokens (device int32 [B]; values are clamped to [0, T]; 0
 * leaves the state bit for bit unchanged). Same q, k, v, a, b as the verify call; no
 * outputs are written. The state is read once and written once. */
GDN_API gdn_status gdn_decode_commit(const void *q, const void *k, const void *v, const float *a,
                                     const float *b, const float *A_log, const float *dt_bias,
                                     int32_t B, int32_t T, int32_t Hk, int32_t Hv, int32_t Dk,
                                     int32_t Dv, float scale, int32_t qk_l2norm, gdn_dtype in_dtype,
                                     const int32_t *accepted, float *state, gdn_stream_t stream);

/* ------------------------------------------------------------ gated RMSNorm ----
 * [TAIL] steps 1-5: y[m, h*Dv + i] = o[m,h,i] / sqrt(mean_i o[m,h,:]^2 + eps) * w[i]
 *                                     * z[m,h,i] * sigmoid(z[m,h,i]).
 * o, z [M, Hv, Dv] in `in_dtype`; weight [Dv] fp32, shared by all heads; y [M, Hv*Dv]
 * in `out_dtype`. Supported: Dv in {16, 32, 64, 128}; M >= 0.
 */
GDN_API gdn_status gdn_gated_rmsnorm_silu(const void *o, const void *z, const float *weight, float eps,
                                  int32_t M, int32_t Hv, int32_t Dv, gdn_dtype in_dtype,
                                  void *y, gdn_dtype out_dtype, gdn_stream_t stream);

/* The same tail with its NVFP4 activation quantisation fused in: y is formed as above,
 * rounded to bf16, and encoded exactly as nvfp4_quantize_act would encode that bf16
 * tensor (so the two-call and fused paths agree bit for bit). K = Hv * Dv.
 * xq [M, K/2], xs [M, K/16]: see nvfp4_quantize_act. */
GDN_API gdn_status gdn_gated_rmsnorm_silu_nvfp4(const void *o, const void *z, const float *weight,
                                        float eps, int32_t M, int32_t Hv, int32_t Dv,
                                        gdn_dtype in_dtype, float global_scale,
                                        uint8_t *xq, uint8_t *xs, gdn_stream_t stream);

/* ------------------------------------------------------------ NVFP4 encode ----
 * [GDN] mechanism i: NVFP4 with 16-element blocks. For each 16 consecutive values of a
 * row of x [M, K] (in `in_dtype`), in fp32 with this order of operations:
 *   amax = max |x_j|;  s = (amax / 6) * global_scale;  sb = E4M3(s) (nearest, ties to
 *   even, saturating at 448);  r = global_scale / sb (0 when sb == 0);
 *   code_j = E2M1(x_j * r) (nearest, ties to even, saturating at 6, sign kept).
 * xq [M, K/2] uint8: element 2j in the low nibble of byte j, 2j+1 in the high nibble.
 * xs [M, K/16] uint8: the E4M3 block scales, row-major.
 * global_scale is the caller's calibrated encode scale, typically 448 * 6 / amax(tensor);
 * it must be finite and > 0. Decoded value: E2M1(code) * E4M3(sb) / global_scale.
 * Supported: K % 32 == 0, M >= 0.
 */
GDN_API gdn_status nvfp4_quantize_act(const void *x, gdn_dtype in_dtype, int32_t M, int32_t K,
                              float global_scale, uint8_t *xq, uint8_t *xs, gdn_stream_t stream);

/* Inverse of nvfp4_quantize_act: y[m, k] = E2M1(code) * E4M3(scale of its 16-value block) /
 * global_scale, each value the correctly rounded fp32 quotient (then rounded to bf16 for a bf16
 * y). xq [M, K/2] (8-byte aligned), xs [M, K/16] as nvfp4_quantize_act writes them; y [M, K] in
 * `out_dtype`. Used to measure what NVFP4 does to activations (quantise, then dequantise).
 * Supported: K % 16 == 0. */
GDN_API gdn_status nvfp4_dequantize_act(const uint8_t *xq, const uint8_t *xs, int32_t M, int32_t K,
                                        float global_scale, gdn_dtype out_dtype, void *y,
                                        gdn_stream_t stream);

/* ------------------------------------------------------------ NVFP4 GEMM ----
 * [GDN] "NVFP4 W4A4 on all linear layers"; [TAIL] step 6 (ssm_out, 4096 -> 2048):
 *   y[m, n] = alpha * sum_k E2M1(a)[m,k] E4M3(as)[m,k/16] E2M1(b)[n,k] E4M3(bs)[n,k/16]
 * with fp32 accumulation on the block-scaled FP4 tensor cores.
 * aq [M, K/2], as [M, K/16]: the activations as nvfp4_quantize_act writes them;
 * bq [N, K/2], bs [N, K/16]: the weight [N, K] (K contiguous), quantised the same way;
 * alpha = 1 / (global_scale_a * global_scale_b); y [M, N] in `out_dtype`.
 * Supported: K % 32 == 0, N % 16 == 0, M >= 0 (K is zero-padded to the 256-value
 * tile inside the kernel; ragged M and N tiles are masked).
 */
GDN_API gdn_status nvfp4_gemm(const uint8_t *aq, const uint8_t *as, const uint8_t *bq, const uint8_t *bs,
                      float alpha, int32_t M, int32_t N, int32_t K, gdn_dtype out_dtype, void *y,
                      gdn_stream_t stream);

/* NVFP4 GEMM whose output columns come from several modules fused into one weight matrix,
 * each quantised with its own calibrated global scale ([GDN] abstract: the global-scale
 * mismatch of per-module-calibrated NVFP4 checkpoints served by kernels that fuse those modules
 * into one GEMM, and its repair): column n is scaled by col_alpha[n] = 1 / (global_scale_a *
 * global_scale of the module column n belongs to), instead of one alpha for the whole output.
 * col_alpha: device fp32 [N]. Other arguments and limits as nvfp4_gemm. */
GDN_API gdn_status nvfp4_gemm_colscale(const uint8_t *aq, const uint8_t *as, const uint8_t *bq,
                                       const uint8_t *bs, const float *col_alpha, int32_t M, int32_t N,
                                       int32_t K, gdn_dtype out_dtype, void *y, gdn_stream_t stream);

/* The col_alpha vector of nvfp4_gemm_colscale for a weight made of n_modules modules stacked
 * along N: module m has widths[m] output columns and was quantised with global scale
 * module_scales[m]; the activations with act_scale. Writes col_alpha[n] = 1 / (act_scale *
 * module_scales[m]) (fp32 IEEE division) for every column n of module m, in order.
 * widths, module_scales: HOST arrays of n_modules (1 <= n_modules <= 64, each width >= 1);
 * col_alpha: device fp32 [sum of widths]. A zero or non-finite product act_scale * scale is
 * GDN_ERR_INVALID_ARG. Enqueued on `stream`. */
GDN_API gdn_status nvfp4_fused_col_alpha(const int32_t *widths, const float *module_scales, int32_t n_modules,
                                         float act_scale, float *col_alpha, gdn_stream_t stream);

/* ------------------------------------------------- Q4_K output projection ----
 * [TAIL] "Q4_K implementation" (the page's comparison format for ssm_out): y [M, N] = a [M, K] w^T
 * with w [N, K] held as Q4_K blocks of 256 values in 144 bytes (f16 d, f16 dmin, 12 bytes of
 * 6-bit sub-block scales / mins, 128 bytes of 4-bit quants; w = d * scale * q - dmin * min; the
 * GGUF K-quant bit positions, which the page calls canonical). The weights are decoded on the fly,
 * rounded to bf16 and multiplied on the tensor cores with fp32 accumulation.
 * a: bf16 [M, K] row-major; w: [N, K/256 * 144] bytes (row n: its K/256 blocks in order); y:
 * [M, N] in out_dtype. Supported: K % 256 == 0, N % 128 == 0; a, w, y 16-byte aligned. */
GDN_API gdn_status q4k_gemm(const void *a, const uint8_t *w, int32_t M, int32_t N, int32_t K, gdn_dtype out_dtype,
                            void *y, gdn_stream_t stream);

/* ------------------------------------------------------ short convolution ----
 * [WALK]: the causal short convolution + SiLU on the layer's q, k, v channels before the scan:
 *   y[t, c] = SiLU(sum_{j<K} weight[c, j] x[t - (K - 1) + j, c])
 * per sequence; the inputs before a sequence's first token are its carried state (the last
 * K - 1 inputs of what came before, oldest first) or zero.
 *
 * x           bf16 [T, ldx] (ldx >= C, ldx % 8 == 0): channels [0, C) of each row are used, so
 *             x can be the q|k|v columns of a wider projection output in place
 * weight      fp32 [C, K], K contiguous
 * cu_seqlens  device int32 [num_seqs + 1] as for gdn_prefill_chunked (non-decreasing,
 *             cu_seqlens[0] = 0, cu_seqlens[num_seqs] = T; empty sequences allowed), or NULL:
 *             num_seqs sequences of T / num_seqs tokens each (T % num_seqs == 0)
 * initial_state  bf16 [num_seqs, K - 1, C], or NULL (zero history)
 * final_state    bf16 [num_seqs, K - 1, C] output, or NULL: each sequence's last K - 1
 *             inputs (continuing initial_state when the sequence is shorter than K - 1). May
 *             alias initial_state; must not overlap x or y.
 * y           bf16, the output as n_parts planes: with part_widths = {w_0, w_1, ...} (host
 *             array, each a multiple of 8, summing to C) plane p holds channels
 *             [w_0 + .. + w_{p-1}, .. + w_p) as a contiguous [T, w_p] block, the planes one
 *             after another (n_parts = 3 and widths {Hk*Dk, Hk*Dk, Hv*Dv} give q, k and v as
 *             gdn_prefill_chunked reads them). n_parts 0 or 1 (part_widths NULL): y is [T, C].
 * Supported: 1 <= K <= 4; C % 8 == 0; n_parts <= 4. A malformed cu_seqlens gives undefined
 * values but no out-of-bounds access of cu_seqlens. */
GDN_API gdn_status gdn_short_conv1d_silu(const void *x, int64_t ldx, const float *weight,
                                         const int32_t *cu_seqlens, int32_t num_seqs, int32_t T,
                                         int32_t C, int32_t K, const void *initial_state,
                                         void *final_state, void *y, const int32_t *part_widths,
                                         int32_t n_parts, gdn_stream_t stream);

/* One decode token per sequence: x bf16 [B, ldx] (channels [0, C) used), conv_state bf16
 * [B, K - 1, C] read and then shifted by one token in place (it ends as the last K - 1 inputs,
 * x included), y as for gdn_short_conv1d_silu with T = B. conv_state must not overlap x or y.
 * Continuing a prefill whose final_state was written gives the same y as one longer prefill. */
GDN_API gdn_status gdn_short_conv1d_silu_decode(const void *x, int64_t ldx, const float *weight,
                                                int32_t B, int32_t C, int32_t K, void *conv_state,
                                                void *y, const int32_t *part_widths, int32_t n_parts,
                                                gdn_stream_t stream);

/* ------------------------------------------------- allocation-free prefill ----
 * No counterpart in the pages this library follows. For callers that cannot allocate device
 * memory - code that runs where cudaMalloc is unavailable or not allowed, or a host framework
 * that owns every allocation - this is gdn_prefill_chunked without the workspace argument: same inputs,
 * outputs, layouts and status codes. The tensor-core path uses a fixed scratch array inside
 * the library instead: 32 MiB (33554432 bytes), held on every GPU that loads the library
 * until the process exits. Sizes whose workspace (gdn_prefill_workspace_bytes) exceeds
 * 32 MiB return GDN_ERR_WORKSPACE before anything is launched. It allocates nothing.
 * The first call on a device looks up the array's device address for that device and keeps
 * it (so the device must not be reset between calls); make that first call before any stream
 * capture on the device.
 * Every call uses the same array: calls that can overlap on the GPU (other streams, other
 * host threads) race on it and corrupt each other's results, so serialise them. What a
 * previous call left in the array does not matter: the path writes all it later reads.
 */
GDN_API gdn_status gdn_prefill_chunked_static_ws(const void *q, const void *k, const void *v,
                                                 const float *a, const float *b,
                                                 const float *A_log, const float *dt_bias,
                                                 const int32_t *cu_seqlens, int32_t num_seqs,
                                                 int32_t T, int32_t Hk, int32_t Hv, int32_t Dk,
                                                 int32_t Dv, float scale, int32_t qk_l2norm,
                                                 gdn_dtype in_dtype, const float *initial_state,
                                                 float *final_state, void *o, gdn_dtype out_dtype,
                                                 gdn_stream_t stream);

/* ----------------------------------------------------------------- helpers ---- */

/* Synchronises `stream`, returns the device status word (GDN_OK or GDN_ERR_TIMEOUT) that
 * kernels set on an expired bounded wait, and clears it. */
GDN_API gdn_status gdn_get_device_status(gdn_stream_t stream);

/* Test support for the timeout path (no counterpart in the pages). Sets, for the current device,
 * the limit of every bounded device-side wait (wait_limit_ns; 0 restores the default of 1 s, larger
 * values are GDN_ERR_INVALID_ARG) and switches that make a kernel skip work so that one of its waits
 * runs out with nothing in flight: GDN_INJECT_SKIP_PREP_LOADS (1) makes the chunked prefill's prep
 * kernel issue none of its tile loads, so each of its CTAs times out waiting for them, records
 * GDN_ERR_TIMEOUT and exits (the later kernels of the call then read an unwritten workspace, so
 * that call's outputs are meaningless). Synchronous; call it with no work of this library in
 * flight on the device, and call gdn_debug_set_wait(0, 0) to restore normal operation. */
#define GDN_INJECT_SKIP_PREP_LOADS 1u
GDN_API gdn_status gdn_debug_set_wait(uint64_t wait_limit_ns, uint32_t inject_flags);

/* Static description of a status code. */
GDN_API const char *gdn_status_string(gdn_status s);

/* Library version, major * 10000 + minor * 100 + patch. */
GDN_API int32_t gdn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GDN_B200_H */
