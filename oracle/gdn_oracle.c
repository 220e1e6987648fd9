/*
 * Oracle for the Gated DeltaNet token mixer and its NVFP4 gated tail.
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and the cpu_baseline /
 * reference legs of bench.py may load this library. The product path never does, and
 * this file shares no code, header, table or constant with the CUDA library.
 *
 * Plain, slow, sequential CPU code:
 *   - the scan is the token-by-token recurrence in fp64 (no chunking, no reordering);
 *   - the gated RMSNorm tail is fp64;
 *   - the NVFP4 encode runs in fp32 with one fixed order of operations, so the GPU can
 *     be compared with it bit for bit; E2M1 and E4M3 rounding is done by searching the
 *     format's finite values for the nearest one (ties to the even code), which is the
 *     definition of round-to-nearest-even, written out.
 *
 * Sources (page title, section):
 *   [GDN]  "Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4 W4A4 for the Recurrent
 *          Half of a Hybrid 27B LLM", abstract: a fixed-size recurrent state; decay and
 *          write-strength gates with softplus/exponential and sigmoid parameterisations
 *          (mechanism ii); each write overwrites the state along the current key
 *          direction (mechanism iii); NVFP4 with 16-element block scaling (mechanism i).
 *          The explicit recurrence is the gated delta rule of Yang, Kautz and
 *          Hatamizadeh, "Gated Delta Networks" (ICLR 2025):
 *              S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *              o_t = S_t q_t,
 *              alpha_t = exp(-exp(A_log) softplus(a_t + dt_bias)), beta_t = sigmoid(b_t).
 *   [TAIL] "Red Lite dev15d - DeltaNet gated tail + Q4_K output projection", section
 *          "Pinned graph semantics", steps 1-6: reshape to value heads x 128, RMSNorm each
 *          head with the one shared norm weight, SiLU(z), multiply, flatten, output
 *          projection; "Real layer-0 GGUF tensors": the norm weight is F32 [128].
 *   [FMT]  OCP Microscaling Formats (MX) v1.0 (E2M1 element encoding) and OCP 8-bit
 *          Floating Point (E4M3FN): value sets used below; IEEE 754 binary16 for the Q4_K
 *          block scales.
 *
 * Readings where the pages are silent:
 *   - q/k are L2-normalised inside the path when qk_l2norm != 0: x * (sum x^2 + eps)^-1/2.
 *   - GQA: v-head h reads k-head h / (Hv / Hk).
 *   - the readout uses the updated state S_t.
 *   - state layout [.., Dv, Dk]: o = S q contracts the last (key) index.
 *   - NVFP4 block encode: amax over 16 values; s = (amax / 6) * gs; sb = E4M3(s);
 *     r = gs / sb (0 if sb == 0); code = E2M1(x * r). Dequant: E2M1(code) * sb / gs.
 *   - E2M1 keeps the sign of values that round to zero (code 0x8).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ---------------------------------------------------------------- gates ---- */

/* softplus(x) = log(1 + e^x), written so that it does not overflow for large x. */
static double softplus(double x) { return x > 0.0 ? x + log1p(exp(-x)) : log1p(exp(x)); }

static double sigmoid(double x) {
    if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
    double e = exp(x);
    return e / (1.0 + e);
}

/* [GDN] mechanism ii: decay through softplus and an exponential, write strength through
 * a sigmoid. Returns log(alpha) in *g so callers can check the decay in log space. */
void oracle_gates(double a, double b, double A_log, double dt_bias,
                  double *g, double *alpha, double *beta) {
    double gg = -exp(A_log) * softplus(a + dt_bias);
    *g = gg;
    *alpha = exp(gg);
    *beta = sigmoid(b);
}

/* ----------------------------------------------------------------- scan ---- */

/*
 * Sequential gated delta rule over every (sequence, v-head) unit in
 * [unit_begin, unit_end); unit = n * Hv + h.
 *
 *   q, k   [T, Hk, Dk]  fp32 values (the bf16 inputs, widened exactly)
 *   v      [T, Hv, Dv]
 *   a, b   [T, Hv]
 *   A_log, dt_bias [Hv]
 *   cu_seqlens [num_seqs + 1]: sequence n covers tokens cu_seqlens[n] .. cu_seqlens[n+1]-1
 *   S0     [num_seqs, Hv, Dv, Dk] fp64, or NULL for a zero initial state
 *   S_out  [num_seqs, Hv, Dv, Dk] fp64 (final state)
 *   o      [T, Hv, Dv] fp64
 * Returns 0, or -1 on bad sizes.
 */
int oracle_gdn_scan(int32_t num_seqs, const int32_t *cu_seqlens,
                    int32_t Hk, int32_t Hv, int32_t Dk, int32_t Dv,
                    const float *q, const float *k, const float *v,
                    const float *a, const float *b,
                    const float *A_log, const float *dt_bias,
                    double scale, int32_t qk_l2norm, double eps,
                    const double *S0, double *S_out, double *o,
                    int32_t unit_begin, int32_t unit_end) {
    if (num_seqs < 1 || Hk <= 0 || Hv <= 0 || Hv % Hk != 0 || Dk <= 0 || Dv <= 0 || Dk > 1024)
        return -1;
    if (unit_begin < 0 || unit_end > num_seqs * Hv) return -1;
    const int32_t group = Hv / Hk;
    double kh[1024], qh[1024];
    double sk[1024];
    if (Dv > 1024) return -1;

    for (int32_t unit = unit_begin; unit < unit_end; ++unit) {
        const int32_t n = unit / Hv, h = unit % Hv, hk = h / group;
        double *S = S_out + (size_t)unit * Dv * Dk;
        if (S0) memcpy(S, S0 + (size_t)unit * Dv * Dk, sizeof(double) * Dv * Dk);
        else memset(S, 0, sizeof(double) * Dv * Dk);

        for (int32_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
            const float *kt = k + ((size_t)t * Hk + hk) * Dk;
            const float *qt = q + ((size_t)t * Hk + hk) * Dk;
            const float *vt = v + ((size_t)t * Hv + h) * Dv;

            /* key and query, optionally L2-normalised per head; the query also takes `scale` */
            double kk = 0.0, qq = 0.0;
            for (int32_t j = 0; j < Dk; ++j) { kk += (double)kt[j] * kt[j]; qq += (double)qt[j] * qt[j]; }
            double kn = qk_l2norm ? 1.0 / sqrt(kk + eps) : 1.0;
            double qn = qk_l2norm ? 1.0 / sqrt(qq + eps) : 1.0;
            for (int32_t j = 0; j < Dk; ++j) { kh[j] = kt[j] * kn; qh[j] = qt[j] * qn * scale; }

            double g, alpha, beta;
            oracle_gates(a[(size_t)t * Hv + h], b[(size_t)t * Hv + h], A_log[h], dt_bias[h],
                         &g, &alpha, &beta);

            /* S <- alpha * S (I - beta k k^T) + beta v k^T, element by element:
             * (S (I - beta k k^T))_ij = S_ij - beta (S k)_i k_j */
            for (int32_t i = 0; i < Dv; ++i) {
                double acc = 0.0;
                for (int32_t j = 0; j < Dk; ++j) acc += S[(size_t)i * Dk + j] * kh[j];
                sk[i] = acc;
            }
            for (int32_t i = 0; i < Dv; ++i)
                for (int32_t j = 0; j < Dk; ++j) {
                    double *s = &S[(size_t)i * Dk + j];
                    *s = alpha * (*s - beta * sk[i] * kh[j]) + beta * (double)vt[i] * kh[j];
                }

            /* o_t = S_t q_t, with the state after this token's write */
            double *ot = o + ((size_t)t * Hv + h) * Dv;
            for (int32_t i = 0; i < Dv; ++i) {
                double acc = 0.0;
                for (int32_t j = 0; j < Dk; ++j) acc += S[(size_t)i * Dk + j] * qh[j];
                ot[i] = acc;
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------- gated RMSNorm ---- */

/*
 * [TAIL] steps 1-5: y[m, h*D + i] = RMSNorm(o[m,h,:])_i * w_i * SiLU(z[m,h,i]),
 * RMSNorm(x)_i = x_i / sqrt(mean_j x_j^2 + eps), one weight vector w [D] for all heads,
 * SiLU(z) = z * sigmoid(z), flattened head-major. Rows [row_begin, row_end) of M.
 */
void oracle_gated_rmsnorm_silu(int32_t M, int32_t Hv, int32_t D,
                               const float *o, const float *z, const float *w, double eps,
                               double *y, int32_t row_begin, int32_t row_end) {
    (void)M;
    for (int32_t m = row_begin; m < row_end; ++m)
        for (int32_t h = 0; h < Hv; ++h) {
            const float *oh = o + ((size_t)m * Hv + h) * D;
            const float *zh = z + ((size_t)m * Hv + h) * D;
            double ss = 0.0;
            for (int32_t i = 0; i < D; ++i) ss += (double)oh[i] * oh[i];
            double inv_rms = 1.0 / sqrt(ss / D + eps);
            double *yh = y + (size_t)m * Hv * D + (size_t)h * D;
            for (int32_t i = 0; i < D; ++i) {
                double normed = (double)oh[i] * inv_rms * (double)w[i];
                double zi = zh[i];
                double silu = zi * sigmoid(zi);
                yh[i] = normed * silu;
            }
        }
}

/* --------------------------------------------------------- number formats ---- */

/* [FMT] E2M1 magnitudes for codes 0..7 (sign is bit 3). */
static const float e2m1_mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

float oracle_e2m1_decode(uint8_t code) {
    float m = e2m1_mag[code & 7];
    return (code & 8) ? -m : m;
}

/* [FMT] E4M3FN: 1 sign, 4 exponent (bias 7), 3 mantissa bits; exponent 0 is subnormal;
 * 0x7F / 0xFF are NaN, so the largest finite magnitude is 0x7E = 448. */
float oracle_e4m3_decode(uint8_t code) {
    int e = (code >> 3) & 15, m = code & 7;
    float mag;
    if ((code & 0x7F) == 0x7F) return NAN;
    if (e == 0) mag = ldexpf((float)m / 8.0f, -6);
    else mag = ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return (code & 0x80) ? -mag : mag;
}

/* Nearest finite E2M1 value to x, ties to the even code; magnitudes of 6 and above
 * saturate to 6 (satfinite). The sign is kept, also when the magnitude rounds to zero.
 * Distances are taken in fp64, where they are exact for the two candidates that bracket x. */
uint8_t oracle_e2m1_encode(float x) {
    double ax = fabs((double)x);
    int best = 7;
    if (ax < 6.0) {
        best = 0;
        for (int c = 1; c < 8; ++c) {
            double d_best = fabs(ax - e2m1_mag[best]), d = fabs(ax - e2m1_mag[c]);
            if (d < d_best || (d == d_best && (c & 1) == 0 && (best & 1) == 1)) best = c;
        }
    }
    return (uint8_t)(best | (signbit(x) ? 8 : 0));
}

/* Nearest finite non-negative E4M3 value to s >= 0, ties to the even code; 448 and above
 * saturate to 448 (satfinite; the block scales are never negative). */
uint8_t oracle_e4m3_encode_nonneg(float s) {
    if (s >= 448.0f) return 0x7E;
    int best = 0;
    double d_best = fabs((double)s - oracle_e4m3_decode(0));
    for (int c = 1; c <= 0x7E; ++c) {
        double d = fabs((double)s - (double)oracle_e4m3_decode((uint8_t)c));
        if (d < d_best || (d == d_best && (c & 1) == 0 && (best & 1) == 1)) { best = c; d_best = d; }
    }
    return (uint8_t)best;
}

/*
 * NVFP4 quantisation of x [M, K] (K % 16 == 0), rows [row_begin, row_end):
 * per 16 consecutive values of a row, one E4M3 scale from the block's largest magnitude
 * and the fp32 global encode scale gs; two E2M1 codes per byte, element 2j in the low
 * nibble of byte j. xq [M, K/2], xs [M, K/16] row-major.
 * Each fp32 operation below is one correctly rounded step, in this order.
 */
void oracle_nvfp4_quantize(int32_t M, int32_t K, const float *x, float gs,
                           uint8_t *xq, uint8_t *xs, int32_t row_begin, int32_t row_end) {
    (void)M;
    for (int32_t m = row_begin; m < row_end; ++m)
        for (int32_t blk = 0; blk < K / 16; ++blk) {
            const float *xb = x + (size_t)m * K + (size_t)blk * 16;
            float amax = 0.0f;
            for (int j = 0; j < 16; ++j) { float ax = fabsf(xb[j]); if (ax > amax) amax = ax; }
            volatile float t = amax / 6.0f;   /* step 1: amax / 6 */
            volatile float s = t * gs;        /* step 2: times the global scale */
            uint8_t sb = oracle_e4m3_encode_nonneg(s);
            float sbf = oracle_e4m3_decode(sb);
            volatile float r = (sb == 0) ? 0.0f : gs / sbf;   /* step 3: reciprocal block scale */
            xs[(size_t)m * (K / 16) + blk] = sb;
            for (int j = 0; j < 16; j += 2) {
                volatile float p0 = xb[j] * r, p1 = xb[j + 1] * r;
                uint8_t c0 = oracle_e2m1_encode(p0), c1 = oracle_e2m1_encode(p1);
                xq[(size_t)m * (K / 2) + (size_t)blk * 8 + j / 2] = (uint8_t)(c0 | (c1 << 4));
            }
        }
}

/* Dequantised values x_hat = E2M1(code) * E4M3(scale) / gs in fp64, rows [row_begin, row_end). */
void oracle_nvfp4_dequantize(int32_t M, int32_t K, const uint8_t *xq, const uint8_t *xs, float gs,
                             double *out, int32_t row_begin, int32_t row_end) {
    (void)M;
    for (int32_t m = row_begin; m < row_end; ++m)
        for (int32_t kk = 0; kk < K; ++kk) {
            uint8_t byte = xq[(size_t)m * (K / 2) + kk / 2];
            uint8_t code = (kk & 1) ? (byte >> 4) : (byte & 15);
            double sc = oracle_e4m3_decode(xs[(size_t)m * (K / 16) + kk / 16]);
            out[(size_t)m * K + kk] = (double)oracle_e2m1_decode(code) * sc / (double)gs;
        }
}

/* ----------------------------------------------------------------- Q4_K ---- */

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 mantissa bits; exponent 0 is subnormal,
 * 31 is inf / NaN. Exact in fp64. */
double oracle_f16_decode(uint16_t h) {
    int e = (h >> 10) & 31, m = h & 1023;
    double mag;
    if (e == 31) mag = m ? NAN : INFINITY;
    else if (e == 0) mag = ldexp((double)m, -24);
    else mag = ldexp(1.0 + (double)m / 1024.0, e - 15);
    return (h & 0x8000) ? -mag : mag;
}

/*
 * [TAIL] "Q4_K implementation": blocks of 256 values in 144 bytes - f16 d, f16 dmin, 12 bytes of
 * packed 6-bit scales and mins for the block's eight sub-blocks of 32 values, 128 bytes of 4-bit
 * quants. The page fixes the sizes and calls the layout canonical; the bit positions read here
 * are the GGUF K-quant ones:
 *   bytes 0-1 d, 2-3 dmin (little-endian f16); bytes 4-15 = sc[12];
 *   sub-block j < 4: scale = sc[j] & 63, min = sc[j + 4] & 63;
 *   sub-block j >= 4: scale = (sc[j + 4] & 15) | ((sc[j - 4] >> 6) << 4),
 *                     min = (sc[j + 4] >> 4) | ((sc[j] >> 6) << 4);
 *   bytes 16-143 = qs[128]: value 64 g + i (g < 4, i < 32) is the low nibble of qs[32 g + i]
 *   (sub-block 2 g), value 64 g + 32 + i its high nibble (sub-block 2 g + 1);
 *   value = d * scale * q - dmin * min.
 * w: rows [N, K / 256 * 144] bytes; out: [N, K] fp64 (exact), rows [row_begin, row_end).
 */
void oracle_q4k_dequantize(int32_t N, int32_t K, const uint8_t *w, double *out, int32_t row_begin,
                           int32_t row_end) {
    (void)N;
    const int32_t nb = K / 256;
    for (int32_t n = row_begin; n < row_end; ++n)
        for (int32_t blk = 0; blk < nb; ++blk) {
            const uint8_t *b = w + ((size_t)n * nb + blk) * 144;
            const double d = oracle_f16_decode((uint16_t)(b[0] | (b[1] << 8)));
            const double dmin = oracle_f16_decode((uint16_t)(b[2] | (b[3] << 8)));
            const uint8_t *sc = b + 4, *qs = b + 16;
            for (int j = 0; j < 8; ++j) {
                int scale, mn;
                if (j < 4) {
                    scale = sc[j] & 63;
                    mn = sc[j + 4] & 63;
                } else {
                    scale = (sc[j + 4] & 15) | ((sc[j - 4] >> 6) << 4);
                    mn = (sc[j + 4] >> 4) | ((sc[j] >> 6) << 4);
                }
                const int g = j / 2, hi = j & 1;
                for (int i = 0; i < 32; ++i) {
                    const int q = hi ? (qs[32 * g + i] >> 4) : (qs[32 * g + i] & 15);
                    out[(size_t)n * K + (size_t)blk * 256 + 32 * j + i] = d * (double)scale * (double)q - dmin * (double)mn;
                }
            }
        }
}

/* ------------------------------------------------- bulk helpers for tests ---- */

void oracle_e2m1_encode_many(int64_t n, const float *x, uint8_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1_encode(x[i]);
}

void oracle_e4m3_encode_many(int64_t n, const float *x, uint8_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode_nonneg(x[i]);
}
