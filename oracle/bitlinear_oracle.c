/*
 * bitlinear_oracle.c -- plain, slow CPU oracle of the BitNet b1.58 BitLinear hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline arm may load this library.  The product path never calls it and
 * shares no code with it (no headers, no helpers, no tables).
 *
 * Pages this restates (titles of the source web pages):
 *   P1 = "BitNet量化感知训练中的梯度传播优化：解决符号函数不可微性的工程实践" (blog.hotdry.top)
 *   P2 = "BitNet 三元权重量化训练工程：直通估计器与梯度裁剪实践" (blog.hotdry.top)
 *   P3 = "BitNet 1.5技术解析：2比特量化在神经网络中的应用与挑战" (intelliparadigm.com)
 *   P4 = "BitNet b1.58：三元权重下的STE设计与优化" (zyxy.net)
 *   P5 = "1.58-bit量化技术突破AI算力与内存墙限制" (intelliparadigm.com)
 *
 * Arithmetic conventions (the pages fix formulas, not precision; these are the
 * readings every function below follows):
 *   - element-wise quantiser arithmetic in IEEE fp32, one rounding per operation,
 *     no fused multiply-add (build with -ffp-contract=off, never -ffast-math);
 *   - round() is round-half-to-even (nearbyintf under the default FE_TONEAREST),
 *     which is what torch.round does in the pages' snippets;
 *   - reductions (sum |W|, sum x^2) and every floating-point contraction are
 *     accumulated in fp64, sequentially, in index order;
 *   - integer contraction in exact int32 (|acc| <= 127*K, far below 2^31).
 *
 * Each function is a direct loop; OpenMP only splits independent rows.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads OpenMP will use (reported beside CPU timings). */
int ora_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* fp32 -> bf16 round-to-nearest-even, from the bf16 definition (top 16 bits of an
 * IEEE binary32).  Used for X_dq and Y when the layer runs in bf16 (P2, "训练管道
 * 集成": bf16 forward).  NaN is returned as a quiet NaN. */
static uint16_t bf16_bits_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x40);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

static float bf16_bits_to_f32(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

void ora_round_bf16(const float* in, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_bits_rne(in[i]);
}

/* ---------------------------------------------------------------------------------
 * RMSNorm statistic (P3 §3.1: BitLinear applies RMSNorm(in_features) to x before the
 * activation quantiser).  The pages do not print RMSNorm; the textbook definition is
 *   r_t = 1 / sqrt( (1/K) sum_k x_{t,k}^2 + eps ).
 * Sum in fp64 in index order; r rounded once to fp32.
 * --------------------------------------------------------------------------------- */
void ora_rmsnorm_rinv(const float* X, int64_t T, int64_t K, float eps, float* rinv) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const float* x = X + t * K;
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k) ss += (double)x[k] * (double)x[k];
        rinv[t] = (float)(1.0 / sqrt(ss / (double)K + (double)eps));
    }
}

/* ---------------------------------------------------------------------------------
 * Per-token absmax int8 activation quantiser (P3 §2.2 activation_quant; P2 "直通估计器
 * 在三元权重量化中的作用": scale_x = 127/max|X|, X_q = clamp(round(X*scale_x),-128,127)).
 * Applied to the RMSNorm output x_hat = x * r_t * g_k (P3 §3.1), one row per token:
 *   x_hat = fl32(fl32(x * r) * g)          (r == NULL: no RMSNorm, x_hat = x)
 *   m     = max_k |x_hat|
 *   s_t   = fl32(127 / max(m, 1e-5))
 *   q     = clamp(round(fl32(x_hat * s_t)), -128, 127)
 *   X_dq  = fl32(q / s_t)                  (the dequantised value the STE forwards)
 * g == NULL means gain 1.  xdq may be NULL.
 * --------------------------------------------------------------------------------- */
void ora_act_quant(const float* X, int64_t T, int64_t K, const float* rinv, const float* g,
                   int8_t* xq, float* s_out, float* xdq) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const float* x = X + t * K;
        float* xh = (float*)malloc(sizeof(float) * (size_t)K);
        for (int64_t k = 0; k < K; ++k) {
            float v = x[k];
            if (rinv) {
                v = v * rinv[t];
                if (g) v = v * g[k];
            }
            xh[k] = v;
        }
        float m = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(xh[k]);
            if (a > m) m = a;
        }
        float s = 127.0f / fmaxf(m, 1e-5f);
        s_out[t] = s;
        for (int64_t k = 0; k < K; ++k) {
            float v = nearbyintf(xh[k] * s);
            if (v < -128.0f) v = -128.0f;
            if (v > 127.0f) v = 127.0f;
            int8_t q = (int8_t)v;
            xq[t * K + k] = q;
            if (xdq) xdq[t * K + k] = (float)q / s;
        }
        free(xh);
    }
}

/* ---------------------------------------------------------------------------------
 * Per-tensor absmean scale (P3 §2.1 weight_quant: 1/mean|w| clamped at 1e-5; P5 §2.2
 * ternary_quantize: gamma = mean|w|):
 *   gamma = max( (float)( sum|W| / n ), 1e-5 )      sum in fp64, index order.
 * --------------------------------------------------------------------------------- */
float ora_absmean_gamma(const float* W, int64_t n) {
    double S = 0.0;
    for (int64_t i = 0; i < n; ++i) S += (double)fabsf(W[i]);
    float mean = (float)(S / (double)n);
    return fmaxf(mean, 1e-5f);
}

/* Ternary round (P5 §2.2: clamp(round(w / gamma), -1, 1); P3 §2.1 round+clamp):
 *   W_q = clamp(round(fl32(W / gamma)), -1, 1). */
void ora_ternary_round(const float* W, int64_t n, float gamma, int8_t* wq) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        float v = nearbyintf(W[i] / gamma);
        if (v < -1.0f) v = -1.0f;
        if (v > 1.0f) v = 1.0f;
        wq[i] = (int8_t)v;
    }
}

/* ---------------------------------------------------------------------------------
 * 2-bit packing (P5 §4.1 memory layout: 00 -> 0, 01 -> +1, 10 -> -1, 11 reserved;
 * P5 §5.1: pack on 64-bit boundaries).  Element (n, k) goes to byte n*(K/4) + k/4,
 * bits 2*(k%4) .. 2*(k%4)+1 (least significant pair first).  K % 32 == 0 keeps every
 * row a whole number of 64-bit words.
 * --------------------------------------------------------------------------------- */
void ora_pack(const int8_t* wq, int64_t N, int64_t K, uint8_t* packed) {
    int64_t row_bytes = K / 4;
    memset(packed, 0, (size_t)(N * row_bytes));
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int8_t v = wq[n * K + k];
            uint8_t code = 0;            /* 0 -> 00 */
            if (v == 1) code = 1;        /* +1 -> 01 */
            else if (v == -1) code = 2;  /* -1 -> 10 */
            packed[n * row_bytes + k / 4] |= (uint8_t)(code << (2 * (k % 4)));
        }
    }
}

/* Decode of one 2-bit code: 00 -> 0, 01 -> +1, 10 -> -1; the reserved 11 decodes to 0. */
static int decode2(unsigned c) {
    if (c == 1u) return 1;
    if (c == 2u) return -1;
    return 0;
}

void ora_unpack(const uint8_t* packed, int64_t N, int64_t K, int8_t* wq) {
    int64_t row_bytes = K / 4;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            unsigned c = (packed[n * row_bytes + k / 4] >> (2 * (k % 4))) & 3u;
            wq[n * K + k] = (int8_t)decode2(c);
        }
}

/* ---------------------------------------------------------------------------------
 * Integer contraction of the forward (P3 §3.1 F.linear(x_quant, w_quant); P5 §3.1
 * W=+1 adds x, W=-1 subtracts x, W=0 skips):
 *   acc[t, n] = sum_k x_q[t, k] * W_q[n, k]          exact int32
 * Computed for the token rows listed in rows[0..nrows) (all rows when rows == NULL),
 * output row r of acc corresponds to token rows[r].
 * --------------------------------------------------------------------------------- */
void ora_int_gemm(const int8_t* xq, const int8_t* wq, int64_t T, int64_t N, int64_t K,
                  const int64_t* rows, int64_t nrows, int32_t* acc) {
    int64_t R = rows ? nrows : T;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        int64_t t = rows ? rows[r] : r;
        for (int64_t n = 0; n < N; ++n) {
            int32_t a = 0;
            for (int64_t k = 0; k < K; ++k) a += (int32_t)xq[t * K + k] * (int32_t)wq[n * K + k];
            acc[r * N + n] = a;
        }
    }
}

/* Output rescale (P3 §3.1: the linear of the dequantised operands times the weight scale;
 * with X_dq = x_q / s_t and W_dq = W_q * gamma the forward is acc * (gamma / s_t), i.e. the
 * integer contraction rescaled by one factor per token):
 *   c_t     = fl32( gamma / s_t )
 *   y[t, n] = fl32( (float)acc[t, n] * c_t ).      s_rows[r] is s of output row r. */
void ora_linear_epilogue(const int32_t* acc, int64_t R, int64_t N, float gamma,
                         const float* s_rows, float* y) {
    for (int64_t r = 0; r < R; ++r) {
        float c = gamma / s_rows[r];
        for (int64_t n = 0; n < N; ++n) {
            float a = (float)acc[r * N + n];
            y[r * N + n] = a * c;
        }
    }
}

/* ---------------------------------------------------------------------------------
 * Straight-through backward of the contraction (P3 §3.2: gradients reach the fp32
 * latent weights through the detach() trick; P5 §3.2 TernarySTE passes grad_output
 * unchanged; P4 §3.2 grad_w = grad_output).  With y = X_dq . W_dq^T and the STE taking
 * d X_dq / d x_hat = I and d W_dq / d W = I, scales treated as constants:
 *   dX_hat[t, k] = sum_n dY[t, n] * W_dq[n, k] = gamma * sum_n dY[t, n] * W_q[n, k]
 *   dW[n, k]     = sum_t dY[t, n] * X_dq[t, k]
 * Both in fp64 accumulation, rounded once to fp32.
 * dX_hat is computed for token rows rows[] (all when NULL); dW for weight rows nrows_w[].
 * --------------------------------------------------------------------------------- */
void ora_grad_input_hat(const float* dY, const int8_t* wq, float gamma, int64_t T, int64_t N,
                        int64_t K, const int64_t* rows, int64_t nrows, float* dxhat) {
    int64_t R = rows ? nrows : T;
#pragma omp parallel
    {
        double* acc = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(static)
        for (int64_t r = 0; r < R; ++r) {
            int64_t t = rows ? rows[r] : r;
            for (int64_t k = 0; k < K; ++k) acc[k] = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                double d = (double)dY[t * N + n];
                const int8_t* w = wq + n * K;
                for (int64_t k = 0; k < K; ++k) acc[k] += d * (double)w[k];
            }
            for (int64_t k = 0; k < K; ++k) dxhat[r * K + k] = (float)((double)gamma * acc[k]);
        }
        free(acc);
    }
}

void ora_grad_weight(const float* dY, const float* xdq, int64_t T, int64_t N, int64_t K,
                     const int64_t* wrows, int64_t nwrows, float* dW) {
    int64_t R = wrows ? nwrows : N;
#pragma omp parallel
    {
        double* acc = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(static)
        for (int64_t r = 0; r < R; ++r) {
            int64_t n = wrows ? wrows[r] : r;
            for (int64_t k = 0; k < K; ++k) acc[k] = 0.0;
            for (int64_t t = 0; t < T; ++t) {
                double d = (double)dY[t * N + n];
                const float* x = xdq + t * K;
                for (int64_t k = 0; k < K; ++k) acc[k] += d * (double)x[k];
            }
            for (int64_t k = 0; k < K; ++k) dW[r * K + k] = (float)acc[k];
        }
        free(acc);
    }
}

/* ---------------------------------------------------------------------------------
 * RMSNorm backward.  The pages apply RMSNorm before the quantiser (P3 §3.1) and the
 * STE passes the gradient of x_hat straight through the quantiser (P3 §2.2
 * activation_quant's detach()), so the gradient w.r.t. the layer input is the
 * textbook derivative of x_hat = x * r * g with r = (mean(x^2) + eps)^(-1/2),
 * evaluated with the saved fp32 r:
 *   u_k  = x_k * r,   h_k = g_k * dX_hat_k,   c = (1/K) sum_k h_k u_k
 *   dX_k = r * (h_k - u_k * c)
 *   dg_k = sum_t dX_hat[t, k] * u[t, k]
 * All in fp64, rounded once to fp32.  Rows rows[] (all when NULL); dg (may be NULL)
 * sums over those rows.
 * --------------------------------------------------------------------------------- */
void ora_rmsnorm_backward(const float* X, const float* rinv, const float* g, const float* dxhat,
                          int64_t T, int64_t K, const int64_t* rows, int64_t nrows,
                          float* dX, float* dg) {
    int64_t R = rows ? nrows : T;
    double* dgacc = NULL;
    if (dg) {
        dgacc = (double*)calloc((size_t)K, sizeof(double));
    }
    for (int64_t r = 0; r < R; ++r) {
        int64_t t = rows ? rows[r] : r;
        const float* x = X + t * K;
        const float* dh = dxhat + r * K;
        double rr = (double)rinv[t];
        double c = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double gk = g ? (double)g[k] : 1.0;
            c += gk * (double)dh[k] * ((double)x[k] * rr);
        }
        c /= (double)K;
        for (int64_t k = 0; k < K; ++k) {
            double gk = g ? (double)g[k] : 1.0;
            double u = (double)x[k] * rr;
            double h = gk * (double)dh[k];
            dX[r * K + k] = (float)(rr * (h - u * c));
            if (dgacc) dgacc[k] += (double)dh[k] * u;
        }
    }
    if (dg) {
        for (int64_t k = 0; k < K; ++k) dg[k] = (float)dgacc[k];
        free(dgacc);
    }
}

/* ---------------------------------------------------------------------------------
 * Decode GEMV over the 2-bit packed weights (P5 §3.1 add / subtract / skip; P5 §4.1
 * codes).  For each of B activation rows:
 *   acc[b, n] = sum_k decode(packed[n, k]) * x_q[b, k]      exact int32
 *   y[b, n]   = fl32( (float)acc * fl32(gamma / s_b) )
 * The loop literally adds, subtracts or skips, as the page describes.
 * --------------------------------------------------------------------------------- */
void ora_gemv(const uint8_t* packed, float gamma, int64_t N, int64_t K, const int8_t* xq,
              const float* s, int64_t B, int32_t* acc, float* y) {
    int64_t row_bytes = K / 4;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < B; ++b) {
            int32_t a = 0;
            for (int64_t k = 0; k < K; ++k) {
                unsigned c = (packed[n * row_bytes + k / 4] >> (2 * (k % 4))) & 3u;
                int w = decode2(c);
                if (w == 1) a += xq[b * K + k];
                else if (w == -1) a -= xq[b * K + k];
            }
            acc[b * N + n] = a;
            float c = gamma / s[b];
            y[b * N + n] = (float)a * c;
        }
    }
}

/* bf16 helpers exposed for tests: decode bf16 bits to fp32 (exact). */
void ora_bf16_to_f32(const uint16_t* in, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_bits_to_f32(in[i]);
}

/* =================================================================================
 * Variants the pages print beside the b1.58 defaults (cheap parameterisations of the
 * two quantisers).  Same arithmetic conventions as above.
 * ================================================================================= */

/* Per-row weight scale (P4 §9 "Quantizer": scale = mean(|x|, dim=1, keepdim=True), one
 * scale per output row), combined with the b1.58 round/clamp of P3 §2.1 / P5 §2.2:
 *   gamma_n   = max( (float)( sum_k |W[n,k]| / K ), 1e-5 )      fp64 sum, index order
 *   W_q[n,k]  = clamp(round(fl32(W[n,k] / gamma_n)), -1, 1). */
void ora_absmean_gamma_rows(const float* W, int64_t N, int64_t K, float* gamma) {
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        double S = 0.0;
        for (int64_t k = 0; k < K; ++k) S += (double)fabsf(W[n * K + k]);
        float mean = (float)(S / (double)K);
        gamma[n] = fmaxf(mean, 1e-5f);
    }
}

void ora_ternary_round_rows(const float* W, int64_t N, int64_t K, const float* gamma, int8_t* wq) {
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            float v = nearbyintf(W[n * K + k] / gamma[n]);
            if (v < -1.0f) v = -1.0f;
            if (v > 1.0f) v = 1.0f;
            wq[n * K + k] = (int8_t)v;
        }
}

/* Zero threshold (P2 "直通估计器在三元权重量化中的作用": tau = 0.7 * scale, |W| < tau
 * quantises to 0; the other weights keep their sign), with the per-tensor gamma:
 *   tau = fl32(tau_factor * gamma);   W_q = 0 if |W| < tau, else sign(W) (sign(0) = 0). */
void ora_ternary_tau(const float* W, int64_t n, float gamma, float tau_factor, int8_t* wq) {
    float tau = tau_factor * gamma;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(W[i]);
        wq[i] = (int8_t)(a < tau ? 0 : (W[i] > 0.0f) - (W[i] < 0.0f));
    }
}

/* Per-tensor activation scale (P5 §5.1 quantize_activation: scale = 127 / max|x| over the
 * whole tensor), applied to x_hat as in ora_act_quant, with the same 1e-5 floor and clamp:
 *   s = fl32(127 / max(max_{t,k} |x_hat|, 1e-5)),  q = clamp(round(fl32(x_hat s)), -128, 127),
 *   X_dq = fl32(q / s).  s_out receives s for every token (one value repeated). */
void ora_act_quant_tensor(const float* X, int64_t T, int64_t K, const float* rinv, const float* g,
                          int8_t* xq, float* s_out, float* xdq) {
    float m = 0.0f;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t k = 0; k < K; ++k) {
            float v = X[t * K + k];
            if (rinv) {
                v = v * rinv[t];
                if (g) v = v * g[k];
            }
            float a = fabsf(v);
            if (a > m) m = a;
        }
    float s = 127.0f / fmaxf(m, 1e-5f);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        s_out[t] = s;
        for (int64_t k = 0; k < K; ++k) {
            float v = X[t * K + k];
            if (rinv) {
                v = v * rinv[t];
                if (g) v = v * g[k];
            }
            float r = nearbyintf(v * s);
            if (r < -128.0f) r = -128.0f;
            if (r > 127.0f) r = 127.0f;
            int8_t q = (int8_t)r;
            xq[t * K + k] = q;
            if (xdq) xdq[t * K + k] = (float)q / s;
        }
    }
}

/* Output rescale with a per-row weight scale: y[t, n] = fl32( (float)acc[t, n] * fl32(gamma_n / s_t) ). */
void ora_linear_epilogue_rows(const int32_t* acc, int64_t R, int64_t N, const float* gamma,
                              const float* s_rows, float* y) {
    for (int64_t r = 0; r < R; ++r)
        for (int64_t n = 0; n < N; ++n) {
            float c = gamma[n] / s_rows[r];
            y[r * N + n] = (float)acc[r * N + n] * c;
        }
}

/* =================================================================================
 * Optimizer step of the latent weight, in the order the pages give it: gradient
 * clipping to a maximum L2 norm (P5 §6.2: clip_grad_norm_ per weight matrix with
 * max_norm 1.0; P3 §6 and P4 §4.1 the same threshold over the model), then AdamW
 * (P2 training pipeline: AdamW; hyper-parameters lr 1e-3, betas (0.9, 0.95), weight decay
 * 0.01, eps 1e-6 from P1 "工程实践：可落地参数配置", optimizer configuration), then
 * the clamp of the latent weight to [-1, 1] (P1 "梯度裁剪与权重约束").  AdamW is the decoupled-weight-decay algorithm of Loshchilov
 * and Hutter with bias-corrected moments:
 *   norm = sqrt(sum_i dW_i^2);  c = min(1, max_norm / (norm + 1e-6))   (c = 1 if max_norm <= 0)
 *   g = c dW;  W <- W - lr wd W;  m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2
 *   W <- W - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps);  W <- clamp(W, -1, 1)
 * All arithmetic in fp64 from the fp32 inputs; W, m, v are stored back rounded to fp32.
 * t is the 1-based index of this step.  Returns c.
 * --------------------------------------------------------------------------------- */
double ora_optimizer_step(float* W, const float* dW, float* m, float* v, int64_t n, double lr, double beta1,
                          double beta2, double eps, double wd, double max_norm, int64_t t) {
    double S = 0.0;
    for (int64_t i = 0; i < n; ++i) S += (double)dW[i] * (double)dW[i];
    double norm = sqrt(S);
    double c = 1.0;
    if (max_norm > 0.0) {
        c = max_norm / (norm + 1e-6);
        if (c > 1.0) c = 1.0;
    }
    double bc1 = 1.0 - pow(beta1, (double)t);
    double bc2 = 1.0 - pow(beta2, (double)t);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double g = c * (double)dW[i];
        double w = (double)W[i];
        w = w - lr * wd * w;
        double mi = beta1 * (double)m[i] + (1.0 - beta1) * g;
        double vi = beta2 * (double)v[i] + (1.0 - beta2) * g * g;
        w = w - lr * (mi / bc1) / (sqrt(vi / bc2) + eps);
        if (w < -1.0) w = -1.0;
        if (w > 1.0) w = 1.0;
        W[i] = (float)w;
        m[i] = (float)mi;
        v[i] = (float)vi;
    }
    return c;
}
