/*
 * ternary_oracle.c — reference oracle for the ternary-weight linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is plain, slow, single-threaded C
 * that restates what the method computes, for the parity tests, the smoke
 * check and the CPU-baseline leg of the benchmark.  Nothing in the product
 * path may include, link or call it, and it shares no code, header, table or
 * helper with the CUDA implementation.
 *
 * What it computes (sources are the pages on VibeVoice-ASR-BitNet):
 *   - Per-tensor ternarisation of a projection matrix W [N x K]:
 *       s = 1 / mean|W| over the whole tensor, codes = round(W * s) clipped
 *       to {-1, 0, +1}.  ("VibeVoice-ASR-BitNet-ONNX" model page,
 *       "Quantization" table, row "LM projections (196 mats)": I2_S ternary,
 *       per-tensor s = 1/mean|W|; "The Paper Says ARM Support" post, section
 *       "What the model is trying to do": every weight becomes -1, 0 or +1.)
 *   - Per-token int8 activation quantisation by absmax, an int32 (here
 *       int64-checked) ternary dot product, and the rescale by absmax/127 and
 *       1/s.  The pages only say the engine uses fused INT8 operations
 *       (xujun.org article, section on heterogeneous quantisation; aitrends
 *       summary, "Technical features"); the formula below is the plainest
 *       reading of absmax int8 quantisation.
 *   - The dot product itself is a plain sum of code * q: ternary weights turn
 *       the multiply into add/subtract (xujun.org article, heterogeneous
 *       quantisation section).
 *
 * Readings taken where the pages are silent (each one is listed in the
 * design notes of the repository):
 *   R1  rounding of W*s and of x*scale is round-half-to-even (IEEE rint).
 *   R2  mean|W| is accumulated in fp64 in a fixed order: each row summed
 *       sequentially over k, then the row sums summed sequentially over n;
 *       the total is divided by N*K.
 *   R3  mean|W| is floored at 1e-5 (an all-zero W then gives all-zero codes).
 *   R4  the activation scale is computed in fp32: amax = max|x| (exact),
 *       scale = 127.0f / amax (IEEE single division), q = rint(x * scale) in
 *       single precision, clamped to [-128, 127].  A row with amax == 0 gives
 *       q == 0 and y == 0.
 *   R5  y = acc * (amax / 127) * mean|W|, evaluated here in fp64.
 *
 * Build: gcc -O1 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (contraction off so that x * scale is a single IEEE multiply).
 */
#include <math.h>
#include <stdint.h>

#define ORC_MEAN_FLOOR 1e-5

/* R2 + R3: mean of |W| over the whole [N x K] tensor. */
double orc_mean_abs(const float *W, int64_t N, int64_t K)
{
    double total = 0.0;
    for (int64_t n = 0; n < N; ++n) {
        double row = 0.0;
        for (int64_t k = 0; k < K; ++k)
            row += fabs((double)W[n * K + k]);
        total += row;
    }
    double mean = total / (double)(N * K);
    if (mean < ORC_MEAN_FLOOR)
        mean = ORC_MEAN_FLOOR;
    return mean;
}

/* Ternarise W with s = 1/mean|W|.  Writes codes[n*K+k] in {-1,0,1} and the
 * mean to *mean_out.  Returns 0, or 1 if W holds a non-finite value (codes
 * are then left unwritten). */
int orc_ternarize(const float *W, int64_t N, int64_t K, double *mean_out,
                  int8_t *codes)
{
    for (int64_t i = 0; i < N * K; ++i)
        if (!isfinite(W[i]))
            return 1;
    double mean = orc_mean_abs(W, N, K);
    double s = 1.0 / mean;
    for (int64_t i = 0; i < N * K; ++i) {
        double r = rint((double)W[i] * s);
        if (r > 1.0)
            r = 1.0;
        if (r < -1.0)
            r = -1.0;
        codes[i] = (int8_t)r;
    }
    *mean_out = mean;
    return 0;
}

/* R4: per-token absmax int8 quantisation of x [M x K]. */
void orc_quantize_act(const float *x, int64_t M, int64_t K, int8_t *q,
                      float *amax)
{
    for (int64_t m = 0; m < M; ++m) {
        const float *row = x + m * K;
        float a = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = fabsf(row[k]);
            if (v > a)
                a = v;
        }
        amax[m] = a;
        if (a == 0.0f) {
            for (int64_t k = 0; k < K; ++k)
                q[m * K + k] = 0;
            continue;
        }
        float scale = 127.0f / a;
        for (int64_t k = 0; k < K; ++k) {
            float v = row[k] * scale;
            float r = rintf(v);
            if (r > 127.0f)
                r = 127.0f;
            if (r < -128.0f)
                r = -128.0f;
            q[m * K + k] = (int8_t)r;
        }
    }
}

/* acc[m*N+n] = sum_k codes[n*K+k] * q[m*K+k].  Summed in int64; returns 0,
 * or 1 if a sum does not fit int32 (acc is still written, truncated). */
int orc_ternary_acc(const int8_t *codes, int64_t N, int64_t K,
                    const int8_t *q, int64_t M, int32_t *acc)
{
    int overflow = 0;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t sum = 0;
            for (int64_t k = 0; k < K; ++k)
                sum += (int64_t)codes[n * K + k] * (int64_t)q[m * K + k];
            if (sum > INT32_MAX || sum < INT32_MIN)
                overflow = 1;
            acc[m * N + n] = (int32_t)sum;
        }
    }
    return overflow;
}

/* R5: y[m*N+n] = acc[m*N+n] * (amax[m] / 127) * mean, in fp64. */
void orc_rescale(const int32_t *acc, int64_t M, int64_t N, const float *amax,
                 double mean, double *y)
{
    for (int64_t m = 0; m < M; ++m) {
        double a = (double)amax[m] / 127.0;
        for (int64_t n = 0; n < N; ++n)
            y[m * N + n] = (double)acc[m * N + n] * a * mean;
    }
}

/* The whole layer on already-ternarised codes: quantise x, accumulate,
 * rescale.  Any of q_out / amax_out / acc_out may be scratch supplied by the
 * caller; all are written.  Returns the overflow flag of orc_ternary_acc. */
int orc_ternary_linear(const float *x, int64_t M, const int8_t *codes,
                       int64_t N, int64_t K, double mean, int8_t *q_out,
                       float *amax_out, int32_t *acc_out, double *y_out)
{
    orc_quantize_act(x, M, K, q_out, amax_out);
    int ovf = orc_ternary_acc(codes, N, K, q_out, M, acc_out);
    orc_rescale(acc_out, M, N, amax_out, mean, y_out);
    return ovf;
}

/* ------------------------------------------------------------------------
 * Decoder-layer chain: the steps on either side of the projections.
 *
 * A layer of the LM decoder (a Qwen2.5-1.5B decoder: "VibeVoice-ASR-BitNet-
 * ONNX" model page, "Layout", where decoder_model_merged maps inputs_embeds
 * and the KV cache to logits) runs q, k and v on one input, attention, o,
 * then gate and up on a second input, SiLU(gate) * up, and down.  The chain
 * keeps those data dependencies and replaces what would need trained weights
 * or a KV cache by weight-free stand-ins (readings taken here, listed with
 * the others in the design notes):
 *   R13 attention is the identity over positions: every token attends only
 *       to itself, so its output is its own v, each KV head repeated for the
 *       query heads of its group (hidden/head_dim query heads, kv/head_dim KV
 *       heads in equal groups).
 *   R14 no normalisation layers (their gains are weights).
 *   R15 a residual connection around each block, added in fp32:
 *       h1 = h + o, then h' = h1 + d.
 *   R16 SiLU(g) * u with SiLU(z) = z / (1 + e^-z), evaluated here in fp64
 *       from the fp32 inputs.
 * ---------------------------------------------------------------------- */

/* R13: a [M x hidden] from v [M x kv_dim]. */
void orc_gqa_expand(const float *v, int64_t M, int64_t kv_dim, int64_t hidden,
                    int64_t head_dim, float *a)
{
    const int64_t n_heads = hidden / head_dim;
    const int64_t n_kv = kv_dim / head_dim;
    const int64_t group = n_heads / n_kv;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t h = 0; h < n_heads; ++h)
            for (int64_t c = 0; c < head_dim; ++c)
                a[m * hidden + h * head_dim + c] = v[m * kv_dim + (h / group) * head_dim + c];
}

/* R15: out = x + y, one IEEE single-precision addition per element. */
void orc_add_f32(const float *x, const float *y, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = x[i] + y[i];
}

/* R16: out = SiLU(g) * u in fp64. */
void orc_silu_mul(const float *g, const float *u, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i) {
        const double z = (double)g[i];
        out[i] = z / (1.0 + exp(-z)) * (double)u[i];
    }
}

/* ------------------------------------------------------------------------
 * I8_S linear with fused bias and ReLU: the int8 side of the model.
 *
 * The audio encoder (VAE tokenizer) keeps int8 weights and int8 activations
 * and replaces GELU by ReLU ("VibeVoice-ASR-BitNet-ONNX" model page,
 * "Quantization" table, row "VAE encoders": I8_S); its fused int8 routines
 * join matmul, bias and ReLU in one pass (aitrends summary, technical
 * features); it is bound by data movement, activations outweighing weights
 * 16 to 1 ("The Paper Says ARM Support" post, "What the model is trying to
 * do").  The pages fix neither the weight scale's granularity nor the
 * rounding; readings taken here:
 *   R17 I8_S weights carry one scale per tensor (the "_S" format of the
 *       ternary weights is per tensor too, and the ONNX page contrasts its
 *       own per-channel int8 weights with it): wq = the absmax int8
 *       quantisation of the whole tensor, the same rule as R4 applied to W
 *       as one row, amax_w = max|W|.
 *   R18 activations are quantised per token as in R4.
 *   R19 y = acc * (amax_x/127) * (amax_w/127) + bias, then ReLU when asked
 *       (max(0, y)); evaluated here in fp64.  A missing bias is zero.
 * ---------------------------------------------------------------------- */

/* R17: wq [N x K] and amax_w of W [N x K]. */
void orc_i8_quantize_weights(const float *W, int64_t N, int64_t K, int8_t *wq,
                             float *amax_w)
{
    orc_quantize_act(W, 1, N * K, wq, amax_w);
}

/* R19: y[m*N+n] from the exact accumulators (orc_ternary_acc computes the
 * int8 dot products for any int8 weights). */
void orc_i8_epilogue(const int32_t *acc, int64_t M, int64_t N,
                     const float *amax_x, float amax_w, const float *bias,
                     int relu, double *y)
{
    const double w = (double)amax_w / 127.0;
    for (int64_t m = 0; m < M; ++m) {
        const double a = (double)amax_x[m] / 127.0;
        for (int64_t n = 0; n < N; ++n) {
            double v = (double)acc[m * N + n] * a * w;
            if (bias)
                v += (double)bias[n];
            if (relu && v < 0.0)
                v = 0.0;
            y[m * N + n] = v;
        }
    }
}

/* ------------------------------------------------------------------------
 * Tensor-parallel split (this library's own; the pages describe one CPU
 * process).  A row-parallel projection quantises each rank's slice of a
 * token row with the absmax of the whole row, which the ranks share:
 *   R20 q = clamp(rint(x * (127 / amax_row)), -128, 127), the R4 rule with
 *       the given amax (a row maximum over all slices), amax == 0 -> q = 0.
 * The partial sums of the slices add up to orc_ternary_acc of the whole row.
 * ---------------------------------------------------------------------- */
void orc_quantize_act_given(const float *x, int64_t M, int64_t K,
                            const float *amax, int8_t *q)
{
    for (int64_t m = 0; m < M; ++m) {
        const float a = amax[m];
        if (a == 0.0f) {
            for (int64_t k = 0; k < K; ++k)
                q[m * K + k] = 0;
            continue;
        }
        const float scale = 127.0f / a;
        for (int64_t k = 0; k < K; ++k) {
            float r = rintf(x[m * K + k] * scale);
            if (r > 127.0f)
                r = 127.0f;
            if (r < -128.0f)
                r = -128.0f;
            q[m * K + k] = (int8_t)r;
        }
    }
}
