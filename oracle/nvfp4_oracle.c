/*
 * nvfp4_oracle.c -- plain, slow CPU reference for the NVFP4 routed-expert MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this code: only the
 * test suite, the smoke check of the package entry module and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or constant generator with the
 * CUDA library; the two meet only on the seeded input bytes.
 *
 * What it follows (page "GLM-5-NVFP4-MTP"):
 *   - "Model Description": the weights are NVFP4, 4-bit values with one FP8 scale per
 *     16 consecutive elements; the model has 256 experts per MoE layer, 8 active per token.
 *   - "What's quantized": only the routed experts' gate, up and down projections are NVFP4.
 * The element type (E2M1), the scale type (E4M3, finite-only "FN" variant), the single fp32
 * global scale per tensor and the block-scale rule "block amax / 6, rounded to E4M3" are the
 * task's definition of that format; every point those sources leave open is resolved by a
 * reading stated next to the code that takes it.
 *
 * Precision: codec steps are done in IEEE fp32 exactly as stated (each operation rounds to
 * nearest even; build with -ffp-contract=off, never -ffast-math); the MoE forward accumulates
 * in fp64 over exactly decoded weights.
 *
 * Every function is deliberately the plainest statement of its definition: encoders search
 * all codes for the nearest value, the MoE loops token by token over the selected experts.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------- */
/* Element and scale formats                                                             */
/* ------------------------------------------------------------------------------------- */

/* E2M1: bit 3 = sign, bits 2..1 = exponent (bias 1), bit 0 = mantissa.
 * Exponent field 0 is subnormal: magnitude = mantissa * 0.5.
 * Otherwise magnitude = (1 + mantissa/2) * 2^(exponent - 1). */
double oracle_e2m1_value(int code)
{
    int s = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag;
    if (e == 0)
        mag = 0.5 * m;
    else
        mag = ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* E4M3 ("FN": finite, no infinities): bit 7 = sign, bits 6..3 = exponent (bias 7),
 * bits 2..0 = mantissa.  Exponent 15 with mantissa 7 is NaN; every other code is finite.
 * Exponent field 0 is subnormal: magnitude = (mantissa/8) * 2^-6. */
double oracle_e4m3_value(int code)
{
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 15;
    int m = code & 7;
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp(m / 8.0, -6);
    else
        mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Nearest E4M3 code to v, ties to the even code, saturating to the largest finite
 * magnitude (448, code 0x7E): any magnitude at or above 448 takes 0x7E ("satfinite").
 * Below that, searching all finite magnitudes for the nearest one is the definition of
 * round-to-nearest.  The sign bit is v's sign bit. */
int oracle_e4m3_encode(float v)
{
    int sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0)
        return sign | 0x7E;
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(a - oracle_e4m3_value(c));
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    return sign | best;
}

/* Nearest E2M1 code to v, ties to the even code (mantissa bit 0); any magnitude at or
 * above 6 saturates to 6 (code 7).  The sign bit is v's sign bit, so a negative value
 * that rounds to zero gives code 0x8 (negative zero).  [Reading: the format sources do not say how a negative value that
 * rounds to zero is stored; keeping the sign bit is the plain IEEE-style choice.] */
int oracle_e2m1_encode(float v)
{
    int sign = signbit(v) ? 0x8 : 0x0;
    double a = fabs((double)v);
    if (a >= 6.0)
        return sign | 0x7;
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c <= 7; ++c) {
        double d = fabs(a - oracle_e2m1_value(c));
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    return sign | best;
}

/* ------------------------------------------------------------------------------------- */
/* bf16                                                                                  */
/* ------------------------------------------------------------------------------------- */

/* bf16 keeps the upper 16 bits of an fp32, so widening is exact. */
float oracle_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* The bf16 nearest to the finite value v, ties to even, with one rounding from v itself.
 * bf16 has 8 significant bits and fp32's exponent range (smallest subnormal 2^-133). */
uint16_t oracle_bf16_round(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0x0000;
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    int e;
    frexp(a, &e);                 /* a = f * 2^e with f in [0.5, 1) */
    int q = e - 8;                /* spacing of bf16 values in [2^(e-1), 2^e) */
    if (q < -133)
        q = -133;                 /* subnormal spacing */
    double r = nearbyint(ldexp(a, -q)) ;  /* default rounding mode: to nearest, ties to even */
    double rv = ldexp(r, q);
    if (rv > 3.3895313892515355e38)       /* above the largest finite bf16 */
        return sign | 0x7F80;
    float f = (float)rv;                  /* exact: rv is a bf16 value */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return sign | (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------------------- */
/* NVFP4 quantize / dequantize                                                           */
/* ------------------------------------------------------------------------------------- */

/* Largest E2M1 magnitude times largest E4M3 magnitude. */
#define NVFP4_E2M1_MAX 6.0f
#define NVFP4_E4M3_MAX 448.0f

/* Global scale of one tensor.  [Reading: the format gives one fp32 global scale per tensor
 * but not how it is chosen.  g = amax / (6 * 448) maps the tensor's largest block onto the
 * top of the E4M3 range, so every block scale fits; an all-zero tensor takes g = 1.] */
float oracle_global_scale(const uint16_t *x, int64_t n)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(oracle_bf16_to_f32(x[i]));
        if (a > amax)
            amax = a;
    }
    if (amax == 0.0f)
        return 1.0f;
    return amax / (NVFP4_E2M1_MAX * NVFP4_E4M3_MAX);
}

/* Quantize one 16-element block with global scale g.
 * Steps, each an fp32 operation rounded to nearest even:
 *   amax_b = max |x_i|;  s = (amax_b / 6) / g;  code_s = E4M3(s)  (satfinite)
 *   d = e4m3_value(code_s) * g;  code_i = E2M1(x_i / d), or 0 when d == 0.
 * [Reading: the block scale is "amax / 6 rounded to E4M3" taken in units of the global
 * scale; the division by 6 comes first, then the division by g.  Elements are divided by
 * the decoded scale times g (not multiplied by a reciprocal).  A block whose decoded scale
 * is zero stores all-zero codes.] */
static void quantize_block(const uint16_t *x, float g, uint8_t *codes, uint8_t *scale_code)
{
    float amax_b = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(oracle_bf16_to_f32(x[i]));
        if (a > amax_b)
            amax_b = a;
    }
    float s = (amax_b / NVFP4_E2M1_MAX) / g;
    int sc = oracle_e4m3_encode(s);
    float sd = (float)oracle_e4m3_value(sc);
    float d = sd * g;
    *scale_code = (uint8_t)sc;
    for (int i = 0; i < 16; ++i) {
        if (d == 0.0f)
            codes[i] = 0;
        else
            codes[i] = (uint8_t)oracle_e2m1_encode(oracle_bf16_to_f32(x[i]) / d);
    }
}

/* x: n_tensors tensors of [rows, cols] bf16, row-major, cols % 16 == 0.
 * packed: [n, rows, cols/2]; byte j of a row holds element 2j in its low nibble and
 * element 2j+1 in its high nibble.  scales: [n, rows, cols/16] E4M3 codes.  g: [n]. */
void oracle_nvfp4_quantize(const uint16_t *x, int64_t n_tensors, int64_t rows, int64_t cols,
                           uint8_t *packed, uint8_t *scales, float *g_out)
{
    int64_t per = rows * cols;
    for (int64_t t = 0; t < n_tensors; ++t) {
        const uint16_t *xt = x + t * per;
        float g = oracle_global_scale(xt, per);
        g_out[t] = g;
        #pragma omp parallel for schedule(static)
        for (int64_t r = 0; r < rows; ++r) {
            for (int64_t b = 0; b < cols / 16; ++b) {
                uint8_t codes[16], sc;
                quantize_block(xt + r * cols + b * 16, g, codes, &sc);
                scales[t * rows * (cols / 16) + r * (cols / 16) + b] = sc;
                uint8_t *dst = packed + t * rows * (cols / 2) + r * (cols / 2) + b * 8;
                for (int j = 0; j < 8; ++j)
                    dst[j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
            }
        }
    }
}

/* ------------------------------------------------------------------------------------- */
/* Calibrated (static) global scales                                                     */
/* ------------------------------------------------------------------------------------- */

/* Per-tensor amax, max |x| over each tensor of `per` elements (exact: bf16 -> fp32).  Page
 * "GLM-5-NVFP4-MTP", "Calibration dataset": several calibration passes are merged by
 * element-wise max.  With merge == 0 amax[t] is set; with merge != 0 it becomes the larger
 * of its value and this pass's, so calling once per pass leaves the merged amax. */
void oracle_nvfp4_amax(const uint16_t *x, int64_t n_tensors, int64_t per, float *amax, int merge)
{
    for (int64_t t = 0; t < n_tensors; ++t) {
        float a = 0.0f;
        for (int64_t i = 0; i < per; ++i) {
            float v = fabsf(oracle_bf16_to_f32(x[t * per + i]));
            if (v > a)
                a = v;
        }
        if (!merge || a > amax[t])
            amax[t] = a;
    }
}

/* Quantize with a given tensor amax (a calibrated one) in place of the tensor's own:
 * g = amax_in / (6 * 448), 1 when amax_in == 0, then every block as in
 * oracle_nvfp4_quantize.  Data beyond the calibrated range saturates: a block scale above
 * 448 is stored as 448 and an element code above 6 as 6 (the E4M3 and E2M1 encoders
 * saturate).  [Reading: amax_in >= 0 and finite; other values are not defined.] */
void oracle_nvfp4_quantize_with_amax(const uint16_t *x, int64_t n_tensors, int64_t rows,
                                     int64_t cols, const float *amax_in, uint8_t *packed,
                                     uint8_t *scales, float *g_out)
{
    int64_t per = rows * cols;
    for (int64_t t = 0; t < n_tensors; ++t) {
        const uint16_t *xt = x + t * per;
        float g = amax_in[t] == 0.0f ? 1.0f : amax_in[t] / (NVFP4_E2M1_MAX * NVFP4_E4M3_MAX);
        g_out[t] = g;
        #pragma omp parallel for schedule(static)
        for (int64_t r = 0; r < rows; ++r) {
            for (int64_t b = 0; b < cols / 16; ++b) {
                uint8_t codes[16], sc;
                quantize_block(xt + r * cols + b * 16, g, codes, &sc);
                scales[t * rows * (cols / 16) + r * (cols / 16) + b] = sc;
                uint8_t *dst = packed + t * rows * (cols / 2) + r * (cols / 2) + b * 8;
                for (int j = 0; j < 8; ++j)
                    dst[j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
            }
        }
    }
}

/* Dequantize: out = bf16( fp32( e2m1 * e4m3 ) * g ).  The first product is exact in fp32
 * (at most 6 significant bits); the multiply by g rounds once in fp32, and the conversion
 * to bf16 rounds a second time.  [Reading: the format sources give no dequantizer; this
 * is the product of the three factors in the order they are stored, in fp32 like g.] */
void oracle_nvfp4_dequantize(const uint8_t *packed, const uint8_t *scales, const float *g,
                             int64_t n_tensors, int64_t rows, int64_t cols, uint16_t *out)
{
    for (int64_t t = 0; t < n_tensors; ++t) {
        #pragma omp parallel for schedule(static)
        for (int64_t r = 0; r < rows; ++r) {
            for (int64_t c = 0; c < cols; ++c) {
                uint8_t byte = packed[t * rows * (cols / 2) + r * (cols / 2) + c / 2];
                int code = (c & 1) ? (byte >> 4) : (byte & 15);
                int sc = scales[t * rows * (cols / 16) + r * (cols / 16) + c / 16];
                float qs = (float)(oracle_e2m1_value(code) * oracle_e4m3_value(sc));
                float v = qs * g[t];
                out[t * rows * cols + r * cols + c] = oracle_bf16_round((double)v);
            }
        }
    }
}

/* ------------------------------------------------------------------------------------- */
/* Routing permutation                                                                   */
/* ------------------------------------------------------------------------------------- */

/* Group the T*K (token, slot) pairs by expert.  counts[e] = number of pairs routed to e;
 * offsets = exclusive prefix sum of counts (E+1 entries); perm lists, expert by expert, the
 * flat pair index t*K+k in ascending order; inv[t*K+k] = position of that pair in perm.
 * Pairs whose id lies outside [0, E) are left out of perm and get inv = -1.
 * Returns the number of such pairs. */
int64_t oracle_route(const int32_t *ids, int64_t T, int64_t K, int64_t E,
                     int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv)
{
    int64_t bad = 0;
    for (int64_t e = 0; e < E; ++e)
        counts[e] = 0;
    for (int64_t p = 0; p < T * K; ++p) {
        if (ids[p] >= 0 && ids[p] < E)
            counts[ids[p]]++;
        else
            bad++;
    }
    offsets[0] = 0;
    for (int64_t e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];
    for (int64_t e = 0; e < E; ++e) {
        int32_t pos = offsets[e];
        for (int64_t p = 0; p < T * K; ++p)
            if (ids[p] == e)
                perm[pos++] = (int32_t)p;
    }
    for (int64_t p = 0; p < T * K; ++p)
        inv[p] = -1;
    for (int64_t j = 0; j < offsets[E]; ++j)
        inv[perm[j]] = (int32_t)j;
    return bad;
}

/* ------------------------------------------------------------------------------------- */
/* Router                                                                                */
/* ------------------------------------------------------------------------------------- */

/* The router's decision per token.  Page "GLM-5-NVFP4-MTP", "Model Description": each
 * token is served by 8 of the 256 experts; "What's quantized" keeps the router in BF16/fp32.
 * The pages do not give the router's function.  Reading taken: p = softmax(logits[t, :]),
 * the K experts of largest p, in descending order of p with the lower index first among
 * equal p, and weights w_k = p_k / (sum of the K selected p).
 * Which p is larger is decided on the fp32 logits, which is the exact order of the
 * real-valued softmax (it is strictly increasing in the logit).  Comparing the fp64-rounded
 * p instead would create false ties where exp underflows or where l - max rounds to the
 * same double.  The weights follow the definition in fp64: softmax over all E, then
 * renormalisation over the selected K.
 *   logits [T, E] fp32  ->  ids [T, K] int32, w [T, K] fp64                              */
void oracle_router(const float *logits, int64_t T, int64_t E, int64_t K, int32_t *ids,
                   double *w)
{
    double *p = (double *)malloc((size_t)E * sizeof(double));
    unsigned char *taken = (unsigned char *)malloc((size_t)E);
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        double m = -INFINITY;
        for (int64_t e = 0; e < E; ++e)
            if ((double)l[e] > m) m = (double)l[e];
        double z = 0.0;
        for (int64_t e = 0; e < E; ++e) {
            p[e] = exp((double)l[e] - m);
            z += p[e];
        }
        for (int64_t e = 0; e < E; ++e) p[e] = p[e] / z;
        memset(taken, 0, (size_t)E);
        double s = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e)   /* strict >: the lower index wins a tie */
                if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
            taken[best] = 1;
            ids[t * K + k] = (int32_t)best;
            w[t * K + k] = p[best];
            s += p[best];
        }
        for (int64_t k = 0; k < K; ++k) w[t * K + k] = w[t * K + k] / s;
    }
    free(p);
    free(taken);
}

/* ------------------------------------------------------------------------------------- */
/* MoE forward                                                                           */
/* ------------------------------------------------------------------------------------- */

/* Exact value of element (r, c) of one NVFP4 matrix with `cols` columns. */
static double nvfp4_weight(const uint8_t *packed, const uint8_t *scales, double g,
                           int64_t cols, int64_t r, int64_t c)
{
    uint8_t byte = packed[r * (cols / 2) + c / 2];
    int code = (c & 1) ? (byte >> 4) : (byte & 15);
    int sc = scales[r * (cols / 16) + c / 16];
    return oracle_e2m1_value(code) * oracle_e4m3_value(sc) * g;   /* exact in fp64 */
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* Routed-expert MoE MLP for the tokens listed in tok[0..n_tok).  For token t:
 *   out[t] = sum over k = 0..K-1 (ascending) of w[t,k] * y_k, where, with e = ids[t,k],
 *   a   = Wgu[e] x_t                          (2I values; rows 0..I-1 gate, I..2I-1 up)
 *   h_j = bf16( silu(a_j) * a_{I+j} )         (SwiGLU, rounded to bf16)
 *   y_k = Wdn[e] h                            (H values)
 * with every weight the exact NVFP4 value e2m1 * e4m3 * g and all sums in fp64.
 * [Readings: gate rows come first in the fused gate/up matrix; h is rounded to bf16 once,
 * as a bf16 matmul input would be; routing weights are fp32; a repeated expert id within a
 * token contributes once per slot; an id outside [0, E) contributes nothing and is counted.]
 * Shapes: x [T,H] bf16; ids, w [T,K]; Wgu packed [E,2I,H/2], scales [E,2I,H/16], g [E];
 * Wdn packed [E,H,I/2], scales [E,H,I/16], g [E].  out [n_tok,H] bf16; out64 (optional)
 * [n_tok,H] fp64.  Returns the number of out-of-range ids met. */
int64_t oracle_moe_forward(const uint16_t *x, const int32_t *ids, const float *w,
                           int64_t T, int64_t H, int64_t I, int64_t E, int64_t K,
                           const uint8_t *wgu, const uint8_t *sgu, const float *ggu,
                           const uint8_t *wdn, const uint8_t *sdn, const float *gdn,
                           const int64_t *tok, int64_t n_tok, uint16_t *out, double *out64)
{
    (void)T;
    int64_t bad = 0;
    double *xt = (double *)malloc(sizeof(double) * H);
    double *a = (double *)malloc(sizeof(double) * 2 * I);
    double *hb = (double *)malloc(sizeof(double) * I);
    double *acc = (double *)malloc(sizeof(double) * H);
    for (int64_t i = 0; i < n_tok; ++i) {
        int64_t t = tok[i];
        for (int64_t c = 0; c < H; ++c) {
            xt[c] = oracle_bf16_to_f32(x[t * H + c]);
            acc[c] = 0.0;
        }
        for (int64_t k = 0; k < K; ++k) {
            int64_t e = ids[t * K + k];
            if (e < 0 || e >= E) {
                bad++;
                continue;
            }
            const uint8_t *pg = wgu + e * (2 * I) * (H / 2);
            const uint8_t *sg = sgu + e * (2 * I) * (H / 16);
            const uint8_t *pd = wdn + e * H * (I / 2);
            const uint8_t *sd = sdn + e * H * (I / 16);
            double g1 = ggu[e], g2 = gdn[e];
            #pragma omp parallel for schedule(static)
            for (int64_t j = 0; j < 2 * I; ++j) {
                double s = 0.0;
                for (int64_t c = 0; c < H; ++c)
                    s += nvfp4_weight(pg, sg, g1, H, j, c) * xt[c];
                a[j] = s;
            }
            for (int64_t j = 0; j < I; ++j)
                hb[j] = oracle_bf16_to_f32(oracle_bf16_round(silu(a[j]) * a[I + j]));
            double wk = w[t * K + k];
            #pragma omp parallel for schedule(static)
            for (int64_t n = 0; n < H; ++n) {
                double s = 0.0;
                for (int64_t c = 0; c < I; ++c)
                    s += nvfp4_weight(pd, sd, g2, I, n, c) * hb[c];
                acc[n] += wk * s;
            }
        }
        for (int64_t c = 0; c < H; ++c) {
            out[i * H + c] = oracle_bf16_round(acc[c]);
            if (out64)
                out64[i * H + c] = acc[c];
        }
    }
    free(xt);
    free(a);
    free(hb);
    free(acc);
    return bad;
}

/* One activation row quantized to NVFP4 as a tensor of its own (its own global scale
 * g = amax(row) / 2688, readings of the codec above) and decoded exactly into v (fp64). */
static void quantize_row_exact(const uint16_t *row, int64_t n, uint8_t *packed, uint8_t *scales,
                               double *v)
{
    float g;
    oracle_nvfp4_quantize(row, 1, 1, n, packed, scales, &g);
    for (int64_t c = 0; c < n; ++c)
        v[c] = nvfp4_weight(packed, scales, (double)g, n, 0, c);
}

/* The routed-expert layer with NVFP4 activations as well as NVFP4 weights ("W4A4"), as a
 * block-scaled FP4 tensor-core GEMM computes it.  Page "GLM-5-NVFP4-MTP", "How to Run",
 * serves the NVFP4 checkpoint with ModelOpt's FP4 quantization and FP4 MoE kernels.  The
 * pages do not say how activations are scaled.  [Reading: each activation row, a token's x
 * for the gate/up projection and a routed pair's bf16 h for the down projection, is
 * quantized with the codec's readings as a tensor of its own, i.e. with a dynamic
 * per-row global scale and per-16 block scales.  Its exact NVFP4 values multiply the exact
 * NVFP4 weights, summed in fp64.  h is rounded to bf16 before it is quantized, as in the
 * W4A16 forward.]  Arguments, shapes, out-of-range ids and return value as
 * oracle_moe_forward. */
int64_t oracle_moe_forward_w4a4(const uint16_t *x, const int32_t *ids, const float *w,
                                int64_t T, int64_t H, int64_t I, int64_t E, int64_t K,
                                const uint8_t *wgu, const uint8_t *sgu, const float *ggu,
                                const uint8_t *wdn, const uint8_t *sdn, const float *gdn,
                                const int64_t *tok, int64_t n_tok, uint16_t *out, double *out64)
{
    (void)T;
    int64_t bad = 0;
    int64_t nmax = H > I ? H : I;
    double *xq = (double *)malloc(sizeof(double) * H);
    double *a = (double *)malloc(sizeof(double) * 2 * I);
    uint16_t *hb = (uint16_t *)malloc(sizeof(uint16_t) * I);
    double *hq = (double *)malloc(sizeof(double) * I);
    double *acc = (double *)malloc(sizeof(double) * H);
    uint8_t *pk = (uint8_t *)malloc((size_t)nmax / 2);
    uint8_t *sc = (uint8_t *)malloc((size_t)nmax / 16);
    for (int64_t i = 0; i < n_tok; ++i) {
        int64_t t = tok[i];
        quantize_row_exact(x + t * H, H, pk, sc, xq);
        for (int64_t c = 0; c < H; ++c) acc[c] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            int64_t e = ids[t * K + k];
            if (e < 0 || e >= E) {
                bad++;
                continue;
            }
            const uint8_t *pg = wgu + e * (2 * I) * (H / 2);
            const uint8_t *sg = sgu + e * (2 * I) * (H / 16);
            const uint8_t *pd = wdn + e * H * (I / 2);
            const uint8_t *sd = sdn + e * H * (I / 16);
            double g1 = ggu[e], g2 = gdn[e];
            #pragma omp parallel for schedule(static)
            for (int64_t j = 0; j < 2 * I; ++j) {
                double s = 0.0;
                for (int64_t c = 0; c < H; ++c)
                    s += nvfp4_weight(pg, sg, g1, H, j, c) * xq[c];
                a[j] = s;
            }
            for (int64_t j = 0; j < I; ++j) hb[j] = oracle_bf16_round(silu(a[j]) * a[I + j]);
            quantize_row_exact(hb, I, pk, sc, hq);
            double wk = w[t * K + k];
            #pragma omp parallel for schedule(static)
            for (int64_t n = 0; n < H; ++n) {
                double s = 0.0;
                for (int64_t c = 0; c < I; ++c)
                    s += nvfp4_weight(pd, sd, g2, I, n, c) * hq[c];
                acc[n] += wk * s;
            }
        }
        for (int64_t c = 0; c < H; ++c) {
            out[i * H + c] = oracle_bf16_round(acc[c]);
            if (out64)
                out64[i * H + c] = acc[c];
        }
    }
    free(xq);
    free(a);
    free(hb);
    free(hq);
    free(acc);
    free(pk);
    free(sc);
    return bad;
}

/* The shared expert: a dense SwiGLU MLP in BF16 that every token passes through, next to
 * the routed experts.  Page "GLM-5-NVFP4-MTP", "What's quantized": only the routed
 * experts' projections are NVFP4 and everything else stays BF16.  A page on the same model
 * family lists the shared experts among its BF16 tensors.  For the tokens tok[0..n_tok):
 *   a   = Wgu x_t                        (2 Is values; rows 0..Is-1 gate, Is..2Is-1 up)
 *   h_j = bf16( silu(a_j) * a_{Is+j} )   (rounded to bf16, as for the routed experts)
 *   y   = Wdn h                          (H values)
 * in fp64 with the bf16 weights exactly.  The layer output is bf16(routed sum + y).
 * [Reading: the shared expert's output is added with weight 1; the pages give no scale.]
 * Shapes: x [T,H] bf16, Wgu [2Is,H] bf16, Wdn [H,Is] bf16; y [n_tok,H] fp64. */
void oracle_shared_expert(const uint16_t *x, int64_t H, int64_t Is, const uint16_t *wgu,
                          const uint16_t *wdn, const int64_t *tok, int64_t n_tok, double *y)
{
    double *xt = (double *)malloc(sizeof(double) * H);
    double *a = (double *)malloc(sizeof(double) * 2 * Is);
    double *hb = (double *)malloc(sizeof(double) * Is);
    for (int64_t i = 0; i < n_tok; ++i) {
        int64_t t = tok[i];
        for (int64_t c = 0; c < H; ++c) xt[c] = oracle_bf16_to_f32(x[t * H + c]);
        #pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < 2 * Is; ++j) {
            double s = 0.0;
            for (int64_t c = 0; c < H; ++c) s += oracle_bf16_to_f32(wgu[j * H + c]) * xt[c];
            a[j] = s;
        }
        for (int64_t j = 0; j < Is; ++j)
            hb[j] = oracle_bf16_to_f32(oracle_bf16_round(silu(a[j]) * a[Is + j]));
        #pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < H; ++n) {
            double s = 0.0;
            for (int64_t c = 0; c < Is; ++c) s += oracle_bf16_to_f32(wdn[n * Is + c]) * hb[c];
            y[i * H + n] = s;
        }
    }
    free(xt);
    free(a);
    free(hb);
}

/* out[i] = bf16(v[i]) for n values (the layer's final rounding of an fp64 sum). */
void oracle_bf16_round_array(const double *v, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_round(v[i]);
}

/* Number of OpenMP threads the oracle's parallel loops use (1 without OpenMP). */
#ifdef _OPENMP
#include <omp.h>
int oracle_threads(void) { return omp_get_max_threads(); }
void oracle_set_threads(int n) { omp_set_num_threads(n); }
#else
int oracle_threads(void) { return 1; }
void oracle_set_threads(int n) { (void)n; }
#endif
