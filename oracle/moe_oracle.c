/*
 * Plain CPU oracle for the routed, weight-quantized Mixture-of-Experts expert layer.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * load this library. The product path never calls it, and it shares no code, header, table or
 * helper with the CUDA library: every number format below is decoded and encoded here from its
 * definition.
 *
 * Precision: weights are dequantized to their exact values and every dot product, the SiLU and
 * the combine run in double. The only roundings are the quantization points the method itself
 * defines (bf16 intermediate for W4A16, E4M3 + f32 scale per 128-group for W8A8), plus the f32
 * rounding of the routing weights, which are f32 values at the library boundary.
 *
 * Sources (web pages), cited by title and section:
 *  [CHORD]  "vLLM x Novita AI: Chord W4A16 INT4 MoE Kernel for Kimi K2.x" (Novita blog).
 *  [SGL]    "SGLang W8A8 Block FP8 quantized kernel config files: analysis and tuning guide"
 *           (xdnf.cn article on SGLang's fp8_kernel.py).
 *  lk_moe   "Lsglang — lk_moe Hybrid Inference for sglang", "Supported models & quant formats"
 *           (MXFP4 and NVFP4 weight formats).
 * Where the pages leave a step open, the reading taken is stated at the step.
 *
 * Parity pins: every exported function is checked, on the CPU, against hand-worked cases, closed
 * forms, invariants, brute force or a library routine (numpy matmul, torch dtype casts) by the
 * oracle tests. The expert-parallel shares are pinned to the whole layer: the full range is the
 * layer bit for bit, and the ranks' shares sum to it. None is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------------ */
/* Number formats                                                                              */
/* ------------------------------------------------------------------------------------------ */

/* bf16 is the upper half of an IEEE binary32: 1 sign, 8 exponent, 7 stored mantissa bits. */
static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 value, ties to even, in ONE rounding (no detour through
 * float, which would round twice). Returns the bit pattern. Values past the largest finite
 * bf16 round to infinity as IEEE round-to-nearest prescribes. */
static uint16_t bf16_round(double v)
{
    if (v != v) return 0x7FC0u;
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (a == 0.0) return sign;
    double q;
    if (a < ldexp(1.0, -126)) {
        /* subnormal bf16: fixed quantum 2^-133 */
        q = nearbyint(a * ldexp(1.0, 133)) * ldexp(1.0, -133);
    } else {
        int ex;
        double m = frexp(a, &ex);               /* a = m * 2^ex, m in [0.5, 1) */
        double r = nearbyint(m * 256.0);        /* 8 significant bits, ties to even */
        q = ldexp(r, ex - 8);
    }
    if (q >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u);
    float f = (float)q;                         /* exact: q has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (uint16_t)((u >> 16) & 0x7FFFu));
}

/* E4M3 "fn" format: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities; S.1111.111 is
 * NaN; largest finite 448 [SGL, "Background": E4M3 has a 4-bit exponent, 3-bit mantissa and a
 * maximum of about 448]. Exponent field 0 holds the subnormals m * 2^-9. */
static double e4m3_value(uint8_t code)
{
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Encode an f32 value as E4M3, nearest with ties to even, saturating to +-448.
 * READING: the pages give no overflow rule; saturation (not NaN) is taken, and with scales
 * amax/448 no in-range input reaches it except through rounding of the quotient. */
static uint8_t e4m3_encode(float x)
{
    uint8_t sign = signbit(x) ? 0x80u : 0u;
    double a = fabs((double)x);
    if (x != x) return 0x7Fu;
    if (a >= 448.0) return (uint8_t)(sign | 0x7Eu);
    if (a < ldexp(1.0, -6)) {
        /* subnormal: step 2^-9; a result of 8 steps is the smallest normal, code 0x08 */
        int r = (int)nearbyint(a * 512.0);
        return (uint8_t)(sign | (uint8_t)r);
    }
    int ex;
    double m = frexp(a, &ex);                   /* a = (2m) * 2^(ex-1), 2m in [1, 2) */
    int e = ex - 1 + 7;
    int r = (int)nearbyint(2.0 * m * 8.0);      /* 8..16 */
    if (r == 16) { r = 8; e += 1; }
    if (e > 15 || (e == 15 && r - 8 == 7)) return (uint8_t)(sign | 0x7Eu);
    return (uint8_t)(sign | (uint8_t)(e << 3) | (uint8_t)(r - 8));
}

/* ------------------------------------------------------------------------------------------ */
/* Step 1: routing                                                                             */
/* ------------------------------------------------------------------------------------------ */

/* Top-k softmax routing, renormalised over the selected experts. The pages only consume the
 * result of routing ([CHORD], "vLLM integration": the indexed path takes the routing buffers);
 * READING: softmax over the E logits, keep the k largest, divide by their sum. Because the full
 * softmax denominator cancels in the renormalisation, w_j = exp(l_j - l_max) / sum over the
 * selected j' of exp(l_j' - l_max). Softmax is monotone, so the selection is by logit.
 * READING: ties go to the lower expert index; slot j holds the j-th selected expert in
 * (logit descending, index ascending) order. */
int orc_route_topk(const float *logits, int T, int E, int k, int32_t *ids, float *w)
{
    if (T < 0 || E < 1 || k < 1 || k > E) return 1;
    char *taken = (char *)malloc((size_t)E);
    if (!taken) return 1;
    for (int t = 0; t < T; ++t) {
        const float *l = logits + (size_t)t * E;
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* strict '>' keeps the lower index on ties */
            }
            taken[best] = 1;
            ids[(size_t)t * k + j] = best;
        }
        double lmax = (double)l[ids[(size_t)t * k]];
        double den = 0.0;
        for (int j = 0; j < k; ++j) den += exp((double)l[ids[(size_t)t * k + j]] - lmax);
        for (int j = 0; j < k; ++j)
            w[(size_t)t * k + j] = (float)(exp((double)l[ids[(size_t)t * k + j]] - lmax) / den);
    }
    free(taken);
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* Step 2: token-to-expert alignment                                                           */
/* ------------------------------------------------------------------------------------------ */

/* moe_align with block size B ([CHORD], "Two kernel families": the indexed path consumes
 * sorted_ids / expert_ids / num_tokens_padded; figure 3, "where padding lives": activations are
 * not padded, the padding guards live in the routing indices; "vLLM integration": the buffers
 * are over-allocated so no host read of the routed count is needed).
 *   flat slot f = t*k + j routes to expert e = ids[f]; c_e = number of slots of e;
 *   P_e = ceil(c_e / B) * B; experts are laid out in ascending e, expert e at offset sum_{e'<e} P_e';
 *   its slots go there in ascending f, the remaining P_e - c_e entries hold the pad value T*k;
 *   expert_ids[b] = expert of block b; num_tokens_padded = sum_e P_e.
 * READINGS: stable (ascending f) order inside an expert; pad value T*k; the buffers have
 * T*k + E*(B-1) entries (the largest possible padded count), entries past num_tokens_padded
 * hold T*k, and block entries past it hold -1. */
int orc_align(const int32_t *ids, int T, int k, int E, int B,
              int32_t *sorted_ids, int32_t *expert_ids, int32_t *num_tokens_padded)
{
    if (T < 0 || k < 1 || E < 1 || B < 1) return 1;
    long n = (long)T * k;
    long cap = n + (long)E * (B - 1);
    long nblk = (cap + B - 1) / B;
    long *cnt = (long *)calloc((size_t)E, sizeof(long));
    if (!cnt) return 1;
    for (long f = 0; f < n; ++f) {
        int e = ids[f];
        if (e < 0 || e >= E) { free(cnt); return 1; }
        cnt[e]++;
    }
    for (long i = 0; i < cap; ++i) sorted_ids[i] = (int32_t)n;
    for (long b = 0; b < nblk; ++b) expert_ids[b] = -1;
    long off = 0;
    for (int e = 0; e < E; ++e) {
        long pos = off;
        for (long f = 0; f < n; ++f)
            if (ids[f] == e) sorted_ids[pos++] = (int32_t)f;
        long padded = (cnt[e] + B - 1) / B * B;
        for (long b = off / B; b < (off + padded) / B; ++b) expert_ids[b] = e;
        off += padded;
    }
    *num_tokens_padded = (int32_t)off;
    free(cnt);
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* Weight formats                                                                              */
/* ------------------------------------------------------------------------------------------ */

/* W4A16 weight element (row r, column c) of a matrix stored as unsigned INT4 codes packed 8 per
 * int32 along the input dimension, with one bf16 scale per 32 consecutive inputs ([CHORD],
 * "vLLM integration": uint4, group 32, BF16 scales, the pack-quantized INT4 group-32 checkpoint
 * shape; "SM90 grouped kernels": codes [G, N, K], scales [G, N, K/32]).
 * READING: nibble j of word w holds column 8w + j in bits [4j, 4j+4); the code carries an
 * implicit zero point of 8, so the value is (q - 8) * scale, exact in double. */
static double w4_value(const int32_t *q, const uint16_t *s, int K, int r, int c)
{
    uint32_t word = (uint32_t)q[(size_t)r * (K / 8) + c / 8];
    int code = (int)((word >> (4 * (c % 8))) & 15u);
    return (double)(code - 8) * bf16_value(s[(size_t)r * (K / 32) + c / 32]);
}

/* E2M1, the 4-bit float of the MXFP4 format (lk_moe page, "Supported models & quant formats"
 * lists MXFP4): 1 sign bit, 2 exponent bits with bias 1, 1 mantissa bit; exponent 0 is the
 * subnormal range (value = mantissa / 2), so the magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
static double e2m1_value(unsigned code)
{
    unsigned e = (code >> 1) & 3u, m = code & 1u;
    double mag = e ? ldexp(1.0 + 0.5 * (double)m, (int)e - 1) : 0.5 * (double)m;
    return (code & 8u) ? -mag : mag;
}

/* MXFP4 weight element: E2M1 code (same packing as the INT4 format: nibble j of int32 word w is
 * input 8w + j) times the power-of-two scale of its 32-input group, a UE8M0 byte s meaning
 * 2^(s - 127). READING: the pages name the format only; this is the OCP microscaling layout with
 * the layer's INT4 nibble order and group-32 scale shape. */
static double fp4_value(const int32_t *q, const uint8_t *s, int K, int r, int c)
{
    uint32_t word = (uint32_t)q[(size_t)r * (K / 8) + c / 8];
    unsigned code = (word >> (4 * (c % 8))) & 15u;
    return e2m1_value(code) * ldexp(1.0, (int)s[(size_t)r * (K / 32) + c / 32] - 127);
}

/* NVFP4 weight element without its tensor scale (lk_moe page, "Supported models & quant
 * formats": NVFP4, compressed-tensors / modelopt): E2M1 code (INT4 nibble order) times the E4M3
 * scale of its 16-input group, scales [rows, K/16] bytes. The per-tensor f32 scale multiplies the
 * whole product and is applied by the caller. READING: the pages name the format only; this is
 * the two-level NVFP4 layout (16-element E4M3 blocks, one f32 scale per weight tensor). */
static double nvfp4_value(const int32_t *q, const uint8_t *s, int K, int r, int c)
{
    uint32_t word = (uint32_t)q[(size_t)r * (K / 8) + c / 8];
    unsigned code = (word >> (4 * (c % 8))) & 15u;
    return e2m1_value(code) * e4m3_value(s[(size_t)r * (K / 16) + c / 16]);
}

/* fmt 0: INT4 (bf16 scales per 32), 1: MXFP4 (UE8M0 scales per 32), 2: NVFP4 (E4M3 per 16) */
static double q4_value(int fmt, const int32_t *q, const void *s, int K, int r, int c)
{
    if (fmt == 2) return nvfp4_value(q, (const uint8_t *)s, K, r, c);
    return fmt ? fp4_value(q, (const uint8_t *)s, K, r, c) : w4_value(q, (const uint16_t *)s, K, r, c);
}

/* ------------------------------------------------------------------------------------------ */
/* FP8 per-token group-128 activation quantization ([SGL], "Background": As is the per
 * token-group quantization scale matrix of the activations; block_size [128, 128]).           */
/* ------------------------------------------------------------------------------------------ */

/* Quantize one group of f32 values: amax = max |v|; scale = max(amax, 1e-10) / 448 in f32;
 * code = E4M3(v / scale) with the f32 quotient.
 * READINGS: the 1e-10 floor for an all-zero group (the pages give none); the scale is kept as
 * an f32 value (not rounded to a power of two). */
static void quant_group_f32(const float *v, int n, uint8_t *q, float *scale)
{
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(v[i]);
        if (a > amax) amax = a;
    }
    float s = (amax > 1e-10f ? amax : 1e-10f) / 448.0f;   /* IEEE f32 division */
    for (int i = 0; i < n; ++i) q[i] = e4m3_encode(v[i] / s);
    *scale = s;
}

/* x: bf16 bits [rows, cols], cols a multiple of 128 -> q [rows, cols], s [rows, cols/128]. */
int orc_fp8_act_quant(const uint16_t *x, int rows, int cols, uint8_t *q, float *s)
{
    if (rows < 0 || cols < 128 || cols % 128) return 1;
    int G = cols / 128;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        float buf[128];
        for (int g = 0; g < G; ++g) {
            for (int i = 0; i < 128; ++i) buf[i] = (float)bf16_value(x[(size_t)r * cols + g * 128 + i]);
            quant_group_f32(buf, 128, q + (size_t)r * cols + g * 128, s + (size_t)r * G + g);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* Steps 3-7: the W4A16 expert layer, for a chosen list of tokens                              */
/* ------------------------------------------------------------------------------------------ */

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* out[i, :] for token tokens[i] (double, [ntok, H]):
 *   route (step 1), then for each selected expert e with weight w:
 *     g_n = sum_c x_c * W13[e][n, c],  u_n = sum_c x_c * W13[e][I + n, c]   (gate rows [0, I),
 *         up rows [I, 2I): READING of the fused gate/up layout, [CHORD] "Kernel optimizations")
 *     h_n = bf16( silu(g_n) * u_n )     (the A16 intermediate: activations are BF16)
 *     y_m = sum_n h_n * W2[e][m, n]
 *   out = sum over the k selected experts of w * y     (the top-k weighted combine).
 * h_out (nullable, bf16 bits [ntok, k, I]) returns the intermediate of each slot.
 * Expert parallelism ([CHORD] "Other deployment details": EP8 / EP16 / EP32, each GPU holding a
 * share of the experts): with the weights of experts [ep_base, ep_base + ep_local) only, the sum
 * above runs over the slots whose expert lies in that range (the routing still ranks all E);
 * ep_base = 0, ep_local = E is the whole layer. Slots outside the range leave h_out untouched. */
static int moe_q4_layer(int fmt, const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                        const int32_t *w13q, const void *w13s, const int32_t *w2q, const void *w2s,
                        const float *g13, const float *g2, const int32_t *tokens, int ntok, double *out,
                        uint16_t *h_out, int ep_base, int ep_local)
{
    const size_t sb = fmt ? 1 : 2;        /* bytes per scale */
    const int gsz = fmt == 2 ? 16 : 32;   /* inputs per scale */
    if (H % 32 || I % 32 || H < 32 || I < 32 || k < 1 || k > E) return 1;
    if (ep_base < 0 || ep_local < 1 || ep_base + ep_local > E) return 1;
    for (int i = 0; i < ntok; ++i)
        if (tokens[i] < 0 || tokens[i] >= T) return 1;
    int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
    float *w = (float *)malloc(sizeof(float) * (size_t)k);
    double *xd = (double *)malloc(sizeof(double) * (size_t)H);
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    if (!ids || !w || !xd || !h) return 1;
    for (int i = 0; i < ntok; ++i) {
        int t = tokens[i];
        orc_route_topk(logits + (size_t)t * E, 1, E, k, ids, w);
        for (int c = 0; c < H; ++c) xd[c] = bf16_value(x[(size_t)t * H + c]);
        double *o = out + (size_t)i * H;
        for (int m = 0; m < H; ++m) o[m] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = ids[j] - ep_base;            /* index among the weights held */
            if (e < 0 || e >= ep_local) continue;
            const int32_t *q13 = w13q + (size_t)e * 2 * I * (H / 8);
            const void *s13 = (const char *)w13s + (size_t)e * 2 * I * (H / gsz) * sb;
            const int32_t *q2 = w2q + (size_t)e * H * (I / 8);
            const void *s2 = (const char *)w2s + (size_t)e * H * (I / gsz) * sb;
            const double ts13 = g13 ? (double)g13[e] : 1.0, ts2 = g2 ? (double)g2[e] : 1.0;
#pragma omp parallel for schedule(static)
            for (int n = 0; n < I; ++n) {
                double g = 0.0, u = 0.0;
                for (int c = 0; c < H; ++c) {
                    g += xd[c] * q4_value(fmt, q13, s13, H, n, c);
                    u += xd[c] * q4_value(fmt, q13, s13, H, I + n, c);
                }
                g *= ts13;
                u *= ts13;
                uint16_t hb = bf16_round(silu(g) * u);
                h[n] = bf16_value(hb);
                if (h_out) h_out[((size_t)i * k + j) * I + n] = hb;
            }
            double wj = (double)w[j];
#pragma omp parallel for schedule(static)
            for (int m = 0; m < H; ++m) {
                double y = 0.0;
                for (int n = 0; n < I; ++n) y += h[n] * q4_value(fmt, q2, s2, I, m, n);
                o[m] += wj * ts2 * y;
            }
        }
    }
    free(ids); free(w); free(xd); free(h);
    return 0;
}

int orc_moe_w4a16(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                  const int32_t *w13q, const uint16_t *w13s, const int32_t *w2q, const uint16_t *w2s,
                  const int32_t *tokens, int ntok, double *out, uint16_t *h_out)
{
    return moe_q4_layer(0, x, logits, T, H, I, E, k, w13q, w13s, w2q, w2s, NULL, NULL, tokens, ntok, out, h_out, 0, E);
}

/* One expert-parallel rank's share of the 4-bit layer (fmt 0 INT4, 1 MXFP4, 2 NVFP4; scales as the
 * single-format functions take them, g13 / g2 NULL except for NVFP4), weights of experts
 * [ep_base, ep_base + ep_local) only. */
int orc_moe_q4_ep(int fmt, const uint16_t *x, const float *logits, int T, int H, int I, int E, int k, int ep_base,
                  int ep_local, const int32_t *w13q, const void *w13s, const float *g13, const int32_t *w2q,
                  const void *w2s, const float *g2, const int32_t *tokens, int ntok, double *out)
{
    if (fmt < 0 || fmt > 2 || (fmt == 2 && (!g13 || !g2))) return 1;
    return moe_q4_layer(fmt, x, logits, T, H, I, E, k, w13q, w13s, w2q, w2s, fmt == 2 ? g13 : NULL,
                        fmt == 2 ? g2 : NULL, tokens, ntok, out, NULL, ep_base, ep_local);
}

/* The same layer with MXFP4 weights (E2M1 codes, UE8M0 group-32 scales [rows, K/32] bytes); the
 * activations stay bf16 and the intermediate is rounded to bf16 as in the W4A16 layer. */
int orc_moe_mxfp4(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                  const int32_t *w13q, const uint8_t *w13s, const int32_t *w2q, const uint8_t *w2s,
                  const int32_t *tokens, int ntok, double *out, uint16_t *h_out)
{
    return moe_q4_layer(1, x, logits, T, H, I, E, k, w13q, w13s, w2q, w2s, NULL, NULL, tokens, ntok, out, h_out, 0, E);
}

/* The same layer with NVFP4 weights: E2M1 codes, E4M3 group-16 scales [rows, K/16] bytes and one
 * f32 tensor scale per expert and matrix (g13 [E] for the fused gate/up, g2 [E] for down):
 * W = E2M1(q) * E4M3(s) * g. READING: one tensor scale for the fused gate/up matrix. */
int orc_moe_nvfp4(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                  const int32_t *w13q, const uint8_t *w13s, const float *g13, const int32_t *w2q,
                  const uint8_t *w2s, const float *g2, const int32_t *tokens, int ntok, double *out,
                  uint16_t *h_out)
{
    if (H % 32 || I % 32) return 1;
    return moe_q4_layer(2, x, logits, T, H, I, E, k, w13q, w13s, w2q, w2s, g13, g2, tokens, ntok, out, h_out, 0, E);
}

/* ------------------------------------------------------------------------------------------ */
/* The W8A8 block-FP8 expert layer, for a chosen list of tokens                                */
/* ------------------------------------------------------------------------------------------ */

/* Decoded E4M3 values, filled from e4m3_value() before any parallel region (a cache of the
 * decoder above, so the inner loops do not call ldexp). */
static double e4m3_table[256];
static int e4m3_table_ready = 0;

static void e4m3_table_init(void)
{
    if (e4m3_table_ready) return;
    for (int c = 0; c < 256; ++c) e4m3_table[c] = e4m3_value((uint8_t)c);
    e4m3_table_ready = 1;
}

/* Block-scaled dot product of one activation row and one weight row over K ([SGL],
 * "Background": each [BLOCK_N, BLOCK_K] = [128, 128] weight block has its own scale, the
 * activations one scale per token and 128-column group):
 *   sum_kb  a_s[kb] * b_s[kb] * sum_{c in block kb} E4M3(a_c) * E4M3(b_c)                     */
static double fp8_row_dot(const uint8_t *a, const float *as, const uint8_t *b, const float *bs, int K)
{
    double acc = 0.0;
    for (int kb = 0; kb < K / 128; ++kb) {
        double part = 0.0;
        for (int c = kb * 128; c < kb * 128 + 128; ++c) part += e4m3_table[a[c]] * e4m3_table[b[c]];
        acc += (double)as[kb] * (double)bs[kb] * part;
    }
    return acc;
}

/* As orc_moe_w4a16 with E4M3 weights W13[e] [2I, H] (scales [2I/128, H/128]) and W2[e] [H, I]
 * (scales [H/128, I/128]); the input is quantized per token and 128-group (orc_fp8_act_quant),
 * and the intermediate a = silu(g)*u is rounded to f32 and quantized the same way before the
 * down projection. READING: the intermediate quantizer sees the f32 value of a, as the input
 * quantizer sees the f32 value of the bf16 input.
 * hq_out/hs_out (nullable) return the quantized intermediate [ntok, k, I] / [ntok, k, I/128].
 * ep_base / ep_local: the expert range whose weights are given, as in moe_q4_layer. */
static int moe_fp8_layer(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                         const uint8_t *w13, const float *w13s, const uint8_t *w2, const float *w2s,
                         const int32_t *tokens, int ntok, double *out, uint8_t *hq_out, float *hs_out,
                         int ep_base, int ep_local)
{
    if (H % 128 || I % 128 || H < 128 || I < 128 || k < 1 || k > E) return 1;
    if (ep_base < 0 || ep_local < 1 || ep_base + ep_local > E) return 1;
    for (int i = 0; i < ntok; ++i)
        if (tokens[i] < 0 || tokens[i] >= T) return 1;
    e4m3_table_init();
    int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
    float *w = (float *)malloc(sizeof(float) * (size_t)k);
    uint8_t *xq = (uint8_t *)malloc((size_t)H);
    float *xs = (float *)malloc(sizeof(float) * (size_t)(H / 128));
    float *a = (float *)malloc(sizeof(float) * (size_t)I);
    uint8_t *hq = (uint8_t *)malloc((size_t)I);
    float *hs = (float *)malloc(sizeof(float) * (size_t)(I / 128));
    if (!ids || !w || !xq || !xs || !a || !hq || !hs) return 1;
    for (int i = 0; i < ntok; ++i) {
        int t = tokens[i];
        orc_route_topk(logits + (size_t)t * E, 1, E, k, ids, w);
        orc_fp8_act_quant(x + (size_t)t * H, 1, H, xq, xs);
        double *o = out + (size_t)i * H;
        for (int m = 0; m < H; ++m) o[m] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = ids[j] - ep_base;            /* index among the weights held */
            if (e < 0 || e >= ep_local) continue;
            const uint8_t *W13 = w13 + (size_t)e * 2 * I * H;
            const float *S13 = w13s + (size_t)e * (2 * I / 128) * (H / 128);
            const uint8_t *W2 = w2 + (size_t)e * H * I;
            const float *S2 = w2s + (size_t)e * (H / 128) * (I / 128);
#pragma omp parallel for schedule(static)
            for (int n = 0; n < I; ++n) {
                double g = fp8_row_dot(xq, xs, W13 + (size_t)n * H, S13 + (size_t)(n / 128) * (H / 128), H);
                double u = fp8_row_dot(xq, xs, W13 + (size_t)(I + n) * H,
                                       S13 + (size_t)((I + n) / 128) * (H / 128), H);
                a[n] = (float)(silu(g) * u);
            }
            for (int gI = 0; gI < I / 128; ++gI) quant_group_f32(a + gI * 128, 128, hq + gI * 128, hs + gI);
            if (hq_out) memcpy(hq_out + ((size_t)i * k + j) * I, hq, (size_t)I);
            if (hs_out) memcpy(hs_out + ((size_t)i * k + j) * (I / 128), hs, sizeof(float) * (size_t)(I / 128));
            double wj = (double)w[j];
#pragma omp parallel for schedule(static)
            for (int m = 0; m < H; ++m)
                o[m] += wj * fp8_row_dot(hq, hs, W2 + (size_t)m * I, S2 + (size_t)(m / 128) * (I / 128), I);
        }
    }
    free(ids); free(w); free(xq); free(xs); free(a); free(hq); free(hs);
    return 0;
}

int orc_moe_fp8(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                const uint8_t *w13, const float *w13s, const uint8_t *w2, const float *w2s,
                const int32_t *tokens, int ntok, double *out, uint8_t *hq_out, float *hs_out)
{
    return moe_fp8_layer(x, logits, T, H, I, E, k, w13, w13s, w2, w2s, tokens, ntok, out, hq_out, hs_out, 0, E);
}

/* One expert-parallel rank's share of the block-FP8 layer (weights of [ep_base, ep_base + ep_local)). */
int orc_moe_fp8_ep(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k, int ep_base,
                   int ep_local, const uint8_t *w13, const float *w13s, const uint8_t *w2, const float *w2s,
                   const int32_t *tokens, int ntok, double *out)
{
    return moe_fp8_layer(x, logits, T, H, I, E, k, w13, w13s, w2, w2s, tokens, ntok, out, NULL, NULL, ep_base,
                         ep_local);
}

/* ------------------------------------------------------------------------------------------ */
/* Dense block-FP8 matmul ([SGL], "Background": w8a8_block_fp8_matmul(A, B, As, Bs, block_size,
 * output_dtype), A the activations [M, K], B the weights [N, K], As [M, K/128], Bs
 * [ceil(N/128), ceil(K/128)]):  C[m, n] = sum_kb As[m, kb] * Bs[n/128, kb] * sum A*B.        */
/* ------------------------------------------------------------------------------------------ */

int orc_fp8_block_matmul(const uint8_t *A, const float *As, const uint8_t *B, const float *Bs,
                         int M, int N, int K, const int32_t *rows, int nrows, double *C)
{
    if (K % 128 || K < 128 || N < 1) return 1;
    for (int i = 0; i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= M) return 1;
    int KB = K / 128;
    e4m3_table_init();
#pragma omp parallel for collapse(2) schedule(static)
    for (int i = 0; i < nrows; ++i)
        for (int n = 0; n < N; ++n) {
            int m = rows[i];
            C[(size_t)i * N + n] = fp8_row_dot(A + (size_t)m * K, As + (size_t)m * KB,
                                               B + (size_t)n * K, Bs + (size_t)(n / 128) * KB, K);
        }
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* Dense channelwise FP8 matmul ([SGL], "JSON format": the channelwise variant is the W8A8 FP8
 * GEMM with one scale per token of the activations and one per channel (output row) of the
 * weights). READING: the pages name the scaling granularity and no formula; the plain reading is
 *   C[m, n] = As[m] * Bs[n] * sum_c E4M3(A[m, c]) * E4M3(B[n, c])
 * with A [M, K], As [M], B [N, K], Bs [N], in double.                                         */
/* ------------------------------------------------------------------------------------------ */

int orc_fp8_channel_matmul(const uint8_t *A, const float *As, const uint8_t *B, const float *Bs,
                           int M, int N, int K, const int32_t *rows, int nrows, double *C)
{
    if (K < 1 || N < 1) return 1;
    for (int i = 0; i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= M) return 1;
    e4m3_table_init();
#pragma omp parallel for collapse(2) schedule(static)
    for (int i = 0; i < nrows; ++i)
        for (int n = 0; n < N; ++n) {
            int m = rows[i];
            const uint8_t *a = A + (size_t)m * K;
            const uint8_t *b = B + (size_t)n * K;
            double dot = 0.0;
            for (int c = 0; c < K; ++c) dot += e4m3_table[a[c]] * e4m3_table[b[c]];
            C[(size_t)i * N + n] = (double)As[m] * (double)Bs[n] * dot;
        }
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* Grouped W4A16 GEMM ([CHORD], "SM90 grouped kernels": the contiguous layout concatenates the
 * rows of each expert, padded to 128-row boundaries, with m_indices holding each row's expert
 * and -1 on padding; the masked layout gives every expert a fixed budget of max_m rows of which
 * masked_m are real, and consumers ignore the rest). Both are, per real row m with expert e:
 *   C[m, n] = sum_c A[m, c] * ((q[e, n, c] - 8) * s[e, n, c / 32])
 * READING: the pages print no formula; this is the plain product of the activation row with the
 * dequantized weights of its expert, A taken as exact bf16 values, in double. The expert of a
 * row is given per row (expert_of_row, -1 = not computed), which covers both layouts.         */
/* ------------------------------------------------------------------------------------------ */

int orc_grouped_w4a16(const uint16_t *A, int M, int K, const int32_t *wq, const uint16_t *ws, int G, int N,
                      const int32_t *expert_of_row, const int32_t *rows, int nrows, double *C)
{
    if (K % 32 || K < 32 || N < 1 || G < 1) return 1;
    for (int i = 0; i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= M) return 1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int i = 0; i < nrows; ++i)
        for (int n = 0; n < N; ++n) {
            int m = rows[i];
            int e = expert_of_row[m];
            double acc = 0.0;
            if (e >= 0 && e < G) {
                const int32_t *q = wq + (size_t)e * N * (K / 8);
                const uint16_t *sc = ws + (size_t)e * N * (K / 32);
                for (int c = 0; c < K; ++c) acc += bf16_value(A[(size_t)m * K + c]) * w4_value(q, sc, K, n, c);
            }
            C[(size_t)i * N + n] = acc;
        }
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* Format primitives exported for the pins                                                     */
/* ------------------------------------------------------------------------------------------ */

void orc_bf16_round(const double *in, uint16_t *out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = bf16_round(in[i]);
}

void orc_bf16_value(const uint16_t *in, double *out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = bf16_value(in[i]);
}

void orc_e4m3_encode(const float *in, uint8_t *out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = e4m3_encode(in[i]);
}

void orc_e4m3_value(const uint8_t *in, double *out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = e4m3_value(in[i]);
}

/* Dequantized W4A16 matrix [N, K] as doubles (used by the pins that reduce to numpy matmul). */
int orc_w4a16_dequant(const int32_t *q, const uint16_t *s, int N, int K, double *out)
{
    if (K % 32 || K < 32) return 1;
    for (int r = 0; r < N; ++r)
        for (int c = 0; c < K; ++c) out[(size_t)r * K + c] = w4_value(q, s, K, r, c);
    return 0;
}

int orc_nvfp4_dequant(const int32_t *q, const uint8_t *s, float g, int N, int K, double *out)
{
    if (K % 32 || K < 32) return 1;
    for (int r = 0; r < N; ++r)
        for (int c = 0; c < K; ++c) out[(size_t)r * K + c] = nvfp4_value(q, s, K, r, c) * (double)g;
    return 0;
}

int orc_mxfp4_dequant(const int32_t *q, const uint8_t *s, int N, int K, double *out)
{
    if (K % 32 || K < 32) return 1;
    for (int r = 0; r < N; ++r)
        for (int c = 0; c < K; ++c) out[(size_t)r * K + c] = fp4_value(q, s, K, r, c);
    return 0;
}

void orc_e2m1_value(const uint8_t *in, double *out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = e2m1_value(in[i] & 15u);
}
