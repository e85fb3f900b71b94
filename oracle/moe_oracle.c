/*
 * moe_oracle.c — plain, slow CPU oracle for the packed-MXFP4 W4A16 top-4
 * MoE expert FFN.  TEST INFRASTRUCTURE ONLY: it is called by tests/, by
 * __graft_entry__.smoke() and by bench.py's CPU-baseline leg, never by the
 * product path.  It shares no code, header, table or helper with the CUDA
 * library.
 *
 * Everything is computed in IEEE double precision with the BF16 rounding
 * points of the definition; each BF16 rounding is ONE rounding (round to
 * nearest, ties to even) of the exact double value, never a double rounding
 * through float.
 *
 * Sources (page title, section):
 *   [MC]  "LFM2.5-24B-A2B — Packed MXFP4 Inference" (model card of the
 *         packed MXFP4 checkpoint): table "Model and quantization" (E2M1 FP4
 *         weights, two per byte, one E8M0 scale per 32 values, BF16
 *         activations, FP32 accumulation with BF16 outputs, top-4 of 64
 *         experts); section "What was optimized" > "Grouped top-4 expert
 *         execution" (gate GEMV, up GEMV, activation and multiplication,
 *         down GEMV, routing-weighted combination that keeps the serial
 *         runner's sequential BF16 multiply/add rounding); section "GPU
 *         routing inside resident-layer graphs" (router projection, sigmoid
 *         scores, expert bias where configured, dynamic top-k, routing
 *         coefficients).
 *   [NV]  "primitive-ai/LFM2.5-24B-A2B-NVFP4A16" (model card of an NVFP4
 *         weight-only build): sections "What's quantized to what" (routed
 *         experts in NVFP4, compute in 16-bit; format nvfp4-pack-quantized;
 *         w1 and w3 of each expert share one global scale).
 *   [CA]  "LFM2.5-8B-A1B — Core AI (.aimodel)": table "Provenance", row
 *         "Weight format" (sym8: symmetric-linear int8 with one scale per
 *         block of 32 along K, read through a gather matvec kernel).
 *   [BW]  "LFM2.5-24B-A2B on Your Own Hardware: The RAM, KV Cache and
 *         Bandwidth Budget": section "Where do the 2.45B active parameters
 *         actually go?" (SwiGLU expert = gate, up, down; H=2048, I=1536).
 *
 * Readings of points the pages leave open:
 *   - E2M1 code c: sign = bit 3, magnitude = {0,0.5,1,1.5,2,3,4,6}[c & 7].
 *   - Nibble order: element 2i is the low nibble of byte i.
 *   - E8M0 e: 2^(e-127); e = 255 is NaN.
 *   - Layout: codes [E][3][rows][K/2] (gate I x H, up I x H, down H x I),
 *     scales [E][3][rows][K/32].
 *   - Router: logits = x . Wr^T (+ bias[e] if given), not rounded; top-k by
 *     logit, descending, ties to the lower expert id; coefficients =
 *     softmax over the k selected logits.
 *   - Sigmoid router (the page's own listing of the routing steps, in its
 *     order): logits l = x . Wr^T (no bias), scores s = 1 / (1 + e^-l), the
 *     expert bias added to the scores for the selection only, top-k of
 *     s + bias (ties to the lower id), coefficients = the selected s
 *     divided by their sum.
 *   - FFN rounding points: g, u -> BF16; s = BF16(silu(g)); h = BF16(s*u);
 *     o = BF16(Wd . h).
 *   - Combine: wb = BF16(w_j); p_j = BF16(o_j * wb_j); y starts at +0 and
 *     y = BF16(y + p_j) for j = 0..k-1 in slot order.
 *   - Stack: xn = BF16(r / sqrt(mean(r^2) + 1e-6)) (weightless RMSNorm
 *     before each layer), r' = BF16(r + y).
 *   - NVFP4 ([NV] names the format only): E2M1 codes packed as above; one
 *     FP8 E4M3 scale per 16 consecutive K elements (scales [E][3][rows][K/16]:
 *     sign, 4 exponent bits with bias 7, 3 mantissa bits, exponent 0
 *     subnormal, S.1111.111 NaN, no infinity); one FP32 multiplier per
 *     expert shared by gate and up and one for down (gscales [E][2]);
 *     w = e2m1(c) * e4m3(s) * g.
 *   - sym8 ([CA] names the format only): one two's-complement int8 q per
 *     weight (codes [E][3][rows][K], one byte each), one IEEE binary16
 *     scale per 32 consecutive K elements (scales [E][3][rows][K/32] as
 *     little-endian 16-bit words); symmetric, so no zero point: w = q * s.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- BF16 -- */

double oracle_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* One RNE rounding of a double to BF16 (8 significant bits, exponent range
 * of binary32, subnormals down to 2^-133, overflow to infinity). */
uint16_t oracle_bf16_from_double(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    if (isnan(v))
        return (uint16_t)(sign | 0x7FC0u);
    double a = fabs(v);
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0)
        return sign;
    int e2;
    frexp(a, &e2);                 /* a in [2^(e2-1), 2^e2) */
    int ebin = e2 - 1;             /* a in [2^ebin, 2^(ebin+1)) */
    int q = (ebin < -126) ? -133 : ebin - 7;   /* exponent of one ulp */
    double units = nearbyint(ldexp(a, -q));    /* ties to even (FE_TONEAREST) */
    double r = ldexp(units, q);
    if (r >= ldexp(1.0, 128))
        return (uint16_t)(sign | 0x7F80u);
    float f = (float)r;            /* exact: <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (uint16_t)(u >> 16));
}

/* ------------------------------------------------------- MXFP4 decode -- */

/* [MC] "Model and quantization": weight values are packed E2M1 FP4.
 * The 16 codes: bit 3 is the sign, bits 0..2 index the magnitudes. */
static const double E2M1_MAGNITUDE[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_value(unsigned code)
{
    double m = E2M1_MAGNITUDE[code & 7u];
    return (code & 8u) ? -m : m;
}

/* [MC] "Model and quantization": E8M0 scale, one per 32 weight values. */
double oracle_e8m0_value(unsigned e)
{
    if (e == 255u)
        return NAN;
    return ldexp(1.0, (int)e - 127);
}

/* Weight element j of a packed row: nibble j of the codes (low nibble first)
 * times the E8M0 scale of its 32-element group. */
static double weight_at(const uint8_t *row_codes, const uint8_t *row_scales,
                        int64_t j)
{
    uint8_t byte = row_codes[j >> 1];
    unsigned nib = (j & 1) ? (unsigned)(byte >> 4) : (unsigned)(byte & 0x0F);
    return oracle_e2m1_value(nib) * oracle_e8m0_value(row_scales[j >> 5]);
}

/* [NV] FP8 E4M3 block scale, one per 16 weight values. */
double oracle_e4m3_value(unsigned b)
{
    unsigned sign = (b >> 7) & 1u, ex = (b >> 3) & 15u, man = b & 7u;
    double m;
    if (ex == 15u && man == 7u)
        return NAN;
    if (ex == 0u)
        m = ldexp((double)man / 8.0, -6);          /* subnormal */
    else
        m = ldexp(1.0 + (double)man / 8.0, (int)ex - 7);
    return sign ? -m : m;
}

/* NVFP4 weight element j of a packed row: the E2M1 code times the E4M3
 * scale of its 16-element block times the tensor's global multiplier. */
static double weight_at_nv(const uint8_t *row_codes, const uint8_t *row_scales,
                           double gscale, int64_t j)
{
    uint8_t byte = row_codes[j >> 1];
    unsigned nib = (j & 1) ? (unsigned)(byte >> 4) : (unsigned)(byte & 0x0F);
    return oracle_e2m1_value(nib) * oracle_e4m3_value(row_scales[j >> 4]) * gscale;
}

/* IEEE 754 binary16 value of the 16-bit pattern b (the sym8 block scale):
 * sign, 5 exponent bits with bias 15, 10 mantissa bits, exponent 0
 * subnormal, exponent 31 infinity or NaN. */
double oracle_f16_value(unsigned b)
{
    unsigned sign = (b >> 15) & 1u, ex = (b >> 10) & 31u, man = b & 1023u;
    double m;
    if (ex == 31u)
        m = man ? NAN : INFINITY;
    else if (ex == 0u)
        m = ldexp((double)man, -24);               /* subnormal */
    else
        m = ldexp(1.0 + (double)man / 1024.0, (int)ex - 15);
    return sign ? -m : m;
}

/* [CA] sym8 weight element j of a row: the signed byte q_j times the
 * binary16 scale of its 32-element block (no zero point). */
static double weight_at_s8(const uint8_t *row_q, const uint8_t *row_scales, int64_t j)
{
    int q = (int)(int8_t)row_q[j];
    const uint8_t *s = row_scales + 2 * (j >> 5);
    return (double)q * oracle_f16_value((unsigned)s[0] | ((unsigned)s[1] << 8));
}

/* sym8 dequantisation of n consecutive elements (n a multiple of 32);
 * scales: the little-endian binary16 words as bytes. */
void oracle_dequant_sym8(const uint8_t *q, const uint8_t *scales, int64_t n, double *out)
{
    for (int64_t j = 0; j < n; ++j)
        out[j] = weight_at_s8(q, scales, j);
}

/* NVFP4 dequantisation of n consecutive elements (n a multiple of 16). */
void oracle_dequant_nvfp4(const uint8_t *codes, const uint8_t *scales,
                          double gscale, int64_t n, double *out)
{
    for (int64_t j = 0; j < n; ++j)
        out[j] = weight_at_nv(codes, scales, gscale, j);
}

/* Dequantise n consecutive elements (n a multiple of 32). */
void oracle_dequant(const uint8_t *codes, const uint8_t *scales, int64_t n,
                    double *out)
{
    for (int64_t j = 0; j < n; ++j)
        out[j] = weight_at(codes, scales, j);
}

/* Same, each value rounded to binary32 (it is exact unless it overflows). */
void oracle_dequant_f32(const uint8_t *codes, const uint8_t *scales, int64_t n,
                        float *out)
{
    for (int64_t j = 0; j < n; ++j)
        out[j] = (float)weight_at(codes, scales, j);
}

/* ------------------------------------------------------------- router -- */

/* Top-k of one token's logits: repeated arg-max over the experts not yet
 * chosen, scanning ids upward with a strict '>' so that equal logits go to
 * the lower id; coefficients = softmax over the k chosen logits.
 * [MC] "GPU routing inside resident-layer graphs": dynamic top-k selection,
 * routing coefficients. */
void oracle_select_topk(const double *logits, int E, int k, int32_t *ids,
                        double *w)
{
    char *taken = (char *)calloc((size_t)E, 1);
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e])
                continue;
            if (best < 0 || logits[e] > logits[best])
                best = e;
        }
        taken[best] = 1;
        ids[j] = best;
    }
    free(taken);
    double lmax = logits[ids[0]];
    double z = 0.0;
    for (int j = 0; j < k; ++j) {
        w[j] = exp(logits[ids[j]] - lmax);
        z += w[j];
    }
    for (int j = 0; j < k; ++j)
        w[j] /= z;
}

/* Sigmoid scoring of one token's unbiased logits: scores s_e = 1/(1+e^-l_e);
 * selection key s_e + bias[e] (bias may be NULL); top-k of the keys by
 * repeated arg-max with a strict '>' scanning ids upward (ties to the lower
 * id); coefficients w_j = s_j / (s_0 + ... + s_{k-1}) of the selected.
 * [MC] "GPU routing inside resident-layer graphs": sigmoid scores, expert
 * bias where configured, dynamic top-k selection, routing coefficients. */
void oracle_select_topk_sigmoid(const double *logits, const float *bias, int E,
                                int k, int32_t *ids, double *w)
{
    double *s = (double *)malloc(sizeof(double) * (size_t)E);
    double *key = (double *)malloc(sizeof(double) * (size_t)E);
    char *taken = (char *)calloc((size_t)E, 1);
    for (int e = 0; e < E; ++e) {
        s[e] = 1.0 / (1.0 + exp(-logits[e]));
        key[e] = s[e] + (bias ? (double)bias[e] : 0.0);
    }
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e])
                continue;
            if (best < 0 || key[e] > key[best])
                best = e;
        }
        taken[best] = 1;
        ids[j] = best;
    }
    double z = 0.0;
    for (int j = 0; j < k; ++j)
        z += s[ids[j]];
    for (int j = 0; j < k; ++j)
        w[j] = s[ids[j]] / z;
    free(taken);
    free(key);
    free(s);
}

/* Router projection for T tokens: logits[t][e] = sum_h x[t][h] * Wr[e][h]
 * (+ bias[e] when bias != NULL), then top-k + softmax.
 * [MC] "GPU routing inside resident-layer graphs": router projection, expert
 * bias where configured. */
void oracle_route(const uint16_t *x, int T, int H, const uint16_t *Wr, int E,
                  const float *bias, int k, int32_t *ids, double *w,
                  double *logits_out)
{
    double *lg = (double *)malloc(sizeof(double) * (size_t)E);
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int h = 0; h < H; ++h)
                s += oracle_bf16_to_double(x[(size_t)t * H + h]) *
                     oracle_bf16_to_double(Wr[(size_t)e * H + h]);
            if (bias)
                s += (double)bias[e];
            lg[e] = s;
            if (logits_out)
                logits_out[(size_t)t * E + e] = s;
        }
        oracle_select_topk(lg, E, k, ids + (size_t)t * k, w + (size_t)t * k);
    }
    free(lg);
}

/* As oracle_route with sigmoid scoring: the logits stay unbiased (they are
 * what logits_out receives) and the bias enters the selection key only. */
void oracle_route_sigmoid(const uint16_t *x, int T, int H, const uint16_t *Wr,
                          int E, const float *bias, int k, int32_t *ids,
                          double *w, double *logits_out)
{
    double *lg = (double *)malloc(sizeof(double) * (size_t)E);
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int h = 0; h < H; ++h)
                s += oracle_bf16_to_double(x[(size_t)t * H + h]) *
                     oracle_bf16_to_double(Wr[(size_t)e * H + h]);
            lg[e] = s;
            if (logits_out)
                logits_out[(size_t)t * E + e] = s;
        }
        oracle_select_topk_sigmoid(lg, bias, E, k, ids + (size_t)t * k,
                                   w + (size_t)t * k);
    }
    free(lg);
}

/* ---------------------------------------------------------- expert FFN -- */

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* Weight formats of the expert matrices. */
enum { FMT_MXFP4 = 0, FMT_NVFP4 = 1, FMT_SYM8 = 2 };

/* Bytes of one row of K weights: codes, and block scales. */
static size_t row_code_bytes(int fmt, int K) { return fmt == FMT_SYM8 ? (size_t)K : (size_t)K / 2; }
static size_t row_scale_bytes(int fmt, int K)
{
    return fmt == FMT_NVFP4 ? (size_t)K / 16 : fmt == FMT_SYM8 ? (size_t)K / 16 : (size_t)K / 32;
}

/* Weight element j of a row in format fmt (g: the NVFP4 multiplier). */
static double weight_fmt(int fmt, const uint8_t *rc, const uint8_t *rs, double g, int64_t j)
{
    if (fmt == FMT_NVFP4)
        return weight_at_nv(rc, rs, g, j);
    if (fmt == FMT_SYM8)
        return weight_at_s8(rc, rs, j);
    return weight_at(rc, rs, j);
}

/* One SwiGLU expert on one BF16 activation vector, for any weight format.
 * [MC] "Grouped top-4 expert execution": gate projection, up projection,
 * activation and multiplication, down projection; "Model and quantization":
 * accumulation wider than BF16, BF16 outputs.  [BW]: the expert is the three
 * matrices gate, up (I x H) and down (H x I).
 *   FMT_MXFP4: codes_e / scales_e: this expert's [3][rows][K/2] /
 *     [3][rows][K/32], gs ignored.
 *   FMT_NVFP4: scales_e [3][rows][K/16] E4M3, gs[0] multiplies gate and up,
 *     gs[1] down.
 *   FMT_SYM8: codes_e [3][rows][K] int8, scales_e [3][rows][K/32] binary16
 *     (2 bytes each), gs ignored.
 *   h_out (nullable): the BF16 SwiGLU output [I].  o_out: BF16 [H]. */
static void expert_any(const uint16_t *x, const uint8_t *codes_e,
                       const uint8_t *scales_e, const float *gs, int fmt,
                       int H, int I, uint16_t *h_out, uint16_t *o_out)
{
    const int nv = fmt == FMT_NVFP4;
    const size_t rcH = row_code_bytes(fmt, H), rsH = row_scale_bytes(fmt, H);
    const size_t rcI = row_code_bytes(fmt, I), rsI = row_scale_bytes(fmt, I);
    const size_t mc = (size_t)I * rcH, ms = (size_t)I * rsH;  /* one matrix */
    const uint8_t *gate_c = codes_e, *up_c = codes_e + mc, *down_c = codes_e + 2 * mc;
    const uint8_t *gate_s = scales_e, *up_s = scales_e + ms, *down_s = scales_e + 2 * ms;
    const double g_gu = nv ? (double)gs[0] : 1.0, g_dn = nv ? (double)gs[1] : 1.0;
    uint16_t *hb = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)I);

#pragma omp parallel for schedule(static)
    for (int i = 0; i < I; ++i) {
        const uint8_t *gc = gate_c + (size_t)i * rcH, *gsc = gate_s + (size_t)i * rsH;
        const uint8_t *uc = up_c + (size_t)i * rcH, *usc = up_s + (size_t)i * rsH;
        double g = 0.0, u = 0.0;
        for (int j = 0; j < H; ++j) {
            double xv = oracle_bf16_to_double(x[j]);
            g += weight_fmt(fmt, gc, gsc, g_gu, j) * xv;
            u += weight_fmt(fmt, uc, usc, g_gu, j) * xv;
        }
        double gb = oracle_bf16_to_double(oracle_bf16_from_double(g));
        double ub = oracle_bf16_to_double(oracle_bf16_from_double(u));
        double sb = oracle_bf16_to_double(oracle_bf16_from_double(silu(gb)));
        hb[i] = oracle_bf16_from_double(sb * ub);
    }

#pragma omp parallel for schedule(static)
    for (int n = 0; n < H; ++n) {
        const uint8_t *dc = down_c + (size_t)n * rcI, *ds = down_s + (size_t)n * rsI;
        double o = 0.0;
        for (int j = 0; j < I; ++j) {
            double wv = weight_fmt(fmt, dc, ds, g_dn, j);
            o += wv * oracle_bf16_to_double(hb[j]);
        }
        o_out[n] = oracle_bf16_from_double(o);
    }
    if (h_out)
        memcpy(h_out, hb, sizeof(uint16_t) * (size_t)I);
    free(hb);
}

/* One MXFP4 expert (expert_any with nv = 0). */
void oracle_expert(const uint16_t *x, const uint8_t *codes_e,
                   const uint8_t *scales_e, int H, int I, uint16_t *h_out,
                   uint16_t *o_out)
{
    expert_any(x, codes_e, scales_e, NULL, FMT_MXFP4, H, I, h_out, o_out);
}

/* One NVFP4 expert: gs = {gate/up multiplier, down multiplier}. */
void oracle_expert_nvfp4(const uint16_t *x, const uint8_t *codes_e,
                         const uint8_t *scales_e, const float *gs, int H, int I,
                         uint16_t *h_out, uint16_t *o_out)
{
    expert_any(x, codes_e, scales_e, gs, FMT_NVFP4, H, I, h_out, o_out);
}

/* One sym8 expert: codes_e [3][rows][K] int8, scales_e [3][rows][K/32]
 * binary16 words (as bytes). */
void oracle_expert_sym8(const uint16_t *x, const uint8_t *codes_e,
                        const uint8_t *scales_e, int H, int I, uint16_t *h_out,
                        uint16_t *o_out)
{
    expert_any(x, codes_e, scales_e, NULL, FMT_SYM8, H, I, h_out, o_out);
}

/* ------------------------------------------------------------- combine -- */

/* Routing-weighted combination in slot order with a BF16 rounding after each
 * multiply and each add ([MC] "Grouped top-4 expert execution": the fused
 * combination keeps the serial runner's sequential BF16 multiply/add
 * rounding).  o: [k][H] BF16, w: [k].  If residual != NULL the result is
 * BF16(residual + y) (one more rounding).  y: [H] BF16. */
void oracle_combine(const uint16_t *o, const double *w, int k, int H,
                    const uint16_t *residual, uint16_t *y)
{
    for (int n = 0; n < H; ++n) {
        double acc = 0.0;
        for (int j = 0; j < k; ++j) {
            double wb = oracle_bf16_to_double(oracle_bf16_from_double(w[j]));
            double p = oracle_bf16_to_double(
                oracle_bf16_from_double(oracle_bf16_to_double(o[(size_t)j * H + n]) * wb));
            acc = oracle_bf16_to_double(oracle_bf16_from_double(acc + p));
        }
        if (residual)
            acc = oracle_bf16_to_double(oracle_bf16_from_double(
                oracle_bf16_to_double(residual[n]) + acc));
        y[n] = oracle_bf16_from_double(acc);
    }
}

/* ---------------------------------------------------------- MoE layer -- */

/* Experts + combine for T tokens with given routing, any weight format.
 *   x [T][H], ids [T][k], w [T][k] (double); codes [E][3*I*H/2] with
 *   scales [E][3*I*H/32] (MXFP4) or [E][3*I*H/16] (NVFP4, with gscales
 *   [E][2]), or codes [E][3*I*H] int8 with scales [E][3*I*H/32] binary16
 *   words (sym8); residual [T][H] or NULL, y [T][H], o_out (nullable)
 *   [T][k][H], h_out (nullable) [T][k][I].
 * An id outside [0, E) gives a zero expert output for that slot. */
static void moe_forward_any(const uint16_t *x, int T, int E, int H, int I, int k,
                            const int32_t *ids, const double *w,
                            const uint8_t *codes, const uint8_t *scales,
                            const float *gscales, int fmt,
                            const uint16_t *residual, uint16_t *y,
                            uint16_t *o_out, uint16_t *h_out)
{
    /* bytes of one expert: three matrices of I x H weights */
    const size_t ce = (size_t)3 * I * row_code_bytes(fmt, H);
    const size_t se = (size_t)3 * I * row_scale_bytes(fmt, H);
    const int nv = fmt == FMT_NVFP4;
    uint16_t *o = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)k * H);
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int e = ids[(size_t)t * k + j];
            uint16_t *hj = h_out ? h_out + ((size_t)t * k + j) * I : NULL;
            if (e < 0 || e >= E) {
                memset(o + (size_t)j * H, 0, sizeof(uint16_t) * (size_t)H);
                if (hj)
                    memset(hj, 0, sizeof(uint16_t) * (size_t)I);
                continue;
            }
            expert_any(x + (size_t)t * H, codes + (size_t)e * ce, scales + (size_t)e * se,
                       nv ? gscales + (size_t)e * 2 : NULL, fmt, H, I, hj,
                       o + (size_t)j * H);
        }
        if (o_out)
            memcpy(o_out + (size_t)t * k * H, o, sizeof(uint16_t) * (size_t)k * H);
        oracle_combine(o, w + (size_t)t * k, k, H,
                       residual ? residual + (size_t)t * H : NULL,
                       y + (size_t)t * H);
    }
    free(o);
}

void oracle_moe_forward(const uint16_t *x, int T, int E, int H, int I, int k,
                        const int32_t *ids, const double *w,
                        const uint8_t *codes, const uint8_t *scales,
                        const uint16_t *residual, uint16_t *y,
                        uint16_t *o_out, uint16_t *h_out)
{
    moe_forward_any(x, T, E, H, I, k, ids, w, codes, scales, NULL, FMT_MXFP4, residual, y,
                    o_out, h_out);
}

void oracle_moe_forward_nvfp4(const uint16_t *x, int T, int E, int H, int I, int k,
                              const int32_t *ids, const double *w,
                              const uint8_t *codes, const uint8_t *scales,
                              const float *gscales, const uint16_t *residual,
                              uint16_t *y, uint16_t *o_out, uint16_t *h_out)
{
    moe_forward_any(x, T, E, H, I, k, ids, w, codes, scales, gscales, FMT_NVFP4, residual, y,
                    o_out, h_out);
}

void oracle_moe_forward_sym8(const uint16_t *x, int T, int E, int H, int I, int k,
                             const int32_t *ids, const double *w,
                             const uint8_t *codes, const uint8_t *scales,
                             const uint16_t *residual, uint16_t *y, uint16_t *o_out,
                             uint16_t *h_out)
{
    moe_forward_any(x, T, E, H, I, k, ids, w, codes, scales, NULL, FMT_SYM8, residual, y,
                    o_out, h_out);
}

/* Full layer: route, experts, combine. */
void oracle_moe_layer(const uint16_t *x, int T, int E, int H, int I, int k,
                      const uint16_t *Wr, const float *bias,
                      const uint8_t *codes, const uint8_t *scales,
                      const uint16_t *residual, int32_t *ids, double *w,
                      uint16_t *y)
{
    oracle_route(x, T, H, Wr, E, bias, k, ids, w, NULL);
    oracle_moe_forward(x, T, E, H, I, k, ids, w, codes, scales, residual, y,
                       NULL, NULL);
}

/* --------------------------------------------------------------- stack -- */

/* Weightless RMSNorm before each MoE layer of the stack:
 * xn = BF16(r / sqrt(mean(r^2) + eps)). */
void oracle_rmsnorm(const uint16_t *r, int T, int H, double eps, uint16_t *xn)
{
    for (int t = 0; t < T; ++t) {
        double ss = 0.0;
        for (int n = 0; n < H; ++n) {
            double v = oracle_bf16_to_double(r[(size_t)t * H + n]);
            ss += v * v;
        }
        double inv = 1.0 / sqrt(ss / H + eps);
        for (int n = 0; n < H; ++n)
            xn[(size_t)t * H + n] =
                oracle_bf16_from_double(oracle_bf16_to_double(r[(size_t)t * H + n]) * inv);
    }
}

/* One decode step through L layers: for each layer, xn = RMSNorm(r), route,
 * experts, combine, r = BF16(r + y).  r is updated in place ([T][H]).
 * Per-layer arrays are passed as arrays of pointers.  ids_out [L][T][k]
 * (nullable). */
void oracle_stack_step(uint16_t *r, int T, int L, int E, int H, int I, int k,
                       const uint16_t *const *Wr, const float *const *bias,
                       const uint8_t *const *codes,
                       const uint8_t *const *scales, double eps,
                       int32_t *ids_out)
{
    uint16_t *xn = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)T * H);
    int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * (size_t)T * k);
    double *w = (double *)malloc(sizeof(double) * (size_t)T * k);
    for (int l = 0; l < L; ++l) {
        oracle_rmsnorm(r, T, H, eps, xn);
        oracle_moe_layer(xn, T, E, H, I, k, Wr[l], bias ? bias[l] : NULL,
                         codes[l], scales[l], r, ids, w, r);
        if (ids_out)
            memcpy(ids_out + (size_t)l * T * k, ids, sizeof(int32_t) * (size_t)T * k);
    }
    free(xn);
    free(ids);
    free(w);
}
