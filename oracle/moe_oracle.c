/*
 * Oracle for the DeepSeek-V3/R1 MoE FFN layer forward: the steps whose
 * results are compared bit for bit (router logits, affinity, top-k
 * selection, gate weights, e4m3 block quantisation, bf16 rounding).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the test-suite, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * constant with the CUDA library: every constant below is derived here from
 * its mathematical definition.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC (no FMA
 * contraction, so every a*b+c below is two roundings unless written fmaf).
 *
 * Sources (page, section):
 *  - "DeepSeek v3 and R1 Model Architecture" (onlylabs.fyi), section "Local
 *    Balanced Routing to Experts": a token is routed by its token-to-expert
 *    affinity; a per-expert bias term is added for routing only.
 *  - "DeepSeek-R1" architecture card (llm-architectures-explained.vercel.app),
 *    "Every architecture field": 256 routed experts, 8 active, gated experts,
 *    1 shared expert.
 *  - "DeepSeek-R1" (aguasto.com), section "Quantization": the checkpoint is
 *    blockwise FP8.
 *  The pages do not state the affinity function, the arithmetic precision,
 *  the tie-break, the tile shapes or the FP8 format; the readings taken here
 *  (sigmoid affinity, FP32 sequential-FMA logits, lowest-index tie-break,
 *  e4m3 with 1x128 / 128x128 tiles and FP32 scales, amax/448 scaling) are
 *  the problem statement's and are listed as readings in the design notes.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- bf16 -- */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
float oracle_bf16_to_f32(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/* Round binary32 -> bf16, to nearest, ties to even (NaN kept quiet). */
uint16_t oracle_bf16_from_f32(float f)
{
    uint32_t u = bits_from_f32(f);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu))
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* ---------------------------------------------------------------- e4m3 -- */
/*
 * OCP 8-bit floating point, E4M3 variant: 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits; no infinities; S.1111.111 is NaN, so the largest
 * finite magnitude is 2^8 * 1.75 = 448; exponent field 0 holds subnormals
 * m * 2^-9.
 */
float oracle_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    float v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexpf((float)m, -9);
    else        v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return s ? -v : v;
}

/* Nearest e4m3 value of v, ties to the even mantissa, magnitudes that round
 * past 448 saturate to 448 (the "satfinite" convention).  Scaling by a power
 * of two is exact, so the only rounding is the rintf (ties to even) of the
 * magnitude measured in quanta of its binade. */
static float pow2f(int e) { return f32_from_bits((uint32_t)(e + 127) << 23); } /* -126..127 */

uint8_t oracle_e4m3_encode(float v)
{
    if (isnan(v)) return 0x7f;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    float a = fabsf(v);
    if (a >= 448.0f) return sign | 0x7e;             /* 448 = exponent 15, mantissa 6 */
    int E = (int)(bits_from_f32(a) >> 23) - 127;     /* a in [2^E, 2^(E+1)) when normal */
    if (E < -6) {
        /* subnormal e4m3 range: quantum 2^-9 */
        int n = (int)rintf(a * 512.0f);               /* 0..8 */
        if (n == 8) return sign | (1 << 3);           /* rounds up to 2^-6 */
        return sign | (uint8_t)n;
    }
    int n = (int)rintf(a * pow2f(3 - E));             /* quantum 2^(E-3): n in 8..16 */
    if (n == 16) { n = 8; E += 1; }
    if (E > 8 || (E == 8 && n > 14)) return sign | 0x7e;    /* past 448 */
    return sign | (uint8_t)(((E + 7) << 3) | (n - 8));
}

/* ------------------------------------------------------ block quantiser -- */
/*
 * Blockwise e4m3 quantisation of a row-major [rows, cols] fp32 matrix
 * (bf16 inputs are widened exactly beforehand).  A tile is block_rows x 128
 * (block_rows = 1 for activations, 128 for weights; the last row-block may be
 * short).  Per tile: amax = max |v|; if amax == 0 the scale is 1 and every
 * code is +0; else scale = amax / 448 and inv = 448 / amax (each one
 * correctly rounded binary32 division) and q = e4m3(v * inv) with one
 * binary32 multiply.  Dequantised value: decode(q) * scale.
 * scales is [ceil(rows / block_rows), cols / 128] row-major.
 */
void oracle_block_quant(const float *in, int rows, int cols, int block_rows,
                        uint8_t *q, float *scales)
{
    int nkb = cols / 128;
    int nrb = (rows + block_rows - 1) / block_rows;
    for (int rb = 0; rb < nrb; ++rb) {
        int r0 = rb * block_rows;
        int r1 = r0 + block_rows < rows ? r0 + block_rows : rows;
        for (int kb = 0; kb < nkb; ++kb) {
            float amax = 0.0f;
            for (int r = r0; r < r1; ++r)
                for (int c = kb * 128; c < kb * 128 + 128; ++c) {
                    float a = fabsf(in[(size_t)r * cols + c]);
                    if (a > amax) amax = a;
                }
            float scale, inv;
            if (amax == 0.0f) { scale = 1.0f; inv = 0.0f; }
            else { scale = amax / 448.0f; inv = 448.0f / amax; }
            scales[(size_t)rb * nkb + kb] = scale;
            for (int r = r0; r < r1; ++r)
                for (int c = kb * 128; c < kb * 128 + 128; ++c) {
                    size_t i = (size_t)r * cols + c;
                    q[i] = amax == 0.0f ? 0 : oracle_e4m3_encode(in[i] * inv);
                }
        }
    }
}

/*
 * UE8M0 variant: the same tiles with power-of-two scales (an 8-bit exponent
 * per tile, no mantissa).  The scale is rounded up to a power of two, so per
 * tile scale = 2^k with k the least integer such that amax / 2^k <= 448.
 * With amax = f * 2^E (frexp: f in [0.5, 1), exact) and 448 = 0.875 * 2^9,
 * k = E - 9 when f <= 0.875 and E - 8 otherwise.  UE8M0 holds 2^-127 ..
 * 2^127, so k is raised to -127 for tiles with amax < 448 * 2^-128 (bf16
 * inputs never need k > 120).  q = e4m3(v * 2^-k): the power-of-two multiply
 * is exact, so each code is the nearest e4m3 value (ties to even) of the
 * exact quotient, and none saturates.  Zero tile: scale 1 (2^0), +0 codes.
 */
void oracle_block_quant_ue8m0(const float *in, int rows, int cols, int block_rows,
                              uint8_t *q, float *scales)
{
    int nkb = cols / 128;
    int nrb = (rows + block_rows - 1) / block_rows;
    for (int rb = 0; rb < nrb; ++rb) {
        int r0 = rb * block_rows;
        int r1 = r0 + block_rows < rows ? r0 + block_rows : rows;
        for (int kb = 0; kb < nkb; ++kb) {
            float amax = 0.0f;
            for (int r = r0; r < r1; ++r)
                for (int c = kb * 128; c < kb * 128 + 128; ++c) {
                    float a = fabsf(in[(size_t)r * cols + c]);
                    if (a > amax) amax = a;
                }
            int k = 0;
            if (amax != 0.0f) {
                int E;
                float f = frexpf(amax, &E);
                k = f > 0.875f ? E - 8 : E - 9;
                if (k < -127) k = -127;
            }
            scales[(size_t)rb * nkb + kb] = ldexpf(1.0f, k);
            for (int r = r0; r < r1; ++r)
                for (int c = kb * 128; c < kb * 128 + 128; ++c) {
                    size_t i = (size_t)r * cols + c;
                    q[i] = amax == 0.0f ? 0 : oracle_e4m3_encode(ldexpf(in[i], -k));
                }
        }
    }
}

/* Same quantiser on bf16 storage. */
void oracle_block_quant_bf16(const uint16_t *in, int rows, int cols, int block_rows,
                             uint8_t *q, float *scales)
{
    size_t n = (size_t)rows * cols;
    float *tmp = (float *)malloc(n * sizeof(float));
    for (size_t i = 0; i < n; ++i) tmp[i] = oracle_bf16_to_f32(in[i]);
    oracle_block_quant(tmp, rows, cols, block_rows, q, scales);
    free(tmp);
}

/* ------------------------------------------------------- router logits -- */
/*
 * l[t,e] = sum_i x[t,i] * W_r[e,i]: binary32, accumulated from +0 in the
 * order i = 0 .. d-1, one fused multiply-add (single rounding) per term.
 */
void oracle_router_logits(const uint16_t *x, const uint16_t *w, int T, int d, int E,
                          float *logits)
{
    float *wf = (float *)malloc((size_t)E * d * sizeof(float));
    float *xf = (float *)malloc((size_t)d * sizeof(float));
    for (size_t i = 0; i < (size_t)E * d; ++i) wf[i] = oracle_bf16_to_f32(w[i]);
    for (int t = 0; t < T; ++t) {
        for (int i = 0; i < d; ++i) xf[i] = oracle_bf16_to_f32(x[(size_t)t * d + i]);
        for (int e = 0; e < E; ++e) {
            const float *we = wf + (size_t)e * d;
            float acc = 0.0f;
            for (int i = 0; i < d; ++i) acc = fmaf(xf[i], we[i], acc);
            logits[(size_t)t * E + e] = acc;
        }
    }
    free(xf);
    free(wf);
}

/* ------------------------------------------------------------- sigmoid -- */
/*
 * sigma(l) = 1 / (1 + exp(-l)) in binary32, with exp evaluated by
 * Cody & Waite's additive range reduction and a Taylor polynomial
 * (W. J. Cody, W. Waite, "Software Manual for the Elementary Functions",
 * 1980): y = clamp(-l, -87, 87); n = rint(y * log2(e)); r = y - n*ln2 with
 * ln2 split into a 12-bit-short head and a tail, each step one fma;
 * p(r) = sum_{i=0..7} r^i / i! by Horner (fma); exp(y) = p * 2^n.
 * |r| <= ln2/2 (+ rounding), so the truncated term r^8/8! stays below 1e-8.
 */
static float c_log2e, c_ln2_hi, c_ln2_lo, c_inv_fact[8];
static int consts_ready = 0;

static void init_consts(void)
{
    if (consts_ready) return;
    const double ln2 = 0.693147180559945309417232121458176568;   /* ln 2 */
    const double log2e = 1.442695040888963407359924681001892137; /* 1/ln 2 */
    c_log2e = (float)log2e;
    c_ln2_hi = f32_from_bits(bits_from_f32((float)ln2) & 0xfffff000u);
    c_ln2_lo = (float)(ln2 - (double)c_ln2_hi);
    double f = 1.0;
    for (int i = 0; i < 8; ++i) { if (i) f *= i; c_inv_fact[i] = (float)(1.0 / f); }
    consts_ready = 1;
}

float oracle_exp_cw(float y)
{
    init_consts();
    if (y > 87.0f) y = 87.0f;
    if (y < -87.0f) y = -87.0f;
    float n = rintf(y * c_log2e);
    float r = fmaf(-n, c_ln2_hi, y);
    r = fmaf(-n, c_ln2_lo, r);
    float p = c_inv_fact[7];
    for (int i = 6; i >= 0; --i) p = fmaf(p, r, c_inv_fact[i]);
    return ldexpf(p, (int)n);
}

float oracle_sigmoid(float l)
{
    float e = oracle_exp_cw(-l);
    return 1.0f / (1.0f + e);
}

/* ----------------------------------------------------- top-k and gates -- */
/*
 * s = sigma(l); sel_e = s_e + b_e (binary32 add; the bias only selects).
 * The k selected experts are taken one by one: each time the unselected
 * expert with the largest sel, the lowest index among equals.  Output in
 * that rank order.  Gates: S = s_{j0} + s_{j1} + ... in rank order
 * (binary32), g_j = (s_j / S) * routed_scale.
 */
void oracle_route(const float *logits, const float *bias, int T, int E, int k,
                  float routed_scale, int32_t *idx, float *gates, float *scores)
{
    float *s = (float *)malloc((size_t)E * sizeof(float));
    float *sel = (float *)malloc((size_t)E * sizeof(float));
    unsigned char *taken = (unsigned char *)malloc((size_t)E);
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            s[e] = oracle_sigmoid(logits[(size_t)t * E + e]);
            sel[e] = s[e] + bias[e];
            taken[e] = 0;
            if (scores) scores[(size_t)t * E + e] = s[e];
        }
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || sel[e] > sel[best]) best = e;
            }
            taken[best] = 1;
            idx[(size_t)t * k + j] = best;
        }
        float S = 0.0f;
        for (int j = 0; j < k; ++j) S = S + s[idx[(size_t)t * k + j]];
        for (int j = 0; j < k; ++j)
            gates[(size_t)t * k + j] = (s[idx[(size_t)t * k + j]] / S) * routed_scale;
    }
    free(taken);
    free(sel);
    free(s);
}

/* ------------------------------------------------------ array helpers -- */

void oracle_bf16_from_f32_array(const float *in, size_t n, uint16_t *out)
{
    for (size_t i = 0; i < n; ++i) out[i] = oracle_bf16_from_f32(in[i]);
}

void oracle_e4m3_encode_array(const float *in, size_t n, uint8_t *out)
{
    for (size_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(in[i]);
}

void oracle_sigmoid_array(const float *in, size_t n, float *out)
{
    for (size_t i = 0; i < n; ++i) out[i] = oracle_sigmoid(in[i]);
}

/* --------------------------------------------------------- RMSNorm ----- */
/*
 * Pre-norm of the FFN input ("DeepSeek-R1" architecture card, "Facts": norm
 * placement pre, norm type RMSNorm; the norm before the MLP produces the MoE
 * input): x_i = bf16( (h_i * rstd) * gamma_i ),
 * rstd = 1 / sqrt( S / d + eps ),  S = sum_i h_i^2.
 * The pages fix no precision or order; both are taken as the kernel's, so
 * the routing decision on x stays reproducible: 32 binary32 partial sums
 * p_l = sum_j h_{l+32j}^2 (fused multiply-add, j ascending), then five
 * pairwise rounds p_l = p_l + p_{l xor off} for off = 16, 8, 4, 2, 1 (all p_l
 * end equal), S = p_0; S / d, the add of eps, the square root and the
 * reciprocal are correctly rounded binary32 operations.
 */
float oracle_rms_rstd(const uint16_t *h, int d, float eps)
{
    float p[32], q[32];
    for (int l = 0; l < 32; ++l) {
        float acc = 0.0f;
        for (int i = l; i < d; i += 32) {
            float v = oracle_bf16_to_f32(h[i]);
            acc = fmaf(v, v, acc);
        }
        p[l] = acc;
    }
    for (int off = 16; off >= 1; off >>= 1) {
        for (int l = 0; l < 32; ++l) q[l] = p[l] + p[l ^ off];
        for (int l = 0; l < 32; ++l) p[l] = q[l];
    }
    float mean = p[0] / (float)d;
    return 1.0f / sqrtf(mean + eps);
}

void oracle_rmsnorm(const uint16_t *h, const uint16_t *gamma, int T, int d, float eps,
                    uint16_t *x, float *rstd_out)
{
    for (int t = 0; t < T; ++t) {
        const uint16_t *ht = h + (size_t)t * d;
        float r = oracle_rms_rstd(ht, d, eps);
        if (rstd_out) rstd_out[t] = r;
        for (int i = 0; i < d; ++i) {
            float v = (oracle_bf16_to_f32(ht[i]) * r) * oracle_bf16_to_f32(gamma[i]);
            x[(size_t)t * d + i] = oracle_bf16_from_f32(v);
        }
    }
}
