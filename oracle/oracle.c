/*
 * oracle.c -- plain, slow, obviously-correct CPU reference for the
 * DeepSeek-V4 hybrid compressed attention hot path (CSA + HCA).
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's
 * CPU-baseline leg load this file's shared library; the GPU product path
 * never does, and nothing here is shared with the CUDA sources.
 *
 * Sources (page titles and sections):
 *   [N8]  "DeepSeek V4: Towards Highly Efficient Million Token Context
 *         Intelligence" (papers.chlience.com reading note), section 8 "HCA":
 *         C = H W^KV, Z = H W^Z, S = Softmax_row(Z_block + B),
 *         C^Comp_i = sum_j S_j (.) C_j  (per-channel softmax over a block).
 *   [N7]  same note, section 7 "CSA": m = 4, lightning indexer
 *         I_{t,s} = sum_h w^I_{t,h} ReLU(q^I_{t,h} . K^IComp_s), Top-k
 *         selection, shared key-value MQA core attention, sliding window.
 *   [N9]  same note, section 9 "CSA/HCA other details": RoPE dims in BF16,
 *         the rest of the KV in FP8; indexer in FP4; 128-token window.
 *   [HF]  "DeepSeek-V4: a million-token context that agents can actually
 *         use" (Hugging Face blog), section "Hybrid attention: CSA and HCA".
 *
 * Where the pages leave the arithmetic open, the reading taken is written
 * next to the code.  Two places must be bit-exact with the GPU, so both
 * sides take their floating-point decisions in the same fp32 sequence:
 *   (1) pooling + FP8 quantisation (codes and scales),
 *   (2) index scores (which decide the top-k sets).
 * Everything else (attention) is computed in fp64.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fopenmp -fPIC -shared -lm.
 * -ffp-contract=off matters: every a*b+c below is two roundings unless it is
 * written as fmaf().  OpenMP only spreads independent outputs (entries,
 * scores, heads, rows) over threads; each output is computed by one thread
 * in the same sequence whatever the thread count, so results do not depend
 * on it.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* Scalar format helpers                                               */
/* ------------------------------------------------------------------ */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 -> fp32 is exact: bf16 is the top half of an fp32. */
float oracle_bf16_to_f32(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/* fp32 -> bf16, round to nearest, ties to even (finite inputs). */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u = bits_from_f32(f);
    if ((u & 0x7F800000u) == 0x7F800000u)           /* inf / nan: truncate */
        return (uint16_t)((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* Threads used by the parallel loops below (n <= 0: the OpenMP default). */
void oracle_set_threads(int n) { omp_set_num_threads(n > 0 ? n : omp_get_num_procs()); }
int oracle_max_threads(void) { return omp_get_max_threads(); }

/* fp64 -> bf16 rounded once, to nearest with ties to even (no detour
 * through fp32, whose own rounding could land on a bf16 midpoint).  With
 * |x| = f 2^e, f in [0.5, 1), the bf16 spacing near x is 2^(e-8) for normal
 * results and 2^-133 below 2^-126; x / spacing is exact in fp64 and
 * nearbyint() rounds it to nearest-even.  Results of magnitude 2^128 or more
 * are +-inf; NaN stays NaN. */
uint16_t oracle_f64_to_bf16(double x)
{
    if (isnan(x)) return 0x7FC0u;
    const uint16_t sign = signbit(x) ? 0x8000u : 0u;
    const double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80u);
    int e;
    frexp(a, &e);
    const int sp = e - 8 > -133 ? e - 8 : -133;       /* log2 of the bf16 spacing */
    const double r = ldexp(nearbyint(ldexp(a, -sp)), sp);
    if (r >= 0x1p128) return (uint16_t)(sign | 0x7F80u);
    const float f = (float)r;                          /* exact: r is a bf16 value */
    return (uint16_t)(sign | (bits_from_f32(f) >> 16));
}

void oracle_f64_to_bf16_array(const double* x, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f64_to_bf16(x[i]);
}

void oracle_f32_to_bf16_array(const float* x, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16(x[i]);
}

/* FP8 e4m3fn: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities,
 * 0x7F/0xFF are NaN, so the largest finite magnitude is 0x7E = 448.  The
 * "/448" in the scale rule fixes this variant. */
double oracle_e4m3_value(uint8_t code)
{
    int e = (code >> 3) & 0xF, f = code & 7;
    double mag = (e == 0) ? ldexp((double)f, -9) : ldexp(1.0 + f / 8.0, e - 7);
    return (code & 0x80) ? -mag : mag;
}

/* fp32 -> e4m3fn, round to nearest with ties to the even code, saturating
 * to +-448 (the "satfinite" rule).  Plain search over the 127 non-negative
 * finite codes, whose values increase with the code; the sign is copied, so
 * a value that rounds to zero keeps its sign (-0 -> 0x80). */
uint8_t oracle_f32_to_e4m3(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0) return sign | 0x7E;
    int lo = 0;                                  /* largest code with value <= a */
    while (lo + 1 <= 0x7E && oracle_e4m3_value((uint8_t)(lo + 1)) <= a) lo++;
    double vlo = oracle_e4m3_value((uint8_t)lo);
    if (vlo == a) return sign | (uint8_t)lo;
    double vhi = oracle_e4m3_value((uint8_t)(lo + 1));
    double dlo = a - vlo, dhi = vhi - a;
    int pick;
    if (dlo < dhi) pick = lo;
    else if (dhi < dlo) pick = lo + 1;
    else pick = (lo & 1) ? lo + 1 : lo;          /* tie: even mantissa */
    return sign | (uint8_t)pick;
}

void oracle_f32_to_e4m3_array(const float* x, uint8_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_e4m3(x[i]);
}

void oracle_exp_neg_array(const float* z, float* out, int64_t n);

/* FP4 e2m1 (OCP microscaling formats): 1 sign bit, 2 exponent bits (bias 1),
 * 1 mantissa bit.  Magnitudes of codes 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
double oracle_e2m1_value(int nib)
{
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    return (nib & 8) ? -mag[nib & 7] : mag[nib & 7];
}

/* ue8m0 scale byte u -> 2^(u-127) (exponent-only scale of the MX formats). */
double oracle_ue8m0_value(uint8_t u) { return ldexp(1.0, (int)u - 127); }

/* ------------------------------------------------------------------ */
/* (1) Softmax-gated pooling  [N8] and [HF] "softmax-gated pooling with a */
/*     learned positional bias"                                        */
/* ------------------------------------------------------------------ */

/* The pages give the pooling formula but no precision or exp.  Reading:
 * fp32 arithmetic in a fixed order, with exp evaluated by one named method
 * so that a GPU kernel can reproduce the bits:
 *   Cody & Waite argument reduction (Cody & Waite, "Software Manual for the
 *   Elementary Functions", 1980): n = rint(z*log2(e)), r = z - n*ln2 with
 *   ln2 split into a short head (trailing mantissa bits zero, so n*LN2_HI
 *   is exact) and a tail; then the Taylor series of e^r to degree 7 in
 *   Horner form with fused multiply-adds; then the scale 2^n.
 * Constants are the correctly rounded fp32 values of their definitions. */
static const uint32_t K_L2E    = 0x3FB8AA3Bu;  /* RN(1/ln 2)                         */
static const uint32_t K_LN2_HI = 0x3F317200u;  /* RN(ln 2) with 9 low mantissa bits 0 */
static const uint32_t K_LN2_LO = 0x35BFBE8Eu;  /* RN(ln 2 - LN2_HI)                   */
static const uint32_t K_INV_FACT[8] = {        /* RN(1/k!), k = 0..7                 */
    0x3F800000u, 0x3F800000u, 0x3F000000u, 0x3E2AAAABu,
    0x3D2AAAABu, 0x3C088889u, 0x3AB60B61u, 0x39500D01u};

float oracle_const(int which)  /* exposed so a test can check each constant */
{
    if (which == 0) return f32_from_bits(K_L2E);
    if (which == 1) return f32_from_bits(K_LN2_HI);
    if (which == 2) return f32_from_bits(K_LN2_LO);
    if (which >= 10 && which < 18) return f32_from_bits(K_INV_FACT[which - 10]);
    return NAN;
}

/* E(z) ~= e^z for z <= 0 (the pooling only ever needs z - max <= 0). */
float oracle_exp_neg(float z)
{
    if (!(z >= -87.0f)) return 0.0f;                 /* e^-87 ~ 1.6e-38: flush */
    float t  = z * f32_from_bits(K_L2E);
    float nf = nearbyintf(t);                        /* ties to even           */
    float r  = fmaf(-nf, f32_from_bits(K_LN2_HI), z);
    r        = fmaf(-nf, f32_from_bits(K_LN2_LO), r);
    float p  = f32_from_bits(K_INV_FACT[7]);
    for (int k = 6; k >= 0; --k) p = fmaf(p, r, f32_from_bits(K_INV_FACT[k]));
    int n = (int)nf;                                 /* -126 <= n <= 0         */
    return p * f32_from_bits((uint32_t)(n + 127) << 23);
}

void oracle_exp_neg_array(const float* z, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_exp_neg(z[i]);
}

/* Pool one block of m tokens into one entry of d channels.
 *   x, gate : [m][d] bf16 rows of the block (token jm+i is row i)
 *   bias    : [m][d] fp32 learned positional bias, row i = position i in block
 * Per channel c (the softmax runs over the block's tokens, per channel, as
 * the (.) product in [N8] implies):
 *   z_i = fp32(gate_i) + b_i          (fp32 add)
 *   zmax = max_i z_i
 *   e_i = E(z_i - zmax)
 *   S   = e_0 + e_1 + ... (fp32, ascending i)
 *   N   = e_0*x_0 + e_1*x_1 + ... (each product rounded, ascending i)
 *   y   = N / S  (one IEEE division)
 * y64 (optional) gets the same pooled value in fp64 with libm exp(), as an
 * independent cross-check of the fp32 sequence, and mag64 (optional) the
 * fp64 sum of p_i |x_i|, the natural scale of the pooled value's error. */
void oracle_pool_block(const uint16_t* x, const uint16_t* gate, const float* bias,
                       int m, int d, float* y, double* y64, double* mag64)
{
    for (int c = 0; c < d; ++c) {
        float zmax = -INFINITY;
        for (int i = 0; i < m; ++i) {
            float z = oracle_bf16_to_f32(gate[(size_t)i * d + c]) + bias[(size_t)i * d + c];
            if (z > zmax) zmax = z;
        }
        float S = 0.0f, N = 0.0f;
        for (int i = 0; i < m; ++i) {
            float z = oracle_bf16_to_f32(gate[(size_t)i * d + c]) + bias[(size_t)i * d + c];
            float e = oracle_exp_neg(z - zmax);
            float xv = oracle_bf16_to_f32(x[(size_t)i * d + c]);
            S = S + e;
            float prod = e * xv;
            N = N + prod;
        }
        y[c] = N / S;
        if (y64) {
            double zm = -INFINITY, s = 0.0, n = 0.0, a = 0.0;
            for (int i = 0; i < m; ++i) {
                double z = (double)oracle_bf16_to_f32(gate[(size_t)i * d + c]) + (double)bias[(size_t)i * d + c];
                if (z > zm) zm = z;
            }
            for (int i = 0; i < m; ++i) {
                double z = (double)oracle_bf16_to_f32(gate[(size_t)i * d + c]) + (double)bias[(size_t)i * d + c];
                double e = exp(z - zm);
                s += e;
                n += e * (double)oracle_bf16_to_f32(x[(size_t)i * d + c]);
                a += e * fabs((double)oracle_bf16_to_f32(x[(size_t)i * d + c]));
            }
            y64[c] = n / s;
            if (mag64) mag64[c] = a / s;
        }
    }
}

/* Storage of one pooled entry ([N9]: RoPE dims BF16, the rest FP8; the
 * scale rule is amax/448 per group of g channels):
 *   channels [0, d - d_rope)  : per group, amax = max |y|, scale = amax/448
 *                               (fp32 division); amax == 0 -> scale 0 and
 *                               codes 0x00; else code = e4m3(y / scale)
 *                               (fp32 division, then RN-even, satfinite)
 *   channels [d - d_rope, d)  : bf16 RN of y. */
void oracle_quant_entry(const float* y, int d, int d_rope, int g,
                        uint8_t* codes, float* scales, uint16_t* rope)
{
    int dn = d - d_rope;
    for (int G = 0; G < dn / g; ++G) {
        float amax = 0.0f;
        for (int c = G * g; c < (G + 1) * g; ++c) {
            float a = fabsf(y[c]);
            if (a > amax) amax = a;
        }
        float scale = amax / 448.0f;
        scales[G] = scale;
        for (int c = G * g; c < (G + 1) * g; ++c)
            codes[c] = (amax == 0.0f) ? 0x00 : oracle_f32_to_e4m3(y[c] / scale);
    }
    for (int c = dn; c < d; ++c) rope[c - dn] = oracle_f32_to_bf16(y[c]);
}

/* ------------------------------------------------------------------ */
/* Entry and query extras  [N9] "Query / KV entry RMSNorm", "Partial     */
/* RoPE", "Attention Sink"                                              */
/* ------------------------------------------------------------------ */

/* RMSNorm of one d-vector (d a power of two) in a fixed fp32 sequence, so
 * that the FP8 codes of a normalised entry can be bit-exact: every square is
 * rounded; ss is the pairwise tree sum over consecutive pairs (level by
 * level: t[i] = t[2i] + t[2i+1]); mean = ss / d; r = sqrt(mean + eps)
 * (IEEE, correctly rounded); out_c = (y_c / r) * w_c.  The pages give no
 * precision or epsilon; eps is an argument (1e-6 in the workloads).
 * out may alias y. */
void oracle_rmsnorm_f32(const float* y, int d, const float* w, float eps, float* out)
{
    float* t = (float*)malloc(sizeof(float) * (size_t)d);
    for (int c = 0; c < d; ++c) t[c] = y[c] * y[c];
    for (int n = d; n > 1; n >>= 1)
        for (int i = 0; i < n / 2; ++i) t[i] = t[2 * i] + t[2 * i + 1];
    const float mean = t[0] / (float)d;
    const float r = sqrtf(mean + eps);
    for (int c = 0; c < d; ++c) out[c] = (y[c] / r) * w[c];
    free(t);
}

/* Partial RoPE on n_r values (the last n_r dims of a vector): pair i =
 * (v[2i], v[2i+1]) is rotated by the angle sign * pos * f_i, where f_i =
 * inv_freq[i] (fp32, the caller's frequency table) and pos an integer
 * position, so the fp64 angle pos * f_i is exact.  fp64 throughout:
 *   (a, b) -> (a cos - b sin, a sin + b cos).
 * The pages fix neither the pairing nor the frequencies; the pairing taken is
 * adjacent dims, the frequencies are an input. */
void oracle_rope_f64(const double* v, int n_r, int64_t pos, const float* inv_freq, int sign, double* out)
{
    for (int i = 0; i < n_r / 2; ++i) {
        const double ang = (double)pos * (double)inv_freq[i];
        const double c = cos(ang), sn = (sign < 0 ? -1.0 : 1.0) * sin(ang);
        const double a = v[2 * i], b = v[2 * i + 1];
        const double x = a * c - b * sn;
        const double y = a * sn + b * c;
        out[2 * i] = x;
        out[2 * i + 1] = y;
    }
}

/* Storage of one entry with the [N9] extras: y (fp32, pooled) is RMS-
 * normalised when norm_w is given; the FP8 dims are quantised as in
 * oracle_quant_entry; the RoPE dims are rotated to the entry's position pos
 * (fp64, then one rounding to bf16) when inv_freq is given. */
static void quant_entry_ex(float* y, int d, int d_rope, int g, const float* norm_w, float eps,
                           const float* inv_freq, int64_t pos, uint8_t* codes, float* scales, uint16_t* rope)
{
    if (norm_w) oracle_rmsnorm_f32(y, d, norm_w, eps, y);
    oracle_quant_entry(y, d, d_rope, g, codes, scales, rope);
    if (inv_freq) {
        const int dn = d - d_rope;
        double v[256], o[256];
        for (int c = 0; c < d_rope; ++c) v[c] = (double)y[dn + c];
        oracle_rope_f64(v, d_rope, pos, inv_freq, +1, o);
        for (int c = 0; c < d_rope; ++c) rope[c] = oracle_f64_to_bf16(o[c]);
    }
}

/* One raw token prepared for the sliding window of the state cache: RMSNorm
 * (norm_w given) in the sequence of oracle_rmsnorm_f32, the non-RoPE dims
 * rounded to bf16 from fp32, the RoPE dims rotated to the token's position in
 * fp64 (inv_freq given) and rounded once to bf16.
 *   x [n][d] bf16, pos [n], out [n][d] bf16. */
void oracle_token_prep(const uint16_t* x, const int64_t* pos, int64_t n, int d, int d_rope,
                       const float* norm_w, float eps, const float* inv_freq, uint16_t* out)
{
    float* y = (float*)malloc(sizeof(float) * (size_t)d);
    const int dn = d - d_rope;
    for (int64_t j = 0; j < n; ++j) {
        for (int c = 0; c < d; ++c) y[c] = oracle_bf16_to_f32(x[(size_t)j * d + c]);
        if (norm_w) oracle_rmsnorm_f32(y, d, norm_w, eps, y);
        for (int c = 0; c < d; ++c) out[(size_t)j * d + c] = oracle_f32_to_bf16(y[c]);
        if (inv_freq) {
            double v[256], o[256];
            for (int c = 0; c < d_rope; ++c) v[c] = (double)y[dn + c];
            oracle_rope_f64(v, d_rope, pos[j], inv_freq, +1, o);
            for (int c = 0; c < d_rope; ++c) out[(size_t)j * d + dn + c] = oracle_f64_to_bf16(o[c]);
        }
    }
    free(y);
}

/* Pool and store n_blocks entries for each of B sequences.
 *   x, gate : [B][x_seq_stride][d] bf16; x points at the first token of
 *             block entry_begin, so block entry_begin+jj is rows jj*m..jj*m+m-1
 *   out     : codes [B][cap][d-d_rope], scales [B][cap][(d-d_rope)/g],
 *             rope [B][cap][d_rope]; entry entry_begin+jj is written.
 * Returns the largest |y32 - y64| / sum_i p_i |x_i| seen (the fp64
 * cross-check of the defined fp32 sequence). */
double oracle_compress_ex(const uint16_t* x, const uint16_t* gate, int64_t x_seq_stride,
                          const float* bias, int m, int B, int64_t n_blocks,
                          int d, int d_rope, int g,
                          uint8_t* codes, float* scales, uint16_t* rope,
                          int64_t cap, int64_t entry_begin,
                          const float* norm_w, float eps, const float* inv_freq, int64_t pos_entry0);

double oracle_compress(const uint16_t* x, const uint16_t* gate, int64_t x_seq_stride,
                       const float* bias, int m, int B, int64_t n_blocks,
                       int d, int d_rope, int g,
                       uint8_t* codes, float* scales, uint16_t* rope,
                       int64_t cap, int64_t entry_begin)
{
    return oracle_compress_ex(x, gate, x_seq_stride, bias, m, B, n_blocks, d, d_rope, g, codes, scales, rope,
                              cap, entry_begin, NULL, 0.0f, NULL, -1);
}

/* oracle_compress with the [N9] extras: each pooled entry is RMS-normalised
 * (norm_w [d], eps) before storage and its RoPE dims rotated to the entry's
 * position, taken as the position of its block's first token, e * m
 * (inv_freq [d_rope/2]); either may be NULL.  pos_entry0: the entry index
 * whose position the first pooled block takes (-1: entry_begin; a test that
 * pools one block of a long sequence into a one-entry buffer passes the
 * block's real index). */
double oracle_compress_ex(const uint16_t* x, const uint16_t* gate, int64_t x_seq_stride,
                          const float* bias, int m, int B, int64_t n_blocks,
                          int d, int d_rope, int g,
                          uint8_t* codes, float* scales, uint16_t* rope,
                          int64_t cap, int64_t entry_begin,
                          const float* norm_w, float eps, const float* inv_freq, int64_t pos_entry0)
{
    const int64_t e_pos0 = pos_entry0 >= 0 ? pos_entry0 : entry_begin;
    int dn = d - d_rope, ng = dn / g;
    double worst = 0.0;
    #pragma omp parallel reduction(max:worst)
    {
        float*  y   = (float*)malloc(sizeof(float) * d);
        double* y64 = (double*)malloc(sizeof(double) * d);
        double* mag = (double*)malloc(sizeof(double) * d);
        #pragma omp for schedule(static)
        for (int64_t be = 0; be < (int64_t)B * n_blocks; ++be) {
            const int b = (int)(be / n_blocks);
            const int64_t jj = be % n_blocks;
            const size_t row = (size_t)b * x_seq_stride + (size_t)jj * m;
            oracle_pool_block(x + row * d, gate + row * d, bias, m, d, y, y64, mag);
            for (int c = 0; c < d; ++c) {
                double den = mag[c] > 1e-30 ? mag[c] : 1e-30;
                double dev = fabs((double)y[c] - y64[c]) / den;
                if (dev > worst) worst = dev;
            }
            int64_t e = entry_begin + jj;
            quant_entry_ex(y, d, d_rope, g, norm_w, eps, inv_freq, (e_pos0 + jj) * m,
                           codes + ((size_t)b * cap + e) * dn,
                           scales + ((size_t)b * cap + e) * ng,
                           rope + ((size_t)b * cap + e) * d_rope);
        }
        free(y); free(y64); free(mag);
    }
    return worst;
}

/* ------------------------------------------------------------------ */
/* (1b) Overlapped CSA compressor and indexer-key compressor  [N7]      */
/* ------------------------------------------------------------------ */
/* [N7] gives CSA two KV streams C_a = H W_a, C_b = H W_b and two gate streams
 * Z_a, Z_b, and builds each compressed entry from 2m adjacent entries with
 * row-wise softmax weights, neighbouring entries' sources overlapping.
 * Reading (the note gives no index formula): entry i pools the m tokens of
 * block i-1 from stream a and the m tokens of block i from stream b, one
 * softmax per channel over those 2m tokens, with a positional bias of 2m
 * rows (rows 0..m-1 for the a-half, m..2m-1 for the b-half).  Each token
 * thus feeds two entries: entry i through stream b and entry i+1 through
 * stream a.  Entry 0 has no previous block: its a-half is absent.  The
 * arithmetic is the fp32 sequence of oracle_pool_block over the 2m tokens in
 * that order (a-half ascending, then b-half ascending).
 * The indexer keys K^IComp_s of [N7] come from the same compressor applied to
 * the indexer-key streams (c channels), then FP4 storage ([N9]: the indexer
 * is FP4): per 32-element block, the OCP MX rule for e2m1: shared exponent
 * X = floor(log2 amax) - 2 (2 = the exponent of e2m1's largest value 6),
 * stored as the ue8m0 byte X + 127 (clamped to 0..254; amax = 0 gives 0),
 * element codes = e2m1(v / 2^X), round to nearest even, saturating at +-6,
 * sign kept. */

/* Pool n token rows (xr[i], gr[i]: d bf16 values each; br[i]: d fp32 bias). */
static void pool_rows(const uint16_t* const* xr, const uint16_t* const* gr, const float* const* br,
                      int n, int d, float* y, double* y64, double* mag64)
{
    for (int c = 0; c < d; ++c) {
        float zmax = -INFINITY;
        for (int i = 0; i < n; ++i) {
            float z = oracle_bf16_to_f32(gr[i][c]) + br[i][c];
            if (z > zmax) zmax = z;
        }
        float S = 0.0f, N = 0.0f;
        for (int i = 0; i < n; ++i) {
            float z = oracle_bf16_to_f32(gr[i][c]) + br[i][c];
            float e = oracle_exp_neg(z - zmax);
            float xv = oracle_bf16_to_f32(xr[i][c]);
            S = S + e;
            float prod = e * xv;
            N = N + prod;
        }
        y[c] = N / S;
        if (y64) {
            double zm = -INFINITY, s = 0.0, nn = 0.0, a = 0.0;
            for (int i = 0; i < n; ++i) {
                double z = (double)oracle_bf16_to_f32(gr[i][c]) + (double)br[i][c];
                if (z > zm) zm = z;
            }
            for (int i = 0; i < n; ++i) {
                double z = (double)oracle_bf16_to_f32(gr[i][c]) + (double)br[i][c];
                double e = exp(z - zm);
                s += e;
                nn += e * (double)oracle_bf16_to_f32(xr[i][c]);
                a += e * fabs((double)oracle_bf16_to_f32(xr[i][c]));
            }
            y64[c] = nn / s;
            if (mag64) mag64[c] = a / s;
        }
    }
}

/* Overlapped pooling of entry jj of sequence b (see above) into y (fp32 d)
 * and y64 (fp64 cross-check, may be NULL).
 *   xa, za, xb, zb : [B][x_seq_stride][d] bf16; row 0 = first token of block
 *                    entry_begin, so the b-half of entry entry_begin+jj is rows
 *                    jj*m .. jj*m+m-1 of xb/zb and, for jj >= 1, its a-half is
 *                    rows (jj-1)*m .. jj*m-1 of xa/za
 *   a_prev, za_prev: [B][x_seq_stride][d], rows 0..m-1 = the a-stream of the
 *                    block before entry_begin (the first entry's a-half); NULL:
 *                    the first entry has no a-half (entry_begin = 0) */
static void pool_overlap_entry(const uint16_t* xa, const uint16_t* za, const uint16_t* xb, const uint16_t* zb,
                               const uint16_t* a_prev, const uint16_t* za_prev, int64_t x_seq_stride,
                               const float* bias, int m, int d, int b, int64_t jj, float* y, double* y64,
                               double* mag64)
{
    const uint16_t* xr[512];
    const uint16_t* gr[512];
    const float* br[512];
    int n = 0;
    const size_t seq = (size_t)b * x_seq_stride;
    const uint16_t* ax = NULL; const uint16_t* az = NULL;
    if (jj >= 1) { ax = xa + (seq + (size_t)(jj - 1) * m) * d; az = za + (seq + (size_t)(jj - 1) * m) * d; }
    else if (a_prev) { ax = a_prev + seq * d; az = za_prev + seq * d; }
    if (ax)
        for (int i = 0; i < m; ++i) { xr[n] = ax + (size_t)i * d; gr[n] = az + (size_t)i * d; br[n] = bias + (size_t)i * d; ++n; }
    for (int i = 0; i < m; ++i) {
        xr[n] = xb + (seq + (size_t)jj * m + i) * d;
        gr[n] = zb + (seq + (size_t)jj * m + i) * d;
        br[n] = bias + (size_t)(m + i) * d;
        ++n;
    }
    pool_rows(xr, gr, br, n, d, y, y64, mag64);
}

/* fp32 -> e2m1 code (4 bits): round to nearest even, saturating at +-6, the
 * sign kept (so -0 and small negatives give 0x8). */
uint8_t oracle_f32_to_e2m1(float v)
{
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    const uint8_t sign = signbit(v) ? 0x8 : 0x0;
    double a = fabs((double)v);
    if (isnan(a)) return 0x7;
    if (a >= 6.0) return (uint8_t)(sign | 0x7);
    int best = 0;
    for (int k = 1; k < 8; ++k) {
        const double dk = fabs(a - mag[k]), db = fabs(a - mag[best]);
        if (dk < db || (dk == db && (k & 1) == 0)) best = k;   /* ties: even code (mantissa bit 0) */
    }
    return (uint8_t)(sign | best);
}

/* One 32-element block: the ue8m0 byte and 16 code bytes (element 2i in the
 * low nibble of byte i). */
void oracle_fp4_quant_block(const float* v, uint8_t* codes, uint8_t* sf)
{
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i) if (fabsf(v[i]) > amax) amax = fabsf(v[i]);
    int X = -127;
    if (amax > 0.0f) {
        int e;
        frexp((double)amax, &e);                 /* amax = f 2^e, f in [0.5, 1): floor(log2 amax) = e - 1 */
        X = (e - 1) - 2;
        if (X < -127) X = -127;
        if (X > 127) X = 127;
    }
    *sf = (uint8_t)(X + 127);
    for (int i = 0; i < 16; ++i) {
        const uint8_t lo = oracle_f32_to_e2m1((float)ldexp((double)v[2 * i], -X));
        const uint8_t hi = oracle_f32_to_e2m1((float)ldexp((double)v[2 * i + 1], -X));
        codes[i] = (uint8_t)(lo | (hi << 4));
    }
}

/* Overlapped CSA compression of n_blocks entries per sequence (FP8/BF16 entry
 * storage as oracle_quant_entry); returns the worst fp32-vs-fp64 deviation. */
double oracle_compress_overlap(const uint16_t* xa, const uint16_t* za, const uint16_t* xb, const uint16_t* zb,
                               const uint16_t* a_prev, const uint16_t* za_prev, int64_t x_seq_stride,
                               const float* bias, int m, int B, int64_t n_blocks, int d, int d_rope, int g,
                               uint8_t* codes, float* scales, uint16_t* rope, int64_t cap, int64_t entry_begin)
{
    const int dn = d - d_rope, ng = dn / g;
    double worst = 0.0;
    #pragma omp parallel reduction(max:worst)
    {
        float* y = (float*)malloc(sizeof(float) * d);
        double* y64 = (double*)malloc(sizeof(double) * d);
        double* mag = (double*)malloc(sizeof(double) * d);
        #pragma omp for schedule(static)
        for (int64_t be = 0; be < (int64_t)B * n_blocks; ++be) {
            const int b = (int)(be / n_blocks);
            const int64_t jj = be % n_blocks;
            pool_overlap_entry(xa, za, xb, zb, a_prev, za_prev, x_seq_stride, bias, m, d, b, jj, y, y64, mag);
            for (int c = 0; c < d; ++c) {
                double den = mag[c] > 1e-30 ? mag[c] : 1e-30;
                double dev = fabs((double)y[c] - y64[c]) / den;
                if (dev > worst) worst = dev;
            }
            const int64_t e = entry_begin + jj;
            oracle_quant_entry(y, d, d_rope, g, codes + ((size_t)b * cap + e) * dn,
                               scales + ((size_t)b * cap + e) * ng, rope + ((size_t)b * cap + e) * d_rope);
        }
        free(y); free(y64); free(mag);
    }
    return worst;
}

/* Indexer keys K^IComp: the overlapped compressor over c-channel indexer-key
 * streams, then FP4 (e2m1 + ue8m0 per 32).  k_codes [B][cap][c/2], k_sf
 * [B][cap][c/32]. */
void oracle_index_key_compress(const uint16_t* xa, const uint16_t* za, const uint16_t* xb, const uint16_t* zb,
                               const uint16_t* a_prev, const uint16_t* za_prev, int64_t x_seq_stride,
                               const float* bias, int m, int B, int64_t n_blocks, int c,
                               uint8_t* k_codes, uint8_t* k_sf, int64_t cap, int64_t entry_begin)
{
    #pragma omp parallel
    {
        float* y = (float*)malloc(sizeof(float) * c);
        #pragma omp for schedule(static)
        for (int64_t be = 0; be < (int64_t)B * n_blocks; ++be) {
            const int b = (int)(be / n_blocks);
            const int64_t jj = be % n_blocks;
            pool_overlap_entry(xa, za, xb, zb, a_prev, za_prev, x_seq_stride, bias, m, c, b, jj, y, NULL, NULL);
            const int64_t e = entry_begin + jj;
            for (int blk = 0; blk < c / 32; ++blk)
                oracle_fp4_quant_block(y + blk * 32, k_codes + ((size_t)b * cap + e) * (c / 2) + blk * 16,
                                       k_sf + ((size_t)b * cap + e) * (c / 32) + blk);
        }
        free(y);
    }
}

/* ------------------------------------------------------------------ */
/* (2) Lightning indexer scores  [N7] eq. I_{t,s}, [N9] "FP4"          */
/* ------------------------------------------------------------------ */

/* Exact FP4 dot of one indexer query head with one indexer key.
 *   qc, kc : c/2 bytes, element 2i in the low nibble of byte i
 *   qs, ks : c/32 ue8m0 bytes, one per block of 32 elements
 * Block b's dot D_b = sum_{i in b} v(q_i) v(k_i) is exact (an integer
 * multiple of 1/4, |D_b| <= 32*36).  The dot is the fp32 sum, in block
 * order b = 0, 1, ..., of the terms t_b = D_b * 2^(eq_b + ek_b), each of
 * which is an exact fp32 value.  With all scale bytes in [123, 127]
 * (2^-4 .. 2^0) every partial sum is exact as well, so the result is the
 * exact dot product, whatever the order; *inexact (if given) is set when a
 * term or the sum is not exact. */
float oracle_fp4_dot(const uint8_t* qc, const uint8_t* qs,
                     const uint8_t* kc, const uint8_t* ks, int c, int* inexact)
{
    float acc = 0.0f;
    double exact = 0.0;
    for (int b = 0; b < c / 32; ++b) {
        int64_t isum = 0;                             /* sum of (2q)(2k) */
        for (int i = b * 32; i < b * 32 + 32; ++i) {
            int qn = (qc[i >> 1] >> ((i & 1) * 4)) & 0xF;
            int kn = (kc[i >> 1] >> ((i & 1) * 4)) & 0xF;
            double qv = oracle_e2m1_value(qn), kv = oracle_e2m1_value(kn);
            isum += (int64_t)llround(2.0 * qv) * (int64_t)llround(2.0 * kv);
        }
        double term = ldexp((double)isum, (int)qs[b] - 127 + (int)ks[b] - 127 - 2);
        float t32 = (float)term;
        if (inexact && (double)t32 != term) *inexact = 1;
        acc = acc + t32;
        exact += term;
    }
    if (inexact && (double)acc != exact) *inexact = 1;
    return acc;
}

/* Index scores for B*Tq queries against Nc_cap indexer keys per sequence.
 *   q_codes [B][Tq][Hi][c/2], q_sf [B][Tq][Hi][c/32], w [B][Tq][Hi] fp32
 *   k_codes [B][Nc_cap][c/2], k_sf [B][Nc_cap][c/32]
 *   q_pos   [B][Tq] absolute position t of each query
 *   scores  [B][Tq][Nc_cap] fp32
 * Eligibility (causal block rule): entry s exists for query t only if its
 * block ends at or before t, i.e. (s+1)*m - 1 <= t.  Ineligible -> -inf.
 * Score: acc = +0; for h = 0..Hi-1 in order: acc = acc + w_h * ReLU(dot_h)
 * (fp32 multiply then fp32 add; ReLU(x) = x > 0 ? x : +0).
 * One key per entry serves every indexer head (K^IComp_s carries no head
 * index in [N7]).  Returns the number of inexact dots seen. */
int64_t oracle_index_scores(const uint8_t* q_codes, const uint8_t* q_sf, const float* w,
                            const uint8_t* k_codes, const uint8_t* k_sf,
                            const int32_t* q_pos, int B, int Tq, int64_t Nc_cap,
                            int Hi, int c, int m, float* scores)
{
    int64_t n_inexact = 0;
    const int cb = c / 2, cs = c / 32;
    for (int b = 0; b < B; ++b) {
        for (int t = 0; t < Tq; ++t) {
            int64_t pos = q_pos[(size_t)b * Tq + t];
            int64_t elig = (pos + 1) / m;
            if (elig > Nc_cap) elig = Nc_cap;
            if (elig < 0) elig = 0;
            float* row = scores + ((size_t)b * Tq + t) * Nc_cap;
            const size_t qi = (size_t)b * Tq + t;
            #pragma omp parallel for schedule(static) reduction(+:n_inexact)
            for (int64_t s = 0; s < Nc_cap; ++s) {
                if (s >= elig) { row[s] = -INFINITY; continue; }
                const uint8_t* kc = k_codes + ((size_t)b * Nc_cap + s) * cb;
                const uint8_t* ks = k_sf + ((size_t)b * Nc_cap + s) * cs;
                float acc = 0.0f;
                for (int h = 0; h < Hi; ++h) {
                    int inexact = 0;
                    float dot = oracle_fp4_dot(q_codes + (qi * Hi + h) * cb, q_sf + (qi * Hi + h) * cs,
                                               kc, ks, c, &inexact);
                    n_inexact += inexact;
                    float relu = dot > 0.0f ? dot : 0.0f;
                    float term = w[qi * Hi + h] * relu;
                    acc = acc + term;
                }
                row[s] = acc;
            }
        }
    }
    return n_inexact;
}

/* ------------------------------------------------------------------ */
/* (3) Top-k selection  [N7] C^SprsComp_t = {C_s | I_{t,s} in Top-k(I_t,:)} */
/* ------------------------------------------------------------------ */

typedef struct { double v; int64_t i; } scored_t;

static int cmp_score_desc_index_asc(const void* a, const void* b)
{
    const scored_t* x = (const scored_t*)a;
    const scored_t* y = (const scored_t*)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->i < y->i) ? -1 : (x->i > y->i);
}
static int cmp_i32(const void* a, const void* b)
{
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/* For each of R rows: the eligible entries are s < min(Nc_cap, (pos+1)/m).
 * Take the min(k, #eligible) largest scores; scores compare as values
 * (+0 == -0), equal scores go to the lower index.  idx[r][:] receives the
 * chosen indices in ascending order, padded with -1; count[r] how many. */
void oracle_topk(const float* scores, const int32_t* q_pos, int R, int64_t Nc_cap,
                 int m, int k, int32_t* idx, int32_t* count)
{
    #pragma omp parallel
    {
    scored_t* buf = (scored_t*)malloc(sizeof(scored_t) * (Nc_cap > 0 ? Nc_cap : 1));
    #pragma omp for schedule(dynamic)
    for (int r = 0; r < R; ++r) {
        int64_t elig = ((int64_t)q_pos[r] + 1) / m;
        if (elig > Nc_cap) elig = Nc_cap;
        if (elig < 0) elig = 0;
        const float* row = scores + (size_t)r * Nc_cap;
        for (int64_t s = 0; s < elig; ++s) { buf[s].v = (double)row[s] + 0.0; buf[s].i = s; }
        qsort(buf, (size_t)elig, sizeof(scored_t), cmp_score_desc_index_asc);
        int64_t kk = elig < k ? elig : k;
        int32_t* out = idx + (size_t)r * k;
        for (int64_t j = 0; j < kk; ++j) out[j] = (int32_t)buf[j].i;
        qsort(out, (size_t)kk, sizeof(int32_t), cmp_i32);
        for (int64_t j = kk; j < k; ++j) out[j] = -1;
        count[r] = (int32_t)kk;
    }
    free(buf);
    }
}

/* ------------------------------------------------------------------ */
/* (4) Core attention  [N7] shared key-value MQA + sliding window,      */
/*     [N8] dense over all compressed entries, [HF] figures 3 and 4    */
/* ------------------------------------------------------------------ */

/* One query token, H heads, one joint softmax over a key list made of
 *   - n_ent compressed entries ent[0..n_ent) of one sequence's cache
 *     (codes [.][d-d_rope] e4m3fn, scales [.][(d-d_rope)/g], rope [.][d_rope]);
 *     the entry is both key and value (shared key-value MQA), dequantised
 *     exactly: code value * scale for the FP8 dims, the bf16 value for the
 *     RoPE dims;
 *   - n_win raw bf16 tokens win[0..n_win) ([n_win][d]), key = value = token.
 * logit_j = softmax_scale * (q_h . k_j); p = softmax(logit); o_h = sum p_j k_j.
 * All in fp64.  out [H][d] fp64, lse [H] fp64 (natural-log log-sum-exp of
 * the scaled logits), either may be NULL.  With no keys at all, o = 0 and
 * lse = -inf. */
void oracle_attend_ex(const uint16_t* q, int H, int d, int d_rope, int g,
                      const uint8_t* codes, const float* scales, const uint16_t* rope,
                      const int64_t* ent, int64_t n_ent,
                      const uint16_t* win, int64_t n_win,
                      float softmax_scale, const float* q_norm_w, float eps, const float* sink,
                      const float* inv_freq, int64_t q_pos, double* out, double* lse);

void oracle_attend(const uint16_t* q, int H, int d, int d_rope, int g,
                   const uint8_t* codes, const float* scales, const uint16_t* rope,
                   const int64_t* ent, int64_t n_ent,
                   const uint16_t* win, int64_t n_win,
                   float softmax_scale, double* out, double* lse)
{
    oracle_attend_ex(q, H, d, d_rope, g, codes, scales, rope, ent, n_ent, win, n_win, softmax_scale,
                     NULL, 0.0f, NULL, NULL, 0, out, lse);
}

/* oracle_attend with the [N9] extras, all in fp64 (each may be NULL):
 *   q_norm_w [d]  : each query head is RMS-normalised, q / sqrt(mean(q^2) +
 *                   eps) * w, before the logits;
 *   inv_freq      : the query's RoPE dims are rotated to its position q_pos
 *                   (the keys carry their own positions already, as stored),
 *                   and the output's RoPE dims are rotated back by -q_pos, so
 *                   that the output, a mix of position-rotated values, carries
 *                   relative positions;
 *   sink [H]      : a per-head logit in the softmax denominator with no value:
 *                   p_j = exp(l_j) / (sum_i exp(l_i) + exp(sink_h)), so the
 *                   attention mass can be below 1.
 * lse includes the sink; with no keys the output is 0 and lse = sink (or
 * -inf without one). */
void oracle_attend_ex(const uint16_t* q, int H, int d, int d_rope, int g,
                      const uint8_t* codes, const float* scales, const uint16_t* rope,
                      const int64_t* ent, int64_t n_ent,
                      const uint16_t* win, int64_t n_win,
                      float softmax_scale, const float* q_norm_w, float eps, const float* sink,
                      const float* inv_freq, int64_t q_pos, double* out, double* lse)
{
    const int dn = d - d_rope, ng = dn / g;
    const int64_t n = n_ent + n_win;
    double* K = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * d);
    for (int64_t j = 0; j < n_ent; ++j) {
        const int64_t e = ent[j];
        double* kr = K + (size_t)j * d;
        for (int c = 0; c < dn; ++c)
            kr[c] = oracle_e4m3_value(codes[(size_t)e * dn + c]) * (double)scales[(size_t)e * ng + c / g];
        for (int c = dn; c < d; ++c)
            kr[c] = (double)oracle_bf16_to_f32(rope[(size_t)e * d_rope + (c - dn)]);
    }
    for (int64_t j = 0; j < n_win; ++j) {
        double* kr = K + (size_t)(n_ent + j) * d;
        for (int c = 0; c < d; ++c) kr[c] = (double)oracle_bf16_to_f32(win[(size_t)j * d + c]);
    }
    #pragma omp parallel
    {
    double* logit = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double* qv = (double*)malloc(sizeof(double) * (size_t)d);
    double* ov = (double*)malloc(sizeof(double) * (size_t)d);
    #pragma omp for schedule(static)
    for (int h = 0; h < H; ++h) {
        const uint16_t* qh = q + (size_t)h * d;
        for (int c = 0; c < d; ++c) qv[c] = (double)oracle_bf16_to_f32(qh[c]);
        if (q_norm_w) {
            double ss = 0.0;
            for (int c = 0; c < d; ++c) ss += qv[c] * qv[c];
            const double r = sqrt(ss / d + (double)eps);
            for (int c = 0; c < d; ++c) qv[c] = qv[c] / r * (double)q_norm_w[c];
        }
        if (inv_freq) oracle_rope_f64(qv + dn, d_rope, q_pos, inv_freq, +1, qv + dn);
        double mx = sink ? (double)sink[h] : -INFINITY;
        for (int64_t j = 0; j < n; ++j) {
            double s = 0.0;
            for (int c = 0; c < d; ++c) s += qv[c] * K[(size_t)j * d + c];
            logit[j] = (double)softmax_scale * s;
            if (logit[j] > mx) mx = logit[j];
        }
        double den = sink ? exp((double)sink[h] - mx) : 0.0;
        for (int64_t j = 0; j < n; ++j) { logit[j] = exp(logit[j] - mx); den += logit[j]; }
        for (int c = 0; c < d; ++c) {
            double o = 0.0;
            for (int64_t j = 0; j < n; ++j) o += logit[j] * K[(size_t)j * d + c];
            ov[c] = n > 0 ? o / den : 0.0;
        }
        if (inv_freq) oracle_rope_f64(ov + dn, d_rope, q_pos, inv_freq, -1, ov + dn);
        if (out) for (int c = 0; c < d; ++c) out[(size_t)h * d + c] = ov[c];
        if (lse) lse[h] = (n > 0 || sink) ? mx + log(den) : -INFINITY;
    }
    free(logit); free(qv); free(ov);
    }
    free(K);
}
