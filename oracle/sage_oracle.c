/*
 * sage_oracle.c -- slow, plain fp64 CPU oracle of the smoothed-INT8-QK / FP8-PV
 * quantized attention forward (SageAttention2 / SageAttention2++ method).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The CUDA product path
 * never links, loads or calls it, and it shares no code, header or constant
 * table with the CUDA path.
 *
 * Sources, cited by page and section:
 *   [SA2-abstract]  "SageAttention2: Efficient Attention with Thorough Outlier
 *                   Smoothing and Per-thread INT4 Quantization" (arXiv 2411.10958),
 *                   abstract: smoothing of Q and K, fine-grained quantization of
 *                   (Q, K), FP8 for (P~, V), two-level accumulation of P~V.
 *   [SA2-notes]     zhaifeiyue.github.io notes on 2411.10958: comparison table and
 *                   the "fine-grained quantization + smoothing" paragraph.
 *   [SA2pp-verdict] pith.science verdict on arXiv 2505.21136, fields key_machinery
 *                   (delta_V = |max V| / Vr per channel, P range Pr),
 *                   core_discovery (Pr x Vr bound) and
 *                   skeptic_critique.load_bearing_attack (Vr = 448 in SageAttention2,
 *                   E4M3 dynamic range 448 * 2^9).
 *   [online-softmax] "Online normalizer calculation for softmax" (Milakov and
 *                   Gimelshein), listed among the references of 2411.10958.
 *
 * The pages give no formula written out in full.  Every step below is the
 * plainest reading consistent with them; the readings are:
 *   - K smoothing subtracts the mean of K over all valid tokens of one head.
 *   - Q smoothing subtracts the mean of the valid rows of each 128-row Q block
 *     and adds back dS[t, j] = qbar_t . K_s[j].
 *   - Q and K are quantized to INT8 per group: g_q consecutive rows inside a
 *     128-row block, g_k consecutive keys inside a 128-key tile;
 *     delta = amax / 127, code = clamp(round-half-even(x / delta), -127, 127).
 *   - P~ = exp(x - m) of the tiled online softmax (tiles of 128 keys) is scaled by
 *     Pr and rounded to E4M3 (static scale 1 / Pr, since P~ <= 1).
 *   - V is scaled per channel by delta_V[c] = max_j |V[j, c]| / Vr and rounded
 *     to E4M3.
 *   - The row sum l uses the unquantized P~; O = acc / Pr * delta_V / l.
 *
 * Precision.  All arithmetic is fp64, except where a floating-point value decides
 * an integer code (an INT8 code, an E4M3 code): there the decision is taken in
 * fp32, the precision of the device kernel, with IEEE correctly rounded fp32
 * operations:
 *   qbar, kbar   : fp64 mean, rounded once to fp32;
 *   x_s          : fp32(x) - qbar   (fp32 subtraction);
 *   delta        : fp32(amax) / 127 (fp32 division);
 *   code         : rint(x_s / delta) with the quotient rounded to fp32;
 *   V code       : E4M3(fp32(v / delta_V));
 *   P code       : E4M3(fp32(P~ * Pr)), P~ itself in fp64.
 * Build with -ffp-contract=off and without -ffast-math so that every float
 * expression rounds as written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_TILE 128 /* Q block rows and KV tile keys; part of the numerics */

/* Planted mistakes for the pins' own tests (tests/test_oracle_mutations.py): a build
 * with ORACLE_MUTATION = k > 0 computes the method with mistake k, which at least one
 * pin must then reject.  The default build (0) compiles every mutation away. */
#ifndef ORACLE_MUTATION
#define ORACLE_MUTATION 0
#endif
#define MUT(k) (ORACLE_MUTATION == (k))

typedef struct {
    int n_q, n_kv, d;
    int g_q, g_k;         /* INT8 group sizes (rows of a Q block, keys of a KV tile) */
    int smooth_q, smooth_k;
    int quant_qk;         /* 1: INT8 codes as in the method; 0: exact (identity);  */
                          /* 2: FP4 (E2M1) codes with two-level scales (see below)  */
    int quant_p;          /* 1: E4M3 P; 0: exact P~ * Pr; 2: FP16 P~ (no Pr scale)  */
    int quant_v;          /* 1: E4M3 V; 0: exact V / delta_V; 2: FP16 V (no scale)  */
    double p_range, v_range;
    double sm_scale;
    int causal;           /* bottom-right aligned: key j visible to row i iff j <= i + n_kv - n_q */
} oracle_cfg_t;

static int ceil_div(int a, int b) { return (a + b - 1) / b; }

/* ------------------------------------------------------------------------- */
/* E4M3 ("e4m3fn": 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no    */
/* infinities, only S.1111.111 is NaN; largest finite 448 = 2^8 * 1.75;       */
/* subnormals m * 2^-9).  Encoding rounds to nearest, ties to even, and        */
/* saturates finite values to +-448 (the "satfinite" behaviour).               */
/* ------------------------------------------------------------------------- */
uint8_t oracle_e4m3_from_f32(float xf)
{
    double x = (double)xf;
    uint8_t sign = (x < 0.0 || (x == 0.0 && signbit(x))) ? 0x80 : 0x00;
    double a = fabs(x);
    if (isnan(x)) return 0x7F;
    if (a == 0.0) return sign;
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    int code;
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: a = q * 2^-9, q in [0, 8]; q = 8 is the smallest normal */
        double q = nearbyint(ldexp(a, 9));
        code = (int)q;
    } else {
        int e;
        double fr = frexp(a, &e);     /* a = fr * 2^e, fr in [0.5, 1) */
        int ex = e - 1;               /* a = (2 fr) * 2^ex, 2 fr in [1, 2) */
        double mant = (2.0 * fr - 1.0) * 8.0;  /* exact */
        double q = MUT(1) ? floor(mant + 0.5) : nearbyint(mant);   /* 1: E4M3 ties away from 0 */
        if (q >= 8.0) { q = 0.0; ex += 1; }
        int be = ex + 7;
        if (be > 15 || (be == 15 && q >= 7.0)) return (uint8_t)(sign | 0x7E);
        code = (be << 3) | (int)q;
    }
    return (uint8_t)(sign | code);
}

double oracle_e4m3_to_f64(uint8_t c)
{
    int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* IEEE binary16 rounding of an fp32 value, returned as its exact fp64 value:
 * 11 significant bits for |x| >= 2^-14, a fixed spacing of 2^-24 below (the
 * subnormals), round to nearest with ties to even, and +-inf from 65520 on (the
 * halfway point above the largest finite value 65504).  Used by the FP16 P / V mode
 * (the "qk_int8_pv_fp16" quantization mode of the SageAttention deployment guide). */
double oracle_f16_round(float xf)
{
    double x = (double)xf;
    if (x == 0.0 || isnan(x)) return x;
    double a = fabs(x);
    if (a >= 65520.0) return copysign(INFINITY, x);
    int e;
    frexp(a, &e);                 /* a in [2^(e-1), 2^e) */
    int q = e - 11;               /* spacing of 11 significant bits */
    if (q < -24) q = -24;         /* subnormal spacing */
    double step = ldexp(1.0, q);
    return copysign((MUT(2) ? trunc(a / step) : nearbyint(a / step)) * step, x);   /* 2: fp16 truncates */
}

/* E2M1 (4-bit: 1 sign, 2 exponent bits with bias 1, 1 mantissa bit; magnitudes
 * 0, 0.5, 1, 1.5, 2, 3, 4, 6; no infinities or NaN).  Encoding rounds to nearest
 * with ties to the even mantissa and saturates to +-6. */
static const double oracle_e2m1_mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_to_f64(uint8_t c)
{
    double v = oracle_e2m1_mag[c & 7];
    return (c & 8) ? -v : v;
}

uint8_t oracle_e2m1_from_f32(float xf)
{
    double x = (double)xf;
    uint8_t sign = (x < 0.0 || (x == 0.0 && signbit(x))) ? 8 : 0;
    double a = fabs(x);
    if (isnan(x) || a >= 6.0) return (uint8_t)(sign | 7);
    int best = 0;
    for (int i = 1; i < 8; ++i) {
        double di = fabs(a - oracle_e2m1_mag[i]), db = fabs(a - oracle_e2m1_mag[best]);
        if (di < db || (di == db && (MUT(3) || (i & 1) == 0))) best = i;  /* ties: even mantissa (3: upward) */
    }
    return (uint8_t)(sign | best);
}

/* Two-level FP4 scales of one 128-row tile of smoothed values (fp32, [128][d], rows
 * past `valid` are 0), the microscaling form of 4-bit Q / K on B200 (block-scaled
 * tcgen05.mma kind::mxf4nvf4; "SageAttention3: Microscaling FP4 Attention", listed
 * among the notes' related papers):
 *   g        = amax over the tile / (6 * 448)          (fp32; 1 if amax = 0)
 *   sf[r][b] = E4M3(fp32(amax of row r, channels 16b..16b+15 / g) / 6)
 *              (1 if that amax is 0; the smallest subnormal 2^-9 if it rounds to 0)
 *   code     = E2M1(fp32(x / fp32(g * sf)))
 * so x ~ g * sf * code.  Writes codes (4-bit values in int8), hat = sf * code (exact),
 * the sf codes, and returns g. */
static float oracle_fp4_tile(const float *xs, int d, int8_t *code, double *hat, uint8_t *sf_code)
{
    float amax = 0.0f;
    for (int i = 0; i < ORACLE_TILE * d; ++i) {
        float a = fabsf(xs[i]);
        if (a > amax) amax = a;
    }
    const float g = (amax == 0.0f) ? 1.0f : amax / (MUT(12) ? 6.0f : 2688.0f);   /* 12: no E4M3 headroom */
    for (int r = 0; r < ORACLE_TILE; ++r)
        for (int b0 = 0; b0 < d; b0 += 16) {
            float am = 0.0f;
            for (int c = b0; c < b0 + 16; ++c) {
                float a = fabsf(xs[(size_t)r * d + c]);
                if (a > am) am = a;
            }
            uint8_t sc = 0x38;  /* 1.0 */
            if (am != 0.0f) {
                sc = oracle_e4m3_from_f32((am / g) / 6.0f);
                if ((sc & 0x7F) == 0 && !MUT(13)) sc = 0x01;   /* 13: an underflowing scale stays 0 */
            }
            sf_code[(size_t)r * (d / 16) + b0 / 16] = sc;
            const double sfv = oracle_e4m3_to_f64(sc);
            const float delta = g * (float)sfv;
            for (int c = b0; c < b0 + 16; ++c) {
                size_t o = (size_t)r * d + c;
                uint8_t e = oracle_e2m1_from_f32(xs[o] / delta);
                code[o] = (int8_t)e;
                hat[o] = sfv * oracle_e2m1_to_f64(e);
            }
        }
    return g;
}

/* INT8 code of an fp32 value for a given fp32 scale: round half to even of the
 * correctly rounded fp32 quotient, then clamp to the symmetric range +-127. */
int8_t oracle_int8_code(float xs, float delta)
{
    float r = xs / delta;
    float n = MUT(4) ? truncf(r) : nearbyintf(r);   /* 4: INT8 codes truncate */
    if (n > 127.0f) n = 127.0f;
    if (n < -127.0f) n = -127.0f;
    return (int8_t)n;
}

/* fp32 group scale from an fp32 absolute maximum: amax / 127, or 1 if amax = 0. */
float oracle_int8_scale(float amax)
{
    if (amax == 0.0f) return 1.0f;
    return amax / 127.0f;
}

/* ------------------------------------------------------------------------- */
/* Pre-pass of one (batch, head): smoothing, INT8 Q/K, FP8 V.                 */
/* Inputs are row-major fp64 copies of the fp16/bf16 tensors (exact):         */
/*   q [n_q][d], k [n_kv][d], v [n_kv][d].                                    */
/* Outputs (caller-allocated; *_pad = ceil(n / 128) * 128):                   */
/*   qbar   [Tq][d]  fp32 block means (0 when smooth_q = 0)                   */
/*   kbar   [d]      fp32 token mean (0 when smooth_k = 0)                    */
/*   q_code [nq_pad][d] int8, q_hat [nq_pad][d] fp64 (the operand the         */
/*          attention multiplies: the code, or the exact smoothed value)      */
/*   dq_row [nq_pad] fp32 scale of each row's group (1 for exact mode)        */
/*   k_code, k_hat [nkv_pad][d], dk_key [nkv_pad]: as for Q                   */
/*   k_s    [n_kv][d] fp64 smoothed K, K - kbar, used for dS                  */
/*   v_code [n_kv][d] E4M3 codes, v_hat [n_kv][d] fp64 decoded (or exact      */
/*          V / delta_V), dv [d] fp32 per-channel scale.                      */
/* ------------------------------------------------------------------------- */
int oracle_prepass(const oracle_cfg_t *cfg, const double *q, const double *k, const double *v,
                   float *qbar, float *kbar,
                   int8_t *q_code, double *q_hat, float *dq_row,
                   int8_t *k_code, double *k_hat, float *dk_key, double *k_s,
                   uint8_t *v_code, double *v_hat, float *dv,
                   uint8_t *q_sf, uint8_t *k_sf)
{
    const int nq = cfg->n_q, nk = cfg->n_kv, d = cfg->d;
    if (nq < 0 || nk < 0 || d <= 0) return 1;
    if (cfg->g_q <= 0 || ORACLE_TILE % cfg->g_q || cfg->g_k <= 0 || ORACLE_TILE % cfg->g_k) return 2;
    const int tq = ceil_div(nq, ORACLE_TILE), nq_pad = tq * ORACLE_TILE;
    const int tk = ceil_div(nk, ORACLE_TILE), nk_pad = tk * ORACLE_TILE;

    /* --- Q: per-block mean (Q smoothing, [SA2-abstract]) --- */
    for (int t = 0; t < tq; ++t) {
        int r0 = t * ORACLE_TILE, r1 = r0 + ORACLE_TILE < nq ? r0 + ORACLE_TILE : nq;
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            if (cfg->smooth_q) {
                for (int i = r0; i < r1; ++i) s += q[(size_t)i * d + c];
                s /= (double)(MUT(5) ? ORACLE_TILE : r1 - r0);   /* 5: ragged block mean over 128 rows */
            }
            qbar[(size_t)t * d + c] = (float)s;
        }
    }
    /* --- Q: smoothed values and INT8 codes per group of g_q rows --- */
    float *xs = (float *)malloc(sizeof(float) * (size_t)ORACLE_TILE * d);
    if (!xs) return 3;
    for (int t = 0; t < tq; ++t) {
        const float *qb = qbar + (size_t)t * d;
        for (int r = 0; r < ORACLE_TILE; ++r) {
            int i = t * ORACLE_TILE + r;
            for (int c = 0; c < d; ++c)
                xs[(size_t)r * d + c] = (i < nq) ? ((float)q[(size_t)i * d + c] - qb[c]) : 0.0f;
        }
        if (cfg->quant_qk == 2) {  /* FP4 codes with two-level scales */
            size_t o0 = (size_t)t * ORACLE_TILE * d;
            const float g = oracle_fp4_tile(xs, d, q_code + o0, q_hat + o0, q_sf + (size_t)t * ORACLE_TILE * (d / 16));
            for (int r = 0; r < ORACLE_TILE; ++r) dq_row[t * ORACLE_TILE + r] = g;
            continue;
        }
        for (int g0 = 0; g0 < ORACLE_TILE; g0 += cfg->g_q) {
            float amax = 0.0f;
            for (int r = g0; r < g0 + cfg->g_q; ++r)
                for (int c = 0; c < d; ++c) {
                    float a = fabsf(xs[(size_t)r * d + c]);
                    if (a > amax) amax = a;
                }
            float delta = cfg->quant_qk ? oracle_int8_scale(amax) : 1.0f;
            for (int r = g0; r < g0 + cfg->g_q; ++r) {
                int i = t * ORACLE_TILE + r;
                dq_row[i] = delta;
                for (int c = 0; c < d; ++c) {
                    size_t o = (size_t)i * d + c;
                    if (cfg->quant_qk) {
                        int8_t code = oracle_int8_code(xs[(size_t)r * d + c], delta);
                        q_code[o] = code;
                        q_hat[o] = (double)code;
                    } else {
                        q_code[o] = 0;
                        q_hat[o] = (i < nq) ? q[o] - (double)qb[c] : 0.0;
                    }
                }
            }
        }
    }
    free(xs);

    /* --- K: per-head token mean (K smoothing, [SA2-notes], [SA2-abstract]) --- */
    for (int c = 0; c < d; ++c) {
        double s = 0.0;
        if (cfg->smooth_k && nk > 0) {
            for (int j = 0; j < nk; ++j) s += k[(size_t)j * d + c];
            s /= (double)nk;
        }
        kbar[c] = (float)s;
    }
    for (int j = 0; j < nk; ++j)
        for (int c = 0; c < d; ++c)
            k_s[(size_t)j * d + c] = k[(size_t)j * d + c] + (MUT(6) ? 1.0 : -1.0) * (double)kbar[c];   /* 6: sign */
    /* --- K: FP4 codes with two-level scales per 128-key tile --- */
    if (cfg->quant_qk == 2) {
        float *ks = (float *)malloc(sizeof(float) * (size_t)ORACLE_TILE * d);
        if (!ks) return 3;
        for (int t = 0; t < tk; ++t) {
            for (int r = 0; r < ORACLE_TILE; ++r) {
                int j = t * ORACLE_TILE + r;
                for (int c = 0; c < d; ++c)
                    ks[(size_t)r * d + c] = (j < nk) ? ((float)k[(size_t)j * d + c] - kbar[c]) : 0.0f;
            }
            size_t o0 = (size_t)t * ORACLE_TILE * d;
            const float g = oracle_fp4_tile(ks, d, k_code + o0, k_hat + o0, k_sf + (size_t)t * ORACLE_TILE * (d / 16));
            for (int r = 0; r < ORACLE_TILE; ++r) dk_key[t * ORACLE_TILE + r] = g;
        }
        free(ks);
    }
    /* --- K: INT8 codes per group of g_k keys inside each 128-key tile --- */
    for (int g0 = 0; cfg->quant_qk != 2 && g0 < nk_pad; g0 += cfg->g_k) {
        float amax = 0.0f;
        for (int j = g0; j < g0 + cfg->g_k - (MUT(17) ? 1 : 0) && j < nk; ++j)   /* 17: group amax misses a key */
            for (int c = 0; c < d; ++c) {
                float a = fabsf((float)k[(size_t)j * d + c] - kbar[c]);
                if (a > amax) amax = a;
            }
        float delta = cfg->quant_qk ? oracle_int8_scale(amax) : 1.0f;
        for (int j = g0; j < g0 + cfg->g_k; ++j) {
            dk_key[j] = delta;
            for (int c = 0; c < d; ++c) {
                size_t o = (size_t)j * d + c;
                if (j >= nk) { k_code[o] = 0; k_hat[o] = 0.0; continue; }
                if (cfg->quant_qk) {
                    int8_t code = oracle_int8_code((float)k[o] - kbar[c], delta);
                    k_code[o] = code;
                    k_hat[o] = (double)code;
                } else {
                    k_code[o] = 0;
                    k_hat[o] = k_s[o];
                }
            }
        }
    }

    /* --- V: per-channel scale delta_V = amax / Vr and E4M3 codes ([SA2pp-verdict]) --- */
    const float vr = (float)cfg->v_range;
    for (int c = 0; c < d; ++c) {
        float amax = 0.0f;
        for (int j = 0; j < nk; ++j) {
            float a = fabsf((float)v[(size_t)j * d + c]);
            if (a > amax) amax = a;
        }
        dv[c] = (amax == 0.0f || cfg->quant_v == 2) ? 1.0f : (MUT(7) ? amax * vr : amax / vr);   /* 7 */
    }
    for (int j = 0; j < nk; ++j)
        for (int c = 0; c < d; ++c) {
            size_t o = (size_t)j * d + c;
            if (cfg->quant_v == 2) {  /* FP16 V, unscaled */
                v_code[o] = 0;
                v_hat[o] = oracle_f16_round((float)v[o]);
            } else if (cfg->quant_v) {
                float qv = (float)v[o] / dv[c];
                v_code[o] = oracle_e4m3_from_f32(qv);
                v_hat[o] = oracle_e4m3_to_f64(v_code[o]);
            } else {
                v_code[o] = 0;
                v_hat[o] = v[o] / (double)dv[c];
            }
        }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Attention of one (batch, head) for a list of 128-row Q blocks, from the    */
/* pre-pass outputs.  For every row i of block t:                             */
/*   S[i,j]  = dq(i) dk(j) (q_hat[i] . k_hat[j]) + dS[t,j],                   */
/*             dS[t,j] = qbar_t . k_s[j]            (Q smoothing bias)        */
/*   x[i,j]  = S[i,j] * sm_scale, masked keys excluded;                        */
/*   tiled online softmax over 128-key tiles in increasing j ([online-softmax]):*/
/*     m' = max(m, max_j x), alpha = exp(m - m'), P~ = exp(x - m'),            */
/*     l  = alpha l + sum P~,  acc = alpha acc + sum_j P8_j v_hat[j],          */
/*     P8 = E4M3(fp32(P~ Pr)) (or P~ Pr exactly when quant_p = 0; FP16(fp32(P~)) */
/*     with Pr = 1 when quant_p = 2);                                          */
/*   O[i,c] = acc[c] / Pr * dv[c] / l   (0 for a row that sees no key).       */
/* With integer codes the dot product q_hat . k_hat is a sum of at most d     */
/* products of magnitude <= 127^2, exact in fp64, i.e. the exact integer      */
/* S_int of the INT8 matmul.                                                  */
/* o is [n_q][d]; row_l, row_m (optional) receive l and the final max m of x.  */
/* ------------------------------------------------------------------------- */
int oracle_attn(const oracle_cfg_t *cfg, const float *qbar, const double *q_hat, const float *dq_row,
                const double *k_hat, const float *dk_key, const double *k_s,
                const double *v_hat, const float *dv,
                const int *qblocks, int n_qblocks, double *o, double *row_l, double *row_m)
{
    const int nq = cfg->n_q, nk = cfg->n_kv, d = cfg->d;
    const int tq = ceil_div(nq, ORACLE_TILE), tk = ceil_div(nk, ORACLE_TILE);
    const long off = MUT(15) ? 0 : (long)nk - (long)nq;   /* 15: causal aligned top-left */
    const double pr = (cfg->quant_p == 2) ? 1.0 : cfg->p_range;  /* FP16 P~ is not scaled */
    for (int b = 0; b < n_qblocks; ++b)
        if (qblocks[b] < 0 || qblocks[b] >= tq) return 1;

    for (int b = 0; b < n_qblocks; ++b) {
        const int t = qblocks[b];
        const int r0 = t * ORACLE_TILE;
        const int r1 = r0 + ORACLE_TILE < nq ? r0 + ORACLE_TILE : nq;
        /* dS for this Q block over all keys */
        double *ds = (double *)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
        if (!ds) return 3;
        for (int j = 0; j < nk; ++j) {
            double s = 0.0;
            for (int c = 0; c < d; ++c)   /* 16: dS from the dequantized K instead of K_s */
                s += (double)qbar[(size_t)t * d + c] *
                     (MUT(16) ? k_hat[(size_t)j * d + c] * (double)dk_key[j] : k_s[(size_t)j * d + c]);
            ds[j] = MUT(8) ? -s : s;   /* 8: dS sign */
        }
        #pragma omp parallel for schedule(dynamic, 4)
        for (int i = r0; i < r1; ++i) {
            double *acc = (double *)calloc((size_t)d, sizeof(double));
            double *x = (double *)malloc(sizeof(double) * ORACLE_TILE);
            char *vis = (char *)malloc(ORACLE_TILE);
            double m = -INFINITY, l = 0.0;
            for (int jt = 0; jt < tk; ++jt) {
                int j0 = jt * ORACLE_TILE, j1 = j0 + ORACLE_TILE < nk ? j0 + ORACLE_TILE : nk;
                double tmax = -INFINITY;
                int any = 0;
                for (int j = j0; j < j1; ++j) {
                    int visible = !cfg->causal || (MUT(9) ? (long)j < (long)i + off : (long)j <= (long)i + off);
                    vis[j - j0] = (char)visible;
                    if (!visible) continue;
                    double dot = 0.0;
                    for (int c = 0; c < d; ++c) dot += q_hat[(size_t)i * d + c] * k_hat[(size_t)j * d + c];
                    double s = (double)dq_row[i] * (double)dk_key[j] * dot + ds[j];
                    x[j - j0] = s * cfg->sm_scale;
                    if (x[j - j0] > tmax && !(MUT(10) && j == j1 - 1)) tmax = x[j - j0];   /* 10: last key missed */
                    any = 1;
                }
                if (!any) continue; /* tile fully masked for this row: skipped */
                double mn = m > tmax ? m : tmax;
                double alpha = (m == -INFINITY) ? 0.0 : exp(MUT(14) ? mn - m : m - mn);   /* 14: inverted */
                l *= alpha;
                for (int c = 0; c < d; ++c) acc[c] *= alpha;
                for (int j = j0; j < j1; ++j) {
                    if (!vis[j - j0]) continue;
                    double p = exp(x[j - j0] - mn);
                    l += p;
                    double p8 = cfg->quant_p == 2 ? oracle_f16_round((float)p)
                                : cfg->quant_p ? oracle_e4m3_to_f64(oracle_e4m3_from_f32((float)(p * pr))) : p * pr;
                    if (p8 == 0.0) continue;
                    for (int c = 0; c < d; ++c) acc[c] += p8 * v_hat[(size_t)j * d + c];
                }
                m = mn;
            }
            for (int c = 0; c < d; ++c)
                o[(size_t)i * d + c] = (l > 0.0) ? acc[c] / (MUT(11) ? 1.0 : pr) * (double)dv[c] / l : 0.0;   /* 11 */
            if (row_l) row_l[i] = l;
            if (row_m) row_m[i] = m;
            free(acc); free(x); free(vis);
        }
        free(ds);
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Textbook full-precision attention of one head, two passes in fp64:         */
/* O = softmax(Q K^T sm_scale + mask) V; a row with no visible key gives 0.   */
/* q [n_q][d], k, v [n_kv][d], o [n_q][d].                                    */
/* ------------------------------------------------------------------------- */
int oracle_ref_attn(int n_q, int n_kv, int d, double sm_scale, int causal,
                    const double *q, const double *k, const double *v, double *o)
{
    const long off = (long)n_kv - (long)n_q;
    #pragma omp parallel for schedule(dynamic, 8)
    for (int i = 0; i < n_q; ++i) {
        double *x = (double *)malloc(sizeof(double) * (size_t)(n_kv > 0 ? n_kv : 1));
        double m = -INFINITY;
        for (int j = 0; j < n_kv; ++j) {
            if (causal && (long)j > (long)i + off) { x[j] = -INFINITY; continue; }
            double s = 0.0;
            for (int c = 0; c < d; ++c) s += q[(size_t)i * d + c] * k[(size_t)j * d + c];
            x[j] = s * sm_scale;
            if (x[j] > m) m = x[j];
        }
        double l = 0.0;
        for (int c = 0; c < d; ++c) o[(size_t)i * d + c] = 0.0;
        if (m != -INFINITY) {
            for (int j = 0; j < n_kv; ++j) {
                if (x[j] == -INFINITY) continue;
                double p = exp(x[j] - m);
                l += p;
                for (int c = 0; c < d; ++c) o[(size_t)i * d + c] += p * v[(size_t)j * d + c];
            }
            for (int c = 0; c < d; ++c) o[(size_t)i * d + c] /= l;
        }
        free(x);
    }
    return 0;
}

/* Number of OpenMP threads the oracle uses (1 when built without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
