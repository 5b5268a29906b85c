/*
 * focus_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, scalar CPU reference of the FOCUS NVFP4 weight
 * fake-quantizer: per-tensor scale s2, forward, straight-through backward for
 * the scale parameters m and q, AdamW on m and q, and the NVFP4 export pack.
 * Only the tests, the package's smoke check and the benchmark's CPU-baseline
 * leg may load this code.  The CUDA library shares nothing with it: no header,
 * table, helper or constant.
 *
 * Sources (page title, then the part of the page):
 *  [card]  "FOCUS NVFP4 scales for Llama-3.2-1B-Instruct (our reproduction)",
 *          section "What this is": the field table (m per 16-element block,
 *          q per 8-element sub-block, s2 = amax(|W|)/(6*448)), the row-major
 *          layout sentence, and the three equations for S_b, c_i and w'_i with
 *          the two rules after them (E2M1 rounds to nearest, ties to even; a
 *          block whose scaled maximum is 0 gets scale 1 before the clamp).
 *          Section "Calibration": AdamW, betas 0.9/0.999, weight decay 0,
 *          lr 5e-3 for m and 1e-3 for q, m starts at 1 and q at 6.
 *  [gist]  "Technische Samenvatting: FOCUS ...", section "Methodologie",
 *          item 1 (scales learned through the straight-through estimator).
 *
 * Readings of points the pages leave open (each also listed in the design
 * notes of the repository):
 *  - Forward arithmetic is IEEE binary32, round to nearest even, one rounding
 *    per operation, no fused multiply-add: m, q and s2 are FP32 on the card,
 *    and a code that depends on a rounding must be decided in the same
 *    precision on both sides.  Build with -ffp-contract=off.
 *  - x_b = fl(fl(A_b*m_b) / fl(6*s2)); "scaled maximum is 0" means x_b == 0.
 *  - e4m3() is round to nearest even (the plain cast).
 *  - sigmoid(q) is the binary32 rounding of 1/(1+exp(-q)) evaluated in
 *    binary64.
 *  - y_i = fl(w_i / D_k) with D_k = fl(fl(S_b*sigma_k)*s2);
 *    w'_i = bf16_rne(fl(fl(c_i*S_b)*s2)).
 *  - E2M1 keeps the sign of zero: a negative input that rounds to 0 gives
 *    code 0x8 and w' = -0.0.
 *  - Straight-through backward: rounding is the identity inside the clamps,
 *    clamps pass the gradient at their end points and block it outside,
 *    and the substitution x == 0 -> 1 blocks it.  The gradient sums are
 *    accumulated in binary64 and rounded to binary32 once.
 *  - AdamW follows the algorithm with decoupled weight decay and bias
 *    correction, step counted from 1, eps 1e-8; evaluated in binary64 from
 *    the binary32 inputs, results rounded to binary32.
 *  - NVFP4 byte layout: element 2j in the low nibble and 2j+1 in the high
 *    nibble of byte j of a row; one E4M3 byte per block, row-major
 *    [out, in/16]; the tensor scale stored is s2 itself.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define FO_OK 0
#define FO_ERR_SHAPE 1
#define FO_ERR_VALUE 2
#define FO_ERR_NONFINITE 3

/* ------------------------------------------------------------------------ */
/* scalar formats                                                            */
/* ------------------------------------------------------------------------ */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 is the upper half of a binary32. */
float fo_bf16_to_f32(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/* Round a binary32 to bf16, nearest with ties to even, by looking at the
 * 16 bits that are dropped. */
uint16_t fo_f32_to_bf16(float f)
{
    uint32_t u = bits_from_f32(f);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep = u >> 16;
    uint32_t dropped = u & 0xFFFFu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (keep & 1u)))
        keep += 1u; /* the next bf16 up in magnitude (may become inf) */
    return (uint16_t)keep;
}

/* Nearest integer to v >= 0, ties to the even integer. */
static double round_half_even(double v)
{
    double lo = floor(v);
    double frac = v - lo;
    if (frac > 0.5) return lo + 1.0;
    if (frac < 0.5) return lo;
    return (fmod(lo, 2.0) == 0.0) ? lo : lo + 1.0;
}

/* E4M3 ("fn": bias 7, no infinities, 0x7F/0xFF are NaN, max 448) decode. */
double fo_e4m3_decode(int byte)
{
    int sign = (byte >> 7) & 1;
    int e = (byte >> 3) & 0xF;
    int mant = byte & 7;
    double v;
    if (e == 15 && mant == 7) return NAN;
    if (e == 0) v = ldexp((double)mant, -9);               /* subnormal: mant * 2^-9 */
    else v = ldexp(1.0 + mant / 8.0, e - 7);                /* normal */
    return sign ? -v : v;
}

/* E4M3 encode of a non-negative finite x: round to nearest, ties to even,
 * values above 448 saturate to 448.  Returns -1 outside the domain.  The
 * quantizer only ever passes x in [2^-6, 448] (the clamp of the S_b
 * equation), where every result is a normal number. */
int fo_e4m3_encode(float xf)
{
    double x = (double)xf;
    if (!(x >= 0.0) || isinf(x)) return -1;
    if (x > 448.0) return 0x7E;
    if (x < ldexp(1.0, -6)) {
        double k = round_half_even(x / ldexp(1.0, -9));     /* 0..8 */
        return (int)k;                                      /* k == 8 is 2^-6 = 0x08 */
    }
    int E;
    frexp(x, &E);                 /* x = f * 2^E, f in [0.5, 1) */
    int e = E - 1;                /* x in [2^e, 2^(e+1)) */
    double k = round_half_even(ldexp(x, -e) * 8.0);         /* 8..16 */
    if (k == 16.0) { e += 1; k = 8.0; }
    if (e > 8 || (e == 8 && k > 14.0)) return 0x7E;        /* cannot happen for x <= 448 */
    return ((e + 7) << 3) | ((int)k - 8);
}

/* E2M1 magnitudes by code 0..7. */
static const double e2m1_mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double fo_e2m1_decode(int code)
{
    double v = e2m1_mag[code & 7];
    return (code & 8) ? -v : v;
}

/* E2M1 encode of u in [-6, 6]: nearest magnitude, ties to the even code
 * (the card's "ties to even"); the sign bit is kept, so -0.1 gives 0x8.
 * The seven midpoints between neighbouring magnitudes decide the code: the
 * code is the number of midpoints below |u|, and at a midpoint the even of
 * the two neighbouring codes wins.  Magnitudes above 6 saturate to 6. */
int fo_e2m1_encode(float uf)
{
    static const double mid[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
    double a = fabs((double)uf);
    int sign = signbit(uf) ? 8 : 0;
    int code = 0;
    for (int j = 0; j < 7; ++j) {
        if (a > mid[j]) code = j + 1;
        else if (a == mid[j]) code = ((j & 1) == 0) ? j : j + 1; /* even of j, j+1 */
    }
    return sign | code;
}

/* sigmoid(q) as a binary32: 1/(1+exp(-q)) in binary64, rounded once. */
float fo_sigmoid(float q)
{
    double e = exp(-(double)q);
    return (float)(1.0 / (1.0 + e));
}

/* ------------------------------------------------------------------------ */
/* the quantizer, block by block                                             */
/* ------------------------------------------------------------------------ */

/* Everything the forward decides for one 16-element block. */
typedef struct {
    float A;          /* max |w| over the block */
    float x;          /* fl(fl(A*m)/fl(6*s2)), before the zero rule and the clamp */
    int inS;          /* 1 when the clamp of S_b passes the gradient */
    int sb;           /* E4M3 byte of S_b */
    float S;          /* value of S_b */
    float sigma[2];   /* sigmoid(q_k) for the two sub-blocks */
    float D[2];       /* fl(fl(S*sigma_k)*s2) */
    float y[16];      /* fl(w_i / D_k) */
    int in[16];       /* 1 when -6 <= y_i <= 6 */
    int code[16];     /* E2M1 code of clamp(y_i, -6, 6) */
    float c[16];      /* its value */
    float wq[16];     /* fl(fl(c*S)*s2) before the bf16 cast */
    int band[16];     /* 1: |y| within 2^-20 relative of a code boundary or of 6; 2: exactly on a midpoint */
} fo_block;

/* Boundaries of the code decision and of the clamp, in |y|. */
static const double y_edges[8] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0};

static int band_of(float y)
{
    double a = fabs((double)y);
    for (int j = 0; j < 8; ++j) {
        if (a == y_edges[j] && j < 7) return 2;
        if (fabs(a - y_edges[j]) <= ldexp(y_edges[j], -20)) return 1;
    }
    return 0;
}

/* The three equations of the card for one block of 16 weights w (given as
 * bf16 bits), with its block factor m_b and its two sub-block logits q2. */
static void quantize_block(const uint16_t *w16, float m_b, const float *q2, float s2, fo_block *B)
{
    float w[16];
    float A = 0.0f;
    for (int i = 0; i < 16; ++i) {
        w[i] = fo_bf16_to_f32(w16[i]);
        float a = fabsf(w[i]);
        if (a > A) A = a;
    }
    B->A = A;

    /* S_b = e4m3(clamp(max|w_b| * m_b / (6*s2), 2^-6, 448)); scale 1 when the scaled max is 0 */
    float num = A * m_b;
    float den = 6.0f * s2;
    float x = num / den;
    B->x = x;
    B->inS = (x != 0.0f) && (x >= 0x1p-6f) && (x <= 448.0f);
    float xc = x;
    if (xc == 0.0f) xc = 1.0f;
    if (xc < 0x1p-6f) xc = 0x1p-6f;
    if (xc > 448.0f) xc = 448.0f;
    B->sb = fo_e4m3_encode(xc);
    B->S = (float)fo_e4m3_decode(B->sb);

    /* c_i = E2M1(clamp(w_i / (S_b * sigmoid(q_k) * s2), -6, 6)); w'_i = c_i * S_b * s2 */
    for (int k = 0; k < 2; ++k) {
        float sig = fo_sigmoid(q2[k]);
        float Ssig = B->S * sig;
        float D = Ssig * s2;
        B->sigma[k] = sig;
        B->D[k] = D;
        for (int j = 0; j < 8; ++j) {
            int i = 8 * k + j;
            float y = w[i] / D;
            float u = y;
            if (u < -6.0f) u = -6.0f;
            if (u > 6.0f) u = 6.0f;
            B->y[i] = y;
            B->in[i] = (y >= -6.0f) && (y <= 6.0f);
            B->code[i] = fo_e2m1_encode(u);
            B->c[i] = (float)fo_e2m1_decode(B->code[i]);
            float cS = B->c[i] * B->S;
            B->wq[i] = cS * s2;
            B->band[i] = band_of(y);
        }
    }
}

/* Straight-through gradients of one block, given the upstream gradient g of
 * w' (bf16 bits).  With y = w/(S*sigma*s2), c = R(clamp(y)), dR/du = 1,
 * S = E4M3(clamp(x)) with dE/dx = 1 and x = A*m/(6*s2):
 *   dw'/dS = s2*(c - in*y),   dS/dm = inS*A/(6*s2)
 *     => dL/dm = inS * (A/6) * sum_i g_i*(c_i - in_i*y_i)
 *   dw'/dsigma = -in*S*s2*y/sigma,   dsigma/dq = sigma*(1-sigma)
 *     => dL/dq_k = -(1-sigma_k) * S * s2 * sum_{i in k} in_i*g_i*y_i          */
static void block_grads(const fo_block *B, const uint16_t *g16, float s2, double *dm, double dq[2])
{
    double sm = 0.0;
    double sq[2] = {0.0, 0.0};
    for (int i = 0; i < 16; ++i) {
        double g = (double)fo_bf16_to_f32(g16[i]);
        double t = B->in[i] ? ((double)B->c[i] - (double)B->y[i]) : (double)B->c[i];
        sm += g * t;
        if (B->in[i]) sq[i / 8] += g * (double)B->y[i];
    }
    *dm = B->inS ? ((double)B->A / 6.0) * sm : 0.0;
    for (int k = 0; k < 2; ++k)
        dq[k] = -(1.0 - (double)B->sigma[k]) * (double)B->S * (double)s2 * sq[k];
}

static int check_shape(int64_t out, int64_t in)
{
    if (out < 0 || in < 0 || (in % 16) != 0) return FO_ERR_SHAPE;
    return FO_OK;
}

static int check_s2(float s2)
{
    if (!(s2 > 0.0f) || isinf(s2)) return FO_ERR_VALUE;
    return FO_OK;
}

/* ------------------------------------------------------------------------ */
/* public entry points (used through ctypes by the tests)                    */
/* ------------------------------------------------------------------------ */

int fo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void fo_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* s2 = amax(|W|) / (6*448), one binary32 division (6*448 = 2688 exactly).
 * Card, field table, row s2. */
int fo_s2(const uint16_t *W, int64_t n, float *s2_out)
{
    float A = 0.0f;
    int bad = 0;
#pragma omp parallel for reduction(max : A) reduction(| : bad)
    for (int64_t i = 0; i < n; ++i) {
        float w = fo_bf16_to_f32(W[i]);
        if (!isfinite(w)) bad = 1;
        float a = fabsf(w);
        if (a > A) A = a;
    }
    if (bad) return FO_ERR_NONFINITE;
    *s2_out = A / 2688.0f;
    return FO_OK;
}

/* Counters the forward reports. */
typedef struct {
    int64_t zero_blocks;   /* x == 0 (scale forced to 1) */
    int64_t clamp_low;     /* 0 < x < 2^-6, or x < 0 */
    int64_t clamp_high;    /* x > 448 */
    int64_t out_of_range;  /* |y| > 6 */
    int64_t band;          /* |y| within 2^-20 relative of a boundary (ties included) */
    int64_t exact_ties;    /* |y| exactly on one of the seven midpoints */
} fo_stats;

/* Forward over a row-major [out, in] tensor.  Every output may be NULL.
 *   Wq     bf16 bits [out, in]   w'
 *   codes  u8 [out, in]          one E2M1 code per element (unpacked)
 *   scales u8 [out, in/16]       E4M3 byte of S_b
 *   band   u8 [out, in]          0 / 1 (near a boundary) / 2 (exactly on a midpoint)
 *   ys     f32 [out, in]         y_i = w_i / D_k                                       */
int fo_fwd(const uint16_t *W, const float *m, const float *q, float s2, int64_t out, int64_t in,
           uint16_t *Wq, uint8_t *codes, uint8_t *scales, uint8_t *band, float *ys, fo_stats *st)
{
    int rc = check_shape(out, in);
    if (rc) return rc;
    if ((rc = check_s2(s2))) return rc;
    const int64_t nb = in / 16;
    int64_t zb = 0, lo = 0, hi = 0, oor = 0, bd = 0, ties = 0;
    int bad = 0;
#pragma omp parallel for reduction(+ : zb, lo, hi, oor, bd, ties) reduction(| : bad) schedule(static)
    for (int64_t r = 0; r < out; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const int64_t blk = r * nb + b;
            const int64_t e0 = r * in + 16 * b;
            if (!isfinite(m[blk]) || !isfinite(q[2 * blk]) || !isfinite(q[2 * blk + 1])) bad = 1;
            for (int i = 0; i < 16; ++i)
                if (!isfinite(fo_bf16_to_f32(W[e0 + i]))) bad = 1;
            fo_block B;
            quantize_block(W + e0, m[blk], q + 2 * blk, s2, &B);
            if (B.x == 0.0f) zb++;
            else if (B.x < 0x1p-6f) lo++;
            else if (B.x > 448.0f) hi++;
            if (scales) scales[blk] = (uint8_t)B.sb;
            for (int i = 0; i < 16; ++i) {
                if (!B.in[i]) oor++;
                if (B.band[i]) bd++;
                if (B.band[i] == 2) ties++;
                if (Wq) Wq[e0 + i] = fo_f32_to_bf16(B.wq[i]);
                if (codes) codes[e0 + i] = (uint8_t)B.code[i];
                if (band) band[e0 + i] = (uint8_t)B.band[i];
                if (ys) ys[e0 + i] = B.y[i];
            }
        }
    }
    if (bad) return FO_ERR_NONFINITE;
    if (st) {
        st->zero_blocks = zb; st->clamp_low = lo; st->clamp_high = hi;
        st->out_of_range = oor; st->band = bd; st->exact_ties = ties;
    }
    return FO_OK;
}

/* Straight-through backward: dm [out, in/16], dq [out, in/8] as binary32.
 * accumulate = 1 adds to what dm and dq hold (the sum is formed in binary64
 * and rounded once). */
int fo_ste_bwd(const uint16_t *W, const uint16_t *dWq, const float *m, const float *q, float s2,
               int64_t out, int64_t in, float *dm, float *dq, int accumulate)
{
    int rc = check_shape(out, in);
    if (rc) return rc;
    if ((rc = check_s2(s2))) return rc;
    const int64_t nb = in / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < out; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const int64_t blk = r * nb + b;
            const int64_t e0 = r * in + 16 * b;
            fo_block B;
            quantize_block(W + e0, m[blk], q + 2 * blk, s2, &B);
            double gm, gq[2];
            block_grads(&B, dWq + e0, s2, &gm, gq);
            if (accumulate) {
                dm[blk] = (float)((double)dm[blk] + gm);
                dq[2 * blk] = (float)((double)dq[2 * blk] + gq[0]);
                dq[2 * blk + 1] = (float)((double)dq[2 * blk + 1] + gq[1]);
            } else {
                dm[blk] = (float)gm;
                dq[2 * blk] = (float)gq[0];
                dq[2 * blk + 1] = (float)gq[1];
            }
        }
    }
    return FO_OK;
}

/* AdamW with decoupled weight decay (Loshchilov & Hutter), bias-corrected
 * moments, step t counted from 1:
 *   p   <- p * (1 - lr*wd)
 *   v1  <- b1*v1 + (1-b1)*g
 *   v2  <- b2*v2 + (1-b2)*g^2
 *   p   <- p - (lr/(1-b1^t)) * v1 / (sqrt(v2)/sqrt(1-b2^t) + eps)
 * Card, "Calibration": betas 0.9/0.999, weight decay 0, constant lr. */
int fo_adamw(float *p, const float *g, float *v1, float *v2, int64_t n, double lr, double b1, double b2,
             double eps, double wd, int64_t step)
{
    if (n < 0) return FO_ERR_SHAPE;
    if (step < 1 || !(lr >= 0.0) || !(eps >= 0.0) || !(b1 >= 0.0 && b1 < 1.0) || !(b2 >= 0.0 && b2 < 1.0))
        return FO_ERR_VALUE;
    const double bc1 = 1.0 - pow(b1, (double)step);
    const double bc2 = 1.0 - pow(b2, (double)step);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double pi = (double)p[i] * (1.0 - lr * wd);
        double gi = (double)g[i];
        double a = b1 * (double)v1[i] + (1.0 - b1) * gi;
        double s = b2 * (double)v2[i] + (1.0 - b2) * gi * gi;
        pi -= (lr / bc1) * a / (sqrt(s) / sqrt(bc2) + eps);
        v1[i] = (float)a;
        v2[i] = (float)s;
        p[i] = (float)pi;
    }
    return FO_OK;
}

/* One calibration step of one tensor, as the composition of the three parts
 * above: forward (w' written when Wq is not NULL), straight-through backward
 * (added to dm_acc / dq_acc when they are not NULL), then AdamW on m and q.
 * gm_out / gq_out (may be NULL) receive the binary32 gradients used. */
int fo_step(const uint16_t *W, const uint16_t *dWq, float *m, float *q, float *m_v1, float *m_v2,
            float *q_v1, float *q_v2, float s2, int64_t out, int64_t in, double lr_m, double lr_q,
            double b1, double b2, double eps, double wd, int64_t step, uint16_t *Wq,
            const float *dm_acc, const float *dq_acc, float *gm_out, float *gq_out)
{
    int rc = check_shape(out, in);
    if (rc) return rc;
    if ((rc = check_s2(s2))) return rc;
    const int64_t nb = out * (in / 16);
    float *gm = gm_out, *gq = gq_out;
    float *own = NULL;
    if (!gm || !gq) {
        own = (float *)malloc(sizeof(float) * 3 * (size_t)(nb > 0 ? nb : 1));
        if (!own) return FO_ERR_VALUE;
        gm = own;
        gq = own + nb;
    }
    if (Wq) {
        rc = fo_fwd(W, m, q, s2, out, in, Wq, NULL, NULL, NULL, NULL, NULL);
        if (rc) goto done;
    }
    if (dm_acc && dq_acc) {
        memcpy(gm, dm_acc, sizeof(float) * (size_t)nb);
        memcpy(gq, dq_acc, sizeof(float) * 2 * (size_t)nb);
        rc = fo_ste_bwd(W, dWq, m, q, s2, out, in, gm, gq, 1);
    } else {
        rc = fo_ste_bwd(W, dWq, m, q, s2, out, in, gm, gq, 0);
    }
    if (rc) goto done;
    rc = fo_adamw(m, gm, m_v1, m_v2, nb, lr_m, b1, b2, eps, wd, step);
    if (rc) goto done;
    rc = fo_adamw(q, gq, q_v1, q_v2, 2 * nb, lr_q, b1, b2, eps, wd, step);
done:
    free(own);
    return rc;
}

/* NVFP4 export: codes u8 [out, in/2] (element 2j low nibble, 2j+1 high),
 * scales u8 [out, in/16] (E4M3 bytes of S_b), tensor scale = s2.
 * Card, "What this is": E2M1 elements, one E4M3 scale per 16 elements, one
 * FP32 scale per tensor. */
int fo_pack(const uint16_t *W, const float *m, const float *q, float s2, int64_t out, int64_t in,
            uint8_t *codes, uint8_t *scales, float *tensor_scale)
{
    int rc = check_shape(out, in);
    if (rc) return rc;
    if ((rc = check_s2(s2))) return rc;
    const int64_t nb = in / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < out; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const int64_t blk = r * nb + b;
            const int64_t e0 = r * in + 16 * b;
            fo_block B;
            quantize_block(W + e0, m[blk], q + 2 * blk, s2, &B);
            scales[blk] = (uint8_t)B.sb;
            for (int j = 0; j < 8; ++j)
                codes[e0 / 2 + j] = (uint8_t)((B.code[2 * j] & 0xF) | ((B.code[2 * j + 1] & 0xF) << 4));
        }
    }
    *tensor_scale = s2;
    return FO_OK;
}

/* ------------------------------------------------------------------------ */
/* FourOverSix: round-to-nearest NVFP4 with a choice of two block targets    */
/* ------------------------------------------------------------------------ */
/*
 * Sources: [card] section "Calibration", the activation bullet: every
 * 16-element block's scale maps the block maximum to 6 or to 4, whichever
 * has the lower error, with one FP32 scale per token; [card] section
 * "Perplexity": round-to-nearest FourOverSix weights are the reference row;
 * "Llama-3.1-8B-Instruct FlipQuant MixFP4 maps", section "What this is": the
 * rest of the format is NVFP4 (16-element blocks, E4M3 scale, FP32 tensor
 * scale).
 *
 * Readings (the pages give the rule in words only):
 *  - The candidate for target T (6 or 4) is the card's block equations with
 *    m = 1, sigmoid = 1 and T in place of 6: x_T = fl(A / fl(T*s)); scale 1
 *    when x_T == 0; S_T = e4m3(clamp(x_T, 2^-6, 448)); D_T = fl(S_T*s);
 *    c_i = E2M1(clamp(fl(w_i/D_T), -6, 6)).  With T = 6 this is plain NVFP4
 *    round to nearest.  These decisions are binary32, as every other
 *    decision of the quantizer.
 *  - "error" is the squared error of the dequantized block,
 *        e_T = sum over i = 0..15 of (w_i - c_i*S_T*s)^2,
 *    taken as a real number: the pages fix no precision for it, so the
 *    definition itself is used, with no rounding.  w_i, c_i, S_T and s are
 *    binary32 values, so every term is a dyadic rational and the comparison
 *    e_4 < e_6 has one exact answer.
 *  - The target 4 is taken only when e_4 < e_6 exactly; equal errors keep 6.
 *  - How the comparison is evaluated (its result is the exact one either
 *    way): both errors are first summed in binary64 in element order,
 *    d_i = w_i - (c_i*S_T)*s (c_i*S_T is exact in binary32, its product with
 *    s exact in binary64, one rounding in the difference), e <- e + d_i*d_i.
 *    Each sum is then within gamma_18 = 18u/(1-18u) < 2^-48.8 of e_T
 *    (u = 2^-53: one rounding in d_i, two in the square, at most fifteen in
 *    the additions), so when the two binary64 sums differ by more than
 *    2^-46 of their sum their order is the exact order.  Otherwise the
 *    difference e_4 - e_6 is formed exactly as a floating-point expansion
 *    and its sign read off (f46_exact_sign below).
 *  - The errors reported are the binary64 sums (exact whenever every d_i^2
 *    and partial sum fits 53 bits, e.g. the hand-derived examples).
 *  - The dequantized value is bf16(fl(fl(c*S)*s)), as w' of the card.
 *  - One scale per token: s_t = fl(A_row / 2688), the tensor scale's formula
 *    over one row.  A row whose maximum is 0 has s_t = 0; its blocks get
 *    scale byte 0x38 (1.0), codes 0 and values 0.
 */

typedef struct {
    int sb[2];         /* E4M3 byte of S_T for T = 6 (index 0) and T = 4 (index 1) */
    int code[2][16];   /* E2M1 codes under each target */
    double err[2];     /* squared error under each target (binary64 sum in element order) */
    double cSs[2][16]; /* c_i*S_T*s of each element under each target (exact in binary64) */
    int four;          /* 1 when the target 4 is chosen */
} fo_f46_block;

/* Error-free transformations in binary64 (exact while nothing overflows and no
 * product underflows): a + b = s + t (Knuth's two-sum), a*b = p + t (the
 * rounding error of the product by one fused multiply-add). */
static void two_sum(double a, double b, double *s, double *t)
{
    double x = a + b;
    double bv = x - a;
    double av = x - bv;
    *s = x;
    *t = (a - av) + (b - bv);
}

static void two_prod(double a, double b, double *p, double *t)
{
    double x = a * b;
    *p = x;
    *t = fma(a, b, -x);
}

/* Adds b to the expansion h[0..n) -- nonoverlapping components in increasing
 * magnitude whose exact sum is the value -- and returns the new length; zero
 * components are dropped.  Grow-Expansion of J. R. Shewchuk, "Adaptive
 * Precision Floating-Point Arithmetic and Fast Robust Geometric Predicates",
 * Discrete & Computational Geometry 18 (1997), with zero elimination.  The sum
 * is exact; the largest component carries the sign of the value. */
static int grow_expansion(double *h, int n, double b)
{
    double q = b;
    int m = 0;
    for (int i = 0; i < n; ++i) {
        double s, t;
        two_sum(q, h[i], &s, &t);
        if (t != 0.0) h[m++] = t;
        q = s;
    }
    if (q != 0.0) h[m++] = q;
    return m;
}

/* Adds sign * (w - v)^2 to the expansion exactly (sign = +1 or -1):
 * w - v = dh + dl exactly, (dh + dl)^2 = dh^2 + 2*dh*dl + dl^2, each product
 * split into two doubles. */
static int add_square(double *h, int n, double w, double v, double sign)
{
    double dh, dl, p, t;
    two_sum(w, -v, &dh, &dl);
    two_prod(dh, dh, &p, &t);
    n = grow_expansion(h, n, sign * p);
    n = grow_expansion(h, n, sign * t);
    two_prod(2.0 * dh, dl, &p, &t);
    n = grow_expansion(h, n, sign * p);
    n = grow_expansion(h, n, sign * t);
    two_prod(dl, dl, &p, &t);
    n = grow_expansion(h, n, sign * p);
    n = grow_expansion(h, n, sign * t);
    return n;
}

/* Sign (-1, 0, +1) of e_4 - e_6 = sum_i (w_i - v4_i)^2 - sum_i (w_i - v6_i)^2,
 * exactly.  Here w_i is a bf16 value (0 or at least 2^-133 in magnitude,
 * at most 2^128) and v_i = c_i*S*s with at most 30 significant bits (0 or at
 * least 2^-156: c >= 1/2, S >= 2^-6, s >= 2^-149), so every part of w_i - v_i
 * is 0 or at least 2^-185 and every square at least 2^-370: far from
 * binary64's underflow and overflow, where two_sum and two_prod are exact. */
int fo_f46_exact_sign(const double *w, const double *v4, const double *v6, int n_el)
{
    double h[16 * 12 + 4];
    int n = 0;
    for (int i = 0; i < n_el && i < 16; ++i) {
        n = add_square(h, n, w[i], v4[i], 1.0);
        n = add_square(h, n, w[i], v6[i], -1.0);
    }
    if (n == 0) return 0;
    return h[n - 1] > 0.0 ? 1 : -1;
}

static void f46_candidate(const float *w, float A, float s, float target, int *sb, int *code, double *cSs,
                          double *err)
{
    float den = target * s;
    float x = A / den;
    if (x == 0.0f) x = 1.0f;
    if (x < 0x1p-6f) x = 0x1p-6f;
    if (x > 448.0f) x = 448.0f;
    *sb = fo_e4m3_encode(x);
    float S = (float)fo_e4m3_decode(*sb);
    float D = S * s;
    double e = 0.0;
    for (int i = 0; i < 16; ++i) {
        float u = w[i] / D;
        if (u < -6.0f) u = -6.0f;
        if (u > 6.0f) u = 6.0f;
        code[i] = fo_e2m1_encode(u);
        float cS = (float)fo_e2m1_decode(code[i]) * S;                 /* exact */
        cSs[i] = (double)cS * (double)s;                               /* exact: at most 30 bits */
        double d = (double)w[i] - cSs[i];
        e = e + d * d;
    }
    *err = e;
}

/* Both candidates of one block of 16 bf16 values with scale s > 0, and the choice. */
static void f46_block(const uint16_t *w16, float s, fo_f46_block *B)
{
    float w[16];
    double wd[16];
    float A = 0.0f;
    for (int i = 0; i < 16; ++i) {
        w[i] = fo_bf16_to_f32(w16[i]);
        wd[i] = (double)w[i];
        float a = fabsf(w[i]);
        if (a > A) A = a;
    }
    f46_candidate(w, A, s, 6.0f, &B->sb[0], B->code[0], B->cSs[0], &B->err[0]);
    f46_candidate(w, A, s, 4.0f, &B->sb[1], B->code[1], B->cSs[1], &B->err[1]);
    const double e6 = B->err[0], e4 = B->err[1];
    if (fabs(e4 - e6) > 0x1p-46 * (e4 + e6))
        B->four = e4 < e6;                                  /* the binary64 order is the exact order */
    else
        B->four = fo_f46_exact_sign(wd, B->cSs[1], B->cSs[0], 16) < 0;
}

/* FourOverSix over a row-major [rows, cols] bf16 tensor (cols % 16 == 0).
 * per_row = 0: s is the tensor scale (s2 of the weights, > 0);
 * per_row = 1: every row gets its own scale s_t, written to row_scales[r].
 * Outputs (each may be NULL):
 *   codes  u8 [rows, cols]        E2M1 code of the chosen target, one per element
 *   scales u8 [rows, cols/16]     E4M3 byte of the chosen scale
 *   Xq     bf16 bits [rows, cols] dequantized values
 *   four   u8 [rows, cols/16]     1 where the target 4 was chosen
 *   errs   f64 [rows, cols/16, 2] squared errors of the targets 6 and 4    */
int fo_f46(const uint16_t *X, int64_t rows, int64_t cols, float s, int per_row, uint8_t *codes,
           uint8_t *scales, uint16_t *Xq, uint8_t *four, double *errs, float *row_scales)
{
    int rc = check_shape(rows, cols);
    if (rc) return rc;
    if (!per_row && (rc = check_s2(s))) return rc;
    if (per_row && !row_scales) return FO_ERR_VALUE;
    const int64_t nb = cols / 16;
    int bad = 0;
#pragma omp parallel for reduction(| : bad) schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *xr = X + r * cols;
        float sr = s;
        for (int64_t i = 0; i < cols; ++i)
            if (!isfinite(fo_bf16_to_f32(xr[i]))) bad = 1;
        if (per_row) {
            float A = 0.0f;
            for (int64_t i = 0; i < cols; ++i) {
                float a = fabsf(fo_bf16_to_f32(xr[i]));
                if (a > A) A = a;
            }
            sr = A / 2688.0f;
            row_scales[r] = sr;
        }
        for (int64_t b = 0; b < nb; ++b) {
            const int64_t blk = r * nb + b;
            const int64_t e0 = r * cols + 16 * b;
            if (sr == 0.0f) {           /* a row of zeros */
                if (scales) scales[blk] = 0x38;
                if (four) four[blk] = 0;
                if (errs) { errs[2 * blk] = 0.0; errs[2 * blk + 1] = 0.0; }
                for (int i = 0; i < 16; ++i) {
                    if (codes) codes[e0 + i] = 0;
                    if (Xq) Xq[e0 + i] = 0;
                }
                continue;
            }
            fo_f46_block B;
            f46_block(xr + 16 * b, sr, &B);
            const int t = B.four;
            const float S = (float)fo_e4m3_decode(B.sb[t]);
            if (scales) scales[blk] = (uint8_t)B.sb[t];
            if (four) four[blk] = (uint8_t)t;
            if (errs) { errs[2 * blk] = B.err[0]; errs[2 * blk + 1] = B.err[1]; }
            for (int i = 0; i < 16; ++i) {
                if (codes) codes[e0 + i] = (uint8_t)B.code[t][i];
                if (Xq) {
                    float cS = (float)fo_e2m1_decode(B.code[t][i]) * S;
                    Xq[e0 + i] = fo_f32_to_bf16(cS * sr);
                }
            }
        }
    }
    return bad ? FO_ERR_NONFINITE : FO_OK;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 round to nearest with one scale per row (per-token activations)     */
/* ------------------------------------------------------------------------ */
/*
 * [card] section "Perplexity", method list: the NVFP4 baseline quantizes
 * activations to NVFP4 with one scale per token.  Read as the card's block
 * equations ("What this is") with m = 1 and sigmoid = 1, applied to each row
 * with its own scale s_t = fl(max_row |x| / 2688) in place of s2:
 *   x_b = fl(A_b / fl(6*s_t)); x_b == 0 -> 1; S_b = e4m3(clamp(x_b, 2^-6, 448))
 *   c_i = E2M1(clamp(fl(x_i / fl(S_b*s_t)), -6, 6));  x'_i = bf16(fl(fl(c_i*S_b)*s_t))
 * A row of zeros gets s_t = 0, scale bytes 0x38 (the zero-block rule), codes 0
 * and values 0.  Outputs as fo_f46 (codes one per element).
 */
int fo_nvfp4_rows(const uint16_t *X, int64_t rows, int64_t cols, uint8_t *codes, uint8_t *scales, uint16_t *Xq,
                  float *row_scales)
{
    int rc = check_shape(rows, cols);
    if (rc) return rc;
    if (!row_scales) return FO_ERR_VALUE;
    const int64_t nb = cols / 16;
    int bad = 0;
#pragma omp parallel for reduction(| : bad) schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *xr = X + r * cols;
        float A_row = 0.0f;
        for (int64_t i = 0; i < cols; ++i) {
            float v = fo_bf16_to_f32(xr[i]);
            if (!isfinite(v)) bad = 1;
            if (fabsf(v) > A_row) A_row = fabsf(v);
        }
        const float st = A_row / 2688.0f;
        row_scales[r] = st;
        for (int64_t b = 0; b < nb; ++b) {
            const int64_t blk = r * nb + b;
            const int64_t e0 = r * cols + 16 * b;
            if (st == 0.0f) {
                if (scales) scales[blk] = 0x38;
                for (int i = 0; i < 16; ++i) {
                    if (codes) codes[e0 + i] = 0;
                    if (Xq) Xq[e0 + i] = 0;
                }
                continue;
            }
            float w[16], A = 0.0f;
            for (int i = 0; i < 16; ++i) {
                w[i] = fo_bf16_to_f32(xr[16 * b + i]);
                if (fabsf(w[i]) > A) A = fabsf(w[i]);
            }
            float x = A / (6.0f * st);
            if (x == 0.0f) x = 1.0f;
            if (x < 0x1p-6f) x = 0x1p-6f;
            if (x > 448.0f) x = 448.0f;
            const int sb = fo_e4m3_encode(x);
            const float S = (float)fo_e4m3_decode(sb);
            const float D = S * st;
            if (scales) scales[blk] = (uint8_t)sb;
            for (int i = 0; i < 16; ++i) {
                float u = w[i] / D;
                if (u < -6.0f) u = -6.0f;
                if (u > 6.0f) u = 6.0f;
                const int c = fo_e2m1_encode(u);
                if (codes) codes[e0 + i] = (uint8_t)c;
                if (Xq) {
                    float cS = (float)fo_e2m1_decode(c) * S;                  /* exact */
                    Xq[e0 + i] = fo_f32_to_bf16(cS * st);
                }
            }
        }
    }
    return bad ? FO_ERR_NONFINITE : FO_OK;
}

/* ------------------------------------------------------------------------ */
/* scale factors in the layout of the sm_100 block-scaled tensor-core GEMM   */
/* ------------------------------------------------------------------------ */
/*
 * Not on the pages: the card deploys the export as plain NVFP4 for standard
 * NVFP4 kernels ("What this is"), and on sm_100 those kernels (cuBLASLt's
 * block-scaled GEMM, the tcgen05 block-scaled MMA) read the E4M3 scale
 * factors of an operand [rows][K/16] in NVIDIA's published 128x4 layout:
 * the scale matrix is padded to a multiple of 128 rows and of 4 columns and
 * cut into atoms of 128 rows x 4 columns (512 bytes), stored atom by atom,
 * the atoms of one 128-row band first (row-major over bands and column
 * groups); inside an atom, scale (r, c) is byte 16*(r mod 32) + 4*(r div 32)
 * + c.  Padding bytes are 0.
 */
int64_t fo_swizzled_bytes(int64_t rows, int64_t cols)
{
    if (rows < 0 || cols < 0) return -1;
    return ((rows + 127) / 128 * 128) * ((cols + 3) / 4 * 4);
}

int fo_scales_swizzle(const uint8_t *lin, int64_t rows, int64_t cols, uint8_t *out)
{
    if (rows < 0 || cols < 0) return FO_ERR_SHAPE;
    const int64_t C = (cols + 3) / 4 * 4;
    memset(out, 0, (size_t)fo_swizzled_bytes(rows, cols));
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            const int64_t atom = (r / 128) * (C / 4) + c / 4;
            const int64_t rr = r % 128;
            out[atom * 512 + 16 * (rr % 32) + 4 * (rr / 32) + c % 4] = lin[r * cols + c];
        }
    }
    return FO_OK;
}

/* ------------------------------------------------------------------------ */
/* MXFP4 variant: 32-element blocks, E8M0 scale, four sub-blocks of 8        */
/* ------------------------------------------------------------------------ */
/*
 * Sources: "Technische Samenvatting: FOCUS ...", section "Probleemstelling"
 * (MXFP4 shares one E8M0 scale per 32 values) and section "Methodologie",
 * items 2 and 3 (the quantization scale is the hardware scale times a
 * learnable coefficient; each hardware block -- 32 values for MXFP4 -- is cut
 * into sub-blocks of 8 with a coefficient each, the dequantization scale
 * stays shared); the card's equations ("What this is") for the structure.
 *
 * Readings (the pages give no MXFP4 formula):
 *  - MXFP4 has no tensor scale.  The block scale follows the format's own
 *    conversion rule (the OCP Microscaling specification: a shared exponent
 *    of floor(log2(max|v|)) minus 2, the largest E2M1 exponent) applied to
 *    the scaled maximum: x_b = fl(A_b * m_b); S_b = 2^(floor(log2 x_b) - 2),
 *    the exponent clamped to E8M0's [-127, 127]; x_b == 0 gives scale 1 (as
 *    the card's zero-block rule); x_b < 0 gives 2^-127.
 *  - c_i = E2M1(clamp(fl(w_i / D_k), -6, 6)) with D_k = fl(S_b * sigmoid(q_k))
 *    for sub-block k = 0..3; w'_i = bf16(fl(c_i * S_b)).
 *  - Straight-through backward as for NVFP4 with s2 = 1 and the power-of-two
 *    rounding passed straight through (S_b = x_b/4 for the gradient):
 *    dm_b = inS * (A_b/4) * sum_i g_i*(in_i ? c_i - y_i : c_i), inS = [x_b >=
 *    2^-125] (inside the exponent clamp; x_b < 2^128 always), and
 *    dq_k = -(1 - sigma_k) * S_b * sum_{i in k} in_i*g_i*y_i.
 *  - Layout: m [out][in/32], q [out][in/8] (q[r][4b+k] for sub-block k of
 *    block b), codes as the NVFP4 pack, E8M0 bytes [out][in/32] (exponent
 *    + 127).
 */

typedef struct {
    float A, x;
    int inS;
    int sb;           /* E8M0 byte */
    float S;
    float sigma[4];
    float y[32];
    int in[32];
    int code[32];
    float c[32];
    float wq[32];     /* fl(c*S) before the bf16 cast */
} fo_mx_block;

/* floor(log2 x) of a positive finite binary32 (exact, from frexp). */
static int floor_log2f(float x)
{
    int e;
    frexpf(x, &e);            /* x = f * 2^e, f in [0.5, 1) */
    return e - 1;
}

static void mx_quantize_block(const uint16_t *w16, float m_b, const float *q4, fo_mx_block *B)
{
    float w[32];
    float A = 0.0f;
    for (int i = 0; i < 32; ++i) {
        w[i] = fo_bf16_to_f32(w16[i]);
        float a = fabsf(w[i]);
        if (a > A) A = a;
    }
    B->A = A;
    float x = A * m_b;
    B->x = x;
    int e;
    if (x == 0.0f) e = 0;
    else if (x < 0.0f) e = -127;
    else {
        e = floor_log2f(x) - 2;
        if (e < -127) e = -127;
        if (e > 127) e = 127;
    }
    B->inS = x >= 0x1p-125f;      /* the exponent clamp: floor(log2 x) >= -125 (x < 2^128 < 2^130 always) */
    B->sb = e + 127;
    B->S = ldexpf(1.0f, e);
    for (int k = 0; k < 4; ++k) {
        float sig = fo_sigmoid(q4[k]);
        float D = B->S * sig;
        B->sigma[k] = sig;
        for (int j = 0; j < 8; ++j) {
            int i = 8 * k + j;
            float y = w[i] / D;
            float u = y;
            if (u < -6.0f) u = -6.0f;
            if (u > 6.0f) u = 6.0f;
            B->y[i] = y;
            B->in[i] = (y >= -6.0f) && (y <= 6.0f);
            B->code[i] = fo_e2m1_encode(u);
            B->c[i] = (float)fo_e2m1_decode(B->code[i]);
            B->wq[i] = B->c[i] * B->S;
        }
    }
}

static int check_shape_mx(int64_t out, int64_t in)
{
    if (out < 0 || in < 0 || (in % 32) != 0) return FO_ERR_SHAPE;
    return FO_OK;
}

/* MXFP4 forward.  Outputs may be NULL: Wq bf16 [out, in]; codes u8 [out, in]
 * (one per element); scales u8 [out, in/32] (E8M0). */
int fo_mx_fwd(const uint16_t *W, const float *m, const float *q, int64_t out, int64_t in, uint16_t *Wq,
              uint8_t *codes, uint8_t *scales)
{
    int rc = check_shape_mx(out, in);
    if (rc) return rc;
    const int64_t nb = in / 32;
    int bad = 0;
#pragma omp parallel for reduction(| : bad) schedule(static)
    for (int64_t r = 0; r < out; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const int64_t blk = r * nb + b;
            const int64_t e0 = r * in + 32 * b;
            if (!isfinite(m[blk])) bad = 1;
            for (int k = 0; k < 4; ++k)
                if (!isfinite(q[4 * blk + k])) bad = 1;
            for (int i = 0; i < 32; ++i)
                if (!isfinite(fo_bf16_to_f32(W[e0 + i]))) bad = 1;
            fo_mx_block B;
            mx_quantize_block(W + e0, m[blk], q + 4 * blk, &B);
            if (scales) scales[blk] = (uint8_t)B.sb;
            for (int i = 0; i < 32; ++i) {
                if (Wq) Wq[e0 + i] = fo_f32_to_bf16(B.wq[i]);
                if (codes) codes[e0 + i] = (uint8_t)B.code[i];
            }
        }
    }
    return bad ? FO_ERR_NONFINITE : FO_OK;
}

/* MXFP4 straight-through backward: dm [out, in/32], dq [out, in/8] as
 * binary32 (sums in binary64, rounded once; accumulate = 1 adds to them). */
int fo_mx_ste_bwd(const uint16_t *W, const uint16_t *dWq, const float *m, const float *q, int64_t out, int64_t in,
                  float *dm, float *dq, int accumulate)
{
    int rc = check_shape_mx(out, in);
    if (rc) return rc;
    const int64_t nb = in / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < out; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const int64_t blk = r * nb + b;
            const int64_t e0 = r * in + 32 * b;
            fo_mx_block B;
            mx_quantize_block(W + e0, m[blk], q + 4 * blk, &B);
            double sm = 0.0, sq[4] = {0.0, 0.0, 0.0, 0.0};
            for (int i = 0; i < 32; ++i) {
                double g = (double)fo_bf16_to_f32(dWq[e0 + i]);
                double t = B.in[i] ? ((double)B.c[i] - (double)B.y[i]) : (double)B.c[i];
                sm += g * t;
                if (B.in[i]) sq[i / 8] += g * (double)B.y[i];
            }
            double gm = B.inS ? ((double)B.A / 4.0) * sm : 0.0;
            dm[blk] = (float)(accumulate ? (double)dm[blk] + gm : gm);
            for (int k = 0; k < 4; ++k) {
                double gq = -(1.0 - (double)B.sigma[k]) * (double)B.S * sq[k];
                dq[4 * blk + k] = (float)(accumulate ? (double)dq[4 * blk + k] + gq : gq);
            }
        }
    }
    return FO_OK;
}
