/*
 * adamw4_oracle.c -- plain, slow, single-precision-canonical CPU oracle of the
 * fused 4-bit AdamW step (ZIP-SR / ZE-EDEN).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header, table or constant generator
 * with the CUDA path: the NF4 table, the Philox generator and every step of
 * the update are written out here independently.
 *
 * Pages cited (title -- site), by the section or paragraph a passage sits in:
 *   [K] "A New Approach to 4-bit AdamW Optimizer Quantization: Rounding in
 *        Preconditioner Space" (kongchang.com)
 *   [L] "ZIP-SR 4-bit AdamW -- Preconditioner-space stochastic rounding --
 *        What does it mean?" (learnaivisually.com)
 *   [D] "ZIP-SR / ZE-EDEN: 4-bit AdamW state quantization" (daiwk.github.io)
 *   [Z] "ZIP-SR and ZE-EDEN: Redesigning 4-bit AdamW Optimizer-State
 *        Quantization in Preconditioner Space" (zhichai.net)
 *
 * Arithmetic: every floating-point operation is an IEEE-754 binary32 (float)
 * operation in round-to-nearest-even, with fused multiply-add only where
 * fmaf() is written.  Build with -ffp-contract=off and without fast-math;
 * denormals are kept (no FTZ/DAZ).  Host-side step scalars are formed in
 * binary64 and rounded to binary32 once.  This fixed evaluation order is the
 * canonical form both implementations follow; the pages give real-number
 * formulas only.
 *
 * Parity pins (tests, CPU only): Philox4x32-10 against the published
 * known-answer vectors; NF4 against an independent library quantile; the
 * worked near-zero example of [L]; exact enumeration of the rounding
 * probabilities over every uniform draw; Monte Carlo unbiasedness; torch's
 * fp32 AdamW for the fp32-state path; byte accounting against [L] and [D].
 */
#include <float.h>
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BLOCK 128          /* values per quantisation block [L, memory paragraph] */
#define ORACLE_VCODE_ZIPSR 0
#define ORACLE_VCODE_ZEEDEN 1
/* State-space variants the pages compare the two methods with ([L, car /
 * stochastic rounding paragraph]: the 834M ablation's state-space round-to-
 * nearest and stochastic rounding on the zero-inclusive code; [L, memory
 * paragraph]: a zero-excluded code with a positive floor and no rescale). */
#define ORACLE_VCODE_ZI_RTN 2
#define ORACLE_VCODE_ZI_SR 3
#define ORACLE_VCODE_ZE_FLOOR 4
/* ZIP-SR deciding on the whole 32-bit draw with one binary64 multiply (the
 * library's option beside the binary32 decision of ZIP-SR itself). */
#define ORACLE_VCODE_ZIPSR_U32 5
#define ORACLE_STREAM_V 0u        /* Philox stream for the v draw (ZIP-SR)        */
#define ORACLE_STREAM_M 1u        /* Philox stream for the LM-head m draw         */

/* ------------------------------------------------------------------------- */
/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As   */
/* Easy as 1, 2, 3", SC'11).  A counter of four 32-bit words and a key of two */
/* words go through ten rounds.  Each round multiplies words 0 and 2 by the   */
/* two round multipliers into 64-bit products; the new words are             */
/*   (hi(M1*x2) ^ x1 ^ k0,  lo(M1*x2),  hi(M0*x0) ^ x3 ^ k1,  lo(M0*x0))       */
/* and the key is bumped by the two Weyl constants between rounds.           */
/* ------------------------------------------------------------------------- */
#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u     /* golden ratio */
#define PHILOX_W1 0xBB67AE85u     /* sqrt(3) - 1  */

void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += PHILOX_W0;
            k1 += PHILOX_W1;
        }
        uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)x0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)x2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t y0 = hi1 ^ x1 ^ k0;
        uint32_t y1 = lo1;
        uint32_t y2 = hi0 ^ x3 ^ k1;
        uint32_t y3 = lo0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* The draw for element e of tensor `tensor_id` at step t on a stream:
 * key = (seed low word, seed high word); counter = (e/4 low, e/4 high, t low
 * word, 2*tensor_id + stream); word e%4 of the output.  The pages are silent
 * on the generator; this keying makes every draw a pure function of
 * (seed, step, tensor, element), so results do not depend on how the work is
 * split. */
uint32_t oracle_draw_word(uint64_t seed, int64_t t, uint32_t tensor_id, uint32_t stream, uint64_t e)
{
    uint64_t quad = e >> 2;
    uint32_t ctr[4] = {(uint32_t)quad, (uint32_t)(quad >> 32), (uint32_t)t,
                       tensor_id * 2u + stream};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    oracle_philox4x32_10(ctr, key, out);
    return out[e & 3u];
}

/* Uniform in [0,1) with 2^-23 granularity: the low 23 bits of the word,
 * scaled by 2^-23 (exact in binary32).  The LM-head first-moment draw and
 * the state-space variants use it. */
float oracle_uniform(uint32_t word)
{
    return (float)(word & 0x7FFFFFu) * 0x1p-23f;
}

/* Uniform in [0,1] from the whole 32-bit word, for the ZIP-SR decision: the
 * word rounded to the nearest binary32, times 2^-32 (exact).  Small words are
 * exact (granularity 2^-32 near zero, where the cell next to zero needs it);
 * above 2^24 the rounding is relative, 2^-24.  So the keep probability
 * p = [h(v)-h(b)]/[h(a)-h(b)] of "ZIP-SR / ZE-EDEN" (Core equation) is
 * realised to within 2^-32 + 2^-23 p, and E[h] to within
 * 2^-32 (h(a)-h(b)) + 2^-23 h(v): unbiased in preconditioner space at the
 * binary32 level, also where h(a) = 1/eps is large ("ZIP-SR 4-bit AdamW --
 * Preconditioner-space stochastic rounding", car / stochastic rounding
 * paragraph: the average multiplier is exact at storage time). */
float oracle_uniform32(uint32_t word)
{
    return (float)word * 0x1p-32f;
}

/* ------------------------------------------------------------------------- */
/* NF4 first-moment codebook [K, Two Complementary Technical Approaches;     */
/* L, ZE-EDEN paragraph].  The pages name NF4 without listing its values.    */
/* NF4 (Dettmers et al., QLoRA, 2023) takes standard-normal quantiles: eight */
/* positive levels at probabilities offset + i*(1/2-offset)/8, i=0..7, seven */
/* negative levels at -quantile(offset + i*(1/2-offset)/7), i=0..6, plus an  */
/* exact zero, all divided by the largest, with offset = 0.9677083.  Here    */
/* the quantile is found by bisection on the upper tail 0.5*erfc(x/sqrt2)    */
/* in binary64, and each normalised level is rounded to binary32 once.       */
/* ------------------------------------------------------------------------- */
static double upper_tail(double x) { return 0.5 * erfc(x * 0.70710678118654752440); }

/* x >= 0 with upper_tail(x) == q (q in (0, 1/2]). */
static double normal_quantile_upper(double q)
{
    double lo = 0.0, hi = 40.0;
    for (int it = 0; it < 2000; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;
        if (upper_tail(mid) > q) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
}

void oracle_nf4_levels_f64(double out[16])
{
    const double offset = 0.9677083;
    double pos[8], neg[7];
    for (int i = 0; i < 8; ++i) {
        double p = offset + (double)i * ((0.5 - offset) / 8.0);
        pos[i] = normal_quantile_upper(1.0 - p);
    }
    for (int i = 0; i < 7; ++i) {
        double p = offset + (double)i * ((0.5 - offset) / 7.0);
        neg[i] = -normal_quantile_upper(1.0 - p);
    }
    double top = pos[0];
    /* ascending: the negatives from most negative, zero, the positives from smallest */
    for (int i = 0; i < 7; ++i) out[i] = neg[i] / top;
    out[7] = 0.0;
    for (int i = 0; i < 8; ++i) out[8 + i] = pos[7 - i] / top;
}

static float g_nf4[16];       /* NF4 levels, ascending, binary32              */
static float g_nf4_mid[15];   /* rounding thresholds between adjacent levels  */
static float g_vz[16];        /* ZIP-SR v code points k/15                    */
static float g_vz_sqrt[16];   /* sqrt of the ZIP-SR code points              */
static float g_vz_mid[15];    /* nearest-point thresholds of the k/15 code     */
static int g_tables_ready = 0;

static void build_tables(void)
{
    if (g_tables_ready) return;
    double lv[16];
    oracle_nf4_levels_f64(lv);
    for (int j = 0; j < 16; ++j) g_nf4[j] = (float)lv[j];
    /* Midpoint of two binary32 levels: exact in binary64, rounded once. */
    for (int j = 0; j < 15; ++j)
        g_nf4_mid[j] = (float)(((double)g_nf4[j] + (double)g_nf4[j + 1]) * 0.5);
    for (int k = 0; k < 16; ++k) {
        g_vz[k] = (float)k / 15.0f;          /* correctly rounded k/15 */
        g_vz_sqrt[k] = sqrtf(g_vz[k]);       /* correctly rounded sqrt  */
    }
    for (int k = 0; k < 15; ++k)
        g_vz_mid[k] = (float)(((double)g_vz[k] + (double)g_vz[k + 1]) * 0.5);
    g_tables_ready = 1;
}

void oracle_tables(float nf4[16], float nf4_mid[15], float vz[16], float vz_sqrt[16])
{
    build_tables();
    memcpy(nf4, g_nf4, sizeof g_nf4);
    memcpy(nf4_mid, g_nf4_mid, sizeof g_nf4_mid);
    memcpy(vz, g_vz, sizeof g_vz);
    memcpy(vz_sqrt, g_vz_sqrt, sizeof g_vz_sqrt);
}

/* ------------------------------------------------------------------------- */
/* Step scalars.  AdamW with decoupled weight decay [K, AdamW and optimizer   */
/* states; L, car paragraph]: w <- w(1 - lr*wd) - lr/(1-b1^t) * m/(sqrt(v)   */
/* /sqrt(1-b2^t) + eps).  The bias correction of v sits inside h(v) exactly  */
/* as in [D, Core equation].                                                 */
/* ------------------------------------------------------------------------- */
typedef struct {
    float step_size;   /* lr / (1 - b1^t)            */
    float rs_bc2;      /* 1 / sqrt(1 - b2^t)         */
    float b1, omb1;    /* b1 and 1 - b1              */
    float b2, omb2;    /* b2 and 1 - b2              */
    float eps;
    float lr;
    int64_t t;         /* 1-based step               */
    uint64_t seed;
    int lm_sr_active;  /* final-10% phase is on      */
} oracle_scalars;

void oracle_make_scalars(float lr, float beta1, float beta2, float eps, int64_t t,
                         int64_t total_steps, uint64_t seed, oracle_scalars *s)
{
    double bc1 = 1.0 - pow((double)beta1, (double)t);
    double bc2 = 1.0 - pow((double)beta2, (double)t);
    s->step_size = (float)((double)lr / bc1);
    s->rs_bc2 = (float)(1.0 / sqrt(bc2));
    s->b1 = beta1;
    s->omb1 = (float)(1.0 - (double)beta1);
    s->b2 = beta2;
    s->omb2 = (float)(1.0 - (double)beta2);
    s->eps = eps;
    s->lr = lr;
    s->t = t;
    s->seed = seed;
    /* "final 10% of training" [Z, Summary; K, Two Complementary Technical
     * Approaches]: the step is in the last tenth when 10*t > 9*T. */
    s->lm_sr_active = (total_steps > 0) && (10 * t > 9 * total_steps);
}

float oracle_decay(float lr, float weight_decay)
{
    return (float)(1.0 - (double)lr * (double)weight_decay);
}

static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Storage of bf16 weights (the library's lower-memory option; the pages keep
 * fp32 weights).  binary32 -> bf16 rounded to nearest, ties to even, the IEEE
 * 754 rounding: keep the top 16 bits after adding 0x7FFF plus the lowest kept
 * bit, so that a value exactly halfway moves to the even neighbour and
 * anything above halfway carries into the kept bits (an overflow of the
 * largest finite values carries into the infinity pattern, as rounding must).
 * A NaN stays a NaN. */
uint16_t oracle_f32_to_bf16(float x)
{
    uint32_t b;
    memcpy(&b, &x, 4);
    if ((b & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((b >> 16) | 0x0040u);
    b += 0x7FFFu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}

void oracle_round_bf16(const float *x, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16(x[i]);
}

static int nibble(const uint8_t *codes, int i)
{
    return (i & 1) ? (codes[i >> 1] >> 4) : (codes[i >> 1] & 15);
}

static void set_nibble(uint8_t *codes, int i, int c)
{
    if (i & 1) codes[i >> 1] = (uint8_t)((codes[i >> 1] & 0x0F) | (c << 4));
    else codes[i >> 1] = (uint8_t)((codes[i >> 1] & 0xF0) | c);
}

/* ------------------------------------------------------------------------- */
/* Per-element moment and weight update, on decoded moments m0, v0            */
/* [D, Method flowchart: "Update working moments" then "Update weights";     */
/*  D, Core equation: weights are updated before the moments are quantised]. */
/* Returns den = sqrt(v1)*rs_bc2 + eps, i.e. 1/h(v1).                        */
/* ------------------------------------------------------------------------- */
float oracle_update_elem(const oracle_scalars *s, float decay, float g, float m0, float v0,
                         float *w, float *m1_out, float *v1_out)
{
    float m1 = fmaf(s->b1, m0, s->omb1 * g);
    float v1 = fmaf(s->b2, v0, s->omb2 * (g * g));
    float den = fmaf(sqrtf(v1), s->rs_bc2, s->eps);
    float w1 = *w * decay;
    *w = fmaf(-s->step_size, m1 / den, w1);
    *m1_out = m1;
    *v1_out = v1;
    return den;
}

/* ------------------------------------------------------------------------- */
/* Quantisers.                                                                */
/* ------------------------------------------------------------------------- */

/* NF4 round-to-nearest: the count of thresholds strictly below x. */
int oracle_nf4_rtn(float x)
{
    build_tables();
    int c = 0;
    for (int j = 0; j < 15; ++j)
        if (x > g_nf4_mid[j]) ++c;
    return c;
}

/* State-space stochastic rounding on the NF4 grid for the LM-head first
 * moment [K, Stochastic rounding; L, ZE-EDEN paragraph]: x between levels a
 * and b goes to a with probability (b - x)/(b - a). */
int oracle_nf4_sr(float x, float u)
{
    build_tables();
    int j = 0;
    for (int i = 1; i <= 14; ++i)
        if (g_nf4[i] <= x) j = i;
    float gap = g_nf4[j + 1] - g_nf4[j];
    int lower = (u * gap) < (g_nf4[j + 1] - x);
    return lower ? j : j + 1;
}

/* ZIP-SR bracket: the k in [0,14] with vz[k] <= x < vz[k+1], or 14 if x is at
 * or above vz[14]. */
int oracle_zipsr_bracket(float x)
{
    build_tables();
    int k = 0;
    for (int i = 1; i <= 14; ++i)
        if (g_vz[i] <= x) k = i;
    return k;
}

/* Zero-inclusive code, state-space round-to-nearest: the count of the
 * binary32 midpoints between adjacent code points strictly below x (a value
 * exactly on a midpoint goes low). */
int oracle_zi_rtn(float x)
{
    build_tables();
    int c = 0;
    for (int k = 0; k < 15; ++k)
        if (x > g_vz_mid[k]) ++c;
    return c;
}

/* Zero-inclusive code, state-space stochastic rounding [K, Stochastic
 * rounding]: x in the bracket [a, b] goes to a with probability
 * (b - x)/(b - a), i.e. when u*(b - a) < b - x. */
int oracle_zi_sr(float x, float u)
{
    build_tables();
    int k = oracle_zipsr_bracket(x);
    int lower = (u * (g_vz[k + 1] - g_vz[k])) < (g_vz[k + 1] - x);
    return lower ? k : k + 1;
}

/* ZIP-SR decision for one element [D, Core equation]: the lower code point a
 * is kept with probability [h(v)-h(b)]/[h(a)-h(b)], h(y) = 1/(sqrt(y)*rs_bc2
 * + eps).  With d = 1/h this is (db - dv)*da / ((db - da)*dv); the element
 * goes low when u*((db-da)*dv) < (db-dv)*da, u = oracle_uniform32(word).  x = v/s, dv = 1/h(v) as used in
 * the weight update, R = sqrt(s)*rs_bc2, so d at code point k is
 * sqrt(k/15)*R + eps.  If da == db in binary32 (h flat across the cell) the
 * preconditioner is the same either way and the rule falls back to state
 * space, which keeps v unbiased. */
int oracle_zipsr_decide(float x, float dv, float R, float eps, float u)
{
    build_tables();
    int k = oracle_zipsr_bracket(x);
    float da = fmaf(g_vz_sqrt[k], R, eps);
    float db = fmaf(g_vz_sqrt[k + 1], R, eps);
    int lower;
    if (da == db) {
        return oracle_zi_sr(x, u);
    } else {
        float lhs = u * ((db - da) * dv);
        float rhs = (db - dv) * da;
        lower = lhs < rhs;
    }
    return lower ? k : k + 1;
}

/* The same decision taken on the whole 32-bit word w of the draw: with
 * u = w 2^-32 (exact in binary64), the element goes low when the binary64
 * product u * B, rounded once, is below rhs, where B = (db-da)*dv and
 * rhs = (db-dv)*da are the binary32 values above (exact in binary64).  P(low)
 * is then p rounded up to a multiple of 2^-32 instead of 2^-23.  The flat-h
 * fallback takes its state-space rule in the same way. */
int oracle_zipsr_decide_u32(float x, float dv, float R, float eps, uint32_t w)
{
    build_tables();
    int k = oracle_zipsr_bracket(x);
    float da = fmaf(g_vz_sqrt[k], R, eps);
    float db = fmaf(g_vz_sqrt[k + 1], R, eps);
    double u = (double)w * 0x1p-32;
    int lower;
    if (da == db) {
        lower = u * (double)(g_vz[k + 1] - g_vz[k]) < (double)(g_vz[k + 1] - x);
    } else {
        float B = (db - da) * dv;
        float rhs = (db - dv) * da;
        lower = u * (double)B < (double)rhs;
    }
    return lower ? k : k + 1;
}

/* ZE-EDEN nearest zero-excluded code point (k+1)/16, ties to even on 16x. */
int oracle_zeeden_code(float x)
{
    float c = rintf(x * 16.0f);
    int k = (int)c - 1;
    if (k < 0) k = 0;
    if (k > 15) k = 15;
    return k;
}

/* Balanced pairwise sum of a[0..n) in index order (n a power of two). */
static float tree_sum(const float *a, int n)
{
    if (n == 1) return a[0];
    return tree_sum(a, n / 2) + tree_sum(a + n / 2, n / 2);
}

/* ZE-EDEN block scale factor [D, Core equation]: ||x||^2 / max(<x,Q(x)>,
 * 1e-12*s^2), evaluated on the normalised block x/s where s^2 cancels, so
 * the floor becomes 1e-12.  Sums run over a balanced pairwise tree of the
 * 128 slots with empty slots contributing zero. */
float oracle_zeeden_factor(const float *xx, const float *xq)
{
    float sxx = tree_sum(xx, ORACLE_BLOCK);
    float sxq = tree_sum(xq, ORACLE_BLOCK);
    return sxx / fmaxf(sxq, 1e-12f);
}

/* ------------------------------------------------------------------------- */
/* One 128-value block of a 4-bit tensor, one step                            */
/* [D, Method flowchart]: decode prior moments -> update working moments ->   */
/* update weights -> ZIP-SR or ZE-EDEN -> pack 4-bit persistent state.        */
/*   w, g        : the block's nvalid weights (in/out) and bf16 gradients     */
/*   mcodes/vcodes: 64 bytes each, element 2i in the low nibble of byte i,    */
/*                  element 2i+1 in the high nibble [D, Local reproduction]   */
/*   mscale/vscale: one binary32 scale per block [L, memory paragraph]        */
/*   elem0       : index of the block's first element within its tensor       */
/* ------------------------------------------------------------------------- */
void oracle_block4(const oracle_scalars *s, float decay, int vcode, int m_sr, uint32_t tensor_id,
                   uint64_t elem0, int nvalid, float *w, const uint16_t *g, uint8_t *mcodes,
                   float *mscale, uint8_t *vcodes, float *vscale)
{
    build_tables();
    float m1[ORACLE_BLOCK], v1[ORACLE_BLOCK], den[ORACLE_BLOCK];

    /* Decode, moment update, weight update. */
    float sm = *mscale, sv = *vscale;
    for (int i = 0; i < nvalid; ++i) {
        float m0 = g_nf4[nibble(mcodes, i)] * sm;
        int cv = nibble(vcodes, i);
        int zero_excluded = (vcode == ORACLE_VCODE_ZEEDEN || vcode == ORACLE_VCODE_ZE_FLOOR);
        float v0 = zero_excluded ? ((float)(cv + 1) * 0.0625f) * sv : g_vz[cv] * sv;
        den[i] = oracle_update_elem(s, decay, bf16_to_f32(g[i]), m0, v0, &w[i], &m1[i], &v1[i]);
    }
    memset(mcodes, 0, ORACLE_BLOCK / 2);
    memset(vcodes, 0, ORACLE_BLOCK / 2);

    /* First moment: absmax scale, NF4 codes. */
    float am = 0.0f;
    for (int i = 0; i < nvalid; ++i) am = fmaxf(am, fabsf(m1[i]));
    if (am < FLT_MIN) {           /* all-zero (or sub-normal) block: zero bytes */
        *mscale = 0.0f;
    } else {
        float inv = 1.0f / am;
        for (int i = 0; i < nvalid; ++i) {
            float x = m1[i] * inv;
            int c;
            if (m_sr) {
                float u = oracle_uniform(oracle_draw_word(s->seed, s->t, tensor_id, ORACLE_STREAM_M,
                                                          elem0 + (uint64_t)i));
                c = oracle_nf4_sr(x, u);
            } else {
                c = oracle_nf4_rtn(x);
            }
            set_nibble(mcodes, i, c);
        }
        *mscale = am;
    }

    /* Second moment: max scale, then ZIP-SR, ZE-EDEN or a state-space variant. */
    float av = 0.0f;
    for (int i = 0; i < nvalid; ++i) av = fmaxf(av, v1[i]);
    if (av < FLT_MIN) {
        *vscale = 0.0f;
        return;
    }
    float inv = 1.0f / av;
    if (vcode == ORACLE_VCODE_ZIPSR || vcode == ORACLE_VCODE_ZIPSR_U32) {
        float R = sqrtf(av) * s->rs_bc2;
        for (int i = 0; i < nvalid; ++i) {
            float x = v1[i] * inv;
            uint32_t w = oracle_draw_word(s->seed, s->t, tensor_id, ORACLE_STREAM_V,
                                          elem0 + (uint64_t)i);
            int c = (vcode == ORACLE_VCODE_ZIPSR)
                        ? oracle_zipsr_decide(x, den[i], R, s->eps, oracle_uniform32(w))
                        : oracle_zipsr_decide_u32(x, den[i], R, s->eps, w);
            set_nibble(vcodes, i, c);
        }
        *vscale = av;
    } else if (vcode == ORACLE_VCODE_ZI_RTN || vcode == ORACLE_VCODE_ZI_SR) {
        for (int i = 0; i < nvalid; ++i) {
            float x = v1[i] * inv;
            int c;
            if (vcode == ORACLE_VCODE_ZI_RTN) {
                c = oracle_zi_rtn(x);
            } else {
                float u = oracle_uniform(oracle_draw_word(s->seed, s->t, tensor_id,
                                                          ORACLE_STREAM_V, elem0 + (uint64_t)i));
                c = oracle_zi_sr(x, u);
            }
            set_nibble(vcodes, i, c);
        }
        *vscale = av;
    } else if (vcode == ORACLE_VCODE_ZE_FLOOR) {
        for (int i = 0; i < nvalid; ++i) set_nibble(vcodes, i, oracle_zeeden_code(v1[i] * inv));
        *vscale = av;
    } else {
        float xx[ORACLE_BLOCK], xq[ORACLE_BLOCK];
        for (int i = 0; i < ORACLE_BLOCK; ++i) { xx[i] = 0.0f; xq[i] = 0.0f; }
        for (int i = 0; i < nvalid; ++i) {
            float x = v1[i] * inv;
            int k = oracle_zeeden_code(x);
            float q = (float)(k + 1) * 0.0625f;
            xx[i] = x * x;
            xq[i] = x * q;
            set_nibble(vcodes, i, k);
        }
        *vscale = av * oracle_zeeden_factor(xx, xq);
    }
}

/* A whole 4-bit tensor, block by block.  Blocks are independent and every
 * draw is keyed by its element, so the optional threads change nothing but
 * the wall time. */
void oracle_step_tensor4(const oracle_scalars *s, float weight_decay, int vcode, int m_sr,
                         uint32_t tensor_id, int64_t numel, float *w, const uint16_t *g,
                         uint8_t *mcodes, float *mscale, uint8_t *vcodes, float *vscale,
                         int nthreads)
{
    float decay = oracle_decay(s->lr, weight_decay);
    int64_t nb = (numel + ORACLE_BLOCK - 1) / ORACLE_BLOCK;
    (void)nthreads;
#ifdef _OPENMP
#pragma omp parallel for schedule(static) num_threads(nthreads > 0 ? nthreads : 1)
#endif
    for (int64_t b = 0; b < nb; ++b) {
        int64_t e0 = b * ORACLE_BLOCK;
        int nvalid = (int)((numel - e0) < ORACLE_BLOCK ? (numel - e0) : ORACLE_BLOCK);
        oracle_block4(s, decay, vcode, m_sr, tensor_id, (uint64_t)e0, nvalid, w + e0, g + e0,
                      mcodes + b * (ORACLE_BLOCK / 2), mscale + b, vcodes + b * (ORACLE_BLOCK / 2),
                      vscale + b);
    }
}

/* A selected list of blocks of one 4-bit tensor, each given as its own
 * buffers (used for sampled checks of full-size runs). */
void oracle_step_blocks4(const oracle_scalars *s, float weight_decay, int vcode, int m_sr,
                         uint32_t tensor_id, int64_t numel, int64_t nsel, const int64_t *blocks,
                         float *w, const uint16_t *g, uint8_t *mcodes, float *mscale,
                         uint8_t *vcodes, float *vscale)
{
    float decay = oracle_decay(s->lr, weight_decay);
    for (int64_t j = 0; j < nsel; ++j) {
        int64_t e0 = blocks[j] * ORACLE_BLOCK;
        int nvalid = (int)((numel - e0) < ORACLE_BLOCK ? (numel - e0) : ORACLE_BLOCK);
        oracle_block4(s, decay, vcode, m_sr, tensor_id, (uint64_t)e0, nvalid,
                      w + j * ORACLE_BLOCK, g + j * ORACLE_BLOCK, mcodes + j * (ORACLE_BLOCK / 2),
                      mscale + j, vcodes + j * (ORACLE_BLOCK / 2), vscale + j);
    }
}

/* fp32-state AdamW for the tensors kept in fp32: normalisation layers and
 * tensors under 4096 elements [L, memory paragraph; D, Local reproduction]. */
void oracle_step_fp32(const oracle_scalars *s, float weight_decay, int64_t numel, float *w,
                      const uint16_t *g, float *m, float *v)
{
    float decay = oracle_decay(s->lr, weight_decay);
    for (int64_t i = 0; i < numel; ++i) {
        float m1, v1;
        oracle_update_elem(s, decay, bf16_to_f32(g[i]), m[i], v[i], &w[i], &m1, &v1);
        m[i] = m1;
        v[i] = v1;
    }
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
