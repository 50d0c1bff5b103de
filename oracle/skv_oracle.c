/*
 * skv_oracle.c -- plain, slow CPU oracle for the Spherical KV (ADA + RDR)
 * paged decode path.
 *
 * TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py load this library.  The product
 * path (long_context_decode_ada_b200/) never links, imports or calls it, and
 * it shares no code, header, table or constant generator with csrc/.
 *
 * What it follows (citations are to the pages about arXiv 2605.18856,
 * "SPHERICAL KV: Angle-Domain Attention and Rate-Distortion Retention for
 * Efficient Long-Context Inference"):
 *   [TS 2.1]  gist.science Technical Summary, section 2.1 Angle-Domain
 *             Attention: key = scalar radius r = |k| + direction angles;
 *             stored as quantised radius r~ and packed angle codes c_theta;
 *             logit l^ ~ |q| r~ f_b(c_theta) computed from the codes;
 *             no dense key is ever materialised.
 *   [TS 2.2]  same page, section 2.2 Rate-Distortion Retention: per state i a
 *             residency z_i and a precision tier b_i under a fixed budget;
 *             distortion surrogate dominated by angular error scaled by the
 *             query and key magnitudes; protected states kept at the top tier;
 *             tier-homogeneous pages read in a single header-guided pass.
 *   [TS 2.3]  same page, section 2.3 System Integration: dense keys ->
 *             spherical codes -> RDR filter/tier -> compressed paged store ->
 *             decode kernel consuming the codes.
 *   [ABS]     arXiv abstract (fugumt.com listing): keep/drop and precision
 *             tiers per token and head under a fixed budget; tier-homogeneous
 *             pages with lightweight metadata.
 * The pages fix none of the numeric details; the concrete scheme below
 * (fp16 radius, per-pair uniform angle code, 2-bit share code, int8 V with a
 * per-token absmax scale, tiers T0/T1/T2/drop) is the pinned reading, and
 * every choice the pages leave open is marked READING.
 *
 * Arithmetic rules: fp64 wherever floating point does not decide a stored
 * integer; integer decisions (codes) are taken in exact integer arithmetic or
 * in exactly-signed fp64 tests; the V quantiser and the RDR slope keys are
 * integer decisions taken in IEEE fp32, the precision the kernels use.
 * Compile with -ffp-contract=off (no fused multiply-add) and no fast-math.
 *
 * Parity pins: every exported function is exercised by tests/test_oracle_*.py
 * against closed forms, brute force, invariants or an independent textbook
 * computation.  Nothing in this file is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <pthread.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_BUDGET 2
#define ORC_ERR_POOL 3

#define TIER_T0 0
#define TIER_T1 1
#define TIER_T2 2
#define TIER_DROP 3

#define PAGE_MAGIC 0x5A
#define HDR_BYTES 16
#define BITS_T1 6
#define BITS_T2 4

typedef unsigned __int128 u128;

/* ------------------------------------------------------------------ */
/* fp16 / bf16 handling, written from the IEEE 754 binary16 definition */
/* ------------------------------------------------------------------ */

/* exact value of an fp16 bit pattern (finite inputs only) */
static double h2d(uint16_t h) {
    int s = h >> 15, e = (h >> 10) & 31, f = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)f, -24);
    else v = ldexp((double)(1024 + f), e - 25);
    return s ? -v : v;
}

/* bf16 bit pattern -> exact value */
static double bf2d(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* fp16 bit pattern -> the bf16 bit pattern of its value rounded to 8
   significant bits, ties to even.  Every finite fp16 value lies inside the
   normal range of bf16 (2^-126 .. 2^128), so only the significand rounds:
   x = m 2^e with m in [2^7, 2^8) after scaling, m rounded to an integer by
   nearbyint (the default rounding mode is to nearest, ties to even), then
   the fields of the result are formed from the rounded m and e. */
static uint16_t h2bf(uint16_t h) {
    double x = h2d(h);
    uint16_t sign = (h & 0x8000) ? 0x8000 : 0;
    if (x < 0) x = -x;
    if (x == 0) return sign;
    int ex;
    frexp(x, &ex);                         /* x in [2^(ex-1), 2^ex) */
    double m = nearbyint(ldexp(x, 8 - ex)); /* in [2^7, 2^8] */
    if (m == 256.0) { m = 128.0; ex += 1; }
    int E = ex - 1 + 127;                  /* biased exponent of 2^(ex-1) */
    return sign | (uint16_t)(E << 7) | (uint16_t)((int)m - 128);
}

/* T0 storage format (process state, tests only: orc_set_t0_bf16): 0 keeps
   the fp16 K and V of a T0 token as they are; 1 stores them as bf16 (each
   component rounded by h2bf), the format of the fused T0 / bf16 decode
   path, read back exactly as bf16. */
static int g_t0_bf16 = 0;
void orc_set_t0_bf16(int on) { g_t0_bf16 = on ? 1 : 0; }
int orc_t0_bf16(void) { return g_t0_bf16; }

/* value of a T0 component as the store holds it */
static double t0_val(uint16_t h) { return g_t0_bf16 ? bf2d(h2bf(h)) : h2d(h); }

/* fp16 value as an integer multiple of 2^-24: value = m * 2^-24, |m| < 2^41 */
static int64_t h2m(uint16_t h) {
    int s = h >> 15, e = (h >> 10) & 31, f = h & 1023;
    int64_t m = (e == 0) ? (int64_t)f : ((int64_t)(1024 + f) << (e - 1));
    return s ? -m : m;
}

/* double -> fp16, one rounding to nearest-even; |x| beyond the fp16 range
   gives +-inf (callers saturate first where the reading says so) */
static uint16_t d2h(double x) {
    uint16_t sign = 0;
    if (x < 0) { sign = 0x8000; x = -x; }
    if (x == 0) return sign;
    if (x < ldexp(1.0, -14)) {                      /* subnormal range */
        double q = nearbyint(ldexp(x, 24));          /* ties to even */
        return sign | (uint16_t)q;                   /* q == 1024 is the smallest normal */
    }
    int ex;
    frexp(x, &ex);                                   /* x in [2^(ex-1), 2^ex) */
    int E = ex - 1;
    double q = nearbyint(ldexp(x, 10 - E));          /* in [1024, 2048] */
    if (q >= 2048) { q = 1024; E += 1; }
    if (E > 15) return sign | 0x7C00;
    return sign | (uint16_t)(((E + 15) << 10) | ((int)q - 1024));
}

/* ------------------------------------------------------------------ */
/* Tables: angle boundaries, share levels, distortion and slope constants */
/* ------------------------------------------------------------------ */

/* Boundary unit vectors between angle codes j and j+1 for a b-bit uniform
   angle quantiser: beta_j = (j + 1/2) * 2*pi / 2^b, rounded to fp32 from
   double cos/sin.  READING: the pages give no rounding rule for the angle
   code; the sector test against these fp32 vectors is the definition of the
   code (it agrees with round(atan2/delta) away from the boundaries). */
static float *g_bx[17], *g_by[17];
static pthread_once_t g_once = PTHREAD_ONCE_INIT;

static void build_tables(void) {
    for (int b = 2; b <= 16; b++) {
        int n = 1 << b;
        g_bx[b] = (float*)malloc(sizeof(float) * n);
        g_by[b] = (float*)malloc(sizeof(float) * n);
        for (int j = 0; j < n; j++) {
            double beta = (j + 0.5) * (2.0 * M_PI / n);
            g_bx[b][j] = (float)cos(beta);
            g_by[b][j] = (float)sin(beta);
        }
    }
}

static void init_once(void) { pthread_once(&g_once, build_tables); }

void orc_boundaries(int b, float* bx, float* by) {
    init_once();
    int n = 1 << b;
    memcpy(bx, g_bx[b], sizeof(float) * n);
    memcpy(by, g_by[b], sizeof(float) * n);
}

/* Share grid.  READING (the pinned scheme says only "2-bit code on a fixed
   grid"): u = (rho_i / r) * sqrt(d/2) is quantised to the levels
   {0.5, 1.0, 1.5, 2.0} with thresholds {0.75, 1.25, 1.75}; the decoded share
   is rho^_i = u_level / sqrt(d/2).
   The non-uniform variant (share grid 1, set per process by
   orc_set_share_grid; tests only) is the Lloyd-Max grid of the Rayleigh
   density that u follows for Gaussian keys, made exact: levels
   {383, 807, 1249, 1831} / 1024 and thresholds sqrt({22, 64, 145} / 64),
   the nearest such values to the optimum (levels 0.3743, 0.7880, 1.2195,
   1.7884; thresholds 0.5811, 1.0037, 1.5039). */
static int g_share_grid = 0;

void orc_set_share_grid(int grid) { g_share_grid = grid ? 1 : 0; }
int orc_share_grid(void) { return g_share_grid; }

double orc_rho_level(int code, int d) {
    static const double U[4] = {0.5, 1.0, 1.5, 2.0};
    static const double LM[4] = {383.0 / 1024, 807.0 / 1024, 1249.0 / 1024, 1831.0 / 1024};
    return (g_share_grid ? LM[code & 3] : U[code & 3]) / sqrt(d / 2.0);
}

/* Relative distortion of each tier, c(tier), for the RDR surrogate [TS 2.2]:
   the expected squared logit error of a tier divided by the expected squared
   logit (the error of dropping the token).  For a b-bit uniform angle
   quantiser with the error eps ~ U[-delta/2, delta/2] and the query uniform
   in direction relative to each pair, E[(cos(phi+eps) - cos phi)^2] /
   E[cos^2 phi] = 2 (1 - sin(delta/2) / (delta/2)).  READING: squared error;
   the share quantisation is ignored, as the pages call the angular error
   dominant.  c(T0) = 0 (dense), c(drop) = 1. */
static double c_angle(int b) {
    double x = M_PI / (double)(1 << b);              /* delta / 2 */
    return 2.0 * (1.0 - sin(x) / x);
}

void orc_distortion(double c[4]) {
    c[TIER_T0] = 0.0;
    c[TIER_T1] = c_angle(BITS_T1);
    c[TIER_T2] = c_angle(BITS_T2);
    c[TIER_DROP] = 1.0;
}

/* bytes per (token, kv head) of each tier at head dim d:
   T0 fp16 K + fp16 V; T1 r~ + one code byte per pair + int8 V + fp16 scale;
   T2 r~ + angle nibble + share crumb per pair + int8 V + fp16 scale. */
int64_t orc_tier_bytes(int tier, int d) {
    switch (tier) {
    case TIER_T0: return 4LL * d;
    case TIER_T1: return 2 + d / 2 + d + 2;
    case TIER_T2: return 2 + d / 4 + d / 8 + d + 2;
    default: return 0;
    }
}

/* Slope per byte of each upgrade step of a token (drop->T2, T2->T1,
   T1->T0): the drop in relative distortion divided by the added bytes,
   rounded to fp32.  Multiplied by u * r^2 this is the RDR priority. */
void orc_kappa(int d, float kappa[3]) {
    double c[4];
    orc_distortion(c);
    kappa[0] = (float)((c[TIER_DROP] - c[TIER_T2]) / (double)orc_tier_bytes(TIER_T2, d));
    kappa[1] = (float)((c[TIER_T2] - c[TIER_T1]) /
                       (double)(orc_tier_bytes(TIER_T1, d) - orc_tier_bytes(TIER_T2, d)));
    kappa[2] = (float)((c[TIER_T1] - c[TIER_T0]) /
                       (double)(orc_tier_bytes(TIER_T0, d) - orc_tier_bytes(TIER_T1, d)));
}

/* ------------------------------------------------------------------ */
/* Encode primitives [TS 2.1]                                          */
/* ------------------------------------------------------------------ */

/* R2 = sum_c m_c^2, exactly, where k_c = m_c * 2^-24.  Returned as lo, hi. */
void orc_norm2(const uint16_t* k, int d, uint64_t out[2]) {
    u128 s = 0;
    for (int c = 0; c < d; c++) {
        int64_t m = h2m(k[c]);
        u128 a = (u128)(m < 0 ? -m : m);
        s += a * a;
    }
    out[0] = (uint64_t)s;
    out[1] = (uint64_t)(s >> 64);
}

/* R2 as a double, correctly rounded (nearest, ties to even): above 64
   significant bits, the top 64 bits are kept with the rest folded into a
   sticky lowest bit, which leaves the rounding of the 53-bit result intact. */
static double r2_double(const uint64_t R2[2]) {
    u128 x = ((u128)R2[1] << 64) | R2[0];
    int shift = 0;
    while ((x >> 64) != 0) {
        int sticky = (int)(x & 1);
        x >>= 1;
        x |= (u128)sticky;
        shift++;
    }
    return ldexp((double)(uint64_t)x, shift);
}

/* Quantised radius r~ = fp16(min(r, 65504)) with r = sqrt(R2) * 2^-24:
   one correctly rounded sqrt in double, one rounding to fp16.  READING: fp16
   for r~ comes from the pinned scheme; saturation is this implementation's choice. */
uint16_t orc_rtilde_from_r2(const uint64_t R2[2]) {
    double r = sqrt(r2_double(R2)) * ldexp(1.0, -24);
    if (r > 65504.0) r = 65504.0;
    return d2h(r);
}

uint16_t orc_rtilde(const uint16_t* k, int d) {
    uint64_t R2[2];
    orc_norm2(k, d, R2);
    return orc_rtilde_from_r2(R2);
}

/* b-bit angle code of the pair (x, y): the sector of the quantiser that the
   point lies in, where sector c spans the angles from boundary c-1 to
   boundary c.  The quadrant is read from the signs; within it, the code
   counts the boundaries that the point lies on or counter-clockwise of
   (a point on a rounded boundary takes the higher code); the cross products
   are exact in fp64 (fp32 x fp16 significands), so the signs are exact.
   (0, 0) -> 0.  Plain definition it realises: round(atan2(y,x)/delta) mod 2^b. */
int orc_angle_code(uint16_t xh, uint16_t yh, int b) {
    init_once();
    double x = h2d(xh), y = h2d(yh);
    int n = 1 << b, per = n / 4;
    if (x == 0.0 && y == 0.0) return 0;
    int q;
    if (x > 0 && y >= 0) q = 0;
    else if (x <= 0 && y > 0) q = 1;
    else if (x < 0 && y <= 0) q = 2;
    else q = 3;
    int cnt = 0;
    for (int j = q * per; j < (q + 1) * per; j++) {
        double side = (double)g_bx[b][j] * y - (double)g_by[b][j] * x;
        if (side >= 0.0) cnt++;
    }
    return (q * per + cnt) % n;
}

/* 2-bit share code of the pair (x, y): how many of the thresholds
   u > {0.75, 1.25, 1.75} hold, u = (rho/r) sqrt(d/2).  Exact integer test:
   u > t  <=>  16 (d/2) rho^2 > (4t)^2 R2 with (4t)^2 = 9, 25, 49; a tie
   goes to the lower code.  Share grid 1: 64 (d/2) rho^2 > {22, 64, 145} R2. */
int orc_rho_code(uint16_t xh, uint16_t yh, const uint64_t R2[2], int d) {
    static const unsigned U16[3] = {9, 25, 49}, U64[3] = {22, 64, 145};
    const unsigned* U = g_share_grid ? U64 : U16;
    int64_t mx = h2m(xh), my = h2m(yh);
    u128 ax = (u128)(mx < 0 ? -mx : mx), ay = (u128)(my < 0 ? -my : my);
    u128 rho2 = ax * ax + ay * ay;
    u128 R = ((u128)R2[1] << 64) | R2[0];
    u128 lhs = rho2 * (u128)((g_share_grid ? 64 : 16) * (d / 2));
    int code = 0;
    for (int j = 0; j < 3; j++)
        if (lhs > (u128)U[j] * R) code++;
    return code;
}

/* int8 V with a per-token absmax scale, taken in IEEE fp32:
   s = fp16(absmax|v| / 127), code = clamp(rint(v / s), -127, 127), s == 0
   gives all-zero codes.  READING: symmetric +-127 range, fp16 scale,
   round-half-even. */
void orc_vquant(const uint16_t* v, int d, int8_t* codes, uint16_t* scale) {
    float amax = 0.0f;
    for (int c = 0; c < d; c++) {
        float a = fabsf((float)h2d(v[c]));
        if (a > amax) amax = a;
    }
    float sf = amax / 127.0f;
    uint16_t sh = d2h((double)sf);
    float s = (float)h2d(sh);
    *scale = sh;
    for (int c = 0; c < d; c++) {
        if (s == 0.0f) { codes[c] = 0; continue; }
        float x = (float)h2d(v[c]) / s;
        float r = nearbyintf(x);
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        codes[c] = (int8_t)r;
    }
}

/* ------------------------------------------------------------------ */
/* Decode side: reconstruction and logits                              */
/* ------------------------------------------------------------------ */

/* k^ from the codes of tier b bits: k^_{2i} = r~ rho^_i cos(2 pi c_i / 2^b),
   k^_{2i+1} = r~ rho^_i sin(2 pi c_i / 2^b).  READING: k^ is not
   renormalised to length r~. */
void orc_reconstruct(const uint16_t* k, int d, int b, double* khat) {
    uint64_t R2[2];
    orc_norm2(k, d, R2);
    double rt = h2d(orc_rtilde_from_r2(R2));
    for (int i = 0; i < d / 2; i++) {
        int c = orc_angle_code(k[2 * i], k[2 * i + 1], b);
        int rc = orc_rho_code(k[2 * i], k[2 * i + 1], R2, d);
        double rho = orc_rho_level(rc, d);
        double ang = 2.0 * M_PI * c / (double)(1 << b);
        khat[2 * i] = rt * rho * cos(ang);
        khat[2 * i + 1] = rt * rho * sin(ang);
    }
}

/* The compressed-domain logit [TS 2.1] in the pinned form
   l = (r~ / sqrt(d)) * sum_i rho^_i * LUT_i[c_i],
   LUT_i[c] = q_{2i} cos(2 pi c / 2^b) + q_{2i+1} sin(2 pi c / 2^b). */
double orc_logit_codes(const double* q, const uint16_t* k, int d, int b) {
    uint64_t R2[2];
    orc_norm2(k, d, R2);
    double rt = h2d(orc_rtilde_from_r2(R2));
    double s = 0.0;
    for (int i = 0; i < d / 2; i++) {
        int c = orc_angle_code(k[2 * i], k[2 * i + 1], b);
        int rc = orc_rho_code(k[2 * i], k[2 * i + 1], R2, d);
        double ang = 2.0 * M_PI * c / (double)(1 << b);
        double lut = q[2 * i] * cos(ang) + q[2 * i + 1] * sin(ang);
        s += orc_rho_level(rc, d) * lut;
    }
    return rt / sqrt((double)d) * s;
}

/* T1 code scheme.  0, the pinned scheme: 6-bit angle and a 2-bit share on
   the uniform 4-level grid, code byte (angle << 2) | share.  1, the variant
   the bytes-versus-logit-error study favours at the same 196 bytes: 5-bit
   angle and a 3-bit share on the uniform 8-level grid u in {0.25, 0.5, ..,
   2.0} (thresholds at the midpoints), code byte (angle << 3) | share.  The
   scheme is process state set by orc_set_t1_scheme (tests only); T2 and the
   allocation do not depend on it. */
static int g_t1_scheme = 0;

void orc_set_t1_scheme(int scheme) { g_t1_scheme = scheme ? 1 : 0; }
int orc_t1_scheme(void) { return g_t1_scheme; }

/* 3-bit share code: how many of the thresholds u > (2j + 3) / 8, j < 7,
   hold; exact integer test 64 (d/2) rho^2 > (2j + 3)^2 R2, ties to the
   lower code. */
int orc_rho_code3(uint16_t xh, uint16_t yh, const uint64_t R2[2], int d) {
    int64_t mx = h2m(xh), my = h2m(yh);
    u128 ax = (u128)(mx < 0 ? -mx : mx), ay = (u128)(my < 0 ? -my : my);
    u128 lhs = (ax * ax + ay * ay) * (u128)(64 * (d / 2));
    u128 R = ((u128)R2[1] << 64) | R2[0];
    int code = 0;
    for (int j = 0; j < 7; j++) {
        unsigned t = 2 * j + 3;
        if (lhs > (u128)(t * t) * R) code++;
    }
    return code;
}

double orc_rho_level3(int code, int d) { return 0.25 * ((code & 7) + 1) / sqrt(d / 2.0); }

/* k^ of a token stored in tier T1 or T2, under the current T1 scheme */
void orc_reconstruct_tier(const uint16_t* k, int d, int tier, double* khat) {
    if (tier != TIER_T1 || g_t1_scheme == 0) {
        orc_reconstruct(k, d, tier == TIER_T1 ? BITS_T1 : BITS_T2, khat);
        return;
    }
    uint64_t R2[2];
    orc_norm2(k, d, R2);
    double rt = h2d(orc_rtilde_from_r2(R2));
    for (int i = 0; i < d / 2; i++) {
        int c = orc_angle_code(k[2 * i], k[2 * i + 1], 5);
        double rho = orc_rho_level3(orc_rho_code3(k[2 * i], k[2 * i + 1], R2, d), d);
        double ang = 2.0 * M_PI * c / 32.0;
        khat[2 * i] = rt * rho * cos(ang);
        khat[2 * i + 1] = rt * rho * sin(ang);
    }
}

/* q . k^ / sqrt(d) with k^ reconstructed (the decompress-then-dot form) */
double orc_logit_recon(const double* q, const uint16_t* k, int d, int b) {
    double* kh = (double*)malloc(sizeof(double) * d);
    orc_reconstruct(k, d, b, kh);
    double s = 0.0;
    for (int c = 0; c < d; c++) s += q[c] * kh[c];
    free(kh);
    return s / sqrt((double)d);
}

/* Variant for the convergence pin: b-bit angle codes, exact shares rho_i/r
   (share_mode 0) or 2-bit shares (share_mode 1) or exact angles with 2-bit
   shares (share_mode 2: the limit b -> infinity of mode 1). */
double orc_logit_variant(const double* q, const uint16_t* k, int d, int b, int share_mode) {
    uint64_t R2[2];
    orc_norm2(k, d, R2);
    double rt = h2d(orc_rtilde_from_r2(R2));
    double r = sqrt(r2_double(R2)) * ldexp(1.0, -24);
    double s = 0.0;
    for (int i = 0; i < d / 2; i++) {
        double x = h2d(k[2 * i]), y = h2d(k[2 * i + 1]);
        double share = (r > 0) ? sqrt(x * x + y * y) / r : 0.0;
        double cs, sn;
        if (share_mode == 2) {
            double nrm = sqrt(x * x + y * y);
            cs = nrm > 0 ? x / nrm : 1.0;
            sn = nrm > 0 ? y / nrm : 0.0;
        } else {
            int c = orc_angle_code(k[2 * i], k[2 * i + 1], b);
            double ang = 2.0 * M_PI * c / (double)(1 << b);
            cs = cos(ang);
            sn = sin(ang);
        }
        if (share_mode >= 1) share = orc_rho_level(orc_rho_code(k[2 * i], k[2 * i + 1], R2, d), d);
        s += share * (q[2 * i] * cs + q[2 * i + 1] * sn);
    }
    return rt / sqrt((double)d) * s;
}

/* Tier/grid variant for the bytes-versus-logit-error study: b-bit angle
   codes (the same coder), and the share u = (rho_i / r) sqrt(d/2) quantised
   to L levels: code = the number of thresholds thresh_u[0..L-2] (ascending)
   that u exceeds, decoded share levels_u[code] / sqrt(d/2); L = 0 keeps the
   exact share.  The radius is r~ as in the tiers.  Returns the logit
   (r~ / sqrt d) sum_i rho^_i (q_{2i} cos + q_{2i+1} sin)(2 pi c_i / 2^b). */
double orc_logit_grid(const double* q, const uint16_t* k, int d, int b, int L,
                      const double* levels_u, const double* thresh_u) {
    uint64_t R2[2];
    orc_norm2(k, d, R2);
    double rt = h2d(orc_rtilde_from_r2(R2));
    double r = sqrt(r2_double(R2)) * ldexp(1.0, -24);
    double sq = sqrt(d / 2.0);
    double s = 0.0;
    for (int i = 0; i < d / 2; i++) {
        double x = h2d(k[2 * i]), y = h2d(k[2 * i + 1]);
        double share = (r > 0) ? sqrt(x * x + y * y) / r : 0.0;
        if (L > 0) {
            double u = share * sq;
            int code = 0;
            for (int j = 0; j < L - 1; j++)
                if (u > thresh_u[j]) code++;
            share = levels_u[code] / sq;
        }
        int c = orc_angle_code(k[2 * i], k[2 * i + 1], b);
        double ang = 2.0 * M_PI * c / (double)(1 << b);
        s += share * (q[2 * i] * cos(ang) + q[2 * i + 1] * sin(ang));
    }
    return rt / sqrt((double)d) * s;
}

/* ------------------------------------------------------------------ */
/* RDR allocation [TS 2.2], [ABS]                                      */
/* ------------------------------------------------------------------ */

typedef struct {
    float key;
    int k;      /* step 0: drop->T2, 1: T2->T1, 2: T1->T0 */
    int h;
    int t;
} step_t;

static int step_cmp(const void* a, const void* b) {
    const step_t* x = (const step_t*)a;
    const step_t* y = (const step_t*)b;
    if (x->key != y->key) return x->key > y->key ? -1 : 1;   /* slope descending */
    if (x->k != y->k) return x->k < y->k ? -1 : 1;           /* then step ascending */
    if (x->h != y->h) return x->h < y->h ? -1 : 1;           /* then head ascending */
    if (x->t != y->t) return x->t < y->t ? -1 : 1;           /* then position ascending */
    return 0;
}

typedef struct {
    float u;
    int t;
} rank_t;

static int rank_cmp(const void* a, const void* b) {
    const rank_t* x = (const rank_t*)a;
    const rank_t* y = (const rank_t*)b;
    if (x->u != y->u) return x->u > y->u ? -1 : 1;           /* utility descending */
    return x->t < y->t ? -1 : (x->t > y->t ? 1 : 0);         /* then position ascending */
}

/* r^2 as fp32: fp32(double(R2) * 2^-48) */
static float r2_float(const uint64_t R2[2]) {
    return (float)(r2_double(R2) * ldexp(1.0, -48));
}

/* Tier choice for every (seq, kv head, token).
   mode 1 (budget): the joint keep/drop + tier decision of [TS 2.2] read as a
   greedy walk down the convex rate-distortion hull: each unprotected token
   offers three upgrade steps (drop->T2, T2->T1, T1->T0) whose priority is
   u * r^2 * kappa_step (fp32, left to right); all steps of one sequence
   (shared by its kv heads: "per token and head under a fixed budget",
   [ABS]) are ordered by (priority desc, step asc, head asc, position asc)
   and the longest prefix whose bytes fit the budget is taken.  The budget
   left for that walk is budget - 512 * protected - Hkv*(P-1)*(512+196+180)
   bytes (room for the partial last page of every tier).  Protected tokens
   are T0 ([TS 2.2] protection constraint, b_max = the top tier).
   mode 0 (quota): per (seq, head), protected tokens are T0; the others are
   ranked by (u desc, position asc) (position order when utility is NULL) and
   the first quota[b][0] go to T0, the next quota[b][1] to T1, the next
   quota[b][2] to T2, the rest are dropped.
   Output tier codes: 0 = T0, 1 = T1, 2 = T2, 3 = dropped; positions at or
   beyond seq_lens[b] are marked dropped. */
int orc_allocate(int B, int Hkv, int Tmax, int d, int P, const int32_t* seq_lens,
                 const uint16_t* K, const float* utility, const uint8_t* protect,
                 int mode, const int64_t* budget, const int32_t* quota, uint8_t* tier_out) {
    if (B < 0 || Hkv <= 0 || Tmax < 0 || d <= 0 || P <= 0) return ORC_ERR_ARG;
    if (mode == 1 && !utility) return ORC_ERR_ARG;
    float kappa[3];
    orc_kappa(d, kappa);
    const int64_t step_bytes[3] = {
        orc_tier_bytes(TIER_T2, d),
        orc_tier_bytes(TIER_T1, d) - orc_tier_bytes(TIER_T2, d),
        orc_tier_bytes(TIER_T0, d) - orc_tier_bytes(TIER_T1, d)};
    int err = ORC_OK;
    for (int b = 0; b < B; b++) {
        int T = seq_lens[b];
        if (T < 0 || T > Tmax) return ORC_ERR_ARG;
        for (int h = 0; h < Hkv; h++)
            for (int t = 0; t < Tmax; t++)
                tier_out[((int64_t)b * Hkv + h) * Tmax + t] = TIER_DROP;
        if (mode == 1) {
            int64_t nprot = 0;
            int64_t nsteps = 0;
            for (int h = 0; h < Hkv; h++)
                for (int t = 0; t < T; t++) {
                    int64_t idx = ((int64_t)b * Hkv + h) * Tmax + t;
                    if (protect && protect[idx]) nprot++;
                    else nsteps += 3;
                }
            int64_t left = budget[b] - nprot * orc_tier_bytes(TIER_T0, d) -
                           (int64_t)Hkv * (P - 1) *
                               (orc_tier_bytes(TIER_T0, d) + orc_tier_bytes(TIER_T1, d) +
                                orc_tier_bytes(TIER_T2, d));
            if (left < 0) { err = ORC_ERR_BUDGET; continue; }
            step_t* st = (step_t*)malloc(sizeof(step_t) * (nsteps > 0 ? nsteps : 1));
            int64_t n = 0;
            for (int h = 0; h < Hkv; h++)
                for (int t = 0; t < T; t++) {
                    int64_t idx = ((int64_t)b * Hkv + h) * Tmax + t;
                    if (protect && protect[idx]) { tier_out[idx] = TIER_T0; continue; }
                    uint64_t R2[2];
                    orc_norm2(K + idx * d, d, R2);
                    float w = utility[idx] * r2_float(R2);
                    for (int k = 0; k < 3; k++) {
                        st[n].key = w * kappa[k];
                        st[n].k = k;
                        st[n].h = h;
                        st[n].t = t;
                        n++;
                    }
                }
            qsort(st, n, sizeof(step_t), step_cmp);
            /* level[h][t] = number of steps taken */
            int64_t used = 0;
            for (int64_t i = 0; i < n; i++) {
                if (used + step_bytes[st[i].k] > left) break;
                used += step_bytes[st[i].k];
                int64_t idx = ((int64_t)b * Hkv + st[i].h) * Tmax + st[i].t;
                /* steps of one token come in order k = 0, 1, 2 */
                tier_out[idx] = (uint8_t)(st[i].k == 0 ? TIER_T2 : (st[i].k == 1 ? TIER_T1 : TIER_T0));
            }
            free(st);
        } else {
            rank_t* rk = (rank_t*)malloc(sizeof(rank_t) * (T > 0 ? T : 1));
            for (int h = 0; h < Hkv; h++) {
                int n = 0;
                for (int t = 0; t < T; t++) {
                    int64_t idx = ((int64_t)b * Hkv + h) * Tmax + t;
                    if (protect && protect[idx]) { tier_out[idx] = TIER_T0; continue; }
                    rk[n].u = utility ? utility[idx] : 0.0f;
                    rk[n].t = t;
                    n++;
                }
                qsort(rk, n, sizeof(rank_t), rank_cmp);
                int64_t c0 = quota[b * 3 + 0], c1 = quota[b * 3 + 1], c2 = quota[b * 3 + 2];
                if (c0 < 0 || c1 < 0 || c2 < 0) { free(rk); return ORC_ERR_ARG; }
                for (int i = 0; i < n; i++) {
                    int64_t idx = ((int64_t)b * Hkv + h) * Tmax + rk[i].t;
                    uint8_t tr = TIER_DROP;
                    if (i < c0) tr = TIER_T0;
                    else if (i < c0 + c1) tr = TIER_T1;
                    else if (i < c0 + c1 + c2) tr = TIER_T2;
                    tier_out[idx] = tr;
                }
            }
            free(rk);
        }
    }
    return err;
}

/* Re-tiering of a store's rows under its budget ([TS 2.2] keep/drop and
   tier per token and head under a fixed budget; [TS 2.3] the retention
   filter between the codes and the store, applied again as tokens age out
   of the protected recent window).  Every resident token keeps its tier
   except those marked in `demote`, which must be T0 (rows leaving the
   recent window, whose exact fp16 keys the store still holds): they take
   the greedy walk of orc_allocate's budget mode among themselves, with the
   budget left after the kept tokens' bytes and the partial-page reserve,
   budget - sum(tier bytes of kept tokens) - Hkv*(P-1)*(512+196+180).
   Their steps, keys, ordering and prefix rule are orc_allocate's.  When the
   kept tokens alone exceed that budget the demoted tokens are dropped and
   ORC_ERR_BUDGET is returned (the store is over budget).  A demote flag on
   a token that is not T0, or on a position past the sequence, is
   ORC_ERR_ARG.  Positions at or beyond seq_lens[b] are dropped. */
int orc_retier(int B, int Hkv, int Tmax, int d, int P, const int32_t* seq_lens,
               const uint16_t* K, const float* utility, const uint8_t* tier_in,
               const uint8_t* demote, const int64_t* budget, uint8_t* tier_out) {
    if (B < 0 || Hkv <= 0 || Tmax < 0 || d <= 0 || P <= 0 || !utility) return ORC_ERR_ARG;
    float kappa[3];
    orc_kappa(d, kappa);
    const int64_t step_bytes[3] = {
        orc_tier_bytes(TIER_T2, d),
        orc_tier_bytes(TIER_T1, d) - orc_tier_bytes(TIER_T2, d),
        orc_tier_bytes(TIER_T0, d) - orc_tier_bytes(TIER_T1, d)};
    int err = ORC_OK;
    for (int b = 0; b < B; b++) {
        int T = seq_lens[b];
        if (T < 0 || T > Tmax) return ORC_ERR_ARG;
        int64_t kept = 0, nsteps = 0;
        for (int h = 0; h < Hkv; h++)
            for (int t = 0; t < Tmax; t++) {
                int64_t idx = ((int64_t)b * Hkv + h) * Tmax + t;
                uint8_t tr = t < T ? tier_in[idx] : TIER_DROP;
                if (demote && demote[idx]) {
                    if (t >= T || tr != TIER_T0) return ORC_ERR_ARG;
                    tier_out[idx] = TIER_DROP;
                    nsteps += 3;
                    continue;
                }
                if (tr > TIER_DROP) return ORC_ERR_ARG;
                tier_out[idx] = tr;
                if (tr != TIER_DROP) kept += orc_tier_bytes(tr, d);
            }
        int64_t left = budget[b] - kept -
                       (int64_t)Hkv * (P - 1) *
                           (orc_tier_bytes(TIER_T0, d) + orc_tier_bytes(TIER_T1, d) +
                            orc_tier_bytes(TIER_T2, d));
        if (left < 0) { err = ORC_ERR_BUDGET; continue; }
        step_t* st = (step_t*)malloc(sizeof(step_t) * (nsteps > 0 ? nsteps : 1));
        int64_t n = 0;
        for (int h = 0; h < Hkv; h++)
            for (int t = 0; t < T; t++) {
                int64_t idx = ((int64_t)b * Hkv + h) * Tmax + t;
                if (!(demote && demote[idx])) continue;
                uint64_t R2[2];
                orc_norm2(K + idx * d, d, R2);
                float w = utility[idx] * r2_float(R2);
                for (int k = 0; k < 3; k++) {
                    st[n].key = w * kappa[k];
                    st[n].k = k;
                    st[n].h = h;
                    st[n].t = t;
                    n++;
                }
            }
        qsort(st, n, sizeof(step_t), step_cmp);
        int64_t used = 0;
        for (int64_t i = 0; i < n; i++) {
            if (used + step_bytes[st[i].k] > left) break;
            used += step_bytes[st[i].k];
            int64_t idx = ((int64_t)b * Hkv + st[i].h) * Tmax + st[i].t;
            tier_out[idx] = (uint8_t)(st[i].k == 0 ? TIER_T2 : (st[i].k == 1 ? TIER_T1 : TIER_T0));
        }
        free(st);
    }
    return err;
}

/* ------------------------------------------------------------------ */
/* Paged store [TS 2.2 tier-homogeneous pages], [TS 2.3], [ABS]        */
/* ------------------------------------------------------------------ */
/*
 * Page payload of tier t with P rows (P a multiple of 16), d = 128:
 *   header (16 B, little endian): u16 count | u8 tier | u8 0x5A |
 *                                  u32 seq | u32 kv_head | u32 tier_page
 *   T0: K fp16 [P][128] at 16, then V fp16 at 16 + 256P
 *   T1: r~ fp16 [P] at 16, codes [P][64] at 16+2P, scale fp16 [P] at 16+66P,
 *       V int8 at 16+68P
 *   T2: r~ at 16, codes [P][48] at 16+2P, scale at 16+50P, V int8 at 16+52P
 * Rows at and beyond count are zero.  The slot stride is the payload rounded
 * up to 128 bytes; stride padding is never written.
 * Within-row orders (the decode kernel reads with lane = 4*t + g, t the token
 * in an 8-row group and g one of four pair groups):
 *   T0 K row r: 16 chunks of 8 dims; chunk c at chunk position c ^ (4*(r&1)).
 *   T1 code row r: byte 16*g + j holds pair 16*(j/4) + 4*g + j%4, as
 *       (angle6 << 2) | share2 (lane g then holds the pairs of the dims
 *       that it reads of a T0 row: chunks 4i + g).
 *   T2 code row r: nibble j of bytes [8g, 8g+8) (low nibble first) holds the
 *       4-bit angle of pair 16*(j/4) + 4*g + j%4; crumb j of bytes
 *       [32+4g, 36+4g) (bits 2j..2j+1 of that little-endian word) its share.
 *   V (all tiers), per 8-row group k, m-tile mt (dims 16mt..16mt+15), lane
 *       L = 4*g + t4 (g = 0..7, t4 = 0..3): the four values
 *       (V[8k+2t4][16mt+g], V[8k+2t4+1][16mt+g], V[8k+2t4][16mt+g+8],
 *        V[8k+2t4+1][16mt+g+8]);
 *       int8: group block of 1024 B, the 4 bytes at
 *             512*(mt/4) + 16*L + 4*(mt%4);
 *       fp16: group block of 2048 B, the 8 bytes at
 *             512*(mt/2) + 16*L + 8*(mt%2).
 */

int64_t orc_page_payload(int tier, int P, int d) {
    return HDR_BYTES + (int64_t)P * orc_tier_bytes(tier, d);
}

int64_t orc_page_stride(int tier, int P, int d) {
    int64_t p = orc_page_payload(tier, P, d);
    return (p + 127) / 128 * 128;
}

static void put16(uint8_t* p, uint16_t v) { p[0] = v & 255; p[1] = v >> 8; }
static void put32(uint8_t* p, uint32_t v) {
    p[0] = v & 255; p[1] = (v >> 8) & 255; p[2] = (v >> 16) & 255; p[3] = v >> 24;
}

/* byte offset, within a group block, of V element (row r, dim dd) */
static int64_t v_frag_offset(int r, int dd, int elem_bytes) {
    int k = r / 8, tr = r % 8, t4 = tr / 2, lo = tr % 2;
    int mt = dd / 16, rem = dd % 16, g = rem % 8, hi = rem / 8;
    int L = 4 * g + t4;
    int e = 2 * hi + lo;
    if (elem_bytes == 1)
        return (int64_t)k * 1024 + 512 * (mt / 4) + 16 * L + 4 * (mt % 4) + e;
    return (int64_t)k * 2048 + 512 * (mt / 2) + 16 * L + 8 * (mt % 2) + 2 * e;
}

/* write token row r of a page of tier `tier` from its fp16 K and V */
static void write_row(uint8_t* page, int tier, int P, int d, int r,
                      const uint16_t* k, const uint16_t* v) {
    if (tier == TIER_T0) {
        uint8_t* ks = page + HDR_BYTES;
        uint8_t* vs = page + HDR_BYTES + (int64_t)256 * P;
        for (int dd = 0; dd < d; dd++) {
            int c = dd / 8, e = dd % 8;
            int pos = c ^ (4 * (r & 1));
            put16(ks + (int64_t)r * 256 + pos * 16 + e * 2, g_t0_bf16 ? h2bf(k[dd]) : k[dd]);
            put16(vs + v_frag_offset(r, dd, 2), g_t0_bf16 ? h2bf(v[dd]) : v[dd]);
        }
        return;
    }
    uint64_t R2[2];
    orc_norm2(k, d, R2);
    uint16_t rt = orc_rtilde_from_r2(R2);
    int8_t v8[128];
    uint16_t sc;
    orc_vquant(v, d, v8, &sc);
    int codes_bytes = (tier == TIER_T1) ? 64 : 48;
    uint8_t* rs = page + HDR_BYTES;
    uint8_t* cs = rs + 2 * P;
    uint8_t* ss = cs + (int64_t)codes_bytes * P;
    uint8_t* vs = ss + 2 * P;
    put16(rs + 2 * r, rt);
    put16(ss + 2 * r, sc);
    uint8_t* row = cs + (int64_t)r * codes_bytes;
    for (int p = 0; p < d / 2; p++) {
        int g = (p / 4) % 4, j = 4 * (p / 16) + p % 4;
        int rho = orc_rho_code(k[2 * p], k[2 * p + 1], R2, d);
        if (tier == TIER_T1 && g_t1_scheme) {
            int th = orc_angle_code(k[2 * p], k[2 * p + 1], 5);
            row[16 * g + j] = (uint8_t)((th << 3) | orc_rho_code3(k[2 * p], k[2 * p + 1], R2, d));
        } else if (tier == TIER_T1) {
            int th = orc_angle_code(k[2 * p], k[2 * p + 1], BITS_T1);
            row[16 * g + j] = (uint8_t)((th << 2) | rho);
        } else {
            int th = orc_angle_code(k[2 * p], k[2 * p + 1], BITS_T2);
            row[8 * g + j / 2] |= (uint8_t)(th << (4 * (j % 2)));
            row[32 + 4 * g + j / 4] |= (uint8_t)(rho << (2 * (j % 4)));
        }
    }
    for (int dd = 0; dd < d; dd++) vs[v_frag_offset(r, dd, 1)] = (uint8_t)v8[dd];
}

/* Pack the tiered tokens into tier-homogeneous pages.
   Per (seq, head): the T0 tokens, then T1, then T2, each in ascending
   position, in chunks of P rows (the last page of a tier may be partial).
   Page slots of tier t are taken from free_t in the order (seq, head, page).
   page_ids[i] = tier << 30 | slot; page_indptr is the CSR offset per
   (seq, head) unit u = b*Hkv + h.  row_of[b][h][t] = (index of the page
   within its unit's list) * P + row, or -1 when the token is not resident.
   Each used slot's payload is fully written (zeros in unused rows). */
int orc_pack(int B, int Hkv, int Tmax, int d, int P, const int32_t* seq_lens,
             const uint16_t* K, const uint16_t* V, const uint8_t* tier,
             const uint32_t* free0, const uint32_t* free1, const uint32_t* free2,
             const int64_t* free_len, int32_t* row_of, int32_t* page_indptr,
             uint32_t* page_ids, int64_t page_cap, uint8_t* pool0, uint8_t* pool1,
             uint8_t* pool2, const int64_t* pool_slots) {
    if (d != 128 || P <= 0 || P % 16 != 0) return ORC_ERR_ARG;
    const uint32_t* fl[3] = {free0, free1, free2};
    uint8_t* pools[3] = {pool0, pool1, pool2};
    int64_t taken[3] = {0, 0, 0};
    int64_t npage = 0;
    int32_t* list = (int32_t*)malloc(sizeof(int32_t) * (Tmax > 0 ? Tmax : 1));
    for (int b = 0; b < B; b++) {
        int T = seq_lens[b];
        for (int h = 0; h < Hkv; h++) {
            int u = b * Hkv + h;
            page_indptr[u] = (int32_t)npage;
            for (int t = 0; t < Tmax; t++) row_of[((int64_t)b * Hkv + h) * Tmax + t] = -1;
            for (int tr = 0; tr < 3; tr++) {
                int n = 0;
                for (int t = 0; t < T; t++)
                    if (tier[((int64_t)b * Hkv + h) * Tmax + t] == tr) list[n++] = t;
                int np = (n + P - 1) / P;
                for (int p = 0; p < np; p++) {
                    if (taken[tr] >= free_len[tr]) { free(list); return ORC_ERR_POOL; }
                    uint32_t slot = fl[tr][taken[tr]++];
                    if ((int64_t)slot >= pool_slots[tr] || npage >= page_cap) {
                        free(list);
                        return ORC_ERR_POOL;
                    }
                    int64_t pidx = npage - page_indptr[u];
                    page_ids[npage++] = ((uint32_t)tr << 30) | slot;
                    uint8_t* page = pools[tr] + (int64_t)slot * orc_page_stride(tr, P, d);
                    memset(page, 0, orc_page_payload(tr, P, d));
                    int cnt = (n - p * P) < P ? (n - p * P) : P;
                    put16(page + 0, (uint16_t)cnt);
                    page[2] = (uint8_t)tr;
                    page[3] = PAGE_MAGIC;
                    put32(page + 4, (uint32_t)b);
                    put32(page + 8, (uint32_t)h);
                    put32(page + 12, (uint32_t)p);
                    for (int r = 0; r < cnt; r++) {
                        int t = list[p * P + r];
                        int64_t idx = ((int64_t)b * Hkv + h) * Tmax + t;
                        write_row(page, tr, P, d, r, K + idx * d, V + idx * d);
                        row_of[idx] = (int32_t)(pidx * P + r);
                    }
                }
            }
        }
    }
    page_indptr[B * Hkv] = (int32_t)npage;
    free(list);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Attention over the resident tokens [TS 2.1], fp64 textbook softmax  */
/* ------------------------------------------------------------------ */

/* For each query head hq of sequence b (kv head h = hq / (Hq/Hkv)):
   the resident tokens are those with tier != dropped; k^ is the dense fp16
   key for T0 and the reconstruction from the codes for T1 (b=6) / T2 (b=4);
   v^ is the fp16 value for T0 and scale * int8 code otherwise;
   l_t = q . k^_t / sqrt(d); out = sum_t softmax(l)_t v^_t; lse = log sum exp l.
   No mask: decode attends over the whole resident cache.  A unit with no
   resident token gives out = 0 and lse = -inf.
   units: optional list of n_units (b, hq) pairs to compute (others untouched);
   NULL computes all B*Hq.  q_kind: 0 fp16, 1 bf16. */
int orc_decode(int B, int Hq, int Hkv, int Tmax, int d, const int32_t* seq_lens,
               const uint16_t* K, const uint16_t* V, const uint8_t* tier,
               const uint16_t* q, int q_kind, double* out, double* lse,
               const int32_t* units, int n_units) {
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0) return ORC_ERR_ARG;
    init_once();
    int G = Hq / Hkv;
    int total = units ? n_units : B * Hq;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int w = 0; w < total; w++) {
        int b = units ? units[2 * w] : w / Hq;
        int hq = units ? units[2 * w + 1] : w % Hq;
        if (b < 0 || b >= B || hq < 0 || hq >= Hq) { bad = 1; continue; }
        int h = hq / G;
        int T = seq_lens[b];
        double* qd = (double*)malloc(sizeof(double) * d);
        for (int c = 0; c < d; c++) {
            uint16_t x = q[((int64_t)b * Hq + hq) * d + c];
            qd[c] = q_kind ? bf2d(x) : h2d(x);
        }
        double* logit = (double*)malloc(sizeof(double) * (T > 0 ? T : 1));
        double* kh = (double*)malloc(sizeof(double) * d);
        double mx = -INFINITY;
        for (int t = 0; t < T; t++) {
            int64_t idx = ((int64_t)b * Hkv + h) * Tmax + t;
            int tr = tier[idx];
            if (tr == TIER_DROP) { logit[t] = -INFINITY; continue; }
            const uint16_t* k = K + idx * d;
            if (tr == TIER_T0)
                for (int c = 0; c < d; c++) kh[c] = t0_val(k[c]);
            else
                orc_reconstruct_tier(k, d, tr, kh);
            double s = 0.0;
            for (int c = 0; c < d; c++) s += qd[c] * kh[c];
            logit[t] = s / sqrt((double)d);
            if (logit[t] > mx) mx = logit[t];
        }
        double* o = out + ((int64_t)b * Hq + hq) * d;
        for (int c = 0; c < d; c++) o[c] = 0.0;
        if (mx == -INFINITY) {
            lse[(int64_t)b * Hq + hq] = -INFINITY;
        } else {
            double l = 0.0;
            int8_t v8[128];
            uint16_t sc;
            for (int t = 0; t < T; t++) {
                if (logit[t] == -INFINITY) continue;
                int64_t idx = ((int64_t)b * Hkv + h) * Tmax + t;
                double wgt = exp(logit[t] - mx);
                l += wgt;
                const uint16_t* v = V + idx * d;
                if (tier[idx] == TIER_T0) {
                    for (int c = 0; c < d; c++) o[c] += wgt * t0_val(v[c]);
                } else {
                    orc_vquant(v, d, v8, &sc);
                    double s = h2d(sc);
                    for (int c = 0; c < d; c++) o[c] += wgt * (s * (double)v8[c]);
                }
            }
            for (int c = 0; c < d; c++) o[c] /= l;
            lse[(int64_t)b * Hq + hq] = mx + log(l);
        }
        free(qd);
        free(logit);
        free(kh);
    }
    return bad ? ORC_ERR_ARG : ORC_OK;
}

/* Outlier flag of a key, for the protection constraint [TS 2.2] (outliers
   are among the states kept at the top tier).  READING: a key is an
   outlier when one of its pairs holds a share far beyond the 2-bit share
   grid: u_i = (rho_i / r) sqrt(d/2) > 4, twice the top level u = 2, where
   the decoded share is under half of the pair's true one.  For Gaussian
   keys u^2 is about Exp(1), so this flags about one key in 10^5 at d = 128;
   a channel scaled up twentyfold flags every key.  Exact integer test:
   (d/2) rho_i^2 > 16 R2; a tie is not an outlier. */
int orc_outlier(const uint16_t* k, int d) {
    uint64_t R2[2];
    orc_norm2(k, d, R2);
    u128 R = ((u128)R2[1] << 64) | R2[0];
    for (int i = 0; i < d / 2; i++) {
        int64_t mx = h2m(k[2 * i]), my = h2m(k[2 * i + 1]);
        u128 ax = (u128)(mx < 0 ? -mx : mx), ay = (u128)(my < 0 ? -my : my);
        u128 rho2 = ax * ax + ay * ay;
        if (rho2 * (u128)(d / 2) > (u128)16 * R) return 1;
    }
    return 0;
}

/* flags[b][h][t] = orc_outlier(K[b][h][t]) for t < seq_lens[b], else 0 */
int orc_outlier_flags(int B, int Hkv, int Tmax, int d, const int32_t* seq_lens,
                      const uint16_t* K, uint8_t* flags) {
    if (B < 0 || Hkv <= 0 || Tmax < 0 || d <= 0 || (d & 1)) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)B * Hkv * Tmax; i++) {
        int b = (int)(i / ((int64_t)Hkv * Tmax));
        int64_t t = i % Tmax;
        flags[i] = t < seq_lens[b] ? (uint8_t)orc_outlier(K + i * d, d) : 0;
    }
    return ORC_OK;
}

/* Attention mass per resident token, the decode-side utility signal.
   READING: [ABS] drives retention by an "estimated future utility" without
   saying how it is estimated; the plainest estimator the decode supplies is
   the softmax weight a token receives, summed over the query heads of its
   kv group.  mass[b][h][t] = sum_{g<G} softmax_t(l_{hq})[t], hq = h G + g,
   with l_t = q . k^_t / sqrt(d) exactly as in orc_decode; 0 for dropped
   tokens and positions >= seq_lens[b].  Every unit with a resident token
   has sum_t mass = G. */
int orc_attention_mass(int B, int Hq, int Hkv, int Tmax, int d, const int32_t* seq_lens,
                       const uint16_t* K, const uint8_t* tier, const uint16_t* q, int q_kind,
                       double* mass) {
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0) return ORC_ERR_ARG;
    init_once();
    int G = Hq / Hkv;
    for (int64_t i = 0; i < (int64_t)B * Hkv * Tmax; i++) mass[i] = 0.0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int w = 0; w < B * Hq; w++) {
        int b = w / Hq, hq = w % Hq, h = hq / G;
        int T = seq_lens[b];
        double* qd = (double*)malloc(sizeof(double) * d);
        for (int c = 0; c < d; c++) {
            uint16_t x = q[((int64_t)b * Hq + hq) * d + c];
            qd[c] = q_kind ? bf2d(x) : h2d(x);
        }
        double* logit = (double*)malloc(sizeof(double) * (T > 0 ? T : 1));
        double* kh = (double*)malloc(sizeof(double) * d);
        double mx = -INFINITY;
        for (int t = 0; t < T; t++) {
            int64_t idx = ((int64_t)b * Hkv + h) * Tmax + t;
            int tr = tier[idx];
            if (tr == TIER_DROP) { logit[t] = -INFINITY; continue; }
            const uint16_t* k = K + idx * d;
            if (tr == TIER_T0)
                for (int c = 0; c < d; c++) kh[c] = t0_val(k[c]);
            else
                orc_reconstruct_tier(k, d, tr, kh);
            double s = 0.0;
            for (int c = 0; c < d; c++) s += qd[c] * kh[c];
            logit[t] = s / sqrt((double)d);
            if (logit[t] > mx) mx = logit[t];
        }
        if (mx != -INFINITY) {
            double l = 0.0;
            for (int t = 0; t < T; t++)
                if (logit[t] != -INFINITY) l += exp(logit[t] - mx);
            for (int t = 0; t < T; t++) {
                if (logit[t] == -INFINITY) continue;
                int64_t idx = ((int64_t)b * Hkv + h) * Tmax + t;
                double p = exp(logit[t] - mx) / l;
#pragma omp atomic
                mass[idx] += p;
            }
        }
        free(qd);
        free(logit);
        free(kh);
    }
    return ORC_OK;
}

/* helpers exposed for pins: fp16 rounding, exact norm as double */
uint16_t orc_d2h(double x) { return d2h(x); }
double orc_h2d(uint16_t h) { return h2d(h); }
double orc_bf2d(uint16_t h) { return bf2d(h); }
uint16_t orc_h2bf(uint16_t h) { return h2bf(h); }
int orc_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
