/*
 * TurboQuant KV-cache oracle — TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of what the TurboQuant KV-cache path
 * computes: the random rotation, the Lloyd–Max codebook, the per-coordinate
 * encoder, the 1-bit QJL sketch of the key residual, the packed cache format,
 * and decode attention over the stored codes. Only tests/, the smoke() entry
 * point and the bench's CPU-baseline leg load this file. It shares no code,
 * header, table or constant generator with the CUDA library: both sides were
 * written separately from the same statement of the method.
 *
 * Sources (page title, section):
 *  [MUNINN]  "[Benchmark] TurboQuant 實測：KV Cache 3-bit 壓縮，真的零損失？"
 *            (ai-muninn.com): §"TurboQuant 是什麼：30 秒懶人包" (rotation,
 *            Lloyd–Max per coordinate, 1-bit QJL residual, unbiased inner
 *            products), §"Lloyd-Max Codebook" (distortion per coordinate),
 *            §"MSE-Only vs QJL：bias 差異確認", §"GB10 速度" (byte counts),
 *            §"壓縮率與精度" (compression ratios with norms).
 *  [WISELY]  "turboquant-kvquant-vllm-benchmark" (ai-coding.wiselychen.com):
 *            §"TurboQuant 是什麼", the three core steps (random rotation;
 *            optimal scalar quantizer per coordinate; 1-bit QJL residual
 *            correction of inner products).
 *  [DIGIPUB] "Google把32B模型壓到5GB顯存，實測后我發現3個坑" (m.digipub.cc):
 *            opening section (Walsh–Hadamard rotation, then scalar quantization).
 *
 * Where the pages leave a step open the oracle takes the plainest reading:
 * codebook for N(0,1/d); K uses (b-1)-bit codes + QJL with m = d rows, V uses
 * b-bit codes; fp16 norms; SplitMix64 tables; strict '>' for the encoder;
 * z >= 0 gives sign bit 1; the packed tile layout of include/tq.h.
 *
 * Pins (tests/test_oracle_*.py check each function against something other
 * than itself): the generator against published SplitMix64 outputs and
 * Gaussian statistics; the rotation against Sylvester-Hadamard identities and
 * scipy's hadamard(); the codebook against the textbook Gaussian Lloyd–Max
 * values, closed forms and independent numerical integration; distortion
 * against the pages' printed values; the encoder against brute-force nearest
 * centroid; the QJL estimator against unbiasedness statistics; attention
 * against textbook softmax attention (torch, fp64) over the reconstructed
 * keys and values; packing by round trip and the pages' byte counts.
 * Parity unpinned: the magnitudes of the pages' bias figures (their trial
 * setup is not given; only the signs are checked).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define TQO_TILE 16
#define TQO_MAXL 128   /* most codebook levels: 7-bit cells */

/* ------------------------------------------------------------------------- */
/* Scalar conversions.                                                        */
/* ------------------------------------------------------------------------- */

/* IEEE binary16 bits -> double (exact). */
double oracle_half_to_double(uint16_t h)
{
    int s = h >> 15, e = (h >> 10) & 31, f = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);
    return s ? -v : v;
}

/* bfloat16 bits -> double (exact): the top half of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* double -> IEEE binary16, round to nearest even; overflow gives infinity. */
uint16_t oracle_double_to_half(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isnan(x)) return 0x7e00;
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);      /* a = f * 2^e, f in [0.5, 1) */
    e -= 1;            /* a = f' * 2^e, f' in [1, 2) */
    if (e < -14) {     /* subnormal range: quantum 2^-24 */
        double n = nearbyint(ldexp(a, 24));
        return sign | (uint16_t)n;   /* n == 1024 encodes 2^-14 correctly */
    }
    double n = nearbyint(ldexp(a, 10 - e));   /* in [1024, 2048] */
    if (n >= 2048.0) { n = 1024.0; e += 1; }
    if (e > 15) return sign | 0x7c00;
    return sign | (uint16_t)(((e + 15) << 10) | ((int)n - 1024));
}

/* Norm storage: fp16, round to nearest even, saturating at 65504 (flag). */
static uint16_t norm_to_half(double v, uint8_t* sat)
{
    if (v > 65504.0) { *sat = 1; return 0x7bff; }
    return oracle_double_to_half(v);
}

/* ------------------------------------------------------------------------- */
/* Counter-based generator (SplitMix64) and the method's random tables.       */
/* ------------------------------------------------------------------------- */

/* SplitMix64 (Steele, Lea, Flood 2014; Vigna's reference code): the generator
 * adds 0x9E3779B97F4A7C15 to its state and returns the state passed through
 * the mixing function below. Draw k (k = 0, 1, ...) of stream s is output
 * k+1 of a generator started at state seed ^ (0x5851F42D4C957F2D * (s+1)). */
static uint64_t sm64_mix(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t oracle_splitmix64_next(uint64_t* state)
{
    *state += 0x9E3779B97F4A7C15ULL;
    return sm64_mix(*state);
}

uint64_t oracle_draw(uint64_t seed, uint32_t stream, uint64_t k)
{
    uint64_t state = seed ^ (0x5851F42D4C957F2DULL * ((uint64_t)stream + 1));
    state += (k + 1) * 0x9E3779B97F4A7C15ULL;
    return sm64_mix(state);
}

/* Standard normal pair by Box–Muller from two 53-bit uniforms of a stream. */
static void gauss_pair(uint64_t seed, uint32_t stream, uint64_t q, double* g0, double* g1)
{
    uint64_t a = oracle_draw(seed, stream, 2 * q);
    uint64_t b = oracle_draw(seed, stream, 2 * q + 1);
    double u1 = ((double)(a >> 11) + 1.0) * 0x1p-53;   /* (0, 1] */
    double u2 = (double)(b >> 11) * 0x1p-53;           /* [0, 1) */
    double r = sqrt(-2.0 * log(u1));
    double th = 2.0 * M_PI * u2;
    *g0 = r * cos(th);
    *g1 = r * sin(th);
}

/* Element e of a standard-normal stream (pairs 2q, 2q+1 share one draw pair). */
double oracle_gauss(uint64_t seed, uint32_t stream, uint64_t e)
{
    double g0, g1;
    gauss_pair(seed, stream, e >> 1, &g0, &g1);
    return (e & 1) ? g1 : g0;
}

/* Rotation signs D (the random ±1 diagonal applied before the WHT):
 * D_i = -1 when the top bit of draw i of stream 0 is set, else +1. */
void oracle_rotation_signs(int d, uint64_t seed, int8_t* D)
{
    for (int i = 0; i < d; ++i)
        D[i] = (oracle_draw(seed, 0, (uint64_t)i) >> 63) ? -1 : 1;
}

/* QJL matrix S (m x d, row-major): i.i.d. N(0,1) from stream 1, element
 * e = j*d + i, each value rounded once to the nearest fp16 value. */
void oracle_qjl_matrix(int m, int d, uint64_t seed, double* S)
{
    for (int e = 0; e < m * d; e += 2) {
        double g0, g1;
        gauss_pair(seed, 1, (uint64_t)(e >> 1), &g0, &g1);
        S[e] = oracle_half_to_double(oracle_double_to_half(g0));
        S[e + 1] = oracle_half_to_double(oracle_double_to_half(g1));
    }
}

/* ------------------------------------------------------------------------- */
/* Lloyd–Max codebook [MUNINN §30 秒懶人包, §Lloyd-Max Codebook; WISELY step 2] */
/* ------------------------------------------------------------------------- */

static double phi(double x) { return exp(-0.5 * x * x) / sqrt(2.0 * M_PI); }
static double Phi(double x) { return 0.5 * erfc(-x / M_SQRT2); }

/* Optimal L = 2^B level scalar quantizer for N(0,1) by Lloyd's iteration:
 * boundaries are midpoints of neighbouring centroids, each centroid is the
 * conditional mean of its cell, (phi(lo) - phi(hi)) / (Phi(hi) - Phi(lo)).
 * Starts from evenly spaced centroids on [-2, 2] and iterates to fp64
 * convergence: once no centroid moves by 1e-12, it continues until the largest
 * step stops shrinking (the fp64 noise floor), so the fixed point is known far
 * below fp32 resolution; the result is made exactly symmetric. Returns 0 on
 * convergence. */
int oracle_lloyd_max_unit(int B, double* c, int* iters_out)
{
    int L = 1 << B;
    double nc[TQO_MAXL];
    for (int j = 0; j < L; ++j) c[j] = -2.0 + 4.0 * (j + 0.5) / L;
    int it, ok = -1;
    double prev = INFINITY;
    for (it = 0; it < 2000000; ++it) {
        double delta = 0.0;
        for (int j = 0; j < L; ++j) {
            double lo = (j == 0) ? -INFINITY : 0.5 * (c[j - 1] + c[j]);
            double hi = (j == L - 1) ? INFINITY : 0.5 * (c[j] + c[j + 1]);
            double plo = (j == 0) ? 0.0 : phi(lo), phi_hi = (j == L - 1) ? 0.0 : phi(hi);
            double mass = Phi(hi) - Phi(lo);
            nc[j] = (plo - phi_hi) / mass;
            double dd = fabs(nc[j] - c[j]);
            if (dd > delta) delta = dd;
        }
        memcpy(c, nc, sizeof(double) * L);
        /* below 1e-12 the iteration is in its linear regime: run it down to
         * the fp64 noise floor, i.e. until the step stops shrinking */
        if (delta == 0.0 || (delta < 1e-12 && delta >= prev)) { ok = 0; break; }
        prev = delta;
    }
    for (int j = 0; j < L / 2; ++j) {
        double s = 0.5 * (c[L - 1 - j] - c[j]);
        c[j] = -s;
        c[L - 1 - j] = s;
    }
    if (iters_out) *iters_out = it + 1;
    return ok;
}

/* Mean squared error of a unit-variance quantizer with centroids c, cells
 * bounded by midpoints, integrated in closed form over each cell. */
double oracle_quantizer_mse_unit(int B, const double* c)
{
    int L = 1 << B;
    double mse = 0.0;
    for (int j = 0; j < L; ++j) {
        double a = (j == 0) ? -INFINITY : 0.5 * (c[j - 1] + c[j]);
        double b = (j == L - 1) ? INFINITY : 0.5 * (c[j] + c[j + 1]);
        double pa = (j == 0) ? 0.0 : phi(a), pb = (j == L - 1) ? 0.0 : phi(b);
        double apa = (j == 0) ? 0.0 : a * pa, bpb = (j == L - 1) ? 0.0 : b * pb;
        double m0 = Phi(b) - Phi(a);        /* integral of phi          */
        double m1 = pa - pb;                /* integral of x phi        */
        double m2 = m0 + apa - bpb;         /* integral of x^2 phi      */
        mse += m2 - 2.0 * c[j] * m1 + c[j] * c[j] * m0;
    }
    return mse;
}

/* Codebook for one head dimension: the unit-variance centroids scaled by
 * 1/sqrt(d) (rotated coordinates of a unit vector are close to N(0, 1/d)),
 * rounded once to fp32; boundaries are the fp32 midpoints of neighbours. */
int oracle_codebook(int B, int d, float* centroids, float* bounds)
{
    double c[TQO_MAXL];
    int rc = oracle_lloyd_max_unit(B, c, NULL);
    int L = 1 << B;
    for (int j = 0; j < L; ++j) centroids[j] = (float)(c[j] / sqrt((double)d));
    for (int j = 0; j + 1 < L; ++j)
        bounds[j] = (float)(0.5 * ((double)centroids[j] + (double)centroids[j + 1]));
    return rc;
}

/* ------------------------------------------------------------------------- */
/* Exact coordinate marginal [WISELY §TurboQuant 是什麼, step 1: a random      */
/* rotation concentrates the coordinates as a Beta distribution]              */
/* ------------------------------------------------------------------------- */

/* Density of one coordinate y of a uniformly random unit vector in R^d, d >= 3:
 *   f_d(y) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) (1 - y^2)^((d-3)/2),  |y| < 1,
 * i.e. (1 + y)/2 ~ Beta((d-1)/2, (d-1)/2). N(0, 1/d) is its large-d limit. */
double oracle_beta_marginal_pdf(int d, double y)
{
    if (!(y > -1.0 && y < 1.0)) return 0.0;
    double logc = lgamma(0.5 * d) - 0.5 * log(M_PI) - lgamma(0.5 * (d - 1));
    return exp(logc + 0.5 * (d - 3) * log1p(-y * y));
}

/* Moments m_k = integral over [lo, hi] of y^k f_d(y) dy, k = 0, 1, 2, by
 * composite Simpson in theta with y = sin(theta): the integrand becomes
 * c_d sin^k(theta) cos^(d-2)(theta), smooth up to the ends of [-1, 1]. */
static void beta_moments(int d, double lo, double hi, double* m0, double* m1, double* m2)
{
    *m0 = *m1 = *m2 = 0.0;
    if (lo < -1.0) lo = -1.0;
    if (hi > 1.0) hi = 1.0;
    if (!(hi > lo)) return;
    const int n = 20000;   /* panels, even */
    double a = asin(lo), b = asin(hi), h = (b - a) / n;
    double logc = lgamma(0.5 * d) - 0.5 * log(M_PI) - lgamma(0.5 * (d - 1));
    double s0 = 0.0, s1 = 0.0, s2 = 0.0;
    for (int i = 0; i <= n; ++i) {
        double th = a + i * h, w = (i == 0 || i == n) ? 1.0 : ((i & 1) ? 4.0 : 2.0);
        double cs = cos(th), sn = sin(th);
        double f = (cs > 0.0) ? w * exp(logc + (d - 2) * log(cs)) : 0.0;
        s0 += f;
        s1 += f * sn;
        s2 += f * sn * sn;
    }
    *m0 = s0 * h / 3.0;
    *m1 = s1 * h / 3.0;
    *m2 = s2 * h / 3.0;
}

/* Lloyd–Max for f_d with L = 2^B levels: midpoint boundaries, centroids the
 * conditional means m1/m0 of their cells. Starts from the N(0,1/d) codebook
 * (d >= 16) or from the uniform quantizer on [-1, 1], and stops like the
 * Gaussian iteration (at the fp64/quadrature noise floor). Symmetrised. */
int oracle_lloyd_max_beta(int d, int B, double* c)
{
    int L = 1 << B;
    if (d >= 16) {
        double g[TQO_MAXL];
        oracle_lloyd_max_unit(B, g, NULL);
        for (int j = 0; j < L; ++j) c[j] = g[j] / sqrt((double)d);
    } else {
        for (int j = 0; j < L; ++j) c[j] = -1.0 + (2.0 * j + 1.0) / L;
    }
    double nc[TQO_MAXL], prev = INFINITY;
    int ok = -1;
    for (int it = 0; it < 100000; ++it) {
        double delta = 0.0;
        for (int j = 0; j < L; ++j) {
            double lo = (j == 0) ? -1.0 : 0.5 * (c[j - 1] + c[j]);
            double hi = (j == L - 1) ? 1.0 : 0.5 * (c[j] + c[j + 1]);
            double m0, m1, m2;
            beta_moments(d, lo, hi, &m0, &m1, &m2);
            nc[j] = m1 / m0;
            double dd = fabs(nc[j] - c[j]);
            if (dd > delta) delta = dd;
        }
        memcpy(c, nc, sizeof(double) * L);
        if (delta == 0.0 || (delta < 1e-13 && delta >= prev)) { ok = 0; break; }
        prev = delta;
    }
    for (int j = 0; j < L / 2; ++j) {
        double s = 0.5 * (c[L - 1 - j] - c[j]);
        c[j] = -s;
        c[L - 1 - j] = s;
    }
    return ok;
}

/* Mean squared error, under f_d, of the quantizer with centroids c (any scale:
 * these are coordinates of a unit vector) and midpoint cells. */
double oracle_quantizer_mse_beta(int d, int B, const double* c)
{
    int L = 1 << B;
    double mse = 0.0;
    for (int j = 0; j < L; ++j) {
        double lo = (j == 0) ? -1.0 : 0.5 * (c[j - 1] + c[j]);
        double hi = (j == L - 1) ? 1.0 : 0.5 * (c[j] + c[j + 1]);
        double m0, m1, m2;
        beta_moments(d, lo, hi, &m0, &m1, &m2);
        mse += m2 - 2.0 * c[j] * m1 + c[j] * c[j] * m0;
    }
    return mse;
}

/* The exact-marginal codebook: oracle_lloyd_max_beta rounded once to fp32,
 * boundaries the fp32 midpoints (the same rounding as oracle_codebook). */
int oracle_codebook_beta(int B, int d, float* centroids, float* bounds)
{
    double c[TQO_MAXL];
    int rc = oracle_lloyd_max_beta(d, B, c);
    int L = 1 << B;
    for (int j = 0; j < L; ++j) centroids[j] = (float)c[j];
    for (int j = 0; j + 1 < L; ++j)
        bounds[j] = (float)(0.5 * ((double)centroids[j] + (double)centroids[j + 1]));
    return rc;
}

/* ------------------------------------------------------------------------- */
/* Rotation [DIGIPUB opening; MUNINN §30 秒懶人包; WISELY step 1]              */
/* ------------------------------------------------------------------------- */

/* Sylvester-Hadamard entry H_ij = (-1)^popcount(i & j). */
static int hsign(int i, int j) { return (__builtin_popcount((unsigned)(i & j)) & 1) ? -1 : 1; }

/* y = Pi u with Pi = H D / sqrt(d): sign flips, then the Walsh–Hadamard
 * transform, written as the explicit matrix product. */
void oracle_rotate(int d, const int8_t* D, const double* u, double* y)
{
    double s = 1.0 / sqrt((double)d);
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += hsign(i, j) * D[j] * u[j];
        y[i] = acc * s;
    }
}

/* u = Pi^T y = D H y / sqrt(d) (H is symmetric). */
void oracle_rotate_inverse(int d, const int8_t* D, const double* y, double* u)
{
    double s = 1.0 / sqrt((double)d);
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += hsign(i, j) * y[j];
        u[i] = D[i] * acc * s;
    }
}

/* ------------------------------------------------------------------------- */
/* Encoder and quantization of one vector                                     */
/* ------------------------------------------------------------------------- */

/* Cell index: the number of boundaries strictly below y. */
int oracle_encode(double y, const float* bounds, int L)
{
    int idx = 0;
    for (int j = 0; j + 1 < L; ++j)
        if (y > (double)bounds[j]) ++idx;
    return idx;
}

static double nearest_boundary_dist(double y, const float* bounds, int L)
{
    double best = INFINITY;
    for (int j = 0; j + 1 < L; ++j) {
        double dd = fabs(y - (double)bounds[j]);
        if (dd < best) best = dd;
    }
    return best;
}

/* Rotated unit vector of a fp16 vector: y = Pi (x / ||x||), written as
 * Pi x / ||x|| (the same value) so that a coordinate whose Walsh–Hadamard sum
 * cancels exactly stays exactly 0 and meets the tie rule of the encoder.
 * Returns ||x||; y = 0 for the zero vector. */
static double rotate_unit(int d, const int8_t* D, const uint16_t* x, double* y)
{
    double xv[256], ss = 0.0;
    for (int i = 0; i < d; ++i) {
        xv[i] = oracle_half_to_double(x[i]);
        ss += xv[i] * xv[i];
    }
    double n = sqrt(ss);
    oracle_rotate(d, D, xv, y);
    for (int i = 0; i < d; ++i) y[i] = (n > 0.0) ? y[i] / n : 0.0;
    return n;
}

/* Keys [MUNINN §30 秒懶人包 step 1 and 2; WISELY steps 1-3]:
 * y = Pi (x/||x||), idx_i = encode(y_i) with the (B_K)-bit codebook,
 * r = y - c[idx], rho = ||r||, z = S r, sign bit s_j = [z_j >= 0].
 * Stores ||x|| and rho as fp16. ydist/zabs report how close each decision was
 * to its threshold (for counting boundary cases in parity tests).
 * With qjl = 0 (the MSE-only key format, [MUNINN §MSE-Only vs QJL]) only the
 * cells and ||x|| are produced: signs, rho and zabs are left at 0. */
void oracle_quantize_keys(int d, int N, const uint16_t* x, const int8_t* D, const double* S,
                          const float* cK, const float* tK, int BK, int qjl,
                          uint8_t* kidx, uint8_t* ksign, uint16_t* knorm, uint16_t* rnorm,
                          double* ydist, double* zabs, uint8_t* sat)
{
    int L = 1 << BK, m = d;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        double y[256], r[256];
        uint8_t s0 = 0;
        double nrm = rotate_unit(d, D, x + (size_t)n * d, y);
        double rr = 0.0;
        for (int i = 0; i < d; ++i) {
            int id = oracle_encode(y[i], tK, L);
            kidx[(size_t)n * d + i] = (uint8_t)id;
            if (ydist) ydist[(size_t)n * d + i] = nearest_boundary_dist(y[i], tK, L);
            r[i] = y[i] - (double)cK[id];
            rr += r[i] * r[i];
        }
        for (int j = 0; j < m; ++j) {
            double z = 0.0;
            if (qjl)
                for (int i = 0; i < d; ++i) z += S[(size_t)j * d + i] * r[i];
            ksign[(size_t)n * m + j] = (qjl && z >= 0.0) ? 1 : 0;
            if (zabs) zabs[(size_t)n * m + j] = qjl ? fabs(z) : 0.0;
        }
        knorm[n] = norm_to_half(nrm, &s0);
        rnorm[n] = qjl ? norm_to_half(sqrt(rr), &s0) : 0;
        if (sat) sat[n] = s0;
    }
}

/* Values: the MSE stage alone with the B_V-bit codebook, plus ||v|| (fp16). */
void oracle_quantize_values(int d, int N, const uint16_t* x, const int8_t* D,
                            const float* cV, const float* tV, int BV,
                            uint8_t* vidx, uint16_t* vnorm, double* ydist, uint8_t* sat)
{
    int L = 1 << BV;
    (void)cV;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        double y[256];
        uint8_t s0 = 0;
        double nrm = rotate_unit(d, D, x + (size_t)n * d, y);
        for (int i = 0; i < d; ++i) {
            vidx[(size_t)n * d + i] = (uint8_t)oracle_encode(y[i], tV, L);
            if (ydist) ydist[(size_t)n * d + i] = nearest_boundary_dist(y[i], tV, L);
        }
        vnorm[n] = norm_to_half(nrm, &s0);
        if (sat) sat[n] = s0;
    }
}

/* ------------------------------------------------------------------------- */
/* Packed cache format (this library's own layout). A format is (B_K, B_V,    */
/* qjl): key cells of B_K bits, value cells of B_V bits, and with qjl = 1 the */
/* 1-bit QJL sketch of the key residual plus its norm rho. With W = B_K +     */
/* qjl + B_V, a stream of one (batch, kv-head) is a run of 16-token tiles of  */
/* 16*(W*d/8 + 4 + 2*qjl) bytes:                                              */
/*   codes:   2*W*d bytes = 32 lane strings of W*d/16 bytes each, stored as   */
/*            chunks of C bytes (C = 16, 8 or 4: the largest dividing the    */
/*            string); chunk c of lane l sits at byte (c*32 + l)*C; a lane    */
/*            string is its chunks in order, bit k = bit (k%8) of byte k/8.   */
/*   K norms: qjl: 64 bytes; for g = 0..7: fp16 {|k_g|, rho_g, |k_g+8|,       */
/*            rho_g+8}. No qjl: 32 bytes; fp16 {|k_g|, |k_g+8|}.              */
/*   V norms: 32 bytes; for g = 0..7: fp16 {|v_g|, |v_g+8|}.                  */
/* Lane l = 4g + t holds, for p = 4kk + r (kk < d/16, r < 4), e in {0,1}:     */
/*   K code of token g + 8(r&1), coordinate 16kk + 8(r>>1) + 2t + e,          */
/*        B_K bits at bit 2*B_K*p + e*B_K;                                    */
/*   (qjl) sign of the same token for QJL row 16kk + 8(r>>1) + 2t + e,        */
/*        at bit B_K*d/2 + 32*(p/16) + 16e + (p%16);                          */
/*   V code of token 2t + 8(r>>1) + e, coordinate 16kk + g + 8(r&1),          */
/*        B_V bits at bit (B_K+qjl)*d/2 + 2*B_V*p + e*B_V.                    */
/* Except for (3, 4, 1), whose key pair and two signs share a byte: the K     */
/* code at bit 8p + 3e (the low 6 bits of byte p), the sign at bit            */
/* 32*(p/4) + 16e + a with a = 6, 7, 14, 15 for p%4 = 0, 1, 2, 3 (the top     */
/* two bits of the bytes of word p/4); the V codes as above.                  */
/* And except for (2, 3, 1), whose value pair and two signs share a byte: the */
/* K codes as above (the first B_K*d/2 bits), then the V code at bit          */
/* B_K*d/2 + 8p + 3e (the low 6 bits of byte p of that region) and the sign   */
/* at bit B_K*d/2 + 32*(p/4) + 16e + a, a as above.                           */
/* The TurboQuant format at b bits is (b-1, b, 1): tiles of 16*(b*d/4 + 6).   */
/* ------------------------------------------------------------------------- */

int64_t oracle_tile_bytes(int d, int kb, int vb, int qjl)
{
    return (int64_t)TQO_TILE * ((int64_t)(kb + qjl + vb) * d / 8 + 4 + 2 * qjl);
}

static int chunk_bytes(int d, int kb, int vb, int qjl)
{
    int sb = (kb + qjl + vb) * d / 16;
    return (sb % 16 == 0) ? 16 : (sb % 8 == 0) ? 8 : 4;
}

static int64_t lane_bit_addr(int C, int lane, int64_t bit)
{
    int64_t byte = bit >> 3;
    int64_t chunk = byte / C, off = byte % C;
    return ((chunk * 32 + lane) * C + off) * 8 + (bit & 7);
}

static void put_bits(uint8_t* tile, int C, int lane, int64_t bit, int nbits, unsigned v)
{
    for (int k = 0; k < nbits; ++k) {
        int64_t a = lane_bit_addr(C, lane, bit + k);
        if ((v >> k) & 1) tile[a >> 3] |= (uint8_t)(1u << (a & 7));
        else tile[a >> 3] &= (uint8_t)~(1u << (a & 7));
    }
}

static unsigned get_bits(const uint8_t* tile, int C, int lane, int64_t bit, int nbits)
{
    unsigned v = 0;
    for (int k = 0; k < nbits; ++k) {
        int64_t a = lane_bit_addr(C, lane, bit + k);
        v |= (unsigned)((tile[a >> 3] >> (a & 7)) & 1) << k;
    }
    return v;
}

/* Whether format (kb, vb, qjl) keeps each key pair and two sign bits in one
 * byte; whether it keeps each value pair and two sign bits in one byte. */
static int key_sign_bytes(int kb, int qjl) { return qjl == 1 && kb == 3; }
static int value_sign_bytes(int kb, int vb, int qjl) { return qjl == 1 && kb == 2 && vb == 3; }

/* Lane-string bit of key code (p, e). */
static int64_t key_bit(int kb, int qjl, int p, int e)
{
    if (key_sign_bytes(kb, qjl)) return 8LL * p + 3 * e;
    return 2LL * kb * p + (int64_t)e * kb;
}

/* Lane-string bit of sign (p, e). Generic layout: sign pair p of a lane has
 * element 0 at bit p%16, element 1 at bit 16 + p%16 of the lane's sign word
 * p/16, after the key codes (sign words start at bit kb*d/2). */
static int64_t sign_bit(int d, int kb, int vb, int qjl, int p, int e)
{
    static const int top[4] = {6, 7, 14, 15};
    if (key_sign_bytes(kb, qjl)) return 32LL * (p / 4) + 16 * e + top[p % 4];
    if (value_sign_bytes(kb, vb, qjl)) return (int64_t)kb * d / 2 + 32LL * (p / 4) + 16 * e + top[p % 4];
    return (int64_t)kb * d / 2 + 32LL * (p / 16) + 16 * e + (p % 16);
}

/* Lane-string bit of value code (p, e): after the key codes and sign words,
 * two vb-bit fields a pair; for (2, 3, 1) byte p of the region after the key
 * codes, element e at bit 3e. */
static int64_t value_bit(int d, int kb, int vb, int qjl, int p, int e)
{
    if (value_sign_bytes(kb, vb, qjl)) return (int64_t)kb * d / 2 + 8LL * p + 3 * e;
    return (int64_t)(kb + qjl) * d / 2 + 2LL * vb * p + (int64_t)e * vb;
}

static void put_half(uint8_t* p, uint16_t h) { p[0] = (uint8_t)(h & 0xff); p[1] = (uint8_t)(h >> 8); }
static uint16_t get_half(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* Byte offsets of token slot n (0..15) of a tile: its |k|, its rho (qjl) and its |v|. */
static void norm_offsets(int d, int kb, int vb, int qjl, int n, int64_t* ok, int64_t* orho,
                         int64_t* ov)
{
    int64_t knoff = 2LL * (kb + qjl + vb) * d, vnoff = knoff + 32 + 32 * qjl;
    int g = n & 7, h = n >> 3;
    if (qjl) {
        *ok = knoff + 8 * g + 4 * h;
        *orho = *ok + 2;
    } else {
        *ok = knoff + 4 * g + 2 * h;
        *orho = -1;
    }
    *ov = vnoff + 4 * g + 2 * h;
}

/* Pack tokens [0, N) of one stream (codes as produced above) into ceil(N/16)
 * tiles; slots past N in the last tile are zero. */
void oracle_pack_stream(int d, int kb, int vb, int qjl, int N, const uint8_t* kidx,
                        const uint8_t* ksign, const uint16_t* knorm, const uint16_t* rnorm,
                        const uint8_t* vidx, const uint16_t* vnorm, uint8_t* out)
{
    int m = d, C = chunk_bytes(d, kb, vb, qjl);
    int64_t TB = oracle_tile_bytes(d, kb, vb, qjl);
    int ntiles = (N + TQO_TILE - 1) / TQO_TILE;
    memset(out, 0, (size_t)(TB * ntiles));
    for (int tl = 0; tl < ntiles; ++tl) {
        uint8_t* tile = out + TB * tl;
        for (int lane = 0; lane < 32; ++lane) {
            int g = lane >> 2, t = lane & 3;
            for (int p = 0; p < d / 4; ++p) {
                int kk = p >> 2, r = p & 3;
                for (int e = 0; e < 2; ++e) {
                    int nk = tl * TQO_TILE + g + 8 * (r & 1);
                    int ik = 16 * kk + 8 * (r >> 1) + 2 * t + e;
                    int nv = tl * TQO_TILE + 2 * t + 8 * (r >> 1) + e;
                    int iv = 16 * kk + g + 8 * (r & 1);
                    if (nk < N) {
                        put_bits(tile, C, lane, key_bit(kb, qjl, p, e), kb, kidx[(size_t)nk * d + ik]);
                        if (qjl)
                            put_bits(tile, C, lane, sign_bit(d, kb, vb, qjl, p, e), 1,
                                     ksign[(size_t)nk * m + ik]);
                    }
                    if (nv < N)
                        put_bits(tile, C, lane, value_bit(d, kb, vb, qjl, p, e), vb,
                                 vidx[(size_t)nv * d + iv]);
                }
            }
        }
        for (int n = 0; n < TQO_TILE; ++n) {
            int tok = tl * TQO_TILE + n;
            if (tok >= N) continue;
            int64_t ok, orho, ov;
            norm_offsets(d, kb, vb, qjl, n, &ok, &orho, &ov);
            put_half(tile + ok, knorm[tok]);
            if (qjl) put_half(tile + orho, rnorm[tok]);
            put_half(tile + ov, vnorm[tok]);
        }
    }
}

/* Inverse of oracle_pack_stream for tokens [0, N) (signs and rho read as 0
 * when qjl = 0). */
void oracle_unpack_stream(int d, int kb, int vb, int qjl, int N, const uint8_t* in, uint8_t* kidx,
                          uint8_t* ksign, uint16_t* knorm, uint16_t* rnorm, uint8_t* vidx,
                          uint16_t* vnorm)
{
    int m = d, C = chunk_bytes(d, kb, vb, qjl);
    int64_t TB = oracle_tile_bytes(d, kb, vb, qjl);
    int ntiles = (N + TQO_TILE - 1) / TQO_TILE;
    for (int tl = 0; tl < ntiles; ++tl) {
        const uint8_t* tile = in + TB * tl;
        for (int lane = 0; lane < 32; ++lane) {
            int g = lane >> 2, t = lane & 3;
            for (int p = 0; p < d / 4; ++p) {
                int kk = p >> 2, r = p & 3;
                for (int e = 0; e < 2; ++e) {
                    int nk = tl * TQO_TILE + g + 8 * (r & 1);
                    int ik = 16 * kk + 8 * (r >> 1) + 2 * t + e;
                    int nv = tl * TQO_TILE + 2 * t + 8 * (r >> 1) + e;
                    int iv = 16 * kk + g + 8 * (r & 1);
                    if (nk < N) {
                        kidx[(size_t)nk * d + ik] =
                            (uint8_t)get_bits(tile, C, lane, key_bit(kb, qjl, p, e), kb);
                        ksign[(size_t)nk * m + ik] =
                            (uint8_t)(qjl ? get_bits(tile, C, lane, sign_bit(d, kb, vb, qjl, p, e), 1) : 0);
                    }
                    if (nv < N)
                        vidx[(size_t)nv * d + iv] =
                            (uint8_t)get_bits(tile, C, lane, value_bit(d, kb, vb, qjl, p, e), vb);
                }
            }
        }
        for (int n = 0; n < TQO_TILE; ++n) {
            int tok = tl * TQO_TILE + n;
            if (tok >= N) continue;
            int64_t ok, orho, ov;
            norm_offsets(d, kb, vb, qjl, n, &ok, &orho, &ov);
            knorm[tok] = get_half(tile + ok);
            rnorm[tok] = qjl ? get_half(tile + orho) : 0;
            vnorm[tok] = get_half(tile + ov);
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Decode attention over the stored codes [MUNINN §30 秒懶人包 step 2: the     */
/* QJL-corrected inner product is unbiased; WISELY step 3]                    */
/* ------------------------------------------------------------------------- */

/* One query head over N cached tokens of its kv head, all in fp64:
 *   q~ = Pi q,  p = S q~,  kappa = sqrt(pi/2)/m,
 *   l_n = |k_n| (<q~, cK[idx_n]> + rho_n kappa <p, 2 s_n - 1>) / sqrt(d),
 *   w = softmax(l),  o = Pi^T sum_n w_n |v_n| cV[vidx_n].
 * With qjl = 0 the QJL term is absent: l_n = |k_n| <q~, cK[idx_n]> / sqrt(d),
 * the MSE-only estimate. N = 0 gives o = 0. logits (if not NULL) receives l. */
void oracle_attend_head(int d, int N, const uint16_t* q, int q_is_bf16, int qjl,
                        const int8_t* D, const double* S, const float* cK, const float* cV,
                        const uint8_t* kidx, const uint8_t* ksign, const uint16_t* knorm,
                        const uint16_t* rnorm, const uint8_t* vidx, const uint16_t* vnorm,
                        double* o, double* logits)
{
    int m = d;
    double qv[256], qt[256], p[256], acc[256];
    for (int i = 0; i < d; ++i)
        qv[i] = q_is_bf16 ? oracle_bf16_to_double(q[i]) : oracle_half_to_double(q[i]);
    oracle_rotate(d, D, qv, qt);
    for (int j = 0; j < m; ++j) {
        double s = 0.0;
        for (int i = 0; i < d; ++i) s += S[(size_t)j * d + i] * qt[i];
        p[j] = s;
    }
    double kappa = sqrt(M_PI / 2.0) / m, inv_sqrt_d = 1.0 / sqrt((double)d);
    double* l = (double*)malloc(sizeof(double) * (N > 0 ? N : 1));
    double lmax = -INFINITY;
    for (int n = 0; n < N; ++n) {
        double ct = 0.0, st = 0.0;
        for (int i = 0; i < d; ++i) ct += qt[i] * (double)cK[kidx[(size_t)n * d + i]];
        if (qjl)
            for (int j = 0; j < m; ++j) st += (ksign[(size_t)n * m + j] ? 1.0 : -1.0) * p[j];
        double kn = oracle_half_to_double(knorm[n]);
        double rn = qjl ? oracle_half_to_double(rnorm[n]) : 0.0;
        l[n] = kn * (ct + rn * kappa * st) * inv_sqrt_d;
        if (l[n] > lmax) lmax = l[n];
        if (logits) logits[n] = l[n];
    }
    for (int i = 0; i < d; ++i) acc[i] = 0.0;
    double den = 0.0;
    for (int n = 0; n < N; ++n) den += exp(l[n] - lmax);
    for (int n = 0; n < N; ++n) {
        double w = exp(l[n] - lmax) / den * oracle_half_to_double(vnorm[n]);
        for (int i = 0; i < d; ++i) acc[i] += w * (double)cV[vidx[(size_t)n * d + i]];
    }
    oracle_rotate_inverse(d, D, acc, o);
    free(l);
}

/* Batched form over (b, query head): codes are stored per (b, kv head) with a
 * stride of `cap` tokens; query head h reads kv head h / (Hq / Hkv). */
void oracle_attend_batch(int d, int B, int Hq, int Hkv, int cap, const int32_t* seq_len,
                         const uint16_t* q, int q_is_bf16, int qjl, const int8_t* D, const double* S,
                         const float* cK, const float* cV,
                         const uint8_t* kidx, const uint8_t* ksign, const uint16_t* knorm,
                         const uint16_t* rnorm, const uint8_t* vidx, const uint16_t* vnorm,
                         double* out, double* logits)
{
    int g = Hq / Hkv, m = d;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            size_t s = (size_t)b * Hkv + h / g;
            size_t base = s * cap;
            oracle_attend_head(d, seq_len[b], q + ((size_t)b * Hq + h) * d, q_is_bf16, qjl, D, S, cK, cV,
                               kidx + base * d, ksign + base * m, knorm + base, rnorm + base,
                               vidx + base * d, vnorm + base, out + ((size_t)b * Hq + h) * d,
                               logits ? logits + ((size_t)b * Hq + h) * cap : NULL);
        }
}

/* ------------------------------------------------------------------------- */
/* Statistics used by the pins                                                */
/* ------------------------------------------------------------------------- */

/* Monte-Carlo distortion per coordinate of the B-bit codebook on uniformly
 * random unit vectors (Gaussian directions from stream 7): the mean over
 * vectors and coordinates of (y_i - c[idx_i])^2 [MUNINN §Lloyd-Max Codebook]. */
double oracle_distortion_mc(int d, int B, int nvec, uint64_t seed)
{
    float c[TQO_MAXL], t[TQO_MAXL];
    oracle_codebook(B, d, c, t);
    int L = 1 << B;
    double total = 0.0;
#pragma omp parallel for reduction(+ : total) schedule(static)
    for (int v = 0; v < nvec; ++v) {
        double y[256], ss = 0.0;
        for (int i = 0; i < d; ++i) {
            y[i] = oracle_gauss(seed, 7, (uint64_t)v * d + i);
            ss += y[i] * y[i];
        }
        double inv = 1.0 / sqrt(ss), part = 0.0;
        for (int i = 0; i < d; ++i) {
            double yi = y[i] * inv;
            double e = yi - (double)c[oracle_encode(yi, t, L)];
            part += e * e;
        }
        total += part;
    }
    return total / ((double)nvec * d);
}

/* Inner-product estimates of <q, k> over fresh random tables per trial
 * (rotation and S from seed0 + trial, S rounded to fp16 as in the method):
 *  est_mse: |k| <Pi q, c[idx]> with the b-bit MSE codebook alone;
 *  est_qjl: |k| (<Pi q, c[idx]> + rho kappa <S Pi q, 2s-1>) with the
 *           (b-1)-bit codebook plus the 1-bit QJL sketch.
 * Norms are kept in fp64 here: the statistic concerns the estimator. */
void oracle_ip_trials(int d, int bits, int ntrials, uint64_t seed0, const double* q,
                      const double* k, double* est_mse, double* est_qjl)
{
    int m = d;
    float cM[TQO_MAXL], tM[TQO_MAXL], cK[TQO_MAXL], tK[TQO_MAXL];
    oracle_codebook(bits, d, cM, tM);
    if (bits > 1) oracle_codebook(bits - 1, d, cK, tK);
    double kn = 0.0;
    for (int i = 0; i < d; ++i) kn += k[i] * k[i];
    kn = sqrt(kn);
    double kappa = sqrt(M_PI / 2.0) / m;
#pragma omp parallel for schedule(dynamic, 16)
    for (int tr = 0; tr < ntrials; ++tr) {
        uint64_t seed = seed0 + (uint64_t)tr;
        int8_t D[256];
        double u[256], y[256], qt[256], r[256];
        double* S = (double*)malloc(sizeof(double) * m * d);
        oracle_rotation_signs(d, seed, D);
        oracle_qjl_matrix(m, d, seed, S);
        for (int i = 0; i < d; ++i) u[i] = k[i] / kn;
        oracle_rotate(d, D, u, y);
        oracle_rotate(d, D, q, qt);
        double em = 0.0, ec = 0.0, rr = 0.0;
        for (int i = 0; i < d; ++i) {
            em += qt[i] * (double)cM[oracle_encode(y[i], tM, 1 << bits)];
            int id = oracle_encode(y[i], tK, 1 << (bits - 1));
            ec += qt[i] * (double)cK[id];
            r[i] = y[i] - (double)cK[id];
            rr += r[i] * r[i];
        }
        double st = 0.0;
        for (int j = 0; j < m; ++j) {
            double z = 0.0, pj = 0.0;
            for (int i = 0; i < d; ++i) {
                z += S[(size_t)j * d + i] * r[i];
                pj += S[(size_t)j * d + i] * qt[i];
            }
            st += (z >= 0.0 ? 1.0 : -1.0) * pj;
        }
        est_mse[tr] = kn * em;
        est_qjl[tr] = kn * (ec + sqrt(rr) * kappa * st);
        free(S);
    }
}
