// Host-side tables of the TurboQuant method: Lloyd–Max codebooks, the random
// sign diagonal D and the QJL matrix S ("[Benchmark] TurboQuant 實測：KV Cache
// 3-bit 壓縮，真的零損失？", ai-muninn.com, §"TurboQuant 是什麼：30 秒懶人包"
// and §"Lloyd-Max Codebook"; "turboquant-kvquant-vllm-benchmark",
// ai-coding.wiselychen.com, §"TurboQuant 是什麼", steps 1-3).
//
// Everything here runs once per context, in fp64, on the host.
#include "tables.h"

#include <cmath>
#include <cstring>

namespace tq {
namespace {

constexpr double kPi = 3.14159265358979323846;

// ---------------------------------------------------------------- generator
// SplitMix64: the state advances by the golden-ratio increment and each output
// is the state passed through a two-round xor-shift-multiply finalizer. A table
// stream s is the generator started at seed ^ (0x5851F42D4C957F2D * (s + 1));
// draw k of the stream is its output number k + 1, so any draw can be computed
// directly from its index.
struct SplitMix64 {
    static constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;
    static uint64_t finalize(uint64_t x)
    {
        x ^= x >> 30;
        x *= 0xBF58476D1CE4E5B9ull;
        x ^= x >> 27;
        x *= 0x94D049BB133111EBull;
        x ^= x >> 31;
        return x;
    }
    static uint64_t at(uint64_t seed, unsigned stream, uint64_t k)
    {
        const uint64_t origin = seed ^ (0x5851F42D4C957F2Dull * (uint64_t(stream) + 1u));
        return finalize(origin + (k + 1u) * kGamma);
    }
};

// Two N(0,1) values from draws 2q and 2q+1 of a stream (Box–Muller on 53-bit
// uniforms u1 in (0,1], u2 in [0,1)).
void normal_pair(uint64_t seed, unsigned stream, uint64_t q, double& z0, double& z1)
{
    const double u1 = (double(SplitMix64::at(seed, stream, 2 * q) >> 11) + 1.0) * 0x1p-53;
    const double u2 = double(SplitMix64::at(seed, stream, 2 * q + 1) >> 11) * 0x1p-53;
    const double radius = std::sqrt(-2.0 * std::log(u1));
    const double angle = 2.0 * kPi * u2;
    z0 = radius * std::cos(angle);
    z1 = radius * std::sin(angle);
}

// ---------------------------------------------------------------- fp16 rounding
// Round a double to the nearest IEEE binary16 value (ties to even) and return
// that value as a double. Works on the binary64 fields directly.
double round_to_half(double v)
{
    if (!(std::fabs(v) < 65520.0)) return std::copysign(INFINITY, v);  // overflow / NaN guard
    if (v == 0.0) return v;
    int exp2;
    std::frexp(std::fabs(v), &exp2);            // |v| in [2^(exp2-1), 2^exp2)
    int lsb_exp = (exp2 - 1) - 10;              // weight of the last kept mantissa bit
    if (lsb_exp < -24) lsb_exp = -24;           // subnormal halves share the 2^-24 step
    const double steps = std::ldexp(v, -lsb_exp);
    double r = std::floor(steps);
    const double frac = steps - r;              // exact: steps has < 53 significant bits
    if (frac > 0.5 || (frac == 0.5 && std::fmod(r, 2.0) != 0.0)) r += 1.0;
    return std::ldexp(r, lsb_exp);
}

// ---------------------------------------------------------------- Lloyd–Max
double std_normal_pdf(double x) { return std::exp(-0.5 * x * x) * 0.39894228040143267794; }
double std_normal_cdf(double x) { return 0.5 * std::erfc(-x * 0.70710678118654752440); }

// Levels of the minimum-MSE quantizer of N(0,1) with n = 2^B cells (Lloyd's
// fixed point: cell edges halfway between levels, each level the mean of the
// density over its cell). Iterated to fp64 convergence, then made exactly
// antisymmetric.
bool gaussian_lloyd_max(int B, double* level)
{
    const int n = 1 << B;
    for (int j = 0; j < n; ++j) level[j] = 3.0 * (2.0 * j + 1.0 - n) / (2.0 * n);
    double edge[kMaxLevels + 1];
    bool converged = false;
    double last_step = INFINITY;
    for (int iter = 0; iter < 4000000 && !converged; ++iter) {
        edge[0] = -INFINITY;
        edge[n] = INFINITY;
        for (int j = 1; j < n; ++j) edge[j] = 0.5 * (level[j - 1] + level[j]);
        double moved = 0.0;
        for (int j = 0; j < n; ++j) {
            const double dens_lo = (j == 0) ? 0.0 : std_normal_pdf(edge[j]);
            const double dens_hi = (j == n - 1) ? 0.0 : std_normal_pdf(edge[j + 1]);
            const double mass = std_normal_cdf(edge[j + 1]) - std_normal_cdf(edge[j]);
            const double updated = (dens_lo - dens_hi) / mass;
            moved = std::fmax(moved, std::fabs(updated - level[j]));
            level[j] = updated;
        }
        // Lloyd's map contracts linearly near the optimum; once steps are
        // below 1e-12, run to the fp64 noise floor (the step stops shrinking).
        converged = moved == 0.0 || (moved < 1e-12 && moved >= last_step);
        last_step = moved;
    }
    for (int j = 0; j < n / 2; ++j) {
        const double a = 0.5 * (level[n - 1 - j] - level[j]);
        level[j] = -a;
        level[n - 1 - j] = a;
    }
    return converged;
}

// Regularized incomplete beta I_x(p, p) for x <= 1/2, by the continued
// fraction of the incomplete beta function (Abramowitz & Stegun 26.5.8)
// evaluated with the modified Lentz method.
double incomplete_beta_sym(double p, double x)
{
    if (x <= 0.0) return 0.0;
    const double a = p, b = p, tiny = 1e-300;
    // I_x(a, b) = x^a (1-x)^b / (a B(a, b)) / g with
    // g = 1 + e1 / (1 + e2 / (1 + ...)), e_{2m+1} = -(a+m)(a+b+m)x / ((a+2m)(a+2m+1)),
    // e_{2m} = m(b-m)x / ((a+2m-1)(a+2m)); Lentz: f = g, C and Dn the running ratios.
    double f = 1.0, C = 1.0, Dn = 0.0;
    for (int i = 1; i <= 100000; ++i) {
        const int m = i / 2;
        const double e = (i & 1) ? -(a + m) * (a + b + m) * x / ((a + 2 * m) * (a + 2 * m + 1))
                                 : m * (b - m) * x / ((a + 2 * m - 1) * (a + 2 * m));
        Dn = 1.0 + e * Dn;
        if (std::fabs(Dn) < tiny) Dn = tiny;
        C = 1.0 + e / C;
        if (std::fabs(C) < tiny) C = tiny;
        Dn = 1.0 / Dn;
        const double step = C * Dn;
        f *= step;
        if (std::fabs(step - 1.0) < 1e-16) break;
    }
    const double front = std::exp(std::lgamma(a + b) - std::lgamma(a) - std::lgamma(b) +
                                  a * std::log(x) + b * std::log1p(-x));
    return front / (a * f);
}

}  // namespace

// Lloyd–Max for the exact marginal of one coordinate of a random unit vector
// in R^d: (1 + y)/2 ~ Beta(p, p), p = (d-1)/2, density c_d (1 - y^2)^((d-3)/2).
// Cell mass from the incomplete beta function (by symmetry always evaluated on
// the lower half), first moment in closed form:
//   int y (1-y^2)^al dy = -(1-y^2)^(al+1) / (2 (al+1)),  al = (d-3)/2.
// Starting point and stopping rule as for the Gaussian iteration.
bool beta_lloyd_max(int B, int d, double* level)
{
    const int n = 1 << B;
    const double p = 0.5 * (d - 1), al = 0.5 * (d - 3);
    const double logc = std::lgamma(0.5 * d) - 0.5 * std::log(M_PI) - std::lgamma(0.5 * (d - 1));
    auto lower = [&](double t) {   // P(y <= t) for t <= 0
        return incomplete_beta_sym(p, 0.5 * (1.0 + t));
    };
    auto mass = [&](double lo, double hi) {   // P(lo < y < hi), -1 <= lo < hi <= 1
        if (hi <= 0.0) return lower(hi) - lower(lo);
        if (lo >= 0.0) return lower(-lo) - lower(-hi);
        return (0.5 - lower(lo)) + (0.5 - lower(-hi));
    };
    auto first = [&](double lo, double hi) {   // E[y; lo < y < hi]
        const double plo = std::exp(logc + (al + 1.0) * std::log1p(-lo * lo));
        const double phi = std::exp(logc + (al + 1.0) * std::log1p(-hi * hi));
        return (plo - phi) / (2.0 * (al + 1.0));
    };
    if (d >= 16) {
        gaussian_lloyd_max(B, level);
        for (int j = 0; j < n; ++j) level[j] /= std::sqrt(double(d));
    } else {
        for (int j = 0; j < n; ++j) level[j] = -1.0 + (2.0 * j + 1.0) / n;
    }
    bool converged = false;
    double last_step = INFINITY;
    for (int iter = 0; iter < 100000 && !converged; ++iter) {
        double moved = 0.0, next[kMaxLevels];
        for (int j = 0; j < n; ++j) {
            const double lo = (j == 0) ? -1.0 : 0.5 * (level[j - 1] + level[j]);
            const double hi = (j == n - 1) ? 1.0 : 0.5 * (level[j] + level[j + 1]);
            next[j] = first(lo, hi) / mass(lo, hi);
            moved = std::fmax(moved, std::fabs(next[j] - level[j]));
        }
        for (int j = 0; j < n; ++j) level[j] = next[j];
        converged = moved == 0.0 || (moved < 1e-13 && moved >= last_step);
        last_step = moved;
    }
    for (int j = 0; j < n / 2; ++j) {
        const double a = 0.5 * (level[n - 1 - j] - level[j]);
        level[j] = -a;
        level[n - 1 - j] = a;
    }
    return converged;
}

bool build_codebook_beta(int B, int d, float* centroids, float* bounds)
{
    double level[kMaxLevels];
    const bool ok = beta_lloyd_max(B, d, level);
    const int n = 1 << B;
    for (int j = 0; j < n; ++j) centroids[j] = float(level[j]);
    for (int j = 0; j + 1 < n; ++j)
        bounds[j] = float((double(centroids[j]) + double(centroids[j + 1])) * 0.5);
    return ok;
}

bool build_codebook(int B, int d, float* centroids, float* bounds)
{
    double unit[kMaxLevels];
    const bool ok = gaussian_lloyd_max(B, unit);
    const int n = 1 << B;
    const double scale = 1.0 / std::sqrt(double(d));
    for (int j = 0; j < n; ++j) centroids[j] = float(unit[j] * scale);
    for (int j = 0; j + 1 < n; ++j)
        bounds[j] = float((double(centroids[j]) + double(centroids[j + 1])) * 0.5);
    return ok;
}

void build_rotation_signs(int d, uint64_t seed, int8_t* signs)
{
    for (int i = 0; i < d; ++i) signs[i] = (SplitMix64::at(seed, 0, uint64_t(i)) >> 63) ? -1 : 1;
}

void build_qjl_matrix(int m, int d, uint64_t seed, float* S)
{
    const uint64_t count = uint64_t(m) * uint64_t(d);
    for (uint64_t e = 0; e < count; e += 2) {
        double z0, z1;
        normal_pair(seed, 1, e / 2, z0, z1);
        S[e] = float(round_to_half(z0));
        S[e + 1] = float(round_to_half(z1));
    }
}

// Relative distance from v > 0 to the nearest IEEE binary16 value (normal range).
static double half_rel_error(double v)
{
    int e;
    std::frexp(v, &e);                          // v in [2^(e-1), 2^e)
    const double steps = std::ldexp(v, 11 - e); // the half spacing there is 2^(e-11)
    return std::fabs(steps - std::nearbyint(steps)) / steps;
}

float choose_decode_scale(const float* centroids, int n, int d)
{
    // The attention kernel decodes codes to fp16 tensor-core operands. A common
    // scale alpha in [1, 2) of the (unit-variance) levels, searched on a 2^-21
    // grid, makes the positive levels land almost on fp16 values; the query
    // operand carries 1/alpha, so the product is unchanged.
    const double sd = std::sqrt(double(d));
    double best = 1.0, best_err = INFINITY;
    for (int k = 0; k < (1 << 21); ++k) {
        const double alpha = 1.0 + std::ldexp(double(k), -21);
        double err = 0.0;
        for (int j = n / 2; j < n && err < best_err; ++j)
            err = std::fmax(err, half_rel_error(double(float(double(centroids[j]) * sd * alpha))));
        if (err < best_err) {
            best_err = err;
            best = alpha;
        }
    }
    return float(best);
}

bool build_host_tables(int d, int kbits, int vbits, int qjl, int codebook, uint64_t seed,
                       HostTables& t)
{
    t.d = d;
    t.bits = vbits;
    t.m = d;
    t.kbits = kbits;
    t.vbits = vbits;
    t.qjl = qjl;
    t.centroids_k.assign(1u << t.kbits, 0.f);
    t.bounds_k.assign((1u << t.kbits) - 1, 0.f);
    t.centroids_v.assign(1u << t.vbits, 0.f);
    t.bounds_v.assign((1u << t.vbits) - 1, 0.f);
    t.signs.assign(d, 1);
    t.S.assign(size_t(t.m) * d, 0.f);
    auto cb = codebook == 1 ? build_codebook_beta : build_codebook;
    t.codebook = codebook;
    bool ok = cb(t.kbits, d, t.centroids_k.data(), t.bounds_k.data());
    ok = cb(t.vbits, d, t.centroids_v.data(), t.bounds_v.data()) && ok;
    build_rotation_signs(d, seed, t.signs.data());
    build_qjl_matrix(t.m, d, seed, t.S.data());
    // cells of more than 4 bits are decoded as fp16 hi + lo parts: no scale needed
    t.alpha_k = t.kbits > 4 ? 1.f : choose_decode_scale(t.centroids_k.data(), 1 << t.kbits, d);
    return ok;
}

}  // namespace tq
