// Host-side builders of the codec's data-independent tables: Lloyd-Max
// codebooks, rotation signs, OCTOPUS-QJL projections, and the layout.
//
// The codebooks follow the explainer's "triplet decomposition" and
// "non-uniform bit allocation" sections (Lloyd-Max quantisers for the
// marginals of xi/eta and of the triplet norm, b+1 and b-1 bits) and the
// abstract ("Lloyd-Max quantized against implementation-matched marginals";
// "data-oblivious ... deterministic given a seed").

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "../../include/octopus.h"

namespace {

// ---------------------------------------------------------------------------
// Gauss-Legendre nodes on [-1, 1] by Newton iteration on P_n (the textbook
// construction: start at cos(pi (i - 1/4) / (n + 1/2)), refine with the
// three-term recurrence for P_n and P_n').
// ---------------------------------------------------------------------------
struct GaussLegendre {
  std::vector<double> x, w;
  explicit GaussLegendre(int n) : x(n), w(n) {
    for (int i = 0; i < (n + 1) / 2; ++i) {
      double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));
      double pp = 0.0;
      for (int it = 0; it < 100; ++it) {
        double p1 = 1.0, p2 = 0.0;
        for (int j = 1; j <= n; ++j) {
          double p3 = p2;
          p2 = p1;
          p1 = ((2.0 * j - 1.0) * z * p2 - (j - 1.0) * p3) / j;
        }
        pp = n * (z * p1 - p2) / (z * z - 1.0);
        double dz = p1 / pp;
        z -= dz;
        if (std::fabs(dz) < 1e-16) break;
      }
      x[i] = -z;
      x[n - 1 - i] = z;
      w[i] = w[n - 1 - i] = 2.0 / ((1.0 - z * z) * pp * pp);
    }
  }
};

// Integral of f over [a, b] split into `pieces` equal panels, each with the rule g.
template <class F>
double integrate(const GaussLegendre& g, F f, double a, double b, int pieces) {
  double acc = 0.0;
  const double h = (b - a) / pieces;
  for (int p = 0; p < pieces; ++p) {
    const double lo = a + p * h, half = 0.5 * h;
    for (size_t k = 0; k < g.x.size(); ++k) acc += half * g.w[k] * f(lo + half * (g.x[k] + 1.0));
  }
  return acc;
}

// ---------------------------------------------------------------------------
// Marginal of xi for a uniform direction on S^2 (by symmetry also of eta).
// The joint density of the octahedral coordinates is 1/(4 pi |v|^3) with v
// the unnormalised inverse-map vector (solid angle of a face element of the
// octahedron |x|+|y|+|z| = 1). Integrating over eta in closed form: for
// x = |xi|, on the upper face |eta| <= 1-x, |v|^2 = 2e^2 - 2(1-x)e + x^2 + (1-x)^2;
// on the unfolded part 1-x <= |eta| <= 1, |v|^2 = 2e^2 - 2(2-x)e + 1 + 2(1-x)^2;
// and the antiderivative of (a e^2 + b e + c)^(-3/2) is
// 2(2ae + b) / ((4ac - b^2) sqrt(a e^2 + b e + c)).
// ---------------------------------------------------------------------------
double quad_antiderivative(double e, double a, double b, double c) {
  return 2.0 * (2.0 * a * e + b) / ((4.0 * a * c - b * b) * std::sqrt(a * e * e + b * e + c));
}

double xi_marginal(double xi) {
  const double x = std::fabs(xi), y = 1.0 - x;
  const double b1 = -2.0 * y, c1 = x * x + y * y;
  const double b2 = -2.0 * (2.0 - x), c2 = 1.0 + 2.0 * y * y;
  const double upper = quad_antiderivative(y, 2.0, b1, c1) - quad_antiderivative(0.0, 2.0, b1, c1);
  const double lower = quad_antiderivative(1.0, 2.0, b2, c2) - quad_antiderivative(y, 2.0, b2, c2);
  return (upper + lower) / (2.0 * M_PI);  // both signs of eta: 2 / (4 pi)
}

// Density of the norm of three coordinates of a uniform unit vector in R^d:
// rho^2 ~ Beta(3/2, (d-3)/2).
struct RhoDensity {
  double log_norm, expo;
  explicit RhoDensity(int d) {
    const double a = 1.5, b = 0.5 * (d - 3);
    log_norm = std::log(2.0) - (std::lgamma(a) + std::lgamma(b) - std::lgamma(a + b));
    expo = 0.5 * (d - 5);
  }
  double operator()(double r) const {
    const double one = 1.0 - r * r;
    if (one <= 0.0 || r <= 0.0) return 0.0;
    return std::exp(log_norm + 2.0 * std::log(r) + expo * std::log(one));
  }
};

// One-dimensional Lloyd-Max on [lo, hi] with a kink-free density except at
// `kink` (panels are split there). Alternates the two optimality
// conditions (midpoint thresholds, conditional-mean centroids) until no
// centroid moves by more than tol.
template <class F>
void lloyd_max(F pdf, double lo, double hi, double kink, int levels, double tol,
               std::vector<double>& c, std::vector<double>& t) {
  static const GaussLegendre g(40);
  c.assign(levels, 0.0);
  t.assign(levels - 1, 0.0);
  // start: equal-width cells
  for (int k = 0; k < levels - 1; ++k) t[k] = lo + (hi - lo) * (k + 1) / levels;
  auto moments = [&](double a, double b, double& m0, double& m1) {
    m0 = m1 = 0.0;
    double pts[3] = {a, b, b};
    int np = 2;
    if (kink > a && kink < b) { pts[1] = kink; pts[2] = b; np = 3; }
    for (int s = 0; s + 1 < np; ++s) {
      const double u = pts[s], v = pts[s + 1];
      const int pieces = 1 + static_cast<int>((v - u) / (hi - lo) * 64.0);
      m0 += integrate(g, pdf, u, v, pieces);
      m1 += integrate(g, [&](double x) { return x * pdf(x); }, u, v, pieces);
    }
  };
  auto centroids = [&]() {
    std::vector<double> out(levels);
    for (int k = 0; k < levels; ++k) {
      const double a = k == 0 ? lo : t[k - 1], b = k == levels - 1 ? hi : t[k];
      double m0, m1;
      moments(a, b, m0, m1);
      out[k] = m0 > 0.0 ? m1 / m0 : 0.5 * (a + b);
    }
    return out;
  };
  c = centroids();
  for (int it = 0; it < 1000000; ++it) {
    for (int k = 0; k < levels - 1; ++k) t[k] = 0.5 * (c[k] + c[k + 1]);
    std::vector<double> cn = centroids();
    double delta = 0.0;
    for (int k = 0; k < levels; ++k) delta = std::fmax(delta, std::fabs(cn[k] - c[k]));
    c.swap(cn);
    if (delta < tol) break;
  }
  for (int k = 0; k < levels - 1; ++k) t[k] = 0.5 * (c[k] + c[k + 1]);
}

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

// Output number n (n >= 1) of SplitMix64 seeded with `seed` (Steele, Lea,
// Flood 2014; finaliser constants as published by Vigna).
inline uint64_t splitmix64_at(uint64_t seed, uint64_t n) {
  uint64_t z = seed + n * kGolden;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

bool supported_d(int d) { return d == 64 || d == 128 || d == 256; }

}  // namespace

extern "C" int octo_layout_init_delta(octo_layout* L, int d, int b, int delta, int qjl, int rounding) {
  if (!L) return OCTO_EINVAL;
  if ((qjl != 0 && qjl != 1) || (rounding != OCTO_ROUND_SCALAR && rounding != OCTO_ROUND_JOINT))
    return OCTO_EINVAL;
  if (!supported_d(d) || b < 2 || b > 4) return OCTO_EUNSUPPORTED;
  const int b_dir = b + delta, b_rho = b - delta;
  if (b_dir < 2 || b_dir > 5 || b_rho < 1 || b_rho > 5) return OCTO_EUNSUPPORTED;
  if (qjl && delta != 1) return OCTO_EUNSUPPORTED;  // the sketch is kept for the OCTOPUS split only
  std::memset(L, 0, sizeof(*L));
  L->d = d;
  L->b = b;
  L->T = (d + 2) / 3;
  L->b_dir = b_dir;
  L->b_rho = b_rho;
  L->code_bits = 2 * b_dir + b_rho;
  L->words = (L->T * L->code_bits + 31) / 32;
  L->n_dir = 1 << L->b_dir;
  L->n_rho = 1 << L->b_rho;
  L->qjl = qjl;
  L->qjl_words = qjl ? d / 32 : 0;
  L->rounding = rounding;
  return OCTO_OK;
}

extern "C" int octo_layout_init(octo_layout* L, int d, int b, int qjl, int rounding) {
  return octo_layout_init_delta(L, d, b, 1, qjl, rounding);
}

extern "C" int octo_codebook_build(const octo_layout* L, float* dir_c, float* dir_t, float* rho_c,
                                   float* rho_t) {
  if (!L || !dir_c || !dir_t || !rho_c || !rho_t) return OCTO_EINVAL;
  if (!supported_d(L->d) || L->b < 2 || L->b > 4) return OCTO_EUNSUPPORTED;
  octo_layout chk;
  const int lc = octo_layout_init_delta(&chk, L->d, L->b, L->b_dir - L->b, L->qjl, L->rounding);
  if (lc != OCTO_OK) return lc;
  if (chk.b_rho != L->b_rho || chk.n_dir != L->n_dir || chk.n_rho != L->n_rho) return OCTO_EINVAL;
  try {
    std::vector<double> c, t;
    lloyd_max(xi_marginal, -1.0, 1.0, 0.0, L->n_dir, 1e-14, c, t);
    const int n = L->n_dir;
    for (int k = 0; k < n; ++k) dir_c[k] = static_cast<float>(0.5 * (c[k] - c[n - 1 - k]));
    for (int k = 0; k < n - 1; ++k) {
      const double a = 0.5 * (c[k] - c[n - 1 - k]), b = 0.5 * (c[k + 1] - c[n - 2 - k]);
      dir_t[k] = static_cast<float>(0.5 * (a + b));
    }
    RhoDensity f(L->d);
    lloyd_max(f, 0.0, 1.0, -1.0, L->n_rho, 1e-15, c, t);
    for (int k = 0; k < L->n_rho; ++k) rho_c[k] = static_cast<float>(c[k]);
    for (int k = 0; k < L->n_rho - 1; ++k) rho_t[k] = static_cast<float>(t[k]);
  } catch (...) {
    return OCTO_EINVAL;
  }
  return OCTO_OK;
}

extern "C" int octo_rotation_build(uint64_t seed, int d, int64_t n_heads, float* signs) {
  if (!signs || n_heads < 1) return OCTO_EINVAL;
  if (!supported_d(d)) return OCTO_EUNSUPPORTED;
  const uint64_t n = static_cast<uint64_t>(n_heads) * static_cast<uint64_t>(d);
  for (uint64_t e = 0; e < n; ++e) signs[e] = (splitmix64_at(seed, e + 1) >> 63) ? -1.0f : 1.0f;
  return OCTO_OK;
}

extern "C" int octo_qjl_build(uint64_t seed, int d, int64_t n_heads, float* S) {
  if (!S || n_heads < 1) return OCTO_EINVAL;
  if (!supported_d(d)) return OCTO_EUNSUPPORTED;
  const uint64_t n = static_cast<uint64_t>(n_heads) * d * d;
  const double two_pi = 2.0 * M_PI;
  for (uint64_t e = 0; e < n; ++e) {
    const uint64_t z1 = splitmix64_at(seed, 2 * e + 1), z2 = splitmix64_at(seed, 2 * e + 2);
    const double u1 = (static_cast<double>(z1 >> 11) + 1.0) * 0x1.0p-53;
    const double u2 = static_cast<double>(z2 >> 11) * 0x1.0p-53;
    S[e] = static_cast<float>(std::sqrt(-2.0 * std::log(u1)) * std::cos(two_pi * u2));
  }
  return OCTO_OK;
}

extern "C" const char* octo_status_string(int status) {
  switch (status) {
    case OCTO_OK: return "OCTO_OK";
    case OCTO_EINVAL: return "OCTO_EINVAL: invalid argument";
    case OCTO_EUNSUPPORTED: return "OCTO_EUNSUPPORTED: shape outside the supported set";
    case OCTO_ECUDA: return "OCTO_ECUDA: CUDA launch or runtime error";
    case OCTO_EWORKSPACE: return "OCTO_EWORKSPACE: workspace too small";
    default: return "unknown octo status";
  }
}

extern "C" int octo_abi_version(void) { return 102; }
