// Host-side parameter setup (float64): random streams, Lloyd-Max codebooks (the
// coordinate codebook and the PolarQuant angle codebooks), unit rotors, the random
// orthogonal rotation Pi and the QJL matrix.
//
// These run once, off the hot path ("pack_rotors_for_triton ... one-time,
// ~0 cost" in "TurboQuant + RotorQuant", section "Usage"); the caller rounds
// the results to the device types and uploads them.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#include "kvrq.h"
#include "kvrq_internal.h"

namespace kvrq {

// ---------------------------------------------------------------- random streams
// splitmix64 (Steele, Lea, Flood, OOPSLA 2014) used as a counter-based
// generator: output k of stream s is mix64(s + (k + 1) * golden_gamma).
static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static inline uint64_t stream_output(uint64_t seed, uint64_t k) {
  return mix64(seed + (k + 1) * 0x9E3779B97F4A7C15ull);
}

// uniform in (0, 1]
static inline double stream_uniform(uint64_t seed, uint64_t k) {
  return (double)((stream_output(seed, k) >> 11) + 1) * 0x1.0p-53;
}

// normal number i: Box-Muller on uniforms 2j and 2j+1 (j = i / 2)
double stream_normal(uint64_t seed, uint64_t i) {
  const uint64_t j = i >> 1;
  const double u1 = stream_uniform(seed, 2 * j);
  const double u2 = stream_uniform(seed, 2 * j + 1);
  const double r = std::sqrt(-2.0 * std::log(u1));
  const double a = 2.0 * M_PI * u2;
  return (i & 1) ? r * std::sin(a) : r * std::cos(a);
}

// ---------------------------------------------------------------- incomplete beta
// Regularized incomplete beta I_x(a, b) by its continued fraction
// (Abramowitz & Stegun 26.5.8), evaluated with the modified Lentz method;
// for x above (a+1)/(a+b+2) the symmetry I_x(a,b) = 1 - I_{1-x}(b,a) is used.
static double beta_cf(double x, double a, double b) {
  const double tiny = 1e-300;
  double c = 1.0;
  double dd = 1.0 - (a + b) * x / (a + 1.0);
  if (std::fabs(dd) < tiny) dd = tiny;
  dd = 1.0 / dd;
  double f = dd;
  for (int m = 1; m <= 100000; ++m) {
    // even term d_{2m}
    double num = m * (b - m) * x / ((a + 2.0 * m - 1.0) * (a + 2.0 * m));
    dd = 1.0 + num * dd;
    if (std::fabs(dd) < tiny) dd = tiny;
    c = 1.0 + num / c;
    if (std::fabs(c) < tiny) c = tiny;
    dd = 1.0 / dd;
    f *= dd * c;
    // odd term d_{2m+1}
    num = -(a + m) * (a + b + m) * x / ((a + 2.0 * m) * (a + 2.0 * m + 1.0));
    dd = 1.0 + num * dd;
    if (std::fabs(dd) < tiny) dd = tiny;
    c = 1.0 + num / c;
    if (std::fabs(c) < tiny) c = tiny;
    dd = 1.0 / dd;
    const double delta = dd * c;
    f *= delta;
    if (std::fabs(delta - 1.0) < 1e-16) break;
  }
  return f;
}

static double ibeta(double x, double a, double b) {
  if (x <= 0.0) return 0.0;
  if (x >= 1.0) return 1.0;
  const double lfront = std::lgamma(a + b) - std::lgamma(a) - std::lgamma(b) + a * std::log(x) +
                        b * std::log1p(-x);
  if (x < (a + 1.0) / (a + b + 2.0)) return std::exp(lfront) * beta_cf(x, a, b) / a;
  return 1.0 - std::exp(lfront) * beta_cf(1.0 - x, b, a) / b;
}

// ---------------------------------------------------------------- coordinate density
// One coordinate X of a uniform unit vector in R^d: X^2 ~ Beta(1/2, (d-1)/2), so
// P(X <= x) = 1/2 + sign(x)/2 * I_{x^2}(1/2, (d-1)/2) and, with
// f(x) = C_d (1-x^2)^((d-3)/2), int x f = -C_d (1-x^2)^((d-1)/2) / (d-1).
struct CoordDensity {
  int d;
  double c_d;
  explicit CoordDensity(int d_) : d(d_) {
    c_d = std::exp(std::lgamma(0.5 * d) - std::lgamma(0.5 * (d - 1))) / std::sqrt(M_PI);
  }
  double cdf(double x) const {
    if (x <= -1.0) return 0.0;
    if (x >= 1.0) return 1.0;
    const double h = 0.5 * ibeta(x * x, 0.5, 0.5 * (d - 1));
    return x >= 0.0 ? 0.5 + h : 0.5 - h;
  }
  double first_moment(double a, double b) const {  // int_a^b x f(x) dx
    a = std::max(-1.0, std::min(1.0, a));
    b = std::max(-1.0, std::min(1.0, b));
    const double e = 0.5 * (d - 1);
    return c_d * (std::pow(1.0 - a * a, e) - std::pow(1.0 - b * b, e)) / (2.0 * e);
  }
};

// ---------------------------------------------------------------- PolarQuant angle density
// ["TurboQuant и PolarQuant", "Полярное преобразование"]: an angle of level l >= 2
// pairs the norms of two k = 2^(l-1)-dimensional Gaussian sub-vectors and has density
// Gamma(k) / (2^(k-2) Gamma(k/2)^2) sin^(k-1)(2 theta) on [0, pi/2]. With
// u = sin^2 theta this is u ~ Beta(k/2, k/2), so P(Theta <= t) = I_{sin^2 t}(k/2, k/2).
// The first moment of a cell follows by parts: int_a^b t f = [t F]_a^b - int_a^b F,
// the last integral by adaptive Simpson quadrature of the smooth, monotone F.
struct AngleDensity {
  double k;
  explicit AngleDensity(int k_) : k(k_) {}
  double cdf(double t) const {
    if (t <= 0.0) return 0.0;
    if (t >= 0.5 * M_PI) return 1.0;
    const double s = std::sin(t);
    return ibeta(s * s, 0.5 * k, 0.5 * k);
  }
  double simpson(double a, double b, double fa, double fm, double fb, double whole, double eps, int depth) const {
    const double m = 0.5 * (a + b), lm = 0.5 * (a + m), rm = 0.5 * (m + b);
    const double flm = cdf(lm), frm = cdf(rm);
    const double left = (m - a) / 6.0 * (fa + 4.0 * flm + fm), right = (b - m) / 6.0 * (fm + 4.0 * frm + fb);
    const double diff = left + right - whole;
    if (depth <= 0 || std::fabs(diff) <= 15.0 * eps) return left + right + diff / 15.0;
    const double e2 = std::max(0.5 * eps, 1e-18);  // below rounding, halving only forces depth
    return simpson(a, m, fa, flm, fm, left, e2, depth - 1) + simpson(m, b, fm, frm, fb, right, e2, depth - 1);
  }
  double first_moment(double a, double b) const {  // int_a^b t f(t) dt
    const double fa = cdf(a), fb = cdf(b), fm = cdf(0.5 * (a + b));
    const double whole = (b - a) / 6.0 * (fa + 4.0 * fm + fb);
    return b * fb - a * fa - simpson(a, b, fa, fm, fb, whole, 1e-15, 24);
  }
};

}  // namespace kvrq

using namespace kvrq;

extern "C" {

int64_t kvrq_packed_words(int64_t n_codes, int bits) {
  if (n_codes < 0 || bits < 1 || bits > 32) return -1;
  return (n_codes * bits + 31) / 32;
}

int kvrq_rq_groups(int d) { return d < 1 ? -1 : (d + 2) / 3; }

kvrq_status kvrq_normals(uint64_t seed, int64_t first, int64_t count, double* out) {
  if (first < 0 || count < 0 || (count > 0 && !out)) return set_error(KVRQ_EINVAL, "kvrq_normals: bad arguments");
  for (int64_t k = 0; k < count; ++k) out[k] = stream_normal(seed, (uint64_t)(first + k));
  return KVRQ_OK;
}

static kvrq_status tq_codebook_init_body(int d, int bits, double tol, int max_iter, double* centroids,
                             double* boundaries, int* iterations) {
  if (d < 2) return set_error(KVRQ_EINVAL, "tq_codebook_init: d must be >= 2");
  if (bits < 1 || bits > 8) return set_error(KVRQ_EINVAL, "tq_codebook_init: bits must be in 1..8");
  if (!(tol > 0.0) || max_iter < 1 || !centroids)
    return set_error(KVRQ_EINVAL, "tq_codebook_init: bad tol/max_iter/centroids");
  const int K = 1 << bits;
  const CoordDensity f(d);
  // Start from an evenly spaced grid over +-3 standard deviations (1/sqrt(d)),
  // kept inside (-1, 1). The density is log-concave, so Lloyd's fixed point is
  // unique and any start reaches it.
  std::vector<double> c(K), lo(K), hi(K);
  const double span = std::min(3.0 / std::sqrt((double)d), 0.999);
  for (int k = 0; k < K; ++k) c[k] = span * (2.0 * k + 1.0 - K) / K;
  int it = 0;
  bool converged = false;
  while (it < max_iter) {
    ++it;
    for (int k = 0; k < K; ++k) {
      lo[k] = k == 0 ? -1.0 : 0.5 * (c[k - 1] + c[k]);
      hi[k] = k == K - 1 ? 1.0 : 0.5 * (c[k] + c[k + 1]);
    }
    double delta = 0.0;
    for (int k = 0; k < K; ++k) {
      const double mass = f.cdf(hi[k]) - f.cdf(lo[k]);
      const double cn = f.first_moment(lo[k], hi[k]) / mass;
      delta = std::max(delta, std::fabs(cn - c[k]));
      c[k] = cn;
    }
    if (delta < tol) {
      converged = true;
      break;
    }
  }
  // the density is even: make the symmetry exact
  std::vector<double> s(K);
  for (int k = 0; k < K; ++k) s[k] = 0.5 * (c[k] - c[K - 1 - k]);
  for (int k = 0; k < K; ++k) centroids[k] = s[k];
  if (boundaries)
    for (int k = 0; k + 1 < K; ++k) boundaries[k] = 0.5 * (s[k] + s[k + 1]);
  if (iterations) *iterations = it;
  if (!converged) return set_error(KVRQ_ENOCONV, "tq_codebook_init: Lloyd-Max did not converge");
  return KVRQ_OK;
}

static kvrq_status pq_angle_codebook_init_body(int level, int bits, double tol, int max_iter, double* centroids,
                                   double* boundaries, int* iterations) {
  if (level < 1 || level > 20) return set_error(KVRQ_EINVAL, "pq_angle_codebook_init: level must be in 1..20");
  if (bits < 1 || bits > 8) return set_error(KVRQ_EINVAL, "pq_angle_codebook_init: bits must be in 1..8");
  if (!(tol > 0.0) || max_iter < 1 || !centroids)
    return set_error(KVRQ_EINVAL, "pq_angle_codebook_init: bad tol/max_iter/centroids");
  const int K = 1 << bits;
  std::vector<double> c(K);
  int it = 0;
  bool converged = false;
  if (level == 1) {
    // uniform on [0, 2 pi): the cells of an even grid are their own fixed point
    for (int k = 0; k < K; ++k) c[k] = (2.0 * k + 1.0) * M_PI / K;
    it = 1;
    converged = true;
  } else {
    const AngleDensity f(1 << (level - 1));
    const double hi_end = 0.5 * M_PI;
    for (int k = 0; k < K; ++k) c[k] = (k + 0.5) * hi_end / K;  // even start; the fixed point is unique
    std::vector<double> lo(K), hi(K);
    while (it < max_iter) {
      ++it;
      for (int k = 0; k < K; ++k) {
        lo[k] = k == 0 ? 0.0 : 0.5 * (c[k - 1] + c[k]);
        hi[k] = k == K - 1 ? hi_end : 0.5 * (c[k] + c[k + 1]);
      }
      double delta = 0.0;
      for (int k = 0; k < K; ++k) {
        const double mass = f.cdf(hi[k]) - f.cdf(lo[k]);
        const double cn = f.first_moment(lo[k], hi[k]) / mass;
        delta = std::max(delta, std::fabs(cn - c[k]));
        c[k] = cn;
      }
      if (delta < tol) {
        converged = true;
        break;
      }
    }
    // the density is symmetric about pi/4: make c[k] + c[K-1-k] = pi/2 exact
    std::vector<double> s(K);
    for (int k = 0; k < K; ++k) s[k] = 0.5 * (c[k] + (hi_end - c[K - 1 - k]));
    c = s;
  }
  for (int k = 0; k < K; ++k) centroids[k] = c[k];
  if (boundaries)
    for (int k = 0; k + 1 < K; ++k) boundaries[k] = 0.5 * (c[k] + c[k + 1]);
  if (iterations) *iterations = it;
  if (!converged) return set_error(KVRQ_ENOCONV, "pq_angle_codebook_init: Lloyd iteration did not converge");
  return KVRQ_OK;
}

kvrq_status rq_rotors_init(int d, uint64_t seed, double* rotors) {
  if (d < 1 || !rotors) return set_error(KVRQ_EINVAL, "rq_rotors_init: d >= 1 and rotors != NULL");
  const int G = (d + 2) / 3;
  for (int g = 0; g < G; ++g) {
    double r[4], ss = 0.0;
    for (int i = 0; i < 4; ++i) {
      r[i] = stream_normal(seed, (uint64_t)(4 * g + i));
      ss += r[i] * r[i];
    }
    const double inv = 1.0 / std::sqrt(ss);
    for (int i = 0; i < 4; ++i) rotors[4 * g + i] = r[i] * inv;
  }
  return KVRQ_OK;
}

kvrq_status qjl_matrix_init(int m, int d, uint64_t seed, double* T) {
  if (m < 1 || d < 1 || !T) return set_error(KVRQ_EINVAL, "qjl_matrix_init: m, d >= 1 and T != NULL");
  const int64_t total = (int64_t)m * d;
  for (int64_t k = 0; k < total; ++k) T[k] = stream_normal(seed, (uint64_t)k);
  return KVRQ_OK;
}

// Householder QR of the d x d Gaussian matrix A (row-major, in place):
// for column k, v = x - alpha e1 with alpha = -sign(x0) ||x||, and the
// trailing block is updated as A <- (I - 2 v v^T / v^T v) A. R_kk = alpha.
// Q = H_0 H_1 ... H_{d-1} is formed by applying the reflectors to I in
// reverse order. Pi = Q diag(sign(R_kk)).
static kvrq_status tq_rotation_init_body(int d, uint64_t seed, double* pi) {
  if (d < 1 || d > 16384 || !pi) return set_error(KVRQ_EINVAL, "tq_rotation_init: 1 <= d <= 16384, pi != NULL");
  const int64_t n = d;
  std::vector<double> A((size_t)(n * n));
  for (int64_t k = 0; k < n * n; ++k) A[(size_t)k] = stream_normal(seed, (uint64_t)k);
  std::vector<double> V((size_t)(n * n), 0.0);  // reflector k in V[k][k..n)
  std::vector<double> rdiag((size_t)n);
  const unsigned hw = std::max(1u, std::min(16u, std::thread::hardware_concurrency()));
  // rows [r0, r1) of a block update, run on several threads for large d
  auto parallel_rows = [&](int64_t r0, int64_t r1, auto&& fn) {
    const int64_t rows = r1 - r0;
    const int64_t nt = (rows * (n - r0) > (1 << 18)) ? (int64_t)hw : 1;
    if (nt <= 1) {
      fn(r0, r1);
      return;
    }
    std::vector<std::thread> th;
    const int64_t chunk = (rows + nt - 1) / nt;
    for (int64_t t = 0; t < nt; ++t) {
      const int64_t a = r0 + t * chunk, b = std::min(r1, a + chunk);
      if (a < b) th.emplace_back([&, a, b] { fn(a, b); });
    }
    for (auto& x : th) x.join();
  };
  std::vector<double> w((size_t)n);
  for (int64_t k = 0; k < n; ++k) {
    double norm2 = 0.0;
    for (int64_t i = k; i < n; ++i) norm2 += A[(size_t)(i * n + k)] * A[(size_t)(i * n + k)];
    const double x0 = A[(size_t)(k * n + k)];
    const double alpha = (x0 >= 0.0 ? -1.0 : 1.0) * std::sqrt(norm2);
    rdiag[(size_t)k] = alpha;
    double* v = &V[(size_t)(k * n)];
    double vv = 0.0;
    for (int64_t i = k; i < n; ++i) {
      v[i] = A[(size_t)(i * n + k)] - (i == k ? alpha : 0.0);
      vv += v[i] * v[i];
    }
    if (vv == 0.0) continue;  // column already reduced; H_k = I
    const double inv = 1.0 / std::sqrt(vv);
    for (int64_t i = k; i < n; ++i) v[i] *= inv;
    // w^T = v^T A[k:, k:], then A[k:, k:] -= 2 v w^T
    std::fill(w.begin(), w.end(), 0.0);
    for (int64_t i = k; i < n; ++i) {
      const double vi = v[i];
      const double* row = &A[(size_t)(i * n)];
      for (int64_t j = k; j < n; ++j) w[(size_t)j] += vi * row[j];
    }
    parallel_rows(k, n, [&](int64_t a, int64_t b) {
      for (int64_t i = a; i < b; ++i) {
        const double f2 = 2.0 * v[i];
        double* row = &A[(size_t)(i * n)];
        for (int64_t j = k; j < n; ++j) row[j] -= f2 * w[(size_t)j];
      }
    });
  }
  // Q = H_0 ... H_{n-1} I: apply H_k for k = n-1 down to 0 to the identity
  std::vector<double> Q((size_t)(n * n), 0.0);
  for (int64_t i = 0; i < n; ++i) Q[(size_t)(i * n + i)] = 1.0;
  for (int64_t k = n - 1; k >= 0; --k) {
    const double* v = &V[(size_t)(k * n)];
    std::fill(w.begin(), w.end(), 0.0);
    for (int64_t i = k; i < n; ++i) {
      const double vi = v[i];
      if (vi == 0.0) continue;
      const double* row = &Q[(size_t)(i * n)];
      for (int64_t j = 0; j < n; ++j) w[(size_t)j] += vi * row[j];
    }
    parallel_rows(k, n, [&](int64_t a, int64_t b) {
      for (int64_t i = a; i < b; ++i) {
        const double f2 = 2.0 * v[i];
        if (f2 == 0.0) continue;
        double* row = &Q[(size_t)(i * n)];
        for (int64_t j = 0; j < n; ++j) row[j] -= f2 * w[(size_t)j];
      }
    });
  }
  for (int64_t i = 0; i < n; ++i)
    for (int64_t j = 0; j < n; ++j) pi[i * n + j] = Q[(size_t)(i * n + j)] * (rdiag[(size_t)j] >= 0.0 ? 1.0 : -1.0);
  return KVRQ_OK;
}

// The entry points that allocate host memory (work vectors, threads) run their bodies guarded.
kvrq_status tq_codebook_init(int d, int bits, double tol, int max_iter, double* centroids, double* boundaries,
                             int* iterations) {
  return guarded("tq_codebook_init", [&] {
    alloc_check();
    return tq_codebook_init_body(d, bits, tol, max_iter, centroids, boundaries, iterations);
  });
}

kvrq_status pq_angle_codebook_init(int level, int bits, double tol, int max_iter, double* centroids,
                                   double* boundaries, int* iterations) {
  return guarded("pq_angle_codebook_init", [&] {
    alloc_check();
    return pq_angle_codebook_init_body(level, bits, tol, max_iter, centroids, boundaries, iterations);
  });
}

kvrq_status tq_rotation_init(int d, uint64_t seed, double* pi) {
  return guarded("tq_rotation_init", [&] {
    alloc_check();
    return tq_rotation_init_body(d, seed, pi);
  });
}

}  // extern "C"
