// Host part of the C ABI: Lloyd-Max codebook solver, Philox parameter
// generator, code-size arithmetic, error reporting.  No device code.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "common.h"

namespace tq {

static thread_local std::string g_last_error;

int set_error(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

void clear_error() { g_last_error.clear(); }

int check_params(const tq_params* p, const char* who) {
  if (!p) return set_error(TQ_EINVAL, "%s: params is NULL", who);
  if (p->d_pad != 128 && p->d_pad != 256)
    return set_error(TQ_EUNSUPPORTED, "%s: d_pad must be 128 or 256 (got %d)", who, p->d_pad);
  if (p->d < 1 || p->d > p->d_pad)
    return set_error(TQ_EINVAL, "%s: d must be in [1, d_pad] (got d=%d, d_pad=%d)", who, p->d, p->d_pad);
  if (p->mode == TQ_MODE_PROD) {
    if (p->bits < 2 || p->bits > 4) return set_error(TQ_EINVAL, "%s: product mode needs bits in 2..4", who);
    if (p->m < 32 || p->m > 256 || (p->m % 32) != 0)
      return set_error(TQ_EINVAL, "%s: m must be a multiple of 32 in [32, 256] (got %d)", who, p->m);
    if (!p->S) return set_error(TQ_EINVAL, "%s: S is NULL in product mode", who);
    if (!aligned(p->S, 16)) return set_error(TQ_EINVAL, "%s: S must be 16-byte aligned", who);
  } else if (p->mode == TQ_MODE_MSE) {
    if (p->bits < 1 || p->bits > 4) return set_error(TQ_EINVAL, "%s: MSE mode needs bits in 1..4", who);
    if (p->m != 0) return set_error(TQ_EINVAL, "%s: m must be 0 in MSE mode", who);
  } else {
    return set_error(TQ_EINVAL, "%s: unknown mode %d", who, p->mode);
  }
  if (p->layout != TQ_LAYOUT_PLANES && p->layout != TQ_LAYOUT_SLICED)
    return set_error(TQ_EINVAL, "%s: unknown code layout %d", who, p->layout);
  if (p->layout == TQ_LAYOUT_SLICED && p->mode != TQ_MODE_MSE)
    return set_error(TQ_EINVAL, "%s: the token-sliced layout holds MSE codes only", who);
  if (!p->centroids || !p->thresholds || !p->signs_D)
    return set_error(TQ_EINVAL, "%s: centroids/thresholds/signs_D must be non-NULL", who);
  if (!aligned(p->centroids, 4) || !aligned(p->thresholds, 4))
    return set_error(TQ_EINVAL, "%s: codebook arrays must be 4-byte aligned", who);
  return TQ_OK;
}

int check_planes(const tq_params* p, const char* who) {
  if (p->layout != TQ_LAYOUT_PLANES)
    return set_error(TQ_EUNSUPPORTED, "%s: needs codes in the canonical bit-plane layout", who);
  return TQ_OK;
}

// ---------------------------------------------------------------------------
// Lloyd-Max solver.  Law: one coordinate of a uniform random unit vector in
// R^d, density C_d (1-t^2)^((d-3)/2) on (-1,1).  Cell masses and first
// moments are integrated numerically (composite Gauss-Legendre); the Lloyd
// iteration alternates midpoint thresholds and conditional-mean centroids.
// ---------------------------------------------------------------------------
namespace {

struct GaussLegendre {
  std::vector<double> x, w;  // nodes/weights on [-1, 1]
  // Legendre P_n(z) and its derivative by the three-term recurrence.
  static void legendre(int n, double z, double* pn, double* dpn) {
    double p0 = 1.0, p1 = z;
    for (int k = 2; k <= n; ++k) {
      double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
      p0 = p1;
      p1 = p2;
    }
    *pn = p1;
    *dpn = n * (z * p1 - p0) / (z * z - 1.0);
  }
  explicit GaussLegendre(int n) : x(n), w(n) {
    for (int i = 0; i < n; ++i) {
      double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));  // initial guess for root i
      double pn, dpn;
      for (int it = 0; it < 100; ++it) {
        legendre(n, z, &pn, &dpn);
        double dz = pn / dpn;
        z -= dz;
        if (std::fabs(dz) < 1e-16) break;
      }
      legendre(n, z, &pn, &dpn);
      x[i] = z;
      w[i] = 2.0 / ((1.0 - z * z) * dpn * dpn);
    }
  }
};

// With t = sin(theta) the cell integrals become integrals of C cos^(d-2)
// (mass) and C sin cos^(d-2) (first moment) over [asin a, asin b]: smooth
// integrands, so composite Gauss-Legendre converges fast even for small d.
struct SphereLaw {
  int d;
  double logC;
  explicit SphereLaw(int dd) : d(dd) {
    logC = std::lgamma(d / 2.0) - 0.5 * std::log(M_PI) - std::lgamma((d - 1) / 2.0);
  }
};

void cell_integrals(const SphereLaw& law, const GaussLegendre& gl, double a, double b, int panels,
                    double* m0, double* m1) {
  const double ta = std::asin(std::max(-1.0, std::min(1.0, a)));
  const double tb = std::asin(std::max(-1.0, std::min(1.0, b)));
  const double h = (tb - ta) / panels;
  double s0 = 0.0, s1 = 0.0;
  for (int pnl = 0; pnl < panels; ++pnl) {
    const double mid = ta + (pnl + 0.5) * h;
    for (size_t i = 0; i < gl.x.size(); ++i) {
      const double th = mid + 0.5 * h * gl.x[i];
      const double cs = std::cos(th);
      const double f = (cs > 0.0) ? std::exp(law.logC + (law.d - 2) * std::log(cs)) * gl.w[i] : 0.0;
      s0 += f;
      s1 += std::sin(th) * f;
    }
  }
  *m0 = s0 * 0.5 * h;
  *m1 = s1 * 0.5 * h;
}

}  // namespace

}  // namespace tq

extern "C" int tq_make_codebook(int d_pad, int kb, float* centroids, float* thresholds) {
  using namespace tq;
  if (!centroids || !thresholds) return set_error(TQ_EINVAL, "tq_make_codebook: NULL output");
  if (!is_pow2(d_pad) || d_pad < 4 || d_pad > 4096)
    return set_error(TQ_EINVAL, "tq_make_codebook: d_pad must be a power of two in [4, 4096]");
  if (kb < 1 || kb > 4) return set_error(TQ_EINVAL, "tq_make_codebook: kb must be in 1..4");
  const int L = 1 << kb;
  SphereLaw law(d_pad);
  GaussLegendre gl(24);
  const double sd = 1.0 / std::sqrt((double)d_pad);
  std::vector<double> c(L), cn(L), edge(L + 1);
  const double spread = std::min(2.5 * sd, 0.9);
  for (int l = 0; l < L; ++l) c[l] = spread * (2.0 * l + 1.0 - L) / L;
  double best = 1e300;
  int best_it = 0;
  bool done = false;
  for (int it = 0; it < 400000 && !done; ++it) {
    edge[0] = -1.0;
    edge[L] = 1.0;
    for (int l = 0; l + 1 < L; ++l) edge[l + 1] = 0.5 * (c[l] + c[l + 1]);
    for (int l = 0; l < L; ++l) {
      double m0, m1;
      cell_integrals(law, gl, edge[l], edge[l + 1], 16, &m0, &m1);
      cn[l] = m1 / m0;
    }
    double step = 0.0;
    for (int l = 0; l < L; ++l) {
      double s = 0.5 * (cn[l] - cn[L - 1 - l]);
      step = std::max(step, std::fabs(s - c[l]));
      c[l] = s;
    }
    step /= sd;
    if (step < 1e-15) done = true;
    if (step < best) {
      best = step;
      best_it = it;
    } else if (best < 1e-12 && it - best_it > 2000) {
      done = true;
    }
  }
  if (!done) return set_error(TQ_EINVAL, "tq_make_codebook: Lloyd-Max iteration did not converge");
  for (int l = 0; l < L; ++l) centroids[l] = (float)c[l];
  for (int l = 0; l + 1 < L; ++l)
    thresholds[l] = (float)(0.5 * ((double)centroids[l] + (double)centroids[l + 1]));
  clear_error();
  return TQ_OK;
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon et al., SC'11) and the parameter streams.
// ---------------------------------------------------------------------------
namespace {

void philox(uint32_t ctr[4], uint32_t k0, uint32_t k1) {
  const uint64_t M0 = 0xD2511F53ull, M1 = 0xCD9E8D57ull;
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    uint64_t p0 = M0 * ctr[0], p1 = M1 * ctr[2];
    uint32_t n0 = (uint32_t)(p1 >> 32) ^ ctr[1] ^ k0;
    uint32_t n1 = (uint32_t)p1;
    uint32_t n2 = (uint32_t)(p0 >> 32) ^ ctr[3] ^ k1;
    uint32_t n3 = (uint32_t)p0;
    ctr[0] = n0;
    ctr[1] = n1;
    ctr[2] = n2;
    ctr[3] = n3;
  }
}

uint32_t stream_word(uint64_t seed, uint32_t stream, uint64_t w) {
  uint32_t c[4] = {(uint32_t)(w >> 2), stream, 0u, 0u};
  philox(c, (uint32_t)seed, (uint32_t)(seed >> 32));
  return c[w & 3];
}

uint16_t f64_to_f16_rne(double v) {
  // IEEE binary16, round to nearest even, via exact scaling in double.
  uint16_t sign = std::signbit(v) ? 0x8000 : 0;
  double a = std::fabs(v);
  if (std::isnan(a)) return 0x7E00;
  if (a >= 65520.0) return sign | 0x7C00;  // rounds to infinity
  if (a < std::ldexp(1.0, -25)) {
    // below half the smallest subnormal (exactly half rounds to even = 0)
    return sign;
  }
  int e;
  std::frexp(a, &e);  // a = f * 2^e, f in [0.5, 1)
  int exp_unbiased = e - 1;
  if (exp_unbiased < -14) {
    // subnormal: value = m * 2^-24
    double mq = std::nearbyint(a * std::ldexp(1.0, 24));  // default rounding: nearest even
    return sign | (uint16_t)mq;                          // mq may reach 1024 = smallest normal
  }
  double frac = a * std::ldexp(1.0, 10 - exp_unbiased);  // in [1024, 2048)
  double mq = std::nearbyint(frac);
  int ex = exp_unbiased;
  if (mq >= 2048.0) {
    mq = 1024.0;
    ++ex;
  }
  if (ex > 15) return sign | 0x7C00;
  return sign | (uint16_t)((ex + 15) << 10) | (uint16_t)((int)mq - 1024);
}

}  // namespace

extern "C" int tq_make_params(int d_pad, int m, uint64_t seed, int8_t* D, uint16_t* S) {
  using namespace tq;
  if (!D) return set_error(TQ_EINVAL, "tq_make_params: D is NULL");
  if (!is_pow2(d_pad) || d_pad > 4096) return set_error(TQ_EINVAL, "tq_make_params: bad d_pad");
  if (m < 0 || m > 4096) return set_error(TQ_EINVAL, "tq_make_params: bad m");
  if (m > 0 && !S) return set_error(TQ_EINVAL, "tq_make_params: S is NULL");
  for (int j = 0; j < d_pad; ++j) D[j] = (stream_word(seed, 0, (uint64_t)j) & 1u) ? -1 : 1;
  const uint64_t n = (uint64_t)m * (uint64_t)d_pad;
  for (uint64_t p = 0; 2 * p < n; ++p) {
    double ua = ((double)stream_word(seed, 1, 2 * p) + 0.5) / 4294967296.0;
    double ub = ((double)stream_word(seed, 1, 2 * p + 1) + 0.5) / 4294967296.0;
    double rad = std::sqrt(-2.0 * std::log(ua));
    double th = 2.0 * M_PI * ub;
    S[2 * p] = f64_to_f16_rne(rad * std::cos(th));
    if (2 * p + 1 < n) S[2 * p + 1] = f64_to_f16_rne(rad * std::sin(th));
  }
  clear_error();
  return TQ_OK;
}

extern "C" int64_t tq_code_bytes(int d_pad, int kb, int m, int64_t n_vec) {
  if (d_pad <= 0 || kb < 0 || m < 0 || n_vec < 0) return -1;
  int64_t tiles = (n_vec + 31) / 32;
  return tiles * 32 * ((int64_t)kb * d_pad / 8 + m / 8);
}

extern "C" const char* tq_last_error(void) { return tq::g_last_error.c_str(); }

extern "C" int tq_version(void) { return 100; }
