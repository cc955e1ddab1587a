// Host side of the polar-coordinate stage 1: table sizes, the Lloyd-Max angle
// tables and code sizes (no device code).
//
// "TurboQuant explainer" (m.163.com), "第一步：PolarQuant": after the random
// rotation the angles of the polar form follow a known Beta law, so each is
// coded with a fixed table.  Level l >= 2 of the recursive pairwise form has
// sin^2 psi ~ Beta(k/2, k/2), k = 2^(l-1): density proportional to
// (sin psi cos psi)^(k-1) on [0, pi/2]; level 1 (the full angle of a
// coordinate pair) is uniform on [0, 2 pi).
#include <algorithm>
#include <cmath>
#include <vector>

#include "common.h"

namespace {

constexpr double kPi = 3.14159265358979323846;

int log2i(int v) {
  int l = 0;
  while ((1 << l) < v) ++l;
  return l;
}

// 24-point Gauss-Legendre nodes and weights on [-1, 1], by Newton's method on P_n.
struct GL24 {
  double x[24], w[24];
  GL24() {
    const int n = 24;
    for (int i = 0; i < n; ++i) {
      double z = std::cos(kPi * (i + 0.75) / (n + 0.5)), dp = 0.0;
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = z;
        for (int k = 2; k <= n; ++k) {
          const double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
          p0 = p1;
          p1 = p2;
        }
        dp = n * (z * p1 - p0) / (z * z - 1.0);
        const double dz = p1 / dp;
        z -= dz;
        if (std::fabs(dz) < 1e-16) break;
      }
      x[i] = z;
      w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
  }
};

// Unnormalised density of psi at level with k coordinates per child radius,
// scaled to 1 at pi/4: ((sin psi cos psi) / (1/2))^(k-1).
double angle_density(double psi, int k) {
  const double s = std::sin(2.0 * psi);  // 2 sin psi cos psi
  if (s <= 0.0) return k == 1 ? 1.0 : 0.0;
  return std::exp((k - 1) * std::log(s));
}

// mass and first moment of the cell [a, b] (panels of 24-point rules)
void angle_cell(const GL24& gl, int k, double a, double b, double* m0, double* m1) {
  const int panels = 64;
  double s0 = 0.0, s1 = 0.0;
  const double h = (b - a) / panels;
  for (int p = 0; p < panels; ++p) {
    const double lo = a + p * h, mid = lo + 0.5 * h;
    for (int i = 0; i < 24; ++i) {
      const double t = mid + 0.5 * h * gl.x[i];
      const double f = gl.w[i] * angle_density(t, k);
      s0 += f;
      s1 += f * t;
    }
  }
  *m0 = 0.5 * h * s0;
  *m1 = 0.5 * h * s1;
}

// Lloyd-Max fixed point of the level's angle law with L cells; false if it does not settle.
bool angle_lloyd(int k, int L, std::vector<double>& c) {
  c.assign(L, kPi / 4);
  if (L == 1) return true;
  static const GL24 gl;
  const double sd = 0.5 / std::sqrt(k + 1.0);  // spread of psi around pi/4
  const double spread = std::min(2.5 * sd, 0.9 * kPi / 4);
  for (int j = 0; j < L; ++j) c[j] = kPi / 4 + spread * (2.0 * j + 1.0 - L) / L;
  std::vector<double> e(L + 1), cn(L);
  double best = 1e300;
  int best_it = 0;
  for (int it = 0; it < 200000; ++it) {
    e[0] = 0.0;
    e[L] = kPi / 2;
    for (int j = 0; j + 1 < L; ++j) e[j + 1] = 0.5 * (c[j] + c[j + 1]);
    for (int j = 0; j < L; ++j) {
      double m0, m1;
      angle_cell(gl, k, e[j], e[j + 1], &m0, &m1);
      cn[j] = m0 > 0.0 ? m1 / m0 : 0.5 * (e[j] + e[j + 1]);
    }
    double step = 0.0;
    for (int j = 0; j < L; ++j) {
      const double s = 0.5 * (cn[j] + (kPi / 2 - cn[L - 1 - j]));  // symmetric about pi/4
      step = std::max(step, std::fabs(s - c[j]));
      c[j] = s;
    }
    if (step < 1e-15) return true;
    if (step < best) {
      best = step;
      best_it = it;
    } else if (best < 1e-12 && it - best_it > 2000) {
      return true;
    }
  }
  return false;
}

}  // namespace

extern "C" int64_t tq_polar_table_floats(int d_pad, int w) {
  if (!tq::is_pow2(d_pad) || d_pad < 4 || d_pad > 4096 || w < 1 || w > 3) return -1;
  const int L1 = 1 << (w + 1), L2 = 1 << (w - 1);
  return 3 * L1 + (int64_t)(log2i(d_pad) - 1) * (4 * L2 - 1);
}

extern "C" int64_t tq_polar_code_bytes(int d_pad, int w, int64_t n_vec) {
  // a record is w * d_pad / 8 whole bytes, so d_pad >= 8 (d_pad 4 at w = 1 would be half a byte)
  if (!tq::is_pow2(d_pad) || d_pad < 8 || w < 1 || w > 3 || n_vec < 0) return -1;
  return n_vec * (int64_t)w * d_pad / 8;
}

extern "C" int tq_polar_make_tables(int d_pad, int w, float* tables) {
  using namespace tq;
  if (!tables) return set_error(TQ_EINVAL, "tq_polar_make_tables: NULL output");
  if (tq_polar_table_floats(d_pad, w) < 0)
    return set_error(TQ_EINVAL, "tq_polar_make_tables: d_pad must be a power of two in [4, 4096], w in 1..3");
  const int L1 = 1 << (w + 1), L2 = 1 << (w - 1);
  for (int j = 0; j < L1; ++j) {
    const float c = (float)((j + 0.5) * (2.0 * kPi / L1));
    tables[j] = c;
    tables[L1 + 2 * j] = (float)std::cos((double)c);
    tables[L1 + 2 * j + 1] = (float)std::sin((double)c);
  }
  float* t = tables + 3 * L1;
  std::vector<double> c;
  for (int lv = 2; lv <= log2i(d_pad); ++lv, t += 4 * L2 - 1) {
    if (!angle_lloyd(1 << (lv - 1), L2, c))
      return set_error(TQ_EINVAL, "tq_polar_make_tables: Lloyd-Max iteration did not converge");
    for (int j = 0; j < L2; ++j) t[j] = (float)c[j];
    for (int j = 0; j + 1 < L2; ++j) t[L2 + j] = (float)(0.5 * ((double)t[j] + (double)t[j + 1]));
    for (int j = 0; j < L2; ++j) {
      t[2 * L2 - 1 + 2 * j] = (float)std::cos((double)t[j]);
      t[2 * L2 - 1 + 2 * j + 1] = (float)std::sin((double)t[j]);
    }
  }
  clear_error();
  return TQ_OK;
}
