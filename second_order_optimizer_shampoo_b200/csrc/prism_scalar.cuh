// Scalar parts of the PRISM step shared by the batched kernels and the
// on-chip small-block kernel: the residual-coefficient tables, the quartic
// J(alpha) from the sketch Gram matrix, its constrained minimiser and the
// per-pass stop rule.  All in fp64 except the stop test, which compares the
// fp32 residual norm.
//
// "Sintesi Tecnica: PRISM", Parte II.1: alpha minimises the fitted residual
// on [l, u]; the stop rule adds the non-finite and stall checks of the
// failure-detection reading.
#pragma once
#include <math.h>

#include "internal.h"

namespace shp {
namespace {

// Coefficients of r_j(alpha) = T[j][0] + T[j][1] alpha + T[j][2] alpha^2 for
// j = d..2d+1, written out from r(xi; alpha) = 1 - (1 - xi) g_d(xi; alpha)^2:
//   d = 1 (f = 1):        r = (1-2a) xi + (2a - a^2) xi^2 + a^2 xi^3
//   d = 2 (f = 1 + xi/2): r = (3/4 - 2a) xi^2 + (1/4 + a) xi^3 + (a - a^2) xi^4 + a^2 xi^5
__device__ const double kRTab1[3][3] = {{1.0, -2.0, 0.0}, {0.0, 2.0, -1.0}, {0.0, 0.0, 1.0}};
__device__ const double kRTab2[4][3] = {
    {0.75, -2.0, 0.0}, {0.25, 1.0, 0.0}, {0.0, 1.0, -1.0}, {0.0, 0.0, 1.0}};

__device__ __forceinline__ double poly4(const double* c, double a) {
  return (((c[4] * a + c[3]) * a + c[2]) * a + c[1]) * a + c[0];
}
__device__ __forceinline__ double dpoly4(const double* c, double a) {
  return ((4.0 * c[4] * a + 3.0 * c[3]) * a + 2.0 * c[2]) * a + c[1];
}
__device__ __forceinline__ double d2poly4(const double* c, double a) {
  return (12.0 * c[4] * a + 6.0 * c[3]) * a + 2.0 * c[2];
}

// Global minimiser of the quartic J on [lo, hi].  J' is monotone between the
// real roots of J'' (a quadratic), so each such piece holds at most one root
// of J'; the root is bracketed, then polished by Newton.  The candidate with
// the least J wins; values within 1e-12 (relative) of the best tie and go to
// the smaller alpha; a constant or non-finite J gives lo.

// Breakpoints lo < (roots of J'' inside) < hi; returns their count, or 0 when
// J is constant or not finite (the minimiser is then lo).
__device__ __forceinline__ int quartic_breaks(const double* c, double lo, double hi,
                                              double* brk) {
  bool finite = true;
  double scale = 0.0;
  for (int i = 0; i < 5; ++i) {
    if (!isfinite(c[i])) finite = false;
    if (i > 0) scale = fmax(scale, fabs(c[i]));
  }
  if (!finite || scale == 0.0) return 0;
  int nb = 0;
  brk[nb++] = lo;
  const double qa = 12.0 * c[4], qb = 6.0 * c[3], qc = 2.0 * c[2];
  double r1 = NAN, r2 = NAN;
  if (qa != 0.0) {
    const double disc = qb * qb - 4.0 * qa * qc;
    if (disc >= 0.0) {
      const double sd = sqrt(disc);
      const double q = -0.5 * (qb + (qb >= 0.0 ? sd : -sd));
      if (q != 0.0) {
        r1 = q / qa;
        r2 = qc / q;
      } else {
        r1 = r2 = 0.0;
      }
    }
  } else if (qb != 0.0) {
    r1 = -qc / qb;
  }
  if (r1 > r2) {
    const double t = r1;
    r1 = r2;
    r2 = t;
  }
  if (r1 > lo && r1 < hi) brk[nb++] = r1;
  if (r2 > lo && r2 < hi && r2 != r1) brk[nb++] = r2;
  brk[nb++] = hi;
  return nb;
}

// Two Newton steps on J' from the bracket midpoint, kept inside [u0, v0].
__device__ __forceinline__ double quartic_polish(const double* c, double u, double v, double u0,
                                                 double v0) {
  double a = 0.5 * (u + v);
  for (int it = 0; it < 2; ++it) {
    const double h = d2poly4(c, a);
    if (h != 0.0) {
      const double an = a - dpoly4(c, a) / h;
      if (an >= u0 && an <= v0) a = an;
    }
  }
  return a;
}

// The candidate with the least J; ties (1e-12 relative) to the smaller alpha.
__device__ __forceinline__ double quartic_pick(const double* c, const double* cand, int nc,
                                               double hi) {
  double best = poly4(c, cand[0]);
  for (int i = 1; i < nc; ++i) best = fmin(best, poly4(c, cand[i]));
  const double thr = best + 1e-12 * fmax(fabs(best), 1e-300);
  double pick = hi;
  for (int i = 0; i < nc; ++i)
    if (poly4(c, cand[i]) <= thr && cand[i] < pick) pick = cand[i];
  return pick;
}

// One thread: each monotone piece with a sign change of J' is bisected.
__device__ double argmin_quartic(const double* c, double lo, double hi) {
  double brk[4];
  const int nb = quartic_breaks(c, lo, hi, brk);
  if (nb == 0) return lo;
  double cand[5];
  int nc = 0;
  cand[nc++] = lo;
  cand[nc++] = hi;
  for (int s = 0; s + 1 < nb; ++s) {
    double u = brk[s], v = brk[s + 1];
    double fu = dpoly4(c, u);
    const double fv = dpoly4(c, v);
    if (fu == 0.0) {
      cand[nc++] = u;
      continue;
    }
    if (fv == 0.0 || (fu < 0.0) == (fv < 0.0)) continue;
    for (int it = 0; it < 200 && v - u > 1e-15 * fmax(1.0, fabs(u)); ++it) {
      const double mid = 0.5 * (u + v);
      const double fm = dpoly4(c, mid);
      if (fm == 0.0) {
        u = v = mid;
        break;
      }
      if ((fm < 0.0) == (fu < 0.0)) {
        u = mid;
        fu = fm;
      } else {
        v = mid;
      }
    }
    const double a = quartic_polish(c, u, v, brk[s], brk[s + 1]);
    if (a > lo && a < hi) cand[nc++] = a;
  }
  return quartic_pick(c, cand, nc, hi);
}

// The same minimiser computed by a whole warp (every lane returns it): each
// round evaluates J' at 32 interior points of the bracket at once and keeps
// the 1/33 sub-interval where its sign first changes, so 10 rounds reach the
// 1e-15 width that bisection needs 50 steps for.  All lanes run identical
// arithmetic, so they agree on every decision.
__device__ double argmin_quartic_warp(const double* c, double lo, double hi) {
  const int lane = threadIdx.x & 31;
  double brk[4];
  const int nb = quartic_breaks(c, lo, hi, brk);
  if (nb == 0) return lo;
  double cand[5];
  int nc = 0;
  cand[nc++] = lo;
  cand[nc++] = hi;
  for (int s = 0; s + 1 < nb; ++s) {
    double u = brk[s], v = brk[s + 1];
    double fu = dpoly4(c, u);
    const double fv = dpoly4(c, v);
    if (fu == 0.0) {
      cand[nc++] = u;
      continue;
    }
    if (fv == 0.0 || (fu < 0.0) == (fv < 0.0)) continue;
    for (int it = 0; it < 16 && v - u > 1e-15 * fmax(1.0, fabs(u)); ++it) {
      // the 32 interior points u + h, u + 2h, .. u + 32h with h = (v - u) / 33
      // (a multiply by the rounded 1/33: any partition of the bracket works,
      // and a division per point is the round's longest dependency)
      const double h = (v - u) * (1.0 / 33.0);
      const double x = u + h * static_cast<double>(lane + 1);
      const double fx = dpoly4(c, x);
      const unsigned m = __ballot_sync(0xffffffffu, fx == 0.0 || (fx < 0.0) != (fu < 0.0));
      const int i = m != 0u ? __ffs(static_cast<int>(m)) - 1 : 32;  // first sign change
      const double nu = i == 0 ? u : u + h * static_cast<double>(i);
      const double nv = i == 32 ? v : u + h * static_cast<double>(i + 1);
      if (i != 0) fu = dpoly4(c, nu);
      u = nu;
      v = nv;
      if (fu == 0.0) {
        v = u;
        break;
      }
    }
    const double a = quartic_polish(c, u, v, brk[s], brk[s + 1]);
    if (a > lo && a < hi) cand[nc++] = a;
  }
  return quartic_pick(c, cand, nc, hi);
}

// Coefficients (alpha^0 .. alpha^4) of J(alpha) = sum_ij r_i(alpha) r_j(alpha) M_ij
// for the d + 2 sketch moments V_d .. V_{2d+1}; M is (d+2) x (d+2).
__device__ void quartic_from_gram(const double (*M)[4], int d, double* coef) {
  const int nv = d + 2;
  double T[4][3];
  for (int i = 0; i < nv; ++i)
    for (int a = 0; a < 3; ++a) T[i][a] = d == 1 ? kRTab1[i][a] : kRTab2[i][a];
  for (int i = 0; i < 5; ++i) coef[i] = 0.0;
  for (int a = 0; a < 3; ++a)
    for (int c = 0; c < 3; ++c) {
      double s = 0.0;
      for (int i = 0; i < nv; ++i)
        for (int j = 0; j < nv; ++j) s += T[i][a] * M[i][j] * T[j][c];
      coef[a + c] += s;
    }
}

// Stop rule of one pass at check k (k updates done), residual r = ||R_k||_F / sqrt(n):
// returns the pass status, or -1 to continue.  prev is the residual of check k - 1.
__device__ __forceinline__ int stop_rule(float r, int k, int max_iter, float tol, float prev,
                                         float stall_below, float stall_ratio) {
  if (!isfinite(r)) return ST_ENONFINITE;
  if (r <= tol) return ST_OK;
  if (k >= max_iter) return ST_ENOCONV;
  if (k >= 1 && prev < stall_below && r > stall_ratio * prev) return ST_ESTALL;
  return -1;
}

}  // namespace
}  // namespace shp
