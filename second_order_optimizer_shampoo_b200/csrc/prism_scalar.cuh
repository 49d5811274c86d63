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

// Coefficient of alpha^t in r_{d+j}(alpha) (j = 0 .. d+1), written out from
// r(xi; alpha) = 1 - (1 - xi) g_d(xi; alpha)^2:
//   d = 1 (f = 1):        r = (1-2a) xi + (2a - a^2) xi^2 + a^2 xi^3
//   d = 2 (f = 1 + xi/2): r = (3/4 - 2a) xi^2 + (1/4 + a) xi^3 + (a - a^2) xi^4 + a^2 xi^5
// Called with compile-time arguments only, so every entry folds into the
// arithmetic that uses it (the zeros vanish).
template <int D>
__device__ __forceinline__ constexpr double rtab(int j, int t) {
  if constexpr (D == 1) {
    constexpr double T[3][3] = {{1.0, -2.0, 0.0}, {0.0, 2.0, -1.0}, {0.0, 0.0, 1.0}};
    return T[j][t];
  } else {
    constexpr double T[4][3] = {
        {0.75, -2.0, 0.0}, {0.25, 1.0, 0.0}, {0.0, 1.0, -1.0}, {0.0, 0.0, 1.0}};
    return T[j][t];
  }
}

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
// the smaller alpha; a constant or non-finite J gives lo.  Everything below
// works on named scalars and fully unrolled loops, so nothing leaves the
// registers (indexed local arrays would go through local memory, and this
// serial fp64 chain is on the critical path of every iteration).

// The breakpoints lo = p0 <= p1 <= p2 <= p3 = hi: p1, p2 are the roots of J''
// inside (lo, hi), an absent one repeating its left neighbour (an empty
// piece).  False when J is constant or not finite (the minimiser is then lo).
__device__ __forceinline__ bool quartic_breaks(const double* c, double lo, double hi,
                                               double& p1, double& p2) {
  bool finite = true;
  double scale = 0.0;
#pragma unroll
  for (int i = 0; i < 5; ++i) {
    if (!isfinite(c[i])) finite = false;
    if (i > 0) scale = fmax(scale, fabs(c[i]));
  }
  if (!finite || scale == 0.0) return false;
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
  p1 = r1 > lo && r1 < hi ? r1 : lo;
  p2 = r2 > lo && r2 < hi && r2 != r1 ? r2 : p1;
  return true;
}

// Newton on J' from the bracket midpoint, each step kept only while it stays
// inside the bracket [u, v] (which holds the root).
__device__ __forceinline__ double quartic_polish(const double* c, double u, double v) {
  double a = 0.5 * (u + v);
#pragma unroll
  for (int it = 0; it < 3; ++it) {
    const double h = d2poly4(c, a);
    if (h == 0.0) break;
    const double an = a - dpoly4(c, a) / h;
    if (!(an >= u && an <= v)) break;
    a = an;
  }
  return a;
}

// The root of J' on the piece [u, v] (J' monotone there) computed by a whole
// warp (every lane returns it), or lo when J' keeps its sign: each round
// evaluates J' at 32 interior points of the bracket at once and keeps the
// 1/33 sub-interval where its sign first changes; four rounds narrow the
// bracket a millionfold (relative), and the Newton polish then converges
// quadratically from inside it.  All lanes run identical arithmetic, so they
// agree on every decision.
__device__ __forceinline__ double piece_root_warp(const double* c, double u, double v,
                                                  double lo, double hi) {
  const int lane = threadIdx.x & 31;
  double fu = dpoly4(c, u);
  const double fv = dpoly4(c, v);
  if (fu == 0.0) return u;
  if (fv == 0.0 || (fu < 0.0) == (fv < 0.0)) return lo;
  const double u0 = u, v0 = v;
  for (int it = 0; it < 16 && v - u > 1e-6 * fmax(1.0, fabs(u)); ++it) {
    // the 32 interior points u + h, u + 2h, .. u + 32h with h = (v - u) / 33
    // (a multiply by the rounded 1/33: any partition of the bracket works)
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
    if (fu == 0.0) return u;
  }
  const double a = quartic_polish(c, fmax(u, u0), fmin(v, v0));
  return a > lo && a < hi ? a : lo;
}

__device__ double argmin_quartic_warp(const double* c, double lo, double hi) {
  double p1, p2;
  if (!quartic_breaks(c, lo, hi, p1, p2)) return lo;
  // candidates: the ends and one root of J' per piece (lo when none: a
  // repeated candidate changes nothing)
  const double a1 = piece_root_warp(c, lo, p1, lo, hi);
  const double a2 = piece_root_warp(c, p1, p2, lo, hi);
  const double a3 = piece_root_warp(c, p2, hi, lo, hi);
  const double cand[5] = {lo, hi, a1, a2, a3};
  double j[5];
  double best = INFINITY;
#pragma unroll
  for (int i = 0; i < 5; ++i) {
    j[i] = poly4(c, cand[i]);
    best = fmin(best, j[i]);
  }
  const double thr = best + 1e-12 * fmax(fabs(best), 1e-300);
  double pick = hi;
#pragma unroll
  for (int i = 0; i < 5; ++i)
    if (j[i] <= thr && cand[i] < pick) pick = cand[i];
  return pick;
}

// Coefficients (alpha^0 .. alpha^4) of J(alpha) = sum_ij r_i(alpha) r_j(alpha) M_ij
// for the D + 2 sketch moments V_D .. V_{2D+1}; M is (D+2) x (D+2) (entries
// past that unused).  U = M T first, then coef[a + c] += T[i][a] U[i][c].
template <int D>
__device__ __forceinline__ void quartic_from_gram_d(const double (&M)[4][4], double* coef) {
  constexpr int NV = D + 2;
  double U[NV][3];
#pragma unroll
  for (int i = 0; i < NV; ++i)
#pragma unroll
    for (int t = 0; t < 3; ++t) {
      double s = 0.0;
#pragma unroll
      for (int j = 0; j < NV; ++j)
        if (rtab<D>(j, t) != 0.0) s = fma(M[i][j], rtab<D>(j, t), s);
      U[i][t] = s;
    }
#pragma unroll
  for (int k = 0; k < 5; ++k) coef[k] = 0.0;
#pragma unroll
  for (int a = 0; a < 3; ++a)
#pragma unroll
    for (int t = 0; t < 3; ++t)
#pragma unroll
      for (int i = 0; i < NV; ++i)
        if (rtab<D>(i, a) != 0.0) coef[a + t] = fma(rtab<D>(i, a), U[i][t], coef[a + t]);
}
__device__ __forceinline__ void quartic_from_gram(const double (&M)[4][4], int d, double* coef) {
  if (d == 1)
    quartic_from_gram_d<1>(M, coef);
  else
    quartic_from_gram_d<2>(M, coef);
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
