// Newton-Schulz/PRISM on chip for small blocks (n <= 64): one CTA per block
// runs every pass of the coupled iteration (or the whole polar iteration)
// with all iterates in shared memory.  HBM is touched only to read the input
// and the sketch slices and to write the result and the report.
//
// Block-diagonal Shampoo ("深度学习中的优化器之Shampoo算法原理与二阶优化机制"
// §3.2) splits large layers into many small preconditioner blocks.  For a
// 64 x 64 block a product is 0.5 MFLOP, far too little for a launch of its
// own, so the batched path's per-iteration launches would dominate; here the
// iteration never leaves the SM.  The steps are exactly those of the batched
// path ("Sintesi Tecnica: PRISM", Parte I-II): residual, stop test, sketched
// alpha fit, Delta = g - I, X + X Delta updates.
//
// Arithmetic: products on the CUDA cores in fp32 FMA (each thread owns a 4 x 4
// output tile and streams float4 operands from shared memory), at least as
// accurate as either fp32 storage mode of the batched path; the alpha fit and
// the norms in fp64.  Four 64 x 68 fp32 buffers (68 KB) per CTA, three CTAs
// per SM.
#include <math.h>

#include "internal.h"
#include "prism_scalar.cuh"
#include "shampoo_prism.h"
#include "shp_common.cuh"

namespace shp {

namespace {

constexpr int SB_NMAX = 64;
// Row stride in floats: rows 4 apart (the two row groups one warp reads) land
// 16 banks apart, so the float4 operand reads are conflict-free.
constexpr int SB_LD = 68;
constexpr int SB_MAT = SB_NMAX * SB_LD;
constexpr int SB_THREADS = 256;
constexpr int SB_PMAX = 16;
constexpr int SB_SMEM = 4 * SB_MAT * static_cast<int>(sizeof(float));
static_assert(4 * SB_NMAX * SB_PMAX <= SB_MAT, "sketch slots must fit one matrix buffer");

struct SmallCfg {
  int d, p, max_iter, fixed_alpha, adaptive;
  float lo, hi, tol, stall_below, stall_ratio, raise_above;
};

// Sum over the CTA; every thread receives the result.
SHP_DEV double block_sum(double v, double* red) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red may still be read by the previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double s = 0.0;
#pragma unroll
  for (int w = 0; w < SB_THREADS / 32; ++w) s += red[w];
  return s;
}

// A thread's 4 x 4 output tile: rows rb, rb + rs, rb + 2 rs, rb + 3 rs and
// columns c0..c0+3.  Products with a row-major left factor use strided rows
// (rs = 16): a warp covers 4 consecutive row indices x 8 column groups, so
// each float4 operand read touches 4 rows (16 banks apart in total) of A and
// 128 contiguous bytes of B, one wavefront each.  Products with a
// transposed left factor read 4 consecutive rows of A^T as one float4 and
// use consecutive rows (rs = 1).
struct Tile {
  int rb, rs, c0;
  SHP_DEV int row(int i) const { return rb + rs * i; }
};

SHP_DEV Tile tile_rows_strided() {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  return Tile{4 * (w >> 1) + (l >> 3), 16, 4 * (8 * (w & 1) + (l & 7))};
}
SHP_DEV Tile tile_rows_consecutive() {
  const int t = static_cast<int>(threadIdx.x);
  return Tile{4 * (t >> 4), 1, 4 * (t & 15)};
}

// acc = op(A) B on tile t, K a multiple of 4.  op(A) = A (row-major M x K) or,
// with AT, the transpose of the row-major K x M matrix A (t.rs must be 1).
template <bool AT>
SHP_DEV void tile_mm(const float* A, const float* B, int K, const Tile& t, float acc[4][4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 2
  for (int k = 0; k < K; k += 4) {
    float a[4][4], b[4][4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const float4 v = *reinterpret_cast<const float4*>(B + (k + kk) * SB_LD + t.c0);
      b[kk][0] = v.x;
      b[kk][1] = v.y;
      b[kk][2] = v.z;
      b[kk][3] = v.w;
    }
    if (AT) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const float4 v = *reinterpret_cast<const float4*>(A + (k + kk) * SB_LD + t.rb);
        a[0][kk] = v.x;
        a[1][kk] = v.y;
        a[2][kk] = v.z;
        a[3][kk] = v.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = *reinterpret_cast<const float4*>(A + t.row(i) * SB_LD + k);
        a[i][0] = v.x;
        a[i][1] = v.y;
        a[i][2] = v.z;
        a[i][3] = v.w;
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i][kk], b[kk][j], acc[i][j]);
  }
}

SHP_DEV void store_row4(float* C, int row, int c0, const float* v) {
  *reinterpret_cast<float4*>(C + row * SB_LD + c0) = make_float4(v[0], v[1], v[2], v[3]);
}

// R = I - op(A) B on the n x n grid; returns this thread's sum of squares.
// Rows of the tile past n are computed from in-buffer data and not stored.
template <bool AT>
SHP_DEV float residual(const float* A, const float* B, int K, int n, float* R, const Tile& t) {
  float nrm = 0.f;
  if (t.rb < n && t.c0 < n) {
    float acc[4][4];
    tile_mm<AT>(A, B, K, t, acc);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = t.row(i);
      if (r >= n) break;
      float v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[j] = (r == t.c0 + j ? 1.f : 0.f) - acc[i][j];
        nrm += v[j] * v[j];
      }
      store_row4(R, r, t.c0, v);
    }
  }
  return nrm;
}

// C = X + A B (X may be A or B, C must be neither), rows x cols, inner K.
SHP_DEV void axpy_mm(const float* A, const float* B, const float* X, int K, int rows, int cols,
                     float* C, const Tile& t) {
  if (t.rb >= rows || t.c0 >= cols) return;
  float acc[4][4];
  tile_mm<false>(A, B, K, t, acc);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = t.row(i);
    if (r >= rows) break;
    const float4 x = *reinterpret_cast<const float4*>(X + r * SB_LD + t.c0);
    const float v[4] = {x.x + acc[i][0], x.y + acc[i][1], x.z + acc[i][2], x.w + acc[i][3]};
    store_row4(C, r, t.c0, v);
  }
}

// Delta = g - I: alpha R in place (d = 1), or W = R/2 + alpha R^2 (d = 2).
// Returns the buffer that holds Delta.
SHP_DEV float* form_delta(int d, float alpha, float* R, float* W, int n, const Tile& t) {
  if (d == 1) {
    for (int e = threadIdx.x; e < n * n; e += SB_THREADS) {
      const int i = e / n, j = e - i * n;
      R[i * SB_LD + j] *= alpha;
    }
    __syncthreads();
    return R;
  }
  if (t.rb < n && t.c0 < n) {
    float acc[4][4];
    tile_mm<false>(R, R, n, t, acc);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = t.row(i);
      if (r >= n) break;
      const float4 q = *reinterpret_cast<const float4*>(R + r * SB_LD + t.c0);
      const float v[4] = {0.5f * q.x + alpha * acc[i][0], 0.5f * q.y + alpha * acc[i][1],
                          0.5f * q.z + alpha * acc[i][2], 0.5f * q.w + alpha * acc[i][3]};
      store_row4(W, r, t.c0, v);
    }
  }
  __syncthreads();
  return W;
}

// Vout = R Vin (n x p, row-major) by the whole CTA; each dot product runs as
// four interleaved partial sums (k mod 4) so that its FMA chain is n/4 long.
SHP_DEV void sketch_power(const float* R, const float* Vin, float* Vout, int n, int p) {
  for (int e = threadIdx.x; e < n * p; e += SB_THREADS) {
    const int row = e / p, col = e - row * p;
    const float* Rr = R + row * SB_LD;
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll 4
    for (int k = 0; k < n; k += 4) {
      const float4 r = *reinterpret_cast<const float4*>(Rr + k);
      s0 = fmaf(r.x, Vin[k * p + col], s0);
      s1 = fmaf(r.y, Vin[(k + 1) * p + col], s1);
      s2 = fmaf(r.z, Vin[(k + 2) * p + col], s2);
      s3 = fmaf(r.w, Vin[(k + 3) * p + col], s3);
    }
    Vout[e] = (s0 + s1) + (s2 + s3);
  }
  __syncthreads();
}

// alpha of degree e from V_e..V_{2e+1} (slot (j - 1) & 3 holds V_j): fp64
// Gram, quartic, minimiser on [lo, hi] by warp 0; every thread gets alpha and,
// through *s_ratio, sqrt(J(alpha)) / ||V_1||_F (the predicted contraction).
SHP_DEV float fit_degree(float* const* slot, int np, int e, double lo, double hi,
                         double (*red)[10], float* s_alpha, float* s_ratio) {
  const int tid = threadIdx.x, nv = e + 2;
  double part[10];
#pragma unroll
  for (int i = 0; i < 10; ++i) part[i] = 0.0;
  for (int q = tid; q < np; q += SB_THREADS) {
    double x[4];
    for (int i = 0; i < nv; ++i) x[i] = static_cast<double>(slot[(e + i - 1) & 3][q]);
    int idx = 0;
    for (int i = 0; i < nv; ++i)
      for (int j = i; j < nv; ++j) part[idx++] += x[i] * x[j];
  }
  const int warp = tid >> 5, lane = tid & 31;
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const double s = warp_sum(part[i]);
    if (lane == 0) red[warp][i] = s;
  }
  __syncthreads();
  if (tid < 32) {  // warp 0: every lane forms J, the warp finds its minimiser
    double M[4][4];
    int idx = 0;
    for (int i = 0; i < nv; ++i)
      for (int j = i; j < nv; ++j) {
        double s = 0.0;
        for (int w = 0; w < SB_THREADS / 32; ++w) s += red[w][idx];
        M[i][j] = M[j][i] = s;
        ++idx;
      }
    double coef[5];
    quartic_from_gram(M, e, coef);
    const double a = argmin_quartic_warp(coef, lo, hi);
    if (tid == 0) {
      *s_alpha = static_cast<float>(a);
      const double base = M[0][0];  // ||V_1||^2 when e = 1
      *s_ratio = base > 0.0 ? static_cast<float>(sqrt(fmax(poly4(coef, a), 0.0) / base)) : 0.f;
    }
  }
  __syncthreads();
  return *s_alpha;
}

// Sketched alpha of one iteration at degree *deg: V_j = R^j S_k (S_k = n x p
// slice in HBM), slot (j - 1) & 3 of the free buffer V holds V_j (S sits in
// slot 3 until V_4 replaces it).  With adaptive degree a block at degree 1
// fits on V_1..V_3 and, when the predicted contraction exceeds raise_above,
// continues to V_5 and fits at degree 2, which *deg keeps from then on.
SHP_DEV float sketch_alpha(const float* R, int n, const SmallCfg& o, const float* Sk, float* V,
                           int* deg, double (*red)[10], float* s_alpha, float* s_ratio) {
  const int p = o.p, np = n * p;
  float* slot[4] = {V, V + np, V + 2 * np, V + 3 * np};
  for (int e = threadIdx.x; e < np; e += SB_THREADS) slot[3][e] = Sk[e];
  __syncthreads();
  sketch_power(R, slot[3], slot[0], n, p);  // V_1
  sketch_power(R, slot[0], slot[1], n, p);  // V_2
  sketch_power(R, slot[1], slot[2], n, p);  // V_3
  float a = 0.f;
  if (*deg == 1) {
    a = fit_degree(slot, np, 1, o.adaptive ? 0.5 : static_cast<double>(o.lo),
                   static_cast<double>(o.hi), red, s_alpha, s_ratio);
    if (!(o.adaptive && *s_ratio > o.raise_above)) return a;
    *deg = 2;
  }
  sketch_power(R, slot[2], slot[3], n, p);  // V_4
  sketch_power(R, slot[3], slot[0], n, p);  // V_5
  return fit_degree(slot, np, 2, o.adaptive ? 0.375 : static_cast<double>(o.lo),
                    static_cast<double>(o.hi), red, s_alpha, s_ratio);
}

// Report slots: resid[b][pass][k] (max_iter + 1 per pass), alpha[b][pass][k]
// and degree[b][pass][k] (max_iter per pass), iters[b][pass], status[b].
struct SmallReport {
  int* status;
  int* iters;
  float* resid;
  float* alpha;
  int* degree;
};

// Coupled Newton-Schulz for A^(1/2), A^(-1/2) (one pass) or A^(-1/4) (a
// second pass on Y_1), one CTA per n x n block.
__global__ void __launch_bounds__(SB_THREADS, 3)
    k_small_inv_root(const float* __restrict__ A, int n, int npass, int power, SmallCfg o,
                     const float* __restrict__ S, float* __restrict__ X, SmallReport rep) {
  count_kernel_run();
  extern __shared__ __align__(16) float sm[];
  __shared__ double red[SB_THREADS / 32][10];
  __shared__ float s_alpha, s_ratio;
  const int b = blockIdx.x, tid = threadIdx.x;
  const Tile ts = tile_rows_strided();
  const int64_t nn = static_cast<int64_t>(n) * n;
  const float* Ab = A + b * nn;
  float *Y = sm, *Z = sm + SB_MAT, *R = sm + 2 * SB_MAT, *W = sm + 3 * SB_MAT;

  // c = ||A||_F (fp64) and Y_0 = (A + A^T) / (2c), the symmetric part (A / c
  // bit for bit when A is symmetric); A^T is read back from L1/L2
  double part = 0.0;
  for (int e = tid; e < nn; e += SB_THREADS) {
    const float v = Ab[e];
    part += static_cast<double>(v) * v;
  }
  const float c = static_cast<float>(sqrt(block_sum(part, red[0])));
  for (int e = tid; e < nn; e += SB_THREADS) {
    const int i = e / n, j = e - i * n;
    Y[i * SB_LD + j] = 0.5f * (Ab[e] + Ab[j * n + i]) / c;
  }
  __syncthreads();

  int status = ST_OK;
  const int mi = o.max_iter;
  for (int pass = 0; pass < npass; ++pass) {
    // Z_0 = I, R_0 = I - Y_0 (pass 2 starts from Y_1)
    float nrm = 0.f;
    for (int e = tid; e < nn; e += SB_THREADS) {
      const int i = e / n, j = e - i * n;
      const float id = i == j ? 1.f : 0.f;
      const float r = id - Y[i * SB_LD + j];
      Z[i * SB_LD + j] = id;
      R[i * SB_LD + j] = r;
      nrm += r * r;
    }
    double n2 = block_sum(nrm, red[0]);
    float prev = INFINITY;
    int deg = o.adaptive ? 1 : o.d;  // the degree of g for this pass (adaptive degree)
    for (int k = 0;; ++k) {
      if (k > 0) n2 = block_sum(residual<false>(Z, Y, n, n, R, ts), red[0]);
      // every thread evaluates the stop rule on the same reduced norm
      const float r = sqrtf(static_cast<float>(n2) / static_cast<float>(n));
      const int st = stop_rule(r, k, mi, o.tol, prev, o.stall_below, o.stall_ratio);
      if (tid == 0 && rep.resid != nullptr) rep.resid[(2 * b + pass) * (mi + 1) + k] = r;
      prev = r;
      if (st >= 0) {
        if (tid == 0 && rep.iters != nullptr) rep.iters[2 * b + pass] = k;
        if (status == ST_OK) status = st;
        break;
      }
      const float alpha =
          o.fixed_alpha ? o.lo
                        : sketch_alpha(R, n, o, S + (static_cast<int64_t>(pass) * mi + k) * n * o.p,
                                       W, &deg, red, &s_alpha, &s_ratio);
      if (tid == 0 && rep.alpha != nullptr) rep.alpha[(2 * b + pass) * mi + k] = alpha;
      if (tid == 0 && rep.degree != nullptr) rep.degree[(2 * b + pass) * mi + k] = deg;
      float* D = form_delta(deg, alpha, R, W, n, ts);
      float* T = deg == 1 ? W : R;  // the buffer Delta does not occupy
      axpy_mm(Y, D, Y, n, n, n, T, ts);  // Y_{k+1} = Y_k + Y_k Delta
      __syncthreads();
      if (k == 0) {  // Z_1 = I + Delta
        for (int e = tid; e < nn; e += SB_THREADS) {
          const int i = e / n, j = e - i * n;
          Y[i * SB_LD + j] = (i == j ? 1.f : 0.f) + D[i * SB_LD + j];
        }
      } else {  // Z_{k+1} = Z_k + Delta Z_k
        axpy_mm(D, Z, Z, n, n, n, Y, ts);
      }
      __syncthreads();
      float* oldZ = Z;
      Z = Y;
      Y = T;
      if (deg == 1)
        W = oldZ;
      else
        R = oldZ;
    }
  }

  double sc;
  const double cd = static_cast<double>(c);
  if (power == SHP_POW_SQRT)
    sc = sqrt(cd);
  else if (power == SHP_POW_INV2)
    sc = 1.0 / sqrt(cd);
  else
    sc = 1.0 / sqrt(sqrt(cd));
  const float scale = static_cast<float>(sc);
  const float* Src = power == SHP_POW_SQRT ? Y : Z;
  float* Xb = X + b * nn;
  for (int e = tid; e < nn; e += SB_THREADS) {
    const int i = e / n, j = e - i * n;
    Xb[e] = scale * Src[i * SB_LD + j];
  }
  if (tid == 0 && rep.status != nullptr) rep.status[b] = status;
}

// Polar factor of an m x n block (m, n <= 64): the tall iteration on G (or on
// G^T when m < n), X_0 = G / ||G||_F, R = I - X^T X, X <- X + X Delta.  With
// `sign` (m == n, G symmetric) the residual is I - X X: the sign function.
__global__ void __launch_bounds__(SB_THREADS, 3)
    k_small_polar(const float* __restrict__ G, int m, int n, SmallCfg o,
                  const float* __restrict__ S, float* __restrict__ Xout, SmallReport rep,
                  int sign, const int* __restrict__ dims, const int64_t* __restrict__ offs,
                  int64_t s_stride) {
  count_kernel_run();
  extern __shared__ __align__(16) float sm[];
  __shared__ double red[SB_THREADS / 32][10];
  __shared__ float s_alpha, s_ratio;
  const int b = blockIdx.x, tid = threadIdx.x;
  const Tile ts = tile_rows_strided(), tc = tile_rows_consecutive();
  int64_t boff = static_cast<int64_t>(b) * m * n;
  if (dims != nullptr) {  // blocks of different shapes, packed at offs[b]
    m = dims[2 * b];
    n = dims[2 * b + 1];
    boff = offs[b];
    if (m < 4 || n < 4 || m > SB_NMAX || n > SB_NMAX || (m & 3) || (n & 3) || boff < 0) {
      if (tid == 0 && rep.status != nullptr) rep.status[b] = ST_EINVAL;
      return;
    }
  }
  const bool tall = m >= n;
  const int rows = tall ? m : n, k_n = tall ? n : m;  // X is rows x k_n
  const int64_t mn = static_cast<int64_t>(m) * n;
  const float* Gb = G + boff;
  float *X = sm, *R = sm + SB_MAT, *W = sm + 2 * SB_MAT, *T = sm + 3 * SB_MAT;

  double part = 0.0;
  for (int e = tid; e < mn; e += SB_THREADS) {
    const float v = Gb[e];
    part += static_cast<double>(v) * v;
  }
  const float c = static_cast<float>(sqrt(block_sum(part, red[0])));
  // X_0 = G / ||G||_F as written (a zero block: 0/0, SHP_ENONFINITE)
  for (int e = tid; e < mn; e += SB_THREADS) {
    const int i = e / n, j = e - i * n;  // G(i, j)
    if (tall)
      X[i * SB_LD + j] = Gb[e] / c;
    else
      X[j * SB_LD + i] = Gb[e] / c;
  }
  __syncthreads();

  const int mi = o.max_iter;
  int status = ST_OK;
  float prev = INFINITY;
  int deg = o.adaptive ? 1 : o.d;
  for (int k = 0;; ++k) {
    // R = I - X^T X (polar) or I - X X (sign of a symmetric X, m == n)
    const double n2 = block_sum(sign ? residual<false>(X, X, rows, k_n, R, ts)
                                     : residual<true>(X, X, rows, k_n, R, tc),
                                red[0]);
    const float r = sqrtf(static_cast<float>(n2) / static_cast<float>(k_n));
    const int st = stop_rule(r, k, mi, o.tol, prev, o.stall_below, o.stall_ratio);
    if (tid == 0 && rep.resid != nullptr) rep.resid[2 * b * (mi + 1) + k] = r;
    prev = r;
    if (st >= 0) {
      if (tid == 0 && rep.iters != nullptr) rep.iters[2 * b] = k;
      status = st;
      break;
    }
    const float alpha =
        o.fixed_alpha ? o.lo
                      : sketch_alpha(R, k_n, o, S + static_cast<int64_t>(k) * s_stride, T, &deg,
                                     red, &s_alpha, &s_ratio);
    if (tid == 0 && rep.alpha != nullptr) rep.alpha[2 * b * mi + k] = alpha;
    if (tid == 0 && rep.degree != nullptr) rep.degree[2 * b * mi + k] = deg;
    float* D = form_delta(deg, alpha, R, W, k_n, ts);
    axpy_mm(X, D, X, k_n, rows, k_n, T, ts);  // X_{k+1} = X_k + X_k Delta
    __syncthreads();
    float* t = X;
    X = T;
    T = t;
  }

  float* Xb = Xout + boff;
  for (int e = tid; e < mn; e += SB_THREADS) {
    const int i = e / n, j = e - i * n;
    Xb[e] = tall ? X[i * SB_LD + j] : X[j * SB_LD + i];
  }
  if (tid == 0 && rep.status != nullptr) rep.status[b] = status;
}

SmallCfg make_cfg(const shp_prism_opts& s) {
  SmallCfg c;
  c.d = s.d;
  c.p = s.p;
  c.max_iter = s.max_iter;
  c.fixed_alpha = s.fixed_alpha;
  c.lo = s.lo;
  c.hi = s.hi;
  c.tol = s.tol;
  c.stall_below = s.stall_below;
  c.stall_ratio = s.stall_ratio;
  c.adaptive = s.adaptive_degree;
  c.raise_above = s.raise_above;
  return c;
}

template <typename K>
cudaError_t prepare(K kern) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SB_SMEM);
}

}  // namespace

bool small_block_ok(int64_t m, int64_t n, int p) {
  return m > 0 && n > 0 && m <= SB_NMAX && n <= SB_NMAX && p <= SB_PMAX;
}

cudaError_t small_inv_root(const float* A, int n, int batch, int power, const shp_prism_opts& o,
                           const float* S, float* X, int* rep_status, int* rep_iters,
                           float* rep_resid, float* rep_alpha, int* rep_degree, cudaStream_t st) {
  if (batch <= 0) return cudaSuccess;
  cudaError_t e = prepare(k_small_inv_root);
  if (e != cudaSuccess) return e;
  const int npass = power == SHP_POW_INV4 ? 2 : 1;
  k_small_inv_root<<<batch, SB_THREADS, SB_SMEM, st>>>(
      A, n, npass, power, make_cfg(o), S, X,
      SmallReport{rep_status, rep_iters, rep_resid, rep_alpha, rep_degree});
  return cudaGetLastError();
}

cudaError_t small_polar(const float* G, int m, int n, int batch, const shp_prism_opts& o,
                        const float* S, float* X, int* rep_status, int* rep_iters,
                        float* rep_resid, float* rep_alpha, int* rep_degree, bool sign,
                        cudaStream_t st) {
  if (batch <= 0) return cudaSuccess;
  cudaError_t e = prepare(k_small_polar);
  if (e != cudaSuccess) return e;
  const int k_n = m >= n ? n : m;
  k_small_polar<<<batch, SB_THREADS, SB_SMEM, st>>>(
      G, m, n, make_cfg(o), S, X,
      SmallReport{rep_status, rep_iters, rep_resid, rep_alpha, rep_degree}, sign ? 1 : 0,
      nullptr, nullptr, static_cast<int64_t>(k_n) * o.p);
  return cudaGetLastError();
}

cudaError_t small_polar_varsize(const float* G, const int* dims, const int64_t* offsets,
                                int batch, const shp_prism_opts& o, const float* S, float* X,
                                int* rep_status, int* rep_iters, float* rep_resid,
                                float* rep_alpha, int* rep_degree, cudaStream_t st) {
  if (batch <= 0) return cudaSuccess;
  cudaError_t e = prepare(k_small_polar);
  if (e != cudaSuccess) return e;
  k_small_polar<<<batch, SB_THREADS, SB_SMEM, st>>>(
      G, 0, 0, make_cfg(o), S, X,
      SmallReport{rep_status, rep_iters, rep_resid, rep_alpha, rep_degree}, 0, dims, offsets,
      static_cast<int64_t>(SB_NMAX) * o.p);
  return cudaGetLastError();
}

uint64_t kernel_runs_small() {
  unsigned long long v = 0;
  if (cudaMemcpyFromSymbol(&v, g_kernel_runs, sizeof(v)) != cudaSuccess) return 0;
  return v;
}

}  // namespace shp
