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
// Arithmetic: products and sketch powers on the tensor cores (warp-level
// mma.sync TF32 with the operands split into two TF32 parts, three products
// per pair: the 3xTF32 split of the batched path) with fp32 iterates; the
// alpha fit and the norms in fp64.  Four 64 x 68 fp32 buffers (68 KB) per
// CTA, three CTAs per SM.
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

// ---------------------------------------------------- products on the tensor cores
// Every product of the iteration is one 64 x 64 (or smaller) matrix in shared
// memory times another; each of the 8 warps computes a 16 x 32 block with
// mma.sync m16n8k8 TF32 (the warp-level MMA: one CTA's whole product is
// 0.26 MFLOP, too small for a tcgen05 issue / TMEM drain round trip per
// product, and the iteration's products depend on each other).  Operands are
// split in registers as x = hi + lo, hi = x rounded to TF32 and lo = the
// remainder rounded to TF32, and each product is lo*hi + hi*lo + hi*hi in the
// fp32 accumulator (the 3xTF32 split of the batched path).
SHP_DEV uint32_t tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

SHP_DEV void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  hi = tf32_rna(x);
  lo = tf32_rna(x - __uint_as_float(hi));
}

SHP_DEV void mma_16x8x8(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// This warp's 16 x 32 block of a 64 x 64 product: warp w covers rows
// 16 (w / 2) .. + 15 and columns 32 (w % 2) .. + 31; in the m16n8 accumulator
// layout a lane holds rows lr and lr + 8 (lr = lane / 4) of its block and the
// column pair lc, lc + 1 (lc = 2 (lane % 4)) of each of the four 8-column
// tiles: acc[nt][q] sits at (row(q / 2), col(nt) + q % 2).
struct WTile {
  int r0, c0, lr, lc;
  SHP_DEV int row(int h) const { return r0 + lr + 8 * h; }
  SHP_DEV int col(int nt) const { return c0 + 8 * nt + lc; }
};

SHP_DEV WTile warp_tile() {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  return WTile{16 * (w >> 1), 32 * (w & 1), l >> 2, 2 * (l & 3)};
}

// acc = op(A) B on the warp's block, op(A) = A (row-major, rows x K) or, with
// AT, the transpose of the row-major K x rows matrix A.  Terms with k >= K
// are zero (K need not be a multiple of 8); rows and columns past the
// operands' extents read in-buffer data whose results the callers do not
// store.  The fragment reads of a row-major operand fall on 32 distinct banks
// (row stride 68 floats); those of a transposed one on 16.
template <bool AT>
SHP_DEV void warp_mm(const float* A, const float* B, int K, const WTile& t, float acc[4][4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  const int lane = threadIdx.x & 31, lk = lane & 3, lm = lane >> 2;
  const int ra = t.r0 + lm, rb = ra + 8;
#pragma unroll 2
  for (int k0 = 0; k0 < K; k0 += 8) {
    const int ka = k0 + lk, kb = ka + 4;
    const bool va = ka < K, vb = kb < K;
    float af[4];
    if (AT) {
      af[0] = va ? A[ka * SB_LD + ra] : 0.f;
      af[1] = va ? A[ka * SB_LD + rb] : 0.f;
      af[2] = vb ? A[kb * SB_LD + ra] : 0.f;
      af[3] = vb ? A[kb * SB_LD + rb] : 0.f;
    } else {
      af[0] = va ? A[ra * SB_LD + ka] : 0.f;
      af[1] = va ? A[rb * SB_LD + ka] : 0.f;
      af[2] = vb ? A[ra * SB_LD + kb] : 0.f;
      af[3] = vb ? A[rb * SB_LD + kb] : 0.f;
    }
    uint32_t ah[4], al[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) split_tf32(af[i], ah[i], al[i]);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int cn = t.c0 + 8 * nt + lm;
      uint32_t bh0, bl0, bh1, bl1;
      split_tf32(va ? B[ka * SB_LD + cn] : 0.f, bh0, bl0);
      split_tf32(vb ? B[kb * SB_LD + cn] : 0.f, bh1, bl1);
      mma_16x8x8(acc[nt], al, bh0, bh1);
      mma_16x8x8(acc[nt], ah, bl0, bl1);
      mma_16x8x8(acc[nt], ah, bh0, bh1);
    }
  }
}

SHP_DEV void store2(float* C, int row, int col, float v0, float v1) {
  *reinterpret_cast<float2*>(C + row * SB_LD + col) = make_float2(v0, v1);
}

// R = I - op(A) B on the n x n grid; returns this thread's sum of squares.
// (The condition on the warp's block origin is the same for all its lanes, as
// mma.sync needs.)
template <bool AT>
SHP_DEV float residual(const float* A, const float* B, int K, int n, float* R, const WTile& t) {
  float nrm = 0.f;
  if (t.r0 < n && t.c0 < n) {
    float acc[4][4];
    warp_mm<AT>(A, B, K, t, acc);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = t.row(h), c = t.col(nt);
        if (r < n && c < n) {  // c even and n % 4 == 0: c + 1 < n too
          const float v0 = (r == c ? 1.f : 0.f) - acc[nt][2 * h];
          const float v1 = (r == c + 1 ? 1.f : 0.f) - acc[nt][2 * h + 1];
          nrm += v0 * v0 + v1 * v1;
          store2(R, r, c, v0, v1);
        }
      }
  }
  return nrm;
}

// C = X + A B (X may be A or B, C must be neither), rows x cols, inner K.
SHP_DEV void axpy_mm(const float* A, const float* B, const float* X, int K, int rows, int cols,
                     float* C, const WTile& t) {
  if (t.r0 >= rows || t.c0 >= cols) return;
  float acc[4][4];
  warp_mm<false>(A, B, K, t, acc);
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = t.row(h), c = t.col(nt);
      if (r < rows && c < cols) {
        const float2 x = *reinterpret_cast<const float2*>(X + r * SB_LD + c);
        store2(C, r, c, x.x + acc[nt][2 * h], x.y + acc[nt][2 * h + 1]);
      }
    }
}

// Delta = g - I: alpha R in place (d = 1), or W = R/2 + alpha R^2 (d = 2).
// Returns the buffer that holds Delta.
SHP_DEV float* form_delta(int d, float alpha, float* R, float* W, int n, const WTile& t) {
  if (d == 1) {
    for (int e = threadIdx.x; e < n * n; e += SB_THREADS) {
      const int i = e / n, j = e - i * n;
      R[i * SB_LD + j] *= alpha;
    }
    __syncthreads();
    return R;
  }
  if (t.r0 < n && t.c0 < n) {
    float acc[4][4];
    warp_mm<false>(R, R, n, t, acc);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = t.row(h), c = t.col(nt);
        if (r < n && c < n) {
          const float2 q = *reinterpret_cast<const float2*>(R + r * SB_LD + c);
          store2(W, r, c, 0.5f * q.x + alpha * acc[nt][2 * h], 0.5f * q.y + alpha * acc[nt][2 * h + 1]);
        }
      }
  }
  __syncthreads();
  return W;
}

// Vout = R Vin (n x p, row-major with row stride p) on the tensor cores, the
// same 3xTF32 split as the products: warp w computes rows 16 (w % 4) .. + 15
// and sketch columns 8 (w / 4) .. + 7 (p <= 16; columns past p and terms past
// n are zero, and rows past n are not stored).
SHP_DEV void sketch_power(const float* R, const float* Vin, float* Vout, int n, int p) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, lk = lane & 3, lm = lane >> 2;
  const int r0 = 16 * (w & 3), c0 = 8 * (w >> 2);
  if (r0 < n && c0 < p) {  // the same for the whole warp, as mma.sync needs
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int ra = r0 + lm, rb = ra + 8, cn = c0 + lm;
    const bool vc = cn < p;
#pragma unroll 2
    for (int k0 = 0; k0 < n; k0 += 8) {
      const int ka = k0 + lk, kb = ka + 4;
      const bool va = ka < n, vb = kb < n;
      const float af[4] = {va ? R[ra * SB_LD + ka] : 0.f, va ? R[rb * SB_LD + ka] : 0.f,
                           vb ? R[ra * SB_LD + kb] : 0.f, vb ? R[rb * SB_LD + kb] : 0.f};
      uint32_t ah[4], al[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) split_tf32(af[i], ah[i], al[i]);
      uint32_t bh0, bl0, bh1, bl1;
      split_tf32(va && vc ? Vin[ka * p + cn] : 0.f, bh0, bl0);
      split_tf32(vb && vc ? Vin[kb * p + cn] : 0.f, bh1, bl1);
      mma_16x8x8(acc, al, bh0, bh1);
      mma_16x8x8(acc, ah, bl0, bl1);
      mma_16x8x8(acc, ah, bh0, bh1);
    }
    const int cc = c0 + 2 * lk;  // the lane's column pair
    if (ra < n) {
      if (cc < p) Vout[ra * p + cc] = acc[0];
      if (cc + 1 < p) Vout[ra * p + cc + 1] = acc[1];
    }
    if (rb < n) {
      if (cc < p) Vout[rb * p + cc] = acc[2];
      if (cc + 1 < p) Vout[rb * p + cc + 1] = acc[3];
    }
  }
  __syncthreads();
}

// alpha of degree E from V_E..V_{2E+1} (slot (j - 1) & 3 holds V_j): fp64
// Gram, quartic, minimiser on [lo, hi] by warp 0; every thread gets alpha and,
// through *s_ratio, sqrt(J(alpha)) / ||V_1||_F (the predicted contraction).
// E is a template argument so that every loop unrolls and the Gram stays in
// registers.
template <int E>
SHP_DEV float fit_degree(float* const* slot, int np, double lo, double hi, double (*red)[10],
                         float* s_alpha, float* s_ratio) {
  constexpr int NV = E + 2;
  const int tid = threadIdx.x;
  double part[10];
#pragma unroll
  for (int i = 0; i < 10; ++i) part[i] = 0.0;
  for (int q = tid; q < np; q += SB_THREADS) {
    double x[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) x[i] = static_cast<double>(slot[(E + i - 1) & 3][q]);
    int idx = 0;
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
      for (int j = i; j < NV; ++j) part[idx++] += x[i] * x[j];
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
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
      for (int j = i; j < NV; ++j) {
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < SB_THREADS / 32; ++w) s += red[w][idx];
        M[i][j] = M[j][i] = s;
        ++idx;
      }
    double coef[5];
    quartic_from_gram_d<E>(M, coef);
    const double a = argmin_quartic_warp(coef, lo, hi);
    if (tid == 0) {
      *s_alpha = static_cast<float>(a);
      const double base = M[0][0];  // ||V_1||^2 when E = 1
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
    a = fit_degree<1>(slot, np, o.adaptive ? 0.5 : static_cast<double>(o.lo),
                      static_cast<double>(o.hi), red, s_alpha, s_ratio);
    if (!(o.adaptive && *s_ratio > o.raise_above)) return a;
    *deg = 2;
  }
  sketch_power(R, slot[2], slot[3], n, p);  // V_4
  sketch_power(R, slot[3], slot[0], n, p);  // V_5
  return fit_degree<2>(slot, np, o.adaptive ? 0.375 : static_cast<double>(o.lo),
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
  const WTile ts = warp_tile();
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
  const WTile ts = warp_tile();
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
                                     : residual<true>(X, X, rows, k_n, R, ts),
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
