// PRISM sketched alpha fit and per-block iteration control.
//
// "Sintesi Tecnica: PRISM", Parte II.1-II.2: the top coefficient alpha of the
// update polynomial g_d(xi; alpha) = f_{d-1}(xi) + alpha xi^d is chosen each
// iteration by a least-squares fit of the next residual on the spectrum of
// R_k, constrained to [l, u], and the fit is made on a Gaussian sketch S so
// that it costs O(n^2 p) instead of traces of high powers of R_k.
//
// With g = f + alpha xi^d the next residual of the square-root family is
//   r(xi; alpha) = 1 - (1 - xi) g^2
//                = [1 - (1-xi) f^2] - 2 alpha (1-xi) xi^d f - alpha^2 (1-xi) xi^{2d},
// a polynomial in xi whose coefficients r_j are quadratics in alpha and vanish
// outside j = d..2d+1.  Hence, with V_j = R_k^j S and M_ij = <V_i, V_j>_F,
//   J(alpha) = ||r(R_k; alpha) S||_F^2 = sum_{i,j} r_i(alpha) r_j(alpha) M_ij,
// a quartic in alpha whose minimiser on [lo, hi] is the new alpha_k.
//
// Kernels: the skinny products V_j = R V_{j-1} on CUDA cores (fp32 FMA, HBM
// bound), the Gram/quartic/argmin per block (fp64), and the stop test.
#include <math.h>

#include "internal.h"
#include "prism_scalar.cuh"
#include "shp_common.cuh"

namespace shp {

namespace {

constexpr int SK_THREADS = 256;
constexpr int SK_GROUPS = 2;  // row groups per warp in one CTA

// Vout = R * Vin for one block: HBM-bound, every byte of R read once.
// Each warp owns ROWS consecutive rows of R per group and streams them with
// 128-bit loads (a lane takes 4 consecutive columns), two 128-column steps
// per iteration so that 2 * ROWS loads per lane are in flight before the
// first is used; a CTA covers GROUPS groups per warp so that one staging of V
// serves 8 * ROWS * GROUPS rows.  V is staged in shared memory transposed,
// Vs[j][c], one 32 KB chunk of columns at a time, with rows padded by 4
// floats so that both the staging stores and the float4 reads of a warp are
// conflict-free.  Rows past n re-read row n-1 (never stored), which keeps
// the loads free of branches.  Requires n % 4 == 0 (16-byte rows).
template <int P>
__global__ void __launch_bounds__(SK_THREADS, 2)
    k_sketch(const float* __restrict__ Rhi, const float* __restrict__ Rlo, int64_t n,
             int64_t rbs, const float* __restrict__ Vin, int64_t vbs, float* __restrict__ Vout,
             int64_t obs, int p, const int* __restrict__ active, const int* __restrict__ it,
             int64_t it_stride) {
  count_kernel_run();
  constexpr int ROWS = P <= 8 ? 4 : 2;
  constexpr int CK = 8192 / P;  // columns per chunk (a multiple of 256)
  constexpr int LDV = CK + 4;
  __shared__ __align__(16) float Vs[P][LDV];
  const int b = blockIdx.y;
  if (active != nullptr && active[b] == 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t cta_row0 = static_cast<int64_t>(blockIdx.x) * (8 * ROWS * SK_GROUPS);
  const float* R = Rhi + b * rbs;
  const float* RL = Rlo != nullptr ? Rlo + b * rbs : nullptr;
  const float* V = Vin + b * vbs + (it != nullptr ? static_cast<int64_t>(*it) * it_stride : 0);
  const bool one_chunk = n <= CK;  // V staged once for every group

  for (int g = 0; g < SK_GROUPS; ++g) {
    const int64_t row0 = cta_row0 + static_cast<int64_t>(g * 8 + warp) * ROWS;
    if (cta_row0 + static_cast<int64_t>(g * 8) * ROWS >= n) break;  // uniform over the CTA
    int64_t roff[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) roff[r] = (row0 + r < n ? row0 + r : n - 1) * n;
    float acc[ROWS][P];
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
#pragma unroll
      for (int j = 0; j < P; ++j) acc[r][j] = 0.f;

    for (int64_t c0 = 0; c0 < n; c0 += CK) {
      if (!(one_chunk && g > 0)) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < CK * (P / 4); idx += SK_THREADS) {
          const int cc = idx / (P / 4), q = 4 * (idx % (P / 4));
          const int64_t col = c0 + cc;
          const float* src = V + col * p + q;
#pragma unroll
          for (int e = 0; e < 4; ++e)
            Vs[q + e][cc] = (col < n && q + e < p) ? __ldg(src + e) : 0.f;
        }
        __syncthreads();
      }
      for (int cc = lane * 4; cc < CK; cc += 256) {
        const int64_t col = c0 + cc;
        if (col >= n) break;
        const bool second = col + 128 < n;
        float4 x0[ROWS], x1[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
          x0[r] = *reinterpret_cast<const float4*>(R + roff[r] + col);
          x1[r] = second ? *reinterpret_cast<const float4*>(R + roff[r] + col + 128)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (RL != nullptr) {
#pragma unroll
          for (int r = 0; r < ROWS; ++r) {
            const float4 y0 = *reinterpret_cast<const float4*>(RL + roff[r] + col);
            x0[r].x += y0.x;
            x0[r].y += y0.y;
            x0[r].z += y0.z;
            x0[r].w += y0.w;
            if (second) {
              const float4 y1 = *reinterpret_cast<const float4*>(RL + roff[r] + col + 128);
              x1[r].x += y1.x;
              x1[r].y += y1.y;
              x1[r].z += y1.z;
              x1[r].w += y1.w;
            }
          }
        }
#pragma unroll
        for (int j = 0; j < P; ++j) {
          const float4 v0 = *reinterpret_cast<const float4*>(&Vs[j][cc]);
          const float4 v1 = *reinterpret_cast<const float4*>(&Vs[j][cc + 128]);
#pragma unroll
          for (int r = 0; r < ROWS; ++r) {
            float a = acc[r][j];
            a = fmaf(x0[r].x, v0.x, a);
            a = fmaf(x0[r].y, v0.y, a);
            a = fmaf(x0[r].z, v0.z, a);
            a = fmaf(x0[r].w, v0.w, a);
            a = fmaf(x1[r].x, v1.x, a);
            a = fmaf(x1[r].y, v1.y, a);
            a = fmaf(x1[r].z, v1.z, a);
            acc[r][j] = fmaf(x1[r].w, v1.w, a);
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
#pragma unroll
      for (int j = 0; j < P; ++j) {
        const float sum = warp_sum(acc[r][j]);
        const int64_t row = row0 + r;
        if (lane == 0 && row < n && j < p) Vout[b * obs + row * p + j] = sum;
      }
    }
  }
}

constexpr int AL_THREADS = 256;

// Per-block alpha of one iteration.  Without adaptive degree: the Gram of
// V_d..V_{2d+1}, the quartic and its minimiser on [lo, hi].  With adaptive
// degree (d = 2): the Gram of V_1..V_5 at once; a block at degree 1 fits on
// V_1..V_3 over [1/2, hi] and, when sqrt(J_1(alpha*)) / ||V_1||_F exceeds
// raise_above, moves to degree 2 (V_2..V_5 over [3/8, hi]) for the rest of
// the pass.  act1/act2 then mark the active blocks at each degree for the
// masked launches that form Delta.
struct AlphaArgs {
  const float* V;
  int64_t n, vbs;
  int p, d, fixed;
  float lo, hi;
  const int* active;
  float* alpha;
  double* Jc;
  float* rep;
  int64_t rep_stride;
  int rep_slot;
  const int* it;
  int adaptive;
  float raise_above;
  int* deg;
  int* act1;
  int* act2;
  int* rep_deg;
};

__global__ void __launch_bounds__(AL_THREADS) k_alpha(AlphaArgs g) {
  count_kernel_run();
  const int b = blockIdx.x;
  if (g.active != nullptr && g.active[b] == 0) {
    if (g.adaptive && threadIdx.x == 0) {
      g.act1[b] = 0;
      g.act2[b] = 0;
    }
    return;
  }
  const int rep_slot = g.rep_slot + (g.it != nullptr ? *g.it : 0);
  if (g.fixed) {  // plain Taylor step: alpha = lo, no sketch needed
    if (threadIdx.x == 0) {
      g.alpha[b] = g.lo;
      if (g.rep != nullptr) g.rep[b * g.rep_stride + rep_slot] = g.lo;
      if (g.rep_deg != nullptr) g.rep_deg[b * g.rep_stride + rep_slot] = g.d;
    }
    return;
  }
  const int first = g.adaptive ? 1 : g.d;     // V_first .. V_{first + nv - 1}
  const int nv = g.adaptive ? 5 : g.d + 2;
  const int64_t len = g.n * g.p;
  const float* Vb = g.V + b * g.vbs + static_cast<int64_t>(first) * len;
  double part[15];
#pragma unroll
  for (int i = 0; i < 15; ++i) part[i] = 0.0;
  for (int64_t e = threadIdx.x; e < len; e += AL_THREADS) {
    double x[5];
    for (int i = 0; i < nv; ++i) x[i] = static_cast<double>(Vb[i * len + e]);
    int idx = 0;
    for (int i = 0; i < nv; ++i)
      for (int j = i; j < nv; ++j) part[idx++] += x[i] * x[j];
  }
  __shared__ double red[AL_THREADS / 32][15];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 15; ++i) {
    const double s = warp_sum(part[i]);
    if (lane == 0) red[warp][i] = s;
  }
  __syncthreads();
  if (threadIdx.x >= 32) return;  // warp 0 forms J and finds its minimiser
  double G[5][5];
  {
    int idx = 0;
    for (int i = 0; i < nv; ++i)
      for (int j = i; j < nv; ++j) {
        double s = 0.0;
        for (int w = 0; w < AL_THREADS / 32; ++w) s += red[w][idx];
        G[i][j] = G[j][i] = s;
        ++idx;
      }
  }
  // fit at degree e on the Gram block starting at V_e (offset e - first)
  auto fit = [&](int e, double lo, double* coef) {
    double M[4][4];
    const int o = e - first;
    for (int i = 0; i < e + 2; ++i)
      for (int j = 0; j < e + 2; ++j) M[i][j] = G[o + i][o + j];
    quartic_from_gram(M, e, coef);
    return argmin_quartic_warp(coef, lo, static_cast<double>(g.hi));
  };
  double coef[5];
  int dcur = g.d;
  double a;
  if (!g.adaptive) {
    a = fit(g.d, static_cast<double>(g.lo), coef);
  } else {
    dcur = g.deg[b];
    if (dcur == 1) {
      a = fit(1, 0.5, coef);
      const double J = poly4(coef, a), base = G[0][0];  // ||V_1||^2 = ||R_k S_k||^2
      if (base > 0.0 && sqrt(fmax(J, 0.0) / base) > static_cast<double>(g.raise_above))
        dcur = 2;
    }
    if (dcur == 2) a = fit(2, 0.375, coef);
  }
  if (threadIdx.x != 0) return;
  g.alpha[b] = static_cast<float>(a);
  if (g.Jc != nullptr)
    for (int i = 0; i < 5; ++i) g.Jc[b * 5 + i] = coef[i];
  if (g.rep != nullptr) g.rep[b * g.rep_stride + rep_slot] = static_cast<float>(a);
  if (g.rep_deg != nullptr) g.rep_deg[b * g.rep_stride + rep_slot] = dcur;
  if (g.adaptive) {
    g.deg[b] = dcur;
    g.act1[b] = dcur == 1;
    g.act2[b] = dcur == 2;
  }
}

__global__ void k_control(BlockState* bs, int* active, const int* it, int batch, int64_t n,
                          int max_iter, float tol, float stall_below, float stall_ratio,
                          float* rep_res, int64_t res_stride, int res_slot, int* rep_iters,
                          int iters_slot) {
  count_kernel_run();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= batch || active[b] == 0) return;
  const int k = *it;
  BlockState& s = bs[b];
  const float r = sqrtf(s.norm2 / static_cast<float>(n));
  s.norm2 = 0.f;
  if (rep_res != nullptr) rep_res[b * res_stride + res_slot + k] = r;
  const int st = stop_rule(r, k, max_iter, tol, s.prev_res, stall_below, stall_ratio);
  s.prev_res = r;
  if (st >= 0) {
    active[b] = 0;
    s.iters = k;
    s.pass_status = st;
    if (s.status == ST_OK) s.status = st;
    if (rep_iters != nullptr) rep_iters[b * 2 + iters_slot] = k;
  }
}

}  // namespace

cudaError_t sketch_pass(const float* Rhi, const float* Rlo, int64_t n, int64_t r_bstride,
                        const float* Vin, int64_t vin_bstride, float* Vout, int64_t vout_bstride,
                        int p, int batch, const int* active, const int* it, int64_t it_stride,
                        cudaStream_t st) {
  if (batch <= 0 || n <= 0) return cudaSuccess;
  const int rows = (p <= 8 ? 4 : 2) * 8 * SK_GROUPS;  // rows per CTA (ROWS x 8 warps x groups)
  dim3 grid(static_cast<unsigned>((n + rows - 1) / rows), batch);
  if (p <= 4)
    k_sketch<4><<<grid, SK_THREADS, 0, st>>>(Rhi, Rlo, n, r_bstride, Vin, vin_bstride, Vout,
                                             vout_bstride, p, active, it, it_stride);
  else if (p <= 8)
    k_sketch<8><<<grid, SK_THREADS, 0, st>>>(Rhi, Rlo, n, r_bstride, Vin, vin_bstride, Vout,
                                             vout_bstride, p, active, it, it_stride);
  else if (p <= 16)
    k_sketch<16><<<grid, SK_THREADS, 0, st>>>(Rhi, Rlo, n, r_bstride, Vin, vin_bstride, Vout,
                                              vout_bstride, p, active, it, it_stride);
  else
    k_sketch<32><<<grid, SK_THREADS, 0, st>>>(Rhi, Rlo, n, r_bstride, Vin, vin_bstride, Vout,
                                              vout_bstride, p, active, it, it_stride);
  return cudaGetLastError();
}

cudaError_t alpha_solve(const float* V, int64_t n, int p, int d, int batch, float lo, float hi,
                        int fixed_alpha, const int* active, float* alpha, double* J_coef,
                        float* report_alpha, int64_t report_stride, int report_slot,
                        const int* it, cudaStream_t st, const AdaptiveDeg* ad) {
  if (batch <= 0) return cudaSuccess;
  AlphaArgs g;
  g.V = V;
  g.n = n;
  g.vbs = static_cast<int64_t>(2 * d + 2) * n * p;
  g.p = p;
  g.d = d;
  g.fixed = fixed_alpha;
  g.lo = lo;
  g.hi = hi;
  g.active = active;
  g.alpha = alpha;
  g.Jc = J_coef;
  g.rep = report_alpha;
  g.rep_stride = report_stride;
  g.rep_slot = report_slot;
  g.it = it;
  g.adaptive = ad != nullptr && ad->enabled;
  g.raise_above = ad != nullptr ? ad->raise_above : 0.f;
  g.deg = ad != nullptr ? ad->deg : nullptr;
  g.act1 = ad != nullptr ? ad->act1 : nullptr;
  g.act2 = ad != nullptr ? ad->act2 : nullptr;
  g.rep_deg = ad != nullptr ? ad->rep_degree : nullptr;
  k_alpha<<<batch, AL_THREADS, 0, st>>>(g);
  return cudaGetLastError();
}

cudaError_t control_step(const Ctl& ctl, int batch, int64_t n, int max_iter, float tol,
                         float stall_below, float stall_ratio, float* report_res,
                         int64_t res_stride, int res_slot, int* report_iters, int iters_slot,
                         cudaStream_t st) {
  if (batch <= 0) return cudaSuccess;
  k_control<<<(batch + 127) / 128, 128, 0, st>>>(ctl.bs, ctl.active, ctl.it, batch, n, max_iter,
                                                 tol, stall_below, stall_ratio, report_res,
                                                 res_stride, res_slot, report_iters, iters_slot);
  return cudaGetLastError();
}

namespace {
__global__ void k_loop_step(const int* active, int* it, int* flag, int batch, int inc,
                            int max_iter, cudaGraphConditionalHandle h) {
  count_kernel_run();
  int any = 0;
  for (int b = threadIdx.x; b < batch; b += blockDim.x) any |= active[b];
  any = __syncthreads_or(any);
  if (threadIdx.x == 0) {
    const int k = *it + inc;
    *it = k;
    const unsigned cond = (any != 0 && k <= max_iter + 1) ? 1u : 0u;
    if (h != 0)
      cudaGraphSetConditional(h, cond);
    else
      *flag = static_cast<int>(cond);
  }
}
}  // namespace

cudaError_t loop_step(const Ctl& ctl, int batch, int inc, int max_iter,
                      cudaGraphConditionalHandle h, cudaStream_t st) {
  k_loop_step<<<1, 256, 0, st>>>(ctl.active, ctl.it, ctl.flag, batch, inc, max_iter, h);
  return cudaGetLastError();
}

uint64_t kernel_runs_sketch() {
  unsigned long long v = 0;
  if (cudaMemcpyFromSymbol(&v, g_kernel_runs, sizeof(v)) != cudaSuccess) return 0;
  return v;
}

}  // namespace shp
