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

// Vout = R * Vin for one block.  Each warp owns ROWS consecutive rows of R
// and streams them with 128-bit loads (a lane takes 4 consecutive columns);
// V is staged in shared memory transposed, Vs[j][c], one 32 KB chunk of
// columns at a time, so that lane reads are conflict-free float4 as well.
// Requires n % 4 == 0 (16-byte rows).
template <int P>
__global__ void __launch_bounds__(SK_THREADS)
    k_sketch(const float* __restrict__ Rhi, const float* __restrict__ Rlo, int64_t n,
             int64_t rbs, const float* __restrict__ Vin, int64_t vbs, float* __restrict__ Vout,
             int64_t obs, int p, const int* __restrict__ active, const int* __restrict__ it,
             int64_t it_stride) {
  count_kernel_run();
  constexpr int ROWS = P <= 16 ? 4 : 2;
  constexpr int CK = 8192 / P;  // columns per chunk: Vs is 32 KB
  __shared__ __align__(16) float Vs[P][CK];
  const int b = blockIdx.y;
  if (active != nullptr && active[b] == 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * (8 * ROWS) + warp * ROWS;
  const float* R = Rhi + b * rbs;
  const float* RL = Rlo != nullptr ? Rlo + b * rbs : nullptr;
  const float* V = Vin + b * vbs + (it != nullptr ? static_cast<int64_t>(*it) * it_stride : 0);
  float acc[ROWS][P];
#pragma unroll
  for (int r = 0; r < ROWS; ++r)
#pragma unroll
    for (int j = 0; j < P; ++j) acc[r][j] = 0.f;

  for (int64_t c0 = 0; c0 < n; c0 += CK) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < CK * P; idx += SK_THREADS) {
      const int cc = idx / P, j = idx % P;
      const int64_t col = c0 + cc;
      Vs[j][cc] = (j < p && col < n) ? V[col * p + j] : 0.f;
    }
    __syncthreads();
    for (int cc = lane * 4; cc < CK; cc += 128) {
      const int64_t col = c0 + cc;
      if (col >= n) break;
      float4 rv[ROWS];
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        const int64_t row = row0 + r;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row < n) {
          x = *reinterpret_cast<const float4*>(R + row * n + col);
          if (RL != nullptr) {
            const float4 y = *reinterpret_cast<const float4*>(RL + row * n + col);
            x.x += y.x;
            x.y += y.y;
            x.z += y.z;
            x.w += y.w;
          }
        }
        rv[r] = x;
      }
#pragma unroll
      for (int j = 0; j < P; ++j) {
        const float4 vj = *reinterpret_cast<const float4*>(&Vs[j][cc]);
#pragma unroll
        for (int r = 0; r < ROWS; ++r)
          acc[r][j] = fmaf(rv[r].x, vj.x,
                           fmaf(rv[r].y, vj.y, fmaf(rv[r].z, vj.z, fmaf(rv[r].w, vj.w, acc[r][j]))));
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

constexpr int AL_THREADS = 256;

__global__ void __launch_bounds__(AL_THREADS)
    k_alpha(const float* __restrict__ V, int64_t n, int p, int d, int64_t vbs, float lo,
            float hi, int fixed, const int* __restrict__ active, float* __restrict__ alpha,
            double* __restrict__ Jc, float* __restrict__ rep, int64_t rep_stride, int rep_slot,
            const int* __restrict__ it) {
  count_kernel_run();
  const int b = blockIdx.x;
  if (active != nullptr && active[b] == 0) return;
  if (it != nullptr) rep_slot += *it;
  if (fixed) {  // plain Taylor step: alpha = lo, no sketch needed
    if (threadIdx.x == 0) {
      alpha[b] = lo;
      if (rep != nullptr) rep[b * rep_stride + rep_slot] = lo;
    }
    return;
  }
  const int nv = d + 2;               // V_d .. V_{2d+1}
  const int64_t len = n * p;
  const float* Vb = V + b * vbs + static_cast<int64_t>(d) * len;
  double part[10];
#pragma unroll
  for (int i = 0; i < 10; ++i) part[i] = 0.0;
  for (int64_t e = threadIdx.x; e < len; e += AL_THREADS) {
    double x[4];
    for (int i = 0; i < nv; ++i) x[i] = static_cast<double>(Vb[i * len + e]);
    int idx = 0;
    for (int i = 0; i < nv; ++i)
      for (int j = i; j < nv; ++j) part[idx++] += x[i] * x[j];
  }
  __shared__ double red[AL_THREADS / 32][10];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const double s = warp_sum(part[i]);
    if (lane == 0) red[warp][i] = s;
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  double M[4][4];
  {
    int idx = 0;
    for (int i = 0; i < nv; ++i)
      for (int j = i; j < nv; ++j) {
        double s = 0.0;
        for (int w = 0; w < AL_THREADS / 32; ++w) s += red[w][idx];
        M[i][j] = M[j][i] = s;
        ++idx;
      }
  }
  double coef[5];
  quartic_from_gram(M, d, coef);
  const double a = argmin_quartic(coef, static_cast<double>(lo), static_cast<double>(hi));
  alpha[b] = static_cast<float>(a);
  if (Jc != nullptr)
    for (int i = 0; i < 5; ++i) Jc[b * 5 + i] = coef[i];
  if (rep != nullptr) rep[b * rep_stride + rep_slot] = static_cast<float>(a);
}

// ------------------------------------------------------------------------
// The whole sketch chain and alpha fit of one block in one cluster.
//
// Eight CTAs (one thread-block cluster) own one block at a time and loop over
// the batch.  CTA r computes rows [r n/8, (r+1) n/8) of every V_j = R V_{j-1},
// j = 1..2d+1, and writes them into the V_j buffer of all eight CTAs through
// distributed shared memory; one cluster barrier per power makes V_j whole
// everywhere.  Only 8 x (the resident clusters) blocks' R (4 MB each at
// n = 1024) are live at a time, so the 2d+1 reads of R after the first come
// from L2.  The fp64 Gram of V_d..V_{2d+1} is reduced over the cluster into
// the leader CTA, whose thread 0 forms the quartic and takes its argmin: the
// same arithmetic as k_sketch + k_alpha, with one launch instead of 2d+2.
constexpr int SC_CS = 8;
constexpr int SC_THREADS = 512;
constexpr int SC_WARPS = SC_THREADS / 32;
constexpr int SC_VFLOATS = 8192;  // n * P per V buffer (32 KB)
// 2 V buffers + own rows of d+2 powers; padded so that one CTA fits per SM
constexpr int SC_SMEM = 120 * 1024;
static_assert((2 * SC_VFLOATS + 4 * (SC_VFLOATS / SC_CS)) * 4 <= SC_SMEM, "sketch chain smem");

SHP_DEV void st_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
SHP_DEV void st_cluster_f64(uint32_t addr, double v) {
  asm volatile("st.shared::cluster.f64 [%0], %1;" ::"r"(addr), "d"(v) : "memory");
}

template <int P>
__global__ void __launch_bounds__(SC_THREADS, 1)
    k_sketch_chain(const float* __restrict__ R, int n, int batch, const float* __restrict__ S,
                   const int* __restrict__ it, int p, int d, float lo, float hi,
                   const int* __restrict__ active, float* __restrict__ alpha,
                   float* __restrict__ rep, int64_t rep_stride, int rep_slot) {
  count_kernel_run();
  extern __shared__ __align__(16) float sc_sm[];
  __shared__ double gpart[SC_WARPS][10];
  __shared__ double gclu[SC_CS][10];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t crank = cluster_rank();
  const int cl = static_cast<int>(blockIdx.x) / SC_CS, ncl = static_cast<int>(gridDim.x) / SC_CS;
  const int rows = (n + SC_CS - 1) / SC_CS;
  const int r_begin = static_cast<int>(crank) * rows;
  const int r_end = r_begin + rows < n ? r_begin + rows : n;
  const int nv = d + 2;
  const int k = it != nullptr ? *it : 0;
  const float* Sk = S + static_cast<int64_t>(k) * n * p;
  float* Vown = sc_sm + 2 * P * n;  // [nv][rows][P]

  for (int b = cl; b < batch; b += ncl) {
    if (active != nullptr && active[b] == 0) continue;  // uniform over the cluster
    float* Vc = sc_sm;          // V_{j-1}, transposed [P][n]
    float* Vn = sc_sm + P * n;  // V_j
    for (int idx = tid; idx < P * n; idx += SC_THREADS) {
      const int j = idx / n, col = idx - j * n;
      Vc[idx] = j < p ? Sk[static_cast<int64_t>(col) * p + j] : 0.f;
    }
    __syncthreads();
    const float* Rb = R + static_cast<int64_t>(b) * n * n;
    for (int jp = 1; jp <= 2 * d + 1; ++jp) {
      // two rows per warp step; each lane takes 4 consecutive columns of
      // every 128-column stripe, four stripes in flight
      for (int row = r_begin + 2 * warp; row < r_end; row += 2 * SC_WARPS) {
        const bool two = row + 1 < r_end;
        const float* r0p = Rb + static_cast<int64_t>(row) * n;
        const float* r1p = two ? r0p + n : r0p;
        float acc0[P], acc1[P];
#pragma unroll
        for (int j = 0; j < P; ++j) acc0[j] = acc1[j] = 0.f;
        for (int c0 = lane * 4; c0 < n; c0 += 512) {
          float4 x0[4], x1[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int c = c0 + 128 * t;
            x0[t] = c < n ? *reinterpret_cast<const float4*>(r0p + c) : make_float4(0, 0, 0, 0);
            x1[t] = c < n ? *reinterpret_cast<const float4*>(r1p + c) : make_float4(0, 0, 0, 0);
          }
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int c = c0 + 128 * t;
            if (c >= n) break;
#pragma unroll
            for (int j = 0; j < P; ++j) {
              const float4 v = *reinterpret_cast<const float4*>(Vc + j * n + c);
              acc0[j] = fmaf(x0[t].x, v.x, fmaf(x0[t].y, v.y, fmaf(x0[t].z, v.z,
                        fmaf(x0[t].w, v.w, acc0[j]))));
              acc1[j] = fmaf(x1[t].x, v.x, fmaf(x1[t].y, v.y, fmaf(x1[t].z, v.z,
                        fmaf(x1[t].w, v.w, acc1[j]))));
            }
          }
        }
#pragma unroll
        for (int j = 0; j < P; ++j) {
          acc0[j] = warp_sum(acc0[j]);
          acc1[j] = warp_sum(acc1[j]);
        }
        // lane q < 8 stores both rows' P values into CTA q's V_j; lane 8 + j
        // keeps column j of the rows this CTA owns (powers d..2d+1)
        if (lane < SC_CS) {
          const uint32_t base = mapa_shared(smem_u32(Vn), static_cast<uint32_t>(lane));
#pragma unroll
          for (int j = 0; j < P; ++j) {
            st_cluster_f32(base + static_cast<uint32_t>((j * n + row) * 4), acc0[j]);
            if (two) st_cluster_f32(base + static_cast<uint32_t>((j * n + row + 1) * 4), acc1[j]);
          }
        } else if (jp >= d && lane < SC_CS + P) {
          const int j = lane - SC_CS;
          float* o = Vown + (static_cast<int64_t>(jp - d) * rows + (row - r_begin)) * P;
          float v0 = 0.f, v1 = 0.f;
#pragma unroll
          for (int jj = 0; jj < P; ++jj) {
            if (jj == j) {
              v0 = acc0[jj];
              v1 = acc1[jj];
            }
          }
          o[j] = v0;
          if (two) o[P + j] = v1;
        }
      }
      cluster_sync();  // V_j complete in every CTA of the cluster
      float* t = Vc;
      Vc = Vn;
      Vn = t;
    }
    // fp64 Gram of the owned rows of V_d .. V_{2d+1}, reduced into the leader
    double part[10];
#pragma unroll
    for (int i = 0; i < 10; ++i) part[i] = 0.0;
    const int cnt = (r_end - r_begin) * P;
    for (int e = tid; e < cnt; e += SC_THREADS) {
      double x[4];
      for (int i = 0; i < nv; ++i) x[i] = static_cast<double>(Vown[static_cast<int64_t>(i) * rows * P + e]);
      int idx = 0;
      for (int i = 0; i < nv; ++i)
        for (int j = i; j < nv; ++j) part[idx++] += x[i] * x[j];
    }
#pragma unroll
    for (int i = 0; i < 10; ++i) {
      const double v = warp_sum(part[i]);
      if (lane == 0) gpart[warp][i] = v;
    }
    __syncthreads();
    if (tid < 10) {
      double v = 0.0;
      for (int w = 0; w < SC_WARPS; ++w) v += gpart[w][tid];
      st_cluster_f64(mapa_shared(smem_u32(&gclu[crank][tid]), 0), v);
    }
    cluster_sync();  // partials in the leader; V buffers free for the next block
    if (crank == 0 && tid == 0) {
      double M[4][4];
      int idx = 0;
      for (int i = 0; i < nv; ++i)
        for (int j = i; j < nv; ++j) {
          double v = 0.0;
          for (int q = 0; q < SC_CS; ++q) v += gclu[q][idx];
          M[i][j] = M[j][i] = v;
          ++idx;
        }
      double coef[5];
      quartic_from_gram(M, d, coef);
      const double a = argmin_quartic(coef, static_cast<double>(lo), static_cast<double>(hi));
      alpha[b] = static_cast<float>(a);
      if (rep != nullptr) rep[b * rep_stride + rep_slot + k] = static_cast<float>(a);
    }
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
  const int rows = p <= 16 ? 4 : 2;
  dim3 grid(static_cast<unsigned>((n + 8 * rows - 1) / (8 * rows)), batch);
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
                        const int* it, cudaStream_t st) {
  if (batch <= 0) return cudaSuccess;
  const int64_t vbs = static_cast<int64_t>(2 * d + 2) * n * p;
  k_alpha<<<batch, AL_THREADS, 0, st>>>(V, n, p, d, vbs, lo, hi, fixed_alpha, active, alpha,
                                        J_coef, report_alpha, report_stride, report_slot, it);
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

bool sketch_chain_ok(int64_t n, int p) {
  const int P = p <= 4 ? 4 : (p <= 8 ? 8 : 16);
  return p <= 16 && n >= 64 && n * P <= SC_VFLOATS;
}

namespace {
constexpr int kMaxDev = 64;
int g_chain_clusters[kMaxDev] = {0};  // resident clusters per device (0 = not queried)

template <int P>
void chain_config(cudaLaunchConfig_t* cfg, cudaLaunchAttribute* attr, cudaStream_t st) {
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = SC_CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg->blockDim = dim3(SC_THREADS, 1, 1);
  cfg->dynamicSmemBytes = SC_SMEM;
  cfg->stream = st;
  cfg->attrs = attr;
  cfg->numAttrs = 1;
}

template <int P>
cudaError_t prepare_chain(int dev) {
  auto kern = k_sketch_chain<P>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SC_SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  chain_config<P>(&cfg, attr, nullptr);
  cfg.gridDim = dim3(SC_CS * 148, 1, 1);
  int mc = 0;
  e = cudaOccupancyMaxActiveClusters(&mc, kern, &cfg);
  if (e != cudaSuccess) return e;
  // every p bucket has the same footprint: keep the smallest answer
  if (g_chain_clusters[dev] == 0 || mc < g_chain_clusters[dev]) g_chain_clusters[dev] = mc < 1 ? 1 : mc;
  return cudaSuccess;
}

template <int P>
cudaError_t launch_chain(const float* R, int n, int batch, const float* S, const int* it, int p,
                         int d, float lo, float hi, const int* active, float* alpha,
                         float* rep, int64_t rep_stride, int rep_slot, cudaStream_t st) {
  auto kern = k_sketch_chain<P>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  chain_config<P>(&cfg, attr, st);
  const int mc = dev < kMaxDev && g_chain_clusters[dev] > 0 ? g_chain_clusters[dev] : 1;
  cfg.gridDim = dim3(SC_CS * (batch < mc ? batch : mc), 1, 1);
  return cudaLaunchKernelEx(&cfg, kern, R, n, batch, S, it, p, d, lo, hi, active, alpha, rep,
                            rep_stride, rep_slot);
}
}  // namespace

cudaError_t sketch_chain_prepare() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev >= kMaxDev) return e;
  if (g_chain_clusters[dev] > 0) return cudaSuccess;
  e = prepare_chain<4>(dev);
  if (e == cudaSuccess) e = prepare_chain<8>(dev);
  if (e == cudaSuccess) e = prepare_chain<16>(dev);
  return e;
}

cudaError_t sketch_chain(const float* R, int64_t n, int batch, const float* S, const int* it,
                         int p, int d, float lo, float hi, const int* active, float* alpha,
                         float* rep, int64_t rep_stride, int rep_slot, cudaStream_t st) {
  if (batch <= 0) return cudaSuccess;
  const int N = static_cast<int>(n);
  if (p <= 4)
    return launch_chain<4>(R, N, batch, S, it, p, d, lo, hi, active, alpha, rep, rep_stride,
                           rep_slot, st);
  if (p <= 8)
    return launch_chain<8>(R, N, batch, S, it, p, d, lo, hi, active, alpha, rep, rep_stride,
                           rep_slot, st);
  return launch_chain<16>(R, N, batch, S, it, p, d, lo, hi, active, alpha, rep, rep_stride,
                          rep_slot, st);
}

uint64_t kernel_runs_sketch() {
  unsigned long long v = 0;
  if (cudaMemcpyFromSymbol(&v, g_kernel_runs, sizeof(v)) != cudaSuccess) return 0;
  return v;
}

}  // namespace shp
