// Bandwidth-bound helpers of the Newton-Schulz passes: Frobenius norms and
// normalisation ("no spectral bounds needed": B = A / ||A||_F puts the
// spectrum in (0, 1]), identity starts, the d = 1 update polynomial
// g = I + alpha R, TF32 hi/lo splitting, and the final scaling of the root.
// All are grid-stride loops over [batch][count] with coalesced accesses.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"
#include "shp_common.cuh"

namespace shp {

namespace {

constexpr int EW_THREADS = 256;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dim3 ew_grid(int64_t count, int batch) {
  int64_t per = (count + EW_THREADS * 8 - 1) / (EW_THREADS * 8);
  if (per < 1) per = 1;
  if (per > 1024) per = 1024;
  return dim3(static_cast<unsigned>(per), static_cast<unsigned>(batch));
}

SHP_DEV void put(int fmt, void* hi, float* lo, int64_t off, float v) {
  if (fmt == OUT_F32) {
    static_cast<float*>(hi)[off] = v;
  } else if (fmt == OUT_SPLIT) {
    const float h = tf32_round(v);
    static_cast<float*>(hi)[off] = h;
    lo[off] = tf32_round(v - h);  // pre-rounded: the tensor core truncates
  } else {
    static_cast<__nv_bfloat16*>(hi)[off] = __float2bfloat16_rn(v);
  }
}
SHP_DEV float get(int fmt, const void* hi, const float* lo, int64_t off) {
  if (fmt == OUT_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(hi)[off]);
  float v = static_cast<const float*>(hi)[off];
  if (fmt == OUT_SPLIT) v += lo[off];
  return v;
}

// Eight bf16 values of one 16-byte word, as fp32 (exact).
SHP_DEV void unpack8(const uint4 u, float* x) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
// Eight fp32 values rounded to bf16 (nearest even) in one 16-byte word.
SHP_DEV uint4 pack8(const float* x) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 t = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&t);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Block-wide sum of a float partial into an fp32 atomic.
SHP_DEV void block_add(float v, float* dst) {
  __shared__ float red[EW_THREADS / 32];
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int w = 0; w < EW_THREADS / 32; ++w) s += red[w];
    atomicAdd(dst, s);
  }
}

__global__ void k_reset(Ctl ctl, int batch, int first, int start_degree) {
  count_kernel_run();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= batch) return;
  if (start_degree > 0 && ctl.deg != nullptr) ctl.deg[b] = start_degree;
  BlockState& s = ctl.bs[b];
  if (first) {
    s.status = ST_OK;
    s.iters1 = 0;
    s.c = 0.f;
    ctl.dnorm[b] = 0.0;
    ctl.tmo[b] = 0;
  } else {
    s.iters1 = s.iters;
  }
  if (b == 0) *ctl.it = 0;
  s.norm2 = 0.f;
  s.prev_res = INFINITY;
  s.iters = 0;
  s.pass_status = ST_OK;
  ctl.active[b] = 1;
  ctl.alpha[b] = 0.f;
  if (ctl.gram != nullptr) {  // the fused alpha's accumulators
    for (int i = 0; i < 15; ++i) ctl.gram[b * 15 + i] = 0.0;
    ctl.gcnt[b] = 0;
  }
  if (b == 0 && ctl.gbar != nullptr) {  // the few-block sketch's grid barrier
    ctl.gbar[0] = 0u;
    ctl.gbar[2] = 0u;
  }
}

__global__ void __launch_bounds__(EW_THREADS)
    k_frob(const void* X, int bf16, int64_t count, double* dnorm, int vec) {
  count_kernel_run();
  const int b = blockIdx.y;
  double acc = 0.0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * EW_THREADS;
  const int64_t e0 = blockIdx.x * static_cast<int64_t>(EW_THREADS) + threadIdx.x;
  if (vec) {  // 16 bytes per load: 8 bf16 or 4 fp32 values (aligned, count a multiple)
    const uint4* p = reinterpret_cast<const uint4*>(
        static_cast<const uint8_t*>(X) + b * count * (bf16 ? 2 : 4));
    const int64_t nv = count / (bf16 ? 8 : 4);
    for (int64_t e = e0; e < nv; e += stride) {
      const uint4 u = p[e];
      if (bf16) {
        float x[8];
        unpack8(u, x);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc += static_cast<double>(x[i]) * x[i];
      } else {
        const float x[4] = {__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z),
                            __uint_as_float(u.w)};
#pragma unroll
        for (int i = 0; i < 4; ++i) acc += static_cast<double>(x[i]) * x[i];
      }
    }
  } else {
    for (int64_t e = e0; e < count; e += stride) {
      const float v = bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(X)[b * count + e])
                           : static_cast<const float*>(X)[b * count + e];
      acc += static_cast<double>(v) * v;
    }
  }
  __shared__ double red[EW_THREADS / 32];
  acc = warp_sum(acc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < EW_THREADS / 32; ++w) s += red[w];
    atomicAdd(&dnorm[b], s);
  }
}

// Start of pass 1 (c = ||A||_F from k_frob): Y_0 = B = (A + A^T) / (2c),
// R_0 = I - B.  Z_0 = I is not stored: the first step writes Z_1 = I + Delta
// directly and k_coupled_finish stands in I for a block that made no step.  The method is stated for a symmetric A and every
// later product is formed on its upper-triangle tiles, so the start takes the
// symmetric part, which is A / c bit for bit when A is symmetric.  A^T comes
// through a padded 32 x 32 shared-memory transpose: both reads are coalesced.
__global__ void __launch_bounds__(EW_THREADS)
    k_coupled_init(const float* A, int64_t n, Ctl ctl, int fmt, float* Yhi, float* Ylo,
                   float* Rhi, float* Rlo, float* Rs) {
  count_kernel_run();
  __shared__ float tt[32][33];
  const int b = blockIdx.y;
  const float c = static_cast<float>(sqrt(ctl.dnorm[b]));
  if (blockIdx.x == 0 && threadIdx.x == 0) ctl.bs[b].c = c;
  const int64_t nn = n * n, T = (n + 31) / 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const float* Ab = A + b * nn;
  float nrm = 0.f;
  for (int64_t t = blockIdx.x; t < T * T; t += gridDim.x) {
    const int64_t i0 = (t / T) * 32, j0 = (t % T) * 32;
    __syncthreads();  // the previous tile's reads of tt are done
    for (int r = ty; r < 32; r += EW_THREADS / 32) {  // tt[x][r] = A(j0 + r, i0 + x)
      const int64_t row = j0 + r, col = i0 + tx;
      tt[tx][r] = (row < n && col < n) ? Ab[row * n + col] : 0.f;
    }
    __syncthreads();
    for (int r = ty; r < 32; r += EW_THREADS / 32) {
      const int64_t row = i0 + r, col = j0 + tx;  // A^T(row, col) = tt[r][tx]
      if (row >= n || col >= n) continue;
      const int64_t off = b * nn + row * n + col;
      const bool diag = row == col;
      const float y = 0.5f * (Ab[row * n + col] + tt[r][tx]) / c;
      const float rr = (diag ? 1.f : 0.f) - y;
      put(fmt, Yhi, Ylo, off, y);
      put(fmt, Rhi, Rlo, off, rr);
      if (Rs != nullptr) Rs[off] = rr;
      nrm += rr * rr;
    }
  }
  block_add(nrm, &ctl.bs[b].norm2);
}

__global__ void __launch_bounds__(EW_THREADS)
    k_coupled_restart(int64_t n, Ctl ctl, int fmt, float* Y0hi, float* Y0lo, const float* Y1hi,
                      const float* Y1lo, float* Rhi, float* Rlo, float* Rs) {
  count_kernel_run();
  const int b = blockIdx.y;
  const bool from1 = (ctl.bs[b].iters1 & 1) != 0;
  const int64_t nn = n * n;
  float nrm = 0.f;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(EW_THREADS) + threadIdx.x; e < nn;
       e += static_cast<int64_t>(gridDim.x) * EW_THREADS) {
    const int64_t off = b * nn + e;
    const bool diag = (e / n) == (e % n);
    float y;
    if (from1) {
      y = get(fmt, Y1hi, Y1lo, off);
      // copy the exact stored pair, not a re-split of its sum
      Y0hi[off] = Y1hi[off];
      if (fmt == OUT_SPLIT) Y0lo[off] = Y1lo[off];
    } else {
      y = get(fmt, Y0hi, Y0lo, off);
    }
    const float r = (diag ? 1.f : 0.f) - y;
    put(fmt, Rhi, Rlo, off, r);
    if (Rs != nullptr) Rs[off] = r;
    nrm += r * r;
  }
  block_add(nrm, &ctl.bs[b].norm2);
}

__global__ void __launch_bounds__(EW_THREADS)
    k_gform_d1(const float* Rhi, const float* Rlo, int64_t n, Ctl ctl, const int* active,
               int fmt, void* ghi, float* glo, void* g2hi, float* g2lo) {
  count_kernel_run();
  const int b = blockIdx.y;
  if (active[b] == 0) return;
  const float a = ctl.alpha[b];
  const int64_t nn = n * n;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(EW_THREADS) + threadIdx.x; e < nn;
       e += static_cast<int64_t>(gridDim.x) * EW_THREADS) {
    const int64_t off = b * nn + e;
    float r = Rhi[off];
    if (Rlo != nullptr) r += Rlo[off];
    const float dlt = a * r;
    put(fmt, ghi, glo, off, dlt);
    if (g2hi != nullptr) put(fmt, g2hi, g2lo, off, (((e / n) == (e % n)) ? 1.f : 0.f) + dlt);
  }
}

__global__ void __launch_bounds__(EW_THREADS)
    k_coupled_finish(int64_t n, Ctl ctl, double e_c, const float* S0hi, const float* S0lo,
                     const float* S1hi, const float* S1lo, float* X, int z_slots) {
  count_kernel_run();
  const int b = blockIdx.y;
  const double c = static_cast<double>(ctl.bs[b].c);
  double sc;
  if (e_c == 0.5)
    sc = sqrt(c);
  else if (e_c == -0.5)
    sc = 1.0 / sqrt(c);
  else
    sc = 1.0 / sqrt(sqrt(c));  // e_c == -0.25
  const float scale = static_cast<float>(sc);
  const bool one = (ctl.bs[b].iters & 1) != 0;
  const float* hi = one ? S1hi : S0hi;
  const float* lo = one ? S1lo : S0lo;
  // Z_0 = I is never stored: a block whose last pass made no step gets I
  const bool identity = z_slots != 0 && ctl.bs[b].iters == 0;
  const int64_t nn = n * n;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(EW_THREADS) + threadIdx.x; e < nn;
       e += static_cast<int64_t>(gridDim.x) * EW_THREADS) {
    const int64_t off = b * nn + e;
    float v;
    if (identity) {
      v = (e / n) == (e % n) ? 1.f : 0.f;
    } else {
      v = hi[off];
      if (lo != nullptr) v += lo[off];
    }
    X[off] = scale * v;
  }
}

__global__ void __launch_bounds__(EW_THREADS)
    k_split(const float* X, int64_t count, float* hi, float* lo) {
  count_kernel_run();
  for (int64_t e = blockIdx.x * static_cast<int64_t>(EW_THREADS) + threadIdx.x; e < count;
       e += static_cast<int64_t>(gridDim.x) * EW_THREADS) {
    const float v = X[e];
    const float h = tf32_round(v);
    hi[e] = h;
    lo[e] = tf32_round(v - h);
  }
}

// The EMA recurrence of the Kronecker factors replayed element by element
// over precomputed products: L <- beta L + (1 - beta) P_t + eps [i == j] for
// t = 0 .. count-1, P: [count][batch][n][n] (both triangles), 4 columns per
// thread (n % 4 == 0).  The products of up to four steps are loaded before
// they are folded in, so the loads overlap.
__global__ void __launch_bounds__(EW_THREADS)
    k_ema_replay(float* L, const float* P, int64_t n, int count, int64_t pstride, float beta,
                 float eps) {
  count_kernel_run();
  const int b = blockIdx.y;
  const int64_t nn = n * n, n4 = nn / 4;
  float4* Lb = reinterpret_cast<float4*>(L + b * nn);
  const float4* Pb = reinterpret_cast<const float4*>(P + b * nn);
  const int64_t ps4 = pstride / 4;
  const float w = 1.f - beta;
  for (int64_t e4 = blockIdx.x * static_cast<int64_t>(EW_THREADS) + threadIdx.x; e4 < n4;
       e4 += static_cast<int64_t>(gridDim.x) * EW_THREADS) {
    const int64_t e = 4 * e4, row = e / n, col = e % n;
    const int dj = static_cast<int>(row - col);  // the diagonal sits at component dj, if in 0..3
    const float ex = dj == 0 ? eps : 0.f, ey = dj == 1 ? eps : 0.f;
    const float ez = dj == 2 ? eps : 0.f, ew = dj == 3 ? eps : 0.f;
    float4 l = Lb[e4];
    for (int t0 = 0; t0 < count; t0 += 4) {
      float4 q[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (t0 + u < count) q[u] = Pb[(t0 + u) * ps4 + e4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (t0 + u < count) {
          l.x = beta * l.x + w * q[u].x + ex;
          l.y = beta * l.y + w * q[u].y + ey;
          l.z = beta * l.z + w * q[u].z + ez;
          l.w = beta * l.w + w * q[u].w + ew;
        }
      }
    }
    Lb[e4] = l;
  }
}

__global__ void __launch_bounds__(EW_THREADS)
    k_polar_init(const void* G, int gbf16, int64_t count, Ctl ctl, int fmt, void* Xhi,
                 float* Xlo, int vec) {
  count_kernel_run();
  const int b = blockIdx.y;
  const float c = static_cast<float>(sqrt(ctl.dnorm[b]));
  if (blockIdx.x == 0 && threadIdx.x == 0) ctl.bs[b].c = c;
  // X_0 = G / ||G||_F as written: a zero block gives 0/0 and stops with
  // SHP_ENONFINITE at its first residual
  if (vec) {  // bf16 to bf16, 8 values per 16-byte load and store
    const uint4* g =
        reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(G) + b * count);
    uint4* x = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(Xhi) + b * count);
    for (int64_t e = blockIdx.x * static_cast<int64_t>(EW_THREADS) + threadIdx.x; e < count / 8;
         e += static_cast<int64_t>(gridDim.x) * EW_THREADS) {
      float v[8];
      unpack8(g[e], v);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = v[i] / c;
      x[e] = pack8(v);
    }
    return;
  }
  for (int64_t e = blockIdx.x * static_cast<int64_t>(EW_THREADS) + threadIdx.x; e < count;
       e += static_cast<int64_t>(gridDim.x) * EW_THREADS) {
    const int64_t off = b * count + e;
    const float v = gbf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(G)[off])
                          : static_cast<const float*>(G)[off];
    put(fmt, Xhi, Xlo, off, v / c);
  }
}

__global__ void __launch_bounds__(EW_THREADS)
    k_polar_finish(int64_t count, Ctl ctl, int fmt, const void* S0hi, const float* S0lo,
                   const void* S1hi, const float* S1lo, void* X, int out_bf16, int vec) {
  count_kernel_run();
  const int b = blockIdx.y;
  const bool one = (ctl.bs[b].iters & 1) != 0;
  const void* hi = one ? S1hi : S0hi;
  const float* lo = one ? S1lo : S0lo;
  if (vec) {  // bf16 to bf16: a 16-byte copy per thread and step
    const uint4* src =
        reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(hi) + b * count);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(X) + b * count);
    for (int64_t e = blockIdx.x * static_cast<int64_t>(EW_THREADS) + threadIdx.x; e < count / 8;
         e += static_cast<int64_t>(gridDim.x) * EW_THREADS)
      dst[e] = src[e];
    return;
  }
  for (int64_t e = blockIdx.x * static_cast<int64_t>(EW_THREADS) + threadIdx.x; e < count;
       e += static_cast<int64_t>(gridDim.x) * EW_THREADS) {
    const int64_t off = b * count + e;
    if (out_bf16 && fmt == OUT_BF16) {
      static_cast<__nv_bfloat16*>(X)[off] = static_cast<const __nv_bfloat16*>(hi)[off];
    } else {
      const float v = get(fmt, hi, lo, off);
      if (out_bf16)
        static_cast<__nv_bfloat16*>(X)[off] = __float2bfloat16_rn(v);
      else
        static_cast<float*>(X)[off] = v;
    }
  }
}

// acc[b] += ||G_b||_F^2 (from dn, fp64), eta[b] = lr / sqrt(1 + acc[b]).
__global__ void k_adaptive_eta(const double* dn, double* acc, float lr, float* eta, int batch) {
  count_kernel_run();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= batch) return;
  const double a = acc[b] + dn[b];
  acc[b] = a;
  eta[b] = static_cast<float>(static_cast<double>(lr) / sqrt(1.0 + a));
}

__global__ void k_write_status(Ctl ctl, int batch, int* out) {
  count_kernel_run();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= batch) return;
  out[b] = ctl.tmo[b] != 0 ? ST_ETIMEOUT : ctl.bs[b].status;
}

}  // namespace

cudaError_t reset_pass(const Ctl& ctl, int batch, int first_pass, cudaStream_t st,
                       int start_degree) {
  k_reset<<<(batch + 127) / 128, 128, 0, st>>>(ctl, batch, first_pass, start_degree);
  return cudaGetLastError();
}

cudaError_t frob_norm2(const void* X, int is_bf16, int64_t count, int batch, const Ctl& ctl,
                       cudaStream_t st) {
  const int vec = aligned16(X) && count % (is_bf16 ? 8 : 4) == 0;
  k_frob<<<ew_grid(count, batch), EW_THREADS, 0, st>>>(X, is_bf16, count, ctl.dnorm, vec);
  return cudaGetLastError();
}

cudaError_t coupled_init(const float* A, int64_t n, int batch, const Ctl& ctl, float* Yhi,
                         float* Ylo, float* Rhi, float* Rlo, float* Rs, cudaStream_t st) {
  const int fmt = Ylo != nullptr ? OUT_SPLIT : OUT_F32;
  k_coupled_init<<<ew_grid(n * n, batch), EW_THREADS, 0, st>>>(A, n, ctl, fmt, Yhi, Ylo, Rhi,
                                                               Rlo, Rs);
  return cudaGetLastError();
}

cudaError_t coupled_restart(int64_t n, int batch, const Ctl& ctl, float* const* Yhi,
                            float* const* Ylo, float* Rhi, float* Rlo, float* Rs,
                            cudaStream_t st) {
  const int fmt = Ylo[0] != nullptr ? OUT_SPLIT : OUT_F32;
  k_coupled_restart<<<ew_grid(n * n, batch), EW_THREADS, 0, st>>>(
      n, ctl, fmt, Yhi[0], Ylo[0], Yhi[1], Ylo[1], Rhi, Rlo, Rs);
  return cudaGetLastError();
}

cudaError_t gform_d1(const float* Rhi, const float* Rlo, int64_t n, int batch, const Ctl& ctl,
                     int fmt, void* ghi, float* glo, void* g2hi, float* g2lo, cudaStream_t st,
                     const int* active) {
  k_gform_d1<<<ew_grid(n * n, batch), EW_THREADS, 0, st>>>(
      Rhi, Rlo, n, ctl, active != nullptr ? active : ctl.active, fmt, ghi, glo, g2hi, g2lo);
  return cudaGetLastError();
}

cudaError_t coupled_finish(int64_t n, int batch, const Ctl& ctl, double c_exponent,
                           const float* const* Shi, const float* const* Slo, float* X_out,
                           bool z_slots, cudaStream_t st) {
  k_coupled_finish<<<ew_grid(n * n, batch), EW_THREADS, 0, st>>>(
      n, ctl, c_exponent, Shi[0], Slo[0], Shi[1], Slo[1], X_out, z_slots ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t split_copy(const float* X, int64_t count, float* hi, float* lo, cudaStream_t st) {
  if (count <= 0) return cudaSuccess;
  k_split<<<ew_grid(count, 1), EW_THREADS, 0, st>>>(X, count, hi, lo);
  return cudaGetLastError();
}

cudaError_t ema_replay(float* L, const float* P, int64_t n, int count, int batch, float beta,
                       float eps, cudaStream_t st) {
  if (count <= 0 || batch <= 0) return cudaSuccess;
  const int64_t n4 = n * n / 4;  // one float4 per thread
  const dim3 grid(static_cast<unsigned>((n4 + EW_THREADS - 1) / EW_THREADS), batch);
  k_ema_replay<<<grid, EW_THREADS, 0, st>>>(
      L, P, n, count, static_cast<int64_t>(batch) * n * n, beta, eps);
  return cudaGetLastError();
}

cudaError_t polar_init(const void* G, int g_bf16, int64_t count, int batch, const Ctl& ctl,
                       int fmt, void* Xhi, float* Xlo, cudaStream_t st) {
  const int vec = g_bf16 && fmt == OUT_BF16 && aligned16(G) && aligned16(Xhi) && count % 8 == 0;
  k_polar_init<<<ew_grid(count, batch), EW_THREADS, 0, st>>>(G, g_bf16, count, ctl, fmt, Xhi,
                                                             Xlo, vec);
  return cudaGetLastError();
}

cudaError_t polar_finish(int64_t count, int batch, const Ctl& ctl, int fmt,
                         const void* const* Shi, const float* const* Slo, void* X_out,
                         int out_bf16, cudaStream_t st) {
  const int vec = out_bf16 && fmt == OUT_BF16 && aligned16(Shi[0]) && aligned16(Shi[1]) &&
                  aligned16(X_out) && count % 8 == 0;
  k_polar_finish<<<ew_grid(count, batch), EW_THREADS, 0, st>>>(
      count, ctl, fmt, Shi[0], Slo[0], Shi[1], Slo[1], X_out, out_bf16, vec);
  return cudaGetLastError();
}

cudaError_t adaptive_step(const float* G, int64_t count, int batch, double* dn, double* acc,
                          float lr, float* eta, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(dn, 0, sizeof(double) * batch, st);
  if (e != cudaSuccess) return e;
  k_frob<<<ew_grid(count, batch), EW_THREADS, 0, st>>>(G, 0, count, dn,
                                                       aligned16(G) && count % 4 == 0);
  k_adaptive_eta<<<(batch + 127) / 128, 128, 0, st>>>(dn, acc, lr, eta, batch);
  return cudaGetLastError();
}

cudaError_t write_status(const Ctl& ctl, int batch, int* report_status, cudaStream_t st) {
  if (report_status == nullptr) return cudaSuccess;
  k_write_status<<<(batch + 127) / 128, 128, 0, st>>>(ctl, batch, report_status);
  return cudaGetLastError();
}

uint64_t kernel_runs_elementwise() {
  unsigned long long v = 0;
  if (cudaMemcpyFromSymbol(&v, g_kernel_runs, sizeof(v)) != cudaSuccess) return 0;
  return v;
}

}  // namespace shp
