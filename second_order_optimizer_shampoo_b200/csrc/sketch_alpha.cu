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
#include <stdlib.h>

#include <string.h>

#include "internal.h"
#include "prism_scalar.cuh"
#include "shp_common.cuh"

namespace shp {

namespace {

constexpr int SK_THREADS = 256;
constexpr int SK_GROUPS = 2;  // row groups per warp in one CTA

// Warp reduction of ROWS x P row sums (acc[r * P + j], one partial per lane)
// by recursive halving: at the step with offset o each lane keeps the half of
// its values selected by its lane bit o and adds the partner's copy of that
// half, so 31 shuffles (for 32 values) leave lane l holding the total of
// value l, where a shuffle tree per value would take 5 per value.  Stores
// row0 + r, column j of Vb (rows >= n and columns >= p are not stored).
template <int ROWS, int P>
SHP_DEV void store_row_sums(float (&acc)[ROWS * P], int lane, int64_t row0, int64_t n, int p,
                            float* Vb) {
  constexpr int NV = ROWS * P;
  static_assert(NV == 16 || NV == 32 || NV == 64, "16, 32 or 64 sums per warp");
  constexpr int STEPS = NV >= 32 ? 5 : 4;
#pragma unroll
  for (int st = 0; st < STEPS; ++st) {
    const int o = 16 >> st;
    const int h = (NV >> st) / 2;
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = up ? acc[i] : acc[i + h];
      const float keep = up ? acc[i + h] : acc[i];
      acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  if constexpr (NV == 16) {  // lanes l and l ^ 1 hold halves of value l >> 1
    acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 1);
    if ((lane & 1) == 0) {
      const int idx = lane >> 1, r = idx / P, j = idx % P;
      if (row0 + r < n && j < p) Vb[(row0 + r) * p + j] = acc[0];
    }
  } else {
#pragma unroll
    for (int k = 0; k < NV / 32; ++k) {  // this lane holds values lane * NV/32 + k
      const int idx = lane * (NV / 32) + k, r = idx / P, j = idx % P;
      if (row0 + r < n && j < p) Vb[(row0 + r) * p + j] = acc[k];
    }
  }
}

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
    float acc[ROWS * P];
#pragma unroll
    for (int i = 0; i < ROWS * P; ++i) acc[i] = 0.f;

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
            float a = acc[r * P + j];
            a = fmaf(x0[r].x, v0.x, a);
            a = fmaf(x0[r].y, v0.y, a);
            a = fmaf(x0[r].z, v0.z, a);
            a = fmaf(x0[r].w, v0.w, a);
            a = fmaf(x1[r].x, v1.x, a);
            a = fmaf(x1[r].y, v1.y, a);
            a = fmaf(x1[r].z, v1.z, a);
            acc[r * P + j] = fmaf(x1[r].w, v1.w, a);
          }
        }
      }
    }
    store_row_sums<ROWS, P>(acc, lane, row0, n, p, Vout + b * obs);
  }
}

// The same product with R streamed through shared memory by TMA, for blocks
// whose V fits in shared memory whole: a persistent grid, one CTA per SM,
// each CTA a contiguous range of work items (RPI = 8 * ROWS rows of one
// block).  Warp 8 (one lane) issues one tiled load per stage (SC = 256
// columns x RPI rows, zero filled past the edges) into an NST-deep ring, so
// up to NST * 32 KB of R is in flight per SM whatever the register file
// holds; warps 0..7 each reduce ROWS rows of a stage against Vs exactly as
// k_sketch does from registers.  Every wait, the V hand-over between items
// of different blocks included, is an mbarrier wait with a bound; one that
// runs out marks the block's timeout flag and the CTA unwinds after its
// copies have landed.
constexpr int ST_SC = 256;  // columns per stage
constexpr int ST_NST = 4;   // ring depth
constexpr int ST_CONS = 8;  // consumer warps

template <int P>
struct SkTma {
  static constexpr int ROWS = P <= 8 ? 4 : 2;
  static constexpr int RPI = ST_CONS * ROWS;        // rows per work item
  static constexpr int STAGE_FLOATS = RPI * ST_SC;  // 32 KB (P <= 8) or 16 KB
  static size_t smem_bytes(int64_t n) {
    const int64_t ldv = (n + ST_SC - 1) / ST_SC * ST_SC + 4;
    return 128 + static_cast<size_t>(ST_NST) * STAGE_FLOATS * 4 + static_cast<size_t>(P) * ldv * 4 +
           (2 * ST_NST + 3) * 8 + 16;
  }
};

// A wait that ran out: flag the block and leave (every other waiter then
// runs out too, or sees the flag first).
constexpr int AL_THREADS = 512;

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
  const int* tmo;  // blocks whose sketch timed out: alpha = NaN
};


// alpha of block b from the Gram G[i][j] = <V_{first+i}, V_{first+j}> of its
// sketch moments (first = d, or 1 with adaptive degree): the quartic J and its
// minimiser on [lo, hi] by the calling warp (every lane takes part in the
// bracketing), the degree rule, and lane 0 writes alpha, J's coefficients and
// the report.  Shared by k_alpha and the fused last sketch pass.
SHP_DEV void alpha_solve_warp(const AlphaArgs& g, int b, const double (&G)[5][5]) {
  const int lane = threadIdx.x & 31;
  const int rep_slot = g.rep_slot + (g.it != nullptr ? *g.it : 0);
  const int first = g.adaptive ? 1 : g.d;  // V_first .. V_{first + nv - 1}
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
  if (lane != 0) return;
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

// Fused alpha of the last sketch pass: a consumer warp's partial Gram of the
// moments over the rows it produced, kept across the items of one block.
struct GramPart {
  double part[15];
  int b, items;
};

SHP_DEV void gram_reset(GramPart& gp) {
#pragma unroll
  for (int i = 0; i < 15; ++i) gp.part[i] = 0.0;
  gp.items = 0;
}

// Adds this warp's rows row0 .. row0 + rows - 1 of V_first .. V_{2d+1} (nv
// vectors of block b, fp32, n x p each) to the partial Gram.
SHP_DEV void gram_add(GramPart& gp, const AlphaArgs& g, int b, int64_t row0, int rows) {
  const int lane = threadIdx.x & 31, nv = g.d + 2;
  const int64_t len = g.n * g.p;
  const float* Vb = g.V + b * g.vbs + static_cast<int64_t>(g.d) * len;
  for (int e = lane; e < rows * g.p; e += 32) {
    const int64_t row = row0 + e / g.p;
    if (row >= g.n) continue;
    const int64_t off = row * g.p + e % g.p;
    double x[5];
#pragma unroll
    for (int i = 0; i < 5; ++i) x[i] = i < nv ? static_cast<double>(Vb[i * len + off]) : 0.0;
    int idx = 0;
#pragma unroll
    for (int i = 0; i < 5; ++i)
#pragma unroll
      for (int j = i; j < 5; ++j, ++idx) gp.part[idx] = fma(x[i], x[j], gp.part[idx]);
  }
  ++gp.items;
}

// Adds the warp's partial Gram of block gp.b into gram[b] and its item count
// into gcnt[b]; the warp whose count completes the block (every item of the
// pass seen by each consumer warp: total items x ST_CONS) solves alpha for it
// and clears the block's accumulators for the next iteration.  A block whose
// sketch timed out gets alpha = NaN.
SHP_DEV void gram_flush(GramPart& gp, const AlphaArgs& g, double* gram, int* gcnt, int total,
                        const int* tmo) {
  const int lane = threadIdx.x & 31;
  if (gp.b < 0 || gp.items == 0) return;
  const int b = gp.b;
#pragma unroll
  for (int i = 0; i < 15; ++i) gp.part[i] = warp_sum(gp.part[i]);
  int last = 0;
  if (lane == 0) {
    for (int i = 0; i < 15; ++i) atomicAdd(&gram[b * 15 + i], gp.part[i]);
    __threadfence();
    last = atomicAdd(&gcnt[b], gp.items) + gp.items == total;
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (last) {
    __threadfence();
    double G[5][5];
    int idx = 0;
    for (int i = 0; i < 5; ++i)
      for (int j = i; j < 5; ++j, ++idx) G[i][j] = G[j][i] = __ldcg(&gram[b * 15 + idx]);
    if (tmo != nullptr && tmo[b] != 0) {
      if (lane == 0) g.alpha[b] = __int_as_float(0x7fc00000);
    } else {
      alpha_solve_warp(g, b, G);
    }
    if (lane == 0) {
      for (int i = 0; i < 15; ++i) gram[b * 15 + i] = 0.0;
      gcnt[b] = 0;
    }
  }
  gram_reset(gp);
}

SHP_DEV void sketch_give_up(volatile int* abort_flag, int* tmo, int b, int lane) {
  *abort_flag = 1;
  __threadfence_block();
  if (lane == 0 && tmo != nullptr) atomicExch(&tmo[b], ST_ETIMEOUT);
}

template <int P>
__global__ void __launch_bounds__(32 * (ST_CONS + 1), 1)
    k_sketch_tma(const __grid_constant__ CUtensorMap tR, int64_t n,
                 const float* __restrict__ Vin, int64_t vbs, float* __restrict__ Vout,
                 int64_t obs, int p, int batch, const int* __restrict__ active,
                 const int* __restrict__ it, int64_t it_stride, int* tmo, int selftest,
                 AlphaArgs fa, double* gram, int* gcnt) {
  count_kernel_run();
  using K = SkTma<P>;
  constexpr int ROWS = K::ROWS, RPI = K::RPI;
  constexpr int NCT = 32 * ST_CONS;  // consumer threads
  extern __shared__ __align__(16) uint8_t sk_smem[];
  float* ring = reinterpret_cast<float*>(
      (reinterpret_cast<uintptr_t>(sk_smem) + 127) & ~static_cast<uintptr_t>(127));
  const int64_t ldv = (n + ST_SC - 1) / ST_SC * ST_SC + 4;
  float* Vs = ring + ST_NST * K::STAGE_FLOATS;
  uint64_t* full = reinterpret_cast<uint64_t*>(Vs + P * ldv);
  uint64_t* empty = full + ST_NST;
  uint64_t* vbar = empty + ST_NST;  // [2] old V released, new V staged
  uint64_t* never = vbar + 2;       // completed by nothing: the self-test's wait
  volatile int* abort_flag = reinterpret_cast<volatile int*>(never + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gpb = (n + RPI - 1) / RPI;  // items per block
  const int64_t items = gpb * batch;
  const int64_t i0 = items * blockIdx.x / gridDim.x, i1 = items * (blockIdx.x + 1) / gridDim.x;
  const int nch = static_cast<int>((n + ST_SC - 1) / ST_SC);
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tR);
    for (int s = 0; s < ST_NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], ST_CONS);
    }
    mbar_init(&vbar[0], ST_CONS);
    mbar_init(&vbar[1], ST_CONS);
    mbar_init(never, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == ST_CONS) {
    // ---------------- producer: one lane issues every copy
    if (lane == 0) {
      int kit = 0;
      int last_b = -1, seen_b = -1;
      bool seen_on = true;
      for (int64_t t = i0; t < i1 && !*abort_flag; ++t) {
        const int b = static_cast<int>(t / gpb);
        if (b != seen_b) {  // one global read per block, not per item
          seen_b = b;
          seen_on = active == nullptr || active[b] != 0;
        }
        if (!seen_on) continue;
        const int r0 = static_cast<int>((t % gpb) * RPI);
        last_b = b;
        for (int c = 0; c < nch; ++c, ++kit) {
          const int s = kit % ST_NST;
          if (kit >= ST_NST && !mbar_wait(&empty[s], ((kit / ST_NST) - 1) & 1, abort_flag)) {
            sketch_give_up(abort_flag, tmo, b, 0);
            break;
          }
          // the full box lands (zeros past the edges); x = c * 256 is aligned
          mbar_arrive_expect_tx(&full[s], K::STAGE_FLOATS * 4u);
          tma_load_3d(ring + s * K::STAGE_FLOATS, &tR, &full[s], c * ST_SC, r0, b);
        }
      }
      // every copy issued has landed before the CTA may exit
      const int first = kit > ST_NST ? kit - ST_NST : 0;
      for (int k = first; k < kit; ++k)
        if (!mbar_wait(&full[k % ST_NST], (k / ST_NST) & 1) && last_b >= 0)
          sketch_give_up(abort_flag, tmo, last_b, 0);
    }
    return;
  }

  // ---------------- consumers: warps 0..7
  int kit = 0, ns = 0;  // stages consumed, V stagings
  int cur_b = -1, seen_b = -1;
  bool seen_on = true;
  GramPart gp;  // fused alpha (gram != nullptr): this warp's partial Gram
  gram_reset(gp);
  gp.b = -1;
  bool aborted = false;
  for (int64_t t = i0; t < i1; ++t) {
    if (*abort_flag) break;
    const int b = static_cast<int>(t / gpb);
    if (b != seen_b) {  // one global read per block, not per item
      seen_b = b;
      seen_on = active == nullptr || active[b] != 0;
    }
    if (!seen_on) continue;
    if (b != cur_b) {  // stage V of block b (all consumer warps; the producer runs on)
      // bounded-wait self-test: the first V hand-over waits on a barrier
      // nothing completes, with the producer's copies already in flight
      if (selftest && !mbar_wait(never, 0, nullptr, SHP_SELFTEST_LIMIT)) {
        sketch_give_up(abort_flag, tmo, b, lane);
        aborted = true;
        break;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&vbar[0]);  // this warp is done with the old V
      if (!mbar_wait(&vbar[0], ns & 1)) {
        sketch_give_up(abort_flag, tmo, b, lane);
        break;
      }
      const float* V = Vin + b * vbs + (it != nullptr ? static_cast<int64_t>(*it) * it_stride : 0);
      for (int64_t idx = threadIdx.x; idx < ldv * (P / 4); idx += NCT) {
        const int64_t col = idx / (P / 4);
        const int q = 4 * static_cast<int>(idx % (P / 4));
        const float* src = V + col * p + q;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          Vs[(q + e) * ldv + col] = (col < n && q + e < p) ? __ldg(src + e) : 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&vbar[1]);  // this warp's part of V is written
      if (!mbar_wait(&vbar[1], ns & 1)) {
        sketch_give_up(abort_flag, tmo, b, lane);
        break;
      }
      ++ns;
      cur_b = b;
    }
    const int64_t r0 = (t % gpb) * RPI;
    float acc[ROWS * P];
#pragma unroll
    for (int i = 0; i < ROWS * P; ++i) acc[i] = 0.f;
    bool ok = true;
    for (int c = 0; c < nch; ++c, ++kit) {
      const int s = kit % ST_NST;
      if (*abort_flag || !mbar_wait(&full[s], (kit / ST_NST) & 1)) {
        sketch_give_up(abort_flag, tmo, b, lane);
        ok = false;
        break;
      }
      const float* st = ring + s * K::STAGE_FLOATS + (warp * ROWS) * ST_SC + lane * 4;
      float4 x0[ROWS], x1[ROWS];
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        x0[r] = *reinterpret_cast<const float4*>(st + r * ST_SC);
        x1[r] = *reinterpret_cast<const float4*>(st + r * ST_SC + 128);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);  // this warp's reads of the stage are done
      // past the last column: R is zero filled and Vs zero padded
      const float* vp = Vs + static_cast<int64_t>(c) * ST_SC + lane * 4;
#pragma unroll
      for (int j = 0; j < P; ++j) {
        const float4 v0 = *reinterpret_cast<const float4*>(vp + j * ldv);
        const float4 v1 = *reinterpret_cast<const float4*>(vp + j * ldv + 128);
        // the ROWS chains advance together: consecutive FMAs are independent
#pragma unroll
        for (int r = 0; r < ROWS; ++r) acc[r * P + j] = fmaf(x0[r].x, v0.x, acc[r * P + j]);
#pragma unroll
        for (int r = 0; r < ROWS; ++r) acc[r * P + j] = fmaf(x0[r].y, v0.y, acc[r * P + j]);
#pragma unroll
        for (int r = 0; r < ROWS; ++r) acc[r * P + j] = fmaf(x0[r].z, v0.z, acc[r * P + j]);
#pragma unroll
        for (int r = 0; r < ROWS; ++r) acc[r * P + j] = fmaf(x0[r].w, v0.w, acc[r * P + j]);
#pragma unroll
        for (int r = 0; r < ROWS; ++r) acc[r * P + j] = fmaf(x1[r].x, v1.x, acc[r * P + j]);
#pragma unroll
        for (int r = 0; r < ROWS; ++r) acc[r * P + j] = fmaf(x1[r].y, v1.y, acc[r * P + j]);
#pragma unroll
        for (int r = 0; r < ROWS; ++r) acc[r * P + j] = fmaf(x1[r].z, v1.z, acc[r * P + j]);
#pragma unroll
        for (int r = 0; r < ROWS; ++r) acc[r * P + j] = fmaf(x1[r].w, v1.w, acc[r * P + j]);
      }
    }
    if (!ok) {
      aborted = true;
      break;
    }
    store_row_sums<ROWS, P>(acc, lane, r0 + warp * ROWS, n, p, Vout + b * obs);
    if (gram != nullptr) {
      if (b != gp.b) {
        gram_flush(gp, fa, gram, gcnt, static_cast<int>(gpb) * ST_CONS, tmo);
        gp.b = b;
      }
      __syncwarp();  // the rows this warp just stored are visible to all its lanes
      gram_add(gp, fa, b, r0 + warp * ROWS, ROWS);
    }
  }
  // a pass that gave up leaves its blocks' counts short: no alpha is solved
  // for them (it stays NaN from the stop test)
  if (gram != nullptr && !aborted && !*abort_flag)
    gram_flush(gp, fa, gram, gcnt, static_cast<int>(gpb) * ST_CONS, tmo);
}

// This thread's partial sums of <V_i, V_j> (i <= j < NV, packed row by row)
// over elements threadIdx.x + k * AL_THREADS; NV is a compile-time constant so
// that the 15 partials and the loaded values stay in registers.  Four
// elements are loaded per step (4 NV loads in flight): the sums are short
// (n p elements per block) and their cost is the load latency, not the fp64
// arithmetic.
template <int NV>
SHP_DEV void gram_partials(const float* __restrict__ Vb, int64_t len, double (&part)[15]) {
#pragma unroll
  for (int i = 0; i < 15; ++i) part[i] = 0.0;
  constexpr int U = 4;
  int64_t e = threadIdx.x;
  for (; e + (U - 1) * AL_THREADS < len; e += U * AL_THREADS) {
    float x[U][NV];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int i = 0; i < NV; ++i) x[u][i] = __ldg(Vb + i * len + e + u * AL_THREADS);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      int idx = 0;
#pragma unroll
      for (int i = 0; i < NV; ++i)
#pragma unroll
        for (int j = i; j < NV; ++j, ++idx)
          part[idx] = fma(static_cast<double>(x[u][i]), static_cast<double>(x[u][j]), part[idx]);
    }
  }
  for (; e < len; e += AL_THREADS) {
    float x[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) x[i] = __ldg(Vb + i * len + e);
    int idx = 0;
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
      for (int j = i; j < NV; ++j, ++idx)
        part[idx] = fma(static_cast<double>(x[i]), static_cast<double>(x[j]), part[idx]);
  }
}

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
  if (g.tmo != nullptr && g.tmo[b] != 0) {  // V is incomplete: no fit
    if (threadIdx.x == 0) {
      g.alpha[b] = __int_as_float(0x7fc00000);
      if (g.Jc != nullptr)
        for (int i = 0; i < 5; ++i) g.Jc[b * 5 + i] = __longlong_as_double(0x7ff8000000000000ll);
    }
    return;
  }
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
  if (nv == 3)
    gram_partials<3>(Vb, len, part);
  else if (nv == 4)
    gram_partials<4>(Vb, len, part);
  else
    gram_partials<5>(Vb, len, part);
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
  alpha_solve_warp(g, b, G);
}

__global__ void k_control(BlockState* bs, int* active, const int* it, int batch, int64_t n,
                          int max_iter, float tol, float stall_below, float stall_ratio,
                          float* rep_res, int64_t res_stride, int res_slot, int* rep_iters,
                          int iters_slot, float* alpha) {
  count_kernel_run();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= batch || active[b] == 0) return;
  // this iteration's alpha is written by the fit; a fit that never completes
  // (a sketch wait that gave up) leaves NaN, which stops the block
  if (alpha != nullptr) alpha[b] = __int_as_float(0x7fc00000);
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

namespace {

template <int P>
bool launch_sketch_tma(const float* R, int64_t n, int64_t rbs, const float* Vin, int64_t vbs,
                       float* Vout, int64_t obs, int p, int batch, const int* active,
                       const int* it, int64_t it_stride, int* tmo, int selftest, cudaStream_t st,
                       cudaError_t* err, const AlphaArgs* fa = nullptr, double* gram = nullptr,
                       int* gcnt = nullptr) {
  const size_t smem = SkTma<P>::smem_bytes(n);
  if (smem > 200 * 1024) return false;  // V does not fit whole: the register kernel
  CUtensorMap tR;
  if (!tensor_map_rows(&tR, R, n, n, batch, n, rbs, ST_SC, SkTma<P>::RPI)) return false;
  auto kern = k_sketch_tma<P>;
  // the attribute allows the largest size used (set once per device and P;
  // calls from several host threads at once may each set it, which is safe)
  static int set_for_dev[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = -1;
  if (dev < 0 || set_for_dev[dev] == 0) {
    *err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (*err != cudaSuccess) return true;
    if (dev >= 0) set_for_dev[dev] = 1;
  }
  int sms = 148;
  if (dev >= 0) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t items = (n + SkTma<P>::RPI - 1) / SkTma<P>::RPI * batch;
  const int grid = static_cast<int>(items < sms ? items : sms);
  AlphaArgs none;
  memset(&none, 0, sizeof(none));
  kern<<<grid, 32 * (ST_CONS + 1), smem, st>>>(tR, n, Vin, vbs, Vout, obs, p, batch, active, it,
                                                it_stride, tmo, selftest, fa ? *fa : none,
                                                fa ? gram : nullptr, fa ? gcnt : nullptr);
  *err = cudaGetLastError();
  return true;
}

}  // namespace

cudaError_t sketch_pass(const float* Rhi, const float* Rlo, int64_t n, int64_t r_bstride,
                        const float* Vin, int64_t vin_bstride, float* Vout, int64_t vout_bstride,
                        int p, int batch, const int* active, const int* it, int64_t it_stride,
                        cudaStream_t st, int* tmo, int selftest) {
  if (batch <= 0 || n <= 0) return cudaSuccess;
  // plain fp32 R with 16-byte aligned rows: the bulk-copy kernel when V fits
  if (Rlo == nullptr && (reinterpret_cast<uintptr_t>(Rhi) & 15) == 0 && n % 4 == 0 &&
      r_bstride % 4 == 0) {
    cudaError_t e = cudaSuccess;
    bool done = false;
    if (p <= 4)
      done = launch_sketch_tma<4>(Rhi, n, r_bstride, Vin, vin_bstride, Vout, vout_bstride, p,
                                  batch, active, it, it_stride, tmo, selftest, st, &e);
    else if (p <= 8)
      done = launch_sketch_tma<8>(Rhi, n, r_bstride, Vin, vin_bstride, Vout, vout_bstride, p,
                                  batch, active, it, it_stride, tmo, selftest, st, &e);
    else if (p <= 16)
      done = launch_sketch_tma<16>(Rhi, n, r_bstride, Vin, vin_bstride, Vout, vout_bstride, p,
                                   batch, active, it, it_stride, tmo, selftest, st, &e);
    if (done) return e;
  }
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

cudaError_t sketch_pass_alpha(const float* R, int64_t n, int64_t r_bstride, const float* Vin,
                              int64_t vin_bstride, float* Vout, int64_t vout_bstride, int p,
                              int batch, const int* active, cudaStream_t st, int* tmo,
                              const float* V, int d, float lo, float hi, float* alpha,
                              float* report_alpha, int64_t report_stride, int report_slot,
                              const int* it, double* gram, int* gcnt, bool* fused,
                              int selftest) {
  *fused = false;
  if (batch <= 0 || n <= 0) return cudaSuccess;
  if (gram != nullptr && gcnt != nullptr && (reinterpret_cast<uintptr_t>(R) & 15) == 0 &&
      n % 4 == 0 && r_bstride % 4 == 0) {
    AlphaArgs g;
    memset(&g, 0, sizeof(g));
    g.tmo = tmo;
    g.V = V;
    g.n = n;
    g.vbs = static_cast<int64_t>(2 * d + 2) * n * p;
    g.p = p;
    g.d = d;
    g.lo = lo;
    g.hi = hi;
    g.active = active;
    g.alpha = alpha;
    g.rep = report_alpha;
    g.rep_stride = report_stride;
    g.rep_slot = report_slot;
    g.it = it;
    cudaError_t e = cudaSuccess;
    bool done = false;
    if (p <= 4)
      done = launch_sketch_tma<4>(R, n, r_bstride, Vin, vin_bstride, Vout, vout_bstride, p, batch,
                                  active, nullptr, 0, tmo, selftest, st, &e, &g, gram, gcnt);
    else if (p <= 8)
      done = launch_sketch_tma<8>(R, n, r_bstride, Vin, vin_bstride, Vout, vout_bstride, p, batch,
                                  active, nullptr, 0, tmo, selftest, st, &e, &g, gram, gcnt);
    else if (p <= 16)
      done = launch_sketch_tma<16>(R, n, r_bstride, Vin, vin_bstride, Vout, vout_bstride, p,
                                   batch, active, nullptr, 0, tmo, selftest, st, &e, &g, gram,
                                   gcnt);
    if (done) {
      *fused = e == cudaSuccess;
      return e;
    }
  }
  return sketch_pass(R, nullptr, n, r_bstride, Vin, vin_bstride, Vout, vout_bstride, p, batch,
                     active, nullptr, 0, st, tmo);
}

cudaError_t alpha_solve(const float* V, int64_t n, int p, int d, int batch, float lo, float hi,
                        int fixed_alpha, const int* active, float* alpha, double* J_coef,
                        float* report_alpha, int64_t report_stride, int report_slot,
                        const int* it, cudaStream_t st, const AdaptiveDeg* ad,
                        const int* tmo) {
  if (batch <= 0) return cudaSuccess;
  AlphaArgs g;
  g.tmo = tmo;
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
                                                 res_stride, res_slot, report_iters, iters_slot,
                                                 ctl.alpha);
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
