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

// Warp reduction of NV per-lane partials by recursive halving: at the step
// with offset o each lane keeps the half of its values selected by its lane
// bit o and adds the partner's copy of that half, so 31 shuffles (for 32
// values) leave lane l holding the total of value l, where a shuffle tree per
// value would take 5 per value.  After 5 steps (NV >= 32) lane l holds the
// totals of values l * (NV / 32) + k in acc[k], k < NV / 32.
template <int NV, int STEPS>
SHP_DEV void halve_lanes(float (&acc)[NV], int lane) {
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
}

// Warp reduction of ROWS x P row sums (acc[r * P + j], one partial per lane);
// stores row0 + r, column j of Vb (rows >= n and columns >= p are not stored).
template <int ROWS, int P>
SHP_DEV void store_row_sums(float (&acc)[ROWS * P], int lane, int64_t row0, int64_t n, int p,
                            float* Vb) {
  constexpr int NV = ROWS * P;
  static_assert(NV == 16 || NV == 32 || NV == 64, "16, 32 or 64 sums per warp");
  halve_lanes<NV, NV >= 32 ? 5 : 4>(acc, lane);
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


// G[i][j] (i, j < NV) from W rows of packed upper-triangle partial sums
// red[w][idx] (idx running over i <= j row by row); unrolled, so G stays in
// registers.
template <int NV, int W>
SHP_DEV void gram_unpack(const double (*red)[15], double (&G)[5][5]) {
  int idx = 0;
#pragma unroll
  for (int i = 0; i < NV; ++i)
#pragma unroll
    for (int j = i; j < NV; ++j, ++idx) {
      double s = 0.0;
#pragma unroll
      for (int w = 0; w < W; ++w) s += red[w][idx];
      G[i][j] = G[j][i] = s;
    }
}

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
    const bool shift = e != first;  // first = 1 and e = 2: the block from V_2
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) M[i][j] = shift ? G[i + 1][j + 1] : G[i][j];
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
#pragma unroll
    for (int i = 0; i < 5; ++i)
#pragma unroll
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

// ---------------------------------------------------------------------------
// Few blocks: every pass of one iteration in one cooperative launch.
// With a handful of blocks a pass of the kernels above is a few microseconds
// of work behind a launch and a pipeline ramp, five times per iteration.
// Here the SMs are shared out evenly among the blocks (cpb CTAs per block),
// and each CTA keeps a contiguous range of rpc rows of one block's R in
// shared memory for the whole iteration; a pass stages V_{j-1} of the block
// from global memory (L2), forms the CTA's rows of V_j = R V_{j-1}, stores
// them, and a grid-wide barrier separates the passes.  The 8 warps split the
// columns (128 per step, a float4 per lane) and reduce RC rows x P columns
// of partial sums at a time, across lanes by halving and then across warps
// in shared memory.  The Gram of the fit needs only the CTA's own rows of
// the moments, so the folded alpha of the last pass needs no further
// barrier.  The barrier is bounded: one that runs out marks every active
// block timed out and sets an abort word that ends the other CTAs' waits,
// and later launches of the call return at once (the word is cleared when a
// pass starts).
constexpr int SC_THREADS = 256;
constexpr int SC_WARPS = SC_THREADS / 32;

template <int P>
struct SkChain {
  static constexpr int RC = P <= 8 ? 8 : 4;  // rows per chunk
  static constexpr int NV = RC * P;          // partial sums per lane
  // the warps' partial sums, later 8 x 15 doubles of the fit's reduction
  static constexpr int RED_BYTES =
      SC_WARPS * NV * 4 > 8 * 15 * 8 ? SC_WARPS * NV * 4 : 8 * 15 * 8;
  static size_t smem_bytes(int64_t rpc, int64_t n) {
    return static_cast<size_t>(rpc * n + P * (n + 4)) * 4 + RED_BYTES;
  }
};

struct ChainArgs {
  const float* R;
  int64_t n, rbs;  // block size and block stride of R
  const float* S;  // S_k = S + (*it) * s_stride, shared by the batch
  int64_t s_stride;
  const int* it;
  float* V;  // V_j of block b at V + b * vbs + j * n * p
  int64_t vbs;
  int p, batch, last;  // passes j = 1 .. last
  int vec;             // p == P and 16-byte aligned S and V: float4 staging
  int cpb;             // CTAs per block: CTA c serves block c / cpb
  int64_t rpc;         // rows per CTA (cpb * rpc >= n)
  const int* active;
  int* tmo;
  unsigned* bar;  // [0] arrivals, [2] abort
  int selftest;   // CTA 0 skips the first barrier, which the others wait out
};

SHP_DEV unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide barrier of a cooperative launch (every CTA resident) on a
// counter that only grows within a pass (cleared when a pass starts): a CTA
// arrives with one atomic add, which also tells it the count that completes
// this barrier (the next multiple of the grid size), and waits until the
// count reaches it, at most `limit` clock cycles or until the abort word is
// set.  One round trip to arrive and one to see the last arrival.  False, in
// every thread of the CTA, for a wait that gave up.
SHP_DEV bool grid_barrier(unsigned* bar, long long limit, bool arrive) {
  __shared__ int ok_s;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned g = gridDim.x;
    __threadfence();  // the CTA's stores (ordered by the block barrier) first
    const unsigned seen = arrive ? atomicAdd(bar, 1u) : ld_acquire_gpu(bar);
    const unsigned target = (seen / g + 1) * g;
    if (seen + 1 != target || !arrive) {
      const long long t0 = clock64();
      while (ld_acquire_gpu(bar) < target) {
        if (ld_acquire_gpu(bar + 2) != 0 || clock64() - t0 > limit) {
          ok = 0;
          break;
        }
      }
    }
    ok_s = ok;
  }
  __syncthreads();
  return ok_s != 0;
}

// The chain's alpha fit for block b: this CTA's partial Gram of V_d ..
// V_{2d+1} over its rows [row0, row0 + rows) goes to its own slot of gpart
// (15 doubles: no contended atomics); the CTA that completes the block's
// count sums the partials of the block's cpb CTAs and solves alpha.
// redd: 8 x 15 doubles of shared scratch.
SHP_DEV void chain_fit(const AlphaArgs& fa, int b, int64_t row0, int64_t rows, double* gpart,
                       int* gcnt, int cpb, double* redd, const int* tmo) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int last_s;
  GramPart gp;
  gram_reset(gp);
  const int64_t w0 = rows * warp / SC_WARPS, w1 = rows * (warp + 1) / SC_WARPS;
  gram_add(gp, fa, b, row0 + w0, static_cast<int>(w1 - w0));
#pragma unroll
  for (int i = 0; i < 15; ++i) gp.part[i] = warp_sum(gp.part[i]);
  if (lane == 0)
#pragma unroll
    for (int i = 0; i < 15; ++i) redd[warp * 15 + i] = gp.part[i];
  __syncthreads();
  if (threadIdx.x < 15) {
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < SC_WARPS; ++w) t += redd[w * 15 + threadIdx.x];
    gpart[blockIdx.x * 15 + threadIdx.x] = t;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();  // the partial before the count
    last_s = atomicAdd(&gcnt[b], 1) == cpb - 1;
    if (last_s) __threadfence();
  }
  __syncthreads();
  if (!last_s) return;
  // the last CTA of block b: 8 groups of 15 threads each sum every 8th CTA
  if (threadIdx.x < 8 * 15) {
    const int c = threadIdx.x % 15, grp = threadIdx.x / 15;
    double acc = 0.0;
#pragma unroll 4
    for (int i = grp; i < cpb; i += 8) acc += __ldcg(&gpart[(b * cpb + i) * 15 + c]);
    redd[grp * 15 + c] = acc;
  }
  __syncthreads();
  if (warp == 0) {
    double G[5][5] = {};
    gram_unpack<5, 8>(reinterpret_cast<const double (*)[15]>(redd), G);
    if (tmo != nullptr && tmo[b] != 0) {
      if (lane == 0) fa.alpha[b] = __int_as_float(0x7fc00000);
    } else {
      alpha_solve_warp(fa, b, G);
    }
    if (lane == 0) gcnt[b] = 0;
  }
}

template <int P>
__global__ void __launch_bounds__(SC_THREADS, 1)
    k_sketch_chain(const ChainArgs c, const AlphaArgs fa, double* gpart, int* gcnt) {
  count_kernel_run();
  constexpr int RC = SkChain<P>::RC, NV = SkChain<P>::NV;
  extern __shared__ __align__(16) float sc_smem[];
  if (ld_acquire_gpu(c.bar + 2) != 0) return;  // an earlier launch of this pass gave up
  const int64_t n = c.n, ldv = n + 4, np = n * c.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = static_cast<int>(blockIdx.x) / c.cpb;
  const int64_t r0 = (static_cast<int64_t>(blockIdx.x) % c.cpb) * c.rpc;
  const int64_t rows = n - r0 < c.rpc ? (n - r0 > 0 ? n - r0 : 0) : c.rpc;
  const bool on = rows > 0 && (c.active == nullptr || c.active[b] != 0);
  float* Rs = sc_smem;           // the CTA's rows r0 .. r0 + rows - 1, n floats each
  float* Vs = Rs + c.rpc * n;    // [P][ldv]: V_{j-1} transposed
  float* red = Vs + P * ldv;     // [warp][NV]: the warps' partial sums (RED_BYTES)
  const int k = c.it != nullptr ? *c.it : 0;

  // R rows into shared memory (16-byte rows), eight loads in flight per thread
  if (on) {
    const float4* src = reinterpret_cast<const float4*>(c.R + b * c.rbs + r0 * n);
    float4* dst = reinterpret_cast<float4*>(Rs);
    const int64_t cnt = rows * n / 4;
    for (int64_t i0 = threadIdx.x; i0 < cnt; i0 += 8 * SC_THREADS) {
      float4 t[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (i0 + u * SC_THREADS < cnt) t[u] = __ldg(src + i0 + u * SC_THREADS);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (i0 + u * SC_THREADS < cnt) dst[i0 + u * SC_THREADS] = t[u];
    }
  }

  for (int j = 1; j <= c.last; ++j) {
    if (j > 1) {
      // V_{j-1} complete in every CTA; the self-test's CTA 0 never arrives
      const bool test = c.selftest && j == 2;
      if (!grid_barrier(c.bar, test ? SHP_SELFTEST_LIMIT : SHP_SPIN_LIMIT,
                        !(test && blockIdx.x == 0))) {
        if (threadIdx.x == 0) {
          atomicExch(c.bar + 2, 1u);
          if (c.tmo != nullptr)
            for (int bb = 0; bb < c.batch; ++bb)
              if (c.active == nullptr || c.active[bb] != 0) atomicExch(&c.tmo[bb], ST_ETIMEOUT);
        }
        return;  // no copy is in flight: plain loads only
      }
    }
    if (!on) continue;  // the barriers are still taken
    // stage V_{j-1} of the block (written by other CTAs: L2 loads)
    const float* src = j == 1 ? c.S + static_cast<int64_t>(k) * c.s_stride
                              : c.V + b * c.vbs + (j - 1) * np;
    if (c.vec) {
      const float4* s4 = reinterpret_cast<const float4*>(src);
      const int64_t cnt = n * (P / 4);
      for (int64_t i0 = threadIdx.x; i0 < cnt; i0 += 8 * SC_THREADS) {
        float4 t[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (i0 + u * SC_THREADS < cnt) t[u] = __ldcg(s4 + i0 + u * SC_THREADS);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int64_t i = i0 + u * SC_THREADS;
          if (i >= cnt) break;
          const int64_t col = i / (P / 4);
          const int q = 4 * static_cast<int>(i % (P / 4));
          Vs[q * ldv + col] = t[u].x;
          Vs[(q + 1) * ldv + col] = t[u].y;
          Vs[(q + 2) * ldv + col] = t[u].z;
          Vs[(q + 3) * ldv + col] = t[u].w;
        }
      }
    } else {
      const int64_t cnt = n * P;
      for (int64_t i0 = threadIdx.x; i0 < cnt; i0 += 8 * SC_THREADS) {
        float t[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int64_t i = i0 + u * SC_THREADS;
          const int q = static_cast<int>(i % P);
          t[u] = i < cnt && q < c.p ? __ldcg(src + (i / P) * c.p + q) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int64_t i = i0 + u * SC_THREADS;
          if (i < cnt) Vs[(i % P) * ldv + i / P] = t[u];
        }
      }
    }
    __syncthreads();
    float* out = c.V + b * c.vbs + j * np;
    for (int64_t l0 = 0; l0 < rows; l0 += RC) {
      float acc[NV];
#pragma unroll
      for (int i = 0; i < NV; ++i) acc[i] = 0.f;
      for (int64_t col = warp * 128 + lane * 4; col < n; col += SC_WARPS * 128) {
        float4 v[P];
#pragma unroll
        for (int q = 0; q < P; ++q) v[q] = *reinterpret_cast<const float4*>(Vs + q * ldv + col);
#pragma unroll
        for (int r = 0; r < RC; ++r) {
          const int64_t l = l0 + r < rows ? l0 + r : rows - 1;  // a spare row: not stored
          const float4 x = *reinterpret_cast<const float4*>(Rs + l * n + col);
#pragma unroll
          for (int q = 0; q < P; ++q) {
            float a = acc[r * P + q];
            a = fmaf(x.x, v[q].x, a);
            a = fmaf(x.y, v[q].y, a);
            a = fmaf(x.z, v[q].z, a);
            acc[r * P + q] = fmaf(x.w, v[q].w, a);
          }
        }
      }
      halve_lanes<NV, 5>(acc, lane);
#pragma unroll
      for (int i = 0; i < NV / 32; ++i) red[warp * NV + lane * (NV / 32) + i] = acc[i];
      __syncthreads();
      if (threadIdx.x < NV) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < SC_WARPS; ++w) sum += red[w * NV + threadIdx.x];
        const int r = threadIdx.x / P, q = threadIdx.x % P;
        if (l0 + r < rows && q < c.p) out[(r0 + l0 + r) * c.p + q] = sum;
      }
      __syncthreads();
    }
  }

  // folded alpha: the Gram over the CTA's rows of V_d .. V_{2d+1}, stored by
  // this CTA and ordered by the block barrier that ended the last chunk
  if (gpart == nullptr || !on) return;
  chain_fit(fa, b, r0, rows, gpart, gcnt, c.cpb, reinterpret_cast<double*>(red), c.tmo);
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
  double G[5][5] = {};
  if (nv == 3)
    gram_unpack<3, AL_THREADS / 32>(red, G);
  else if (nv == 4)
    gram_unpack<4, AL_THREADS / 32>(red, G);
  else
    gram_unpack<5, AL_THREADS / 32>(red, G);
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

// The cooperative launch of k_sketch_chain: the SMs are shared out evenly
// among the blocks (cpb CTAs of rpc rows each per block).  False (nothing
// launched) when the batch has more blocks than SMs, a CTA's rows do not fit
// in shared memory, or the device cannot launch the grid cooperatively.
template <int P>
bool launch_sketch_chain(ChainArgs c, const AlphaArgs* fa, double* gpart, int* gcnt,
                         cudaStream_t st, cudaError_t* err) {
  int dev = 0, sms = 0, coop = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess ||
      sms <= 0 || coop == 0 || c.batch > sms)
    return false;
  const int64_t cpb_max = sms / c.batch;
  c.rpc = (c.n + cpb_max - 1) / cpb_max;
  c.cpb = static_cast<int>((c.n + c.rpc - 1) / c.rpc);  // every CTA has rows
  const size_t smem = SkChain<P>::smem_bytes(c.rpc, c.n);
  if (smem > 200 * 1024) return false;
  auto kern = k_sketch_chain<P>;
  static int set_for_dev[64];
  if (set_for_dev[dev] == 0) {
    *err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (*err != cudaSuccess) return true;
    set_for_dev[dev] = 1;
  }
  const int grid = c.cpb * c.batch;
  if (grid > kChainMaxCtas) return false;  // the partial-Gram slots
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, SC_THREADS, smem) !=
          cudaSuccess ||
      static_cast<int64_t>(per_sm) * sms < grid)
    return false;
  AlphaArgs none;
  memset(&none, 0, sizeof(none));
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(SC_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  *err = cudaLaunchKernelEx(&cfg, kern, c, fa != nullptr ? *fa : none,
                            fa != nullptr ? gpart : nullptr, fa != nullptr ? gcnt : nullptr);
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

cudaError_t sketch_chain(const float* R, int64_t n, int64_t r_bstride, const float* S,
                         int64_t s_stride, const int* it, float* V, int p, int d, int batch,
                         const int* active, int* tmo, unsigned* bar, float lo, float hi,
                         float* alpha, float* report_alpha, int64_t report_stride,
                         int report_slot, double* gpart, int* gcnt, cudaStream_t st, bool* done,
                         int selftest) {
  *done = false;
  if (batch <= 0 || n <= 0 || bar == nullptr || p < 1 || p > 16) return cudaSuccess;
  if ((reinterpret_cast<uintptr_t>(R) & 15) != 0 || n % 4 != 0 || r_bstride % 4 != 0)
    return cudaSuccess;
  const int P = p <= 4 ? 4 : (p <= 8 ? 8 : 16);
  ChainArgs c;
  memset(&c, 0, sizeof(c));
  c.R = R;
  c.n = n;
  c.rbs = r_bstride;
  c.S = S;
  c.s_stride = s_stride;
  c.it = it;
  c.V = V;
  c.vbs = static_cast<int64_t>(2 * d + 2) * n * p;
  c.p = p;
  c.batch = batch;
  c.last = 2 * d + 1;
  c.vec = p == P && (reinterpret_cast<uintptr_t>(S) & 15) == 0 &&
          (reinterpret_cast<uintptr_t>(V) & 15) == 0 && s_stride % 4 == 0;
  c.active = active;
  c.tmo = tmo;
  c.bar = bar;
  c.selftest = selftest;
  AlphaArgs g;
  memset(&g, 0, sizeof(g));
  const bool fit = gpart != nullptr && gcnt != nullptr;
  if (fit) {
    g.tmo = tmo;
    g.V = V;
    g.n = n;
    g.vbs = c.vbs;
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
  }
  cudaError_t e = cudaSuccess;
  bool launched = false;
  if (P == 4)
    launched = launch_sketch_chain<4>(c, fit ? &g : nullptr, gpart, gcnt, st, &e);
  else if (P == 8)
    launched = launch_sketch_chain<8>(c, fit ? &g : nullptr, gpart, gcnt, st, &e);
  else
    launched = launch_sketch_chain<16>(c, fit ? &g : nullptr, gpart, gcnt, st, &e);
  *done = launched && e == cudaSuccess;
  return e;
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
