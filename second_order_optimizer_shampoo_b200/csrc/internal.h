// Host-side interfaces between the C-ABI layer (api.cu) and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "shampoo_prism.h"

namespace shp {

// Kernels run so far on the current device, per translation unit (device
// counters read back with a synchronous copy).
uint64_t kernel_runs_gemm();
uint64_t kernel_runs_sketch();
uint64_t kernel_runs_elementwise();
uint64_t kernel_runs_small();

enum Mode { MODE_TF32 = 0, MODE_3XTF32 = 1, MODE_BF16 = 2 };
enum EpiKind {
  EPI_STORE = 0,
  EPI_RESID = 1,
  EPI_GPOLY = 2,
  EPI_EMA = 3,
  EPI_APPLY = 4,
  EPI_AXPY = 5,
  EPI_MOMENTUM = 6
};
enum OutFmt { OUT_F32 = 0, OUT_SPLIT = 1, OUT_BF16 = 2 };

// Per-block outcome codes (mirrors shp_status in include/shampoo_prism.h).
enum {
  ST_OK = 0,
  ST_EINVAL = 1,  // a block's own arguments are out of range (per-block shapes)
  ST_ENOCONV = 16,
  ST_ESTALL = 17,
  ST_ENONFINITE = 18,
  ST_ETIMEOUT = 19
};

// A batched row-major operand in HBM.  `hi` holds the fp32 value (TF32 mode),
// the TF32-rounded high part (split mode, with `lo` = tf32(value - hi), so
// that hi + lo equals the value to within 2^-22 relative) or bf16.  The
// tensor cores truncate fp32 operands to TF32, hence both parts are stored
// already rounded to nearest.
//   mn == false (K-major): element (i, k) of the logical M x K (or N x K
//     for B^T) operand sits at hi[i * ld + k];
//   mn == true  (MN-major): element (i, k) sits at hi[k * ld + i].
struct Operand {
  const void* hi;
  const float* lo;
  bool mn;
  int64_t ld;       // elements between consecutive memory rows
  int64_t bstride;  // elements between batch members
};

// What the epilogue does with accumulator element acc(i, j) of block b.
//   STORE: v = s0 * acc
//   RESID: v = [i==j] - acc, and norm2[b] += v^2
//   GPOLY: v = s1 * aux(i,j) + alpha[b] * acc   (Delta = g - I; out2 gets I + Delta)
//   EMA:   v = s0 * out(i,j) + s1 * acc + s2 * [i==j]   (read-modify-write)
//   APPLY: v = out(i,j) + s0 * eta[b] * acc              (read-modify-write)
//   AXPY:  v = aux(i,j) + s0 * acc                       (X + X Delta)
//   MOMENTUM: m = s1 * aux(i,j) + acc, v = out(i,j) + s0 * eta[b] * m; out2 gets m
// (eta[b] = alpha[b] when alpha is non-null, else 1).
// v is written to `out` (and to `out2` when non-null) in `out_fmt`.  The
// update polynomial is kept as Delta = g - I and applied as X + X Delta so
// that its small part keeps full relative precision in every storage format
// (g itself would round to 2^-8 near 1 in bf16).
struct EpiParams {
  int kind;
  int out_fmt;
  void* out_hi;
  float* out_lo;
  void* out2_hi;
  float* out2_lo;
  float* out_plain;  // optional plain fp32 copy of v (same layout as out)
  void* out_b16;     // optional bf16 copy of v (same layout as out)
  int64_t ldo, bso;
  const void* aux_hi;
  const float* aux_lo;
  int aux_fmt;  // OUT_F32 / OUT_SPLIT / OUT_BF16
  int64_t lda_aux, bs_aux;
  const float* alpha;
  float s0, s1, s2;
  float* norm2;       // norm2[b * norm2_stride] accumulates ||v||^2 (RESID)
  int norm2_stride;
  const int* active;  // blocks with active[b] == 0 are skipped (may be null)
  int* status;        // receives ST_ETIMEOUT if a pipeline wait runs out (may be null)
  int M, N;
  // The result is symmetric (M == N; any kind but MOMENTUM, whose out2 is not
  // of the form I + v): the persistent kernel computes the tiles on and above
  // the diagonal and writes each off-diagonal tile's mirror image too (to out,
  // out2, out_plain and out_b16); other kernels compute it all.  Read-modify-write and
  // aux operands are read on the upper tiles only, so they must be symmetric.
  int sym;
  // bounded-wait self-test (persistent kernel): the producer first waits on a
  // barrier nothing completes; status[0] receives ST_ETIMEOUT
  int selftest;
  // set by the persistent kernel's launcher: a bf16 result whose rows (and
  // aux rows) start on 16-byte boundaries takes the lane-per-row epilogue
  int vec;
};

// C[b] (M x N) = A[b] (M x K) * B[b] (K x N) on tcgen05 tensor cores,
// followed by the epilogue.  A and B must share `mode`'s storage type.
cudaError_t gemm_tc(int mode, const Operand& A, const Operand& B, int M, int N, int K,
                    int batch, const EpiParams& ep, cudaStream_t st);

// 3-D fp32 tensor map over [batch][rows][inner] (row stride ld, batch stride
// bstride, in elements) with a box of box_rows x box_inner, no swizzle and
// zero fill outside the tensor.  False if cuTensorMapEncodeTiled rejects it.
bool tensor_map_rows(CUtensorMap* m, const float* ptr, int64_t inner, int64_t rows,
                     int64_t batch, int64_t ld, int64_t bstride, int box_inner, int box_rows);

// 4-D int8 map over [blocks][slices][rows][kb_bytes] (the K-blocked digit
// slices of the Ozaki-scheme products, ozaki.cu; kb_bytes 64 or 128) with a
// box of all slices x box_rows x kb_bytes and the swizzle of that row
// length, zero fill past `rows`.
bool tensor_map_slices(CUtensorMap* m, const int8_t* ptr, int64_t rows, int slices,
                       int64_t blocks, int kb_bytes, int box_rows);

// ---- PRISM sketch and alpha (sketch_alpha.cu)
// Vout[b] = R[b] * Vin[b]; R is n x n (hi + lo when lo != null); V is n x p.
// vin_bstride == 0 shares Vin across the batch.  When `it` is non-null the
// input is Vin + (*it) * it_stride (the sketch slice of the current iteration).
// A pipeline wait of the bulk-copy variant that runs out sets tmo[b] (if
// non-null) to ST_ETIMEOUT.  selftest (bulk-copy variant only): the first V
// hand-over waits on a barrier nothing completes, so that wait runs out.
cudaError_t sketch_pass(const float* Rhi, const float* Rlo, int64_t n, int64_t r_bstride,
                        const float* Vin, int64_t vin_bstride, float* Vout, int64_t vout_bstride,
                        int p, int batch, const int* active, const int* it, int64_t it_stride,
                        cudaStream_t st, int* tmo = nullptr, int selftest = 0);
// V is stored per block as [2d+2][n][p] (slot j holds V_j; slot 0 unused).
// Gram of V_d..V_{2d+1}, the
// quartic J(alpha) and its minimiser on [lo, hi]; writes alpha[b] and, when
// non-null, J_coef[b][5] and report_alpha[b * stride + slot (+ *it)].
// Adaptive degree state of a call (all [batch] device arrays): the current
// degree of each block, the active blocks at degree 1 and 2 (masks of the
// launches that form Delta), and the report's degree trajectory (may be null).
struct AdaptiveDeg {
  int enabled;
  float raise_above;
  int* deg;
  int* act1;
  int* act2;
  int* rep_degree;
};
// With ad enabled (d = 2): V holds V_1..V_5 and each block fits at its
// current degree, raising it by the rule of shp_prism_opts.adaptive_degree.
// tmo (may be null): a block whose flag is set (a sketch wait ran out, so V
// is incomplete) gets alpha = NaN and NaN coefficients instead of a fit.
// The last sketch pass V_{2d+1} = R V_2d with the alpha fit folded in: each
// consumer warp adds its rows' partial Gram of V_d .. V_{2d+1} (fp64) into
// gram[b] and the warp that completes a block solves its alpha (fitted alpha
// at fixed degree d; V is the moment stack [batch][2d+2][n][p]).  *fused
// tells whether the fused kernel ran; when it did not (R not 16-byte aligned,
// V too large for shared memory) the pass ran plain and the caller fits.
cudaError_t sketch_pass_alpha(const float* R, int64_t n, int64_t r_bstride, const float* Vin,
                              int64_t vin_bstride, float* Vout, int64_t vout_bstride, int p,
                              int batch, const int* active, cudaStream_t st, int* tmo,
                              const float* V, int d, float lo, float hi, float* alpha,
                              float* report_alpha, int64_t report_stride, int report_slot,
                              const int* it, double* gram, int* gcnt, bool* fused,
                              int selftest = 0);
// Every pass V_1 = R S_k .. V_{2d+1} of one iteration in one cooperative
// launch (S_k = S + (*it) * s_stride, shared by the batch; V as above), for a
// batch whose rows of R fit in the CTAs' shared memory (no more blocks than
// SMs).  With gpart/gcnt non-null the alpha fit of fixed degree d is folded
// in: each CTA writes its partial Gram to its own slot of gpart
// ([kChainMaxCtas][15] doubles) and the CTA that completes a block's count
// in gcnt[b] (zero on entry; left zero) sums them and solves alpha.  bar:
// three words of device scratch (arrivals, unused, abort) that reset_pass
// clears; a grid barrier that runs out
// sets tmo of every active block to ST_ETIMEOUT and the abort word, and
// later launches then return at once.  selftest: CTA 0 skips the first
// barrier, which the others wait out with the short limit.  *done = false:
// not eligible, nothing launched (the caller runs the passes one by one).
cudaError_t sketch_chain(const float* R, int64_t n, int64_t r_bstride, const float* S,
                         int64_t s_stride, const int* it, float* V, int p, int d, int batch,
                         const int* active, int* tmo, unsigned* bar, float lo, float hi,
                         float* alpha, float* report_alpha, int64_t report_stride,
                         int report_slot, double* gpart, int* gcnt, cudaStream_t st, bool* done,
                         int selftest = 0);
constexpr int kChainMaxCtas = 512;
cudaError_t alpha_solve(const float* V, int64_t n, int p, int d, int batch, float lo, float hi,
                        int fixed_alpha, const int* active, float* alpha, double* J_coef,
                        float* report_alpha, int64_t report_stride, int report_slot,
                        const int* it, cudaStream_t st, const AdaptiveDeg* ad = nullptr,
                        const int* tmo = nullptr);

// ---- per-block control (sketch_alpha.cu)
struct BlockState {
  float norm2;     // ||R_k||_F^2 accumulated by the residual epilogue
  float prev_res;  // residual of the previous iteration
  float c;         // Frobenius norm of the input (normalisation)
  int iters;       // update steps taken in the current pass
  int iters1;      // update steps taken in pass 1 (set when pass 2 starts)
  int status;      // first non-OK outcome over the passes
  int pass_status;
  int pad;
};
// Workspace-resident control block of one call.
struct Ctl {
  BlockState* bs;
  int* active;
  int* deg;       // current degree of each block (adaptive degree)
  int* act1;      // active blocks at degree 1 / 2 (adaptive degree)
  int* act2;
  double* dnorm;  // ||input||_F^2 per block
  int* tmo;       // ST_ETIMEOUT flags from the GEMM pipeline
  float* alpha;   // alpha_k per block
  int* it;        // iteration index k of the current pass (device-side loop)
  int* flag;      // loop condition for the host-driven diagnostic loop
  double* gram;   // [batch][15] sketch Gram accumulated by the fused last pass
  int* gcnt;      // [batch] items of the fused last pass seen so far
  unsigned* gbar;  // [4] grid barrier of the few-block sketch: arrivals, -, abort
  double* gpart;   // [kChainMaxCtas][15] its CTAs' partial Grams
};
// Stop test of iteration k = *ctl.it for every active block.
cudaError_t control_step(const Ctl& ctl, int batch, int64_t n, int max_iter, float tol,
                         float stall_below, float stall_ratio, float* report_res,
                         int64_t res_stride, int res_slot, int* report_iters, int iters_slot,
                         cudaStream_t st);
// End of an iteration of the device-side loop: *ctl.it += inc, then the
// graph conditional `h` = (some block still active and *it <= max_iter + 1);
// with h == 0 the condition goes to *ctl.flag instead (host-driven loop).
cudaError_t loop_step(const Ctl& ctl, int batch, int inc, int max_iter,
                      cudaGraphConditionalHandle h, cudaStream_t st);

// ---- elementwise (elementwise.cu)
// Start of a pass: active = 1, counters cleared; first_pass also clears the
// status, the timeout flags and the input norms; otherwise iters1 = iters.
// start_degree > 0 also sets every block's degree (adaptive degree).
cudaError_t reset_pass(const Ctl& ctl, int batch, int first_pass, cudaStream_t st,
                       int start_degree = 0);
// dnorm[b] += ||X[b]||_F^2 (X fp32 or bf16, rows x cols contiguous per block).
cudaError_t frob_norm2(const void* X, int is_bf16, int64_t count, int batch, const Ctl& ctl,
                       cudaStream_t st);
// c = sqrt(dnorm); Y = (A + A^T) / (2c); R = I - Y; norm2 = ||R||_F^2.
// Z_0 = I is implied (the first step writes Z_1; see coupled_finish).
// (lo pointers null in TF32 mode; Rs, when non-null, gets a plain fp32 R.)
cudaError_t coupled_init(const float* A, int64_t n, int batch, const Ctl& ctl, float* Yhi,
                         float* Ylo, float* Rhi, float* Rlo, float* Rs, cudaStream_t st);
// Pass 2: Y[0] <- Y[iters1 % 2]; R = I - Y; norm2 = ||R||_F^2 (Z_0 = I implied).
cudaError_t coupled_restart(int64_t n, int batch, const Ctl& ctl, float* const* Yhi,
                            float* const* Ylo, float* Rhi, float* Rlo, float* Rs,
                            cudaStream_t st);
// Delta = alpha[b] R (d = 1) in `fmt`; I + Delta into (g2hi, g2lo) when non-null.
// `active` overrides ctl.active (the degree-1 mask under adaptive degree).
cudaError_t gform_d1(const float* Rhi, const float* Rlo, int64_t n, int batch, const Ctl& ctl,
                     int fmt, void* ghi, float* glo, void* g2hi, float* g2lo, cudaStream_t st,
                     const int* active = nullptr);
// X_out[b] = c_b^e * S[iters_b % 2][b] (hi + lo), S = the two ping-pong slots;
// with z_slots (S holds Z, whose Z_0 = I is not stored) a block that made no
// step in its last pass gets c_b^e * I.
cudaError_t coupled_finish(int64_t n, int batch, const Ctl& ctl, double c_exponent,
                           const float* const* Shi, const float* const* Slo, float* X_out,
                           bool z_slots, cudaStream_t st);
// hi = tf32(X), lo = X - hi.
// L[b] <- beta L[b] + (1 - beta) P[t][b] + eps I for t = 0 .. count-1 in
// turn (the EMA recurrence over precomputed products P: [count][batch][n][n]).
cudaError_t ema_replay(float* L, const float* P, int64_t n, int count, int batch, float beta,
                       float eps, cudaStream_t st);
cudaError_t split_copy(const float* X, int64_t count, float* hi, float* lo, cudaStream_t st);
// X0 = G / ||G||_F (uses dnorm) in `fmt`.
cudaError_t polar_init(const void* G, int g_bf16, int64_t count, int batch, const Ctl& ctl,
                       int fmt, void* Xhi, float* Xlo, cudaStream_t st);
// X_out[b] = slot[iters_b % 2][b] in the output storage (bf16 or fp32).
cudaError_t polar_finish(int64_t count, int batch, const Ctl& ctl, int fmt,
                         const void* const* Shi, const float* const* Slo, void* X_out,
                         int out_bf16, cudaStream_t st);
// Adaptive step of the update ([Shampoo] 5.1): acc[b] += ||G_b||_F^2 (G fp32,
// count elements per block; dn is [batch] fp64 scratch), eta[b] = lr / sqrt(1 + acc[b]).
cudaError_t adaptive_step(const float* G, int64_t count, int batch, double* dn, double* acc,
                          float lr, float* eta, cudaStream_t st);
// report.status[b] = ETIMEOUT if flagged, else bs[b].status.
cudaError_t write_status(const Ctl& ctl, int batch, int* report_status, cudaStream_t st);

// ---- on-chip small blocks (small_block.cu): one CTA per block runs the
// whole iteration in shared memory; products in fp32 FMA.
// True when an m x n input (n x n for inverse roots) and sketch width p fit.
bool small_block_ok(int64_t m, int64_t n, int p);
// power: SHP_POW_*; report pointers may be null (layouts as the ABI's report).
cudaError_t small_inv_root(const float* A, int n, int batch, int power,
                           const shp_prism_opts& o, const float* S, float* X,
                           int* rep_status, int* rep_iters, float* rep_resid, float* rep_alpha,
                           int* rep_degree, cudaStream_t st);
// Blocks of different shapes: block b is dims[2b] x dims[2b+1] (<= 64,
// multiples of 4) at G + offsets[b] / X + offsets[b]; sketch slices are
// 64 x p and a block uses their first min(m_b, n_b) rows.
cudaError_t small_polar_varsize(const float* G, const int* dims, const int64_t* offsets,
                                int batch, const shp_prism_opts& o, const float* S, float* X,
                                int* rep_status, int* rep_iters, float* rep_resid,
                                float* rep_alpha, int* rep_degree, cudaStream_t st);
// sign: the sign function of a symmetric square G (R = I - X X).
cudaError_t small_polar(const float* G, int m, int n, int batch, const shp_prism_opts& o,
                        const float* S, float* X, int* rep_status, int* rep_iters,
                        float* rep_resid, float* rep_alpha, int* rep_degree, bool sign,
                        cudaStream_t st);

// ---- fp64-grade products on the int8 tensor cores (ozaki.cu)
// Digit slices of an fp64 matrix X (rows x cols): the row slicing serves X
// as the left operand A, the column slicing (that of X^T) as the right
// operand B.  Both are K-blocked: [batch][K / 64][S][rows of the operand][64]
// with K padded to oz_ldk(K) (K = cols for `rows`, rows for `cols`).
struct OzSlices {
  int8_t* rows;    // [batch][cols / 64][S][rows][64], weights rscale
  int8_t* cols;    // [batch][rows / 64][S][cols][64], weights cscale
  double* rscale;  // [batch][rows]
  double* cscale;  // [batch][cols]
};
// Epilogue of one Ozaki product C = A B (acc = the fp64 value of C):
//   STORE v = s0 acc; RESID v = [i==j] - acc, norm2 += v^2;
//   GPOLY v = s1 aux + alpha[b] acc (out2 = I + v); AXPY v = aux + s0 acc.
// out, out2 and aux are fp64 [batch][M][N] (ld / batch strides in elements);
// sa [batch][M] and sb [batch][N] are the slice weights of A and B.
struct OzEpi {
  int kind;
  double* out;
  double* out2;
  int64_t ldo, bso;
  const double* aux;
  int64_t lda, bsa;
  const double* sa;
  const double* sb;
  const float* alpha;
  float s0, s1;
  float* norm2;
  int norm2_stride;
  const int* active;
  int* status;
  int M, N;
  // maxima keys (high word of |v|) of out and out2 by row [batch][M] and by
  // column [batch][N], folded in with atomicMax (may be null)
  unsigned* rmax;
  unsigned* cmax;
  unsigned* rmax2;
  unsigned* cmax2;
  int selftest;  // as EpiParams::selftest
};
int64_t oz_ldk(int64_t k);                                     // K padded to whole blocks
size_t oz_slices_bytes(int64_t rows, int64_t k, int64_t batch);  // one slicing's digits
int oz_slice_count();
// Slices of X ([batch][rows][cols] at ld / bs); out.rows / out.cols may be
// null to skip that slicing; maxbuf holds the row maxima keys [batch][rows]
// and then the column ones [batch][cols]: with have_max they were folded in
// by the epilogue that wrote X (after oz_clear_max), otherwise they are
// computed here first.  x32 (may be null) gets a plain fp32 copy of X.
// Blocks with active[b] == 0 are skipped.
cudaError_t oz_slice(const double* X, int rows, int cols, int64_t ld, int64_t bs, int batch,
                     const int* active, unsigned* maxbuf, bool have_max, const OzSlices& out,
                     float* x32, cudaStream_t st);
cudaError_t oz_clear_max(unsigned* maxbuf, int rows, int cols, int batch, cudaStream_t st);
// C = A B from A's row slices ([batch][S][M][oz_ldk(K)]) and B's column
// slices ([batch][S][N][oz_ldk(K)]), then the epilogue.
cudaError_t gemm_oz(const int8_t* Arows, const int8_t* Bcols, int M, int N, int K, int batch,
                    const OzEpi& ep, cudaStream_t st);
// fp64 storage kernels of the inverse-root passes (see the fp32 versions).
cudaError_t oz_init(const float* A, int64_t n, int batch, const Ctl& ctl, double* Y, double* R,
                    cudaStream_t st);
cudaError_t oz_restart(int64_t n, int batch, const Ctl& ctl, const double* Y, double* R,
                       cudaStream_t st);
cudaError_t oz_gform_d1(const double* R, int64_t n, int batch, const Ctl& ctl, double* D,
                        double* D2, cudaStream_t st, const int* active = nullptr);
cudaError_t oz_finish(int64_t n, int batch, const Ctl& ctl, double c_exponent, const double* S,
                      float* X_out, bool z_slots, cudaStream_t st);
uint64_t kernel_runs_ozaki();


}  // namespace shp
