/*
 * shampoo_prism.h - C ABI of the B200 (sm_100a) Shampoo preconditioner step
 * with PRISM-accelerated Newton-Schulz matrix functions.
 *
 * Sources of the operations (page title, section):
 *   [Shampoo]  "深度学习中的优化器之Shampoo算法原理与二阶优化机制"
 *              (algorithm.idocdown.com): 2.2-2.3 statistics and update,
 *              3.1 matrix roots, 3.2 block-diagonal approximation,
 *              6.3 shampoo_update(W, G, L, R, beta, epsilon, lr).
 *   [PRISM]    "Sintesi Tecnica: PRISM" (gist.science): Parte I residual-form
 *              iteration X_{k+1} = X_k f(R_k); Parte II.1 polynomial
 *              g_d(xi; alpha) = f_{d-1}(xi) + alpha xi^d, alpha fitted by least
 *              squares and constrained to [l, u]; Parte II.2 Gaussian sketch.
 *
 * Conventions shared by every entry point
 *   - Matrices are fp32 (or bf16 where stated), row-major, contiguous, and a
 *     batch of B matrices is B consecutive matrices (stride rows*cols).
 *   - Every pointer argument is DEVICE memory owned by the caller unless it is
 *     documented as host memory.  The library never allocates, frees or keeps
 *     a caller pointer after the call returns; scratch memory is the caller's
 *     `ws` buffer of at least shp_workspace_bytes(...) bytes, 256-byte aligned.
 *   - Column counts of fp32 matrices must be multiples of 4 and of bf16
 *     matrices multiples of 8 (16-byte rows for the tensor-memory-access
 *     unit); base pointers must be 16-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronise the host.
 *   - The return value is decided before any launch: SHP_OK, SHP_EINVAL
 *     (bad argument, nothing launched), SHP_EUNSUPPORTED, or SHP_ECUDA (a
 *     CUDA runtime error at launch; the stream may hold partial work).
 *     Numerical outcomes are per-block codes written to `report.status` on the
 *     device; the caller reads them after synchronising the stream.
 *   - No exceptions cross this boundary.  State kept between calls: cached
 *     kernel attributes, and up to 16 instantiated CUDA graphs of the matrix
 *     functions keyed by every pointer, size and option of a call (a repeated
 *     call with the same buffers replays its graph; the oldest
 *     entry is replaced).
 */
#ifndef SHAMPOO_PRISM_H
#define SHAMPOO_PRISM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* shp_stream; /* cudaStream_t */

typedef enum {
  SHP_OK = 0,
  SHP_EINVAL = 1,
  SHP_EUNSUPPORTED = 2,
  SHP_ECUDA = 3,
  /* per-block outcomes, written to report.status */
  SHP_ENOCONV = 16,    /* max_iter update steps taken, residual still above tol  */
  SHP_ESTALL = 17,     /* residual stopped shrinking once small (precision floor) */
  SHP_ENONFINITE = 18, /* residual became NaN or Inf                              */
  SHP_ETIMEOUT = 19    /* a bounded wait inside a kernel ran out                  */
} shp_status;

typedef enum {
  SHP_TF32 = 0,   /* fp32 storage, products on TF32 tensor cores                  */
  SHP_3XTF32 = 1, /* fp32 storage split as hi (TF32) + lo; acc += hh + hl + lh     */
  SHP_BF16 = 2,   /* bf16 storage, fp32 accumulation (polar factor only)           */
  SHP_OZAKI = 3   /* fp64 storage; every product split into five int8 digit slices
                     per operand and accumulated exactly on the int8 tensor cores
                     (about 2^-40 of the row/column maxima per product; inverse
                     roots only; see shp_matmul_f64)                               */
} shp_precision;

typedef enum {
  SHP_POW_INV4 = 0, /* A^(-1/4): the Shampoo preconditioner power ([Shampoo] 2.3) */
  SHP_POW_INV2 = 1, /* A^(-1/2)                                                    */
  SHP_POW_SQRT = 2  /* A^(1/2)                                                     */
} shp_power;

typedef enum { SHP_OP_INV_ROOT = 0, SHP_OP_POLAR = 1, SHP_OP_ALPHA_FIT = 2, SHP_OP_APPLY = 3,
               SHP_OP_GRAM_EMA = 4, SHP_OP_GRAM_EMA_STEPS = 5 } shp_op;

/* Knobs of a PRISM Newton-Schulz pass ([PRISM] Parte I-II).
 *   d           degree of g_d; 1 or 2
 *   p           sketch width, 1..32
 *   lo, hi      alpha interval [l, u]; [1/2, 1] for d = 1 as printed, the
 *               Taylor coefficient 3/8 and 1 for d = 2
 *   tol         stop when ||R_k||_F / sqrt(n) <= tol (checked before an update)
 *   max_iter    at most this many update steps per pass (<= 256)
 *   prec        SHP_TF32 / SHP_3XTF32 / SHP_OZAKI (inverse roots); SHP_BF16
 *               only for polar storage
 *   fixed_alpha 1: alpha = lo every step (plain Taylor Newton-Schulz; with
 *               d = 2 and lo = 3/8 this is Chebyshev's third-order method for
 *               the inverse square root, which PRISM accelerates by fitting
 *               alpha instead)
 *   stall_below, stall_ratio: stop with SHP_ESTALL when the previous residual
 *               is below stall_below and the new one exceeds stall_ratio times it
 *   adaptive_degree 1: every pass starts at degree 1 and raises to d (= 2) for
 *               the rest of the pass once the sketched degree-1 fit predicts a
 *               contraction ||r(R_k) S_k||_F / ||R_k S_k||_F above raise_above
 *               ([PRISM] 方法论 3, adaptive degree selection); the interval of
 *               degree e is then [c_e, hi] with c_e its Taylor coefficient
 *               (1/2, 3/8) and lo is not used; needs fixed_alpha = 0
 *   host_loop   0 (default): the iteration loop runs on the device inside a
 *               cached CUDA graph (a conditional WHILE node), with no host
 *               synchronisation; 1: the same kernels are launched from a host
 *               loop that synchronises the stream once per iteration to read
 *               the loop condition (for profilers and launch tracers that do
 *               not look inside CUDA graphs; slower, never captured)
 */
typedef struct {
  int d;
  int p;
  float lo, hi;
  float tol;
  int max_iter;
  int prec;
  int fixed_alpha;
  float stall_below;
  float stall_ratio;
  int adaptive_degree;
  float raise_above;
  int host_loop;
} shp_prism_opts;

/* Optional per-block trajectory, all device pointers, each may be NULL.
 *   status [B]                      final shp_status of the block
 *   iters  [B][2]                   update steps in pass 1 and pass 2
 *   resid  [B][2][max_iter + 1]     ||R_k||_F / sqrt(n) at every k
 *   alpha  [B][2][max_iter]         alpha_k used at every update
 *   degree [B][2][max_iter]         degree of g used at every update
 * Entries after a block stops are left untouched. */
typedef struct {
  int32_t* status;
  int32_t* iters;
  float* resid;
  float* alpha;
  int32_t* degree;
} shp_prism_report;

/* Bytes of scratch the call `op` needs for these sizes (0 if none).  For
 * SHP_OP_INV_ROOT / SHP_OP_ALPHA_FIT m is ignored (pass n); for SHP_OP_POLAR
 * and SHP_OP_APPLY m x n is the matrix shape.  Returns 0 on bad arguments. */
size_t shp_workspace_bytes(int op, int64_t m, int64_t n, int64_t batch,
                           const shp_prism_opts* opts);

/* Kronecker-factor statistics, one EMA step ([Shampoo] 2.2-2.3, step 2):
 *   L <- beta L + (1 - beta) G G^T + eps I      (L: m x m, in place)
 *   R <- beta R + (1 - beta) G^T G + eps I      (R: n x n, in place)
 * G: [batch][m][n] fp32; L: [batch][m][m]; R: [batch][n][n].
 * prec: SHP_TF32 or SHP_3XTF32 (the latter needs workspace for the split G).
 * Either L or R may be NULL to skip that factor.  L and R are symmetric by
 * construction and must be on entry: each product is formed on its tiles on
 * and above the diagonal, and the result is written to both triangles. */
int shampoo_gram_ema(const float* G, int64_t m, int64_t n, int64_t batch, float* L, float* R,
                     float beta, float eps, int prec, void* ws, size_t ws_bytes,
                     shp_stream stream);

/* `count` successive EMA steps of the Kronecker factors, one per gradient of
 * the stack G: [count][batch][m][n] fp32 ([Shampoo] 2.3 step 2 applied for
 * t = 1 .. count):
 *   L <- beta L + (1 - beta) G_t G_t^T + eps I,  R <- beta R + (1 - beta) G_t^T G_t + eps I.
 * The result equals `count` calls of shampoo_gram_ema with G_1 .. G_count up
 * to rounding order: every product G_t G_t^T is formed as that call forms it
 * (one batched launch over t and the blocks), then the recurrence is replayed
 * element by element in fp32.  For training loops that hold several
 * gradients at once (accumulated micro-batches, a replayed window).
 * count * batch <= 65535.  Workspace: shp_workspace_bytes(SHP_OP_GRAM_EMA_STEPS,
 * m, n, count * batch, opts with prec) -- the products of both factors (and
 * the split G for SHP_3XTF32).  L, R, prec, NULL factors and errors as in
 * shampoo_gram_ema. */
int shampoo_gram_ema_steps(const float* G, int64_t count, int64_t m, int64_t n, int64_t batch,
                           float* L, float* R, float beta, float eps, int prec, void* ws,
                           size_t ws_bytes, shp_stream stream);

/* Matrix power of a batch of SPD matrices by coupled Newton-Schulz with PRISM
 * alpha ([PRISM] Parte I-II; [Shampoo] 2.3 step 3 and 3.1):
 *   c = ||A||_F, B = (A + A^T) / (2c) (A / c for a symmetric A);
 *   pass 1: Y_0 = B, Z_0 = I, for k = 0, 1, ...:
 *   R_k = I - Z_k Y_k, stop test, alpha_k = argmin_{[lo,hi]} ||r(R_k;alpha) S_k||_F,
 *   g = g_d(R_k; alpha_k), Y_{k+1} = Y_k g, Z_{k+1} = g Z_k.
 *   SHP_POW_SQRT -> sqrt(c) Y;  SHP_POW_INV2 -> Z / sqrt(c);
 *   SHP_POW_INV4 -> pass 2 on Y (same recurrence) and c^(-1/4) Z.
 * A: [batch][n][n] fp32 SPD; X_out: [batch][n][n] fp32 (may not alias A).
 * S: [S_count][n][p] fp32 Gaussian sketches shared by the batch; pass 1
 *   iteration k uses S[k], pass 2 uses S[max_iter + k]; S_count must be
 *   >= max_iter (one pass) or >= 2 * max_iter (SHP_POW_INV4).
 * Output of a block that stopped without converging is its last iterate.
 * prec SHP_OZAKI keeps the iterates in fp64 and forms every product from
 * int8 digit slices (n <= 26000); it is the path for ill-conditioned inputs
 * (condition 1e6 and above), where fp32 storage cannot reach 1e-5.
 * Otherwise, blocks with n <= 64 and p <= 16 run on chip, one CTA per block
 * with fp32 products for either precision; they need a 256-byte workspace
 * and allow batch > 65535. */
int matfn_inv_root(const float* A, int64_t n, int64_t batch, int power,
                   const shp_prism_opts* opts, const float* S, int64_t S_count, float* X_out,
                   const shp_prism_report* report, void* ws, size_t ws_bytes, shp_stream stream);

/* Polar factor U V^T of a batch of m x n matrices (the Muon orthogonalisation;
 * [PRISM] Parte I with R_k = I - X_k^T X_k):
 *   X_0 = G / ||G||_F; R_k = I - X_k^T X_k; stop test; alpha_k from S[k];
 *   X_{k+1} = X_k g_d(R_k; alpha_k).  A wide G (m < n) is handled as G^T.
 * G, X_out: [batch][m][n], bf16 (storage = SHP_BF16; the iterate is kept in
 *   bf16 with fp32 accumulation) or fp32 (storage = SHP_TF32 / SHP_3XTF32).
 * S: [S_count][min(m,n)][p] fp32, S_count >= max_iter.
 * fp32 inputs with m, n <= 64 and p <= 16 run on chip (as matfn_inv_root). */
int matfn_polar(const void* G, int storage, int64_t m, int64_t n, int64_t batch,
                const shp_prism_opts* opts, const float* S, int64_t S_count, void* X_out,
                const shp_prism_report* report, void* ws, size_t ws_bytes, shp_stream stream);

/* Polar factors of a batch of small blocks of different shapes, each on chip
 * (one CTA per block, fp32 products): block b is the row-major m_b x n_b
 * matrix at G + offsets[b] and its factor goes to X_out + offsets[b].
 *   dims    [batch][2] int32 (m_b, n_b), each in 4..64 and a multiple of 4
 *   offsets [batch] int64 element offsets of the blocks in G and X_out
 *   S       [S_count][64][p] fp32 (p <= 16); block b uses the first
 *           min(m_b, n_b) rows of slice k at iteration k
 * dims and offsets are DEVICE arrays, read by the kernel: a block whose
 * dims are out of range gets report.status SHP_EINVAL and is left untouched.
 * The batched polar decomposition of variable-size diagonal blocks (e.g. the
 * groups of close eigenvalues of a block-rotation optimizer). */
int matfn_polar_varsize(const float* G, const int32_t* dims, const int64_t* offsets,
                        int64_t batch, const shp_prism_opts* opts, const float* S,
                        int64_t S_count, float* X_out, const shp_prism_report* report,
                        shp_stream stream);

/* Matrix sign function of a batch of symmetric n x n matrices ([PRISM] Parte I:
 * the residual of sign functions is R_k = I - X_k^2):
 *   X_0 = A / ||A||_F; R_k = I - X_k X_k; stop test; alpha_k from S[k];
 *   X_{k+1} = X_k g_d(R_k; alpha_k)  ->  sign(A) = Q sign(Lambda) Q^T.
 * A, X_out: [batch][n][n], bf16 or fp32 storage as in matfn_polar (A must be
 * symmetric and nonsingular; for an SPD A the result is I).  Workspace:
 * shp_workspace_bytes(SHP_OP_POLAR, n, n, batch, opts with prec = storage). */
int matfn_sign(const void* A, int storage, int64_t n, int64_t batch, const shp_prism_opts* opts,
               const float* S, int64_t S_count, void* X_out, const shp_prism_report* report,
               void* ws, size_t ws_bytes, shp_stream stream);

/* One sketched alpha fit ([PRISM] Parte II.1-II.2) on given residuals:
 *   V_0 = S, V_j = R V_{j-1} (j <= 2d+1), M_ij = <V_i, V_j>_F (i, j = d..2d+1),
 *   J(alpha) = sum_ij r_i(alpha) r_j(alpha) M_ij,  alpha* = argmin_{[lo,hi]} J.
 * R: [batch][n][n] fp32 (n a multiple of 4); S: [n][p] fp32 shared by the batch;
 * alpha_out: [batch] fp32; J_coef_out: [batch][5] fp64 coefficients of
 * alpha^0..alpha^4, or NULL.  The passes stream R through shared memory by TMA
 * when V fits there (n * p up to about 16K), else through registers; their
 * pipeline waits are bounded, and a block whose wait runs out (which only a
 * device fault can cause) gets alpha_out = NaN and NaN coefficients. */
int prism_alpha_fit(const float* R, int64_t n, int64_t batch, const float* S, int p, int d,
                    float lo, float hi, float* alpha_out, double* J_coef_out, void* ws,
                    size_t ws_bytes, shp_stream stream);

/* Preconditioned update ([Shampoo] 2.3 step 4; 6.3):
 *   W <- W - lr * Lroot * G * Rroot        (in place)
 * W, G: [batch][m][n]; Lroot: [batch][m][m]; Rroot: [batch][n][n]; fp32.
 * prec: SHP_TF32 or SHP_3XTF32. */
int shampoo_apply(float* W, const float* G, const float* Lroot, const float* Rroot, int64_t m,
                  int64_t n, int64_t batch, float lr, int prec, void* ws, size_t ws_bytes,
                  shp_stream stream);

/* Preconditioned update with the variants of [Shampoo] 5.1-5.2, P = Lroot G Rroot:
 *   adaptive step (gnorm2_acc non-NULL): acc[b] += ||G[b]||_F^2 and
 *     eta_b = lr / sqrt(1 + acc[b]); otherwise eta_b = lr;
 *   momentum (M non-NULL), the recursion as the page prints it:
 *     M <- gamma M + P,  W <- W - eta_b M;  otherwise W <- W - eta_b P.
 * W, G, M: [batch][m][n] fp32 (W and M updated in place; M 16-byte aligned);
 * gnorm2_acc: [batch] fp64 running sums, updated in place; Lroot, Rroot as in
 * shampoo_apply.  With M = gnorm2_acc = NULL this is shampoo_apply.
 * Workspace: shp_workspace_bytes(SHP_OP_APPLY, m, n, batch, opts). */
int shampoo_apply_ex(float* W, float* M, double* gnorm2_acc, const float* G, const float* Lroot,
                     const float* Rroot, int64_t m, int64_t n, int64_t batch, float lr,
                     float gamma, int prec, void* ws, size_t ws_bytes, shp_stream stream);

/* ---- Utilities (no counterpart on the pages; building blocks of the calls
 * above, exposed for measurement and tests). ---- */

/* C[b] = A[b] * B[b] on the tensor cores, the product every call above is
 * built from.  Logical shapes: A is M x K, B is K x N, C is M x N fp32
 * (bf16 for SHP_BF16), all row-major with no padding.  a_trans = 1 reads A
 * from an K x M row-major buffer (A^T stored), b_trans = 1 reads B from an
 * N x K row-major buffer.  prec: SHP_TF32 (fp32 inputs), SHP_BF16 (bf16
 * inputs), or SHP_3XTF32 with A_lo/B_lo the low parts from shp_split_tf32
 * (A/B then hold the high parts); A_lo/B_lo are ignored otherwise.
 * One kernel launch; no workspace. */
int shp_matmul(const void* A, const float* A_lo, int a_trans, const void* B, const float* B_lo,
               int b_trans, void* C, int64_t M, int64_t N, int64_t K, int64_t batch, int prec,
               shp_stream stream);

/* C[b] = A[b] * B[b] in fp64-grade arithmetic on the int8 tensor cores (the
 * Ozaki scheme: Ozaki, Ogita, Oishi, Rump, Numer. Algorithms 2012; the
 * integer-unit form of Ootomo, Ozaki, Yokota, IJHPCA 2024).  Each row of A
 * and each column of B is scaled by a power of two and written as five
 * signed 8-bit digits; the 15 digit products of weight >= 2^-32 are
 * accumulated exactly in int32 and combined in fp64, so |C - AB|_ij is about
 * K 2^-40 max_k|A_ik| max_k|B_kj| (or below).  A: [batch][M][K], B:
 * [batch][K][N], C: [batch][M][N], fp64 row-major, N even, K <= 26000; a NaN
 * or Inf in a row of A or a column of B makes that row/column of C NaN.
 * Workspace: shp_matmul_f64_workspace_bytes(M, N, K, batch). */
size_t shp_matmul_f64_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t batch);
int shp_matmul_f64(const double* A, const double* B, double* C, int64_t M, int64_t N, int64_t K,
                   int64_t batch, void* ws, size_t ws_bytes, shp_stream stream);

/* shp_matmul_f64 for an operand that does not change between calls: with
 * SHP_MATMUL_REUSE_A (SHP_MATMUL_REUSE_B) the digit slices of A (B) are not
 * formed again but taken from `ws` as the previous call with the same A (B),
 * sizes and workspace left them (e.g. applying one fixed matrix to many
 * right-hand sides); the product is then a single GEMM launch.  Reusing
 * slices of an operand whose values changed gives the product with the old
 * values.  With SHP_MATMUL_ACCUMULATE the product is added to C
 * (C <- C + A B, in place).  flags = 0 is shp_matmul_f64. */
#define SHP_MATMUL_REUSE_A 1
#define SHP_MATMUL_REUSE_B 2
#define SHP_MATMUL_ACCUMULATE 4
int shp_matmul_f64_ex(const double* A, const double* B, double* C, int64_t M, int64_t N,
                      int64_t K, int64_t batch, int flags, void* ws, size_t ws_bytes,
                      shp_stream stream);

/* hi = TF32(x) (round to nearest), lo = TF32(x - hi), for `count` floats. */
int shp_split_tf32(const float* X, int64_t count, float* hi, float* lo, shp_stream stream);

/* Number of kernels this library has launched in the process so far
 * (host-side counter, all threads and devices). */
uint64_t shp_kernel_launches(void);

/* ---- Alpha fit with no caller workspace (no counterpart on the pages). ----
 *
 * Same result as prism_alpha_fit, but the sketch vectors live in a fixed
 * device array inside the library instead of a caller workspace, so the
 * caller allocates nothing.  It is meant for callers that cannot allocate in
 * the middle of their work: an optimizer step running under a framework whose
 * caching allocator owns the free device memory (a raw cudaMalloc can fail
 * there, and cudaFree synchronises the whole device), or a latency-bound loop
 * that must not take the implicit synchronisation of cudaMalloc/cudaFree.
 *
 *   Limit: ((2d+2) * n * p + 1) * batch * 4 bytes <= SHP_NOALLOC_SCRATCH_BYTES
 *          (e.g. n = 1024, p = 8, d = 2: batch <= 21); larger sizes return
 *          SHP_EUNSUPPORTED before any launch.
 *   Memory: every GPU that loads the library holds SHP_NOALLOC_SCRATCH_BYTES
 *          until the process exits.
 *   Set-up: the first call on a device looks up the array's device address
 *          (cudaGetSymbolAddress) with that device current; make that first
 *          call before any stream capture.
 *   Sharing: all calls use the same array, which keeps the previous call's
 *          contents (the sketch vectors need no clearing; the per-block
 *          timeout flags stored after them are cleared by every call); calls
 *          that overlap on the GPU race on it, so serialise them (one stream,
 *          one thread).
 * Arguments, layouts, the NaN alpha of a timed-out block and the other return
 * codes are those of prism_alpha_fit. */
#define SHP_NOALLOC_SCRATCH_BYTES (4u << 20)
int prism_alpha_fit_noalloc(const float* R, int64_t n, int64_t batch, const float* S, int p,
                            int d, float lo, float hi, float* alpha_out, double* J_coef_out,
                            shp_stream stream);

/* ---- Self-test of the bounded waits (no counterpart on the pages). ----
 * Every pipeline wait inside the kernels is bounded: a wait that runs out
 * records SHP_ETIMEOUT, the other roles of the CTA give up at their next
 * wait, the copies and tensor-core operations already issued are waited for,
 * tensor memory is freed, and the stream stays usable.  This call makes one
 * such wait run out on purpose, by pointing it at a barrier nothing completes
 * (limit about 10 ms), in one small launch of the kernel `which` selects:
 *   SHP_SELFTEST_GEMM    persistent CTA-pair GEMM: the producer's first wait
 *                        (nothing issued yet)
 *   SHP_SELFTEST_OZAKI   Ozaki-scheme GEMM: the same wait
 *   SHP_SELFTEST_SKETCH  TMA sketch: the consumers' first V hand-over, with
 *                        the producer's copies in flight (they are drained),
 *                        in the first pass of a whole alpha fit (d = 1)
 *   SHP_SELFTEST_SKETCH_ALPHA  the last sketch pass with the alpha fit folded
 *                        in (as inside the matrix-function loops): the same
 *                        hand-over in that pass; no warp completes the block,
 *                        so no alpha is solved
 *   SHP_SELFTEST_SKETCH_CHAIN  the few-block sketch (every pass of an
 *                        iteration and the fit in one cooperative launch, as
 *                        the loops use it when the batch's R fits in shared
 *                        memory): its first grid barrier, which CTA 0 never
 *                        reaches; no alpha is solved
 * status: one device int32, set to SHP_ETIMEOUT by the kernel (cleared
 * first).  alpha_out: one device float (may be NULL), for the sketch cases
 * the fit's alpha, which must come out NaN (no fit on incomplete vectors; the
 * folded case leaves the NaN it starts from, as the stop test sets it).
 * ws: at least SHP_SELFTEST_WS_BYTES of device scratch, 256-byte aligned
 * (zeroed by the call).  Returns SHP_OK once launched. */
#define SHP_SELFTEST_GEMM 0
#define SHP_SELFTEST_OZAKI 1
#define SHP_SELFTEST_SKETCH 2
#define SHP_SELFTEST_SKETCH_ALPHA 3
#define SHP_SELFTEST_SKETCH_CHAIN 4
#define SHP_SELFTEST_WS_BYTES (4u << 20)
int shp_selftest_bounded_wait(int which, int32_t* status, float* alpha_out, void* ws,
                              size_t ws_bytes, shp_stream stream);

/* Human-readable name of a status code (static storage). */
const char* shp_status_string(int status);

/* Name of the CUDA error (e.g. "cudaErrorInvalidValue") behind the latest
 * SHP_ECUDA returned on this host thread, or "none" (static storage). */
const char* shp_last_cuda_error(void);

/* Library version, e.g. "0.1.0" (static storage). */
const char* shp_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SHAMPOO_PRISM_H */
