// C ABI of the library (declared in include/shampoo_prism.h): argument
// validation, workspace carving and the launch sequence of each operation.
// Nothing here touches matrix data on the host; every step runs in the
// kernels of gemm_tc.cu, sketch_alpha.cu and elementwise.cu.
#include <math.h>
#include <stdlib.h>
#include <stdint.h>
#include <string.h>

#include "internal.h"
#include "shampoo_prism.h"

#include <mutex>
#include <vector>

using namespace shp;

namespace {

constexpr size_t kAlign = 256;

// Carves aligned sub-buffers out of the caller's workspace.  With a null base
// it only measures.
struct Arena {
  uint8_t* base;
  size_t used = 0;
  explicit Arena(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <class T>
  T* take(size_t count) {
    used = (used + kAlign - 1) & ~(kAlign - 1);
    T* p = base != nullptr ? reinterpret_cast<T*>(base + used) : nullptr;
    used += count * sizeof(T);
    return p;
  }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool opts_ok(const shp_prism_opts* o) {
  if (o == nullptr) return false;
  if (o->d != 1 && o->d != 2) return false;
  if (o->p < 1 || o->p > 32) return false;
  if (!(isfinite(o->lo) && isfinite(o->hi)) || o->lo > o->hi) return false;
  if (!(o->tol >= 0.f)) return false;
  if (o->max_iter < 1 || o->max_iter > 256) return false;
  if (o->prec != SHP_TF32 && o->prec != SHP_3XTF32 && o->prec != SHP_BF16 &&
      o->prec != SHP_OZAKI)
    return false;
  if (!(o->stall_below >= 0.f) || !(o->stall_ratio >= 0.f)) return false;
  if (o->adaptive_degree != 0 &&
      (o->d != 2 || o->fixed_alpha != 0 || !(o->raise_above >= 0.f)))
    return false;
  if (o->host_loop != 0 && o->host_loop != 1) return false;
  return true;
}

Ctl carve_ctl(Arena& a, int64_t batch) {
  Ctl c;
  c.bs = a.take<BlockState>(batch);
  c.active = a.take<int>(batch);
  c.deg = a.take<int>(batch);
  c.act1 = a.take<int>(batch);
  c.act2 = a.take<int>(batch);
  c.dnorm = a.take<double>(batch);
  c.tmo = a.take<int>(batch);
  c.alpha = a.take<float>(batch);
  c.it = a.take<int>(1);
  c.flag = a.take<int>(1);
  c.gram = a.take<double>(batch * 15);
  c.gcnt = a.take<int>(batch);
  c.gbar = a.take<unsigned>(4);
  c.gpart = a.take<double>(static_cast<size_t>(kChainMaxCtas) * 15);
  return c;
}

// Iterate buffers: two ping-pong slots for the iterates (Y and Z, or X), and
// R and g.  `lo` parts exist only in split (3xTF32) mode.
struct Bufs {
  float* Yhi[2];
  float* Ylo[2];
  float* Zhi[2];
  float* Zlo[2];
  float* Rhi;
  float* Rlo;
  float* Rs;  // plain fp32 R read by the sketch passes (= Rhi in TF32 mode)
  float* ghi;
  float* glo;
  float* V;
  Ctl ctl;
};

Bufs carve_inv_root(Arena& a, int64_t n, int64_t batch, const shp_prism_opts* o) {
  Bufs b;
  const bool split = o->prec == SHP_3XTF32;
  const size_t nn = static_cast<size_t>(n) * n * batch;
  for (int s = 0; s < 2; ++s) {
    b.Yhi[s] = a.take<float>(nn);
    b.Ylo[s] = split ? a.take<float>(nn) : nullptr;
    b.Zhi[s] = a.take<float>(nn);
    b.Zlo[s] = split ? a.take<float>(nn) : nullptr;
  }
  b.Rhi = a.take<float>(nn);
  b.Rlo = split ? a.take<float>(nn) : nullptr;
  b.Rs = split ? a.take<float>(nn) : b.Rhi;
  b.ghi = a.take<float>(nn);
  b.glo = split ? a.take<float>(nn) : nullptr;
  b.V = a.take<float>(static_cast<size_t>(2 * o->d + 2) * n * o->p * batch);
  b.ctl = carve_ctl(a, batch);
  return b;
}

// fp64 iterates (updated in place: every product reads the digit slices,
// and the epilogue reads and writes an element of Y or Z only at its own
// position), their slices, a plain fp32 R for the sketch.
struct OzBufs {
  double* Y;
  double* Z;
  double* R;
  double* D;  // Delta = g - I
  float* Rs;
  OzSlices sY, sZ, sR, sD;
  unsigned* maxbuf;   // row and column maxima keys of the matrix being sliced
  unsigned* maxbuf2;  // ... of Z_1 = I + Delta, written beside Delta
  float* V;
  Ctl ctl;
};

OzSlices carve_slices(Arena& a, int64_t rows, int64_t cols, int64_t batch, bool want_rows,
                      bool want_cols) {
  OzSlices s{};
  s.rows = want_rows ? a.take<int8_t>(oz_slices_bytes(rows, cols, batch)) : nullptr;
  s.cols = want_cols ? a.take<int8_t>(oz_slices_bytes(cols, rows, batch)) : nullptr;
  s.rscale = want_rows ? a.take<double>(static_cast<size_t>(rows) * batch) : nullptr;
  s.cscale = want_cols ? a.take<double>(static_cast<size_t>(cols) * batch) : nullptr;
  return s;
}

OzBufs carve_inv_root_oz(Arena& a, int64_t n, int64_t batch, const shp_prism_opts* o) {
  OzBufs b;
  const size_t nn = static_cast<size_t>(n) * n * batch;
  b.Y = a.take<double>(nn);
  b.Z = a.take<double>(nn);
  b.R = a.take<double>(nn);
  b.D = a.take<double>(nn);
  b.Rs = a.take<float>(nn);
  b.sY = carve_slices(a, n, n, batch, true, true);
  b.sZ = carve_slices(a, n, n, batch, true, true);
  b.sR = carve_slices(a, n, n, batch, true, true);
  b.sD = carve_slices(a, n, n, batch, true, true);
  b.maxbuf = a.take<unsigned>(static_cast<size_t>(2 * n) * batch);
  b.maxbuf2 = a.take<unsigned>(static_cast<size_t>(2 * n) * batch);
  b.V = a.take<float>(static_cast<size_t>(2 * o->d + 2) * n * o->p * batch);
  b.ctl = carve_ctl(a, batch);
  return b;
}

struct PolarBufs {
  void* Xhi[2];
  float* Xlo[2];
  float* Rhi;
  float* Rlo;
  float* Rs;  // plain fp32 R read by the sketch passes
  uint16_t* Rb;  // bf16 copy of R, the operands of R R (bf16 storage)
  void* ghi;
  float* glo;
  float* V;
  Ctl ctl;
};

PolarBufs carve_polar(Arena& a, int64_t m, int64_t n, int64_t batch, int storage,
                      const shp_prism_opts* o) {
  PolarBufs b;
  const int64_t k = m < n ? m : n;
  const bool split = storage == SHP_3XTF32;
  const bool bf = storage == SHP_BF16;
  const size_t mn = static_cast<size_t>(m) * n * batch, kk = static_cast<size_t>(k) * k * batch;
  for (int s = 0; s < 2; ++s) {
    b.Xhi[s] = bf ? static_cast<void*>(a.take<uint16_t>(mn)) : static_cast<void*>(a.take<float>(mn));
    b.Xlo[s] = split ? a.take<float>(mn) : nullptr;
  }
  b.Rhi = a.take<float>(kk);
  b.Rlo = split ? a.take<float>(kk) : nullptr;
  b.Rs = split ? a.take<float>(kk) : b.Rhi;
  b.Rb = bf ? a.take<uint16_t>(kk) : nullptr;
  b.ghi = bf ? static_cast<void*>(a.take<uint16_t>(kk)) : static_cast<void*>(a.take<float>(kk));
  b.glo = split ? a.take<float>(kk) : nullptr;
  b.V = a.take<float>(static_cast<size_t>(2 * o->d + 2) * k * o->p * batch);
  b.ctl = carve_ctl(a, batch);
  return b;
}

EpiParams epi(int kind, int fmt, void* hi, float* lo, int64_t ldo, int64_t bso, int M, int N,
              const Ctl* ctl) {
  EpiParams e;
  memset(&e, 0, sizeof(e));
  e.kind = kind;
  e.out_fmt = fmt;
  e.out_hi = hi;
  e.out_lo = lo;
  e.ldo = ldo;
  e.bso = bso;
  e.s0 = 1.f;
  e.M = M;
  e.N = N;
  if (ctl != nullptr) {
    e.active = ctl->active;
    e.status = ctl->tmo;
    e.alpha = ctl->alpha;
    e.norm2 = &ctl->bs[0].norm2;
    e.norm2_stride = static_cast<int>(sizeof(BlockState) / sizeof(float));
  }
  return e;
}

Operand op(const void* hi, const float* lo, bool mn, int64_t ld, int64_t bs) {
  Operand o;
  o.hi = hi;
  o.lo = lo;
  o.mn = mn;
  o.ld = ld;
  o.bstride = bs;
  return o;
}

// The CUDA error behind this host thread's latest SHP_ECUDA.
thread_local cudaError_t g_last_cuda = cudaSuccess;

#define CK(x)                           \
  do {                                  \
    const cudaError_t ck_e_ = (x);      \
    if (ck_e_ != cudaSuccess) {         \
      g_last_cuda = ck_e_;              \
      return SHP_ECUDA;                 \
    }                                   \
  } while (0)

// The sketch passes and the alpha solve of iteration k = *ctl.it:
// V_1 = R S[k] (S_pass is the pass's first slice), V_j = R V_{j-1}
// (j <= 2d+1), then the Gram, the quartic and its argmin.
int sketch_and_alpha(const float* Rs, int64_t n, int batch, const float* S_pass, float* V,
                     const shp_prism_opts* o, const Ctl& ctl, float* rep_alpha,
                     int64_t rep_stride, int rep_slot_base, cudaStream_t st,
                     int* rep_degree = nullptr) {
  const int64_t np = n * o->p, nn = n * n;
  const int64_t vbs = static_cast<int64_t>(2 * o->d + 2) * np;
  // a fitted alpha at fixed degree is solved inside the last pass (no alpha launch)
  const bool fuse = !o->fixed_alpha && !o->adaptive_degree && ctl.gram != nullptr;
  bool chained = false;
  if (!o->fixed_alpha) {
    // few blocks: every pass (and the fit) in one cooperative launch
    CK(sketch_chain(Rs, n, nn, S_pass, np, ctl.it, V, o->p, o->d, batch, ctl.active, ctl.tmo,
                    ctl.gbar, o->lo, o->hi, ctl.alpha, rep_alpha, rep_stride, rep_slot_base,
                    fuse ? ctl.gpart : nullptr, fuse ? ctl.gcnt : nullptr, st, &chained));
    if (chained && fuse) return SHP_OK;
  }
  if (!o->fixed_alpha && !chained) {
    CK(sketch_pass(Rs, nullptr, n, nn, S_pass, 0, V + np, vbs, o->p, batch, ctl.active, ctl.it,
                   np, st, ctl.tmo));
    const int last = 2 * o->d + 1;
    for (int j = 2; j <= last; ++j) {
      if (fuse && j == last) {
        bool fused = false;
        CK(sketch_pass_alpha(Rs, n, nn, V + (j - 1) * np, vbs, V + j * np, vbs, o->p, batch,
                             ctl.active, st, ctl.tmo, V, o->d, o->lo, o->hi, ctl.alpha,
                             rep_alpha, rep_stride, rep_slot_base, ctl.it, ctl.gram, ctl.gcnt,
                             &fused));
        if (fused) return SHP_OK;
      } else {
        CK(sketch_pass(Rs, nullptr, n, nn, V + (j - 1) * np, vbs, V + j * np, vbs, o->p, batch,
                       ctl.active, nullptr, 0, st, ctl.tmo));
      }
    }
  }
  AdaptiveDeg ad{o->adaptive_degree, o->raise_above, ctl.deg, ctl.act1, ctl.act2, rep_degree};
  CK(alpha_solve(V, n, o->p, o->d, batch, o->lo, o->hi, o->fixed_alpha, ctl.active, ctl.alpha,
                 nullptr, rep_alpha, rep_stride, rep_slot_base, ctl.it, st, &ad));
  return SHP_OK;
}

// ------------------------------------------------------------------------
// Device-side iteration loop.  Each Newton-Schulz pass is recorded into a CUDA
// graph: the k = 0 step, then a conditional WHILE node whose body runs two
// steps (odd k on ping-pong slot 1, then even k on slot 0).  After every step
// a one-CTA kernel advances the device iteration counter; the one after the
// even step sets the condition to "some block still active".  Blocks stop
// independently in k_control, and every kernel of a step returns at once for
// a stopped block, so the even step of the body pass in which the last block
// stopped is a few empty launches (an IF node around it measured costlier
// than that).  No host synchronisation.  Graphs are cached by the call's
// pointers and sizes.

struct CallKey {
  int op, device, power, storage;
  const void* a;
  void* x;
  const void* s;
  int64_t s_count, m, n, batch;
  shp_prism_opts o;
  void* ws;
  size_t ws_bytes;
  const void* rep[5];
};

struct CachedGraph {
  CallKey key;
  cudaGraph_t graph;
  cudaGraphExec_t exec;
};

std::mutex g_graph_mu;
std::vector<CachedGraph> g_graphs;
constexpr size_t kGraphCacheMax = 16;
constexpr int kMaxDev = 64;
cudaStream_t g_cap[kMaxDev][2] = {};  // the pass and its WHILE body

// Adds a conditional node after the current capture frontier of `st`, makes
// it the new frontier and returns its body graph.
cudaError_t add_conditional(cudaStream_t st, cudaGraphConditionalHandle h,
                            cudaGraphConditionalNodeType type, cudaGraph_t* body) {
  cudaStreamCaptureStatus cs;
  const cudaGraphNode_t* deps = nullptr;
  size_t nd = 0;
  cudaGraph_t g = nullptr;
  cudaError_t e = cudaStreamGetCaptureInfo(st, &cs, nullptr, &g, &deps, &nd);
  if (e != cudaSuccess) return e;
  if (cs != cudaStreamCaptureStatusActive) return cudaErrorStreamCaptureInvalidated;
  cudaGraphNodeParams p = {cudaGraphNodeTypeConditional};
  p.conditional.handle = h;
  p.conditional.type = type;
  p.conditional.size = 1;
  cudaGraphNode_t node;
  e = cudaGraphAddNode(&node, g, deps, nd, &p);
  if (e != cudaSuccess) return e;
  *body = p.conditional.phGraph_out[0];
  return cudaStreamUpdateCaptureDependencies(st, &node, 1, cudaStreamSetCaptureDependencies);
}

// iter(cur, first, stream) launches one step on ping-pong slot `cur`.
// With g == nullptr the same steps run from a host loop that reads the
// condition back after every step (opts.host_loop = 1, for profilers and
// launch tracers that do not look inside conditional graphs).
template <class Iter>
int record_loop(cudaStream_t const* cs, cudaGraph_t g, const Ctl& ctl, int batch, int max_iter,
                Iter iter) {
  if (g == nullptr) {
    int r = iter(0, true, cs[0]);
    if (r != SHP_OK) return r;
    CK(loop_step(ctl, batch, 1, max_iter, 0, cs[0]));
    for (int k = 1;; ++k) {
      int flag = 0;
      CK(cudaMemcpyAsync(&flag, ctl.flag, sizeof(int), cudaMemcpyDeviceToHost, cs[0]));
      CK(cudaStreamSynchronize(cs[0]));
      if (flag == 0) break;
      r = iter(k & 1, false, cs[0]);
      if (r != SHP_OK) return r;
      CK(loop_step(ctl, batch, 1, max_iter, 0, cs[0]));
    }
    return SHP_OK;
  }
  const cudaStreamCaptureMode mode = cudaStreamCaptureModeRelaxed;
  int r = iter(0, true, cs[0]);
  if (r != SHP_OK) return r;
  cudaGraphConditionalHandle hw;
  CK(cudaGraphConditionalHandleCreate(&hw, g, 0, cudaGraphCondAssignDefault));
  CK(loop_step(ctl, batch, 1, max_iter, hw, cs[0]));
  cudaGraph_t body = nullptr;
  CK(add_conditional(cs[0], hw, cudaGraphCondTypeWhile, &body));
  CK(cudaStreamBeginCaptureToGraph(cs[1], body, nullptr, nullptr, 0, mode));
  // two steps per pass of the body, the second without a conditional of its
  // own: an IF node costs more than the step it would skip, which (all blocks
  // stopped) is a few launches that return at once
  r = iter(1, false, cs[1]);
  if (r == SHP_OK && loop_step(ctl, batch, 1, max_iter, 0, cs[1]) != cudaSuccess) r = SHP_ECUDA;
  if (r == SHP_OK) r = iter(0, false, cs[1]);
  if (r == SHP_OK && loop_step(ctl, batch, 1, max_iter, hw, cs[1]) != cudaSuccess) r = SHP_ECUDA;
  cudaGraph_t g1 = nullptr;
  if (cudaStreamEndCapture(cs[1], &g1) != cudaSuccess && r == SHP_OK) r = SHP_ECUDA;
  return r;
}

// Finds or records (rec(capture streams, graph)) the graph of `key` and
// launches it on `user`.
template <class Rec>
int run_graph(CallKey key, Rec rec, cudaStream_t user) {
  CK(cudaGetDevice(&key.device));
  if (key.device < 0 || key.device >= kMaxDev) return SHP_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_graph_mu);
  for (auto& c : g_graphs)
    if (memcmp(&c.key, &key, sizeof(key)) == 0) {
      CK(cudaGraphLaunch(c.exec, user));
      return SHP_OK;
    }
  cudaStream_t* cs = g_cap[key.device];
  for (int i = 0; i < 2; ++i)
    if (cs[i] == nullptr) CK(cudaStreamCreateWithFlags(&cs[i], cudaStreamNonBlocking));
  cudaGraph_t g = nullptr;
  CK(cudaGraphCreate(&g, 0));
  if (cudaStreamBeginCaptureToGraph(cs[0], g, nullptr, nullptr, 0,
                                    cudaStreamCaptureModeRelaxed) != cudaSuccess) {
    cudaGraphDestroy(g);
    return SHP_ECUDA;
  }
  int r = rec(static_cast<cudaStream_t const*>(cs), g);
  cudaGraph_t g0 = nullptr;
  if (cudaStreamEndCapture(cs[0], &g0) != cudaSuccess && r == SHP_OK) r = SHP_ECUDA;
  cudaGraphExec_t exec = nullptr;
  if (r == SHP_OK && cudaGraphInstantiate(&exec, g, 0) != cudaSuccess) r = SHP_ECUDA;
  if (r != SHP_OK) {
    cudaGetLastError();
    cudaGraphDestroy(g);
    return r;
  }
  if (g_graphs.size() >= kGraphCacheMax) {
    cudaGraphExecDestroy(g_graphs.front().exec);
    cudaGraphDestroy(g_graphs.front().graph);
    g_graphs.erase(g_graphs.begin());
  }
  g_graphs.push_back(CachedGraph{key, g, exec});
  CK(cudaGraphLaunch(exec, user));
  return SHP_OK;
}

// Runs `rec` on the user's stream with host-driven loops (opts.host_loop),
// else through the graph cache.
template <class Rec>
int dispatch(const CallKey& key, Rec rec, cudaStream_t user) {
  if (key.o.host_loop != 0) {
    cudaStream_t cs[3] = {user, user, user};
    return rec(static_cast<cudaStream_t const*>(cs), static_cast<cudaGraph_t>(nullptr));
  }
  return run_graph(key, rec, user);
}

CallKey make_key(int opk) {
  CallKey k;
  memset(&k, 0, sizeof(k));
  k.op = opk;
  return k;
}

}  // namespace

extern "C" {

const char* shp_version(void) { return "0.1.0"; }

uint64_t shp_kernel_launches(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return 0;
  return kernel_runs_gemm() + kernel_runs_sketch() + kernel_runs_elementwise() +
         kernel_runs_small() + kernel_runs_ozaki();
}

int shp_split_tf32(const float* X, int64_t count, float* hi, float* lo, shp_stream stream) {
  if (!X || !hi || !lo || count < 0) return SHP_EINVAL;
  CK(split_copy(X, count, hi, lo, static_cast<cudaStream_t>(stream)));
  return SHP_OK;
}

int shp_matmul(const void* A, const float* A_lo, int a_trans, const void* B, const float* B_lo,
               int b_trans, void* C, int64_t M, int64_t N, int64_t K, int64_t batch, int prec,
               shp_stream stream) {
  if (!A || !B || !C || M <= 0 || N <= 0 || K <= 0 || batch <= 0) return SHP_EINVAL;
  if (prec != SHP_TF32 && prec != SHP_3XTF32 && prec != SHP_BF16) return SHP_EINVAL;
  if (prec == SHP_3XTF32 && (!A_lo || !B_lo)) return SHP_EINVAL;
  const int64_t q = prec == SHP_BF16 ? 8 : 4;  // elements per 16 bytes
  // every memory row (M, N or K long, per the transposes) must be 16-byte aligned
  if ((a_trans ? M : K) % q || (b_trans ? K : N) % q || N % q) return SHP_EINVAL;
  if (!aligned16(A) || !aligned16(B) || !aligned16(C)) return SHP_EINVAL;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX || batch > 65535) return SHP_EUNSUPPORTED;
  const int mode = prec == SHP_BF16 ? MODE_BF16 : (prec == SHP_3XTF32 ? MODE_3XTF32 : MODE_TF32);
  const bool split = prec == SHP_3XTF32;
  // A^T stored (K x M) is the MN-major view of A; B stored (K x N) is MN-major,
  // B^T stored (N x K) is K-major.
  Operand a = op(A, split ? A_lo : nullptr, a_trans != 0, a_trans ? M : K, M * K);
  Operand b = op(B, split ? B_lo : nullptr, b_trans == 0, b_trans ? K : N, K * N);
  EpiParams e = epi(EPI_STORE, prec == SHP_BF16 ? OUT_BF16 : OUT_F32, C, nullptr, N, M * N,
                    static_cast<int>(M), static_cast<int>(N), nullptr);
  CK(gemm_tc(mode, a, b, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K),
             static_cast<int>(batch), e, static_cast<cudaStream_t>(stream)));
  return SHP_OK;
}

const char* shp_last_cuda_error(void) {
  if (g_last_cuda == cudaSuccess) return "none";
  return cudaGetErrorName(g_last_cuda);
}

const char* shp_status_string(int s) {
  switch (s) {
    case SHP_OK: return "ok";
    case SHP_EINVAL: return "invalid argument";
    case SHP_EUNSUPPORTED: return "unsupported";
    case SHP_ECUDA: return "CUDA runtime error";
    case SHP_ENOCONV: return "not converged within max_iter";
    case SHP_ESTALL: return "residual stalled";
    case SHP_ENONFINITE: return "non-finite residual";
    case SHP_ETIMEOUT: return "bounded wait timed out";
    default: return "unknown status";
  }
}

size_t shp_workspace_bytes(int opk, int64_t m, int64_t n, int64_t batch,
                           const shp_prism_opts* o) {
  if (n <= 0 || batch <= 0) return 0;
  Arena a(nullptr);
  switch (opk) {
    case SHP_OP_INV_ROOT:
      if (!opts_ok(o)) return 0;
      if (o->prec == SHP_OZAKI) {
        carve_inv_root_oz(a, n, batch, o);
        break;
      }
      if (small_block_ok(n, n, o->p)) return kAlign;  // on-chip path: no scratch
      carve_inv_root(a, n, batch, o);
      break;

    case SHP_OP_POLAR:
      if (!opts_ok(o) || m <= 0) return 0;
      if (o->prec != SHP_BF16 && small_block_ok(m, n, o->p)) return kAlign;
      carve_polar(a, m, n, batch, o->prec, o);
      break;
    case SHP_OP_ALPHA_FIT: {
      const int d = o != nullptr ? o->d : 2, p = o != nullptr ? o->p : 32;
      a.take<float>(static_cast<size_t>(2 * d + 2) * n * p * batch);
      a.take<int>(static_cast<size_t>(batch));  // timeout flags of the sketch passes
      break;
    }
    case SHP_OP_APPLY: {
      // per-block norms and steps; T = Lroot G (m x n); split mode also
      // needs hi/lo copies of the inputs
      const int prec = o != nullptr ? o->prec : SHP_3XTF32;
      const size_t mn = static_cast<size_t>(m) * n * batch;
      a.take<double>(static_cast<size_t>(batch));
      a.take<float>(static_cast<size_t>(batch));
      a.take<float>(mn);
      if (prec == SHP_3XTF32) {
        a.take<float>(mn);
        a.take<float>(static_cast<size_t>(m) * m * batch * 2);
        a.take<float>(mn * 2);
        a.take<float>(static_cast<size_t>(n) * n * batch * 2);
      }
      break;
    }
    case SHP_OP_GRAM_EMA: {
      const int prec = o != nullptr ? o->prec : SHP_3XTF32;
      if (prec == SHP_3XTF32) a.take<float>(static_cast<size_t>(m) * n * batch * 2);
      break;
    }
    case SHP_OP_GRAM_EMA_STEPS: {  // batch = count x blocks
      const int prec = o != nullptr ? o->prec : SHP_3XTF32;
      if (prec == SHP_3XTF32) a.take<float>(static_cast<size_t>(m) * n * batch * 2);
      a.take<float>(static_cast<size_t>(m) * m * batch);  // the products G G^T
      a.take<float>(static_cast<size_t>(n) * n * batch);  // and G^T G
      break;
    }
    default:
      return 0;
  }
  return a.used + kAlign;
}

int shampoo_gram_ema(const float* G, int64_t m, int64_t n, int64_t batch, float* L, float* R,
                     float beta, float eps, int prec, void* ws, size_t ws_bytes,
                     shp_stream stream) {
  if (G == nullptr || m <= 0 || n <= 0 || batch <= 0 || m % 4 || n % 4) return SHP_EINVAL;
  if (!aligned16(G) || (L && !aligned16(L)) || (R && !aligned16(R))) return SHP_EINVAL;
  if (prec != SHP_TF32 && prec != SHP_3XTF32) return SHP_EINVAL;
  if (!isfinite(beta) || !isfinite(eps)) return SHP_EINVAL;
  if (m > INT32_MAX || n > INT32_MAX || batch > 65535) return SHP_EUNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float* Ghi = G;
  const float* Glo = nullptr;
  if (prec == SHP_3XTF32) {
    shp_prism_opts o{};
    o.prec = prec;
    if (ws == nullptr || ws_bytes < shp_workspace_bytes(SHP_OP_GRAM_EMA, m, n, batch, &o))
      return SHP_EINVAL;
    Arena a(reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(ws) + kAlign - 1) & ~(kAlign - 1)));
    float* hi = a.take<float>(static_cast<size_t>(m) * n * batch);
    float* lo = a.take<float>(static_cast<size_t>(m) * n * batch);
    CK(split_copy(G, m * n * batch, hi, lo, st));
    Ghi = hi;
    Glo = lo;
  }
  const int mode = prec == SHP_3XTF32 ? MODE_3XTF32 : MODE_TF32;
  const int M = static_cast<int>(m), N = static_cast<int>(n), B = static_cast<int>(batch);
  if (L != nullptr) {  // L <- beta L + (1-beta) G G^T + eps I
    EpiParams e = epi(EPI_EMA, OUT_F32, L, nullptr, m, m * m, M, M, nullptr);
    e.s0 = beta;
    e.s1 = 1.f - beta;
    e.s2 = eps;
    e.sym = 1;  // G G^T and L symmetric: upper-triangle tiles, mirrored
    CK(gemm_tc(mode, op(Ghi, Glo, false, n, m * n), op(Ghi, Glo, false, n, m * n), M, M, N, B, e,
               st));
  }
  if (R != nullptr) {  // R <- beta R + (1-beta) G^T G + eps I
    EpiParams e = epi(EPI_EMA, OUT_F32, R, nullptr, n, n * n, N, N, nullptr);
    e.s0 = beta;
    e.s1 = 1.f - beta;
    e.s2 = eps;
    e.sym = 1;
    CK(gemm_tc(mode, op(Ghi, Glo, true, n, m * n), op(Ghi, Glo, true, n, m * n), N, N, M, B, e,
               st));
  }
  return SHP_OK;
}

int shampoo_gram_ema_steps(const float* G, int64_t count, int64_t m, int64_t n, int64_t batch,
                           float* L, float* R, float beta, float eps, int prec, void* ws,
                           size_t ws_bytes, shp_stream stream) {
  if (G == nullptr || count <= 0 || m <= 0 || n <= 0 || batch <= 0 || m % 4 || n % 4)
    return SHP_EINVAL;
  if (!aligned16(G) || (L && !aligned16(L)) || (R && !aligned16(R))) return SHP_EINVAL;
  if (prec != SHP_TF32 && prec != SHP_3XTF32) return SHP_EINVAL;
  if (!isfinite(beta) || !isfinite(eps)) return SHP_EINVAL;
  if (m > INT32_MAX || n > INT32_MAX || count > 65535 || count * batch > 65535)
    return SHP_EUNSUPPORTED;
  const int64_t cb = count * batch;
  shp_prism_opts o{};
  o.prec = prec;
  if (ws == nullptr || ws_bytes < shp_workspace_bytes(SHP_OP_GRAM_EMA_STEPS, m, n, cb, &o))
    return SHP_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Arena a(reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(ws) + kAlign - 1) & ~(kAlign - 1)));
  const float* Ghi = G;
  const float* Glo = nullptr;
  if (prec == SHP_3XTF32) {
    float* hi = a.take<float>(static_cast<size_t>(m) * n * cb);
    float* lo = a.take<float>(static_cast<size_t>(m) * n * cb);
    CK(split_copy(G, m * n * cb, hi, lo, st));
    Ghi = hi;
    Glo = lo;
  }
  float* PL = a.take<float>(static_cast<size_t>(m) * m * cb);
  float* PR = a.take<float>(static_cast<size_t>(n) * n * cb);
  const int mode = prec == SHP_3XTF32 ? MODE_3XTF32 : MODE_TF32;
  const int M = static_cast<int>(m), N = static_cast<int>(n), CB = static_cast<int>(cb);
  // every step's product in one batched launch (each formed exactly as the
  // one-step call forms it), then the recurrence replayed element by element
  if (L != nullptr) {
    EpiParams e = epi(EPI_STORE, OUT_F32, PL, nullptr, m, m * m, M, M, nullptr);
    e.sym = 1;
    CK(gemm_tc(mode, op(Ghi, Glo, false, n, m * n), op(Ghi, Glo, false, n, m * n), M, M, N, CB, e,
               st));
    CK(ema_replay(L, PL, m, static_cast<int>(count), static_cast<int>(batch), beta, eps, st));
  }
  if (R != nullptr) {
    EpiParams e = epi(EPI_STORE, OUT_F32, PR, nullptr, n, n * n, N, N, nullptr);
    e.sym = 1;
    CK(gemm_tc(mode, op(Ghi, Glo, true, n, m * n), op(Ghi, Glo, true, n, m * n), N, N, M, CB, e,
               st));
    CK(ema_replay(R, PR, n, static_cast<int>(count), static_cast<int>(batch), beta, eps, st));
  }
  return SHP_OK;
}

}  // extern "C"

namespace {

// W <- W - eta P (or the momentum form) with P = Lroot G Rroot; shared by
// shampoo_apply and shampoo_apply_ex.
int apply_impl(float* W, float* Mom, double* acc, const float* G, const float* Lroot,
               const float* Rroot, int64_t m, int64_t n, int64_t batch, float lr, float gamma,
               int prec, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!W || !G || !Lroot || !Rroot || m <= 0 || n <= 0 || batch <= 0 || m % 4 || n % 4)
    return SHP_EINVAL;
  if (!aligned16(W) || !aligned16(G) || !aligned16(Lroot) || !aligned16(Rroot)) return SHP_EINVAL;
  if ((Mom && !aligned16(Mom)) || !isfinite(lr) || !isfinite(gamma)) return SHP_EINVAL;
  if (prec != SHP_TF32 && prec != SHP_3XTF32) return SHP_EINVAL;
  if (m > INT32_MAX || n > INT32_MAX || batch > 65535) return SHP_EUNSUPPORTED;
  shp_prism_opts o{};
  o.prec = prec;
  if (ws == nullptr || ws_bytes < shp_workspace_bytes(SHP_OP_APPLY, m, n, batch, &o))
    return SHP_EINVAL;
  Arena a(reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(ws) + kAlign - 1) & ~(kAlign - 1)));
  const size_t mn = static_cast<size_t>(m) * n * batch;
  const int mode = prec == SHP_3XTF32 ? MODE_3XTF32 : MODE_TF32;
  const int fmt = prec == SHP_3XTF32 ? OUT_SPLIT : OUT_F32;
  double* dn = a.take<double>(static_cast<size_t>(batch));
  float* eta = a.take<float>(static_cast<size_t>(batch));
  float* Thi = a.take<float>(mn);
  float* Tlo = prec == SHP_3XTF32 ? a.take<float>(mn) : nullptr;
  const int M = static_cast<int>(m), N = static_cast<int>(n), B = static_cast<int>(batch);
  if (acc != nullptr)  // [Shampoo] 5.1: acc += ||G||_F^2, eta = lr / sqrt(1 + acc)
    CK(adaptive_step(G, m * n, B, dn, acc, lr, eta, st));
  const float *Lh = Lroot, *Ll = nullptr, *Gh = G, *Gl = nullptr, *Rh = Rroot, *Rl = nullptr;
  if (prec == SHP_3XTF32) {
    const size_t mm = static_cast<size_t>(m) * m * batch, nn = static_cast<size_t>(n) * n * batch;
    float* p = a.take<float>(mm * 2);
    CK(split_copy(Lroot, mm, p, p + mm, st));
    Lh = p;
    Ll = p + mm;
    p = a.take<float>(mn * 2);
    CK(split_copy(G, mn, p, p + mn, st));
    Gh = p;
    Gl = p + mn;
    p = a.take<float>(nn * 2);
    CK(split_copy(Rroot, nn, p, p + nn, st));
    Rh = p;
    Rl = p + nn;
  }
  // T = Lroot G
  EpiParams e1 = epi(EPI_STORE, fmt, Thi, Tlo, n, m * n, M, N, nullptr);
  CK(gemm_tc(mode, op(Lh, Ll, false, m, m * m), op(Gh, Gl, true, n, m * n), M, N, M, B, e1, st));
  // W <- W - eta T Rroot, or M <- gamma M + T Rroot and W <- W - eta M ([Shampoo] 5.2)
  EpiParams e2 = epi(Mom ? EPI_MOMENTUM : EPI_APPLY, OUT_F32, W, nullptr, n, m * n, M, N, nullptr);
  e2.s0 = acc != nullptr ? -1.f : -lr;
  e2.alpha = acc != nullptr ? eta : nullptr;
  if (Mom != nullptr) {
    e2.aux_hi = Mom;
    e2.aux_fmt = OUT_F32;
    e2.lda_aux = n;
    e2.bs_aux = m * n;
    e2.out2_hi = Mom;
    e2.s1 = gamma;
  }
  CK(gemm_tc(mode, op(Thi, Tlo, false, n, m * n), op(Rh, Rl, true, n, n * n), M, N, N, B, e2, st));
  return SHP_OK;
}

// The inverse-root passes with fp64 iterates and Ozaki-scheme products: the
// same recurrence and launch order as the split path, each product from the
// digit slices of its operands, each new iterate sliced after it is formed.
int inv_root_oz(const float* A, int64_t n, int64_t batch, int power, const shp_prism_opts* o,
                const float* S, int64_t S_count, float* X_out, const shp_prism_report* rep,
                void* ws, size_t ws_bytes, cudaStream_t stream) {
  const int npass = power == SHP_POW_INV4 ? 2 : 1;
  if (!o->fixed_alpha && (S == nullptr || S_count < static_cast<int64_t>(npass) * o->max_iter))
    return SHP_EINVAL;
  if (!aligned16(A) || !aligned16(X_out)) return SHP_EINVAL;
  if (n > 26000 || batch > 65535) return SHP_EUNSUPPORTED;  // int32 level sums stay exact
  if (ws == nullptr || ws_bytes < shp_workspace_bytes(SHP_OP_INV_ROOT, n, n, batch, o))
    return SHP_EINVAL;
  CallKey key = make_key(3);
  key.power = power;
  key.a = A;
  key.x = X_out;
  key.s = S;
  key.s_count = S_count;
  key.n = n;
  key.batch = batch;
  key.o = *o;
  key.ws = ws;
  key.ws_bytes = ws_bytes;
  if (rep != nullptr) {
    key.rep[0] = rep->status;
    key.rep[1] = rep->iters;
    key.rep[2] = rep->resid;
    key.rep[3] = rep->alpha;
    key.rep[4] = rep->degree;
  }
  auto record = [&](cudaStream_t const* cs, cudaGraph_t g) -> int {
    Arena a(reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(ws) + kAlign - 1) &
                                    ~(kAlign - 1)));
    OzBufs w = carve_inv_root_oz(a, n, batch, o);
    const Ctl& ctl = w.ctl;
    const int N = static_cast<int>(n), B = static_cast<int>(batch);
    const int64_t nn = n * n;
    const int mi = o->max_iter;
    float* rep_res = rep != nullptr ? rep->resid : nullptr;
    float* rep_alpha = rep != nullptr ? rep->alpha : nullptr;
    int* rep_iters = rep != nullptr ? rep->iters : nullptr;
    int* rep_degree = rep != nullptr ? rep->degree : nullptr;
    // have_max: the maxima in `mb` were folded in by the epilogue that wrote X
    auto slice = [&](const double* X, const OzSlices& sl, float* x32, unsigned* mb,
                     bool have_max, cudaStream_t st) {
      return oz_slice(X, N, N, n, nn, B, ctl.active, mb, have_max, sl, x32, st);
    };
    // product of the left operand's row slices and the right one's column
    // slices; the epilogue folds the maxima of `out` into w.maxbuf
    auto epi = [&](int kind, double* out, const OzSlices& l, const OzSlices& r) {
      OzEpi e;
      memset(&e, 0, sizeof(e));
      e.kind = kind;
      e.out = out;
      e.ldo = n;
      e.bso = nn;
      e.sa = l.rscale;
      e.sb = r.cscale;
      e.alpha = ctl.alpha;
      e.s0 = 1.f;
      e.norm2 = &ctl.bs[0].norm2;
      e.norm2_stride = static_cast<int>(sizeof(BlockState) / sizeof(float));
      e.active = ctl.active;
      e.status = ctl.tmo;
      e.M = N;
      e.N = N;
      e.rmax = w.maxbuf;
      e.cmax = w.maxbuf + static_cast<int64_t>(B) * N;
      return e;
    };
    for (int pass = 0; pass < npass; ++pass) {
      CK(reset_pass(ctl, B, pass == 0, cs[0], o->adaptive_degree ? 1 : o->d));
      if (pass == 0) {
        CK(frob_norm2(A, 0, nn, B, ctl, cs[0]));
        CK(oz_init(A, n, B, ctl, w.Y, w.R, cs[0]));
        CK(slice(w.Y, w.sY, nullptr, w.maxbuf, false, cs[0]));
      } else {  // Y is pass 1's result, its slices are current
        CK(oz_restart(n, B, ctl, w.Y, w.R, cs[0]));
      }
      CK(slice(w.R, w.sR, w.Rs, w.maxbuf, false, cs[0]));
      const float* S_pass =
          S != nullptr ? S + static_cast<int64_t>(pass) * mi * n * o->p : nullptr;
      auto iter = [&](int, bool first, cudaStream_t st) -> int {
        if (!first) {  // R_k = I - Z_k Y_k and ||R_k||_F^2
          OzEpi e = epi(EPI_RESID, w.R, w.sZ, w.sY);
          CK(oz_clear_max(w.maxbuf, N, N, B, st));
          CK(gemm_oz(w.sZ.rows, w.sY.cols, N, N, N, B, e, st));
          CK(slice(w.R, w.sR, w.Rs, w.maxbuf, true, st));
        }
        CK(control_step(ctl, B, n, mi, o->tol, o->stall_below, o->stall_ratio, rep_res,
                        2 * (mi + 1), pass * (mi + 1), rep_iters, pass, st));
        int r = sketch_and_alpha(w.Rs, n, B, S_pass, w.V, o, ctl, rep_alpha, 2 * mi, pass * mi,
                                 st, rep_degree);
        if (r != SHP_OK) return r;
        double* z1 = first ? w.Z : nullptr;  // Z_1 = I + Delta (Z_0 = I is not stored)
        // Delta comes from the GEMM epilogue (which folds in its maxima) unless
        // some or all blocks form it elementwise (d = 1, adaptive degree)
        const bool d_max = o->d == 2 && !o->adaptive_degree;
        if (o->adaptive_degree) CK(oz_gform_d1(w.R, n, B, ctl, w.D, z1, st, ctl.act1));
        if (o->d == 2) {  // Delta = R/2 + alpha R^2 in the R R epilogue
          OzEpi e = epi(EPI_GPOLY, w.D, w.sR, w.sR);
          if (o->adaptive_degree) e.active = ctl.act2;
          e.out2 = z1;
          if (z1 != nullptr) {
            e.rmax2 = w.maxbuf2;
            e.cmax2 = w.maxbuf2 + static_cast<int64_t>(B) * N;
            CK(oz_clear_max(w.maxbuf2, N, N, B, st));
          }
          e.aux = w.R;
          e.lda = n;
          e.bsa = nn;
          e.s1 = 0.5f;
          CK(oz_clear_max(w.maxbuf, N, N, B, st));
          CK(gemm_oz(w.sR.rows, w.sR.cols, N, N, N, B, e, st));
        } else {
          CK(oz_gform_d1(w.R, n, B, ctl, w.D, z1, st));
        }
        CK(slice(w.D, w.sD, nullptr, w.maxbuf, d_max, st));
        if (first) CK(slice(w.Z, w.sZ, nullptr, w.maxbuf2, d_max, st));
        {  // Y_{k+1} = Y_k + Y_k Delta (in place)
          OzEpi e = epi(EPI_AXPY, w.Y, w.sY, w.sD);
          e.aux = w.Y;
          e.lda = n;
          e.bsa = nn;
          CK(oz_clear_max(w.maxbuf, N, N, B, st));
          CK(gemm_oz(w.sY.rows, w.sD.cols, N, N, N, B, e, st));
          CK(slice(w.Y, w.sY, nullptr, w.maxbuf, true, st));
        }
        if (!first) {  // Z_{k+1} = Z_k + Delta Z_k (in place)
          OzEpi e = epi(EPI_AXPY, w.Z, w.sD, w.sZ);
          e.aux = w.Z;
          e.lda = n;
          e.bsa = nn;
          CK(oz_clear_max(w.maxbuf, N, N, B, st));
          CK(gemm_oz(w.sD.rows, w.sZ.cols, N, N, N, B, e, st));
          CK(slice(w.Z, w.sZ, nullptr, w.maxbuf, true, st));
        }
        return SHP_OK;
      };
      int r = record_loop(cs, g, ctl, B, mi, iter);
      if (r != SHP_OK) return r;
    }
    if (power == SHP_POW_SQRT)
      CK(oz_finish(n, B, ctl, 0.5, w.Y, X_out, false, cs[0]));
    else
      CK(oz_finish(n, B, ctl, power == SHP_POW_INV2 ? -0.5 : -0.25, w.Z, X_out, true, cs[0]));
    if (rep != nullptr) CK(write_status(ctl, B, rep->status, cs[0]));
    return SHP_OK;
  };
  return dispatch(key, record, stream);
}

}  // namespace

extern "C" {

int shp_selftest_bounded_wait(int which, int32_t* status, float* alpha_out, void* ws,
                              size_t ws_bytes, shp_stream stream) {
  if (status == nullptr || ws == nullptr || ws_bytes < SHP_SELFTEST_WS_BYTES) return SHP_EINVAL;
  if (which != SHP_SELFTEST_GEMM && which != SHP_SELFTEST_OZAKI && which != SHP_SELFTEST_SKETCH &&
      which != SHP_SELFTEST_SKETCH_ALPHA && which != SHP_SELFTEST_SKETCH_CHAIN)
    return SHP_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CK(cudaMemsetAsync(status, 0, sizeof(int32_t), st));
  CK(cudaMemsetAsync(ws, 0, SHP_SELFTEST_WS_BYTES, st));
  Arena a(reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(ws) + kAlign - 1) & ~(kAlign - 1)));
  constexpr int n = 256, p = 8;  // one 256 x 256 product (a single CTA-pair tile)
  if (which == SHP_SELFTEST_GEMM) {
    float* A = a.take<float>(n * n);
    float* B = a.take<float>(n * n);
    float* C = a.take<float>(n * n);
    EpiParams e = epi(EPI_STORE, OUT_F32, C, nullptr, n, n * n, n, n, nullptr);
    e.status = status;
    e.selftest = 1;
    CK(gemm_tc(MODE_TF32, op(A, nullptr, false, n, n * n), op(B, nullptr, true, n, n * n), n, n,
               n, 1, e, st));
  } else if (which == SHP_SELFTEST_OZAKI) {
    const OzSlices sa = carve_slices(a, n, n, 1, true, false);
    const OzSlices sb = carve_slices(a, n, n, 1, false, true);
    double* C = a.take<double>(n * n);
    OzEpi e;
    memset(&e, 0, sizeof(e));
    e.kind = EPI_STORE;
    e.out = C;
    e.ldo = n;
    e.bso = n * n;
    e.sa = sa.rscale;
    e.sb = sb.cscale;
    e.s0 = 1.f;
    e.M = n;
    e.N = n;
    e.status = status;
    e.selftest = 1;
    CK(gemm_oz(sa.rows, sb.cols, n, n, n, 1, e, st));
  } else if (which == SHP_SELFTEST_SKETCH_ALPHA) {
    // the folded last pass of a d = 1 fit (V_3 = R V_2) times out; alpha starts
    // as the stop test leaves it, NaN, and nothing may overwrite it
    float* R = a.take<float>(n * n);
    float* V = a.take<float>(4 * n * p);
    double* gram = a.take<double>(15);
    int* gcnt = a.take<int>(1);
    float* alpha = alpha_out != nullptr ? alpha_out : a.take<float>(1);
    const int64_t np = static_cast<int64_t>(n) * p;
    CK(cudaMemsetAsync(alpha, 0xff, sizeof(float), st));  // a NaN pattern
    bool fused = false;
    CK(sketch_pass_alpha(R, n, n * n, V + 2 * np, 4 * np, V + 3 * np, 4 * np, p, 1, nullptr, st,
                         status, V, 1, 0.5f, 1.f, alpha, nullptr, 0, 0, nullptr, gram, gcnt,
                         &fused, 1));
    if (!fused) return SHP_EUNSUPPORTED;  // the folded kernel is the TMA one (n p fits)
  } else if (which == SHP_SELFTEST_SKETCH_CHAIN) {
    // the few-block sketch of one block (d = 1, passes and fit in one
    // cooperative launch) whose first grid barrier is never completed
    float* R = a.take<float>(n * n);
    float* S = a.take<float>(n * p);
    float* V = a.take<float>(4 * n * p);
    double* gpart = a.take<double>(static_cast<size_t>(kChainMaxCtas) * 15);
    int* gcnt = a.take<int>(1);
    unsigned* bar = a.take<unsigned>(4);
    float* alpha = alpha_out != nullptr ? alpha_out : a.take<float>(1);
    CK(cudaMemsetAsync(alpha, 0xff, sizeof(float), st));  // a NaN pattern
    bool done = false;
    CK(sketch_chain(R, n, n * n, S, 0, nullptr, V, p, 1, 1, nullptr, status, bar, 0.5f, 1.f,
                    alpha, nullptr, 0, 0, gpart, gcnt, st, &done, 1));
    if (!done) return SHP_EUNSUPPORTED;
  } else {  // the alpha fit of one block (d = 1) whose first sketch pass times out
    float* R = a.take<float>(n * n);
    float* S = a.take<float>(n * p);
    float* V = a.take<float>(4 * n * p);
    float* alpha = alpha_out != nullptr ? alpha_out : a.take<float>(1);
    const int64_t np = static_cast<int64_t>(n) * p;
    CK(sketch_pass(R, nullptr, n, n * n, S, 0, V + np, 4 * np, p, 1, nullptr, nullptr, 0, st,
                   status, 1));
    for (int j = 2; j <= 3; ++j)
      CK(sketch_pass(R, nullptr, n, n * n, V + (j - 1) * np, 4 * np, V + j * np, 4 * np, p, 1,
                     nullptr, nullptr, 0, st, status));
    CK(alpha_solve(V, n, p, 1, 1, 0.5f, 1.f, 0, nullptr, alpha, nullptr, nullptr, 0, 0, nullptr,
                   st, nullptr, status));
  }
  if (a.used > SHP_SELFTEST_WS_BYTES - kAlign) return SHP_EUNSUPPORTED;  // cannot happen
  return SHP_OK;
}

size_t shp_matmul_f64_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t batch) {
  if (M <= 0 || N <= 0 || K <= 0 || batch <= 0) return 0;
  Arena a(nullptr);
  carve_slices(a, M, K, batch, true, false);
  carve_slices(a, K, N, batch, false, true);
  a.take<unsigned>(static_cast<size_t>(M + 2 * K + N) * batch);
  return a.used + kAlign;
}

int shp_matmul_f64(const double* A, const double* B, double* C, int64_t M, int64_t N, int64_t K,
                   int64_t batch, void* ws, size_t ws_bytes, shp_stream stream) {
  return shp_matmul_f64_ex(A, B, C, M, N, K, batch, 0, ws, ws_bytes, stream);
}

int shp_matmul_f64_ex(const double* A, const double* B, double* C, int64_t M, int64_t N,
                      int64_t K, int64_t batch, int flags, void* ws, size_t ws_bytes,
                      shp_stream stream) {
  if (!A || !B || !C || M <= 0 || N <= 0 || K <= 0 || batch <= 0 || N % 2) return SHP_EINVAL;
  if (flags & ~(SHP_MATMUL_REUSE_A | SHP_MATMUL_REUSE_B | SHP_MATMUL_ACCUMULATE))
    return SHP_EINVAL;
  if (!aligned16(A) || !aligned16(B) || !aligned16(C)) return SHP_EINVAL;
  if (M > INT32_MAX || N > INT32_MAX || K > 26000 || batch > 65535) return SHP_EUNSUPPORTED;
  if (ws == nullptr || ws_bytes < shp_matmul_f64_workspace_bytes(M, N, K, batch)) return SHP_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Arena a(reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(ws) + kAlign - 1) & ~(kAlign - 1)));
  const OzSlices sa = carve_slices(a, M, K, batch, true, false);
  const OzSlices sb = carve_slices(a, K, N, batch, false, true);
  unsigned* maxbuf = a.take<unsigned>(static_cast<size_t>(M + 2 * K + N) * batch);
  const int m = static_cast<int>(M), nc = static_cast<int>(N), k = static_cast<int>(K);
  const int bt = static_cast<int>(batch);
  if (!(flags & SHP_MATMUL_REUSE_A))
    CK(oz_slice(A, m, k, K, M * K, bt, nullptr, maxbuf, false, sa, nullptr, st));
  if (!(flags & SHP_MATMUL_REUSE_B))
    CK(oz_slice(B, k, nc, N, K * N, bt, nullptr, maxbuf + (M + K) * batch, false, sb, nullptr,
                st));
  OzEpi e;
  memset(&e, 0, sizeof(e));
  e.kind = (flags & SHP_MATMUL_ACCUMULATE) ? EPI_AXPY : EPI_STORE;
  e.out = C;
  e.ldo = N;
  e.bso = M * N;
  if (flags & SHP_MATMUL_ACCUMULATE) {  // C <- C + A B, element by element in place
    e.aux = C;
    e.lda = N;
    e.bsa = M * N;
  }
  e.sa = sa.rscale;
  e.sb = sb.cscale;
  e.s0 = 1.f;
  e.M = m;
  e.N = nc;
  CK(gemm_oz(sa.rows, sb.cols, m, nc, k, bt, e, st));
  return SHP_OK;
}

int shampoo_apply(float* W, const float* G, const float* Lroot, const float* Rroot, int64_t m,
                  int64_t n, int64_t batch, float lr, int prec, void* ws, size_t ws_bytes,
                  shp_stream stream) {
  return apply_impl(W, nullptr, nullptr, G, Lroot, Rroot, m, n, batch, lr, 0.f, prec, ws,
                    ws_bytes, static_cast<cudaStream_t>(stream));
}

int shampoo_apply_ex(float* W, float* M, double* gnorm2_acc, const float* G, const float* Lroot,
                     const float* Rroot, int64_t m, int64_t n, int64_t batch, float lr,
                     float gamma, int prec, void* ws, size_t ws_bytes, shp_stream stream) {
  return apply_impl(W, M, gnorm2_acc, G, Lroot, Rroot, m, n, batch, lr, gamma, prec, ws,
                    ws_bytes, static_cast<cudaStream_t>(stream));
}

int prism_alpha_fit(const float* R, int64_t n, int64_t batch, const float* S, int p, int d,
                    float lo, float hi, float* alpha_out, double* J_coef_out, void* ws,
                    size_t ws_bytes, shp_stream stream) {
  if (!R || !S || !alpha_out || n <= 0 || batch <= 0 || p < 1 || p > 32 || (d != 1 && d != 2))
    return SHP_EINVAL;
  if (n % 4 || !aligned16(R)) return SHP_EINVAL;
  if (!(isfinite(lo) && isfinite(hi)) || lo > hi) return SHP_EINVAL;
  if (batch > 65535) return SHP_EUNSUPPORTED;
  shp_prism_opts o{};
  o.d = d;
  o.p = p;
  if (ws == nullptr || ws_bytes < shp_workspace_bytes(SHP_OP_ALPHA_FIT, n, n, batch, &o))
    return SHP_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Arena a(reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(ws) + kAlign - 1) & ~(kAlign - 1)));
  float* V = a.take<float>(static_cast<size_t>(2 * d + 2) * n * p * batch);
  int* tmo = a.take<int>(static_cast<size_t>(batch));
  const int64_t np = n * p, vbs = static_cast<int64_t>(2 * d + 2) * np;
  const int B = static_cast<int>(batch);
  CK(cudaMemsetAsync(tmo, 0, sizeof(int) * static_cast<size_t>(batch), st));
  CK(sketch_pass(R, nullptr, n, n * n, S, 0, V + np, vbs, p, B, nullptr, nullptr, 0, st, tmo));
  for (int j = 2; j <= 2 * d + 1; ++j)
    CK(sketch_pass(R, nullptr, n, n * n, V + (j - 1) * np, vbs, V + j * np, vbs, p, B, nullptr,
                   nullptr, 0, st, tmo));
  CK(alpha_solve(V, n, p, d, B, lo, hi, 0, nullptr, alpha_out, J_coef_out, nullptr, 0, 0,
                 nullptr, st, nullptr, tmo));
  return SHP_OK;
}

int matfn_inv_root(const float* A, int64_t n, int64_t batch, int power,
                   const shp_prism_opts* o, const float* S, int64_t S_count, float* X_out,
                   const shp_prism_report* rep, void* ws, size_t ws_bytes, shp_stream stream) {
  if (!A || !X_out || !opts_ok(o) || n <= 0 || batch <= 0 || n % 4) return SHP_EINVAL;
  if (power != SHP_POW_INV4 && power != SHP_POW_INV2 && power != SHP_POW_SQRT) return SHP_EINVAL;
  if (o->prec == SHP_OZAKI)
    return inv_root_oz(A, n, batch, power, o, S, S_count, X_out, rep, ws, ws_bytes,
                       static_cast<cudaStream_t>(stream));
  if (o->prec != SHP_TF32 && o->prec != SHP_3XTF32) return SHP_EINVAL;
  const int npass = power == SHP_POW_INV4 ? 2 : 1;
  if (!o->fixed_alpha && (S == nullptr || S_count < static_cast<int64_t>(npass) * o->max_iter))
    return SHP_EINVAL;
  if (!aligned16(A) || !aligned16(X_out)) return SHP_EINVAL;
  if (n > INT32_MAX || batch > INT32_MAX) return SHP_EUNSUPPORTED;
  if (ws == nullptr || ws_bytes < shp_workspace_bytes(SHP_OP_INV_ROOT, n, n, batch, o))
    return SHP_EINVAL;
  if (small_block_ok(n, n, o->p)) {  // one CTA per block, the whole iteration on chip
    CK(small_inv_root(A, static_cast<int>(n), static_cast<int>(batch), power, *o, S, X_out,
                      rep ? rep->status : nullptr, rep ? rep->iters : nullptr,
                      rep ? rep->resid : nullptr, rep ? rep->alpha : nullptr,
                      rep ? rep->degree : nullptr, static_cast<cudaStream_t>(stream)));
    return SHP_OK;
  }
  if (batch > 65535) return SHP_EUNSUPPORTED;
  CallKey key = make_key(0);
  key.power = power;
  key.a = A;
  key.x = X_out;
  key.s = S;
  key.s_count = S_count;
  key.n = n;
  key.batch = batch;
  key.o = *o;
  key.ws = ws;
  key.ws_bytes = ws_bytes;
  if (rep != nullptr) {
    key.rep[0] = rep->status;
    key.rep[1] = rep->iters;
    key.rep[2] = rep->resid;
    key.rep[3] = rep->alpha;
    key.rep[4] = rep->degree;
  }
  auto record = [&](cudaStream_t const* cs, cudaGraph_t g) -> int {
    Arena a(reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(ws) + kAlign - 1) &
                                    ~(kAlign - 1)));
    Bufs w = carve_inv_root(a, n, batch, o);
    const Ctl& ctl = w.ctl;
    const bool split = o->prec == SHP_3XTF32;
    const int mode = split ? MODE_3XTF32 : MODE_TF32;
    const int fmt = split ? OUT_SPLIT : OUT_F32;
    const int N = static_cast<int>(n), B = static_cast<int>(batch);
    const int64_t nn = n * n;
    const int mi = o->max_iter;
    float* rep_res = rep != nullptr ? rep->resid : nullptr;
    float* rep_alpha = rep != nullptr ? rep->alpha : nullptr;
    int* rep_iters = rep != nullptr ? rep->iters : nullptr;
    int* rep_degree = rep != nullptr ? rep->degree : nullptr;
    for (int pass = 0; pass < npass; ++pass) {
      CK(reset_pass(ctl, B, pass == 0, cs[0], o->adaptive_degree ? 1 : o->d));
      if (pass == 0) {
        CK(frob_norm2(A, 0, nn, B, ctl, cs[0]));
        CK(coupled_init(A, n, B, ctl, w.Yhi[0], w.Ylo[0], w.Rhi, w.Rlo,
                        split ? w.Rs : nullptr, cs[0]));
      } else {
        CK(coupled_restart(n, B, ctl, w.Yhi, w.Ylo, w.Rhi, w.Rlo,
                           split ? w.Rs : nullptr, cs[0]));
      }
      const float* S_pass =
          S != nullptr ? S + static_cast<int64_t>(pass) * mi * n * o->p : nullptr;
      // one step of the coupled iteration on ping-pong slot `cur`; the k = 0
      // step has R_0 = I - B from the start kernel and Z_1 = g (Z_0 = I)
      auto iter = [&](int cur, bool first, cudaStream_t st) -> int {
        const int nxt = cur ^ 1;
        // Every product here is formed in full, although Z_k Y_k, R_k^2,
        // Y_k g and g Z_k are symmetric in exact arithmetic: Z_k and Y_k only
        // commute up to rounding, and keeping one triangle (mirroring) turns
        // that non-commuting error into a symmetric one the coupled pair no
        // longer corrects.  In fp32 at cond 1e6 it costs the inverse root two
        // orders of magnitude of accuracy (residual and R^2 mirrored) or
        // diverges (updates mirrored).
        if (!first) {  // R_k = I - Z_k Y_k and ||R_k||_F^2
          EpiParams e = epi(EPI_RESID, fmt, w.Rhi, w.Rlo, n, nn, N, N, &ctl);
          if (split) e.out_plain = w.Rs;
          CK(gemm_tc(mode, op(w.Zhi[cur], w.Zlo[cur], false, n, nn),
                     op(w.Yhi[cur], w.Ylo[cur], true, n, nn), N, N, N, B, e, st));
        }
        CK(control_step(ctl, B, n, mi, o->tol, o->stall_below, o->stall_ratio, rep_res,
                        2 * (mi + 1), pass * (mi + 1), rep_iters, pass, st));
        int r = sketch_and_alpha(w.Rs, n, B, S_pass, w.V, o, ctl, rep_alpha, 2 * mi, pass * mi,
                                 st, rep_degree);
        if (r != SHP_OK) return r;
        float* z2hi = first ? w.Zhi[nxt] : nullptr;
        float* z2lo = first ? w.Zlo[nxt] : nullptr;
        // adaptive degree: blocks at degree 1 and 2 take the two launches below,
        // each masked to its own blocks
        if (o->adaptive_degree)
          CK(gform_d1(w.Rhi, w.Rlo, n, B, ctl, fmt, w.ghi, w.glo, z2hi, z2lo, st, ctl.act1));
        if (o->d == 2) {  // Delta = g - I = R/2 + alpha R^2 in the R R epilogue
          EpiParams e = epi(EPI_GPOLY, fmt, w.ghi, w.glo, n, nn, N, N, &ctl);
          if (o->adaptive_degree) e.active = ctl.act2;
          e.out2_hi = z2hi;
          e.out2_lo = z2lo;
          e.aux_hi = w.Rhi;
          e.aux_lo = w.Rlo;
          e.aux_fmt = fmt;
          e.lda_aux = n;
          e.bs_aux = nn;
          e.s1 = 0.5f;
          CK(gemm_tc(mode, op(w.Rhi, w.Rlo, false, n, nn), op(w.Rhi, w.Rlo, true, n, nn), N, N,
                     N, B, e, st));
        } else {
          CK(gform_d1(w.Rhi, w.Rlo, n, B, ctl, fmt, w.ghi, w.glo, z2hi, z2lo, st));
        }
        {  // Y_{k+1} = Y_k g = Y_k + Y_k Delta
          EpiParams e = epi(EPI_AXPY, fmt, w.Yhi[nxt], w.Ylo[nxt], n, nn, N, N, &ctl);
          e.aux_hi = w.Yhi[cur];
          e.aux_lo = w.Ylo[cur];
          e.aux_fmt = fmt;
          e.lda_aux = n;
          e.bs_aux = nn;
          CK(gemm_tc(mode, op(w.Yhi[cur], w.Ylo[cur], false, n, nn),
                     op(w.ghi, w.glo, true, n, nn), N, N, N, B, e, st));
        }
        if (!first) {  // Z_{k+1} = g Z_k = Z_k + Delta Z_k
          EpiParams e = epi(EPI_AXPY, fmt, w.Zhi[nxt], w.Zlo[nxt], n, nn, N, N, &ctl);
          e.aux_hi = w.Zhi[cur];
          e.aux_lo = w.Zlo[cur];
          e.aux_fmt = fmt;
          e.lda_aux = n;
          e.bs_aux = nn;
          CK(gemm_tc(mode, op(w.ghi, w.glo, false, n, nn),
                     op(w.Zhi[cur], w.Zlo[cur], true, n, nn), N, N, N, B, e, st));
        }
        return SHP_OK;
      };
      int r = record_loop(cs, g, ctl, B, mi, iter);
      if (r != SHP_OK) return r;
    }
    if (power == SHP_POW_SQRT) {
      const float* sh[2] = {w.Yhi[0], w.Yhi[1]};
      const float* sl[2] = {w.Ylo[0], w.Ylo[1]};
      CK(coupled_finish(n, B, ctl, 0.5, sh, sl, X_out, false, cs[0]));
    } else {
      const float* sh[2] = {w.Zhi[0], w.Zhi[1]};
      const float* sl[2] = {w.Zlo[0], w.Zlo[1]};
      CK(coupled_finish(n, B, ctl, power == SHP_POW_INV2 ? -0.5 : -0.25, sh, sl, X_out, true,
                        cs[0]));
    }
    if (rep != nullptr) CK(write_status(ctl, B, rep->status, cs[0]));
    return SHP_OK;
  };
  return dispatch(key, record, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// The polar iteration (R = I - X^T X, or I - X X^T for a wide G) and, with
// `sign`, the sign iteration of a symmetric square matrix (R = I - X X): the
// two differ only in the orientation of the first factor of the residual.
int polar_impl(const void* G, int storage, int64_t m, int64_t n, int64_t batch,
               const shp_prism_opts* o, const float* S, int64_t S_count, void* X_out,
               const shp_prism_report* rep, void* ws, size_t ws_bytes, shp_stream stream,
               bool sign) {
  if (!G || !X_out || !opts_ok(o) || m <= 0 || n <= 0 || batch <= 0) return SHP_EINVAL;
  if (storage != SHP_TF32 && storage != SHP_3XTF32 && storage != SHP_BF16) return SHP_EINVAL;
  const bool bf = storage == SHP_BF16;
  if (bf ? (n % 8 != 0 || m % 8 != 0) : (n % 4 != 0 || m % 4 != 0)) return SHP_EINVAL;
  if (!o->fixed_alpha && (S == nullptr || S_count < o->max_iter)) return SHP_EINVAL;
  if (!aligned16(G) || !aligned16(X_out)) return SHP_EINVAL;
  if (m > INT32_MAX || n > INT32_MAX || batch > INT32_MAX) return SHP_EUNSUPPORTED;
  shp_prism_opts oo = *o;
  oo.prec = storage;
  if (ws == nullptr || ws_bytes < shp_workspace_bytes(SHP_OP_POLAR, m, n, batch, &oo))
    return SHP_EINVAL;
  if (!bf && small_block_ok(m, n, o->p)) {  // one CTA per block, the whole iteration on chip
    CK(small_polar(static_cast<const float*>(G), static_cast<int>(m), static_cast<int>(n),
                   static_cast<int>(batch), oo, S, static_cast<float*>(X_out),
                   rep ? rep->status : nullptr, rep ? rep->iters : nullptr,
                   rep ? rep->resid : nullptr, rep ? rep->alpha : nullptr,
                   rep ? rep->degree : nullptr, sign, static_cast<cudaStream_t>(stream)));
    return SHP_OK;
  }
  if (batch > 65535) return SHP_EUNSUPPORTED;
  CallKey key = make_key(sign ? 2 : 1);
  key.storage = storage;
  key.a = G;
  key.x = X_out;
  key.s = S;
  key.s_count = S_count;
  key.m = m;
  key.n = n;
  key.batch = batch;
  key.o = oo;
  key.ws = ws;
  key.ws_bytes = ws_bytes;
  if (rep != nullptr) {
    key.rep[0] = rep->status;
    key.rep[1] = rep->iters;
    key.rep[2] = rep->resid;
    key.rep[3] = rep->alpha;
    key.rep[4] = rep->degree;
  }
  auto record = [&](cudaStream_t const* cs, cudaGraph_t g) -> int {
    Arena a(reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(ws) + kAlign - 1) &
                                    ~(kAlign - 1)));
    PolarBufs w = carve_polar(a, m, n, batch, storage, &oo);
    const Ctl& ctl = w.ctl;
    const bool tall = m >= n;
    const int64_t k = tall ? n : m;  // Gram size
    const int xmode = bf ? MODE_BF16 : (storage == SHP_3XTF32 ? MODE_3XTF32 : MODE_TF32);
    const int xfmt = bf ? OUT_BF16 : (storage == SHP_3XTF32 ? OUT_SPLIT : OUT_F32);
    // R R: bf16 storage multiplies the bf16 copy of R (fp32 accumulation,
    // as the iterate's own products); R itself stays fp32 for R/2 and the
    // sketch
    const int rmode = xmode;
    const int rfmt = storage == SHP_3XTF32 ? OUT_SPLIT : OUT_F32;
    const int M = static_cast<int>(m), N = static_cast<int>(n), K = static_cast<int>(k);
    const int B = static_cast<int>(batch);
    const int64_t mn = m * n, kk = k * k;
    const int mi = o->max_iter;
    float* rep_res = rep != nullptr ? rep->resid : nullptr;
    float* rep_alpha = rep != nullptr ? rep->alpha : nullptr;
    int* rep_iters = rep != nullptr ? rep->iters : nullptr;
    int* rep_degree = rep != nullptr ? rep->degree : nullptr;
    CK(reset_pass(ctl, B, 1, cs[0], o->adaptive_degree ? 1 : o->d));
    CK(frob_norm2(G, bf, mn, B, ctl, cs[0]));
    CK(polar_init(G, bf, mn, B, ctl, xfmt, w.Xhi[0], w.Xlo[0], cs[0]));
    auto iter = [&](int cur, bool, cudaStream_t st) -> int {
      const int nxt = cur ^ 1;
      {  // R = I - X^T X (tall) or I - X X^T (wide), and ||R||_F^2
        EpiParams e = epi(EPI_RESID, rfmt, w.Rhi, w.Rlo, k, kk, K, K, &ctl);
        if (rfmt == OUT_SPLIT) e.out_plain = w.Rs;
        e.out_b16 = w.Rb;
        // X^T X is a Gram matrix, symmetric in any arithmetic: upper-triangle
        // tiles, mirrored.  X X (sign) is symmetric only while X is, and X
        // picks up a rounding-level asymmetry from X + X Delta: keeping one
        // triangle of X X there raised the residual floor tenfold (fp32,
        // 512^2: 8e-6 instead of 3.5e-7), so it is formed in full.
        e.sym = sign ? 0 : 1;
        if (sign)  // X X
          CK(gemm_tc(xmode, op(w.Xhi[cur], w.Xlo[cur], false, n, mn),
                     op(w.Xhi[cur], w.Xlo[cur], true, n, mn), K, K, M, B, e, st));
        else if (tall)
          CK(gemm_tc(xmode, op(w.Xhi[cur], w.Xlo[cur], true, n, mn),
                     op(w.Xhi[cur], w.Xlo[cur], true, n, mn), K, K, M, B, e, st));
        else
          CK(gemm_tc(xmode, op(w.Xhi[cur], w.Xlo[cur], false, n, mn),
                     op(w.Xhi[cur], w.Xlo[cur], false, n, mn), K, K, N, B, e, st));
      }
      CK(control_step(ctl, B, k, mi, o->tol, o->stall_below, o->stall_ratio, rep_res,
                      2 * (mi + 1), 0, rep_iters, 0, st));
      int r = sketch_and_alpha(w.Rs, k, B, S, w.V, o, ctl, rep_alpha, 2 * mi, 0, st, rep_degree);
      if (r != SHP_OK) return r;
      if (o->adaptive_degree)  // degree-1 blocks; the R R launch below takes the others
        CK(gform_d1(w.Rhi, w.Rlo, k, B, ctl, xfmt, w.ghi, w.glo, nullptr, nullptr, st,
                    ctl.act1));
      if (o->d == 2) {  // Delta = g - I = R/2 + alpha R^2, stored like X
        EpiParams e = epi(EPI_GPOLY, xfmt, w.ghi, w.glo, k, kk, K, K, &ctl);
        if (o->adaptive_degree) e.active = ctl.act2;
        e.sym = sign ? 0 : 1;  // R exactly symmetric (mirrored above): R R and Delta too
        e.aux_hi = w.Rhi;
        e.aux_lo = w.Rlo;
        e.aux_fmt = rfmt;
        e.lda_aux = k;
        e.bs_aux = kk;
        e.s1 = 0.5f;
        if (bf)
          CK(gemm_tc(rmode, op(w.Rb, nullptr, false, k, kk), op(w.Rb, nullptr, true, k, kk), K, K,
                     K, B, e, st));
        else
          CK(gemm_tc(rmode, op(w.Rhi, w.Rlo, false, k, kk), op(w.Rhi, w.Rlo, true, k, kk), K, K,
                     K, B, e, st));
      } else {
        CK(gform_d1(w.Rhi, w.Rlo, k, B, ctl, xfmt, w.ghi, w.glo, nullptr, nullptr, st));
      }
      // X <- X g = X + X Delta (tall), X <- g^T X = X + Delta^T X (wide)
      EpiParams e = epi(EPI_AXPY, xfmt, w.Xhi[nxt], w.Xlo[nxt], n, mn, M, N, &ctl);
      e.aux_hi = w.Xhi[cur];
      e.aux_lo = w.Xlo[cur];
      e.aux_fmt = xfmt;
      e.lda_aux = n;
      e.bs_aux = mn;
      if (tall)
        CK(gemm_tc(xmode, op(w.Xhi[cur], w.Xlo[cur], false, n, mn),
                   op(w.ghi, w.glo, true, k, kk), M, N, N, B, e, st));
      else  // the tall iteration applied to X^T
        CK(gemm_tc(xmode, op(w.ghi, w.glo, true, k, kk),
                   op(w.Xhi[cur], w.Xlo[cur], true, n, mn), M, N, M, B, e, st));
      return SHP_OK;
    };
    int r = record_loop(cs, g, ctl, B, mi, iter);
    if (r != SHP_OK) return r;
    const void* sh[2] = {w.Xhi[0], w.Xhi[1]};
    const float* sl[2] = {w.Xlo[0], w.Xlo[1]};
    CK(polar_finish(mn, B, ctl, xfmt, sh, sl, X_out, bf ? 1 : 0, cs[0]));
    if (rep != nullptr) CK(write_status(ctl, B, rep->status, cs[0]));
    return SHP_OK;
  };
  return dispatch(key, record, static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

int matfn_polar(const void* G, int storage, int64_t m, int64_t n, int64_t batch,
                const shp_prism_opts* o, const float* S, int64_t S_count, void* X_out,
                const shp_prism_report* rep, void* ws, size_t ws_bytes, shp_stream stream) {
  return polar_impl(G, storage, m, n, batch, o, S, S_count, X_out, rep, ws, ws_bytes, stream,
                    false);
}

int matfn_polar_varsize(const float* G, const int32_t* dims, const int64_t* offsets,
                        int64_t batch, const shp_prism_opts* o, const float* S, int64_t S_count,
                        float* X_out, const shp_prism_report* rep, shp_stream stream) {
  if (!G || !dims || !offsets || !X_out || !opts_ok(o) || batch <= 0) return SHP_EINVAL;
  if (o->p > 16) return SHP_EINVAL;
  if (!o->fixed_alpha && (S == nullptr || S_count < o->max_iter)) return SHP_EINVAL;
  if (!aligned16(G) || !aligned16(X_out)) return SHP_EINVAL;
  if (batch > INT32_MAX) return SHP_EUNSUPPORTED;
  CK(small_polar_varsize(G, dims, reinterpret_cast<const int64_t*>(offsets),
                         static_cast<int>(batch), *o, S, X_out, rep ? rep->status : nullptr,
                         rep ? rep->iters : nullptr, rep ? rep->resid : nullptr,
                         rep ? rep->alpha : nullptr, rep ? rep->degree : nullptr,
                         static_cast<cudaStream_t>(stream)));
  return SHP_OK;
}

int matfn_sign(const void* A, int storage, int64_t n, int64_t batch, const shp_prism_opts* o,
               const float* S, int64_t S_count, void* X_out, const shp_prism_report* rep,
               void* ws, size_t ws_bytes, shp_stream stream) {
  return polar_impl(A, storage, n, n, batch, o, S, S_count, X_out, rep, ws, ws_bytes, stream,
                    true);
}

}  // extern "C"
