// prism_alpha_fit_noalloc: the sketched alpha fit without a caller workspace.
//
// prism_alpha_fit needs (2d+2) * n * p * batch floats of scratch for the
// sketch vectors V_j = R^j S, which the caller normally provides.  Some callers
// cannot hand out device memory in the middle of their work: an optimizer step
// running inside a framework whose caching allocator already owns the free
// device memory (a raw cudaMalloc there can fail, and cudaFree synchronises
// the whole device), or a latency-critical loop that must not stall on the
// implicit synchronisation of cudaMalloc/cudaFree.  This variant keeps its
// scratch in a fixed device array owned by the library instead.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds these SHP_NOALLOC_SCRATCH_BYTES until the process exits.
// Host code cannot use the variable's name as a device address (it names a
// host-side shadow), so the address is looked up with cudaGetSymbolAddress,
// once per device, with that device current, on the first call made on it.
// That first call should therefore come before any stream capture.
//
// All calls share the one array and it keeps the previous call's contents.
// The sketch vectors need no clearing (each pass writes every element it
// later reads); the per-block timeout flags after them are cleared at the
// start of every call (cudaMemsetAsync, which allocates nothing).  Calls that
// overlap on the GPU (on different streams, or from different host threads)
// race on the array.
//
// A bounded pipeline wait of the sketch passes that runs out (which only a
// device fault can cause) sets its block's flag, and that block's alpha comes
// out as NaN rather than as a fit on incomplete vectors.
#include <math.h>

#include <mutex>

#include "internal.h"
#include "shampoo_prism.h"

namespace {

constexpr size_t kScratchFloats = SHP_NOALLOC_SCRATCH_BYTES / sizeof(float);

static __device__ __align__(256) float g_alpha_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_alpha_scratch on the current device (looked up once).
cudaError_t scratch_address(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_alpha_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int prism_alpha_fit_noalloc(const float* R, int64_t n, int64_t batch, const float* S,
                                       int p, int d, float lo, float hi, float* alpha_out,
                                       double* J_coef_out, shp_stream stream) {
  if (!R || !S || !alpha_out || n <= 0 || batch <= 0 || p < 1 || p > 32 || (d != 1 && d != 2))
    return SHP_EINVAL;
  if (n % 4 || (reinterpret_cast<uintptr_t>(R) & 15u) != 0) return SHP_EINVAL;
  if (!(isfinite(lo) && isfinite(hi)) || lo > hi) return SHP_EINVAL;
  if (batch > 65535 || n > INT32_MAX) return SHP_EUNSUPPORTED;
  const int64_t np = n * p;
  const int64_t vbs = static_cast<int64_t>(2 * d + 2) * np;
  // V for every block, then one timeout flag per block
  if ((vbs + 1) * batch > static_cast<int64_t>(kScratchFloats)) return SHP_EUNSUPPORTED;
  float* V = nullptr;
  if (scratch_address(&V) != cudaSuccess) return SHP_ECUDA;
  int* tmo = reinterpret_cast<int*>(V + vbs * batch);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int B = static_cast<int>(batch);
  if (cudaMemsetAsync(tmo, 0, sizeof(int) * static_cast<size_t>(batch), st) != cudaSuccess)
    return SHP_ECUDA;
  if (shp::sketch_pass(R, nullptr, n, n * n, S, 0, V + np, vbs, p, B, nullptr, nullptr, 0, st,
                       tmo) != cudaSuccess)
    return SHP_ECUDA;
  for (int j = 2; j <= 2 * d + 1; ++j)
    if (shp::sketch_pass(R, nullptr, n, n * n, V + (j - 1) * np, vbs, V + j * np, vbs, p, B,
                         nullptr, nullptr, 0, st, tmo) != cudaSuccess)
      return SHP_ECUDA;
  if (shp::alpha_solve(V, n, p, d, B, lo, hi, 0, nullptr, alpha_out, J_coef_out, nullptr, 0, 0,
                       nullptr, st, nullptr, tmo) != cudaSuccess)
    return SHP_ECUDA;
  return SHP_OK;
}
