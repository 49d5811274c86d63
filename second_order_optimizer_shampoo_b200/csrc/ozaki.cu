// fp64-grade products on the int8 tensor cores (the Ozaki scheme), and the
// fp64 storage kernels of the inverse-root iteration that uses them.
//
// Why: the coupled Newton-Schulz iteration for A^(-1/4) of an SPD matrix of
// condition 1e6 ("Sintesi Tecnica: PRISM", Parte I; Shampoo tutorial 3.1)
// needs products and storage well beyond fp32 to stay within 1e-5 of the
// eigendecomposition result: fp32 storage with exactly rounded products ends
// near 2e-4, the fp64 iteration near 7e-6.  The split-precision idea the
// PRISM pages mention is taken here to its integer form: an error-free
// splitting of each operand into int8 digit slices whose products the int8
// tensor cores accumulate exactly in int32 (Ozaki, Ogita, Oishi, Rump,
// "Error-free transformations of matrix multiplication", Numer. Algorithms
// 2012; the integer-unit variant of Ootomo, Ozaki and Yokota, "DGEMM on
// integer matrix multiplication unit", IJHPCA 2024).
//
// Splitting (our own fixed-point form of it).  Row i of A (and column j of B)
// gets a power-of-two exponent e with max_k |A_ik| < 2^e.  Then
//   T_ik = rint(A_ik * 127 * 2^(32 - e))          (|T| < 127 * 2^32 + 1)
// is written in balanced base 256 as T = sum_s D_s 256^(4 - s) with
// D_1..D_4 in [-128, 127] (two's-complement low bytes, exact) and the top
// digit D_0 in [-127, 127], so A_ik = sigma_i sum_s D_s 2^(-8s) up to 2^-40
// of the row maximum, sigma_i = 2^e / 127.  A product keeps the digit pairs
// with s + t <= 4 ("levels" L = s + t, 15 int8 GEMMs):
//   C_ij = sigma_i tau_j sum_L 2^(-8L) sum_{s+t=L} (D^A_s D^B_t)_ij.
// Every level sum is an exact int32 (|D| <= 128, so a level of at most 5
// products over K terms stays below 5 * 2^14 * K < 2^31 for K <= 26000).
//
// Kernel k_gemm_oz: one cluster of two CTAs per SM pair, persistent over
// 256 x 96 output tiles.  Warp 0 loads all five slices of a 64-byte K step of
// A (128 rows per CTA) and of B^T (48 rows per CTA) with one 4-D TMA copy
// each into a 4-deep ring; the leader's warp 1 issues 30 tcgen05.mma
// kind::i8 (M = 256, N = 96, K = 32) per stage into five int32 accumulators
// (TMEM columns 0..479); warps 2..13 first drain their 32 columns of the five
// accumulators into fp64 registers and release TMEM (the next tile's products
// start then), and only after that apply the scales and the elementwise
// update, store (each thread owns one row, 16-byte stores) and fold the row
// and column maxima of the output into the arrays the next slicing reads.
// Five accumulators fill TMEM, so this split is what overlaps a tile's
// epilogue traffic with the next tile's products.  No TMA multicast.
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "shp_common.cuh"

namespace shp {

namespace {

constexpr int OZ_S = 5;                              // digit slices per operand
constexpr int OZ_BN = 96;                            // tile columns (pair tile 256 x 96)
#ifndef OZ_KB_BYTES
#define OZ_KB_BYTES 64
#endif
constexpr int OZ_BK = OZ_KB_BYTES;                   // K bytes per stage = per slice K block
// the shared-memory swizzle that matches a K row of OZ_BK bytes
constexpr uint32_t OZ_SW_LAYOUT = OZ_BK == 128 ? 2u : 4u;    // 128-byte / 64-byte swizzle
constexpr uint32_t OZ_SW_SBO = 8u * OZ_BK;                   // bytes between 8-row groups
static_assert(OZ_BK == 64 || OZ_BK == 128, "K rows of 64 or 128 bytes");
#ifndef OZ_STAGES_N
#define OZ_STAGES_N (OZ_BK == 128 ? 2 : 4)
#endif
constexpr int OZ_STAGES = OZ_STAGES_N;
constexpr int OZ_A_SLICE = 128 * OZ_BK;              // one slice of A per CTA: 8 KB
constexpr int OZ_B_SLICE = (OZ_BN / 2) * OZ_BK;      // one slice of B^T per CTA: 3 KB
constexpr int OZ_A_BYTES = OZ_S * OZ_A_SLICE;
constexpr int OZ_B_BYTES = OZ_S * OZ_B_SLICE;
constexpr int OZ_STAGE = OZ_A_BYTES + OZ_B_BYTES;    // 55 KB
constexpr int OZ_SMEM = 1024 + OZ_STAGES * OZ_STAGE + 256;
constexpr uint32_t OZ_TMEM_COLS = 512;               // 5 x 96 used
static_assert(OZ_S * OZ_BN <= 512, "level accumulators must fit in TMEM");
static_assert(OZ_SMEM <= 232448, "ozaki GEMM exceeds shared memory");
static_assert(OZ_A_SLICE % (8 * OZ_BK) == 0 && OZ_B_SLICE % (8 * OZ_BK) == 0,
              "slices start on swizzle atoms");

// ------------------------------------------------------------- device helpers
SHP_DEV void tma_load_4d_pair(void* dst, const CUtensorMap* map, uint32_t mbar, int x, int y,
                              int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(mbar), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

SHP_DEV void mma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// The same product with the A operand held in the tensor core's collector
// buffer across consecutive instructions: FILL reads A from shared memory and
// keeps it, USE takes the kept copy, LAST takes it and frees the buffer.  The
// products of one A digit slice against several B slices then read that slice
// from shared memory once instead of once per product.
enum { COLL_FILL = 0, COLL_USE = 1, COLL_LAST = 2 };
template <int C>
SHP_DEV void mma_i8_pair_coll(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                              uint32_t accumulate) {
  if constexpr (C == COLL_FILL)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8.collector::a::fill [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
  else if constexpr (C == COLL_USE)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8.collector::a::use [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8.collector::a::lastuse [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// kind::i8 instruction descriptor: D s32, A and B signed 8-bit, both K-major.
constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// 32 lanes x 16 consecutive 32-bit columns, no wait (the caller waits once
// for several loads).
SHP_DEV void tmem_ld16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
SHP_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Exponent of a row (column) maximum from the high word of |max| (the key the
// absmax kernel reduces): e with max < 2^e, scale factor 2^-e and the weight
// sigma = 2^e / 127.  key 0: an all-zero row (factor 0, sigma 0); a
// non-finite maximum (or one >= 2^1022) gives sigma = NaN, so a NaN or Inf
// anywhere in the row reaches every product that uses it.
SHP_DEV void oz_scale_of(unsigned key, double& factor, double& sigma) {
  const int E = static_cast<int>(key >> 20);  // biased exponent of the maximum
  if (key == 0u) {
    factor = 0.0;
    sigma = 0.0;
    return;
  }
  if (E >= 2045) {
    factor = 0.0;
    sigma = __longlong_as_double(0x7ff8000000000000ll);
    return;
  }
  const int e = (E == 0 ? 1 : E) - 1022;  // max < 2^e (subnormal maxima take E = 1)
  factor = __longlong_as_double(static_cast<long long>(1023 - e) << 52);  // 2^-e
  sigma = __longlong_as_double(static_cast<long long>(1023 + e) << 52) * (1.0 / 127.0);
}

// Exact conversions through the fp64 adder instead of the (much narrower)
// conversion unit: an int32 v is the double with high word 0x43300000 and low
// word v ^ 2^31, less 2^52 + 2^31; rint(t) for |t| < 2^51 is the low part of
// t + 1.5 * 2^52 (the addition rounds to nearest even, as rint does).
SHP_DEV double i32_to_f64(uint32_t v) {
  return __hiloint2double(0x43300000, static_cast<int>(v ^ 0x80000000u)) - 4503601774854144.0;
}
SHP_DEV long long rint_to_i64(double t) {
  return __double_as_longlong(t + 6755399441055744.0) - 0x4338000000000000ll;
}

// Digit slices of four consecutive elements x[0..3] that share the factor
// 2^-e of their row (or column): T = rint(x 2^-e 127 2^32) in balanced base
// 256.  With U = T + 0x80808080 the low word holds D_4 .. D_1 offset by 128
// byte by byte (so XOR 0x80 gives each digit's two's-complement byte) and the
// high word is D_0; w[s] receives the four elements' digit s, one per byte.
SHP_DEV void oz_digits4(const double (&x)[4], double factor, uint32_t (&w)[OZ_S]) {
  uint32_t lo[4], hi[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const long long T = rint_to_i64((x[e] * factor) * 545460846592.0);  // 127 * 2^32
    const long long U = T + 0x80808080ll;
    lo[e] = static_cast<uint32_t>(U) ^ 0x80808080u;
    hi[e] = static_cast<uint32_t>(U >> 32);
  }
  // 4 x 4 byte transpose: byte k of lo[e] is digit 4 - k of element e
  const uint32_t t0 = __byte_perm(lo[0], lo[1], 0x5140), t1 = __byte_perm(lo[0], lo[1], 0x7362);
  const uint32_t t2 = __byte_perm(lo[2], lo[3], 0x5140), t3 = __byte_perm(lo[2], lo[3], 0x7362);
  w[4] = __byte_perm(t0, t2, 0x5410);
  w[3] = __byte_perm(t0, t2, 0x7632);
  w[2] = __byte_perm(t1, t3, 0x5410);
  w[1] = __byte_perm(t1, t3, 0x7632);
  w[0] = __byte_perm(__byte_perm(hi[0], hi[1], 0x0040), __byte_perm(hi[2], hi[3], 0x0040), 0x5410);
}

// ------------------------------------------------------------- slicing
constexpr int SL_T = 64;  // tile edge of the slicing kernels

SHP_DEV unsigned abs_key(double x) {
  return static_cast<unsigned>(static_cast<unsigned long long>(__double_as_longlong(x)) >> 32) &
         0x7fffffffu;
}

// rmax[b][i] = max_j key(|X_ij|), cmax[b][j] = max_i key(|X_ij|) (atomicMax on
// the high word of |x|, monotonic for non-negative doubles; NaN above all).
__global__ void __launch_bounds__(256)
    k_oz_absmax(const double* __restrict__ X, int rows, int cols, int64_t ld, int64_t bs,
                const int* __restrict__ active, unsigned* rmax, unsigned* cmax) {
  count_kernel_run();
  const int b = blockIdx.z;
  if (active != nullptr && active[b] == 0) return;
  __shared__ unsigned cm[8][SL_T];
  const int r0 = blockIdx.y * SL_T, c0 = blockIdx.x * SL_T;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const double* Xb = X + b * bs;
  const int c = c0 + 2 * tx;
  unsigned ck0 = 0u, ck1 = 0u;
  for (int k = 0; k < SL_T / 8; ++k) {
    const int r = r0 + ty + 8 * k;
    unsigned k0 = 0u, k1 = 0u;
    if (r < rows) {
      if (c < cols) k0 = abs_key(Xb[static_cast<int64_t>(r) * ld + c]);
      if (c + 1 < cols) k1 = abs_key(Xb[static_cast<int64_t>(r) * ld + c + 1]);
    }
    ck0 = max(ck0, k0);
    ck1 = max(ck1, k1);
    unsigned rk = max(k0, k1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rk = max(rk, __shfl_xor_sync(0xffffffffu, rk, o));
    if (tx == 0 && r < rows && rk != 0u) atomicMax(&rmax[static_cast<int64_t>(b) * rows + r], rk);
  }
  cm[ty][2 * tx] = ck0;
  cm[ty][2 * tx + 1] = ck1;
  __syncthreads();
  if (threadIdx.x < SL_T) {
    unsigned m = 0u;
#pragma unroll
    for (int w = 0; w < 8; ++w) m = max(m, cm[w][threadIdx.x]);
    const int cc = c0 + threadIdx.x;
    if (cc < cols && m != 0u) atomicMax(&cmax[static_cast<int64_t>(b) * cols + cc], m);
  }
}

// Digit slices of a 64 x 64 tile of X.  Slices are stored K-blocked, so that
// the copy of one 64-byte K step of every slice of a 128-row tile is one
// contiguous stretch of memory: digit s of element (row, k) of an operand
// with R rows sits at [b][k / 64][s][row][k % 64].  Row slicing (A role, K =
// the column index) goes to rsl with weights rscale[b][i], column slicing (B
// role, K = the row index: the row slicing of X^T) to csl with weights
// cscale[b][j].  Either output may be null.  Past the matrix edge the last K
// block holds digits of 0.  x32, when non-null, gets a plain fp32 copy of X.
__global__ void __launch_bounds__(256)
    k_oz_slice(const double* __restrict__ X, int rows, int cols, int64_t ld, int64_t bs,
               const int* __restrict__ active, const unsigned* __restrict__ rmax,
               const unsigned* __restrict__ cmax, int8_t* rsl, int8_t* csl, double* rscale,
               double* cscale, float* x32) {
  count_kernel_run();
  const int b = blockIdx.z;
  if (active != nullptr && active[b] == 0) return;
  __shared__ double tile[SL_T][SL_T + 1];
  const int r0 = blockIdx.y * SL_T, c0 = blockIdx.x * SL_T;
  const double* Xb = X + b * bs;
  {
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (int k = 0; k < SL_T / 8; ++k) {
      const int r = ty + 8 * k;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int cc = 2 * tx + h;
        double v = 0.0;
        if (r0 + r < rows && c0 + cc < cols) {
          v = Xb[static_cast<int64_t>(r0 + r) * ld + c0 + cc];
          if (x32 != nullptr) x32[b * bs + static_cast<int64_t>(r0 + r) * ld + c0 + cc] = static_cast<float>(v);
        }
        tile[r][cc] = v;
      }
    }
  }
  __syncthreads();
  const int idx = threadIdx.x >> 2, seg = (threadIdx.x & 3) * 16;
  // row slicing: this thread's row r0 + idx, columns c0 + seg .. + 15
  const int64_t nkb_r = (cols + OZ_BK - 1) / OZ_BK, nkb_c = (rows + OZ_BK - 1) / OZ_BK;
  if (rsl != nullptr && r0 + idx < rows) {
    const int r = r0 + idx;
    double f, sg;
    oz_scale_of(rmax[static_cast<int64_t>(b) * rows + r], f, sg);
    if (blockIdx.x == 0 && seg == 0 && rscale != nullptr) rscale[static_cast<int64_t>(b) * rows + r] = sg;
    uint32_t w[OZ_S][4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      double x[4];
      uint32_t d[OZ_S];
#pragma unroll
      for (int e = 0; e < 4; ++e) x[e] = tile[idx][seg + 4 * g + e];
      oz_digits4(x, f, d);
#pragma unroll
      for (int q = 0; q < OZ_S; ++q) w[q][g] = d[q];
    }
#pragma unroll
    for (int q = 0; q < OZ_S; ++q) {
      int8_t* dst =
          rsl + ((((b * nkb_r + c0 / OZ_BK) * OZ_S + q) * rows + r) * OZ_BK) + c0 % OZ_BK + seg;
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[q][0], w[q][1], w[q][2], w[q][3]);
    }
  }
  // column slicing: this thread's column c0 + idx, rows r0 + seg .. + 15
  if (csl != nullptr && c0 + idx < cols) {
    const int c = c0 + idx;
    double f, sg;
    oz_scale_of(cmax[static_cast<int64_t>(b) * cols + c], f, sg);
    if (blockIdx.y == 0 && seg == 0 && cscale != nullptr) cscale[static_cast<int64_t>(b) * cols + c] = sg;
    uint32_t w[OZ_S][4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      double x[4];
      uint32_t d[OZ_S];
#pragma unroll
      for (int e = 0; e < 4; ++e) x[e] = tile[seg + 4 * g + e][idx];
      oz_digits4(x, f, d);
#pragma unroll
      for (int q = 0; q < OZ_S; ++q) w[q][g] = d[q];
    }
#pragma unroll
    for (int q = 0; q < OZ_S; ++q) {
      int8_t* dst =
          csl + ((((b * nkb_c + r0 / OZ_BK) * OZ_S + q) * cols + c) * OZ_BK) + r0 % OZ_BK + seg;
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[q][0], w[q][1], w[q][2], w[q][3]);
    }
  }
}

// ------------------------------------------------------------- the GEMM
constexpr int OZ_EPI_WARPS = 12;  // 4 TMEM lane quarters x 3 groups of 32 columns
constexpr int OZ_THREADS = 32 * (2 + OZ_EPI_WARPS);

SHP_DEV void tmem_ld8_nowait(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr));
}

// Phase 1 of a tile's epilogue: this thread's row, 32 columns of the five
// level accumulators, combined in fp64 (exact up to the last bits): the TMEM
// accumulators are free again once every warp has done this.
SHP_DEV void oz_drain(uint32_t taddr, double (&acc)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t l[OZ_S][8];
#pragma unroll
    for (int L = 0; L < OZ_S; ++L)
      tmem_ld8_nowait(taddr + static_cast<uint32_t>(L * OZ_BN + 8 * c), l[L]);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      double t = i32_to_f64(l[OZ_S - 1][j]);
#pragma unroll
      for (int L = OZ_S - 2; L >= 0; --L) t = fma(t, 0.00390625, i32_to_f64(l[L][j]));
      acc[8 * c + j] = t;
    }
  }
}

// Maximum over the warp's 32 rows of each of 8 column keys, by recursive
// halving (9 shuffles): lanes 4c .. 4c + 3 end with the maximum of column c.
SHP_DEV uint32_t col_max8(uint32_t (&k)[8], int lane) {
#pragma unroll
  for (int st = 0; st < 3; ++st) {
    const int o = 16 >> st, h = 4 >> st;
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const uint32_t send = up ? k[i] : k[i + h];
      const uint32_t keep = up ? k[i + h] : k[i];
      k[i] = max(keep, __shfl_xor_sync(0xffffffffu, send, o));
    }
  }
  uint32_t v = k[0];
  v = max(v, __shfl_xor_sync(0xffffffffu, v, 2));
  v = max(v, __shfl_xor_sync(0xffffffffu, v, 1));
  return v;
}

// Phase 2: scales, the kind's elementwise update, fp64 stores (16 bytes at a
// time; a thread owns one row) and the row/column maxima of what is stored,
// which the next slicing needs.  Rows past M take part in the shuffles only.
SHP_DEV double oz_finish_tile(const double (&acc)[32], const OzEpi& ep, int b, int row, int col00,
                              int lane) {
  const bool rowok = row < ep.M;
  const double sa = rowok ? ep.sa[static_cast<int64_t>(b) * ep.M + row] : 0.0;
  const double alpha = ep.alpha != nullptr ? static_cast<double>(ep.alpha[b]) : 0.0;
  const double* sb = ep.sb + static_cast<int64_t>(b) * ep.N;
  double nrm = 0.0;
  uint32_t rk = 0u, rk2 = 0u;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int col0 = col00 + 8 * c;
    const int nv = col0 >= ep.N ? 0 : (ep.N - col0 < 8 ? ep.N - col0 : 8);  // 0, 4 or 8
    const bool ok = rowok && nv > 0;
    const int64_t off = static_cast<int64_t>(b) * ep.bso + static_cast<int64_t>(row) * ep.ldo + col0;
    double x[8];
    if (ok && (ep.kind == EPI_GPOLY || ep.kind == EPI_AXPY)) {
      const double* ap = ep.aux + static_cast<int64_t>(b) * ep.bsa + static_cast<int64_t>(row) * ep.lda + col0;
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        double2 a2 = make_double2(0.0, 0.0);
        if (j < nv) a2 = *reinterpret_cast<const double2*>(ap + j);
        x[j] = a2.x;
        x[j + 1] = a2.y;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) x[j] = 0.0;
    }
    double out[8];
    const int dcol = row - col0;  // column j of this chunk is on the diagonal when j == dcol
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const double v = ok && j < nv ? acc[8 * c + j] * sa * __ldg(sb + col0 + j) : 0.0;
      switch (ep.kind) {
        case EPI_RESID: out[j] = (j == dcol ? 1.0 : 0.0) - v; break;
        case EPI_GPOLY: out[j] = static_cast<double>(ep.s1) * x[j] + alpha * v; break;
        case EPI_AXPY: out[j] = x[j] + static_cast<double>(ep.s0) * v; break;
        default: out[j] = static_cast<double>(ep.s0) * v; break;
      }
    }
    uint32_t ck[8], ck2[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const bool in = ok && j < nv;
      if (in && ep.kind == EPI_RESID) nrm += out[j] * out[j];
      ck[j] = in ? abs_key(out[j]) : 0u;
      ck2[j] = in ? abs_key(out[j] + (j == dcol ? 1.0 : 0.0)) : 0u;
      rk = max(rk, ck[j]);
      rk2 = max(rk2, ck2[j]);
    }
    if (ok) {
      double* op = ep.out + off;
#pragma unroll
      for (int j = 0; j < 8; j += 2)
        if (j < nv) *reinterpret_cast<double2*>(op + j) = make_double2(out[j], out[j + 1]);
      if (ep.out2 != nullptr) {  // I + Delta
        double* o2 = ep.out2 + off;
#pragma unroll
        for (int j = 0; j < 8; j += 2)
          if (j < nv)
            *reinterpret_cast<double2*>(o2 + j) = make_double2(
                out[j] + (j == dcol ? 1.0 : 0.0), out[j + 1] + (j + 1 == dcol ? 1.0 : 0.0));
      }
    }
    if (ep.cmax != nullptr) {
      const uint32_t m = col_max8(ck, lane);
      if ((lane & 3) == 0 && (lane >> 2) < nv && m != 0u)
        atomicMax(&ep.cmax[static_cast<int64_t>(b) * ep.N + col0 + (lane >> 2)], m);
      if (ep.out2 != nullptr) {
        const uint32_t m2 = col_max8(ck2, lane);
        if ((lane & 3) == 0 && (lane >> 2) < nv && m2 != 0u)
          atomicMax(&ep.cmax2[static_cast<int64_t>(b) * ep.N + col0 + (lane >> 2)], m2);
      }
    }
  }
  if (ep.rmax != nullptr && rowok) {
    if (rk != 0u) atomicMax(&ep.rmax[static_cast<int64_t>(b) * ep.M + row], rk);
    if (ep.out2 != nullptr && rk2 != 0u)
      atomicMax(&ep.rmax2[static_cast<int64_t>(b) * ep.M + row], rk2);
  }
  return nrm;
}

//   full[s]/empty[s]: operand ring (the leader's full barrier counts both
//                     CTAs' bytes; empty is signalled to both by the commit)
//   accf:             the five level accumulators of the current tile complete
//   acce:             ... drained into registers (12 epilogue warps x 2 CTAs
//                     arrive on the leader's)
__global__ void __launch_bounds__(OZ_THREADS, 1)
    k_gemm_oz(const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tB,
              int K, OzEpi ep, int batch) {
  count_kernel_run();
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int ncl = static_cast<int>(gridDim.x) / 2, cl = static_cast<int>(blockIdx.x) / 2;
  const int tiles_n = (ep.N + OZ_BN - 1) / OZ_BN, tiles_m = (ep.M + 255) / 256;
  const int per_b = tiles_n * tiles_m;
  const int ntiles = per_b * batch;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OZ_STAGES * OZ_STAGE);
  uint64_t* empty = full + OZ_STAGES;
  uint64_t* accf = empty + OZ_STAGES;
  uint64_t* acce = accf + 1;
  uint64_t* drain = acce + 1;
  uint64_t* never = drain + 1;  // completed by nothing: the self-test's wait
  volatile int* abort_flag = reinterpret_cast<volatile int*>(never + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1) + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < OZ_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    mbar_init(acce, 2 * OZ_EPI_WARPS);
    mbar_init(drain, 1);
    mbar_init(never, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tA);
    tma_prefetch_desc(&tB);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, OZ_TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int KB = (K + OZ_BK - 1) / OZ_BK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs load their halves)
      const uint32_t tx = 2u * OZ_STAGE;
      int kit = 0;
      bool stop = false;
      // bounded-wait self-test: before any copy is issued, wait on a barrier
      // nothing completes; it runs out, and the CTA unwinds with nothing in flight
      if (ep.selftest && !mbar_wait(never, 0, nullptr, SHP_SELFTEST_LIMIT)) {
        *abort_flag = 1;
        if (ep.status != nullptr) atomicExch(&ep.status[0], ST_ETIMEOUT);
        stop = true;
      }
      for (int t = cl; t < ntiles && !stop; t += ncl) {
        const int b = t / per_b, r = t % per_b;
        if (ep.active != nullptr && ep.active[b] == 0) continue;
        const int tm = r / tiles_n, tn = r % tiles_n;
        const int m0 = tm * 256 + static_cast<int>(rank) * 128;
        const int nb0 = tn * OZ_BN + static_cast<int>(rank) * (OZ_BN / 2);
        for (int kb = 0; kb < KB; ++kb, ++kit) {
          const int s = kit % OZ_STAGES;
          if (kit >= OZ_STAGES &&
              (*abort_flag || !mbar_wait(&empty[s], ((kit / OZ_STAGES) - 1) & 1, abort_flag))) {
            *abort_flag = 1;
            if (ep.status != nullptr) atomicExch(&ep.status[b], ST_ETIMEOUT);
            stop = true;
            break;
          }
          uint8_t* st = smem + s * OZ_STAGE;
          if (leader) mbar_arrive_expect_tx(&full[s], tx);
          const uint32_t fbar = mapa_shared(smem_u32(&full[s]), 0);
          tma_load_4d_pair(st, &tA, fbar, 0, m0, 0, b * KB + kb);
          tma_load_4d_pair(st + OZ_A_BYTES, &tB, fbar, 0, nb0, 0, b * KB + kb);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer: per 32-byte K step, level L = s + t takes
      // the digit products D^A_s D^B_t into accumulator L
      constexpr uint32_t idesc = idesc_i8(256, OZ_BN);
      int kit = 0, tl = 0;
      bool stop = false;
      for (int t = cl; t < ntiles && !stop; t += ncl) {
        const int b = t / per_b;
        if (ep.active != nullptr && ep.active[b] == 0) continue;
        if (tl >= 1 && (*abort_flag || !mbar_wait(acce, (tl - 1) & 1, abort_flag))) {
          *abort_flag = 1;
          if (ep.status != nullptr) atomicExch(&ep.status[b], ST_ETIMEOUT);
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++kit) {
          const int s = kit % OZ_STAGES;
          if (*abort_flag || !mbar_wait(&full[s], (kit / OZ_STAGES) & 1, abort_flag)) {
            *abort_flag = 1;
            if (ep.status != nullptr) atomicExch(&ep.status[b], ST_ETIMEOUT);
            stop = true;
            break;
          }
          tc_fence_after();
          // the descriptors' start-address field holds address >> 4 (shared
          // memory addresses stay below 2^18, so adding offsets >> 4 to the
          // base descriptor never carries out of the field)
          const uint32_t base = smem_u32(smem + s * OZ_STAGE);
          const uint64_t ad0 = smem_desc(base, 16, OZ_SW_SBO, OZ_SW_LAYOUT);
          const uint64_t bd0 = smem_desc(base + OZ_A_BYTES, 16, OZ_SW_SBO, OZ_SW_LAYOUT);
          // A slice sa meets B slices 0 .. S-1-sa (level sa + sb); the first
          // product of a k-step into each level comes from sa = 0
#pragma unroll
          for (int ks = 0; ks < OZ_BK / 32; ++ks) {
#pragma unroll
            for (int sa = 0; sa < OZ_S; ++sa) {
              const uint64_t ad = ad0 + static_cast<uint64_t>((sa * OZ_A_SLICE + ks * 32) >> 4);
              const uint32_t acc = (kb > 0 || ks > 0 || sa > 0) ? 1u : 0u;
#pragma unroll
              for (int sb = 0; sb < OZ_S - sa; ++sb) {
                const uint64_t bd = bd0 + static_cast<uint64_t>((sb * OZ_B_SLICE + ks * 32) >> 4);
                const uint32_t d = tmem + static_cast<uint32_t>((sa + sb) * OZ_BN);
                if (sa == OZ_S - 1)
                  mma_i8_pair(d, ad, bd, idesc, acc);
                else if (sb == 0)
                  mma_i8_pair_coll<COLL_FILL>(d, ad, bd, idesc, acc);
                else if (sb < OZ_S - 1 - sa)
                  mma_i8_pair_coll<COLL_USE>(d, ad, bd, idesc, acc);
                else
                  mma_i8_pair_coll<COLL_LAST>(d, ad, bd, idesc, acc);
              }
            }
          }
          mma_commit_pair(&empty[s], 3);
        }
        if (stop) break;
        mma_commit_pair(accf, 3);
        ++tl;
      }
    }
    if (lane == 0 && leader) mma_commit_pair(drain, 3);  // after every MMA issued above
  } else {
    // ---------------- epilogue warps 2..13 (both CTAs, each on its TMEM rows):
    // drain the accumulators, release them to the next tile's products, then
    // finish this tile while those run
    const int q = warp & 3, g = (warp - 2) >> 2;
    int tl = 0;
    for (int t = cl; t < ntiles; t += ncl) {
      const int b = t / per_b, r = t % per_b;
      if (ep.active != nullptr && ep.active[b] == 0) continue;
      if (*abort_flag || !mbar_wait(accf, tl & 1, abort_flag)) {
        *abort_flag = 1;
        if (lane == 0 && ep.status != nullptr) atomicExch(&ep.status[b], ST_ETIMEOUT);
        break;
      }
      __syncwarp();
      tc_fence_after();
      double acc[32];
      oz_drain(tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(32 * g), acc);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(acce), 0));
      const int tm = r / tiles_n, tn = r % tiles_n;
      const int row = tm * 256 + static_cast<int>(rank) * 128 + q * 32 + lane;
      double nrm = oz_finish_tile(acc, ep, b, row, tn * OZ_BN + 32 * g, lane);
      if (ep.kind == EPI_RESID) {
        nrm = warp_sum(nrm);
        if (lane == 0)
          atomicAdd(&ep.norm2[static_cast<int64_t>(b) * ep.norm2_stride], static_cast<float>(nrm));
      }
      ++tl;
    }
  }

  if (warp == 1) mbar_wait(drain, 0);  // bounded; immediate unless a wait above gave up
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) tmem_dealloc_pair(tmem, OZ_TMEM_COLS);
}

// ------------------------------------------------------------- fp64 storage kernels
constexpr int EW = 256;

dim3 ew_grid64(int64_t count, int batch) {
  int64_t per = (count + EW * 8 - 1) / (EW * 8);
  if (per < 1) per = 1;
  if (per > 1024) per = 1024;
  return dim3(static_cast<unsigned>(per), static_cast<unsigned>(batch));
}

SHP_DEV void block_add64(double v, float* dst) {
  __shared__ double red[EW / 32];
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < EW / 32; ++w) s += red[w];
    atomicAdd(dst, static_cast<float>(s));
  }
}

// Pass 1 start: c = ||A||_F (fp64 from k_frob), Y_0 = (A + A^T) / (2c) and
// R_0 = I - Y_0 in fp64, ||R_0||^2; A^T through a padded 32 x 32 tile.
__global__ void __launch_bounds__(EW)
    k_oz_init(const float* A, int64_t n, Ctl ctl, double* Y, double* R) {
  count_kernel_run();
  __shared__ float tt[32][33];
  const int b = blockIdx.y;
  const double c = sqrt(ctl.dnorm[b]);
  if (blockIdx.x == 0 && threadIdx.x == 0) ctl.bs[b].c = static_cast<float>(c);
  const int64_t nn = n * n, T = (n + 31) / 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const float* Ab = A + b * nn;
  double nrm = 0.0;
  for (int64_t t = blockIdx.x; t < T * T; t += gridDim.x) {
    const int64_t i0 = (t / T) * 32, j0 = (t % T) * 32;
    __syncthreads();
    for (int r = ty; r < 32; r += EW / 32) {
      const int64_t row = j0 + r, col = i0 + tx;
      tt[tx][r] = (row < n && col < n) ? Ab[row * n + col] : 0.f;
    }
    __syncthreads();
    for (int r = ty; r < 32; r += EW / 32) {
      const int64_t row = i0 + r, col = j0 + tx;
      if (row >= n || col >= n) continue;
      const int64_t off = b * nn + row * n + col;
      const double y = 0.5 * (static_cast<double>(Ab[row * n + col]) + static_cast<double>(tt[r][tx])) / c;
      const double rr = (row == col ? 1.0 : 0.0) - y;
      Y[off] = y;
      R[off] = rr;
      nrm += rr * rr;
    }
  }
  block_add64(nrm, &ctl.bs[b].norm2);
}

// Pass 2 start: Y (kept in place) is the pass-1 result; R_0 = I - Y, ||R_0||^2.
__global__ void __launch_bounds__(EW) k_oz_restart(int64_t n, Ctl ctl, const double* Y, double* R) {
  count_kernel_run();
  const int b = blockIdx.y;
  const int64_t nn = n * n;
  double nrm = 0.0;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(EW) + threadIdx.x; e < nn;
       e += static_cast<int64_t>(gridDim.x) * EW) {
    const int64_t off = b * nn + e;
    const double r = ((e / n) == (e % n) ? 1.0 : 0.0) - Y[off];
    R[off] = r;
    nrm += r * r;
  }
  block_add64(nrm, &ctl.bs[b].norm2);
}

// d = 1: Delta = alpha R; I + Delta into D2 when non-null (Z_1 of the first step).
__global__ void __launch_bounds__(EW)
    k_oz_gform_d1(const double* R, int64_t n, Ctl ctl, const int* active, double* D, double* D2) {
  count_kernel_run();
  const int b = blockIdx.y;
  if (active[b] == 0) return;
  const double a = static_cast<double>(ctl.alpha[b]);
  const int64_t nn = n * n;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(EW) + threadIdx.x; e < nn;
       e += static_cast<int64_t>(gridDim.x) * EW) {
    const int64_t off = b * nn + e;
    const double dl = a * R[off];
    D[off] = dl;
    if (D2 != nullptr) D2[off] = ((e / n) == (e % n) ? 1.0 : 0.0) + dl;
  }
}

// X_out = c^e * S (fp32 output); with z_slots a block whose last pass made no
// step gets c^e * I (Z_0 = I is never stored).
__global__ void __launch_bounds__(EW)
    k_oz_finish(int64_t n, Ctl ctl, double e_c, const double* S, float* X, int z_slots) {
  count_kernel_run();
  const int b = blockIdx.y;
  const double c = sqrt(ctl.dnorm[b]);
  double sc;
  if (e_c == 0.5)
    sc = sqrt(c);
  else if (e_c == -0.5)
    sc = 1.0 / sqrt(c);
  else
    sc = 1.0 / sqrt(sqrt(c));
  const bool identity = z_slots != 0 && ctl.bs[b].iters == 0;
  const int64_t nn = n * n;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(EW) + threadIdx.x; e < nn;
       e += static_cast<int64_t>(gridDim.x) * EW) {
    const int64_t off = b * nn + e;
    const double v = identity ? ((e / n) == (e % n) ? 1.0 : 0.0) : S[off];
    X[off] = static_cast<float>(sc * v);
  }
}

}  // namespace

// ------------------------------------------------------------- host side
int64_t oz_ldk(int64_t k) { return (k + OZ_BK - 1) / OZ_BK * OZ_BK; }

size_t oz_slices_bytes(int64_t rows, int64_t k, int64_t batch) {
  return static_cast<size_t>(OZ_S) * rows * oz_ldk(k) * batch;
}

int oz_slice_count() { return OZ_S; }

cudaError_t oz_clear_max(unsigned* maxbuf, int rows, int cols, int batch, cudaStream_t st) {
  return cudaMemsetAsync(maxbuf, 0, sizeof(unsigned) * static_cast<size_t>(batch) * (rows + cols),
                         st);
}

cudaError_t oz_slice(const double* X, int rows, int cols, int64_t ld, int64_t bs, int batch,
                     const int* active, unsigned* maxbuf, bool have_max, const OzSlices& out,
                     float* x32, cudaStream_t st) {
  if (rows <= 0 || cols <= 0 || batch <= 0) return cudaSuccess;
  unsigned* rmax = maxbuf;
  unsigned* cmax = maxbuf + static_cast<int64_t>(batch) * rows;
  if (!have_max) {
    cudaError_t e = oz_clear_max(maxbuf, rows, cols, batch, st);
    if (e != cudaSuccess) return e;
    const dim3 grid((cols + SL_T - 1) / SL_T, (rows + SL_T - 1) / SL_T, batch);
    k_oz_absmax<<<grid, 256, 0, st>>>(X, rows, cols, ld, bs, active, rmax, cmax);
  }
  // the slicing tiles cover whole K blocks (digits 0 past the matrix edge)
  const dim3 grid2((oz_ldk(cols) + SL_T - 1) / SL_T, (oz_ldk(rows) + SL_T - 1) / SL_T, batch);
  k_oz_slice<<<grid2, 256, 0, st>>>(X, rows, cols, ld, bs, active, rmax, cmax, out.rows,
                                    out.cols, out.rscale, out.cscale, x32);
  return cudaGetLastError();
}

cudaError_t gemm_oz(const int8_t* Arows, const int8_t* Bcols, int M, int N, int K, int batch,
                    const OzEpi& ep, cudaStream_t st) {
  if (M <= 0 || N <= 0 || K <= 0 || batch <= 0) return cudaSuccess;
  static_assert(OZ_BK % SL_T == 0, "a K block of the slice layout is whole slicing tiles");
  CUtensorMap ma, mb;
  const int64_t nkb = (K + OZ_BK - 1) / OZ_BK;
  if (!tensor_map_slices(&ma, Arows, M, OZ_S, nkb * batch, OZ_BK, 128) ||
      !tensor_map_slices(&mb, Bcols, N, OZ_S, nkb * batch, OZ_BK, OZ_BN / 2))
    return cudaErrorInvalidValue;
  static int attr_set[64];
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = -1;
  if (dev < 0 || attr_set[dev] == 0) {
    cudaError_t e =
        cudaFuncSetAttribute(k_gemm_oz, cudaFuncAttributeMaxDynamicSharedMemorySize, OZ_SMEM);
    if (e != cudaSuccess) return e;
    if (dev >= 0) attr_set[dev] = 1;
  }
  if (dev >= 0) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int ntiles = ((N + OZ_BN - 1) / OZ_BN) * ((M + 255) / 256) * batch;
  int ncl = sms / 2;
  if (ncl > ntiles) ncl = ntiles;
  if (ncl < 1) ncl = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * ncl, 1, 1);
  cfg.blockDim = dim3(OZ_THREADS, 1, 1);
  cfg.dynamicSmemBytes = OZ_SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_gemm_oz, ma, mb, K, ep, batch);
}

cudaError_t oz_init(const float* A, int64_t n, int batch, const Ctl& ctl, double* Y, double* R,
                    cudaStream_t st) {
  k_oz_init<<<ew_grid64(n * n, batch), EW, 0, st>>>(A, n, ctl, Y, R);
  return cudaGetLastError();
}

cudaError_t oz_restart(int64_t n, int batch, const Ctl& ctl, const double* Y, double* R,
                       cudaStream_t st) {
  k_oz_restart<<<ew_grid64(n * n, batch), EW, 0, st>>>(n, ctl, Y, R);
  return cudaGetLastError();
}

cudaError_t oz_gform_d1(const double* R, int64_t n, int batch, const Ctl& ctl, double* D,
                        double* D2, cudaStream_t st, const int* active) {
  k_oz_gform_d1<<<ew_grid64(n * n, batch), EW, 0, st>>>(
      R, n, ctl, active != nullptr ? active : ctl.active, D, D2);
  return cudaGetLastError();
}

cudaError_t oz_finish(int64_t n, int batch, const Ctl& ctl, double c_exponent, const double* S,
                      float* X_out, bool z_slots, cudaStream_t st) {
  k_oz_finish<<<ew_grid64(n * n, batch), EW, 0, st>>>(n, ctl, c_exponent, S, X_out,
                                                      z_slots ? 1 : 0);
  return cudaGetLastError();
}

uint64_t kernel_runs_ozaki() {
  unsigned long long v = 0;
  if (cudaMemcpyFromSymbol(&v, g_kernel_runs, sizeof(v)) != cudaSuccess) return 0;
  return v;
}

}  // namespace shp
