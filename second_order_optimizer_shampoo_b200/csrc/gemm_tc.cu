// Batched GEMM on the sm_100a tensor cores (tcgen05) with fused epilogues.
//
// Every dense product of the Shampoo step and of the PRISM Newton-Schulz
// iteration (G G^T, G^T G, Z_k Y_k, R_k^2, Y_k g, g Z_k, X_k^T X_k, X_k g and
// the two products of the preconditioned update) runs through this kernel.
// The PRISM summary ("Sintesi Tecnica: PRISM", Contributi Chiave 3) stresses
// that the method stays dominated by GEMMs; this is that GEMM.
//
// Design (one CTA per 128 x BN output tile, BN in {64, 128, 256}):
//   warp 0 lane 0  - TMA producer: 128-byte-swizzled tiles of A and B (and of
//                    their low parts in split mode) into a STAGES-deep ring;
//   warp 1 lane 0  - MMA issuer: tcgen05.mma (M = 128, N = BN) into a TMEM
//                    accumulator, tcgen05.commit frees each smem stage;
//   all 8 warps    - epilogue: tcgen05.ld 32 lanes x 32 columns, transpose
//                    through padded smem so each warp store is one coalesced
//                    128-byte row segment, fused elementwise op, store.
// Modes: TF32 (fp32 operands read as TF32), 3xTF32 (operands kept as a TF32
// high part plus an fp32 remainder; acc += Ah*Bh + Ah*Bl + Al*Bh), BF16.
// No TMA multicast is used anywhere.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "internal.h"
#include "shp_common.cuh"

namespace shp {

namespace {

constexpr int EPI_BYTES = 8 * 32 * 33 * 4;  // epilogue staging, reuses stage memory

// Tiling.  Every operand row of a stage is one 128-byte K row (32 fp32 / 64
// bf16 elements); the split mode holds four tiles per stage (A and B, high
// and low parts).  PAIR = false: one CTA computes 128 x BN.  PAIR = true: a
// cluster of two CTAs computes 256 x BN with one tcgen05 MMA of M = 256; each
// CTA stages 128 rows of A and BN/2 rows (or columns) of B, which halves the
// B traffic per SM and leaves room for deeper pipelines.
template <int MODE, bool PAIR>
struct Cfg {
  static constexpr bool SPLIT = MODE == MODE_3XTF32;
  static constexpr int ESZ = MODE == MODE_BF16 ? 2 : 4;
  static constexpr int ROWB = 128;               // bytes of one K-major row per stage
  static constexpr int BK = ROWB / ESZ;          // K elements per stage
  static constexpr int UK = MODE == MODE_BF16 ? 16 : 8;  // K per MMA instruction
  static constexpr int KSTEPS = BK / UK;
  static constexpr int CHUNK = 128 / ESZ;        // MN elements per 128-byte MN chunk
  // K-major: 128B swizzle, 8-row core groups of 1024 B.
  static constexpr uint32_t K_LAYOUT = 2u;
  static constexpr uint32_t K_SBO = 1024u;
  // MN-major smem layout: 32-bit operands need the 32-byte-atom 128B swizzle
  // (period 4 rows); 16-bit operands use the plain 128B swizzle (8 rows).
  static constexpr uint32_t MN_LAYOUT = ESZ == 4 ? 1u : 2u;
  static constexpr uint32_t MN_SBO = ESZ == 4 ? 512u : 1024u;
  static constexpr int A_BYTES = 128 * ROWB;
  static constexpr int B_BYTES_MAX = (PAIR ? 128 : 256) * ROWB;
  static constexpr int PART_BYTES = A_BYTES + B_BYTES_MAX;
  static constexpr int STAGE_BYTES = PART_BYTES * (SPLIT ? 2 : 1);
  static constexpr int STAGES = (196608 / STAGE_BYTES) < 8 ? (196608 / STAGE_BYTES) : 8;
  static constexpr int PP_STAGES = STAGES;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 256;
  static_assert(STAGES * STAGE_BYTES >= EPI_BYTES, "epilogue staging must fit in the stages");
  static_assert(STAGES >= 2, "need a double-buffered pipeline");
};

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

// The epilogue update of RP consecutive rows of one column (EpiKind): acc
// a[r], aux x[r], old output w[r]; row dr is on the diagonal (or none).
// v[r] is what `out` receives, v2[r] what `out2` receives; returns the sum
// of squares of the first nrows values for RESID.  The kind is tested once.
template <int RP>
SHP_DEV float epi_rows(const EpiParams& ep, const float* a, const float* x, const float* w,
                       int dr, int nrows, float alpha, float eta, float* v, float* v2) {
  float sq = 0.f;
  switch (ep.kind) {
    case EPI_RESID:
#pragma unroll
      for (int r = 0; r < RP; ++r) {
        v[r] = (r == dr ? 1.f : 0.f) - a[r];
        if (r < nrows) sq += v[r] * v[r];
      }
      break;
    case EPI_GPOLY:
#pragma unroll
      for (int r = 0; r < RP; ++r) v[r] = ep.s1 * x[r] + alpha * a[r];
      break;
    case EPI_AXPY:
#pragma unroll
      for (int r = 0; r < RP; ++r) v[r] = x[r] + ep.s0 * a[r];
      break;
    case EPI_EMA:
#pragma unroll
      for (int r = 0; r < RP; ++r)
        v[r] = ep.s0 * w[r] + ep.s1 * a[r] + (r == dr ? ep.s2 : 0.f);
      break;
    case EPI_APPLY: {
      const float c = ep.s0 * eta;
#pragma unroll
      for (int r = 0; r < RP; ++r) v[r] = w[r] + c * a[r];
      break;
    }
    case EPI_MOMENTUM: {
      const float c = ep.s0 * eta;
#pragma unroll
      for (int r = 0; r < RP; ++r) {
        v2[r] = ep.s1 * x[r] + a[r];
        v[r] = w[r] + c * v2[r];
      }
      return 0.f;
    }
    default:
#pragma unroll
      for (int r = 0; r < RP; ++r) v[r] = ep.s0 * a[r];
      break;
  }
  if (ep.out2_hi != nullptr) {  // I + Delta
#pragma unroll
    for (int r = 0; r < RP; ++r) v2[r] = v[r] + (r == dr ? 1.f : 0.f);
  }
  return sq;
}

// Stores v[r] at off + r * ld for r < nrows in format fmt (one branch).
template <int RP>
SHP_DEV void store_rows(int fmt, void* hi, float* lo, int64_t off, int64_t ld, const float* v,
                        int nrows) {
  if (fmt == OUT_F32) {
    float* p = static_cast<float*>(hi) + off;
#pragma unroll
    for (int r = 0; r < RP; ++r)
      if (r < nrows) p[r * ld] = v[r];
  } else if (fmt == OUT_SPLIT) {
    float* p = static_cast<float*>(hi) + off;
    float* q = lo + off;
#pragma unroll
    for (int r = 0; r < RP; ++r) {
      if (r < nrows) {
        const float h = tf32_round(v[r]);
        p[r * ld] = h;
        q[r * ld] = tf32_round(v[r] - h);  // pre-rounded: the tensor core truncates
      }
    }
  } else {
    __nv_bfloat16* p = static_cast<__nv_bfloat16*>(hi) + off;
#pragma unroll
    for (int r = 0; r < RP; ++r)
      if (r < nrows) p[r * ld] = __float2bfloat16_rn(v[r]);
  }
}

// Epilogue of one CTA's 128 x BN accumulator, by 8 warps.  Warp (q, h) reads
// TMEM lanes 32q..32q+31 (q must be the warp's position in its warpgroup, the
// lane quarter the hardware grants it) and every other 32-column chunk
// starting at h.  Each chunk is transposed through padded shared memory `st`
// (32 x 33 floats per warp) so that a lane owns one column: its RP loads and
// RP stores per pass are independent and every warp access is one coalesced
// 128-byte row segment.  DUAL adds the second (cross-term) accumulator that
// sits BN columns further.  Returns this warp's sum of squares (RESID).
template <bool DUAL, int RP>
SHP_DEV float epilogue_tile(float* st, uint32_t tmem, const EpiParams& ep, int b, int m0, int n0,
                            int BN, int q, int h, int lane, bool mirror = false) {
  const float alpha = ep.alpha != nullptr ? ep.alpha[b] : 0.f;  // GPOLY
  const float eta = ep.alpha != nullptr ? ep.alpha[b] : 1.f;    // APPLY, MOMENTUM
  const bool diag_tile = (m0 < n0 + BN) && (n0 < m0 + 128);
  const int row0 = m0 + q * 32;
  const int rcount = ep.M - row0 < 32 ? ep.M - row0 : 32;
  const bool need_aux = ep.kind == EPI_GPOLY || ep.kind == EPI_AXPY || ep.kind == EPI_MOMENTUM;
  const bool need_old = ep.kind == EPI_EMA || ep.kind == EPI_APPLY || ep.kind == EPI_MOMENTUM;
  const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
  float nrm = 0.f;
  for (int c = h; c < BN / 32; c += 2) {
    {
      float v[32];
      tmem_ld32(trow + static_cast<uint32_t>(c * 32), v);
      if (DUAL) {
        float w[32];
        tmem_ld32(trow + static_cast<uint32_t>(BN + c * 32), w);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += w[j];
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) st[lane * 33 + j] = v[j];
    }
    __syncwarp();
    const int gj = n0 + c * 32 + lane;
    const bool colok = gj < ep.N && rcount > 0;
    const int64_t obase =
        static_cast<int64_t>(b) * ep.bso + static_cast<int64_t>(row0) * ep.ldo + gj;
    const int64_t abase =
        static_cast<int64_t>(b) * ep.bs_aux + static_cast<int64_t>(row0) * ep.lda_aux + gj;
#pragma unroll 1
    for (int r0 = 0; r0 < 32; r0 += RP) {
      float a[RP], x[RP], w[RP];
#pragma unroll
      for (int r = 0; r < RP; ++r) a[r] = st[(r0 + r) * 33 + lane];
      if (colok) {
        // All RP (or 2 RP) loads of a pass are issued before any is used:
        // rows past the edge re-read the last valid row (their results are
        // never stored), so no load sits behind a branch that would make the
        // warp wait for it before issuing the next.
        if (need_aux) {
          if (ep.aux_fmt == OUT_BF16) {
            const __nv_bfloat16* p = static_cast<const __nv_bfloat16*>(ep.aux_hi) + abase;
#pragma unroll
            for (int r = 0; r < RP; ++r) {
              const int rr = r0 + r < rcount ? r0 + r : rcount - 1;
              x[r] = __bfloat162float(p[static_cast<int64_t>(rr) * ep.lda_aux]);
            }
          } else {
            const float* p = static_cast<const float*>(ep.aux_hi) + abase;
#pragma unroll
            for (int r = 0; r < RP; ++r) {
              const int rr = r0 + r < rcount ? r0 + r : rcount - 1;
              x[r] = p[static_cast<int64_t>(rr) * ep.lda_aux];
            }
            if (ep.aux_fmt == OUT_SPLIT) {
              const float* pl = ep.aux_lo + abase;
              float y[RP];
#pragma unroll
              for (int r = 0; r < RP; ++r) {
                const int rr = r0 + r < rcount ? r0 + r : rcount - 1;
                y[r] = pl[static_cast<int64_t>(rr) * ep.lda_aux];
              }
#pragma unroll
              for (int r = 0; r < RP; ++r) x[r] += y[r];
            }
          }
        } else {
#pragma unroll
          for (int r = 0; r < RP; ++r) x[r] = 0.f;
        }
        if (need_old) {
          const float* p = static_cast<const float*>(ep.out_hi) + obase;
#pragma unroll
          for (int r = 0; r < RP; ++r) {
            const int rr = r0 + r < rcount ? r0 + r : rcount - 1;
            w[r] = p[static_cast<int64_t>(rr) * ep.ldo];
          }
        } else {
#pragma unroll
          for (int r = 0; r < RP; ++r) w[r] = 0.f;
        }
        // One branch on the kind and one on each format per pass, then
        // straight-line loops over the RP rows.
        const int nrows = rcount - r0 < RP ? rcount - r0 : RP;
        const int dr = diag_tile ? gj - row0 - r0 : -1;  // row of the diagonal, if here
        float v[RP], v2[RP];
        nrm += epi_rows<RP>(ep, a, x, w, dr, nrows, alpha, eta, v, v2);
        const int64_t off = obase + static_cast<int64_t>(r0) * ep.ldo;
        store_rows<RP>(ep.out_fmt, ep.out_hi, ep.out_lo, off, ep.ldo, v, nrows);
        if (ep.out2_hi != nullptr)
          store_rows<RP>(ep.out_fmt, ep.out2_hi, ep.out2_lo, off, ep.ldo, v2, nrows);
        if (ep.out_plain != nullptr)
          store_rows<RP>(OUT_F32, ep.out_plain, nullptr, off, ep.ldo, v, nrows);
        if (ep.out_b16 != nullptr)
          store_rows<RP>(OUT_BF16, ep.out_b16, nullptr, off, ep.ldo, v, nrows);
        if (mirror) {
#pragma unroll
          for (int r = 0; r < RP; ++r) st[(r0 + r) * 33 + lane] = v[r];
        }
      }
    }
    __syncwarp();
    if (mirror) {
      // the chunk's values, now in st, also go to the transposed position:
      // lane = row of the tile, so each store is one coalesced row segment
      if (lane < rcount) {
        const int64_t mcol = static_cast<int64_t>(row0 + lane);
#pragma unroll 4
        for (int j = 0; j < 32; ++j) {
          const int mrow = n0 + c * 32 + j;
          if (mrow >= ep.N) break;
          const int64_t off = static_cast<int64_t>(b) * ep.bso + mrow * ep.ldo + mcol;
          const float v = st[lane * 33 + j];
          put(ep.out_fmt, ep.out_hi, ep.out_lo, off, v);
          // a mirrored tile holds no diagonal element, so out2 = I + v is v here
          if (ep.out2_hi != nullptr) put(ep.out_fmt, ep.out2_hi, ep.out2_lo, off, v);
          if (ep.out_plain != nullptr) ep.out_plain[off] = v;
          if (ep.out_b16 != nullptr) put(OUT_BF16, ep.out_b16, nullptr, off, v);
        }
      }
      __syncwarp();
    }
  }
  return nrm;
}

// Tile r of one batch member: row-major over tiles_m x tiles_n, or, for a
// symmetric result, row by row over the tiles with tn >= tm.
SHP_DEV void tile_coords(int r, int tiles_n, bool sym, int& tm, int& tn) {
  if (!sym) {
    tm = r / tiles_n;
    tn = r % tiles_n;
    return;
  }
  tm = 0;
  while (r >= tiles_n - tm) {
    r -= tiles_n - tm;
    ++tm;
  }
  tn = tm + r;
}

template <int MODE, bool A_MN, bool B_MN, bool PAIR>
__global__ void __launch_bounds__(256, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tAl,
              const __grid_constant__ CUtensorMap tB, const __grid_constant__ CUtensorMap tBl,
              int K, int BN, EpiParams ep) {
  count_kernel_run();
  using C = Cfg<MODE, PAIR>;
  const int b = blockIdx.z;
  if (ep.active != nullptr && ep.active[b] == 0) return;  // uniform over a CTA pair
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  // a symmetric result on square tiles (one CTA each): blockIdx.x enumerates
  // the tiles on and above the diagonal; off-diagonal ones also write their
  // mirror image
  const bool sym = !PAIR && ep.sym != 0 && ep.M == ep.N && BN == 128;
  int tmi = static_cast<int>(blockIdx.y), tni = static_cast<int>(PAIR ? blockIdx.x >> 1 : blockIdx.x);
  if (sym) tile_coords(static_cast<int>(blockIdx.x), (ep.N + 127) / 128, true, tmi, tni);
  const int m0 = PAIR ? tmi * 256 + static_cast<int>(rank) * 128 : tmi * 128;
  const int n0 = tni * BN;
  const int bn_cta = PAIR ? BN / 2 : BN;        // B rows (or columns) this CTA stages
  const int nb0 = n0 + static_cast<int>(rank) * bn_cta;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* done = empty + C::STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Split mode keeps the two small cross products (hi*lo, lo*hi) in a second
  // accumulator: the tensor cores add into the accumulator with truncation,
  // so the large hi*hi sum should take as few of those additions as possible.
  const uint32_t ncols = static_cast<uint32_t>(C::SPLIT ? 2 * BN : BN);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tA);
    tma_prefetch_desc(&tB);
    if (C::SPLIT) {
      tma_prefetch_desc(&tAl);
      tma_prefetch_desc(&tBl);
    }
  }
  if (warp == 1) {
    if (PAIR)
      tmem_alloc_pair(tmem_slot, ncols);
    else
      tmem_alloc(tmem_slot, ncols);
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync();  // peer barriers initialised, both TMEM allocations done
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int KB = (K + C::BK - 1) / C::BK;
  const uint32_t b_bytes = static_cast<uint32_t>(bn_cta) * C::ROWB;
  const uint32_t tx = (C::A_BYTES + b_bytes) * (C::SPLIT ? 2u : 1u) * (PAIR ? 2u : 1u);
  bool timed_out = false;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer (both CTAs of a pair load their halves;
    // completion is counted on the leader's full barrier)
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % C::STAGES;
      if (kb >= C::STAGES && !mbar_wait(&empty[s], ((kb / C::STAGES) - 1) & 1)) {
        timed_out = true;
        break;
      }
      uint8_t* st = smem + s * C::STAGE_BYTES;
      const int k0 = kb * C::BK;
      if (leader) mbar_arrive_expect_tx(&full[s], tx);
      const uint32_t fbar = PAIR ? mapa_shared(smem_u32(&full[s]), 0) : smem_u32(&full[s]);
#pragma unroll 1
      for (int part = 0; part < (C::SPLIT ? 2 : 1); ++part) {
        const CUtensorMap* ma = part ? &tAl : &tA;
        const CUtensorMap* mb = part ? &tBl : &tB;
        uint8_t* sa = st + part * C::PART_BYTES;
        uint8_t* sb = sa + C::A_BYTES;
        if (A_MN) {
          for (int i = 0; i < 128 / C::CHUNK; ++i) {
            if (PAIR)
              tma_load_3d_pair(sa + i * C::BK * 128, ma, fbar, m0 + i * C::CHUNK, k0, b);
            else
              tma_load_3d(sa + i * C::BK * 128, ma, &full[s], m0 + i * C::CHUNK, k0, b);
          }
        } else {
          if (PAIR)
            tma_load_3d_pair(sa, ma, fbar, k0, m0, b);
          else
            tma_load_3d(sa, ma, &full[s], k0, m0, b);
        }
        if (B_MN) {
          for (int i = 0; i < bn_cta / C::CHUNK; ++i) {
            if (PAIR)
              tma_load_3d_pair(sb + i * C::BK * 128, mb, fbar, nb0 + i * C::CHUNK, k0, b);
            else
              tma_load_3d(sb + i * C::BK * 128, mb, &full[s], nb0 + i * C::CHUNK, k0, b);
          }
        } else {
          if (PAIR)
            tma_load_3d_pair(sb, mb, fbar, k0, nb0, b);
          else
            tma_load_3d(sb, mb, &full[s], k0, nb0, b);
        }
      }
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ---------------- MMA issuer (the leader of a pair issues for both SMs)
    const uint32_t idesc =
        instr_desc(MODE == MODE_BF16 ? 1u : 2u, A_MN, B_MN, PAIR ? 256 : 128, BN);
    const uint32_t mn_lbo = C::BK * 128;  // bytes between 128-byte MN chunks
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % C::STAGES;
      if (!mbar_wait(&full[s], (kb / C::STAGES) & 1)) {
        timed_out = true;
        break;
      }
      tc_fence_after();
      const uint32_t base = smem_u32(smem + s * C::STAGE_BYTES);
#pragma unroll
      for (int ks = 0; ks < C::KSTEPS; ++ks) {
        uint64_t ad[2], bd[2];
#pragma unroll
        for (int part = 0; part < (C::SPLIT ? 2 : 1); ++part) {
          const uint32_t sa = base + part * C::PART_BYTES;
          const uint32_t sb = sa + C::A_BYTES;
          ad[part] = A_MN ? smem_desc(sa + ks * C::UK * 128, mn_lbo, C::MN_SBO, C::MN_LAYOUT)
                          : smem_desc(sa + ks * C::UK * C::ESZ, 16, C::K_SBO, C::K_LAYOUT);
          bd[part] = B_MN ? smem_desc(sb + ks * C::UK * 128, mn_lbo, C::MN_SBO, C::MN_LAYOUT)
                          : smem_desc(sb + ks * C::UK * C::ESZ, 16, C::K_SBO, C::K_LAYOUT);
        }
        const uint32_t acc0 = (kb > 0 || ks > 0) ? 1u : 0u;
        if (MODE == MODE_BF16) {
          if (PAIR)
            mma_f16_pair(tmem, ad[0], bd[0], idesc, acc0);
          else
            mma_f16(tmem, ad[0], bd[0], idesc, acc0);
        } else if (C::SPLIT) {
          const uint32_t tsmall = tmem + static_cast<uint32_t>(BN);
          if (PAIR) {
            mma_tf32_pair(tmem, ad[0], bd[0], idesc, acc0);
            mma_tf32_pair(tsmall, ad[0], bd[1], idesc, acc0);
            mma_tf32_pair(tsmall, ad[1], bd[0], idesc, 1u);
          } else {
            mma_tf32(tmem, ad[0], bd[0], idesc, acc0);
            mma_tf32(tsmall, ad[0], bd[1], idesc, acc0);
            mma_tf32(tsmall, ad[1], bd[0], idesc, 1u);
          }
        } else {
          if (PAIR)
            mma_tf32_pair(tmem, ad[0], bd[0], idesc, acc0);
          else
            mma_tf32(tmem, ad[0], bd[0], idesc, acc0);
        }
      }
      if (PAIR)
        mma_commit_pair(&empty[s], 3);
      else
        mma_commit(&empty[s]);
    }
    if (PAIR)
      mma_commit_pair(done, 3);
    else
      mma_commit(done);
  }

  // ---------------- epilogue (all 8 warps of each CTA, on its own TMEM rows)
  if (!mbar_wait(done, 0)) timed_out = true;
  __syncwarp();
  tc_fence_after();
  const bool mirror = sym && tmi != tni;
  float nrm = epilogue_tile<C::SPLIT, 16>(reinterpret_cast<float*>(smem) + warp * (32 * 33), tmem,
                                          ep, b, m0, n0, BN, warp & 3, warp >> 2, lane, mirror);
  if (mirror) nrm *= 2.f;
  if (ep.kind == EPI_RESID) {
    nrm = warp_sum(nrm);
    if (lane == 0) atomicAdd(&ep.norm2[static_cast<int64_t>(b) * ep.norm2_stride], nrm);
  }
  if (timed_out && ep.status != nullptr) atomicExch(&ep.status[b], ST_ETIMEOUT);

  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync();
  if (warp == 1) {
    if (PAIR)
      tmem_dealloc_pair(tmem, ncols);
    else
      tmem_dealloc(tmem, ncols);
  }
}

// Persistent CTA-pair GEMM (BN = 256, M >= 256): one cluster of two CTAs per
// SM pair loops over the output tiles (tile t, t + #clusters, ...).  Warp 0
// streams operands, warp 1 of the leader issues the MMAs, warps 2..9 run the
// epilogue.  TMEM holds two 256-column accumulators: while the epilogue
// drains tile i from one, the MMAs of tile i+1 fill the other, so the
// epilogue's memory traffic hides behind the next main loop.
//   full[s]/empty[s]: operand ring (leader's full counts both CTAs' bytes;
//                     empty is signalled to both CTAs by the leader's commit)
//   accf[u]:          accumulator u complete (leader's commit, both CTAs)
//   acce[u]:          accumulator u drained (8 epilogue warps x 2 CTAs arrive
//                     on the leader's barrier)
// ------------------------------------------ lane-per-row epilogue (bf16 out)
// Eight consecutive values of format fmt at element offset off, as fp32
// (bf16: one 16-byte load; fp32: two; split: two of hi and two of lo).
SHP_DEV void ld8(int fmt, const void* hi, const float* lo, int64_t off, float* x) {
  if (fmt == OUT_BF16) {
    const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(hi) + off);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(hi) + off);
    const float4 a = p[0], b = p[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    if (fmt == OUT_SPLIT) {
      const float4* q = reinterpret_cast<const float4*>(lo + off);
      const float4 c = q[0], d = q[1];
      x[0] += c.x; x[1] += c.y; x[2] += c.z; x[3] += c.w;
      x[4] += d.x; x[5] += d.y; x[6] += d.z; x[7] += d.w;
    }
  }
}

SHP_DEV float ld1(int fmt, const void* hi, const float* lo, int64_t off) {
  if (fmt == OUT_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(hi)[off]);
  const float h = static_cast<const float*>(hi)[off];
  return fmt == OUT_SPLIT ? h + lo[off] : h;
}

// Eight values rounded to bf16, one 16-byte store at element offset off.
SHP_DEV void st8_bf16(void* hi, int64_t off, const float* v) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 t = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&t);
  }
  *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(hi) + off) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Epilogue of one CTA's 128 x 256 accumulator into a bf16 result, by 8 warps
// with a lane per row: warp (q, h) reads TMEM lanes 32q..32q+31 (the lane
// quarter of its warpgroup position q) and the 32-column chunks c = h, h + 2,
// ...; lane i holds row m0 + 32q + i of the chunk in registers, reads that
// row's aux values and writes its 32 results as four 16-byte stores, with no
// shared-memory pass and every load of a chunk issued before any use.  For
// bf16 rows (64 bytes per chunk) this measured faster than a lane-per-column
// epilogue transposed through shared memory: four times fewer instructions
// outweigh the less coalesced stores; for fp32 rows the transposed epilogue
// wins and is used instead.  Chunks that cross the matrix edge go element by
// element.  A mirrored off-diagonal tile of a symmetric result is also
// written transposed: there lanes hold consecutive columns of the image, so
// those stores are coalesced.  Needs ep.vec (16-byte aligned rows) and an
// out2_hi/out_plain-free store, or out2 in bf16 too.  Returns this lane's sum
// of squares (RESID).
SHP_DEV float epilogue_lane_rows(uint32_t tmem, const EpiParams& ep, int b, int m0, int n0, int q,
                                 int h, int lane, bool mirror) {
  const float alpha = ep.alpha != nullptr ? ep.alpha[b] : 0.f;  // GPOLY
  const float eta = ep.alpha != nullptr ? ep.alpha[b] : 1.f;    // APPLY, MOMENTUM
  const bool need_aux = ep.kind == EPI_GPOLY || ep.kind == EPI_AXPY || ep.kind == EPI_MOMENTUM;
  const bool need_old = ep.kind == EPI_EMA || ep.kind == EPI_APPLY || ep.kind == EPI_MOMENTUM;
  const int row = m0 + q * 32 + lane;
  const bool rowok = row < ep.M;
  const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
  const int64_t obase = static_cast<int64_t>(b) * ep.bso + static_cast<int64_t>(row) * ep.ldo;
  const int64_t abase =
      static_cast<int64_t>(b) * ep.bs_aux + static_cast<int64_t>(row) * ep.lda_aux;
  float nrm = 0.f;
  for (int c = h; c < 8; c += 2) {
    const int cb = n0 + c * 32;
    float a[32];
    tmem_ld32(trow + static_cast<uint32_t>(c * 32), a);  // the whole warp
    if (rowok && cb < ep.N) {
      if (cb + 32 <= ep.N) {
        float x[32], w[32];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          if (need_aux) {
            ld8(ep.aux_fmt, ep.aux_hi, ep.aux_lo, abase + cb + 8 * g, x + 8 * g);
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) x[8 * g + j] = 0.f;
          }
          if (need_old) {  // read-modify-write kinds store fp32 (never this path)
            ld8(OUT_F32, ep.out_hi, nullptr, obase + cb + 8 * g, w + 8 * g);
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) w[8 * g + j] = 0.f;
          }
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float v[8], v2[8];
          nrm += epi_rows<8>(ep, a + 8 * g, x + 8 * g, w + 8 * g, row - cb - 8 * g, 8, alpha, eta,
                             v, v2);
          st8_bf16(ep.out_hi, obase + cb + 8 * g, v);
          if (ep.out2_hi != nullptr) st8_bf16(ep.out2_hi, obase + cb + 8 * g, v2);
#pragma unroll
          for (int j = 0; j < 8; ++j) a[8 * g + j] = v[j];  // kept for the mirror image
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int col = cb + j;
          if (col < ep.N) {
            float x = need_aux ? ld1(ep.aux_fmt, ep.aux_hi, ep.aux_lo, abase + col) : 0.f;
            float w = need_old ? static_cast<const float*>(ep.out_hi)[obase + col] : 0.f;
            float v, v2;
            nrm += epi_rows<1>(ep, &a[j], &x, &w, col == row ? 0 : -1, 1, alpha, eta, &v, &v2);
            put(OUT_BF16, ep.out_hi, nullptr, obase + col, v);
            if (ep.out2_hi != nullptr) put(OUT_BF16, ep.out2_hi, nullptr, obase + col, v2);
            a[j] = v;
          }
        }
      }
      if (mirror) {
        // the image of column cb + j is row cb + j; lanes write its
        // consecutive columns m0 + 32q + lane.  A mirrored tile holds no
        // diagonal element, so out2 = I + v is v there.
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (cb + j < ep.N) {
            const int64_t off = static_cast<int64_t>(b) * ep.bso +
                                static_cast<int64_t>(cb + j) * ep.ldo + row;
            put(OUT_BF16, ep.out_hi, nullptr, off, a[j]);
            if (ep.out2_hi != nullptr) put(OUT_BF16, ep.out2_hi, nullptr, off, a[j]);
          }
        }
      }
    }
  }
  return nrm;
}

// Byte offset of 16-byte group g of row r in a box of 64-byte rows stored
// with the tensor maps' 64-byte swizzle (address bits 4-5 XOR bits 7-8).
SHP_DEV uint32_t sw64_off(int r, int g) {
  return static_cast<uint32_t>(r * 64 + ((g ^ ((r >> 1) & 3)) << 4));
}

// The lane-per-row epilogue with bulk-tensor (TMA) traffic, for bf16 results
// with no out2 (ep.vec == 2): per 32-column chunk, each
// lane packs its row's 32 results into the warp's 32 x 32 bf16 box `wbuf`
// (64-byte swizzle: conflict-free, four 16-byte stores per lane) and lane 0
// stores the box with one tensor store (tO), which also clips rows and
// columns outside the matrix.  A bf16 aux box arrives in `wbuf + 2048` by
// tensor load (tX) on the warp's barrier `abar`, one chunk ahead: the caller
// issues the tile's first chunk, each chunk issues the next; an fp32 or split
// aux is read directly, each lane its row's 32 values.  `apar` is the
// barrier's phase; `pending` tracks a load in flight (drained before exit).
// The caller runs it only for warps with rows inside the matrix (no tensor
// access starts past the last row).  Returns this lane's sum of squares
// (RESID), or sets `stop` if a wait gave up.
SHP_DEV float epilogue_rows_tma(uint32_t tmem, const CUtensorMap* tO, const CUtensorMap* tX,
                                uint8_t* wbuf, uint64_t* abar, uint32_t& apar, bool& pending,
                                const EpiParams& ep, int b, int m0, int n0, int q, int h,
                                int lane, bool mirror, volatile int* abort_flag, bool& stop) {
  const float alpha = ep.alpha != nullptr ? ep.alpha[b] : 0.f;  // GPOLY
  const bool need_aux = ep.kind == EPI_GPOLY || ep.kind == EPI_AXPY || ep.kind == EPI_MOMENTUM;
  const int row0 = m0 + q * 32;
  const int row = row0 + lane;
  const int vrows = row < ep.M ? 8 : 0;
  const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
  uint8_t* obuf = wbuf;
  uint8_t* xbuf = wbuf + 2048;
  float nrm = 0.f;
  for (int c = h; c < 8; c += 2) {
    const int cb = n0 + c * 32;
    if (cb >= ep.N) break;
    float a[32];
    tmem_ld32(trow + static_cast<uint32_t>(c * 32), a);  // the whole warp
    float x[32];
    if (need_aux && ep.aux_fmt != OUT_BF16) {  // fp32 / split aux: the lane's row, direct
      const int64_t abase = static_cast<int64_t>(b) * ep.bs_aux +
                            static_cast<int64_t>(row) * ep.lda_aux + cb;
      if (row < ep.M && cb + 32 <= ep.N) {
#pragma unroll
        for (int g = 0; g < 4; ++g) ld8(ep.aux_fmt, ep.aux_hi, ep.aux_lo, abase + 8 * g, x + 8 * g);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          x[j] = row < ep.M && cb + j < ep.N ? ld1(ep.aux_fmt, ep.aux_hi, ep.aux_lo, abase + j)
                                             : 0.f;
      }
    } else if (need_aux) {
      if (!mbar_wait(abar, apar, abort_flag)) {
        stop = true;
        return nrm;
      }
      apar ^= 1u;
      pending = false;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const uint4 u = *reinterpret_cast<const uint4*>(xbuf + sw64_off(lane, g));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          x[8 * g + 2 * i] = __uint_as_float(w[i] << 16);
          x[8 * g + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
      }
      __syncwarp();  // every lane has read the box
      const int cn = c + 2;
      if (cn < 8 && n0 + cn * 32 < ep.N) {
        if (lane == 0) {
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(abar, 2048);
          tma_load_3d(xbuf, tX, abar, n0 + cn * 32, row0, b);
        }
        pending = true;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) x[j] = 0.f;
    }
    float v[32];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const int nv = ep.N - cb - 8 * g;  // columns of this group inside the matrix
      float w0[8], v2[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) w0[j] = 0.f;
      nrm += epi_rows<8>(ep, a + 8 * g, x + 8 * g, w0, row - cb - 8 * g,
                         nv < vrows ? (nv > 0 ? nv : 0) : vrows, alpha, 1.f, v + 8 * g, v2);
    }
    if (lane == 0) bulk_wait_read_all();  // the previous store has read obuf
    __syncwarp();
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 t = __floats2bfloat162_rn(v[8 * g + 2 * i], v[8 * g + 2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&t);
      }
      *reinterpret_cast<uint4*>(obuf + sw64_off(lane, g)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_3d(tO, obuf, cb, row0, b);
      bulk_commit();
    }
    if (mirror && row < ep.M) {
      // the image of column cb + j is row cb + j; lanes write its
      // consecutive columns row0 + lane (a mirrored tile holds no diagonal)
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (cb + j < ep.N)
          put(OUT_BF16, ep.out_hi, nullptr,
              static_cast<int64_t>(b) * ep.bso + static_cast<int64_t>(cb + j) * ep.ldo + row, v[j]);
      }
    }
  }
  return nrm;
}

template <int MODE, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(320, 1)
    k_gemm_pp(const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tAl,
              const __grid_constant__ CUtensorMap tB, const __grid_constant__ CUtensorMap tBl,
              const __grid_constant__ CUtensorMap tO, const __grid_constant__ CUtensorMap tX,
              int K, EpiParams ep, int batch) {
  count_kernel_run();
  using C = Cfg<MODE, true>;
  constexpr int BN = 256;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int ncl = static_cast<int>(gridDim.x) / 2, cl = static_cast<int>(blockIdx.x) / 2;
  const int tiles_n = (ep.N + BN - 1) / BN, tiles_m = (ep.M + 255) / 256;
  // symmetric result (M == N): only the tiles on and above the diagonal
  const bool sym = ep.sym != 0 && ep.M == ep.N;
  const int per_b = sym ? tiles_n * (tiles_n + 1) / 2 : tiles_n * tiles_m;
  const int ntiles = per_b * batch;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* stage_epi = reinterpret_cast<float*>(smem + C::PP_STAGES * C::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(stage_epi + 8 * 32 * 33);
  uint64_t* empty = full + C::PP_STAGES;
  uint64_t* accf = empty + C::PP_STAGES;
  uint64_t* acce = accf + 2;
  uint64_t* drain = acce + 2;  // all MMAs of this pair complete (before TMEM is freed)
  uint64_t* never = drain + 1;  // completed by nothing: the self-test's wait
  uint64_t* auxb = never + 1;   // per epilogue warp: its aux box has landed (ep.vec == 2)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(auxb + 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(auxb + 8) + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::PP_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(&accf[u], 1);
      mbar_init(&acce[u], 16);
    }
    mbar_init(drain, 1);
    mbar_init(never, 1);
    for (int w = 0; w < 8; ++w) mbar_init(&auxb[w], 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tA);
    tma_prefetch_desc(&tB);
    if (C::SPLIT) {
      tma_prefetch_desc(&tAl);
      tma_prefetch_desc(&tBl);
    }
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, 2 * BN);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // peer barriers initialised, both TMEM allocations done
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int KB = (K + C::BK - 1) / C::BK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs)
      const uint32_t tx = (C::A_BYTES + 128u * C::ROWB) * (C::SPLIT ? 2u : 1u) * 2u;
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
        int tm, tn;
        tile_coords(r, tiles_n, sym, tm, tn);
        const int m0 = tm * 256 + static_cast<int>(rank) * 128;
        const int nb0 = tn * BN + static_cast<int>(rank) * 128;
        for (int kb = 0; kb < KB; ++kb, ++kit) {
          const int s = kit % C::PP_STAGES;
          if (kit >= C::PP_STAGES &&
              (*abort_flag || !mbar_wait(&empty[s], ((kit / C::PP_STAGES) - 1) & 1, abort_flag))) {
            *abort_flag = 1;
            if (ep.status != nullptr) atomicExch(&ep.status[b], ST_ETIMEOUT);
            stop = true;
            break;
          }
          uint8_t* st = smem + s * C::STAGE_BYTES;
          const int k0 = kb * C::BK;
          if (leader) mbar_arrive_expect_tx(&full[s], tx);
          const uint32_t fbar = mapa_shared(smem_u32(&full[s]), 0);
#pragma unroll 1
          for (int part = 0; part < (C::SPLIT ? 2 : 1); ++part) {
            const CUtensorMap* ma = part ? &tAl : &tA;
            const CUtensorMap* mb = part ? &tBl : &tB;
            uint8_t* sa = st + part * C::PART_BYTES;
            uint8_t* sb = sa + C::A_BYTES;
            if (A_MN) {
              for (int i = 0; i < 128 / C::CHUNK; ++i)
                tma_load_3d_pair(sa + i * C::BK * 128, ma, fbar, m0 + i * C::CHUNK, k0, b);
            } else {
              tma_load_3d_pair(sa, ma, fbar, k0, m0, b);
            }
            if (B_MN) {
              for (int i = 0; i < 128 / C::CHUNK; ++i)
                tma_load_3d_pair(sb + i * C::BK * 128, mb, fbar, nb0 + i * C::CHUNK, k0, b);
            } else {
              tma_load_3d_pair(sb, mb, fbar, k0, nb0, b);
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (leader of the pair)
      const uint32_t idesc = instr_desc(MODE == MODE_BF16 ? 1u : 2u, A_MN, B_MN, 256, BN);
      const uint32_t mn_lbo = C::BK * 128;
      int kit = 0, tl = 0;
      bool stop = false;
      for (int t = cl; t < ntiles && !stop; t += ncl) {
        const int b = t / per_b;
        if (ep.active != nullptr && ep.active[b] == 0) continue;
        const int u = tl & 1, use = tl >> 1;
        if (use >= 1 && (*abort_flag || !mbar_wait(&acce[u], (use - 1) & 1, abort_flag))) {
          *abort_flag = 1;
          if (ep.status != nullptr) atomicExch(&ep.status[b], ST_ETIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t dacc = tmem + static_cast<uint32_t>(u * BN);
        for (int kb = 0; kb < KB; ++kb, ++kit) {
          const int s = kit % C::PP_STAGES;
          if (*abort_flag || !mbar_wait(&full[s], (kit / C::PP_STAGES) & 1, abort_flag)) {
            *abort_flag = 1;
            if (ep.status != nullptr) atomicExch(&ep.status[b], ST_ETIMEOUT);
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t base = smem_u32(smem + s * C::STAGE_BYTES);
#pragma unroll
          for (int ks = 0; ks < C::KSTEPS; ++ks) {
            uint64_t ad[2], bd[2];
#pragma unroll
            for (int part = 0; part < (C::SPLIT ? 2 : 1); ++part) {
              const uint32_t sa = base + part * C::PART_BYTES;
              const uint32_t sb = sa + C::A_BYTES;
              ad[part] = A_MN ? smem_desc(sa + ks * C::UK * 128, mn_lbo, C::MN_SBO, C::MN_LAYOUT)
                              : smem_desc(sa + ks * C::UK * C::ESZ, 16, C::K_SBO, C::K_LAYOUT);
              bd[part] = B_MN ? smem_desc(sb + ks * C::UK * 128, mn_lbo, C::MN_SBO, C::MN_LAYOUT)
                              : smem_desc(sb + ks * C::UK * C::ESZ, 16, C::K_SBO, C::K_LAYOUT);
            }
            const uint32_t acc0 = (kb > 0 || ks > 0) ? 1u : 0u;
            if (MODE == MODE_BF16) {
              mma_f16_pair(dacc, ad[0], bd[0], idesc, acc0);
            } else {
              mma_tf32_pair(dacc, ad[0], bd[0], idesc, acc0);
              if (C::SPLIT) {
                mma_tf32_pair(dacc, ad[0], bd[1], idesc, 1u);
                mma_tf32_pair(dacc, ad[1], bd[0], idesc, 1u);
              }
            }
          }
          mma_commit_pair(&empty[s], 3);
        }
        mma_commit_pair(&accf[u], 3);
        ++tl;
      }
    }
    if (lane == 0 && leader) mma_commit_pair(drain, 3);  // after every MMA issued above
  } else {
    // ---------------- epilogue warps 2..9 (both CTAs, each on its TMEM rows)
    const int q = warp & 3, h = (warp - 2) >> 2;
    float* st = stage_epi + (warp - 2) * (32 * 33);
    // the bulk-tensor epilogue's 4 KB per warp (out box, aux box) in the same region
    uint8_t* wbuf = reinterpret_cast<uint8_t*>(stage_epi) + (warp - 2) * 4096;
    uint64_t* abar = &auxb[warp - 2];
    const bool tma_epi = ep.vec == 2;
    const bool aux_tma =
        tma_epi && (ep.kind == EPI_GPOLY || ep.kind == EPI_AXPY) && ep.aux_fmt == OUT_BF16;
    uint32_t apar = 0;
    bool pending = false;
    int tl = 0;
    for (int t = cl; t < ntiles; t += ncl) {
      const int b = t / per_b, r = t % per_b;
      if (ep.active != nullptr && ep.active[b] == 0) continue;
      const int u = tl & 1, use = tl >> 1;
      int tm, tn;
      tile_coords(r, tiles_n, sym, tm, tn);
      const int m0 = tm * 256 + static_cast<int>(rank) * 128;
      const int n0 = tn * BN;
      // rows of this warp inside the matrix (tensor traffic only for those)
      const bool rows_in = m0 + q * 32 < ep.M;
      if (aux_tma && rows_in && n0 + h * 32 < ep.N) {  // the first aux box, during the wait
        if (lane == 0) {
          mbar_arrive_expect_tx(abar, 2048);
          tma_load_3d(wbuf + 2048, &tX, abar, n0 + h * 32, m0 + q * 32, b);
        }
        pending = true;
      }
      if (*abort_flag || !mbar_wait(&accf[u], use & 1, abort_flag)) {
        *abort_flag = 1;
        if (lane == 0 && ep.status != nullptr) atomicExch(&ep.status[b], ST_ETIMEOUT);
        break;
      }
      __syncwarp();
      tc_fence_after();
      // an off-diagonal tile of a symmetric result also writes its mirror image
      // and counts twice in ||R||^2
      const bool mirror = sym && tn != tm;
      float nrm;
      if (tma_epi && !rows_in) {
        nrm = 0.f;
      } else if (tma_epi) {
        bool stop = false;
        nrm = epilogue_rows_tma(tmem + static_cast<uint32_t>(u * BN), &tO, &tX, wbuf, abar, apar,
                                pending, ep, b, m0, n0, q, h, lane, mirror, abort_flag, stop);
        if (stop) {
          *abort_flag = 1;
          if (lane == 0 && ep.status != nullptr) atomicExch(&ep.status[b], ST_ETIMEOUT);
          break;
        }
      } else if (ep.vec) {
        nrm = epilogue_lane_rows(tmem + static_cast<uint32_t>(u * BN), ep, b, m0, n0, q, h, lane,
                                 mirror);
      } else {
        nrm = epilogue_tile<false, 16>(st, tmem + static_cast<uint32_t>(u * BN), ep, b, m0, n0, BN,
                                       q, h, lane, mirror);
      }
      if (mirror) nrm *= 2.f;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&acce[u]), 0));
      if (ep.kind == EPI_RESID) {
        nrm = warp_sum(nrm);
        if (lane == 0) atomicAdd(&ep.norm2[static_cast<int64_t>(b) * ep.norm2_stride], nrm);
      }
      ++tl;
    }
    if (tma_epi) {
      // nothing of this warp's bulk traffic may outlive the CTA: a tensor load
      // left in flight by a wait that gave up lands first (bounded wait), and
      // the tensor stores complete
      if (pending) mbar_wait(abar, apar);
      if (lane == 0) bulk_wait_all();
      __syncwarp();
    }
  }

  if (warp == 1) mbar_wait(drain, 0);  // bounded; immediate unless a wait above gave up
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) tmem_dealloc_pair(tmem, 2 * BN);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map over [batch][rows][inner] with the given box and swizzle, zero
// fill outside the tensor.
bool make_map(CUtensorMap* m, const void* ptr, int esz, int64_t inner, int64_t rows,
              int64_t batch, int64_t ld, int64_t bstride, int box_inner, int box_rows,
              CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld * esz),
                           static_cast<cuuint64_t>((batch > 1 ? bstride : rows * ld) * esz)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  3, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int MODE, bool AMN, bool BMN, bool PAIR>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& al, const CUtensorMap& b,
                   const CUtensorMap& bl, int M, int N, int K, int BN, int batch,
                   const EpiParams& ep, cudaStream_t st) {
  using C = Cfg<MODE, PAIR>;
  auto kern = k_gemm_tc<MODE, AMN, BMN, PAIR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  const int tq = (N + 127) / 128;
  const bool sym = !PAIR && ep.sym != 0 && M == N && BN == 128;
  cfg.gridDim = PAIR  ? dim3(2 * ((N + BN - 1) / BN), (M + 255) / 256, batch)
                : sym ? dim3(tq * (tq + 1) / 2, 1, batch)
                      : dim3((N + BN - 1) / BN, (M + 127) / 128, batch);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = PAIR ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, al, b, bl, K, BN, ep);
}

// The lane-per-row epilogue applies: a bf16 result (and out2, if any) with no
// plain fp32 copy, and every row the epilogue reads or writes starting on a
// 16-byte boundary (base pointers aligned, row and batch strides whole
// multiples of 16 bytes in each buffer's element size).
bool lane_rows_ok(const EpiParams& ep) {
  auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  auto st = [](int64_t ld, int64_t bs, int esz) {
    return (ld * esz) % 16 == 0 && (bs * esz) % 16 == 0;
  };
  if (ep.out_fmt != OUT_BF16 || ep.out_plain != nullptr || ep.out_b16 != nullptr) return false;
  if (!al(ep.out_hi) || !st(ep.ldo, ep.bso, 2)) return false;
  if (ep.out2_hi != nullptr && !al(ep.out2_hi)) return false;
  const bool need_aux = ep.kind == EPI_GPOLY || ep.kind == EPI_AXPY || ep.kind == EPI_MOMENTUM;
  const bool need_old = ep.kind == EPI_EMA || ep.kind == EPI_APPLY || ep.kind == EPI_MOMENTUM;
  if (need_old) return false;  // read-modify-write kinds keep fp32 storage
  if (need_aux) {
    const int ea = ep.aux_fmt == OUT_BF16 ? 2 : 4;
    if (!al(ep.aux_hi) || !st(ep.lda_aux, ep.bs_aux, ea)) return false;
    if (ep.aux_fmt == OUT_SPLIT && !al(ep.aux_lo)) return false;
  }
  return true;
}

template <int MODE, bool AMN, bool BMN>
cudaError_t launch_pp(const CUtensorMap& a, const CUtensorMap& al, const CUtensorMap& b,
                      const CUtensorMap& bl, int M, int N, int K, int batch, const EpiParams& ep_in,
                      cudaStream_t st) {
  using C = Cfg<MODE, true>;
  EpiParams ep = ep_in;
  ep.vec = lane_rows_ok(ep) ? 1 : 0;
  // bf16 result boxes of 32 x 32 by tensor store (and bf16 aux boxes by
  // tensor load) when there is no second output
  CUtensorMap tO, tX;
  memset(&tO, 0, sizeof(tO));
  memset(&tX, 0, sizeof(tX));
  const bool need_aux = ep.kind == EPI_GPOLY || ep.kind == EPI_AXPY || ep.kind == EPI_MOMENTUM;
  if (ep.vec && ep.out2_hi == nullptr && ep.kind != EPI_MOMENTUM &&
      make_map(&tO, ep.out_hi, 2, N, M, batch, ep.ldo, ep.bso, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B) &&
      (!need_aux || ep.aux_fmt != OUT_BF16 ||
       make_map(&tX, ep.aux_hi, 2, N, M, batch, ep.lda_aux, ep.bs_aux, 32, 32,
                CU_TENSOR_MAP_SWIZZLE_64B)))
    ep.vec = 2;
  constexpr int SMEM = 1024 + C::PP_STAGES * C::STAGE_BYTES + 8 * 32 * 33 * 4 + 320;
  static_assert(SMEM <= 232448, "persistent pair kernel exceeds shared memory");
  auto kern = k_gemm_pp<MODE, AMN, BMN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int tn = (N + 255) / 256;
  const int ntiles = (ep.sym && M == N ? tn * (tn + 1) / 2 : tn * ((M + 255) / 256)) * batch;
  int ncl = sms / 2;
  if (ncl > ntiles) ncl = ntiles;
  if (ncl < 1) ncl = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * ncl, 1, 1);
  cfg.blockDim = dim3(320, 1, 1);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, al, b, bl, tO, tX, K, ep, batch);
}

template <int MODE>
cudaError_t dispatch_pp(bool amn, bool bmn, const CUtensorMap& a, const CUtensorMap& al,
                        const CUtensorMap& b, const CUtensorMap& bl, int M, int N, int K,
                        int batch, const EpiParams& ep, cudaStream_t st) {
  if (!amn && !bmn) return launch_pp<MODE, false, false>(a, al, b, bl, M, N, K, batch, ep, st);
  if (!amn && bmn) return launch_pp<MODE, false, true>(a, al, b, bl, M, N, K, batch, ep, st);
  if (amn && !bmn) return launch_pp<MODE, true, false>(a, al, b, bl, M, N, K, batch, ep, st);
  return launch_pp<MODE, true, true>(a, al, b, bl, M, N, K, batch, ep, st);
}

template <int MODE, bool PAIR>
cudaError_t dispatch(bool amn, bool bmn, const CUtensorMap& a, const CUtensorMap& al,
                     const CUtensorMap& b, const CUtensorMap& bl, int M, int N, int K, int BN,
                     int batch, const EpiParams& ep, cudaStream_t st) {
  if (!amn && !bmn)
    return launch<MODE, false, false, PAIR>(a, al, b, bl, M, N, K, BN, batch, ep, st);
  if (!amn && bmn)
    return launch<MODE, false, true, PAIR>(a, al, b, bl, M, N, K, BN, batch, ep, st);
  if (amn && !bmn)
    return launch<MODE, true, false, PAIR>(a, al, b, bl, M, N, K, BN, batch, ep, st);
  return launch<MODE, true, true, PAIR>(a, al, b, bl, M, N, K, BN, batch, ep, st);
}

template <int MODE>
cudaError_t dispatch_pair(bool pair, bool amn, bool bmn, const CUtensorMap& a,
                          const CUtensorMap& al, const CUtensorMap& b, const CUtensorMap& bl,
                          int M, int N, int K, int BN, int batch, const EpiParams& ep,
                          cudaStream_t st) {
  if (pair) return dispatch_pp<MODE>(amn, bmn, a, al, b, bl, M, N, K, batch, ep, st);
  return dispatch<MODE, false>(amn, bmn, a, al, b, bl, M, N, K, BN, batch, ep, st);
}

}  // namespace

bool tensor_map_slices(CUtensorMap* m, const int8_t* ptr, int64_t rows, int slices,
                       int64_t blocks, int kb_bytes, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr || (kb_bytes != 64 && kb_bytes != 128)) return false;
  const cuuint64_t kb = static_cast<cuuint64_t>(kb_bytes);
  cuuint64_t dims[4] = {kb, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(slices),
                        static_cast<cuuint64_t>(blocks)};
  cuuint64_t strides[3] = {kb, static_cast<cuuint64_t>(rows) * kb,
                           static_cast<cuuint64_t>(slices) * rows * kb};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(kb_bytes), static_cast<cuuint32_t>(box_rows),
                       static_cast<cuuint32_t>(slices), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<int8_t*>(ptr), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  kb_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool tensor_map_rows(CUtensorMap* m, const float* ptr, int64_t inner, int64_t rows,
                     int64_t batch, int64_t ld, int64_t bstride, int box_inner, int box_rows) {
  return make_map(m, ptr, 4, inner, rows, batch, ld, bstride, box_inner, box_rows,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
}

cudaError_t gemm_tc(int mode, const Operand& A, const Operand& B, int M, int N, int K,
                    int batch, const EpiParams& ep, cudaStream_t st) {
  if (M <= 0 || N <= 0 || K <= 0 || batch <= 0) return cudaSuccess;
  const int esz = mode == MODE_BF16 ? 2 : 4;
  const int rowb = 128;  // Cfg<MODE>::ROWB
  const int bk = rowb / esz, chunk = 128 / esz;
  const CUtensorMapSwizzle k_swz = rowb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  int BN = N > 128 ? 256 : (N > 64 ? 128 : 64);
  // CTA pairs (M = 256 per MMA) for full-width tiles; small problems keep one
  // CTA per 128-row tile.  When the 256 x 256 tiles would leave most SM pairs
  // idle (a few blocks, e.g. the two Kronecker factors of one weight), one CTA
  // per 128 x 128 tile puts four times as many SMs to work.
  bool pair = M >= 256 && BN == 256;
  if (pair && !ep.selftest) {  // the self-test exercises the persistent pair kernel
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int tn = (N + 255) / 256, tm = (M + 255) / 256;
    const int64_t tiles = static_cast<int64_t>(ep.sym && M == N ? tn * (tn + 1) / 2 : tn * tm) * batch;
    if (2 * tiles < sms) {
      pair = false;
      BN = 128;
      // a single block's product still leaves half the SMs idle at 128 x 128:
      // 128 x 64 tiles (a symmetric result keeps 128 x 128 and its upper
      // triangle)
      const int64_t t128 = static_cast<int64_t>((N + 127) / 128) * ((M + 127) / 128) * batch;
      if (!(ep.sym && M == N) && 2 * t128 <= sms) BN = 64;
    }
  }
  const int bn_cta = pair ? BN / 2 : BN;
  CUtensorMap ma, mal, mb, mbl;
  bool ok = true;
  // A: logical M x K.
  // MN-major tiles of 32-bit data use the 32-byte-atom swizzle (see Cfg).
  const CUtensorMapSwizzle mn_swz =
      esz == 4 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B;
  auto mapA = [&](CUtensorMap* m, const void* p) {
    return A.mn ? make_map(m, p, esz, M, K, batch, A.ld, A.bstride, chunk, bk, mn_swz)
                : make_map(m, p, esz, K, M, batch, A.ld, A.bstride, bk, 128, k_swz);
  };
  // B: logical K x N.
  auto mapB = [&](CUtensorMap* m, const void* p) {
    return B.mn ? make_map(m, p, esz, N, K, batch, B.ld, B.bstride, chunk, bk, mn_swz)
                : make_map(m, p, esz, K, N, batch, B.ld, B.bstride, bk, bn_cta, k_swz);
  };
  ok = ok && mapA(&ma, A.hi) && mapB(&mb, B.hi);
  if (mode == MODE_3XTF32) {
    if (A.lo == nullptr || B.lo == nullptr) return cudaErrorInvalidValue;
    ok = ok && mapA(&mal, A.lo) && mapB(&mbl, B.lo);
  } else {
    mal = ma;
    mbl = mb;
  }
  if (!ok) return cudaErrorInvalidValue;
  switch (mode) {
    case MODE_TF32:
      return dispatch_pair<MODE_TF32>(pair, A.mn, B.mn, ma, mal, mb, mbl, M, N, K, BN, batch,
                                      ep, st);
    case MODE_3XTF32:
      return dispatch_pair<MODE_3XTF32>(pair, A.mn, B.mn, ma, mal, mb, mbl, M, N, K, BN, batch,
                                        ep, st);
    case MODE_BF16:
      return dispatch_pair<MODE_BF16>(pair, A.mn, B.mn, ma, mal, mb, mbl, M, N, K, BN, batch,
                                      ep, st);
  }
  return cudaErrorInvalidValue;
}

uint64_t kernel_runs_gemm() {
  unsigned long long v = 0;
  if (cudaMemcpyFromSymbol(&v, g_kernel_runs, sizeof(v)) != cudaSuccess) return 0;
  return v;
}

}  // namespace shp
