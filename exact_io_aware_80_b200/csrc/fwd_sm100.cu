// fwd_sm100.cu -- attention forward on the sm_100a tensor-core path:
// TMA tile loads, tcgen05 MMAs with accumulators in tensor memory (TMEM),
// and warp-specialised roles.
//
// What it computes is the tiled online softmax of "FlashAttention 심층 분석"
// (section 3): for each query row, walk the key tiles, keep a running max m
// and running sum l, rescale the output accumulator when m grows, and divide
// by l at the end; the N x N score matrix never reaches HBM.
//
// How it maps onto one B200 SM: a persistent grid of one CTA per SM (384
// threads = 3 warpgroups) walks the (row block, head, batch) work tiles,
// longest causal row blocks first; the next tile's Q/K/V loads and first
// score MMAs overlap the current tile's epilogue.  Per work tile:
//   * two 128-row query tiles Q0, Q1 share every K/V tile the CTA loads: 256
//     consecutive rows of one head, or (causal or block-sparse GQA with an even
//     group) the same 128 rows of two heads of one KV group, whose key ranges
//     then coincide;
//   * warp 8 (one thread) issues TMA loads: Q0/Q1 once, then 128-key K and V
//     tiles into a two-stage shared-memory ring (128-byte swizzle);
//   * warp 9 (one thread) issues the tcgen05 MMAs: S_t = Q_t K_j^T into TMEM
//     (fp32, 128 columns per tile), and O_t += P_t V_j with P_t read from
//     TMEM, where the softmax warps wrote it over S_t as 16-bit pairs;
//   * warps 0-3 own the rows of Q0 and warps 4-7 those of Q1, one query row
//     per thread (TMEM lane = row): each reads its 128 scores with
//     tcgen05.ld, updates m and l in the log2 domain
//     (t = s * scale * log2 e, p = 2^(t - m)), writes P back with tcgen05.st
//     and, only when the row max grew by more than 2^8, rescales its O row
//     in TMEM (the reference max may otherwise stay stale: O and l share it,
//     so O / l is unchanged and every p stays <= 256);
//   * the MMA thread queues PV for tile 0 and the next S for tile 0 while
//     the tile-1 softmax runs, and vice versa, so the tensor core and the
//     exponential units overlap.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
// Causal tiles beyond the diagonal are skipped; the diagonal and ragged
// tail tiles are masked per row.
//
// The same kernel, instantiated with F8, is the FP8 forward pass (FA-3's
// low-precision variant; see fp8_quant.cu for the operand formats): Q, K and
// the transposed V arrive as E4M3 codes, the MMAs run as kind::f8f6f4 (K = 32
// per instruction), every block's scores are scaled by the Q and K block
// scales, P is rounded to E4M3 for the P V product, and the epilogue applies
// V's scale.
//
// Instantiated with SPARSE, it is block-sparse attention ("FlashAttention-2
// (KO)", FA-1 results: the IO-aware kernel extended with a block-sparse
// pattern): a uint8 table [B, Hq, ceil(Nq/128), ceil(Nk/128)] marks the
// 128 x 128 blocks that are computed.  A work tile visits only the K/V tiles
// that either of its query tiles marks, a query tile masks the blocks it does
// not mark, and a work tile with none writes O = 0 and LSE = -inf directly.
//
// Instantiated with DROP, it applies dropout to P ("FlashAttention 심층 분석",
// section 2: dropout is one of the fused steps): Philox4x32-10 calls (common.cuh:
// one call per 2 x 4 block of query/key pairs, one 16-bit value per pair) give
// every row its 128 keep bits per key tile, and the dropped entries of P are zeroed before
// the P V product; l keeps the sum of the undropped p, so LSE is that of the
// scores, and the epilogue multiplies O by 1 / (1 - p).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace fa {
namespace {

using namespace sm100;

constexpr int kBM = 128;     // query rows per tile (= TMEM lanes)
constexpr int kBN = 128;     // keys per K/V tile
constexpr int kTiles = 2;    // query tiles per CTA
constexpr int kStages = 2;   // K/V ring depth
constexpr int kWarpLoad = 8;
constexpr int kWarpMma = 9;   // warps 10 and 11 only complete the third warpgroup
constexpr int kThreads = 384;
// Register split: launched at 168 per thread (384 x 168 = 64512); the
// load/MMA warpgroup drops to 104 and the two softmax warpgroups rise to 200
// (2 x 128 x 200 + 128 x 104 = 64512).
constexpr int kRegsSoftmax = 200;
constexpr int kRegsControl = 104;
// Of every eight column pairs of a score block, how many take the FMA-pipe exponential
// (exp2_fma2) instead of ex2.approx: 16-bit operands, FP8 operands, 16-bit with dropout (whose
// Philox multiplies share the FMA pipe).
#ifndef FA_FWD_EXP2_EIGHTHS
#define FA_FWD_EXP2_EIGHTHS 2
#endif
#ifndef FA_FWD_F8_EXP2_EIGHTHS
#define FA_FWD_F8_EXP2_EIGHTHS 2
#endif
#ifndef FA_FWD_DROP_EXP2_EIGHTHS
#define FA_FWD_DROP_EXP2_EIGHTHS 2
#endif
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsControl <= kThreads * 168, "register split exceeds the launch");
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when m grows by more than 2^8
__host__ __device__ constexpr uint32_t col_s(int t) { return 128u * t; }        // S_t / P_t
__host__ __device__ constexpr uint32_t col_o(int t) { return 256u + 128u * t; }  // O_t

template <int D, bool F8>
struct Smem {
  static constexpr int kPanel = 128 * 128;  // one [128 rows][128 bytes] swizzled panel
  // a Q, K or V tile: 16-bit [128][D] as D / 64 panels, or E4M3 [128][D = 128] as one panel
  static constexpr int kTile = F8 ? 128 * D : (D / 64) * kPanel;
  static constexpr int kStageBytes = 2 * kPanel;  // one 64-column O panel per query tile
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTiles * kTile;
  static constexpr int kOffV = kOffK + kStages * kTile;
  static constexpr int kOffStage = kOffV + kStages * kTile;  // two 16 KB halves, one per query tile: O panels
                                                             // on their way to a TMA store
  static constexpr int kOffBar = kOffStage + kStageBytes;
  // kBarQ/kBarQEmpty: the query tiles of a work tile landed / may be replaced; kBarO + t: tile t's
  // last PV finished; kBarOFree + t: the epilogue of tile t has read O_t from TMEM;
  // kBarStageFull + t: a panel of tile t's rows is in tile t's half of the stage buffer;
  // kBarStageDone + t: the TMA store of that panel has read it
  enum { kBarQ = 0, kBarKFull = 1, kBarKEmpty = 3, kBarVFull = 5, kBarVEmpty = 7, kBarS = 9, kBarP = 11, kBarO = 13,
         kBarDrain = 15, kBarQEmpty = 16, kBarOFree = 17, kBarStageFull = 19, kBarStageDone = 21, kNumBars = 23 };
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmem + 4;
  static constexpr int kBytes = kOffAbort + 4 + 1024;  // + slack to align the base to 1024 B
  static_assert(kBytes <= 232448, "shared memory per CTA exceeded");
};

struct Params {
  void* o;
  float* lse;
  int B, Hq, Hkv, Nq, Nk;
  float scale_log2;
  int* status;
  int num_mblk;  // row units per (b, head unit): 256 rows, or 128 with paired heads
  int num_work;  // num_mblk * head units * B work tiles
  int pair;      // 1: the two query tiles are heads h, h + 1 (one KV group) over the same 128 rows
  // FP8 only: Q / K scales per 128-row block ([B,Hq,nqb], [B,Hkv,nkb]), V scale per head [B,Hkv]
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  int nqb, nkb;  // 128-row blocks of Nq and Nk (FP8 scales and the block-sparse table)
  const uint8_t* block_mask;  // block-sparse only: [B, Hq, nqb, nkb], nonzero = computed
  Dropout drop;               // dropout only
  // fp32 accumulator of the merged result (ACC only): O [B,Nq,Hq,D], LSE [B,Hq,Nq]; acc_mode 0: set,
  // 1: merge and keep, 2: merge into the outputs o, lse
  float* acc_o;
  float* acc_lse;
  int acc_mode;
};

// Log-sum-exp merge of this launch's row (O_part = r * inv, LSE_part = lse) with the fp32
// accumulator row ("FlashAttention 심층 분석", Flash-Decoding: partial results over disjoint key
// ranges combine by their log-sum-exp).  Mode 0 stores the part; otherwise the merged row
// replaces r (inv becomes 1) and lse, and mode 1 also stores it back.
template <int D>
__device__ __forceinline__ void merge_acc_row(const Params& p, long orow, long lrow, uint32_t (&r)[D], float& inv,
                                              float& lse) {
  float4* acc = reinterpret_cast<float4*>(p.acc_o + orow * D);
  if (p.acc_mode == 0) {
#pragma unroll
    for (int c = 0; c < D / 4; ++c)
      acc[c] = make_float4(__uint_as_float(r[4 * c]) * inv, __uint_as_float(r[4 * c + 1]) * inv,
                           __uint_as_float(r[4 * c + 2]) * inv, __uint_as_float(r[4 * c + 3]) * inv);
    p.acc_lse[lrow] = lse;
    return;
  }
  const float la = p.acc_lse[lrow];
  const float mx = fmaxf(la, lse);
  float wa = 0.f, wp = 0.f;
  if (mx != -INFINITY) {
    wa = ex2((la - mx) * kLog2e);
    wp = ex2((lse - mx) * kLog2e);
  }
  const float s = wa + wp;
  const float ia = s > 0.f ? wa / s : 0.f, ip = s > 0.f ? wp * inv / s : 0.f;
#pragma unroll
  for (int c = 0; c < D / 4; ++c) {
    const float4 a = acc[c];
    const float4 m = make_float4(ia * a.x + ip * __uint_as_float(r[4 * c]), ia * a.y + ip * __uint_as_float(r[4 * c + 1]),
                                 ia * a.z + ip * __uint_as_float(r[4 * c + 2]),
                                 ia * a.w + ip * __uint_as_float(r[4 * c + 3]));
    r[4 * c] = __float_as_uint(m.x);
    r[4 * c + 1] = __float_as_uint(m.y);
    r[4 * c + 2] = __float_as_uint(m.z);
    r[4 * c + 3] = __float_as_uint(m.w);
    if (p.acc_mode == 1) acc[c] = m;
  }
  lse = s > 0.f ? mx + lg2(s) * kLn2 : -INFINITY;
  if (p.acc_mode == 1) p.acc_lse[lrow] = lse;
  inv = 1.f;
}

// Work tile w of the persistent schedule: row block, query head, batch.  Causal
// row blocks are enumerated longest first (all heads and batches of one length
// together).  CTA i takes one tile per round k, snaking across the grid:
// w = k G + i on even rounds and k G + (G - 1 - i) on odd ones, which balances
// the decreasing tile lengths across SMs (work_index below).
struct Work {
  int mblk, hq, b;  // row unit, first query head, batch
};
// The two query tiles of a work tile: rows 256 mblk .. + 255 of head hq (tile t: 128 rows at
// 256 mblk + 128 t), or, with paired heads, rows 128 mblk .. + 127 of heads hq and hq + 1, which
// share one KV head (GQA groups of even size) and so need exactly the same K/V tiles -- no key
// tile is computed for one query tile and masked away for the other.
__device__ __forceinline__ int tile_row(const Params& p, const Work& x, int t) {
  return p.pair ? x.mblk * kBM : x.mblk * (kTiles * kBM) + t * kBM;
}
__device__ __forceinline__ int tile_head(const Params& p, const Work& x, int t) { return x.hq + (p.pair ? t : 0); }
__device__ __forceinline__ int work_index(int round) {
  const int G = gridDim.x, i = blockIdx.x;
  return round * G + ((round & 1) ? (G - 1 - i) : i);
}
template <bool CAUSAL>
__device__ __forceinline__ Work work_at(const Params& p, int w) {
  const int hunits = p.pair ? p.Hq / 2 : p.Hq;
  const int per_len = hunits * p.B;
  const int r = w / per_len, rest = w % per_len;
  Work x;
  x.mblk = CAUSAL ? p.num_mblk - 1 - r : r;
  x.hq = (rest % hunits) * (p.pair ? 2 : 1);
  x.b = rest / hunits;
  return x;
}

template <typename T, int D, bool CAUSAL, bool F8, bool SPARSE, bool DROP, bool ACC = false>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO, Params p) {
  using L = Smem<D, F8>;
  constexpr int kExpFma8 = F8 ? FA_FWD_F8_EXP2_EIGHTHS : DROP ? FA_FWD_DROP_EXP2_EIGHTHS : FA_FWD_EXP2_EIGHTHS;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* gb = smem_raw + (sb - raw);
  auto bar = [&](int i) { return sb + L::kOffBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + L::kOffAbort);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int off = p.Nk - p.Nq;
  auto blocks_of = [&](const Work& x) {  // K/V tiles a work tile visits (causal rows stop at their diagonal)
    const int rows_end = (x.mblk + 1) * (p.pair ? kBM : kTiles * kBM);
    const int n_end = CAUSAL ? min(p.Nk, rows_end + off) : p.Nk;
    return (n_end + kBN - 1) / kBN;
  };
  // block-sparse: the table row of query tile t of a work tile (null past Nq), and the first
  // K/V tile >= j below nblk that either query tile marks (j itself for dense attention)
  auto mask_row = [&](const Work& x, int t) -> const uint8_t* {
    const int qb = tile_row(p, x, t) / kBM;
    if (qb >= p.nqb) return nullptr;
    const long mi = (((long)x.b * p.Hq + tile_head(p, x, t)) * p.nqb + qb) * p.nkb;
    if (!FA_IN_BOUNDS(p.status, mi + p.nkb - 1, (long)p.B * p.Hq * p.nqb * p.nkb)) return nullptr;
    return p.block_mask + mi;
  };
  auto next_vis = [&](const Work& x, int j, int nblk) {
    if constexpr (SPARSE) {
      const uint8_t* r0 = mask_row(x, 0);
      const uint8_t* r1 = mask_row(x, 1);
      while (j < nblk && !(r0[j] || (r1 && r1[j]))) ++j;
    }
    return j;
  };

  if (tid == 0) {
    for (int i = 0; i < L::kNumBars; ++i)
      mbar_init(bar(i), (i == L::kBarP || i == L::kBarP + 1 || i == L::kBarOFree || i == L::kBarOFree + 1 ||
                         i == L::kBarStageFull || i == L::kBarStageFull + 1)
                            ? kBM
                            : 1);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kWarpMma) {
    tmem_alloc(sb + L::kOffTmem, 512);
    tmem_relinquish();
  }
  if (warp == kWarpLoad && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(gb + L::kOffTmem);

  if (warp >= kWarpLoad) {
   regs_decrease<kRegsControl>();
   if (warp == kWarpLoad) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int last_u[kStages] = {-1, -1};
      int last_q = -1;
      int g = 0;  // K/V tiles loaded so far by this CTA (ring position)
      int we = 0;  // work tiles with at least one K/V tile so far (the per-work-tile barrier phases)
      for (int wl = 0, w = work_index(0); w < p.num_work; w = work_index(++wl)) {
        const Work x = work_at<CAUSAL>(p, w);
        const int hk = x.hq / (p.Hq / p.Hkv);
        const int nblk = blocks_of(x);
        if constexpr (SPARSE) {
          if (next_vis(x, 0, nblk) >= nblk) continue;  // nothing to load: the softmax warps write zeros
        } else {
          we = wl;  // every dense work tile visits a K/V tile
        }
        // the previous tile's last score MMAs must have read Q before it is replaced
        if (we > 0 && !mbar_wait(bar(L::kBarQEmpty), (we - 1) & 1, abort_flag, p.status)) break;
        mbar_expect_tx(bar(L::kBarQ), kTiles * L::kTile);
#pragma unroll
        for (int t = 0; t < kTiles; ++t) {
          if constexpr (F8) {
            tma_load_4d(sb + L::kOffQ + t * L::kTile, &tmQ, bar(L::kBarQ), 0, tile_head(p, x, t), tile_row(p, x, t),
                        x.b);
          } else {
#pragma unroll
            for (int pn = 0; pn < D / 64; ++pn)
              tma_load_4d(sb + L::kOffQ + t * L::kTile + pn * L::kPanel, &tmQ, bar(L::kBarQ), 64 * pn,
                          tile_head(p, x, t), tile_row(p, x, t), x.b);
          }
        }
        last_q = we++;
        bool stop = false;
        for (int j = next_vis(x, 0, nblk); j < nblk; j = next_vis(x, j + 1, nblk), ++g) {
          const int st = g & 1, u = g >> 1;
          if (u > 0 && !mbar_wait(bar(L::kBarKEmpty + st), (u - 1) & 1, abort_flag, p.status)) {
            stop = true;
            break;
          }
          mbar_expect_tx(bar(L::kBarKFull + st), L::kTile);
          if constexpr (F8) {
            tma_load_4d(sb + L::kOffK + st * L::kTile, &tmK, bar(L::kBarKFull + st), 0, hk, j * kBN, x.b);
          } else {
#pragma unroll
            for (int pn = 0; pn < D / 64; ++pn)
              tma_load_4d(sb + L::kOffK + st * L::kTile + pn * L::kPanel, &tmK, bar(L::kBarKFull + st), 64 * pn, hk,
                          j * kBN, x.b);
          }
          if (u > 0 && !mbar_wait(bar(L::kBarVEmpty + st), (u - 1) & 1, abort_flag, p.status)) {
            last_u[st] = u;  // K of this use is in flight
            stop = true;
            break;
          }
          mbar_expect_tx(bar(L::kBarVFull + st), L::kTile);
          if constexpr (F8) {
            // V transposed: [d rows][128 keys], keys innermost
            tma_load_4d(sb + L::kOffV + st * L::kTile, &tmV, bar(L::kBarVFull + st), j * kBN, 0, hk, x.b);
          } else {
#pragma unroll
            for (int pn = 0; pn < D / 64; ++pn)
              tma_load_4d(sb + L::kOffV + st * L::kTile + pn * L::kPanel, &tmV, bar(L::kBarVFull + st), 64 * pn, hk,
                          j * kBN, x.b);
          }
          last_u[st] = u;
        }
        if (stop) break;
      }
      if (*abort_flag) {
        // let every copy this thread issued land before the CTA releases its shared memory
        if (last_q >= 0) wait_drain(bar(L::kBarQ), last_q & 1, p.status);
        for (int st = 0; st < kStages; ++st)
          if (last_u[st] >= 0) {
            wait_drain(bar(L::kBarKFull + st), last_u[st] & 1, p.status);
            wait_drain(bar(L::kBarVFull + st), last_u[st] & 1, p.status);
          }
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr bool kBf16 = Elem<T>::kBf16;
      constexpr uint32_t idq = F8 ? idesc_e4m3(kBM, kBN) : idesc_f16(kBf16, kBM, kBN, false);
      constexpr uint32_t idv = F8 ? idesc_e4m3(kBM, D) : idesc_f16(kBf16, kBM, D, true);
      auto qk = [&](int t, int st) {
        if constexpr (F8) {
          // 32 E4M3 values of d = 32 bytes per step along the 128-byte rows
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            const uint64_t a = sdesc_sw128(sb + L::kOffQ + t * L::kTile + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(sb + L::kOffK + st * L::kTile + kk * 32, 16, 1024);
            mma_ss_f8(tbase + col_s(t), a, bd, idq, kk > 0 ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t ko = (kk >> 2) * L::kPanel + (kk & 3) * 32;
            const uint64_t a = sdesc_sw128(sb + L::kOffQ + t * L::kTile + ko, 16, 1024);
            const uint64_t bd = sdesc_sw128(sb + L::kOffK + st * L::kTile + ko, 16, 1024);
            mma_ss(tbase + col_s(t), a, bd, idq, kk > 0 ? 1u : 0u);
          }
        }
      };
      auto pv = [&](int t, int st, bool first) {
        if constexpr (F8) {
          // P: 4 E4M3 codes per TMEM column (32 keys = 8 columns per step); V^T K-major
#pragma unroll
          for (int kk = 0; kk < kBN / 32; ++kk) {
            const uint64_t bd = sdesc_sw128(sb + L::kOffV + st * L::kTile + kk * 32, 16, 1024);
            mma_ts_f8(tbase + col_o(t), tbase + col_s(t) + kk * 8, bd, idv, (!first || kk > 0) ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            // V stored [keys][d]: B is N(=d)-major; 16 keys = two 8-row groups of 128 B
            const uint64_t bd = sdesc_sw128(sb + L::kOffV + st * L::kTile + kk * 2048, L::kPanel, 1024);
            mma_ts(tbase + col_o(t), tbase + col_s(t) + kk * 8, bd, idv, (!first || kk > 0) ? 1u : 0u);
          }
        }
      };
      bool ok = true;
      int g = 0;  // K/V tiles consumed so far by this CTA; S/P barriers complete once per tile
      int we = 0;  // work tiles with at least one K/V tile so far
      for (int wl = 0, w = work_index(0); ok && w < p.num_work; w = work_index(++wl)) {
        const Work x = work_at<CAUSAL>(p, w);
        const int nblk = blocks_of(x);
        const int j0 = next_vis(x, 0, nblk);
        if constexpr (SPARSE) {
          if (j0 >= nblk) continue;
        } else {
          we = wl;
        }
        ok = mbar_wait(bar(L::kBarQ), we & 1, abort_flag, p.status) &&
             mbar_wait(bar(L::kBarKFull + (g & 1)), (g >> 1) & 1, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        // the previous tile's last PV ran before these in issue order; its S/P buffers are free
        qk(0, g & 1);
        mma_commit(bar(L::kBarS + 0));
        qk(1, g & 1);
        mma_commit(bar(L::kBarS + 1));
        mma_commit(bar(L::kBarKEmpty + (g & 1)));
        if (next_vis(x, j0 + 1, nblk) >= nblk) mma_commit(bar(L::kBarQEmpty));
        for (int j = j0; j < nblk; ++g) {
          const int jn = next_vis(x, j + 1, nblk);  // the next K/V tile of this work tile
          const int st = g & 1, u = g >> 1;
          const bool more = jn < nblk;
          const int st1 = (g + 1) & 1, u1 = (g + 1) >> 1;
          ok = mbar_wait(bar(L::kBarVFull + st), u & 1, abort_flag, p.status) &&
               mbar_wait(bar(L::kBarP + 0), g & 1, abort_flag, p.status);
          // the first PV of a tile overwrites O_0: the previous tile's epilogue must have read it
          if (ok && j == j0 && we > 0) ok = mbar_wait(bar(L::kBarOFree + 0), (we - 1) & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
          pv(0, st, j == j0);
          if (!more) mma_commit(bar(L::kBarO + 0));
          if (more) {
            ok = mbar_wait(bar(L::kBarKFull + st1), u1 & 1, abort_flag, p.status);
            if (!ok) break;
            tc_fence_after();
            qk(0, st1);  // overwrites S0/P0 after PV0 in issue order
            mma_commit(bar(L::kBarS + 0));
          }
          ok = mbar_wait(bar(L::kBarP + 1), g & 1, abort_flag, p.status);
          if (ok && j == j0 && we > 0) ok = mbar_wait(bar(L::kBarOFree + 1), (we - 1) & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
          pv(1, st, j == j0);
          if (!more) {
            mma_commit(bar(L::kBarO + 1));
            mma_commit(bar(L::kBarVEmpty + st));  // inside a work tile the softmax warps free V (below)
          }
          if (more) {
            qk(1, st1);
            mma_commit(bar(L::kBarS + 1));  // also frees K of tile g + 1 and V of tile g (see the softmax)
            if (next_vis(x, jn + 1, nblk) >= nblk) mma_commit(bar(L::kBarQEmpty));  // last score MMAs issued
          }
          j = jn;
        }
        ++we;
      }
      // no MMA may still run when TMEM is released
      mma_commit(bar(L::kBarDrain));
      wait_drain(bar(L::kBarDrain), 0, p.status);
    }
   }
  } else {
    regs_increase<kRegsSoftmax>();
    // ------------------------------------------------------------------ softmax + epilogue
    const int t = warp >> 2;
    const int wq = warp & 3;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tbase + lane_off + col_s(t);
    const uint32_t tO = tbase + lane_off + col_o(t);
    const float c = p.scale_log2;
    bool ok = true;
    int g = 0;  // K/V tiles processed so far by this CTA
    int we = 0;  // work tiles with at least one K/V tile so far
    for (int wl = 0, w = work_index(0); ok && w < p.num_work; w = work_index(++wl)) {
      const Work x = work_at<CAUSAL>(p, w);
      const int h = tile_head(p, x, t), b = x.b;
      const int nblk = blocks_of(x);
      const int row_first = tile_row(p, x, t);
      const int row = row_first + wq * 32 + lane;
      const int j0 = next_vis(x, 0, nblk);
      if constexpr (SPARSE) {
        if (j0 >= nblk) {
          // block-sparse work tile with no K/V tile: every row attends to nothing
          if (row < p.Nq) {
            const long oi = (((long)b * p.Nq + row) * p.Hq + h) * D;
            if (FA_IN_BOUNDS(p.status, oi + D - 1, (long)p.B * p.Nq * p.Hq * D)) {
              uint4* orow = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + oi);
#pragma unroll
              for (int i = 0; i < D / 8; ++i) orow[i] = make_uint4(0u, 0u, 0u, 0u);
            }
            const long li = ((long)b * p.Hq + h) * p.Nq + row;
            if (FA_IN_BOUNDS(p.status, li, (long)p.B * p.Hq * p.Nq)) p.lse[li] = -INFINITY;
          }
          continue;
        }
      } else {
        we = wl;
      }
      const uint8_t* mrow = nullptr;  // this query tile's block-sparse table row
      if constexpr (SPARSE) mrow = mask_row(x, t);
      const int hk = h / (p.Hq / p.Hkv);
      float cq = c;  // FP8: times the Q tile's block scale
      if constexpr (F8) {
        const long si = ((long)b * p.Hq + h) * p.nqb + min(row_first / kBM, p.nqb - 1);
        cq = FA_IN_BOUNDS(p.status, si, (long)p.B * p.Hq * p.nqb) ? c * p.q_scale[si] : 0.f;
      }
      float m_ref = -INFINITY, l = 0.f;
      for (int j = j0; j < nblk; j = next_vis(x, j + 1, nblk), ++g) {
        uint32_t keep[4] = {0u, 0u, 0u, 0u};  // dropout: bit c = (this row, key j kBN + c) kept
        if constexpr (DROP) {
          // drawn before the scores arrive (they need neither), four independent Philox calls at a
          // time.  Lanes 2m and 2m + 1 hold the two rows of one query pair, which share every call
          // (a key quad): each lane makes the calls of every other quad, keeps both rows' bits and
          // hands the other row's to its partner (lane ^ 1)
          const uint32_t rh = (uint32_t)row >> 1, bh = (uint32_t)(b * p.Hq + h);
          const int e = row & 1;  // == lane & 1
          uint32_t own[4] = {0u, 0u, 0u, 0u}, other[4] = {0u, 0u, 0u, 0u};
#pragma unroll 1
          for (int t2 = 0; t2 < 4; ++t2) {
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
              const int c = 32 * wd + 8 * t2 + 4 * e;  // keys j kBN + c .. c + 3: this lane's quad
              const uint4 w = philox4x32_10((uint32_t)(j * kBN + c) >> 2, rh, bh, p.drop.offset, p.drop.seed_lo,
                                            p.drop.seed_hi);
              const uint32_t even = keep_quad(w.x, w.y, p.drop.thr), odd = keep_quad(w.z, w.w, p.drop.thr);
              own[wd] |= (e ? odd : even) << (c & 31);
              other[wd] |= (e ? even : odd) << (c & 31);
            }
          }
#pragma unroll
          for (int wd = 0; wd < 4; ++wd) keep[wd] = own[wd] | __shfl_xor_sync(0xffffffffu, other[wd], 1);
        }
        float cj = cq;  // FP8: times the K block's scale, loaded before the scores arrive
        if constexpr (F8) {
          const long si = ((long)b * p.Hkv + hk) * p.nkb + j;
          cj = FA_IN_BOUNDS(p.status, si, (long)p.B * p.Hkv * p.nkb) ? cq * p.k_scale[si] : 0.f;
        }
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarS + t), g & 1, abort_flag, p.status));
        if (!ok) break;
        if (t == 1 && wq == 0 && lane == 0 && j != j0) {
          // S_1 of tile g is complete, and with it every MMA issued before it: the score MMAs
          // of tile g (its K stage is free) and P_1 V of tile g - 1 (its V stage is free).  This
          // arrival stands in for two MMA commits per key tile; the first tile of a work tile
          // and the last one's V are still freed by commits.
          mbar_arrive(bar(L::kBarKEmpty + (g & 1)));
          mbar_arrive(bar(L::kBarVEmpty + ((g - 1) & 1)));
        }
        tc_fence_after();
        float s[kBN];
        {
          uint32_t r0[32], r1[32], r2[32], r3[32];
          tmem_ld32(tS + 0, r0);
          tmem_ld32(tS + 32, r1);
          tmem_ld32(tS + 64, r2);
          tmem_ld32(tS + 96, r3);
          tmem_wait_ld();
          reg_fence(r0);
          reg_fence(r1);
          reg_fence(r2);
          reg_fence(r3);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            s[i] = __uint_as_float(r0[i]);
            s[32 + i] = __uint_as_float(r1[i]);
            s[64 + i] = __uint_as_float(r2[i]);
            s[96 + i] = __uint_as_float(r3[i]);
          }
        }
        const int kbase = j * kBN;
        bool on = true;  // block-sparse: this query tile computes block (., j)
        if constexpr (SPARSE) on = mrow && mrow[j];
        if (!on || kbase + kBN > p.Nk || (CAUSAL && kbase + kBN - 1 > row_first + off)) {
          int lim = on ? p.Nk - kbase : 0;
          if (CAUSAL) lim = min(lim, row + off + 1 - kbase);
#pragma unroll
          for (int i = 0; i < kBN; ++i)
            if (i >= lim) s[i] = -INFINITY;
        }
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < kBN; i += 8) {
          mx[0] = max3(mx[0], s[i], s[i + 1]);
          mx[1] = max3(mx[1], s[i + 2], s[i + 3]);
          mx[2] = max3(mx[2], s[i + 4], s[i + 5]);
          mx[3] = max3(mx[3], s[i + 6], s[i + 7]);
        }
        const float mxs = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * cj;
        const bool resc = mxs > m_ref + kRescaleThreshold;
        const float corr = resc ? ex2(m_ref - mxs) : 1.f;
        if (resc) m_ref = mxs;
        l *= corr;
        const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
        const float2 c2 = make_float2(cj, cj), nm2 = make_float2(-mu, -mu);
        float2 rs0 = make_float2(0.f, 0.f), rs1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const int c0 = 64 * half + 2 * i;
            const float2 a = exp2_pair8<kExpFma8>(__ffma2_rn(make_float2(s[c0], s[c0 + 1]), c2, nm2), 32 * half + i);
            const float2 bb =
                exp2_pair8<kExpFma8>(__ffma2_rn(make_float2(s[c0 + 2], s[c0 + 3]), c2, nm2), 32 * half + i + 1);
            rs0 = __fadd2_rn(rs0, a);
            rs1 = __fadd2_rn(rs1, bb);
            float2 ad = a, bd = bb;  // the weights of the P V product
            if constexpr (DROP) {
              const uint32_t kw = keep[c0 >> 5], sh = c0 & 31;
              ad.x = (kw >> sh) & 1u ? a.x : 0.f;
              ad.y = (kw >> (sh + 1)) & 1u ? a.y : 0.f;
              bd.x = (kw >> (sh + 2)) & 1u ? bb.x : 0.f;
              bd.y = (kw >> (sh + 3)) & 1u ? bb.y : 0.f;
            }
            if constexpr (F8) {
              pk[i >> 1] = pack_e4m3x4(ad.x, ad.y, bd.x, bd.y);  // keys c0 .. c0 + 3 in one column
            } else {
              pk[i] = Elem<T>::pack(ad.x, ad.y);
              pk[i + 1] = Elem<T>::pack(bd.x, bd.y);
            }
          }
          if constexpr (F8) {
            tmem_st16(tS + 16 * half, *reinterpret_cast<const uint32_t(*)[16]>(pk));
          } else {
            tmem_st32(tS + 32 * half, pk);
          }
        }
        l += (rs0.x + rs0.y) + (rs1.x + rs1.y);
        if (__any_sync(0xffffffffu, resc && j > j0)) {
#pragma unroll
          for (int q = 0; q < D / 32; ++q) {
            uint32_t r[32];
            tmem_ld32(tO + q * 32, r);
            tmem_wait_ld();
            reg_fence(r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * corr);
            tmem_st32(tO + q * 32, r);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(L::kBarP + t));
      }
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarO + t), we & 1, abort_flag, p.status));
      uint32_t r[D];
      if (ok) {
        // O_t: TMEM -> registers, then hand the TMEM columns back to the MMA thread at once
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < D / 32; ++q) tmem_ld32(tO + q * 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32 * q));
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < D / 32; ++q) reg_fence(*reinterpret_cast<uint32_t(*)[32]>(r + 32 * q));
        tc_fence_before();
        mbar_arrive(bar(L::kBarOFree + t));
      }
      if (ok) {
        float num = 1.f;  // FP8: V's scale; dropout: 1 / (1 - p)
        if constexpr (F8) num = FA_IN_BOUNDS(p.status, (long)b * p.Hkv + hk, (long)p.B * p.Hkv) ? p.v_scale[(long)b * p.Hkv + hk] : 0.f;
        if constexpr (DROP) num = p.drop.inv_keep;
        // block-sparse: a row that saw no visible key keeps m_ref = -inf (its l holds only the
        // clamped polynomial exp2 of -inf): O = 0 and LSE = -inf
        const bool any = SPARSE ? (l > 0.f && m_ref != -INFINITY) : l > 0.f;
        float inv = any ? num / l : 0.f;
        float lse_row = any ? (m_ref + lg2(l)) * kLn2 : -INFINITY;
        if constexpr (ACC) {
          const long orow = ((long)b * p.Nq + row) * p.Hq + h, lrow = ((long)b * p.Hq + h) * p.Nq + row;
          if (row < p.Nq && FA_IN_BOUNDS(p.status, orow, (long)p.B * p.Nq * p.Hq) &&
              FA_IN_BOUNDS(p.status, lrow, (long)p.B * p.Hq * p.Nq))
            merge_acc_row<D>(p, orow, lrow, r, inv, lse_row);
        }
        if (row < p.Nq && FA_IN_BOUNDS(p.status, ((long)b * p.Hq + h) * p.Nq + row, (long)p.B * p.Hq * p.Nq))
          p.lse[((long)b * p.Hq + h) * p.Nq + row] = lse_row;
        // O / l as 16-bit, one 64-column panel at a time, through this tile's own half of the
        // stage buffer (16 KB, laid out as the TMA box expects: 128-byte rows, 16-byte chunk c of
        // row r at chunk c ^ (r & 7)); the two tiles' halves are separate, so their epilogues
        // overlap.  One thread of the tile stores each panel; rows past Nq are clipped by the map.
        const int rr = wq * 32 + lane;
        const uint32_t half = sb + L::kOffStage + t * L::kPanel;
        auto o2 = [&](int i) { return Elem<T>::pack(__uint_as_float(r[i]) * inv, __uint_as_float(r[i + 1]) * inv); };
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn) {
          const int u = we * (D / 64) + pn;  // uses of this tile's half so far
          if (u > 0)
            ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarStageDone + t), (u - 1) & 1, abort_flag, p.status));
          if (!ok) break;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int cc = 8 * pn + c;
            st_shared_v4(half + rr * 128 + ((c ^ (rr & 7)) << 4), o2(8 * cc), o2(8 * cc + 2), o2(8 * cc + 4),
                         o2(8 * cc + 6));
          }
          fence_proxy_async_smem();
          mbar_arrive(bar(L::kBarStageFull + t));
          if (wq == 0 && lane == 0) {
            ok = mbar_wait(bar(L::kBarStageFull + t), u & 1, abort_flag, p.status);
            if (ok) {
              tma_store_4d(&tmO, half, 64 * pn, h, row_first, b);
              bulk_commit();
              bulk_wait_read_all();
              mbar_arrive(bar(L::kBarStageDone + t));
            }
          }
          ok = __all_sync(0xffffffffu, ok);
        }
      }
      ++we;
    }
    // stores must be complete before the CTA exits
    if (wq == 0 && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <typename T, int D, bool CAUSAL>
cudaError_t launch(const AttnArgs& a, cudaStream_t s) {
  CUtensorMap mq, mk, mv, mo;
  const bool bf16 = Elem<T>::kBf16;
  if (!make_map(&mq, a.q, bf16, D, a.Hq, a.Nq, a.B, kBM) || !make_map(&mk, a.k, bf16, D, a.Hkv, a.Nk, a.B, kBN) ||
      !make_map(&mv, a.v, bf16, D, a.Hkv, a.Nk, a.B, kBN) || !make_map(&mo, a.o, bf16, D, a.Hq, a.Nq, a.B, kBM))
    return cudaErrorInvalidValue;
  // paired heads for even GQA groups when the two query tiles' key ranges would differ otherwise
  // (causal, block-sparse); non-causal dense tiles need the same keys either way
  const int pair = ((a.Hq / a.Hkv) % 2 == 0 && (CAUSAL || a.block_mask)) ? 1 : 0;
  const int unit = pair ? kBM : kTiles * kBM;
  const int num_mblk = (a.Nq + unit - 1) / unit;
  const long long num_work = (long long)num_mblk * (pair ? a.Hq / 2 : a.Hq) * a.B;
  if (num_work > (1ll << 31) - 1) return cudaErrorInvalidValue;
  Params p{a.o, a.lse, a.B, a.Hq, a.Hkv, a.Nq, a.Nk, a.scale * kLog2e, a.status, num_mblk, (int)num_work, pair,
           nullptr, nullptr, nullptr, (a.Nq + kBM - 1) / kBM, (a.Nk + kBN - 1) / kBN, a.block_mask,
           Dropout{a.drop_thr, a.drop_inv_keep, a.seed_lo, a.seed_hi, a.drop_offset}, a.acc_o, a.acc_lse, a.acc_mode};
  if (a.acc_o) {
    auto kern = fwd_sm100_kernel<T, D, CAUSAL, false, false, false, true>;
    const int smem = Smem<D, false>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<long long>(num_work, device_sm_count());
    kern<<<grid, kThreads, smem, s>>>(mq, mk, mv, mo, p);
    return cudaGetLastError();
  }
  if (a.drop_p > 0.f) {
    auto kern = fwd_sm100_kernel<T, D, CAUSAL, false, false, true>;
    const int smem = Smem<D, false>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<long long>(num_work, device_sm_count());
    kern<<<grid, kThreads, smem, s>>>(mq, mk, mv, mo, p);
    return cudaGetLastError();
  }
  if (a.block_mask) {
    auto kern = fwd_sm100_kernel<T, D, CAUSAL, false, true, false>;
    const int smem = Smem<D, false>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<long long>(num_work, device_sm_count());
    kern<<<grid, kThreads, smem, s>>>(mq, mk, mv, mo, p);
    return cudaGetLastError();
  }
  auto kern = fwd_sm100_kernel<T, D, CAUSAL, false, false, false>;
  const int smem = Smem<D, false>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM (the shared-memory footprint allows no more), looping over work tiles
  const int grid = (int)std::min<long long>(num_work, device_sm_count());
  kern<<<grid, kThreads, smem, s>>>(mq, mk, mv, mo, p);
  return cudaGetLastError();
}

// FP8: d = 128.  Q/K maps over E4M3 [B][N][H][128] (box 128 bytes x 1 x 128 rows x 1),
// V map over the transposed codes [B][Hkv][128][Nk_pad] (box 128 keys x 128 rows x 1 x 1).
template <typename T, bool CAUSAL>
cudaError_t launch_f8(const Fp8AttnArgs& a, cudaStream_t s) {
  constexpr int D = 128;
  const uint64_t npad = (uint64_t)(a.Nk + 15) / 16 * 16;
  const uint64_t dq[4] = {D, (uint64_t)a.Hq, (uint64_t)a.Nq, (uint64_t)a.B};
  const uint64_t sq[3] = {D, (uint64_t)a.Hq * D, (uint64_t)a.Nq * a.Hq * D};
  const uint64_t dk[4] = {D, (uint64_t)a.Hkv, (uint64_t)a.Nk, (uint64_t)a.B};
  const uint64_t sk[3] = {D, (uint64_t)a.Hkv * D, (uint64_t)a.Nk * a.Hkv * D};
  const uint64_t dv[4] = {npad, D, (uint64_t)a.Hkv, (uint64_t)a.B};
  const uint64_t sv[3] = {npad, D * npad, (uint64_t)a.Hkv * D * npad};
  const uint32_t box_qk[4] = {128, 1, kBM, 1}, box_v[4] = {kBN, D, 1, 1};
  CUtensorMap mq, mk, mv, mo;
  if (!make_map_u8(&mq, a.q8, dq, sq, box_qk) || !make_map_u8(&mk, a.k8, dk, sk, box_qk) ||
      !make_map_u8(&mv, a.v8t, dv, sv, box_v) || !make_map(&mo, a.o, Elem<T>::kBf16, D, a.Hq, a.Nq, a.B, kBM))
    return cudaErrorInvalidValue;
  const int pair = ((a.Hq / a.Hkv) % 2 == 0 && CAUSAL) ? 1 : 0;
  const int unit = pair ? kBM : kTiles * kBM;
  const int num_mblk = (a.Nq + unit - 1) / unit;
  const long long num_work = (long long)num_mblk * (pair ? a.Hq / 2 : a.Hq) * a.B;
  if (num_work > (1ll << 31) - 1) return cudaErrorInvalidValue;
  const float sl2 = a.scale * kLog2e / (a.rotated ? (float)D : 1.f);
  Params p{a.o, a.lse, a.B, a.Hq, a.Hkv, a.Nq, a.Nk, sl2, a.status, num_mblk, (int)num_work, pair,
           a.q_scale, a.k_scale, a.v_scale, (a.Nq + kBM - 1) / kBM, (a.Nk + kBN - 1) / kBN, nullptr, Dropout{},
           nullptr, nullptr, 0};
  auto kern = fwd_sm100_kernel<T, D, CAUSAL, true, false, false>;
  const int smem = Smem<D, true>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = (int)std::min<long long>(num_work, device_sm_count());
  kern<<<grid, kThreads, smem, s>>>(mq, mk, mv, mo, p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const AttnArgs& a, cudaStream_t s) {
  if (a.d == 128) return a.causal ? launch<T, 128, true>(a, s) : launch<T, 128, false>(a, s);
  return a.causal ? launch<T, 64, true>(a, s) : launch<T, 64, false>(a, s);
}

}  // namespace

bool fwd_sm100_supported(const AttnArgs& a) {
  return (a.d == 64 || a.d == 128) && tma_available();
}

cudaError_t launch_fwd_sm100(const AttnArgs& a, cudaStream_t s) {
  return a.bf16 ? launch_t<__nv_bfloat16>(a, s) : launch_t<__half>(a, s);
}

cudaError_t launch_fwd_fp8_sm100(const Fp8AttnArgs& a, cudaStream_t s) {
  if (a.bf16) return a.causal ? launch_f8<__nv_bfloat16, true>(a, s) : launch_f8<__nv_bfloat16, false>(a, s);
  return a.causal ? launch_f8<__half, true>(a, s) : launch_f8<__half, false>(a, s);
}

}  // namespace fa
