// bwd_sm100.cu -- attention backward on the sm_100a tensor-core path (TMA,
// tcgen05 MMAs with accumulators in tensor memory, warp-specialised roles).
//
// The gradients are the chain rule of the definition, with P recomputed from
// the stored log-sum-exp ("FlashAttention 심층 분석", section 4: keep only the
// softmax statistics, rebuild P on chip):
//   P = exp(scale q.k - LSE),  dP = dO V^T,  dS = P * (dP - D),  D = rowsum(dO * O)
//   dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
// Two kernels, no atomics (bitwise-reproducible results):
//
// dK/dV: one CTA per (128-key tile, KV head, batch).  K and V stay in shared
//   memory; Q and dO tiles of the group's query heads stream through a
//   two-stage TMA ring.  TMEM holds S^T (keys x queries, later P^T as 16-bit
//   pairs), dP^T (later dS^T), and the dV and dK accumulators (512 columns).
//   Per query tile the MMA thread issues S^T = K Q^T, dP^T = V dO^T,
//   dV += P^T dO and dK += dS^T Q (the last two read P^T / dS^T from TMEM);
//   it queues the next tile's S^T behind dV and the next dP^T behind dK, so
//   the tensor core works while the four elementwise warps (one key row per
//   thread) turn S^T into P^T and dP^T into dS^T.
//
// dQ: one CTA per (128-row query tile, query head, batch).  Q and dO stay in
//   shared memory; K tiles stream through a three-stage ring and V tiles
//   through a two-stage ring.  TMEM: two S buffers (scores, later dS as
//   16-bit pairs), dP, and the dQ accumulator.  Per key tile: S = Q K^T,
//   dP = dO V^T, then dQ += dS K; S for tile j+2 is queued behind dQ_j so the
//   exponentials of one tile overlap the MMAs of the next.
//
// Both kernels write their outputs through shared memory (buffers that are
// free once the last MMA has run) and TMA stores.
//
// With DROP both kernels regenerate the forward pass's dropout mask (Philox
// values from the same counters, common.cuh): dV uses P * M, and dS =
// P * (M * dP / (1 - p) - D); dV is scaled by 1 / (1 - p) when stored.  A
// third warpgroup (384 threads, setmaxnreg split) draws each tile's keep bits
// into a two-slot shared-memory ring one tile ahead of the elementwise warps;
// the dQ kernel's DROP variant keeps one V stage to make room for it.
//
// Every mbarrier wait is bounded (sm100.cuh) and the roles drain in-flight
// copies and MMAs before tensor memory is released.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace fa {
namespace {

using namespace sm100;

constexpr int kT = 128;        // rows of every tile (keys or queries) = TMEM lanes
constexpr int kThreads = 192;  // warps 0-3 elementwise, 4 TMA, 5 MMA
// dK/dV with dropout: a third warpgroup (warps 8-11, one warp per SM sub-partition) draws the
// keep bits; warps 6-7 idle.  The 384 threads launch with 168 registers each; each role's branch
// then moves its warpgroup to its own budget.
constexpr int kThreadsDrop = 384;
constexpr int kRegsElem = 256, kRegsCtrl = 104, kRegsRng = 104;
static_assert(128 * (kRegsElem + kRegsCtrl + kRegsRng) <= kThreadsDrop * 168, "register split exceeds the launch");
// Of every eight column pairs, how many exponentials take the FMA pipe (exp2_fma2) instead of
// ex2.approx, without and with dropout (whose keep-bit generator shares the multiply pipe, so
// there every exponential goes to ex2.approx: 2.91 -> 2.87 ms for the dropout backward at N=8192).
#ifndef FA_BWD_EXP2_EIGHTHS
#define FA_BWD_EXP2_EIGHTHS 2
#endif
#ifndef FA_BWD_DROP_EXP2_EIGHTHS
#define FA_BWD_DROP_EXP2_EIGHTHS 0
#endif
template <bool DROP>
constexpr int kExp8 = DROP ? FA_BWD_DROP_EXP2_EIGHTHS : FA_BWD_EXP2_EIGHTHS;
constexpr int kWarpLoad = 4;
constexpr int kWarpMma = 5;
constexpr int kPanel = 128 * 128;  // [128 rows][64 cols] 16-bit panel, bytes

struct Params {
  const float* lse;
  const float* dvec;
  void* out0;  // dK (dK/dV kernel) or dQ
  void* out1;  // dV (dK/dV kernel)
  int B, Hq, Hkv, Nq, Nk;
  float scale;
  float scale_log2;
  int* status;
  Dropout drop;  // DROP only
  // ACC only: fp32 accumulators the results are added into (set when acc_init): acc0 = dK or dQ,
  // acc1 = dV, laid out like the 16-bit outputs
  float* acc0;
  float* acc1;
  int acc_init;
};

// One row of D fp32 TMEM columns, times `mul`, added into (or, with init, stored to) the fp32
// row `dst` of an accumulator; the row is this thread's own, so no other thread touches it.
// Every lane of the warp must call it (tcgen05.ld is warp-collective); lanes whose row lies
// outside the tensor pass active = false and touch no memory.
template <int D>
__device__ __forceinline__ void acc_row(uint32_t taddr, float* dst, float mul, bool init, bool active) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int q = 0; q < D / 32; ++q) {
    uint32_t x[32];
    tmem_ld32(taddr + q * 32, x);
    tmem_wait_ld();
    reg_fence(x);
    if (!active) continue;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float4 v = make_float4(__uint_as_float(x[4 * c]) * mul, __uint_as_float(x[4 * c + 1]) * mul,
                             __uint_as_float(x[4 * c + 2]) * mul, __uint_as_float(x[4 * c + 3]) * mul);
      if (!init) {
        const float4 o = d4[q * 8 + c];
        v.x += o.x;
        v.y += o.y;
        v.z += o.z;
        v.w += o.w;
      }
      d4[q * 8 + c] = v;
    }
  }
}

// One row of D fp32 TMEM columns, times `mul`, as 16-bit values into a stage tile laid out as
// a TMA box with 128-byte swizzle: 64-column panels of 128-byte rows, 16-byte chunk c of row r
// at chunk c ^ (r & 7).
template <typename T, int D>
__device__ __forceinline__ void stage_row(uint32_t taddr, uint32_t stage, int r, float mul) {
#pragma unroll
  for (int q = 0; q < D / 32; ++q) {
    uint32_t x[32];
    tmem_ld32(taddr + q * 32, x);
    tmem_wait_ld();
    reg_fence(x);
    auto pk = [&](int i) { return Elem<T>::pack(__uint_as_float(x[i]) * mul, __uint_as_float(x[i + 1]) * mul); };
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      const int cg = q * 4 + c4;  // 16-byte chunk of the row
      st_shared_v4(stage + (cg >> 3) * kPanel + r * 128 + (((cg & 7) ^ (r & 7)) << 4), pk(8 * c4), pk(8 * c4 + 2),
                   pk(8 * c4 + 4), pk(8 * c4 + 6));
    }
  }
}

// 128 fp32 TMEM columns of this thread's lane into s[].
__device__ __forceinline__ void load_row128(uint32_t taddr, float (&s)[kT]) {
  uint32_t r0[32], r1[32], r2[32], r3[32];
  tmem_ld32(taddr + 0, r0);
  tmem_ld32(taddr + 32, r1);
  tmem_ld32(taddr + 64, r2);
  tmem_ld32(taddr + 96, r3);
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

// dS = P (dP - d) column by column, written back as 16-bit pairs over the
// first 64 columns starting at `tds`; reads dP 32 columns at a time from `tdp`.
// The caller passes d negated: per column (dcol[c] = -D_c) or per row (drow = -D_i).
// When tds == tdp the writes trail the reads (columns 16c.. after 32c.. are read).
// With DROP, element c uses M * dP / (1 - p): keep bit c of `keep` (128 bits) and inv_keep.
template <typename T, bool PER_COL_D, bool DROP = false>
__device__ __forceinline__ void write_ds(uint32_t tdp, uint32_t tds, const float (&p)[kT], const float* dcol,
                                         float drow, const uint32_t (&keep)[4] = {}, float inv_keep = 1.f) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t r[32];
    tmem_ld32(tdp + q * 32, r);
    tmem_wait_ld();
    reg_fence(r);
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c0 = q * 32 + 2 * i;
      const float2 nd = PER_COL_D ? reinterpret_cast<const float2*>(dcol)[c0 >> 1] : make_float2(drow, drow);
      float2 dp = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
      if constexpr (DROP) {
        dp.x = (keep[c0 >> 5] >> (c0 & 31)) & 1u ? dp.x * inv_keep : 0.f;
        dp.y = (keep[c0 >> 5] >> ((c0 + 1) & 31)) & 1u ? dp.y * inv_keep : 0.f;
      }
      const float2 ds = __fmul2_rn(make_float2(p[c0], p[c0 + 1]), __fadd2_rn(dp, nd));
      pk[i] = Elem<T>::pack(ds.x, ds.y);
    }
    tmem_st16(tds + q * 16, pk);
  }
}

// ===========================================================================
// dK / dV
// ===========================================================================
template <int D>
struct DkdvSmem {
  static constexpr int kTile = (D / 64) * kPanel;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTile;
  static constexpr int kOffQ = 2 * kTile;   // 2 stages
  static constexpr int kOffDO = 4 * kTile;  // 2 stages
  static constexpr int kOffLse = 6 * kTile;  // [2][128] fp32, log2 domain
  static constexpr int kOffD = kOffLse + 2 * kT * 4;
  static constexpr int kOffKeep = kOffD + 2 * kT * 4;  // dropout: [2][128 keys] x 128 keep bits
  static constexpr int kOffBar = kOffKeep + 2 * kT * 16;
  // kBarOut: the elementwise threads have staged dK and dV (in the two free Q stages);
  // kBarKeepFull / kBarKeepEmpty: a slot of the keep-bit ring written / read
  enum { kBarKV = 0, kBarQFull = 1, kBarQEmpty = 3, kBarS = 5, kBarDP = 6, kBarP = 7, kBarDS = 8, kBarDone = 9,
         kBarDrain = 10, kBarLse = 11, kBarOut = 13, kBarKeepFull = 14, kBarKeepEmpty = 16, kNumBars = 18 };
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmem + 4;
  static constexpr int kBytes = kOffAbort + 4 + 1024;
};
// TMEM columns: S^T / P^T, dP^T / dS^T, dV, dK
constexpr uint32_t kColST = 0, kColDPT = 128, kColDV = 256, kColDK = 384;

template <typename T, int D, bool CAUSAL, bool DROP, bool ACC = false>
__global__ void __launch_bounds__(DROP ? kThreadsDrop : kThreads, 1)
    bwd_dkdv_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                          const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                          Params p) {
  using L = DkdvSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* gb = smem_raw + (sb - raw);
  auto bar = [&](int i) { return sb + L::kOffBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + L::kOffAbort);
  float* s_lse = reinterpret_cast<float*>(gb + L::kOffLse);
  float* s_d = reinterpret_cast<float*>(gb + L::kOffD);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // grid (Hkv, key tiles, B), dispatched x-fastest: small key tiles see the most
  // query tiles, so every head's longest work starts first
  const int kt = blockIdx.y;
  const int hk = blockIdx.x, b = blockIdx.z;
  const int G = p.Hq / p.Hkv;
  const int k0 = kt * kT;
  const int off = p.Nk - p.Nq;
  const int mstart = CAUSAL ? max(0, k0 - off) / kT : 0;
  const int nq = (p.Nq + kT - 1) / kT;
  const int per_head = nq - mstart;
  const int nt = G * per_head;  // query tiles this CTA visits
  // the dQ kernel, launched next on the stream as a programmatic dependent, reads none of this
  // kernel's outputs: let its CTAs start on SMs this grid frees (its last CTA waits for this grid)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (tid == 0) {
    for (int i = 0; i < L::kNumBars; ++i)
      mbar_init(bar(i), (i == L::kBarP || i == L::kBarDS || i >= L::kBarLse) ? kT : 1);
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
    prefetch_tmap(&tmDO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(gb + L::kOffTmem);

  if (warp >= 4 && warp < 8) {
   if constexpr (DROP) regs_decrease<kRegsCtrl>();
   if (warp == kWarpLoad) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int last_u[2] = {-1, -1};
      mbar_expect_tx(bar(L::kBarKV), 2 * L::kTile);
#pragma unroll
      for (int pn = 0; pn < D / 64; ++pn) {
        tma_load_4d(sb + L::kOffK + pn * kPanel, &tmK, bar(L::kBarKV), 64 * pn, hk, k0, b);
        tma_load_4d(sb + L::kOffV + pn * kPanel, &tmV, bar(L::kBarKV), 64 * pn, hk, k0, b);
      }
      for (int t = 0; t < nt; ++t) {
        const int st = t & 1, u = t >> 1;
        const int h = hk * G + t / per_head;
        const int i0 = (mstart + t % per_head) * kT;
        if (u > 0 && !mbar_wait(bar(L::kBarQEmpty + st), (u - 1) & 1, abort_flag, p.status)) break;
        mbar_expect_tx(bar(L::kBarQFull + st), 2 * L::kTile);
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn) {
          tma_load_4d(sb + L::kOffQ + st * L::kTile + pn * kPanel, &tmQ, bar(L::kBarQFull + st), 64 * pn, h, i0, b);
          tma_load_4d(sb + L::kOffDO + st * L::kTile + pn * kPanel, &tmDO, bar(L::kBarQFull + st), 64 * pn, h, i0,
                      b);
        }
        last_u[st] = u;
      }
      if (*abort_flag) {
        wait_drain(bar(L::kBarKV), 0, p.status);
        for (int st = 0; st < 2; ++st)
          if (last_u[st] >= 0) wait_drain(bar(L::kBarQFull + st), last_u[st] & 1, p.status);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr bool kBf16 = Elem<T>::kBf16;
      constexpr uint32_t id_kk = idesc_f16(kBf16, kT, kT, false);  // S^T, dP^T: both operands K(=d)-major
      constexpr uint32_t id_mn = idesc_f16(kBf16, kT, D, true);    // dV, dK: B = [queries][d], d contiguous
      auto kmajor = [&](uint32_t dst, uint32_t a_base, uint32_t b_base) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * kPanel + (kk & 3) * 32;
          mma_ss(tbase + dst, sdesc_sw128(a_base + ko, 16, 1024), sdesc_sw128(b_base + ko, 16, 1024), id_kk,
                 kk > 0 ? 1u : 0u);
        }
      };
      auto accum = [&](uint32_t dst, uint32_t a_col, uint32_t b_base, bool first) {
#pragma unroll
        for (int kk = 0; kk < kT / 16; ++kk)
          mma_ts(tbase + dst, tbase + a_col + kk * 8, sdesc_sw128(b_base + kk * 2048, kPanel, 1024), id_mn,
                 (!first || kk > 0) ? 1u : 0u);
      };
      const uint32_t sK = sb + L::kOffK, sV = sb + L::kOffV;
      auto sQ = [&](int st) { return sb + L::kOffQ + st * L::kTile; };
      auto sDO = [&](int st) { return sb + L::kOffDO + st * L::kTile; };
      bool ok = mbar_wait(bar(L::kBarKV), 0, abort_flag, p.status) &&
                mbar_wait(bar(L::kBarQFull), 0, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        kmajor(kColST, sK, sQ(0));
        mma_commit(bar(L::kBarS));
        kmajor(kColDPT, sV, sDO(0));
        mma_commit(bar(L::kBarDP));
        for (int t = 0; t < nt; ++t) {
          const int st = t & 1;
          const bool more = t + 1 < nt;
          ok = mbar_wait(bar(L::kBarP), t & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
          accum(kColDV, kColST, sDO(st), t == 0);
          if (more) {
            ok = mbar_wait(bar(L::kBarQFull + (st ^ 1)), ((t + 1) >> 1) & 1, abort_flag, p.status);
            if (!ok) break;
            tc_fence_after();
            kmajor(kColST, sK, sQ(st ^ 1));  // overwrites P^T after the dV MMA in issue order
            mma_commit(bar(L::kBarS));
          }
          ok = mbar_wait(bar(L::kBarDS), t & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
          accum(kColDK, kColDPT, sQ(st), t == 0);
          mma_commit(bar(L::kBarQEmpty + st));
          if (more) {
            kmajor(kColDPT, sV, sDO(st ^ 1));  // overwrites dS^T after the dK MMA in issue order
            mma_commit(bar(L::kBarDP));
          }
        }
        if (ok) mma_commit(bar(L::kBarDone));
      }
      mma_commit(bar(L::kBarDrain));
      wait_drain(bar(L::kBarDrain), 0, p.status);
    }
  }
  } else if (DROP && warp >= 8) {
    if constexpr (DROP) regs_decrease<kRegsRng>();
    // ------------------------------------------------------------------ keep bits (dropout)
    // thread rt draws the keep bits of key k0 + rt for every query tile into ring slot t & 1.
    // Lanes 4m .. 4m + 3 hold the four keys of one key quad, which share every Philox call:
    // each lane makes the calls of every fourth query pair, which give two bits (the pair's
    // queries) for each key of the quad, and the lanes swap them (lane ^ 1, ^ 2, ^ 3); four
    // independent calls are in flight at a time.
    const int rt = tid - 256;
    const int key = k0 + rt;
    const uint32_t jq = (uint32_t)key >> 2, thr = p.drop.thr;
    const int r = key & 3;  // == lane & 3
    uint4* ring = reinterpret_cast<uint4*>(gb + L::kOffKeep);
    for (int t = 0; t < nt; ++t) {
      const int slot = t & 1;
      if (t >= 2 && !__all_sync(0xffffffffu, mbar_wait(bar(L::kBarKeepEmpty + slot), ((t >> 1) - 1) & 1,
                                                       abort_flag, p.status)))
        break;
      const int i0 = (mstart + t % per_head) * kT;
      const uint32_t bh = (uint32_t)(b * p.Hq + hk * G + t / per_head);
      uint32_t a0[4] = {0u, 0u, 0u, 0u}, a1[4] = {0u, 0u, 0u, 0u};  // bits of keys 4 jq + k at this
      uint32_t a2[4] = {0u, 0u, 0u, 0u}, a3[4] = {0u, 0u, 0u, 0u};  // lane's query pairs, by word
#pragma unroll 1
      for (int t2 = 0; t2 < 4; ++t2) {
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
          // the call of the 2 x 4 block (queries i0 + cc, + 1) x (keys 4 jq .. 4 jq + 3)
          const int cc = 32 * wd + 8 * t2 + 2 * r;
          const uint4 w = philox4x32_10(jq, (uint32_t)(i0 + cc) >> 1, bh, p.drop.offset, p.drop.seed_lo,
                                        p.drop.seed_hi);
          const int sh = cc & 31;
          a0[wd] |= keep_pair(w.x & 0xFFFFu, w.z & 0xFFFFu, thr) << sh;
          a1[wd] |= keep_pair(w.x >> 16, w.z >> 16, thr) << sh;
          a2[wd] |= keep_pair(w.y & 0xFFFFu, w.w & 0xFFFFu, thr) << sh;
          a3[wd] |= keep_pair(w.y >> 16, w.w >> 16, thr) << sh;
        }
      }
      uint32_t keep[4];
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) {
        auto pick = [&](int k) { return k == 0 ? a0[wd] : k == 1 ? a1[wd] : k == 2 ? a2[wd] : a3[wd]; };
        uint32_t kw = pick(r);
        kw |= __shfl_xor_sync(0xffffffffu, pick(r ^ 1), 1);
        kw |= __shfl_xor_sync(0xffffffffu, pick(r ^ 2), 2);
        kw |= __shfl_xor_sync(0xffffffffu, pick(r ^ 3), 3);
        keep[wd] = kw;
      }
      ring[slot * kT + rt] = make_uint4(keep[0], keep[1], keep[2], keep[3]);
      mbar_arrive(bar(L::kBarKeepFull + slot));
    }
  } else {
    if constexpr (DROP) regs_increase<kRegsElem>();
    // ------------------------------------------------------------------ elementwise: one key row per thread
    const int wq = warp;
    const int jrow = wq * 32 + lane;
    const int key = k0 + jrow;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tST = tbase + lane_off + kColST, tDPT = tbase + lane_off + kColDPT;
    const float c = p.scale_log2;
    auto fetch = [&](int t, float& lv, float& dv) {
      const int h = hk * G + t / per_head;
      const int i = (mstart + t % per_head) * kT + tid;
      const long idx = ((long)b * p.Hq + h) * p.Nq + i;
      const bool in = i < p.Nq && FA_IN_BOUNDS(p.status, idx, (long)p.B * p.Hq * p.Nq);
      lv = in ? -p.lse[idx] * kLog2e : -INFINITY;  // negated; rows past Nq get P = 0
      dv = in ? -p.dvec[idx] : 0.f;                 // negated
    };
    // LSE and D of query tile t sit in shared buffer t & 1; every elementwise thread
    // writes one entry and arrives on kBarLse + buffer.  Waiting for buffer t & 1
    // also proves every thread finished reading it in iteration t - 2.
    {
      float lv, dv;
      fetch(0, lv, dv);
      s_lse[tid] = lv;
      s_d[tid] = dv;
      mbar_arrive(bar(L::kBarLse));
    }
    bool ok = true;
    for (int t = 0; t < nt; ++t) {
      const int buf = t & 1;
      const int i0 = (mstart + t % per_head) * kT;
      float nl = 0.f, nd = 0.f;
      if (t + 1 < nt) fetch(t + 1, nl, nd);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarLse + buf), (t >> 1) & 1, abort_flag, p.status));
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarS), t & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      float pv[kT];
      load_row128(tST, pv);
      const float2* nl2 = reinterpret_cast<const float2*>(s_lse + buf * kT);
      const float2 c2 = make_float2(c, c);
#pragma unroll
      for (int cc = 0; cc < kT; cc += 2) {
        const float2 x =
            exp2_pair8<kExp8<DROP>>(__ffma2_rn(make_float2(pv[cc], pv[cc + 1]), c2, nl2[cc >> 1]), cc >> 1);
        pv[cc] = x.x;
        pv[cc + 1] = x.y;
      }
      if (CAUSAL && k0 + kT - 1 > i0 + off) {
        const int lim = key - off - i0;  // queries i0 + cc with cc < lim cannot see this key
#pragma unroll
        for (int cc = 0; cc < kT; ++cc)
          if (cc < lim) pv[cc] = 0.f;
      }
      uint32_t keep[4] = {0u, 0u, 0u, 0u};  // dropout: bit cc = (query i0 + cc, this key) kept
      if constexpr (DROP) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarKeepFull + (t & 1)), (t >> 1) & 1, abort_flag, p.status));
        if (!ok) break;
        const uint4 kq = reinterpret_cast<const uint4*>(gb + L::kOffKeep)[(t & 1) * kT + jrow];
        keep[0] = kq.x;
        keep[1] = kq.y;
        keep[2] = kq.z;
        keep[3] = kq.w;
        mbar_arrive(bar(L::kBarKeepEmpty + (t & 1)));
      }
      {
        auto pd = [&](int c) { return DROP && !((keep[c >> 5] >> (c & 31)) & 1u) ? 0.f : pv[c]; };
        uint32_t pk0[32], pk1[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          pk0[i] = Elem<T>::pack(pd(2 * i), pd(2 * i + 1));
          pk1[i] = Elem<T>::pack(pd(64 + 2 * i), pd(64 + 2 * i + 1));
        }
        tmem_st32(tST + 0, pk0);
        tmem_st32(tST + 32, pk1);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(L::kBarP));

      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarDP), t & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      write_ds<T, true, DROP>(tDPT, tDPT, pv, s_d + buf * kT, 0.f, keep, p.drop.inv_keep);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(L::kBarDS));
      if (t + 1 < nt) {
        s_lse[(buf ^ 1) * kT + tid] = nl;
        s_d[(buf ^ 1) * kT + tid] = nd;
        mbar_arrive(bar(L::kBarLse + (buf ^ 1)));
      }
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarDone), 0, abort_flag, p.status));
    if (ACC && ok) {
      // added into the fp32 accumulators, one key row per thread
      tc_fence_after();
      const long rowoff = (((long)b * p.Nk + key) * p.Hkv + hk) * D;
      const bool active = key < p.Nk && FA_IN_BOUNDS(p.status, rowoff + D - 1, (long)p.B * p.Nk * p.Hkv * D);
      acc_row<D>(tbase + lane_off + kColDV, p.acc1 + rowoff, DROP ? p.drop.inv_keep : 1.f, p.acc_init != 0, active);
      acc_row<D>(tbase + lane_off + kColDK, p.acc0 + rowoff, p.scale, p.acc_init != 0, active);
    } else if (ok) {
      // every MMA has run, so the Q and dO buffers are free: dV and dK leave through them by TMA
      // (rows past Nk are clipped by the tensor maps)
      tc_fence_after();
      stage_row<T, D>(tbase + lane_off + kColDV, sb + L::kOffQ, jrow, DROP ? p.drop.inv_keep : 1.f);
      stage_row<T, D>(tbase + lane_off + kColDK, sb + L::kOffDO, jrow, p.scale);
      fence_proxy_async_smem();
      mbar_arrive(bar(L::kBarOut));
      if (tid == 0 && mbar_wait(bar(L::kBarOut), 0, abort_flag, p.status)) {
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn) {
          tma_store_4d(&tmDV, sb + L::kOffQ + pn * kPanel, 64 * pn, hk, k0, b);
          tma_store_4d(&tmDK, sb + L::kOffDO + pn * kPanel, 64 * pn, hk, k0, b);
        }
        bulk_commit();
        bulk_wait_all();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ===========================================================================
// dQ
// ===========================================================================
template <int D, bool DROP>
struct DqSmem {
  static constexpr int kTile = (D / 64) * kPanel;
  static constexpr int kVStages = DROP ? 1 : 2;  // with dropout one V stage makes room for the keep ring
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kTile;
  static constexpr int kOffK = 2 * kTile;  // 3 stages
  static constexpr int kOffV = 5 * kTile;  // kVStages stages
  static constexpr int kOffKeep = kOffV + kVStages * kTile;  // dropout: [2][128 rows] x 128 keep bits
  static constexpr int kOffBar = kOffKeep + (DROP ? 2 * kT * 16 : 0);
  // kBarOut: the elementwise threads have staged dQ (in the free Q buffer);
  // kBarKeepFull / kBarKeepEmpty: a slot of the keep-bit ring written / read
  enum { kBarQ = 0, kBarKFull = 1, kBarKEmpty = 4, kBarVFull = 7, kBarVEmpty = 9, kBarS = 11, kBarDP = 13,
         kBarDS = 14, kBarDone = 15, kBarDrain = 16, kBarOut = 17, kBarKeepFull = 18, kBarKeepEmpty = 20,
         kNumBars = 22 };
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmem + 4;
  static constexpr int kBytes = kOffAbort + 4 + 1024;
};
// TMEM columns: S buffers (scores, later dS), dP, dQ
__host__ __device__ constexpr uint32_t col_s(int buf) { return 128u * buf; }
constexpr uint32_t kColDP = 256, kColDQ = 384;

template <typename T, int D, bool CAUSAL, bool DROP, bool ACC = false>
__global__ void __launch_bounds__(DROP ? kThreadsDrop : kThreads, 1)
    bwd_dq_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                        const __grid_constant__ CUtensorMap tmDQ, Params p) {
  using L = DqSmem<D, DROP>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* gb = smem_raw + (sb - raw);
  auto bar = [&](int i) { return sb + L::kOffBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + L::kOffAbort);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // grid (Hq, row tiles, B), dispatched x-fastest: longest causal rows first across all heads
  const int mblk = CAUSAL ? (int)(gridDim.y - 1 - blockIdx.y) : (int)blockIdx.y;
  const int h = blockIdx.x, b = blockIdx.z;
  const int hk = h / (p.Hq / p.Hkv);
  const int m0 = mblk * kT;
  const int off = p.Nk - p.Nq;
  const int n_end = CAUSAL ? min(p.Nk, m0 + kT + off) : p.Nk;
  const int n = (n_end + kT - 1) / kT;

  if (tid == 0) {
    for (int i = 0; i < L::kNumBars; ++i) mbar_init(bar(i), (i == L::kBarDS || i >= L::kBarOut) ? kT : 1);
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
    prefetch_tmap(&tmDO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(gb + L::kOffTmem);

  if (warp >= 4 && warp < 8) {
   if constexpr (DROP) regs_decrease<kRegsCtrl>();
   if (warp == kWarpLoad) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int last_k[3] = {-1, -1, -1}, last_v[2] = {-1, -1};
      constexpr int VS = L::kVStages;
      mbar_expect_tx(bar(L::kBarQ), 2 * L::kTile);
#pragma unroll
      for (int pn = 0; pn < D / 64; ++pn) {
        tma_load_4d(sb + L::kOffQ + pn * kPanel, &tmQ, bar(L::kBarQ), 64 * pn, h, m0, b);
        tma_load_4d(sb + L::kOffDO + pn * kPanel, &tmDO, bar(L::kBarQ), 64 * pn, h, m0, b);
      }
      for (int j = 0; j < n; ++j) {
        const int ks = j % 3, ku = j / 3, vs = j % VS, vu = j / VS;
        if (ku > 0 && !mbar_wait(bar(L::kBarKEmpty + ks), (ku - 1) & 1, abort_flag, p.status)) break;
        mbar_expect_tx(bar(L::kBarKFull + ks), L::kTile);
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn)
          tma_load_4d(sb + L::kOffK + ks * L::kTile + pn * kPanel, &tmK, bar(L::kBarKFull + ks), 64 * pn, hk, j * kT,
                      b);
        last_k[ks] = ku;
        if (vu > 0 && !mbar_wait(bar(L::kBarVEmpty + vs), (vu - 1) & 1, abort_flag, p.status)) break;
        mbar_expect_tx(bar(L::kBarVFull + vs), L::kTile);
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn)
          tma_load_4d(sb + L::kOffV + vs * L::kTile + pn * kPanel, &tmV, bar(L::kBarVFull + vs), 64 * pn, hk, j * kT,
                      b);
        last_v[vs] = vu;
      }
      if (*abort_flag) {
        wait_drain(bar(L::kBarQ), 0, p.status);
        for (int s3 = 0; s3 < 3; ++s3)
          if (last_k[s3] >= 0) wait_drain(bar(L::kBarKFull + s3), last_k[s3] & 1, p.status);
        for (int s2 = 0; s2 < VS; ++s2)
          if (last_v[s2] >= 0) wait_drain(bar(L::kBarVFull + s2), last_v[s2] & 1, p.status);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr bool kBf16 = Elem<T>::kBf16;
      constexpr uint32_t id_kk = idesc_f16(kBf16, kT, kT, false);  // S, dP
      constexpr uint32_t id_mn = idesc_f16(kBf16, kT, D, true);    // dQ: B = K as [keys][d]
      auto kmajor = [&](uint32_t dst, uint32_t a_base, uint32_t b_base) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * kPanel + (kk & 3) * 32;
          mma_ss(tbase + dst, sdesc_sw128(a_base + ko, 16, 1024), sdesc_sw128(b_base + ko, 16, 1024), id_kk,
                 kk > 0 ? 1u : 0u);
        }
      };
      const uint32_t sQ = sb + L::kOffQ, sDO = sb + L::kOffDO;
      auto sK = [&](int j) { return sb + L::kOffK + (j % 3) * L::kTile; };
      auto sV = [&](int j) { return sb + L::kOffV + (j % L::kVStages) * L::kTile; };
      auto issue_s = [&](int j) -> bool {
        if (!mbar_wait(bar(L::kBarKFull + j % 3), (j / 3) & 1, abort_flag, p.status)) return false;
        tc_fence_after();
        kmajor(col_s(j & 1), sQ, sK(j));
        mma_commit(bar(L::kBarS + (j & 1)));
        return true;
      };
      auto issue_dp = [&](int j) -> bool {
        if (!mbar_wait(bar(L::kBarVFull + j % L::kVStages), (j / L::kVStages) & 1, abort_flag, p.status)) return false;
        tc_fence_after();
        kmajor(kColDP, sDO, sV(j));
        mma_commit(bar(L::kBarDP));  // without dropout this also frees V of tile j (see the elementwise warps)
        if constexpr (DROP) mma_commit(bar(L::kBarVEmpty + j % L::kVStages));  // one V stage: free it at once
        return true;
      };
      bool ok = mbar_wait(bar(L::kBarQ), 0, abort_flag, p.status);
      ok = ok && issue_s(0) && issue_dp(0);
      if (ok && n > 1) ok = issue_s(1);
      if (ok) {
        for (int j = 0; j < n; ++j) {
          ok = mbar_wait(bar(L::kBarDS), j & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kT / 16; ++kk)
            mma_ts(tbase + kColDQ, tbase + col_s(j & 1) + kk * 8, sdesc_sw128(sK(j) + kk * 2048, kPanel, 1024), id_mn,
                   (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(L::kBarKEmpty + j % 3));
          if (j + 1 < n && !(ok = issue_dp(j + 1))) break;  // dP_j was read before dS_j was signalled
          if (j + 2 < n && !(ok = issue_s(j + 2))) break;   // reuses S buffer j after the dQ MMA
        }
        if (ok) mma_commit(bar(L::kBarDone));
      }
      mma_commit(bar(L::kBarDrain));
      wait_drain(bar(L::kBarDrain), 0, p.status);
    }
  }
  } else if (DROP && warp >= 8) {
    if constexpr (DROP) regs_decrease<kRegsRng>();
    // ------------------------------------------------------------------ keep bits (dropout)
    // thread rt draws the keep bits of query row m0 + rt for every key tile into ring slot j & 1.
    // Lanes 2m and 2m + 1 hold one query pair: each makes the calls of every other key quad and
    // hands the other row's bits to lane ^ 1; four independent calls are in flight at a time.
    const int rt = tid - 256;
    const int row = m0 + rt;
    const uint32_t bh = (uint32_t)(b * p.Hq + h), rh = (uint32_t)row >> 1;
    const int e = row & 1;  // == lane & 1
    uint4* ring = reinterpret_cast<uint4*>(gb + L::kOffKeep);
    for (int j = 0; j < n; ++j) {
      const int slot = j & 1;
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(bar(L::kBarKeepEmpty + slot), ((j >> 1) - 1) & 1,
                                                       abort_flag, p.status)))
        break;
      const int kb = j * kT;
      uint32_t own[4] = {0u, 0u, 0u, 0u}, other[4] = {0u, 0u, 0u, 0u};
#pragma unroll 1
      for (int t2 = 0; t2 < 4; ++t2) {
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
          const int cc = 32 * wd + 8 * t2 + 4 * e;  // keys kb + cc .. cc + 3
          const uint4 w = philox4x32_10((uint32_t)(kb + cc) >> 2, rh, bh, p.drop.offset, p.drop.seed_lo,
                                        p.drop.seed_hi);
          const uint32_t even = keep_quad(w.x, w.y, p.drop.thr), odd = keep_quad(w.z, w.w, p.drop.thr);
          own[wd] |= (e ? odd : even) << (cc & 31);
          other[wd] |= (e ? even : odd) << (cc & 31);
        }
      }
      uint32_t keep[4];
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) keep[wd] = own[wd] | __shfl_xor_sync(0xffffffffu, other[wd], 1);
      ring[slot * kT + rt] = make_uint4(keep[0], keep[1], keep[2], keep[3]);
      mbar_arrive(bar(L::kBarKeepFull + slot));
    }
  } else {
    if constexpr (DROP) regs_increase<kRegsElem>();
    // ------------------------------------------------------------------ elementwise: one query row per thread
    const int wq = warp;
    const int row = m0 + wq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const float c = p.scale_log2;
    const long idx = ((long)b * p.Hq + h) * p.Nq + row;
    const bool in = row < p.Nq && FA_IN_BOUNDS(p.status, idx, (long)p.B * p.Hq * p.Nq);
    const float nlse2 = in ? -p.lse[idx] * kLog2e : -INFINITY;  // rows past Nq get P = 0
    const float ndrow = in ? -p.dvec[idx] : 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const uint32_t tS = tbase + lane_off + col_s(j & 1);
      const int kb = j * kT;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarS + (j & 1)), (j >> 1) & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      float pv[kT];
      load_row128(tS, pv);
      const float2 c2 = make_float2(c, c), nl2 = make_float2(nlse2, nlse2);
#pragma unroll
      for (int cc = 0; cc < kT; cc += 2) {
        const float2 x = exp2_pair8<kExp8<DROP>>(__ffma2_rn(make_float2(pv[cc], pv[cc + 1]), c2, nl2), cc >> 1);
        pv[cc] = x.x;
        pv[cc + 1] = x.y;
      }
      if (kb + kT > p.Nk || (CAUSAL && kb + kT - 1 > m0 + off)) {
        int lim = p.Nk - kb;
        if (CAUSAL) lim = min(lim, row + off + 1 - kb);
#pragma unroll
        for (int cc = 0; cc < kT; ++cc)
          if (cc >= lim) pv[cc] = 0.f;
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarDP), j & 1, abort_flag, p.status));
      if (!ok) break;
      if (!DROP && tid == 0) {
        // dP of tile j is complete, so its V stage (read by no other MMA) is free: this arrival
        // stands in for an MMA commit per key tile.  With two V stages the next load into it has
        // a tile of slack; the dropout variant's single V stage is freed by the commit instead.
        mbar_arrive(bar(L::kBarVEmpty + j % L::kVStages));
      }
      tc_fence_after();
      uint32_t keep[4] = {0u, 0u, 0u, 0u};  // dropout: bit cc = (this query, key kb + cc) kept
      if constexpr (DROP) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarKeepFull + (j & 1)), (j >> 1) & 1, abort_flag, p.status));
        if (!ok) break;
        const uint4 kq = reinterpret_cast<const uint4*>(gb + L::kOffKeep)[(j & 1) * kT + wq * 32 + lane];
        keep[0] = kq.x;
        keep[1] = kq.y;
        keep[2] = kq.z;
        keep[3] = kq.w;
        mbar_arrive(bar(L::kBarKeepEmpty + (j & 1)));
      }
      write_ds<T, false, DROP>(tbase + lane_off + kColDP, tS, pv, nullptr, ndrow, keep, p.drop.inv_keep);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(L::kBarDS));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarDone), 0, abort_flag, p.status));
    if (ACC && ok) {
      tc_fence_after();
      const long rowoff = (((long)b * p.Nq + row) * p.Hq + h) * D;
      const bool active = row < p.Nq && FA_IN_BOUNDS(p.status, rowoff + D - 1, (long)p.B * p.Nq * p.Hq * D);
      acc_row<D>(tbase + lane_off + kColDQ, p.acc0 + rowoff, p.scale, p.acc_init != 0, active);
    } else if (ok) {
      // every MMA has run, so the Q buffer is free: dQ leaves through it by TMA (rows past Nq clipped)
      tc_fence_after();
      stage_row<T, D>(tbase + lane_off + kColDQ, sb + L::kOffQ, wq * 32 + lane, p.scale);
      fence_proxy_async_smem();
      mbar_arrive(bar(L::kBarOut));
      if (tid == 0 && mbar_wait(bar(L::kBarOut), 0, abort_flag, p.status)) {
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn) tma_store_4d(&tmDQ, sb + L::kOffQ + pn * kPanel, 64 * pn, h, m0, b);
        bulk_commit();
        bulk_wait_all();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
  // launched as a programmatic dependent of the dK/dV kernel: the grid must not complete before
  // that kernel has (later work on the stream waits only for this grid), so the last CTA waits
  // for it; without that launch attribute the wait returns at once
  if (blockIdx.x == gridDim.x - 1 && blockIdx.y == gridDim.y - 1 && blockIdx.z == gridDim.z - 1)
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct Maps {
  CUtensorMap q, k, v, dO, dq, dk, dv;
};

// Loads of Q, K, V, dO; stores of whichever of dQ, dK, dV the launch writes.
bool make_maps(Maps& m, const BwdArgs& a, bool kv_out, bool q_out) {
  const bool bf16 = a.bf16 != 0;
  bool ok = make_map(&m.q, a.q, bf16, a.d, a.Hq, a.Nq, a.B, kT) && make_map(&m.k, a.k, bf16, a.d, a.Hkv, a.Nk, a.B, kT) &&
            make_map(&m.v, a.v, bf16, a.d, a.Hkv, a.Nk, a.B, kT) &&
            make_map(&m.dO, a.dout, bf16, a.d, a.Hq, a.Nq, a.B, kT);
  if (ok && kv_out)
    ok = make_map(&m.dk, a.dk, bf16, a.d, a.Hkv, a.Nk, a.B, kT) && make_map(&m.dv, a.dv, bf16, a.d, a.Hkv, a.Nk, a.B, kT);
  if (ok && q_out) ok = make_map(&m.dq, a.dq, bf16, a.d, a.Hq, a.Nq, a.B, kT);
  return ok;
}

// The dropout kernels' register split assumes the launch register count it was sized against;
// a kernel compiled with fewer would wait forever in setmaxnreg.inc, so it is not launched.
template <typename K>
bool split_fits(K kern) {
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return false;
  return fa.numRegs * kThreadsDrop >= 128 * (kRegsElem + kRegsCtrl + kRegsRng);
}

Params params(const BwdArgs& a, void* out0, void* out1, float* acc0, float* acc1) {
  return Params{a.lse,  a.dvec,      out0,  out1, a.B, a.Hq, a.Hkv, a.Nq, a.Nk, a.scale, a.scale * kLog2e, a.status,
                Dropout{a.drop_thr, a.drop_inv_keep, a.seed_lo, a.seed_hi, a.drop_offset}, acc0, acc1, a.acc_init};
}

template <typename T, int D, bool CAUSAL>
cudaError_t launch_dkdv(const BwdArgs& a, cudaStream_t s) {
  Maps m;
  const bool acc = a.acc_k != nullptr;
  if (!make_maps(m, a, !acc, false)) return cudaErrorInvalidValue;
  const bool drop = a.drop_p > 0.f;
  if (acc && drop) return cudaErrorInvalidValue;
  auto kern = acc ? bwd_dkdv_sm100_kernel<T, D, CAUSAL, false, true>
                  : drop ? bwd_dkdv_sm100_kernel<T, D, CAUSAL, true> : bwd_dkdv_sm100_kernel<T, D, CAUSAL, false>;
  const int smem = DkdvSmem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if (drop && !split_fits(kern)) return cudaErrorInvalidConfiguration;
  dim3 grid(a.Hkv, (a.Nk + kT - 1) / kT, a.B);
  kern<<<grid, drop ? kThreadsDrop : kThreads, smem, s>>>(m.q, m.k, m.v, m.dO, m.dk, m.dv,
                                                          params(a, a.dk, a.dv, a.acc_k, a.acc_v));
  return cudaGetLastError();
}

template <typename T, int D, bool CAUSAL>
cudaError_t launch_dq(const BwdArgs& a, cudaStream_t s) {
  Maps m;
  const bool acc = a.acc_q != nullptr;
  if (!make_maps(m, a, false, !acc)) return cudaErrorInvalidValue;
  const bool drop = a.drop_p > 0.f;
  if (acc && drop) return cudaErrorInvalidValue;
  auto kern = acc ? bwd_dq_sm100_kernel<T, D, CAUSAL, false, true>
                  : drop ? bwd_dq_sm100_kernel<T, D, CAUSAL, true> : bwd_dq_sm100_kernel<T, D, CAUSAL, false>;
  const int smem = drop ? DqSmem<D, true>::kBytes : DqSmem<D, false>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if (drop && !split_fits(kern)) return cudaErrorInvalidConfiguration;
  dim3 grid(a.Hq, (a.Nq + kT - 1) / kT, a.B);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(drop ? kThreadsDrop : kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr{};
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  if (a.after_dkdv) {  // the previous launch on the stream is this backward's dK/dV kernel
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kern, m.q, m.k, m.v, m.dO, m.dq, params(a, a.dq, nullptr, a.acc_q, nullptr));
}

}  // namespace

#define FA_DISPATCH_SM100(FN, a, s)                                                                        \
  do {                                                                                                     \
    if (a.bf16) {                                                                                          \
      if (a.d == 128) return a.causal ? FN<__nv_bfloat16, 128, true>(a, s) : FN<__nv_bfloat16, 128, false>(a, s); \
      return a.causal ? FN<__nv_bfloat16, 64, true>(a, s) : FN<__nv_bfloat16, 64, false>(a, s);           \
    }                                                                                                      \
    if (a.d == 128) return a.causal ? FN<__half, 128, true>(a, s) : FN<__half, 128, false>(a, s);         \
    return a.causal ? FN<__half, 64, true>(a, s) : FN<__half, 64, false>(a, s);                           \
  } while (0)

cudaError_t launch_bwd_dkdv_sm100(const BwdArgs& a, cudaStream_t s) { FA_DISPATCH_SM100(launch_dkdv, a, s); }
cudaError_t launch_bwd_dq_sm100(const BwdArgs& a, cudaStream_t s) { FA_DISPATCH_SM100(launch_dq, a, s); }

}  // namespace fa
