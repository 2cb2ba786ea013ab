// fwd_sm100.cu -- attention forward on the sm_100a tensor-core path:
// TMA tile loads, tcgen05 MMAs with accumulators in tensor memory (TMEM),
// and warp-specialised roles.
//
// What it computes is the tiled online softmax of "FlashAttention 심층 분석"
// (section 3): for each query row, walk the key tiles, keep a running max m
// and running sum l, rescale the output accumulator when m grows, and divide
// by l at the end; the N x N score matrix never reaches HBM.
//
// How it maps onto one B200 SM (one CTA per SM, 320 threads):
//   * two 128-row query tiles Q0, Q1 share every K/V tile the CTA loads;
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
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

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
constexpr int kWarpMma = 9;
constexpr int kThreads = 320;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when m grows by more than 2^8
__host__ __device__ constexpr uint32_t col_s(int t) { return 128u * t; }        // S_t / P_t
__host__ __device__ constexpr uint32_t col_o(int t) { return 256u + 128u * t; }  // O_t

template <int D>
struct Smem {
  static constexpr int kPanel = 128 * 128;  // one [128 rows][64 cols] 16-bit panel, bytes
  static constexpr int kTile = (D / 64) * kPanel;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTiles * kTile;
  static constexpr int kOffV = kOffK + kStages * kTile;
  static constexpr int kOffBar = kOffV + kStages * kTile;
  enum { kBarQ = 0, kBarKFull = 1, kBarKEmpty = 3, kBarVFull = 5, kBarVEmpty = 7, kBarS = 9, kBarP = 11, kBarO = 13,
         kBarDrain = 14, kNumBars = 15 };
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmem + 4;
  static constexpr int kBytes = kOffAbort + 4 + 1024;  // + slack to align the base to 1024 B
};

struct Params {
  void* o;
  float* lse;
  int B, Hq, Hkv, Nq, Nk;
  float scale_log2;
  int* status;
};

template <typename T, int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, Params p) {
  using L = Smem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* gb = smem_raw + (sb - raw);
  auto bar = [&](int i) { return sb + L::kOffBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + L::kOffAbort);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // grid (Hq, row blocks, B): blocks are dispatched x-fastest, so every head's
  // longest causal row block starts before any shorter one
  const int mblk = CAUSAL ? (int)(gridDim.y - 1 - blockIdx.y) : (int)blockIdx.y;
  const int h = blockIdx.x, b = blockIdx.z;
  const int hk = h / (p.Hq / p.Hkv);
  const int m0 = mblk * (kTiles * kBM);
  const int off = p.Nk - p.Nq;
  const int n_end = CAUSAL ? min(p.Nk, m0 + kTiles * kBM + off) : p.Nk;
  const int nblk = (n_end + kBN - 1) / kBN;

  if (tid == 0) {
    for (int i = 0; i < L::kNumBars; ++i) mbar_init(bar(i), (i == L::kBarP || i == L::kBarP + 1) ? kBM : 1);
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
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(gb + L::kOffTmem);

  if (warp == kWarpLoad) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int last_u[kStages] = {-1, -1};
      mbar_expect_tx(bar(L::kBarQ), kTiles * L::kTile);
#pragma unroll
      for (int t = 0; t < kTiles; ++t)
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn)
          tma_load_4d(sb + L::kOffQ + t * L::kTile + pn * L::kPanel, &tmQ, bar(L::kBarQ), 64 * pn, h, m0 + t * kBM, b);
      for (int j = 0; j < nblk; ++j) {
        const int st = j & 1, u = j >> 1;
        if (u > 0 && !mbar_wait(bar(L::kBarKEmpty + st), (u - 1) & 1, abort_flag, p.status)) break;
        mbar_expect_tx(bar(L::kBarKFull + st), L::kTile);
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn)
          tma_load_4d(sb + L::kOffK + st * L::kTile + pn * L::kPanel, &tmK, bar(L::kBarKFull + st), 64 * pn, hk,
                      j * kBN, b);
        if (u > 0 && !mbar_wait(bar(L::kBarVEmpty + st), (u - 1) & 1, abort_flag, p.status)) {
          last_u[st] = u;  // K of this use is in flight
          break;
        }
        mbar_expect_tx(bar(L::kBarVFull + st), L::kTile);
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn)
          tma_load_4d(sb + L::kOffV + st * L::kTile + pn * L::kPanel, &tmV, bar(L::kBarVFull + st), 64 * pn, hk,
                      j * kBN, b);
        last_u[st] = u;
      }
      if (*abort_flag) {
        // let every copy this thread issued land before the CTA releases its shared memory
        wait_drain(bar(L::kBarQ), 0, p.status);
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
      constexpr uint32_t idq = idesc_f16(kBf16, kBM, kBN, false);
      constexpr uint32_t idv = idesc_f16(kBf16, kBM, D, true);
      auto qk = [&](int t, int st) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * L::kPanel + (kk & 3) * 32;
          const uint64_t a = sdesc_sw128(sb + L::kOffQ + t * L::kTile + ko, 16, 1024);
          const uint64_t bd = sdesc_sw128(sb + L::kOffK + st * L::kTile + ko, 16, 1024);
          mma_ss(tbase + col_s(t), a, bd, idq, kk > 0 ? 1u : 0u);
        }
      };
      auto pv = [&](int t, int st, bool first) {
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // V stored [keys][d]: B is N(=d)-major; 16 keys = two 8-row groups of 128 B
          const uint64_t bd = sdesc_sw128(sb + L::kOffV + st * L::kTile + kk * 2048, L::kPanel, 1024);
          mma_ts(tbase + col_o(t), tbase + col_s(t) + kk * 8, bd, idv, (!first || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(bar(L::kBarQ), 0, abort_flag, p.status) &&
                mbar_wait(bar(L::kBarKFull), 0, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        qk(0, 0);
        mma_commit(bar(L::kBarS + 0));
        qk(1, 0);
        mma_commit(bar(L::kBarS + 1));
        mma_commit(bar(L::kBarKEmpty + 0));
        for (int j = 0; j < nblk; ++j) {
          const int st = j & 1, u = j >> 1;
          const bool more = j + 1 < nblk;
          const int st1 = (j + 1) & 1, u1 = (j + 1) >> 1;
          ok = mbar_wait(bar(L::kBarVFull + st), u & 1, abort_flag, p.status) &&
               mbar_wait(bar(L::kBarP + 0), j & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
          pv(0, st, j == 0);
          if (more) {
            ok = mbar_wait(bar(L::kBarKFull + st1), u1 & 1, abort_flag, p.status);
            if (!ok) break;
            tc_fence_after();
            qk(0, st1);  // overwrites S0/P0 after PV0 in issue order
            mma_commit(bar(L::kBarS + 0));
          }
          ok = mbar_wait(bar(L::kBarP + 1), j & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
          pv(1, st, j == 0);
          mma_commit(bar(L::kBarVEmpty + st));
          if (more) {
            qk(1, st1);
            mma_commit(bar(L::kBarS + 1));
            mma_commit(bar(L::kBarKEmpty + st1));
          }
        }
        if (ok) mma_commit(bar(L::kBarO));
      }
      // no MMA may still run when TMEM is released
      mma_commit(bar(L::kBarDrain));
      wait_drain(bar(L::kBarDrain), 0, p.status);
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int t = warp >> 2;
    const int wq = warp & 3;
    const int row_first = m0 + t * kBM;
    const int row = row_first + wq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tbase + lane_off + col_s(t);
    const uint32_t tO = tbase + lane_off + col_o(t);
    const float c = p.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarS + t), j & 1, abort_flag, p.status));
      if (!ok) break;
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
      if (kbase + kBN > p.Nk || (CAUSAL && kbase + kBN - 1 > row_first + off)) {
        int lim = p.Nk - kbase;
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
      const float mxs = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c;
      const bool resc = mxs > m_ref + kRescaleThreshold;
      const float corr = resc ? ex2(m_ref - mxs) : 1.f;
      if (resc) m_ref = mxs;
      l *= corr;
      const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
      uint32_t pk0[32], pk1[32];
      const float2 c2 = make_float2(c, c), nm2 = make_float2(-mu, -mu);
      float2 rs0 = make_float2(0.f, 0.f), rs1 = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float2 x0 = __ffma2_rn(make_float2(s[2 * i], s[2 * i + 1]), c2, nm2);
        const float2 x1 = __ffma2_rn(make_float2(s[64 + 2 * i], s[64 + 2 * i + 1]), c2, nm2);
        const float2 a = make_float2(ex2(x0.x), ex2(x0.y)), bb = make_float2(ex2(x1.x), ex2(x1.y));
        rs0 = __fadd2_rn(rs0, a);
        rs1 = __fadd2_rn(rs1, bb);
        pk0[i] = Elem<T>::pack(a.x, a.y);
        pk1[i] = Elem<T>::pack(bb.x, bb.y);
      }
      l += (rs0.x + rs0.y) + (rs1.x + rs1.y);
      tmem_st32(tS + 0, pk0);
      tmem_st32(tS + 32, pk1);
      if (__any_sync(0xffffffffu, resc && j > 0)) {
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
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarO), 0, abort_flag, p.status));
    if (ok) {
      tc_fence_after();
      const bool valid = row < p.Nq;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint16_t* orow = static_cast<uint16_t*>(p.o) + (((long)b * p.Nq + row) * p.Hq + h) * D;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        uint32_t r[32];
        tmem_ld32(tO + q * 32, r);
        tmem_wait_ld();
        reg_fence(r);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = Elem<T>::pack(__uint_as_float(r[8 * v + 0]) * inv, __uint_as_float(r[8 * v + 1]) * inv);
            w.y = Elem<T>::pack(__uint_as_float(r[8 * v + 2]) * inv, __uint_as_float(r[8 * v + 3]) * inv);
            w.z = Elem<T>::pack(__uint_as_float(r[8 * v + 4]) * inv, __uint_as_float(r[8 * v + 5]) * inv);
            w.w = Elem<T>::pack(__uint_as_float(r[8 * v + 6]) * inv, __uint_as_float(r[8 * v + 7]) * inv);
            dst[v] = w;
          }
        }
      }
      if (valid) p.lse[((long)b * p.Hq + h) * p.Nq + row] = l > 0.f ? (m_ref + lg2(l)) * kLn2 : -INFINITY;
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

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <typename T, int D, bool CAUSAL>
cudaError_t launch(const AttnArgs& a, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  const bool bf16 = Elem<T>::kBf16;
  if (!make_map(&mq, a.q, bf16, D, a.Hq, a.Nq, a.B, kBM) || !make_map(&mk, a.k, bf16, D, a.Hkv, a.Nk, a.B, kBN) ||
      !make_map(&mv, a.v, bf16, D, a.Hkv, a.Nk, a.B, kBN))
    return cudaErrorInvalidValue;
  Params p{a.o, a.lse, a.B, a.Hq, a.Hkv, a.Nq, a.Nk, a.scale * kLog2e, a.status};
  auto kern = fwd_sm100_kernel<T, D, CAUSAL>;
  const int smem = Smem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.Hq, (a.Nq + kTiles * kBM - 1) / (kTiles * kBM), a.B);
  kern<<<grid, kThreads, smem, s>>>(mq, mk, mv, p);
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

}  // namespace fa
