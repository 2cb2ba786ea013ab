// fwd_mma.cu -- attention forward on warp-level MMA (mma.sync m16n8k16).
//
// One CTA = 4 warps = one 64-row query tile of one (b, h_q); each warp owns 16
// query rows.  K/V tiles of 64 keys stream through a two-stage cp.async ring
// in shared memory, S = Q K^T stays in registers, and the online softmax of
// "FlashAttention 심층 분석" section 3 runs per row in the log2 domain:
//   t = s * scale * log2(e),  m' = max(m, rowmax t),  p = 2^(t - m'),
//   l = 2^(m - m') l + rowsum p,  O = 2^(m - m') O + P V,
// and at the end O /= l, LSE = ln2 * (m + log2 l).  P is rounded to the input
// dtype for the PV product; l is summed from the unrounded fp32 values, so
// the LSE carries only fp32 rounding (the 16-bit rounding of P would move it
// by up to 2^-9 relative).
//
// This is the compact, portable forward (any Nq, Nk, d in {64, 128}); the
// tcgen05 kernel in fwd_sm100.cu is the fast path for sm_100a.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace fa {
namespace {

constexpr int kBM = 64;
constexpr int kBN = 64;
constexpr int kThreads = 128;

template <typename T, int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 2) fwd_mma_kernel(AttnArgs p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int kTile = kBM * D * 2;
  const uint32_t sQ = smem_u32(smem);
  auto sK = [&](int st) { return sQ + kTile * (1 + 2 * st); };
  auto sV = [&](int st) { return sQ + kTile * (2 + 2 * st); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mb = CAUSAL ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x;  // longest tiles first
  const int h = blockIdx.y, b = blockIdx.z;
  const int G = p.Hq / p.Hkv, hk = h / G;
  const int Nq = p.Nq, Nk = p.Nk, off = Nk - Nq;
  const int m0 = mb * kBM;
  const long ldq = (long)p.Hq * D, ldk = (long)p.Hkv * D;
  const uint16_t* gq = static_cast<const uint16_t*>(p.q) + ((long)b * Nq * p.Hq + h) * D;
  const uint16_t* gk = static_cast<const uint16_t*>(p.k) + ((long)b * Nk * p.Hkv + hk) * D;
  const uint16_t* gv = static_cast<const uint16_t*>(p.v) + ((long)b * Nk * p.Hkv + hk) * D;

  const int n_end = CAUSAL ? min(Nk, m0 + kBM + off) : Nk;
  const int nblocks = (n_end + kBN - 1) / kBN;

  load_tile_async<kBM, D, kThreads>(sQ, gq, m0, Nq, ldq, tid);
  load_tile_async<kBN, D, kThreads>(sK(0), gk, 0, Nk, ldk, tid);
  load_tile_async<kBN, D, kThreads>(sV(0), gv, 0, Nk, ldk, tid);
  cp_async_commit();

  float acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  uint32_t qf[D / 16][4];
  const float c = p.scale * kLog2e;
  const int row_w = warp * 16;
  const int r_lo = m0 + row_w + (lane >> 2);
  const int r_hi = r_lo + 8;

  for (int j = 0; j < nblocks; ++j) {
    const int st = j & 1;
    if (j + 1 < nblocks) {
      load_tile_async<kBN, D, kThreads>(sK(st ^ 1), gk, (j + 1) * kBN, Nk, ldk, tid);
      load_tile_async<kBN, D, kThreads>(sV(st ^ 1), gv, (j + 1) * kBN, Nk, ldk, tid);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (j == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) frag_a<kBM>(qf[kk], sQ, row_w, kk * 16, lane);
    }

    // S = Q K_j^T
    float s[kBN / 8][4];
#pragma unroll
    for (int i = 0; i < kBN / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < kBN / 16; ++np) {
        uint32_t bb[4];
        frag_b_nk<kBN>(bb, sK(st), np * 16, kk * 16, lane);
        mma16816<T>(s[2 * np], qf[kk], bb[0], bb[1]);
        mma16816<T>(s[2 * np + 1], qf[kk], bb[2], bb[3]);
      }
    }

    // ragged tail and causal diagonal
    const int n0 = j * kBN;
    if (n0 + kBN > Nk || (CAUSAL && n0 + kBN - 1 > m0 + off)) {
#pragma unroll
      for (int nb = 0; nb < kBN / 8; ++nb) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = n0 + nb * 8 + 2 * (lane & 3) + (e & 1);
          const int row = (e < 2) ? r_lo : r_hi;
          if (key >= Nk || (CAUSAL && key > row + off)) s[nb][e] = -INFINITY;
        }
      }
    }

    // online softmax (log2 domain)
    float rmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nb = 0; nb < kBN / 8; ++nb) {
      rmax[0] = fmaxf(rmax[0], fmaxf(s[nb][0], s[nb][1]));
      rmax[1] = fmaxf(rmax[1], fmaxf(s[nb][2], s[nb][3]));
    }
    float mu[2], corr[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float mnew = fmaxf(m_run[e], quad_max(rmax[e]) * c);
      mu[e] = (mnew == -INFINITY) ? 0.f : mnew;
      corr[e] = ex2(m_run[e] - mu[e]);
      m_run[e] = mnew;
    }
    uint32_t pa[kBN / 16][4];
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int nb = 0; nb < kBN / 8; ++nb) {
      const float p0 = ex2(fmaf(s[nb][0], c, -mu[0])), p1 = ex2(fmaf(s[nb][1], c, -mu[0]));
      const float p2 = ex2(fmaf(s[nb][2], c, -mu[1])), p3 = ex2(fmaf(s[nb][3], c, -mu[1]));
      rs[0] += p0 + p1;
      rs[1] += p2 + p3;
      pa[nb >> 1][(nb & 1) * 2 + 0] = Elem<T>::pack(p0, p1);
      pa[nb >> 1][(nb & 1) * 2 + 1] = Elem<T>::pack(p2, p3);
    }
    l_run[0] = l_run[0] * corr[0] + rs[0];
    l_run[1] = l_run[1] * corr[1] + rs[1];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      acc[i][0] *= corr[0];
      acc[i][1] *= corr[0];
      acc[i][2] *= corr[1];
      acc[i][3] *= corr[1];
    }

    // O += P V_j
#pragma unroll
    for (int kk = 0; kk < kBN / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {
        uint32_t bb[4];
        frag_b_kn<kBN>(bb, sV(st), kk * 16, np * 16, lane);
        mma16816<T>(acc[2 * np], pa[kk], bb[0], bb[1]);
        mma16816<T>(acc[2 * np + 1], pa[kk], bb[2], bb[3]);
      }
    }
    __syncthreads();
  }

  // epilogue: O / l, LSE
  uint16_t* go = static_cast<uint16_t*>(p.o) + ((long)b * Nq * p.Hq + h) * D;
  float inv[2], lse[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const float l = quad_sum(l_run[e]);
    inv[e] = l > 0.f ? 1.f / l : 0.f;
    lse[e] = l > 0.f ? (m_run[e] + lg2(l)) * kLn2 : -INFINITY;
  }
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const int col = i * 8 + 2 * (lane & 3);
    if (r_lo < Nq)
      *reinterpret_cast<uint32_t*>(go + r_lo * ldq + col) = Elem<T>::pack(acc[i][0] * inv[0], acc[i][1] * inv[0]);
    if (r_hi < Nq)
      *reinterpret_cast<uint32_t*>(go + r_hi * ldq + col) = Elem<T>::pack(acc[i][2] * inv[1], acc[i][3] * inv[1]);
  }
  if ((lane & 3) == 0) {
    float* gl = p.lse + ((long)b * p.Hq + h) * Nq;
    if (r_lo < Nq) gl[r_lo] = lse[0];
    if (r_hi < Nq) gl[r_hi] = lse[1];
  }
}

template <typename T, int D, bool CAUSAL>
cudaError_t launch(const AttnArgs& a, cudaStream_t s) {
  const int smem = 5 * kBM * D * 2;
  auto kern = fwd_mma_kernel<T, D, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.Nq + kBM - 1) / kBM, a.Hq, a.B);
  kern<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const AttnArgs& a, cudaStream_t s) {
  if (a.d == 128) return a.causal ? launch<T, 128, true>(a, s) : launch<T, 128, false>(a, s);
  return a.causal ? launch<T, 64, true>(a, s) : launch<T, 64, false>(a, s);
}

}  // namespace

cudaError_t launch_fwd_mma(const AttnArgs& a, cudaStream_t s) {
  return a.bf16 ? launch_t<__nv_bfloat16>(a, s) : launch_t<__half>(a, s);
}

}  // namespace fa
