// decode.cu -- split-KV decode for one-token queries ("FlashAttention 심층
// 분석", Flash-Decoding): the key axis of each sequence is cut into splits
// that are processed in parallel, each producing a normalised partial output
// O_s and its log-sum-exp LSE_s; a second kernel merges the splits by
// log-sum-exp.
//
// Partial pass: one CTA per (split s, KV head h_kv, sequence b).  The
// Hq/Hkv query rows of the GQA group share every K/V byte the CTA reads, so
// the KV cache crosses HBM exactly once.  K/V tiles of 64 keys stream through
// a three-stage cp.async ring (two CTAs per SM); each of the four warps takes 16 keys of every
// tile, keeps its own running (m, l, O) for the group's rows, and the warps
// are merged through shared memory at the end.  The group's rows (padded to
// the 16-row MMA shape) multiply the tiles on the tensor cores; the pass is
// bound by HBM reads of the cache, not by the arithmetic.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace fa {
namespace {

constexpr int kThreads = 128;
constexpr int kTileN = 64;
constexpr int kStages = 3;  // 3 x 32 KB K/V stages: two CTAs fit on an SM
constexpr int kRows = 16;  // MMA rows; the group's query heads, zero-padded

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 2) decode_split_kernel(DecodeArgs p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int kTile = kTileN * D * 2;
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sStage0 = sQ + kRows * D * 2;
  auto sK = [&](int st) { return sStage0 + kTile * (2 * st); };
  auto sV = [&](int st) { return sStage0 + kTile * (2 * st + 1); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int G = p.Hq / p.Hkv;
  const int S = p.num_splits;
  int n = p.seqlens[b];
  n = n < 0 ? 0 : (n > p.Nk_max ? p.Nk_max : n);
  const int lo = s * p.chunk;
  const int hi = min(lo + p.chunk, n);
  const long part0 = ((long)b * p.Hq + (long)hk * G) * S + s;  // (b, h = hk*G + g, s) = part0 + g*S

  const long nparts = (long)p.B * p.Hq * S;
  if (hi <= lo) {
    for (int i = tid; i < G * D; i += kThreads) {
      const long oi = (part0 + (long)(i / D) * S) * D + (i % D);
      if (FA_IN_BOUNDS(p.status, oi, nparts * D)) p.o_part[oi] = 0.f;
    }
    if (tid < G && FA_IN_BOUNDS(p.status, part0 + (long)tid * S, nparts)) p.lse_part[part0 + (long)tid * S] = -INFINITY;
    return;
  }
  const int ntiles = (hi - lo + kTileN - 1) / kTileN;
  const long ldk = (long)p.Hkv * D;
  const uint16_t* gq = static_cast<const uint16_t*>(p.q) + ((long)b * p.Hq + (long)hk * G) * D;
  const uint16_t* gk = static_cast<const uint16_t*>(p.k) + ((long)b * p.Nk_max * p.Hkv + hk) * D;
  const uint16_t* gv = static_cast<const uint16_t*>(p.v) + ((long)b * p.Nk_max * p.Hkv + hk) * D;

  load_tile_async<kRows, D, kThreads>(sQ, gq, 0, G, D, tid);
#pragma unroll
  for (int t = 0; t < kStages - 1; ++t) {
    if (t < ntiles) {
      load_tile_async<kTileN, D, kThreads>(sK(t), gk, lo + t * kTileN, hi, ldk, tid);
      load_tile_async<kTileN, D, kThreads>(sV(t), gv, lo + t * kTileN, hi, ldk, tid);
    }
    cp_async_commit();
  }

  float acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  uint32_t qf[D / 16][4];
  const float c = p.scale * kLog2e;

  for (int t = 0; t < ntiles; ++t) {
    const int st = t % kStages;
    {
      const int tn = t + kStages - 1;
      if (tn < ntiles) {
        load_tile_async<kTileN, D, kThreads>(sK(tn % kStages), gk, lo + tn * kTileN, hi, ldk, tid);
        load_tile_async<kTileN, D, kThreads>(sV(tn % kStages), gv, lo + tn * kTileN, hi, ldk, tid);
      }
      cp_async_commit();
    }
    cp_async_wait<kStages - 1>();
    __syncthreads();
    if (t == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) frag_a<kRows>(qf[kk], sQ, 0, kk * 16, lane);
    }

    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t bb[4];
      frag_b_nk<kTileN>(bb, sK(st), warp * 16, kk * 16, lane);
      mma16816<T>(sc[0], qf[kk], bb[0], bb[1]);
      mma16816<T>(sc[1], qf[kk], bb[2], bb[3]);
    }
    const int key0 = lo + t * kTileN + warp * 16;
    if (key0 + 16 > hi) {
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (key0 + nb * 8 + 2 * (lane & 3) + (e & 1) >= hi) sc[nb][e] = -INFINITY;
    }
    float mu[2], corr[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float rm = fmaxf(fmaxf(sc[0][2 * e], sc[0][2 * e + 1]), fmaxf(sc[1][2 * e], sc[1][2 * e + 1]));
      const float mnew = fmaxf(m_run[e], quad_max(rm) * c);
      mu[e] = (mnew == -INFINITY) ? 0.f : mnew;
      corr[e] = ex2(m_run[e] - mu[e]);
      m_run[e] = mnew;
    }
    uint32_t pa[4];
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
      const float p0 = ex2(fmaf(sc[nb][0], c, -mu[0])), p1 = ex2(fmaf(sc[nb][1], c, -mu[0]));
      const float p2 = ex2(fmaf(sc[nb][2], c, -mu[1])), p3 = ex2(fmaf(sc[nb][3], c, -mu[1]));
      rs[0] += p0 + p1;
      rs[1] += p2 + p3;
      pa[nb * 2 + 0] = Elem<T>::pack(p0, p1);
      pa[nb * 2 + 1] = Elem<T>::pack(p2, p3);
    }
    l_run[0] = l_run[0] * corr[0] + rs[0];
    l_run[1] = l_run[1] * corr[1] + rs[1];
#pragma unroll
    for (int np = 0; np < D / 16; ++np) {
      uint32_t bb[4];
      frag_b_kn<kTileN>(bb, sV(st), warp * 16, np * 16, lane);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * np][e] *= corr[e >> 1];
        acc[2 * np + 1][e] *= corr[e >> 1];
      }
      mma16816<T>(acc[2 * np], pa, bb[0], bb[1]);
      mma16816<T>(acc[2 * np + 1], pa, bb[2], bb[3]);
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  __syncthreads();

  // merge the four warps: per warp m[16], l[16], O[16][D] (fp32) in the stage buffers
  float* red_o = reinterpret_cast<float*>(smem + kRows * D * 2);  // [4][16][D]
  float* red_m = red_o + 4 * kRows * D;                             // [4][16]
  float* red_l = red_m + 4 * kRows;                                 // [4][16]
  const int r0 = lane >> 2;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const float l = quad_sum(l_run[e]);
    if ((lane & 3) == 0) {
      red_m[warp * kRows + r0 + 8 * e] = m_run[e];
      red_l[warp * kRows + r0 + 8 * e] = l;
    }
  }
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const int col = i * 8 + 2 * (lane & 3);
    float* o0 = red_o + (warp * kRows + r0) * D + col;
    float* o1 = red_o + (warp * kRows + r0 + 8) * D + col;
    o0[0] = acc[i][0];
    o0[1] = acc[i][1];
    o1[0] = acc[i][2];
    o1[1] = acc[i][3];
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += kThreads) {
    const int g = idx / D, col = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, red_m[w * kRows + g]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float f = ex2(red_m[w * kRows + g] - M);
      L += red_l[w * kRows + g] * f;
      O += red_o[(w * kRows + g) * D + col] * f;
    }
    const long oi = (part0 + (long)g * S) * D + col;
    if (FA_IN_BOUNDS(p.status, oi, nparts * D)) p.o_part[oi] = O / L;
    if (col == 0 && FA_IN_BOUNDS(p.status, part0 + (long)g * S, nparts)) p.lse_part[part0 + (long)g * S] = (M + lg2(L)) * kLn2;
  }
}

// Combine: one CTA per (h_q, b), one thread per output column.
template <typename T, int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(CombineArgs p) {
  const int h = blockIdx.x, b = blockIdx.y, col = threadIdx.x;
  const int S = p.num_splits;
  const long base = ((long)b * p.Hq + h) * S;
  if (!FA_IN_BOUNDS(p.status, base + S - 1, (long)p.B * p.Hq * S)) return;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, p.lse_part[base + s]);
  float L = 0.f, O = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < S; ++s) {
      const float w = __expf(p.lse_part[base + s] - M);
      L += w;
      O += w * p.o_part[(base + s) * D + col];
    }
  }
  const float out = L > 0.f ? O / L : 0.f;
  uint16_t* go = static_cast<uint16_t*>(p.o) + ((long)b * p.Hq + h) * D;
  T v;
  if constexpr (Elem<T>::kBf16) v = __float2bfloat16_rn(out); else v = __float2half_rn(out);
  if (FA_IN_BOUNDS(p.status, ((long)b * p.Hq + h) * D + col, (long)p.B * p.Hq * D)) go[col] = *reinterpret_cast<uint16_t*>(&v);
  if (col == 0 && FA_IN_BOUNDS(p.status, (long)b * p.Hq + h, (long)p.B * p.Hq))
    p.lse[(long)b * p.Hq + h] = L > 0.f ? M + logf(L) : -INFINITY;
}

template <typename T, int D>
cudaError_t launch_split(const DecodeArgs& a, cudaStream_t s) {
  const int smem_pipe = kRows * D * 2 + kStages * 2 * kTileN * D * 2;
  const int smem_red = kRows * D * 2 + (4 * kRows * D + 8 * kRows) * 4;
  const int smem = smem_pipe > smem_red ? smem_pipe : smem_red;
  auto kern = decode_split_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.num_splits, a.Hkv, a.B);
  kern<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
  dim3 grid(a.Hq, a.B);
  decode_combine_kernel<T, D><<<grid, D, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_split(const DecodeArgs& a, cudaStream_t s) {
  if (a.bf16) return a.d == 128 ? launch_split<__nv_bfloat16, 128>(a, s) : launch_split<__nv_bfloat16, 64>(a, s);
  return a.d == 128 ? launch_split<__half, 128>(a, s) : launch_split<__half, 64>(a, s);
}

cudaError_t launch_decode_combine(const CombineArgs& a, cudaStream_t s) {
  if (a.bf16) return a.d == 128 ? launch_combine<__nv_bfloat16, 128>(a, s) : launch_combine<__nv_bfloat16, 64>(a, s);
  return a.d == 128 ? launch_combine<__half, 128>(a, s) : launch_combine<__half, 64>(a, s);
}

}  // namespace fa
