// bwd.cu -- attention backward with P recomputed from the stored LSE
// ("FlashAttention 심층 분석", section 4: keep only the softmax statistics and
// rebuild S and P on chip).  The gradient equations are the chain rule of
// the definition (the pages give none):
//   D_i  = sum_c dO_ic O_ic                       (preprocess kernel)
//   P_ij = exp(scale q_i.k_j - LSE_i)             (masked entries 0)
//   dP   = dO V^T,   dS = P * (dP - D)
//   dV   = P^T dO,   dK = scale dS^T Q,   dQ = scale dS K
// dK and dV of a KV head are summed over the Hq/Hkv query heads of its GQA
// group inside one CTA, and dQ is produced by a separate kernel, so no
// atomics are used and the result is bitwise reproducible.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace fa {
namespace {

constexpr int kThreads = 128;
constexpr int kB = 64;  // rows of every tile (keys or queries)

// ---------------------------------------------------------------------------
// D = rowsum(dO * O)
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(BwdArgs p) {
  constexpr int TPR = D / 8;  // threads per row, 16 bytes each
  const long R = (long)p.B * p.Nq * p.Hq;
  const long gt = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const long r = gt / TPR;
  const int part = (int)(gt % TPR);
  float acc = 0.f;
  if (r < R) {
    const uint4 o = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.o) + r * D) + part);
    const uint4 g = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.dout) + r * D) + part);
    const uint32_t ov[4] = {o.x, o.y, o.z, o.w};
    const uint32_t gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 a = Elem<T>::unpack(ov[i]), c = Elem<T>::unpack(gv[i]);
      acc = fmaf(a.x, c.x, acc);
      acc = fmaf(a.y, c.y, acc);
    }
  }
#pragma unroll
  for (int w = 1; w < TPR; w <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
  if (part == 0 && r < R) {
    const long bb = r / ((long)p.Nq * p.Hq);
    const int i = (int)((r / p.Hq) % p.Nq);
    const int h = (int)(r % p.Hq);
    p.dvec[(bb * p.Hq + h) * p.Nq + i] = acc;
  }
}

// ---------------------------------------------------------------------------
// dK, dV: one CTA per (64-key tile, h_kv, b); loops over the group's query
// heads and the query tiles that can see the key tile.
// ---------------------------------------------------------------------------
template <typename T, int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 2) bwd_dkdv_kernel(BwdArgs p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int kTile = kB * D * 2;
  const uint32_t sK = smem_u32(smem);
  const uint32_t sV = sK + kTile;
  auto sQ = [&](int st) { return sK + kTile * (2 + 2 * st); };
  auto sdO = [&](int st) { return sK + kTile * (3 + 2 * st); };
  float* s_lse = reinterpret_cast<float*>(smem + 6 * kTile);  // [2][64], log2 domain
  float* s_dv = s_lse + 2 * kB;                                // [2][64]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * kB, hk = blockIdx.y, b = blockIdx.z;
  const int G = p.Hq / p.Hkv;
  const int Nq = p.Nq, Nk = p.Nk, off = Nk - Nq;
  const long ldq = (long)p.Hq * D, ldk = (long)p.Hkv * D;
  const int mstart = CAUSAL ? max(0, n0 - off) / kB : 0;
  const int nmb = (Nq + kB - 1) / kB;
  const int per_head = nmb - mstart;
  const int total = G * per_head;
  const float c = p.scale * kLog2e;

  const uint16_t* gk = static_cast<const uint16_t*>(p.k) + ((long)b * Nk * p.Hkv + hk) * D;
  const uint16_t* gv = static_cast<const uint16_t*>(p.v) + ((long)b * Nk * p.Hkv + hk) * D;
  auto q_base = [&](int h) { return static_cast<const uint16_t*>(p.q) + ((long)b * Nq * p.Hq + h) * D; };
  auto do_base = [&](int h) { return static_cast<const uint16_t*>(p.dout) + ((long)b * Nq * p.Hq + h) * D; };

  load_tile_async<kB, D, kThreads>(sK, gk, n0, Nk, ldk, tid);
  load_tile_async<kB, D, kThreads>(sV, gv, n0, Nk, ldk, tid);
  // tile 0
  {
    const int h = hk * G, m0 = mstart * kB;
    load_tile_async<kB, D, kThreads>(sQ(0), q_base(h), m0, Nq, ldq, tid);
    load_tile_async<kB, D, kThreads>(sdO(0), do_base(h), m0, Nq, ldq, tid);
    if (tid < kB) {
      const int i = m0 + tid;
      const long idx = ((long)b * p.Hq + h) * Nq + i;
      s_lse[tid] = i < Nq ? p.lse[idx] * kLog2e : INFINITY;
      s_dv[tid] = i < Nq ? p.dvec[idx] : 0.f;
    }
  }
  cp_async_commit();

  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.f;
  const int key_lo = n0 + warp * 16 + (lane >> 2);

  for (int t = 0; t < total; ++t) {
    const int st = t & 1;
    const int m0 = (mstart + t % per_head) * kB;
    float nx_lse = 0.f, nx_dv = 0.f;
    if (t + 1 < total) {
      const int h1 = hk * G + (t + 1) / per_head;
      const int m1 = (mstart + (t + 1) % per_head) * kB;
      load_tile_async<kB, D, kThreads>(sQ(st ^ 1), q_base(h1), m1, Nq, ldq, tid);
      load_tile_async<kB, D, kThreads>(sdO(st ^ 1), do_base(h1), m1, Nq, ldq, tid);
      if (tid < kB) {
        const int i = m1 + tid;
        const long idx = ((long)b * p.Hq + h1) * Nq + i;
        nx_lse = i < Nq ? p.lse[idx] * kLog2e : INFINITY;
        nx_dv = i < Nq ? p.dvec[idx] : 0.f;
      }
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    // S^T = K Q^T  (rows: this warp's 16 keys; cols: 64 queries)
    float sp[kB / 8][4];
#pragma unroll
    for (int i = 0; i < kB / 8; ++i) sp[i][0] = sp[i][1] = sp[i][2] = sp[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t ka[4];
      frag_a<kB>(ka, sK, warp * 16, kk * 16, lane);
#pragma unroll
      for (int np = 0; np < kB / 16; ++np) {
        uint32_t bb[4];
        frag_b_nk<kB>(bb, sQ(st), np * 16, kk * 16, lane);
        mma16816<T>(sp[2 * np], ka, bb[0], bb[1]);
        mma16816<T>(sp[2 * np + 1], ka, bb[2], bb[3]);
      }
    }
    // P^T = exp2(S^T c - LSE_q log2e), masked
    const bool need_mask = (n0 + kB > Nk) || (CAUSAL && n0 + kB - 1 > m0 + off);
#pragma unroll
    for (int nb = 0; nb < kB / 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qc = nb * 8 + 2 * (lane & 3) + (e & 1);
        float pv = ex2(fmaf(sp[nb][e], c, -s_lse[st * kB + qc]));
        if (need_mask) {
          const int key = key_lo + ((e >> 1) << 3);
          if (key >= Nk || (CAUSAL && key > m0 + qc + off)) pv = 0.f;
        }
        sp[nb][e] = pv;
      }
    }
    // dP^T = V dO^T
    float dp[kB / 8][4];
#pragma unroll
    for (int i = 0; i < kB / 8; ++i) dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t va[4];
      frag_a<kB>(va, sV, warp * 16, kk * 16, lane);
#pragma unroll
      for (int np = 0; np < kB / 16; ++np) {
        uint32_t bb[4];
        frag_b_nk<kB>(bb, sdO(st), np * 16, kk * 16, lane);
        mma16816<T>(dp[2 * np], va, bb[0], bb[1]);
        mma16816<T>(dp[2 * np + 1], va, bb[2], bb[3]);
      }
    }
    // dV += P^T dO
#pragma unroll
    for (int kk = 0; kk < kB / 16; ++kk) {
      uint32_t pa[4];
      pa[0] = Elem<T>::pack(sp[2 * kk][0], sp[2 * kk][1]);
      pa[1] = Elem<T>::pack(sp[2 * kk][2], sp[2 * kk][3]);
      pa[2] = Elem<T>::pack(sp[2 * kk + 1][0], sp[2 * kk + 1][1]);
      pa[3] = Elem<T>::pack(sp[2 * kk + 1][2], sp[2 * kk + 1][3]);
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {
        uint32_t bb[4];
        frag_b_kn<kB>(bb, sdO(st), kk * 16, np * 16, lane);
        mma16816<T>(dv[2 * np], pa, bb[0], bb[1]);
        mma16816<T>(dv[2 * np + 1], pa, bb[2], bb[3]);
      }
    }
    // dS^T = P^T (dP^T - D_q);  dK += dS^T Q
#pragma unroll
    for (int kk = 0; kk < kB / 16; ++kk) {
      float ds[2][4];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int nb = 2 * kk + u;
          const int qc = nb * 8 + 2 * (lane & 3) + (e & 1);
          ds[u][e] = sp[nb][e] * (dp[nb][e] - s_dv[st * kB + qc]);
        }
      uint32_t da[4];
      da[0] = Elem<T>::pack(ds[0][0], ds[0][1]);
      da[1] = Elem<T>::pack(ds[0][2], ds[0][3]);
      da[2] = Elem<T>::pack(ds[1][0], ds[1][1]);
      da[3] = Elem<T>::pack(ds[1][2], ds[1][3]);
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {
        uint32_t bb[4];
        frag_b_kn<kB>(bb, sQ(st), kk * 16, np * 16, lane);
        mma16816<T>(dk[2 * np], da, bb[0], bb[1]);
        mma16816<T>(dk[2 * np + 1], da, bb[2], bb[3]);
      }
    }
    if (t + 1 < total && tid < kB) {
      s_lse[(st ^ 1) * kB + tid] = nx_lse;
      s_dv[(st ^ 1) * kB + tid] = nx_dv;
    }
    __syncthreads();
  }

  uint16_t* gdk = static_cast<uint16_t*>(p.dk) + ((long)b * Nk * p.Hkv + hk) * D;
  uint16_t* gdv = static_cast<uint16_t*>(p.dv) + ((long)b * Nk * p.Hkv + hk) * D;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const int col = i * 8 + 2 * (lane & 3);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int key = key_lo + 8 * u;
      if (key < Nk) {
        *reinterpret_cast<uint32_t*>(gdk + key * ldk + col) =
            Elem<T>::pack(dk[i][2 * u] * p.scale, dk[i][2 * u + 1] * p.scale);
        *reinterpret_cast<uint32_t*>(gdv + key * ldk + col) = Elem<T>::pack(dv[i][2 * u], dv[i][2 * u + 1]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// dQ: one CTA per (64-query tile, h_q, b); loops over the visible key tiles.
// ---------------------------------------------------------------------------
template <typename T, int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 2) bwd_dq_kernel(BwdArgs p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int kTile = kB * D * 2;
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sdO = sQ + kTile;
  auto sK = [&](int st) { return sQ + kTile * (2 + 2 * st); };
  auto sV = [&](int st) { return sQ + kTile * (3 + 2 * st); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mb = CAUSAL ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int G = p.Hq / p.Hkv, hk = h / G;
  const int Nq = p.Nq, Nk = p.Nk, off = Nk - Nq;
  const int m0 = mb * kB;
  const long ldq = (long)p.Hq * D, ldk = (long)p.Hkv * D;
  const uint16_t* gq = static_cast<const uint16_t*>(p.q) + ((long)b * Nq * p.Hq + h) * D;
  const uint16_t* gdo = static_cast<const uint16_t*>(p.dout) + ((long)b * Nq * p.Hq + h) * D;
  const uint16_t* gk = static_cast<const uint16_t*>(p.k) + ((long)b * Nk * p.Hkv + hk) * D;
  const uint16_t* gv = static_cast<const uint16_t*>(p.v) + ((long)b * Nk * p.Hkv + hk) * D;
  const int n_end = CAUSAL ? min(Nk, m0 + kB + off) : Nk;
  const int nblocks = (n_end + kB - 1) / kB;
  const float c = p.scale * kLog2e;

  load_tile_async<kB, D, kThreads>(sQ, gq, m0, Nq, ldq, tid);
  load_tile_async<kB, D, kThreads>(sdO, gdo, m0, Nq, ldq, tid);
  load_tile_async<kB, D, kThreads>(sK(0), gk, 0, Nk, ldk, tid);
  load_tile_async<kB, D, kThreads>(sV(0), gv, 0, Nk, ldk, tid);
  cp_async_commit();

  const int r_lo = m0 + warp * 16 + (lane >> 2);
  float lse2[2], dvr[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int i = r_lo + 8 * u;
    const long idx = ((long)b * p.Hq + h) * Nq + i;
    lse2[u] = i < Nq ? p.lse[idx] * kLog2e : INFINITY;
    dvr[u] = i < Nq ? p.dvec[idx] : 0.f;
  }
  float dq[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;

  for (int j = 0; j < nblocks; ++j) {
    const int st = j & 1;
    if (j + 1 < nblocks) {
      load_tile_async<kB, D, kThreads>(sK(st ^ 1), gk, (j + 1) * kB, Nk, ldk, tid);
      load_tile_async<kB, D, kThreads>(sV(st ^ 1), gv, (j + 1) * kB, Nk, ldk, tid);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    float s[kB / 8][4], dp[kB / 8][4];
#pragma unroll
    for (int i = 0; i < kB / 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[i][e] = dp[i][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t qa[4], oa[4];
      frag_a<kB>(qa, sQ, warp * 16, kk * 16, lane);
      frag_a<kB>(oa, sdO, warp * 16, kk * 16, lane);
#pragma unroll
      for (int np = 0; np < kB / 16; ++np) {
        uint32_t bk[4], bv[4];
        frag_b_nk<kB>(bk, sK(st), np * 16, kk * 16, lane);
        frag_b_nk<kB>(bv, sV(st), np * 16, kk * 16, lane);
        mma16816<T>(s[2 * np], qa, bk[0], bk[1]);
        mma16816<T>(s[2 * np + 1], qa, bk[2], bk[3]);
        mma16816<T>(dp[2 * np], oa, bv[0], bv[1]);
        mma16816<T>(dp[2 * np + 1], oa, bv[2], bv[3]);
      }
    }
    const int n0 = j * kB;
    const bool need_mask = (n0 + kB > Nk) || (CAUSAL && n0 + kB - 1 > m0 + off);
#pragma unroll
    for (int kk = 0; kk < kB / 16; ++kk) {
      float ds[2][4];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int nb = 2 * kk + u;
          float pv = ex2(fmaf(s[nb][e], c, -lse2[e >> 1]));
          if (need_mask) {
            const int key = n0 + nb * 8 + 2 * (lane & 3) + (e & 1);
            const int row = r_lo + ((e >> 1) << 3);
            if (key >= Nk || (CAUSAL && key > row + off)) pv = 0.f;
          }
          ds[u][e] = pv * (dp[nb][e] - dvr[e >> 1]);
        }
      uint32_t da[4];
      da[0] = Elem<T>::pack(ds[0][0], ds[0][1]);
      da[1] = Elem<T>::pack(ds[0][2], ds[0][3]);
      da[2] = Elem<T>::pack(ds[1][0], ds[1][1]);
      da[3] = Elem<T>::pack(ds[1][2], ds[1][3]);
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {
        uint32_t bb[4];
        frag_b_kn<kB>(bb, sK(st), kk * 16, np * 16, lane);
        mma16816<T>(dq[2 * np], da, bb[0], bb[1]);
        mma16816<T>(dq[2 * np + 1], da, bb[2], bb[3]);
      }
    }
    __syncthreads();
  }

  uint16_t* gdq = static_cast<uint16_t*>(p.dq) + ((long)b * Nq * p.Hq + h) * D;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const int col = i * 8 + 2 * (lane & 3);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int row = r_lo + 8 * u;
      if (row < Nq)
        *reinterpret_cast<uint32_t*>(gdq + row * ldq + col) =
            Elem<T>::pack(dq[i][2 * u] * p.scale, dq[i][2 * u + 1] * p.scale);
    }
  }
}

template <typename T, int D>
cudaError_t launch_pre_t(const BwdArgs& a, cudaStream_t s) {
  const long R = (long)a.B * a.Nq * a.Hq;
  const long threads = R * (D / 8);
  const int blocks = (int)((threads + 255) / 256);
  bwd_pre_kernel<T, D><<<blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

template <typename T, int D, bool CAUSAL>
cudaError_t launch_dkdv_t(const BwdArgs& a, cudaStream_t s) {
  const int smem = 6 * kB * D * 2 + 4 * kB * 4;
  auto kern = bwd_dkdv_kernel<T, D, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.Nk + kB - 1) / kB, a.Hkv, a.B);
  kern<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <typename T, int D, bool CAUSAL>
cudaError_t launch_dq_t(const BwdArgs& a, cudaStream_t s) {
  const int smem = 6 * kB * D * 2;
  auto kern = bwd_dq_kernel<T, D, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.Nq + kB - 1) / kB, a.Hq, a.B);
  kern<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_preprocess(const BwdArgs& a, cudaStream_t s) {
  if (a.bf16) return a.d == 128 ? launch_pre_t<__nv_bfloat16, 128>(a, s) : launch_pre_t<__nv_bfloat16, 64>(a, s);
  return a.d == 128 ? launch_pre_t<__half, 128>(a, s) : launch_pre_t<__half, 64>(a, s);
}

#define FA_DISPATCH_BWD(FN, a, s)                                                          \
  do {                                                                                     \
    if (a.bf16) {                                                                          \
      if (a.d == 128) return a.causal ? FN<__nv_bfloat16, 128, true>(a, s)                 \
                                      : FN<__nv_bfloat16, 128, false>(a, s);               \
      return a.causal ? FN<__nv_bfloat16, 64, true>(a, s) : FN<__nv_bfloat16, 64, false>(a, s); \
    }                                                                                      \
    if (a.d == 128) return a.causal ? FN<__half, 128, true>(a, s) : FN<__half, 128, false>(a, s); \
    return a.causal ? FN<__half, 64, true>(a, s) : FN<__half, 64, false>(a, s);            \
  } while (0)

cudaError_t launch_bwd_dkdv(const BwdArgs& a, cudaStream_t s) { FA_DISPATCH_BWD(launch_dkdv_t, a, s); }
cudaError_t launch_bwd_dq(const BwdArgs& a, cudaStream_t s) { FA_DISPATCH_BWD(launch_dq_t, a, s); }

}  // namespace fa
