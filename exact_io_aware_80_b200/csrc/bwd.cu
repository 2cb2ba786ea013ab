// bwd.cu -- backward preprocess: D_i = sum_c dO_ic O_ic, the row term of the
// softmax Jacobian (D_i = sum_j P_ij dP_ij) that the dK/dV and dQ kernels of
// bwd_sm100.cu subtract from dP.  HBM-bound: each row of O and dO is read once
// with 16-byte loads and reduced across the threads that share the row.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace fa {
namespace {

// ---------------------------------------------------------------------------
// D = rowsum(dO * O)
// ---------------------------------------------------------------------------
// D / 8 threads share a row (16 bytes each), so a warp reads 256 contiguous bytes of
// each of 32 / (D / 8) rows per load; each thread takes kRowsPerThread rows of one
// (b, h), consecutive query positions, and issues all of their loads before any
// arithmetic so that every thread has 2 * kRowsPerThread 16-byte loads in flight.
// A warp's rows are consecutive positions i of one (b, h), so the D values it writes
// are contiguous; consecutive warps take consecutive heads at the same positions, so
// the warps in flight together read neighbouring memory (position i of every head is
// one contiguous stretch of O and dO).
constexpr int kRowsPerThread = 8;

template <typename T, int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(BwdArgs p) {
  constexpr int TPR = D / 8;         // threads per row
  constexpr int RPW = 32 / TPR;      // rows per warp per load
  constexpr int WROWS = RPW * kRowsPerThread;  // rows per warp
  const int lane = threadIdx.x & 31;
  const long warp = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int part = lane % TPR, sub = lane / TPR;
  const long groups = (p.Nq + WROWS - 1) / WROWS;  // position groups per (b, h)
  const long BH = (long)p.B * p.Hq;
  if (warp >= BH * groups) return;
  const long bb = warp / (groups * p.Hq);  // batch, then position group, then head (fastest)
  const long rest = warp % (groups * p.Hq);
  const int h = (int)(rest % p.Hq);
  const int i0 = (int)(rest / p.Hq) * WROWS;
  const long bh = bb * p.Hq + h;
  uint4 o[kRowsPerThread], g[kRowsPerThread];
#pragma unroll
  for (int k = 0; k < kRowsPerThread; ++k) {
    const int i = i0 + k * RPW + sub;
    const long off = ((bb * p.Nq + i) * p.Hq + h) * D;
    if (i < p.Nq && FA_IN_BOUNDS(p.status, off + D - 1, (long)p.B * p.Nq * p.Hq * D)) {
      o[k] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.o) + off) + part);
      g[k] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.dout) + off) + part);
    } else {
      o[k] = g[k] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
#pragma unroll
  for (int k = 0; k < kRowsPerThread; ++k) {
    const uint32_t ov[4] = {o[k].x, o[k].y, o[k].z, o[k].w};
    const uint32_t gv[4] = {g[k].x, g[k].y, g[k].z, g[k].w};
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 a = Elem<T>::unpack(ov[e]), c = Elem<T>::unpack(gv[e]);
      acc = fmaf(a.x, c.x, acc);
      acc = fmaf(a.y, c.y, acc);
    }
#pragma unroll
    for (int w = 1; w < TPR; w <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
    const int i = i0 + k * RPW + sub;
    if (part == 0 && i < p.Nq && FA_IN_BOUNDS(p.status, bh * p.Nq + i, (long)p.B * p.Hq * p.Nq))
      p.dvec[bh * p.Nq + i] = acc;
  }
}

template <typename T, int D>
cudaError_t launch_pre_t(const BwdArgs& a, cudaStream_t s) {
  constexpr int WROWS = (32 / (D / 8)) * kRowsPerThread;
  const long warps = (long)a.B * a.Hq * ((a.Nq + WROWS - 1) / WROWS);
  const long blocks = (warps + 7) / 8;
  if (blocks > 0x7fffffffL) return cudaErrorInvalidValue;
  bwd_pre_kernel<T, D><<<(unsigned)blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_preprocess(const BwdArgs& a, cudaStream_t s) {
  if (a.bf16) return a.d == 128 ? launch_pre_t<__nv_bfloat16, 128>(a, s) : launch_pre_t<__nv_bfloat16, 64>(a, s);
  return a.d == 128 ? launch_pre_t<__half, 128>(a, s) : launch_pre_t<__half, 64>(a, s);
}

}  // namespace fa
