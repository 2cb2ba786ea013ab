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

template <typename T, int D>
cudaError_t launch_pre_t(const BwdArgs& a, cudaStream_t s) {
  const long R = (long)a.B * a.Nq * a.Hq;
  const long threads = R * (D / 8);
  const int blocks = (int)((threads + 255) / 256);
  bwd_pre_kernel<T, D><<<blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_preprocess(const BwdArgs& a, cudaStream_t s) {
  if (a.bf16) return a.d == 128 ? launch_pre_t<__nv_bfloat16, 128>(a, s) : launch_pre_t<__nv_bfloat16, 64>(a, s);
  return a.d == 128 ? launch_pre_t<__half, 128>(a, s) : launch_pre_t<__half, 64>(a, s);
}

}  // namespace fa
