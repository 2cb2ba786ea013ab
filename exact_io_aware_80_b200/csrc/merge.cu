// merge.cu -- log-sum-exp merge of partial attention results (context-parallel
// ring attention: each rank attends its queries to one key/value chunk at a
// time and folds the partial result into an accumulator).
//
// The merge is the split-combine of "FlashAttention 심층 분석" ("Flash-Decoding":
// partial results over key ranges are merged by their log-sum-exp): for a row
// with accumulated (O_a, L_a) and a partial (O_p, L_p) over disjoint keys,
//   L = ln(e^{L_a} + e^{L_p}),  O = e^{L_a - L} O_a + e^{L_p - L} O_p,
// with -inf for a row that has seen no key (weight 0; both -inf gives O = 0).
// One warp per (b, row, head); fp32 accumulator, 16-bit partials and output.
// Also here: the fp32 accumulation of 16-bit gradient partials and the final
// cast (the backward of the ring sums per-chunk dQ / dK / dV contributions).
// HBM-bound: per row it moves 4 d (accumulator in) + 2 d (partial) + 4 d
// (accumulator out) bytes, or 2 d for the final 16-bit output.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace fa {
namespace {

// mode 0: acc = part; 1: acc = merge(acc, part); 2: out (16-bit) = merge(acc, part), lse_acc updated
template <typename T, int D>
__global__ void __launch_bounds__(128) lse_merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc,
                                                         const T* __restrict__ o_part,
                                                         const float* __restrict__ lse_part, T* __restrict__ o_out,
                                                         long rows, int N, int H, int mode) {
  const long r = (long)blockIdx.x * 4 + (threadIdx.x >> 5);  // row index over [B][N][H]
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const int h = (int)(r % H);
  const long bn = r / H;
  const int n = (int)(bn % N);
  const long b = bn / N;
  const long li = (b * H + h) * N + n;  // lse index [B][H][N]
  const float lp = lse_part[li];
  float wa = 0.f, wp = 1.f, L = lp;
  if (mode != 0) {
    const float la = lse_acc[li];
    const float m = fmaxf(la, lp);
    if (m == -INFINITY) {
      wa = 0.f;
      wp = 0.f;
      L = -INFINITY;
    } else {
      const float ea = expf(la - m), ep = expf(lp - m);
      L = m + logf(ea + ep);
      wa = expf(la - L);
      wp = expf(lp - L);
    }
  } else if (lp == -INFINITY) {
    wp = 0.f;
  }
  constexpr int kPer = D / 32;  // elements per lane
  const long base = r * D + lane * kPer;
  float a[kPer], pv[kPer];
#pragma unroll
  for (int i = 0; i < kPer; i += 2) {
    const float2 f = Elem<T>::unpack(*reinterpret_cast<const uint32_t*>(o_part + base + i));
    pv[i] = f.x;
    pv[i + 1] = f.y;
  }
  if (mode != 0) {
#pragma unroll
    for (int i = 0; i < kPer; ++i) a[i] = o_acc[base + i];
  } else {
#pragma unroll
    for (int i = 0; i < kPer; ++i) a[i] = 0.f;
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) a[i] = wa * a[i] + wp * pv[i];
  if (mode == 2) {
#pragma unroll
    for (int i = 0; i < kPer; i += 2) *reinterpret_cast<uint32_t*>(o_out + base + i) = Elem<T>::pack(a[i], a[i + 1]);
  } else {
#pragma unroll
    for (int i = 0; i < kPer; ++i) o_acc[base + i] = a[i];
  }
  if (lane == 0) lse_acc[li] = L;
}

template <typename T, int D>
cudaError_t launch_merge_t(const MergeArgs& a, cudaStream_t s) {
  const long rows = (long)a.B * a.N * a.H;
  const long blocks = (rows + 3) / 4;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  lse_merge_kernel<T, D><<<(unsigned)blocks, 128, 0, s>>>(a.o_acc, a.lse_acc, static_cast<const T*>(a.o_part),
                                                          a.lse_part, static_cast<T*>(a.o_out), rows, a.N, a.H, a.mode);
  return cudaGetLastError();
}

// acc = (init ? 0 : acc) + part (16-bit), 8 elements per thread
template <typename T>
__global__ void accumulate_kernel(float* __restrict__ acc, const T* __restrict__ part, long n8, int init) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const uint4 w = reinterpret_cast<const uint4*>(part)[i];
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
  float4* a4 = reinterpret_cast<float4*>(acc) + 2 * i;
  float4 lo = init ? make_float4(0.f, 0.f, 0.f, 0.f) : a4[0];
  float4 hi = init ? make_float4(0.f, 0.f, 0.f, 0.f) : a4[1];
  const float2 f0 = Elem<T>::unpack(u[0]), f1 = Elem<T>::unpack(u[1]), f2 = Elem<T>::unpack(u[2]),
               f3 = Elem<T>::unpack(u[3]);
  lo.x += f0.x; lo.y += f0.y; lo.z += f1.x; lo.w += f1.y;
  hi.x += f2.x; hi.y += f2.y; hi.z += f3.x; hi.w += f3.y;
  a4[0] = lo;
  a4[1] = hi;
}

// out (16-bit) = acc, 8 elements per thread
template <typename T>
__global__ void cast_kernel(const float* __restrict__ acc, T* __restrict__ out, long n8) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 lo = reinterpret_cast<const float4*>(acc)[2 * i], hi = reinterpret_cast<const float4*>(acc)[2 * i + 1];
  reinterpret_cast<uint4*>(out)[i] = make_uint4(Elem<T>::pack(lo.x, lo.y), Elem<T>::pack(lo.z, lo.w),
                                                Elem<T>::pack(hi.x, hi.y), Elem<T>::pack(hi.z, hi.w));
}

}  // namespace

cudaError_t launch_accumulate(float* acc, const void* part, long n, int init, int bf16, cudaStream_t s) {
  const long n8 = n / 8;
  const long blocks = (n8 + 255) / 256;
  if (n8 == 0) return cudaSuccess;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  if (bf16)
    accumulate_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(acc, static_cast<const __nv_bfloat16*>(part), n8,
                                                                        init);
  else
    accumulate_kernel<__half><<<(unsigned)blocks, 256, 0, s>>>(acc, static_cast<const __half*>(part), n8, init);
  return cudaGetLastError();
}

cudaError_t launch_cast(const float* acc, void* out, long n, int bf16, cudaStream_t s) {
  const long n8 = n / 8;
  const long blocks = (n8 + 255) / 256;
  if (n8 == 0) return cudaSuccess;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  if (bf16)
    cast_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(acc, static_cast<__nv_bfloat16*>(out), n8);
  else
    cast_kernel<__half><<<(unsigned)blocks, 256, 0, s>>>(acc, static_cast<__half*>(out), n8);
  return cudaGetLastError();
}

cudaError_t launch_lse_merge(const MergeArgs& a, cudaStream_t s) {
  if (a.bf16) return a.d == 128 ? launch_merge_t<__nv_bfloat16, 128>(a, s) : launch_merge_t<__nv_bfloat16, 64>(a, s);
  return a.d == 128 ? launch_merge_t<__half, 128>(a, s) : launch_merge_t<__half, 64>(a, s);
}

}  // namespace fa
