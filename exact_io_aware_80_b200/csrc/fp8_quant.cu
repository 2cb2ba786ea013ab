// fp8_quant.cu -- E4M3 operands for the FP8 forward pass.
//
// "FlashAttention-2 (KO)" (FA-3 paragraph) names low-precision FP8 with
// incoherent processing as FlashAttention-3's forward path; the pages give no
// formats, so the library fixes them:
//   * E4M3 codes (round to nearest even, saturating to +-448) via
//     cvt.rn.satfinite.e4m3x2.f32;
//   * Q and K: one fp32 scale per (batch, head, 128-row block), s = amax / 448
//     (1 when the block is all zero), code = E4M3(y / s) with a correctly
//     rounded fp32 division; optionally the rows are first multiplied by the
//     caller's +-1 signs and by the unnormalised d x d Walsh-Hadamard matrix
//     (butterflies (a, b) -> (a + b, a - b) for h = 1, 2, 4, ..., d / 2, in
//     fp32), which multiplies every score by d;
//   * V: one scale per (batch, kv head) over all keys, codes stored transposed
//     as [B, Hkv, d, Nk_pad] (Nk_pad = Nk rounded up to 16; zero codes in the
//     padding) so that the P V product reads V K-major.
// These kernels move Nq x d (or Nk x d) 16-bit values once; they are bound by
// HBM bandwidth and run once per input, outside the attention kernel.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace fa {
namespace {

constexpr int kRows = 128;  // rows per quantization block (= threads per CTA)

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

template <typename T>
__device__ __forceinline__ void load_row(const T* src, float* y, int d) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  for (int i = 0; i < d / 8; ++i) {
    const uint4 w = s4[i];
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = Elem<T>::unpack(u[k]);
      y[8 * i + 2 * k] = f.x;
      y[8 * i + 2 * k + 1] = f.y;
    }
  }
}

// In-place unnormalised Walsh-Hadamard transform of y[0..D), fp32 butterflies
// in the order h = 1, 2, 4, ..., D / 2.
template <int D>
__device__ __forceinline__ void fwht(float (&y)[D]) {
#pragma unroll
  for (int h = 1; h < D; h *= 2)
#pragma unroll
    for (int i = 0; i < D; ++i)
      if ((i & h) == 0) {
        const float a = y[i], b = y[i + h];
        y[i] = __fadd_rn(a, b);
        y[i + h] = __fsub_rn(a, b);
      }
}

// Block maximum of v over the CTA's 128 threads.
__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  v = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  return v;
}

__device__ __forceinline__ float scale_of(float amax) { return amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f; }

// grid (row blocks, H, B), 128 threads: thread r quantises row 128 blockIdx.x + r.
template <typename T, int D>
__global__ void __launch_bounds__(kRows) quant_qk_kernel(const T* __restrict__ x, uint8_t* __restrict__ x8,
                                                          float* __restrict__ scales, const float* __restrict__ signs,
                                                          int N, int H) {
  __shared__ float red[4];
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int n = j * kRows + threadIdx.x;
  const bool valid = n < N;
  const long row = ((long)b * N + n) * H + h;
  float y[D];
  if (valid) {
    load_row(x + row * D, y, D);
  } else {
#pragma unroll
    for (int i = 0; i < D; ++i) y[i] = 0.f;
  }
  if (signs) {
#pragma unroll
    for (int i = 0; i < D; ++i) y[i] = y[i] * signs[i];  // exact: +-1
    fwht<D>(y);
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < D; ++i) amax = fmaxf(amax, fabsf(y[i]));
  amax = block_max(amax, red);
  const float s = scale_of(amax);
  if (threadIdx.x == 0) scales[((long)b * H + h) * gridDim.x + j] = s;
  if (!valid) return;
  uint4* dst = reinterpret_cast<uint4*>(x8 + row * D);
#pragma unroll
  for (int i = 0; i < D / 16; ++i) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = 16 * i + 4 * k;
      const uint32_t lo = e4m3x2(__fdiv_rn(y[c], s), __fdiv_rn(y[c + 1], s));
      const uint32_t hi = e4m3x2(__fdiv_rn(y[c + 2], s), __fdiv_rn(y[c + 3], s));
      w[k] = lo | (hi << 16);
    }
    dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// grid (row blocks, Hkv, B): amax of every 128-key block of V into part[b][h][j].
template <typename T, int D>
__global__ void __launch_bounds__(kRows) v_amax_kernel(const T* __restrict__ v, float* __restrict__ part, int Nk,
                                                        int H) {
  __shared__ float red[4];
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int n = j * kRows + threadIdx.x;
  float amax = 0.f;
  if (n < Nk) {
    float y[D];
    load_row(v + (((long)b * Nk + n) * H + h) * D, y, D);
#pragma unroll
    for (int i = 0; i < D; ++i) amax = fmaxf(amax, fabsf(y[i]));
  }
  amax = block_max(amax, red);
  if (threadIdx.x == 0) part[((long)b * H + h) * gridDim.x + j] = amax;
}

// grid (row blocks, Hkv, B): quantise 128 keys of V with the head's scale and
// write them transposed, [d][128 keys] per block, through shared memory.
template <typename T, int D>
__global__ void __launch_bounds__(kRows) v_quant_kernel(const T* __restrict__ v, const float* __restrict__ part,
                                                         uint8_t* __restrict__ v8t, float* __restrict__ scale,
                                                         int Nk, int H, int Npad) {
  __shared__ __align__(16) uint8_t tile[D][kRows + 16];
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nb = gridDim.x;
  float amax = 0.f;
  const float* ph = part + ((long)b * H + h) * nb;
  for (int i = 0; i < nb; ++i) amax = fmaxf(amax, ph[i]);
  const float s = scale_of(amax);
  if (j == 0 && threadIdx.x == 0) scale[(long)b * H + h] = s;
  const int r = threadIdx.x, n = j * kRows + r;
  if (n < Nk) {
    float y[D];
    load_row(v + (((long)b * Nk + n) * H + h) * D, y, D);
#pragma unroll
    for (int c = 0; c < D; c += 2) {
      const uint16_t p = e4m3x2(__fdiv_rn(y[c], s), __fdiv_rn(y[c + 1], s));
      tile[c][r] = (uint8_t)(p & 0xFF);
      tile[c + 1][r] = (uint8_t)(p >> 8);
    }
  } else {
#pragma unroll
    for (int c = 0; c < D; ++c) tile[c][r] = 0;
  }
  __syncthreads();
  // row c of the block: keys 128 j .. 128 j + 127, clipped to Npad (a multiple of 16)
  const int nkeys = min(kRows, Npad - j * kRows);
  uint8_t* base = v8t + ((long)b * H + h) * D * (long)Npad + (long)j * kRows;
  for (int e = threadIdx.x; e < D * (kRows / 16); e += kRows) {
    const int c = e / (kRows / 16), q = e % (kRows / 16);
    if (16 * q < nkeys) {
      const uint32_t* t4 = reinterpret_cast<const uint32_t*>(&tile[c][16 * q]);
      *reinterpret_cast<uint4*>(base + (long)c * Npad + 16 * q) = make_uint4(t4[0], t4[1], t4[2], t4[3]);
    }
  }
}

template <typename T, int D>
cudaError_t launch_qk(const Fp8QuantArgs& a, cudaStream_t s) {
  dim3 grid((a.N + kRows - 1) / kRows, a.H, a.B);
  quant_qk_kernel<T, D><<<grid, kRows, 0, s>>>(static_cast<const T*>(a.x), static_cast<uint8_t*>(a.x8), a.scales,
                                              a.signs, a.N, a.H);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_v(const Fp8QuantArgs& a, cudaStream_t s) {
  dim3 grid((a.N + kRows - 1) / kRows, a.H, a.B);
  v_amax_kernel<T, D><<<grid, kRows, 0, s>>>(static_cast<const T*>(a.x), a.work, a.N, a.H);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  v_quant_kernel<T, D><<<grid, kRows, 0, s>>>(static_cast<const T*>(a.x), a.work, static_cast<uint8_t*>(a.x8),
                                             a.scales, a.N, a.H, (a.N + 15) / 16 * 16);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fp8_quant_qk(const Fp8QuantArgs& a, cudaStream_t s) {
  if (a.bf16) return a.d == 128 ? launch_qk<__nv_bfloat16, 128>(a, s) : launch_qk<__nv_bfloat16, 64>(a, s);
  return a.d == 128 ? launch_qk<__half, 128>(a, s) : launch_qk<__half, 64>(a, s);
}

cudaError_t launch_fp8_quant_v(const Fp8QuantArgs& a, cudaStream_t s) {
  if (a.bf16) return a.d == 128 ? launch_v<__nv_bfloat16, 128>(a, s) : launch_v<__nv_bfloat16, 64>(a, s);
  return a.d == 128 ? launch_v<__half, 128>(a, s) : launch_v<__half, 64>(a, s);
}

}  // namespace fa
