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
//
// These kernels move each 16-bit input once (V twice: its per-head scale
// needs the amax of every key first) and are bound by HBM bandwidth.  One CTA
// of 128 threads takes one 128-row block of one head: the block is staged in
// shared memory with coalesced 16-byte cp.async copies (a row is contiguous,
// rows of one head are H * d elements apart), each thread then works on one
// row in registers (rotation, block amax, division, E4M3 packing), and the
// codes leave through shared memory with coalesced 16-byte stores.  The Q, K
// and V-amax blocks of a forward pass run in one persistent launch whose CTAs
// stage their next block while working on the current one; V's transposing
// encode is a second launch, since it needs the head's amax.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <algorithm>

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

// In-place unnormalised Walsh-Hadamard transform of y[0..D), fp32 butterflies
// (a, b) -> (a + b, a - b) in the order h = 1, 2, 4, ..., D / 2.  From h = 2 on, the
// butterflies of elements i and i + 1 run as one packed f32x2 instruction each
// (a - b as the fused a + (-1) b: the product is exact, so it rounds once, as a
// subtraction does).
template <int D>
__device__ __forceinline__ void fwht(float (&y)[D]) {
#pragma unroll
  for (int i = 0; i < D; i += 2) {
    const float a = y[i], b = y[i + 1];
    y[i] = __fadd_rn(a, b);
    y[i + 1] = __fsub_rn(a, b);
  }
#pragma unroll
  for (int h = 2; h < D; h *= 2)
#pragma unroll
    for (int i = 0; i < D; i += 2)
      if ((i & h) == 0) {
        const float2 a = make_float2(y[i], y[i + 1]), b = make_float2(y[i + h], y[i + h + 1]);
        const float2 sum = __fadd2_rn(a, b), dif = __ffma2_rn(b, make_float2(-1.f, -1.f), a);
        y[i] = sum.x;
        y[i + 1] = sum.y;
        y[i + h] = dif.x;
        y[i + h + 1] = dif.y;
      }
}

// y / s correctly rounded to fp32, for one divisor and many dividends, without a division per
// element: r = RN(1 / s), q1 = RN(y r), then one correction q = q1 + (y - q1 s) r with fused
// multiply-adds.  With r correctly rounded and q1 within an ulp of y / s, the corrected quotient
// is RN(y / s) (Markstein's theorem for FMA-based division), provided no intermediate leaves
// the normal range, which holds for 2^-90 <= s <= 2^90 whenever |y / s| >= 2^-11; other divisors
// take the IEEE division.  Smaller quotients may come out inexact, but every value below 2^-10
// has the E4M3 code +-0 (the smallest code, 2^-9, takes values from 2^-10 up), and q keeps y's
// sign, which q1 carries: the only case where the correction can flip it is y = -0 (q1 = -0,
// q = +0), so q1's sign bit is OR-ed into q.  The choice between the two forms is made once per
// block by the caller (div2<true> or div2<false>), so that the per-element code has no branch.
struct Divider {
  float s, r;
  bool fast;
  template <bool FAST>
  __device__ __forceinline__ float2 div2(float2 y) const {
    if constexpr (!FAST) {
      return make_float2(__fdiv_rn(y.x, s), __fdiv_rn(y.y, s));
    } else {
      const float2 q1 = __fmul2_rn(y, make_float2(r, r));
      const float2 e = __ffma2_rn(q1, make_float2(-s, -s), y);
      const float2 q = __ffma2_rn(e, make_float2(r, r), q1);
      return make_float2(__int_as_float(__float_as_int(q.x) | (__float_as_int(q1.x) & 0x80000000)),
                         __int_as_float(__float_as_int(q.y) | (__float_as_int(q1.y) & 0x80000000)));
    }
  }
};
__device__ __forceinline__ Divider make_divider(float s) {
  Divider d;
  d.s = s;
  d.r = __frcp_rn(s);
  d.fast = s >= 0x1p-90f && s <= 0x1p90f;
  return d;
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

// Staged rows: D 16-bit values plus 16 bytes of padding, so that 8 threads reading
// 16 bytes of 8 consecutive rows hit distinct banks (row stride = 4 banks mod 32).
template <int D>
struct Stage {
  static constexpr int kRowBytes = 2 * D + 16;
  static constexpr int kBytes = kRows * kRowBytes;
  static constexpr int kChunks = D / 8;  // 16-byte chunks per row
};

// Rows n0 .. n0 + 127 of head h, batch b of x [B, N, H, D] into the stage (rows
// past N as zeros): 16-byte cp.async copies, consecutive threads on consecutive
// chunks.  Issued only; the caller commits and waits.
template <typename T, int D>
__device__ __forceinline__ void issue_rows(const T* x, uint8_t* st, int N, int H, int b, int h, int n0) {
  using S = Stage<D>;
  const uint32_t base = smem_u32(st);
#pragma unroll 4
  for (int e = threadIdx.x; e < kRows * S::kChunks; e += kRows) {
    const int r = e / S::kChunks, c = e % S::kChunks;
    const int n = n0 + r;
    const bool ok = n < N;
    const T* src = x + (((long)b * N + (ok ? n : 0)) * H + h) * D + 8 * c;
    cp_async16(base + r * S::kRowBytes + 16 * c, src, ok);
  }
}
// Row r of the stage as fp32.
template <typename T, int D>
__device__ __forceinline__ void read_row(const uint8_t* st, int r, float (&y)[D]) {
  const uint4* s4 = reinterpret_cast<const uint4*>(st + r * Stage<D>::kRowBytes);
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
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

// E4M3 codes of one row y / s, 16 at a time into row[0 .. D / 16).
template <int D, bool FAST>
__device__ __forceinline__ void encode_row(const float (&y)[D], const Divider& dv, uint4* row) {
#pragma unroll
  for (int i = 0; i < D / 16; ++i) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = 16 * i + 4 * k;
      const float2 lo = dv.div2<FAST>(make_float2(y[c], y[c + 1]));
      const float2 hi = dv.div2<FAST>(make_float2(y[c + 2], y[c + 3]));
      w[k] = (uint32_t)e4m3x2(lo.x, lo.y) | ((uint32_t)e4m3x2(hi.x, hi.y) << 16);
    }
    row[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// One 128-row block of Q or K: (signs, Walsh-Hadamard), block amax, scale, E4M3 codes.
template <typename T, int D>
__device__ __forceinline__ void quant_rows_block(const QuantJob& job, const float* signs, int j, int h, int b, int B,
                                                 uint8_t* st, float* red, int* status) {
  using S = Stage<D>;
  const int r = threadIdx.x;
  float y[D];
  read_row<T, D>(st, r, y);
  if (signs) {  // the rotation signs, staged in shared memory by the kernel
    const float4* s4 = reinterpret_cast<const float4*>(signs);
#pragma unroll
    for (int i = 0; i < D / 4; ++i) {
      const float4 g = s4[i];
      const float2 a = __fmul2_rn(make_float2(y[4 * i], y[4 * i + 1]), make_float2(g.x, g.y));  // exact: +-1
      const float2 c = __fmul2_rn(make_float2(y[4 * i + 2], y[4 * i + 3]), make_float2(g.z, g.w));
      y[4 * i] = a.x;
      y[4 * i + 1] = a.y;
      y[4 * i + 2] = c.x;
      y[4 * i + 3] = c.y;
    }
    fwht<D>(y);
  }
  float am[4] = {0.f, 0.f, 0.f, 0.f};  // four independent chains
#pragma unroll
  for (int i = 0; i < D; i += 4)
#pragma unroll
    for (int k = 0; k < 4; ++k) am[k] = fmaxf(am[k], fabsf(y[i + k]));
  float amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
  amax = block_max(amax, red);  // its barriers also order every read of the stage before the writes below
  const float s = scale_of(amax);
  if (r == 0 && FA_IN_BOUNDS(status, ((long)b * job.H + h) * job.nblk + j, (long)B * job.H * job.nblk))
    job.scales[((long)b * job.H + h) * job.nblk + j] = s;
  const Divider dv = make_divider(s);
  // codes of row r over the first D bytes of its own stage row
  uint4* row = reinterpret_cast<uint4*>(st + r * S::kRowBytes);
  if (dv.fast)
    encode_row<D, true>(y, dv, row);
  else
    encode_row<D, false>(y, dv, row);
  __syncthreads();
  // D code bytes per row, 16 at a time, consecutive threads on consecutive chunks of a row
  constexpr int C8 = D / 16;
  const int n0 = j * kRows;
#pragma unroll 4
  for (int e = threadIdx.x; e < kRows * C8; e += kRows) {
    const int rr = e / C8, c = e % C8;
    const int n = n0 + rr;
    const long ci = (((long)b * job.N + n) * job.H + h) * D + 16 * c;
    if (n < job.N && FA_IN_BOUNDS(status, ci + 15, (long)B * job.N * job.H * D))
      *reinterpret_cast<uint4*>(job.x8 + ci) = *reinterpret_cast<const uint4*>(st + rr * S::kRowBytes + 16 * c);
  }
}

// Amax of one staged 128-key block of V into part[b][h][j] (rows past N were staged as zeros).
template <typename T, int D>
__device__ __forceinline__ void v_amax_block(const QuantJob& job, int j, int h, int b, int B, const uint8_t* st,
                                             float* red, int* status) {
  float y[D];
  read_row<T, D>(st, threadIdx.x, y);
  float am[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < D; i += 4)
#pragma unroll
    for (int k = 0; k < 4; ++k) am[k] = fmaxf(am[k], fabsf(y[i + k]));
  const float amax = block_max(fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3])), red);
  if (threadIdx.x == 0 && FA_IN_BOUNDS(status, ((long)b * job.H + h) * job.nblk + j, (long)B * job.H * job.nblk))
    job.scales[((long)b * job.H + h) * job.nblk + j] = amax;
}

// One persistent launch over up to three jobs (Q rows, K rows, V block maxima).  The flat
// block index walks job 0's blocks (j fastest, then h, then b), then job 1's, then job 2's;
// CTA i takes blocks i, i + G, i + 2G, ... and stages block i + G into its second buffer
// while it works on block i, so the copies overlap the arithmetic.
struct BlockRef {
  int job, j, h, b;
};
__device__ __forceinline__ BlockRef block_ref(const QuantJobs& jobs, long id, int B) {
  int k = 0;
  while (k < jobs.n - 1 && id >= (long)jobs.job[k].nblk * jobs.job[k].H * B) {
    id -= (long)jobs.job[k].nblk * jobs.job[k].H * B;
    ++k;
  }
  const int nb = jobs.job[k].nblk, H = jobs.job[k].H;
  return BlockRef{k, (int)(id % nb), (int)((id / nb) % H), (int)(id / ((long)nb * H))};
}

template <typename T, int D>
__device__ __forceinline__ void issue_block(const QuantJobs& jobs, const BlockRef& r, uint8_t* st) {
  const QuantJob& job = jobs.job[r.job];
  issue_rows<T, D>(static_cast<const T*>(job.x), st, job.N, job.H, r.b, r.h, r.j * kRows);
}

template <typename T, int D>
__global__ void __launch_bounds__(kRows, 3) quant_kernel(QuantJobs jobs, const float* __restrict__ signs, int B,
                                                      long total) {
  extern __shared__ __align__(16) uint8_t q_smem[];  // two stages
  __shared__ float red[4];
  __shared__ __align__(16) float s_signs[D];
  uint8_t* stage[2] = {q_smem, q_smem + Stage<D>::kBytes};
  if (signs)
    for (int i = threadIdx.x; i < D; i += kRows) s_signs[i] = signs[i];
  const float* sg = signs ? s_signs : nullptr;  // visible to every thread after the loop's first barrier
  // V's encode, launched next as a programmatic dependent, may stage its V rows meanwhile; it
  // waits for this grid before it reads the block maxima
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  long id = blockIdx.x;
  if (id < total) issue_block<T, D>(jobs, block_ref(jobs, id, B), stage[0]);
  cp_async_commit();
  for (int it = 0; id < total; ++it, id += gridDim.x) {
    const long nxt = id + gridDim.x;
    if (nxt < total) issue_block<T, D>(jobs, block_ref(jobs, nxt, B), stage[(it + 1) & 1]);
    cp_async_commit();
    cp_async_wait<1>();  // this block's copies have landed (the next block's may still fly)
    __syncthreads();
    const BlockRef r = block_ref(jobs, id, B);
    const QuantJob& job = jobs.job[r.job];
    if (job.kind == kQuantRows)
      quant_rows_block<T, D>(job, sg, r.j, r.h, r.b, B, stage[it & 1], red, jobs.status);
    else
      v_amax_block<T, D>(job, r.j, r.h, r.b, B, stage[it & 1], red, jobs.status);
    __syncthreads();  // every thread is done with this buffer before it is refilled
  }
  cp_async_wait<0>();
}

// Codes of a staged V block, transposed: thread t takes the column pair (2p, 2p + 1),
// p = t mod (D / 2), over the keys [K g, K g + K) with g = t div (D / 2) and K = 128 / (128 / (D / 2))
// = D / 2 keys; one 32-bit shared-memory read gives both columns of a key (rows past Nk were
// staged as zeros).  Code row c of out holds the 128 keys of column c (kRows + 16 bytes per row).
template <typename T, int D, bool FAST>
__device__ __forceinline__ void encode_columns(const uint8_t* st, uint8_t* out, const Divider& dv) {
  using S = Stage<D>;
  constexpr int kOutRow = kRows + 16;
  constexpr int P = D / 2, K = P;
  static_assert(kRows % P == 0 && (kRows / P) * K == kRows, "column pairs x key groups = threads");
  const int p = threadIdx.x % P, g = threadIdx.x / P;
#pragma unroll 2
  for (int k16 = 0; k16 < K / 16; ++k16) {
    const int key0 = K * g + 16 * k16;
    uint32_t w0[4], w1[4];  // codes of column 2p and 2p + 1
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float2 f[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        f[e] = Elem<T>::unpack(*reinterpret_cast<const uint32_t*>(st + (key0 + 4 * q + e) * S::kRowBytes + 4 * p));
      const float2 a0 = dv.div2<FAST>(make_float2(f[0].x, f[1].x)), b0 = dv.div2<FAST>(make_float2(f[2].x, f[3].x));
      const float2 a1 = dv.div2<FAST>(make_float2(f[0].y, f[1].y)), b1 = dv.div2<FAST>(make_float2(f[2].y, f[3].y));
      w0[q] = (uint32_t)e4m3x2(a0.x, a0.y) | ((uint32_t)e4m3x2(b0.x, b0.y) << 16);
      w1[q] = (uint32_t)e4m3x2(a1.x, a1.y) | ((uint32_t)e4m3x2(b1.x, b1.y) << 16);
    }
    *reinterpret_cast<uint4*>(out + (2 * p) * kOutRow + key0) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
    *reinterpret_cast<uint4*>(out + (2 * p + 1) * kOutRow + key0) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
  }
}

// One 128-key block of V: the head's scale from the block maxima, then codes written
// transposed ([d][128 keys] for the block) through shared memory.
template <typename T, int D>
__global__ void __launch_bounds__(kRows) v_quant_kernel(const T* __restrict__ v, const float* __restrict__ part,
                                                         uint8_t* __restrict__ v8t, float* __restrict__ scale,
                                                         int Nk, int H, int Npad, int* status) {
  using S = Stage<D>;
  constexpr int kOutRow = kRows + 16;  // bytes per transposed code row (+ padding)
  extern __shared__ __align__(16) uint8_t vq_smem[];  // the stage, then D transposed code rows
  uint8_t* st = vq_smem;
  uint8_t* out = vq_smem + S::kBytes;
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nb = gridDim.x;
  __shared__ float red[4];
  issue_rows<T, D>(v, st, Nk, H, b, h, j * kRows);
  cp_async_commit();
  // the head's amax over its block maxima, while the block's copies are in flight.  Launched as a
  // programmatic dependent of the kernel that wrote them: wait for that grid first (without the
  // launch attribute the wait returns at once)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  float amax = 0.f;
  const float* ph = part + ((long)b * H + h) * nb;
  for (int i = threadIdx.x; i < nb; i += kRows) amax = fmaxf(amax, ph[i]);
  amax = block_max(amax, red);
  cp_async_wait<0>();
  __syncthreads();
  const float s = scale_of(amax);
  if (j == 0 && threadIdx.x == 0 && FA_IN_BOUNDS(status, (long)b * H + h, (long)gridDim.z * H)) scale[(long)b * H + h] = s;
  const Divider dv = make_divider(s);
  if (dv.fast)
    encode_columns<T, D, true>(st, out, dv);
  else
    encode_columns<T, D, false>(st, out, dv);
  __syncthreads();
  // row c of the block: keys 128 j .. 128 j + 127, clipped to Npad (a multiple of 16); codes of
  // keys past Nk are zeros
  const int nkeys = min(kRows, Npad - j * kRows);
  uint8_t* base = v8t + ((long)b * H + h) * D * (long)Npad + (long)j * kRows;
  for (int e = threadIdx.x; e < D * (kRows / 16); e += kRows) {
    const int c = e / (kRows / 16), q = e % (kRows / 16);
    const long vi = (((long)b * H + h) * D + c) * (long)Npad + (long)j * kRows + 16 * q;
    if (16 * q < nkeys && FA_IN_BOUNDS(status, vi + 15, (long)gridDim.z * H * D * Npad))
      *reinterpret_cast<uint4*>(base + (long)c * Npad + 16 * q) = *reinterpret_cast<const uint4*>(out + c * kOutRow + 16 * q);
  }
}

template <int D>
struct VQuantSmem {
  static constexpr int kBytes = Stage<D>::kBytes + D * (kRows + 16);
};

template <typename T, int D>
cudaError_t launch_jobs(const QuantJobs& jobs, const float* signs, int B, cudaStream_t s) {
  long blocks = 0;
  for (int k = 0; k < jobs.n; ++k) blocks += (long)jobs.job[k].nblk * jobs.job[k].H * B;
  if (blocks < 1 || blocks > 0x7fffffffL) return cudaErrorInvalidValue;
  constexpr int smem = 2 * Stage<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(quant_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_kernel<T, D>, kRows, smem);
  if (e != cudaSuccess) return e;
  const long grid = std::min<long>(blocks, (long)std::max(per_sm, 1) * device_sm_count());
  quant_kernel<T, D><<<(unsigned)grid, kRows, smem, s>>>(jobs, signs, B, blocks);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_v_quant(const void* v, const float* part, void* v8t, float* scale, int B, int H, int Nk,
                           int* status, cudaStream_t s) {
  constexpr int smem = VQuantSmem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(v_quant_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // always launched right after the quant_kernel launch that writes `part`, on the same stream
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((Nk + kRows - 1) / kRows, H, B);
  cfg.blockDim = dim3(kRows);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr{};
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, v_quant_kernel<T, D>, static_cast<const T*>(v), part, static_cast<uint8_t*>(v8t),
                            scale, Nk, H, (Nk + 15) / 16 * 16, status);
}

template <int D>
cudaError_t jobs_d(const QuantJobs& jobs, const float* signs, int B, bool bf16, cudaStream_t s) {
  return bf16 ? launch_jobs<__nv_bfloat16, D>(jobs, signs, B, s) : launch_jobs<__half, D>(jobs, signs, B, s);
}
template <int D>
cudaError_t vq_d(const void* v, const float* part, void* v8t, float* scale, int B, int H, int Nk, bool bf16,
                 int* status, cudaStream_t s) {
  return bf16 ? launch_v_quant<__nv_bfloat16, D>(v, part, v8t, scale, B, H, Nk, status, s)
              : launch_v_quant<__half, D>(v, part, v8t, scale, B, H, Nk, status, s);
}

QuantJob rows_job(const void* x, void* x8, float* scales, int H, int N) {
  return QuantJob{x, static_cast<uint8_t*>(x8), scales, N, H, (N + kRows - 1) / kRows, kQuantRows};
}
QuantJob amax_job(const void* v, float* part, int H, int N) {
  return QuantJob{v, nullptr, part, N, H, (N + kRows - 1) / kRows, kQuantAmax};
}

}  // namespace

cudaError_t launch_fp8_quant_qk(const Fp8QuantArgs& a, cudaStream_t s) {
  QuantJobs jobs{};
  jobs.n = 1;
  jobs.status = a.status;
  jobs.job[0] = rows_job(a.x, a.x8, a.scales, a.H, a.N);
  return a.d == 128 ? jobs_d<128>(jobs, a.signs, a.B, a.bf16, s) : jobs_d<64>(jobs, a.signs, a.B, a.bf16, s);
}

cudaError_t launch_fp8_quant_v(const Fp8QuantArgs& a, cudaStream_t s) {
  QuantJobs jobs{};
  jobs.n = 1;
  jobs.status = a.status;
  jobs.job[0] = amax_job(a.x, a.work, a.H, a.N);
  cudaError_t e = a.d == 128 ? jobs_d<128>(jobs, nullptr, a.B, a.bf16, s) : jobs_d<64>(jobs, nullptr, a.B, a.bf16, s);
  if (e != cudaSuccess) return e;
  return a.d == 128 ? vq_d<128>(a.x, a.work, a.x8, a.scales, a.B, a.H, a.N, a.bf16, a.status, s)
                    : vq_d<64>(a.x, a.work, a.x8, a.scales, a.B, a.H, a.N, a.bf16, a.status, s);
}

cudaError_t launch_fp8_quant_qkv(const Fp8QkvArgs& a, cudaStream_t s) {
  QuantJobs jobs{};
  jobs.n = 3;
  jobs.status = a.status;
  jobs.job[0] = rows_job(a.q, a.q8, a.q_scale, a.Hq, a.Nq);
  jobs.job[1] = rows_job(a.k, a.k8, a.k_scale, a.Hkv, a.Nk);
  jobs.job[2] = amax_job(a.v, a.work, a.Hkv, a.Nk);
  cudaError_t e = a.d == 128 ? jobs_d<128>(jobs, a.signs, a.B, a.bf16, s) : jobs_d<64>(jobs, a.signs, a.B, a.bf16, s);
  if (e != cudaSuccess) return e;
  return a.d == 128 ? vq_d<128>(a.v, a.work, a.v8t, a.v_scale, a.B, a.Hkv, a.Nk, a.bf16, a.status, s)
                    : vq_d<64>(a.v, a.work, a.v8t, a.v_scale, a.B, a.Hkv, a.Nk, a.bf16, a.status, s);
}

}  // namespace fa
