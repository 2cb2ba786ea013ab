// common.cuh -- device helpers shared by the attention kernels (sm_100a).
//
// Shared-memory tile layout used by every kernel: a tile of R rows x D
// 16-bit columns is stored as D/64 column panels of [R][64] elements; each
// row of a panel is 128 bytes, and its eight 16-byte chunks are permuted by
// chunk' = chunk ^ (row & 7).  This is the 128-byte swizzle that the Tensor
// Memory Accelerator writes (CU_TENSOR_MAP_SWIZZLE_128B) and that tcgen05
// shared-memory descriptors read (layout type SWIZZLE_128B), so the same
// tiles serve ldmatrix, cp.async, TMA and tcgen05 without bank conflicts.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Device status word codes (mirrors fa_status in fa.h).
constexpr int kStatusTimeout = -5;
constexpr int kStatusBounds = -6;

// Index checks of the FA_CHECKS build (libfa_checks.so): FA_IN_BOUNDS(status, i, n) is true
// when 0 <= i < n; otherwise it records kStatusBounds in the status word (no trap) and the
// caller skips the access.  In the normal build it is the constant true and costs nothing.
__device__ __forceinline__ bool in_bounds_or_flag(int* status, long long i, long long n) {
  if (i >= 0 && i < n) return true;
  if (status) atomicCAS(status, 0, kStatusBounds);
  return false;
}
#ifdef FA_CHECKS
#define FA_IN_BOUNDS(status, i, n) ::fa::in_bounds_or_flag((status), (long long)(i), (long long)(n))
#else
#define FA_IN_BOUNDS(status, i, n) ((void)(status), (void)(i), (void)(n), true)
#endif

// Philox4x32 with 10 rounds (Salmon, Moraes, Dror, Shaw, "Parallel random
// numbers: as easy as 1, 2, 3", SC 2011): per round, with M0 = 0xD2511F53 and
// M1 = 0xCD9E8D57, (c0, c1, c2, c3) -> (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2),
// hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)); the key is bumped by the Weyl constants
// (0x9E3779B9, 0xBB67AE85) before every round but the first.  Used for the
// dropout mask, which the backward kernels regenerate from the same counters.
__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                                               uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = c0 * 0xD2511F53u, hi0 = __umulhi(c0, 0xD2511F53u);
    const uint32_t lo1 = c2 * 0xCD9E8D57u, hi1 = __umulhi(c2, 0xCD9E8D57u);
    c0 = hi1 ^ c1 ^ k0;
    c1 = lo1;
    c2 = hi0 ^ c3 ^ k1;
    c3 = lo0;
  }
  return make_uint4(c0, c1, c2, c3);
}

// Dropout of one (b, h_q): one Philox call per 2 x 4 block of (query i, key j),
// counter (j >> 2, i >> 1, b * Hq + h, offset), key = the 64-bit seed.  The
// call's four words are eight 16-bit values (low half first); value
// e = 4 (i & 1) + (j & 3), the half e & 1 of word e >> 1, decides (i, j): kept
// iff it is >= thr = floor(p 2^16).
struct Dropout {
  uint32_t thr;       // floor(p * 2^16)
  float inv_keep;     // 1 / (1 - p)
  uint32_t seed_lo, seed_hi, offset;
};

// Keep bits of one row of a 2 x 4 block from the row's two words (a: keys 0-1, b: keys 2-3):
// bit k = key k of the quad.
__device__ __forceinline__ uint32_t keep_quad(uint32_t a, uint32_t b, uint32_t thr) {
  return (uint32_t)((a & 0xFFFFu) >= thr) | ((uint32_t)((a >> 16) >= thr) << 1) |
         ((uint32_t)((b & 0xFFFFu) >= thr) << 2) | ((uint32_t)((b >> 16) >= thr) << 3);
}
// Keep bits of one key of a 2 x 4 block for both rows, from the key's value in the even-row word
// (ve) and the odd-row word (vo): bit 0 = even row, bit 1 = odd row.
__device__ __forceinline__ uint32_t keep_pair(uint32_t ve, uint32_t vo, uint32_t thr) {
  return (uint32_t)(ve >= thr) | ((uint32_t)(vo >= thr) << 1);
}

// ---------------------------------------------------------------------------
// element types
// ---------------------------------------------------------------------------
template <typename T>
struct Elem;

template <>
struct Elem<__nv_bfloat16> {
  static constexpr bool kBf16 = true;
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __device__ __forceinline__ static float2 unpack(uint32_t u) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(v);
  }
};

template <>
struct Elem<__half> {
  static constexpr bool kBf16 = false;
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __device__ __forceinline__ static float2 unpack(uint32_t u) {
    __half2 v = *reinterpret_cast<__half2*>(&u);
    return __half22float2(v);
  }
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// D += A * B for one m16n8k16 tile, fp32 accumulate.
template <typename T>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (Elem<T>::kBf16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// 16-byte global->shared copy; zero-fills the destination when !valid.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// ---------------------------------------------------------------------------
// swizzled tile addressing (see the layout note at the top of this file)
// ---------------------------------------------------------------------------
// Byte offset of element (r, col) in an R-row tile; col is a multiple of 8.
template <int R>
__device__ __forceinline__ uint32_t swz(int r, int col) {
  return static_cast<uint32_t>((col >> 6) * (R * 128) + r * 128 + ((((col >> 3) & 7) ^ (r & 7)) << 4));
}

// Copy a [R][D] tile of 16-bit elements from global rows row0.. (row stride
// `ld` elements) into a swizzled shared tile with cp.async.  Rows at or past
// `nrows` are zero-filled.  All NT threads of the block take part.
template <int R, int D, int NT>
__device__ __forceinline__ void load_tile_async(uint32_t smem, const uint16_t* g, int row0, int nrows, long ld,
                                                int tid) {
  constexpr int kChunks = R * D / 8;
#pragma unroll
  for (int c = tid; c < kChunks; c += NT) {
    const int r = c / (D / 8);
    const int col = (c % (D / 8)) * 8;
    const int gr = row0 + r;
    const bool ok = gr < nrows;
    const uint16_t* src = g + (ok ? (long)gr * ld + col : 0);
    cp_async16(smem + swz<R>(r, col), src, ok);
  }
}

// A-operand fragment (16 rows x 16 k) of a row-major swizzled tile at
// rows r0.., columns k0.. .
template <int R>
__device__ __forceinline__ void frag_a(uint32_t (&a)[4], uint32_t tile, int r0, int k0, int lane) {
  ldsm_x4(tile + swz<R>(r0 + (lane & 15), k0 + ((lane >> 4) << 3)), a[0], a[1], a[2], a[3]);
}

// B-operand fragments for two n8 blocks (n0.., n0+8..) x k16 (k0..) from a
// tile stored [n][k] (k contiguous): b[0],b[1] for block n0, b[2],b[3] for n0+8.
template <int R>
__device__ __forceinline__ void frag_b_nk(uint32_t (&b)[4], uint32_t tile, int n0, int k0, int lane) {
  ldsm_x4(tile + swz<R>(n0 + (lane & 7) + ((lane >> 4) << 3), k0 + (((lane >> 3) & 1) << 3)), b[0], b[1], b[2],
          b[3]);
}

// B-operand fragments for two n8 blocks x k16 from a tile stored [k][n]
// (n contiguous), via the transposing ldmatrix.
template <int R>
__device__ __forceinline__ void frag_b_kn(uint32_t (&b)[4], uint32_t tile, int k0, int n0, int lane) {
  ldsm_x4_t(tile + swz<R>(k0 + (lane & 7) + (((lane >> 3) & 1) << 3), n0 + ((lane >> 4) << 3)), b[0], b[1], b[2],
            b[3]);
}

__device__ __forceinline__ float quad_max(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
  return x;
}
__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

}  // namespace fa
