// decode_noalloc.cu -- split-KV decode for callers that cannot allocate device
// memory.
//
// Who needs it: a serving runtime that plans all of its device memory up front
// and forbids allocation on the request path (cudaMalloc can synchronise the
// device and fragments a pre-planned pool), code that runs inside another
// library's allocator or memory callback (allocating there would re-enter that
// allocator), and latency-bound callers for which the first-touch cost of a
// fresh allocation is not acceptable.  Such callers can still pass their own
// inputs and outputs, but not a workspace for the split partials.
//
// This entry point runs the same partial and combine kernels as
// fa_decode_splitkv + fa_decode_combine, with the partials placed in a static
// device array that is part of this library's module image.  Every GPU that
// loads libfa.so holds that array from load until process exit.  The array's
// name is, in host code, only a host-side stand-in for the symbol: handing it
// to a kernel would fault (or silently use host memory where the GPU can reach
// it), so the device address is looked up with cudaGetSymbolAddress, once per
// device, with that device current, and that address is what the kernels get.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "fa.h"
#include "kernels.h"

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[FA_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device (looked up on the
// first call on each device; later calls reuse it).
fa_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return FA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return FA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Bytes of partials for S splits: O_s fp32 [B,Hq,S,d], then LSE_s fp32 [B,Hq,S] at a 256-byte boundary.
size_t partial_bytes(int B, int Hq, int S, int d, size_t* lse_offset) {
  const size_t o = (size_t)B * Hq * S * d * sizeof(float);
  const size_t off = (o + 255) / 256 * 256;
  if (lse_offset) *lse_offset = off;
  return off + (size_t)B * Hq * S * sizeof(float);
}

}  // namespace

extern "C" fa_status fa_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, const int* seqlens_k,
                                       void* o, float* lse, int B, int Hq, int Hkv, int Nk_max, int d, float scale,
                                       int num_splits, fa_dtype dt, fa_stream_t stream) {
  if (!q || !k_cache || !v_cache || !seqlens_k || !o || !lse) return FA_ERR_INVALID;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nk_max < 1 || Hq % Hkv != 0) return FA_ERR_INVALID;
  if (dt != FA_FP16 && dt != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (Hq / Hkv > 16) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || Hq > 65535 || Hkv > 65535) return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(seqlens_k, 4))
    return FA_ERR_ALIGN;
  const int max_splits = (Nk_max + 63) / 64;
  int S = num_splits;
  if (S <= 0) {
    // the library's suggestion, reduced until the partials fit the scratch array
    S = fa_decode_num_splits(B, Hkv, Nk_max, d, 0);
    while (S > 1 && partial_bytes(B, Hq, S, d, nullptr) > FA_DECODE_NOALLOC_SCRATCH_BYTES) --S;
  }
  if (S > max_splits || S > 65535) return FA_ERR_INVALID;
  size_t lse_off = 0;
  if (partial_bytes(B, Hq, S, d, &lse_off) > FA_DECODE_NOALLOC_SCRATCH_BYTES) return FA_ERR_UNSUPPORTED;

  void* scratch = nullptr;
  const fa_status st = scratch_address(&scratch);
  if (st != FA_OK) return st;
  float* o_part = static_cast<float*>(scratch);
  float* lse_part = reinterpret_cast<float*>(static_cast<unsigned char*>(scratch) + lse_off);
  const int bf16 = dt == FA_BF16 ? 1 : 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Every (b, h, split) entry the combine reads is written by the partial pass of
  // this same call (an empty split writes O_s = 0, LSE_s = -inf), so nothing left
  // in the array by an earlier call is ever read and nothing needs clearing.
  fa::DecodeArgs da{q, k_cache, v_cache, seqlens_k, o_part, lse_part, B, Hq, Hkv, Nk_max, d, S,
                    fa_decode_chunk(Nk_max, S), scale, bf16, nullptr};
  cudaError_t e = fa::launch_decode_split(da, s);
  if (e != cudaSuccess) return FA_ERR_CUDA;
  fa::CombineArgs ca{o_part, lse_part, seqlens_k, o, lse, B, Hq, d, S, bf16};
  e = fa::launch_decode_combine(ca, s);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
