// kernels.h -- host-side launchers of the attention kernels (internal to libfa.so).
// Arguments are validated by the C ABI in fa_api.cu before any launcher runs.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  int B, Hq, Hkv, Nq, Nk, d;
  int causal;
  float scale;
  int bf16;  // 1: bf16, 0: fp16
  int* status;
  const uint8_t* block_mask = nullptr;  // block-sparse forward: [B, Hq, ceil(Nq/128), ceil(Nk/128)]
  // dropout (drop_p > 0): keep threshold floor(p 2^16), 1 / (1 - p), Philox key and counter offset
  float drop_p = 0.f;
  uint32_t drop_thr = 0;
  float drop_inv_keep = 1.f;
  uint32_t seed_lo = 0, seed_hi = 0, drop_offset = 0;
  // merge into an fp32 accumulator (acc_o != nullptr): O [B,Nq,Hq,d] and LSE [B,Hq,Nq] fp32;
  // acc_mode 0: acc = this result; 1: acc = merge(acc, result); 2: o, lse = merge(acc, result)
  float* acc_o = nullptr;
  float* acc_lse = nullptr;
  int acc_mode = 0;
};

struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const void* dout;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  float* dvec;  // D [B,Hq,Nq] fp32 workspace
  int B, Hq, Hkv, Nq, Nk, d;
  int causal;
  float scale;
  int bf16;
  int* status;
  float drop_p = 0.f;
  uint32_t drop_thr = 0;
  float drop_inv_keep = 1.f;
  uint32_t seed_lo = 0, seed_hi = 0, drop_offset = 0;
  // add into fp32 accumulators instead of writing 16-bit gradients (acc_q / acc_k / acc_v !=
  // nullptr): dQ [B,Nq,Hq,d], dK and dV [B,Nk,Hkv,d]; acc_init: set instead of add
  float* acc_q = nullptr;
  float* acc_k = nullptr;
  float* acc_v = nullptr;
  int acc_init = 0;
  // the dQ launch directly follows this backward's dK/dV launch on the same stream: it may
  // start as a programmatic dependent (the two kernels share inputs, not outputs)
  int after_dkdv = 0;
};

struct DecodeArgs {
  const void* q;
  const void* k;
  const void* v;
  const int* seqlens;
  float* o_part;    // [B,Hq,S,d]
  float* lse_part;  // [B,Hq,S]
  int B, Hq, Hkv, Nk_max, d;
  int num_splits, chunk;
  float scale;
  int bf16;
  int* status;
};

struct CombineArgs {
  const float* o_part;
  const float* lse_part;
  const int* seqlens;
  void* o;
  float* lse;
  int B, Hq, d, num_splits;
  int bf16;
  int* status = nullptr;  // index checks of the FA_CHECKS build
};

// FP8 operand preparation (fp8_quant.cu).  Q/K: x [B,N,H,d] 16-bit -> x8 codes [B,N,H,d],
// scales [B,H,ceil(N/128)], optional rotation signs [d].  V: x [B,N,H,d] -> x8 codes
// [B,H,d,Npad] (Npad = N rounded up to 16), scales [B,H], work = per-block amax
// [B,H,ceil(N/128)] fp32.
struct Fp8QuantArgs {
  const void* x;
  void* x8;
  float* scales;
  const float* signs;
  float* work;
  int B, H, N, d;
  int bf16;
  int* status = nullptr;  // index checks of the FA_CHECKS build
};

// One quantization job of the fused launch: E4M3 codes and block scales of the rows of
// x [B, N, H, d] (kQuantRows), or the amax of every 128-row block of x into `scales`
// (kQuantAmax, the first pass over V).
constexpr int kQuantRows = 0, kQuantAmax = 1;
struct QuantJob {
  const void* x;
  uint8_t* x8;
  float* scales;
  int N, H, nblk, kind;
};
struct QuantJobs {
  QuantJob job[3];
  int n;
  int* status;  // index checks of the FA_CHECKS build
};
// Q, K and V of one forward pass quantized together (two launches).
struct Fp8QkvArgs {
  const void *q, *k, *v;
  void *q8, *k8, *v8t;
  float *q_scale, *k_scale, *v_scale;
  const float* signs;
  float* work;
  int B, Hq, Hkv, Nq, Nk, d;
  int bf16;
  int* status = nullptr;  // index checks of the FA_CHECKS build
};

// FP8 forward: E4M3 Q/K codes [B,N,H,d] with block scales, V codes transposed
// [B,Hkv,d,Nk_pad] with one scale per head; O in the 16-bit type `bf16` names.
struct Fp8AttnArgs {
  const void* q8;
  const float* q_scale;
  const void* k8;
  const float* k_scale;
  const void* v8t;
  const float* v_scale;
  void* o;
  float* lse;
  int B, Hq, Hkv, Nq, Nk, d;
  int causal;
  float scale;  // softmax scale of the original scores
  int rotated;  // Q and K were rotated: the scores are d times the original ones
  int bf16;
  int* status;
};

// Log-sum-exp merge of a partial attention result (merge.cu): o_acc fp32 [B,N,H,d], lse_acc
// [B,H,N]; o_part 16-bit [B,N,H,d], lse_part [B,H,N]; mode 0 acc = part, 1 acc = merge,
// 2 o_out (16-bit [B,N,H,d]) = merge and lse_acc updated.
struct MergeArgs {
  float* o_acc;
  float* lse_acc;
  const void* o_part;
  const float* lse_part;
  void* o_out;
  int B, N, H, d;
  int mode;
  int bf16;
};
cudaError_t launch_lse_merge(const MergeArgs& a, cudaStream_t s);
// acc fp32[n] = (init ? 0 : acc) + part 16-bit[n]; out 16-bit[n] = acc (n a multiple of 8).
cudaError_t launch_accumulate(float* acc, const void* part, long n, int init, int bf16, cudaStream_t s);
cudaError_t launch_cast(const float* acc, void* out, long n, int bf16, cudaStream_t s);

// TMA descriptors (tma.cu).  make_map: 4-D map over a BSHD tensor [B][N][H][D]
// (innermost d, then head, row, batch); box = 64 columns (128 bytes, 128-byte
// swizzle) x 1 head x `rows` rows x 1 batch.  Out-of-range rows read as zero.
bool tma_available();
// Streaming multiprocessors of the current device (148 if the query fails).
int device_sm_count();
bool make_map(CUtensorMap* m, const void* base, bool bf16, int D, int H, int N, int B, int rows);
// 4-D map over bytes: dims (innermost first), strides of dims 1..3 in bytes, box,
// 128-byte swizzle (the box's innermost extent must be 128 bytes).
bool make_map_u8(CUtensorMap* m, const void* base, const uint64_t dims[4], const uint64_t strides[3],
                 const uint32_t box[4]);

// Forward on tcgen05 / TMEM / TMA (warp-specialised), d = 128 and 64.
cudaError_t launch_fwd_sm100(const AttnArgs& a, cudaStream_t s);
bool fwd_sm100_supported(const AttnArgs& a);

// FP8 forward on tcgen05 kind::f8f6f4, d = 128 (fwd_sm100.cu).
cudaError_t launch_fwd_fp8_sm100(const Fp8AttnArgs& a, cudaStream_t s);
cudaError_t launch_fp8_quant_qk(const Fp8QuantArgs& a, cudaStream_t s);
cudaError_t launch_fp8_quant_v(const Fp8QuantArgs& a, cudaStream_t s);
cudaError_t launch_fp8_quant_qkv(const Fp8QkvArgs& a, cudaStream_t s);

cudaError_t launch_bwd_preprocess(const BwdArgs& a, cudaStream_t s);
// Backward dK/dV and dQ on tcgen05 / TMEM / TMA, d = 128 and 64.
cudaError_t launch_bwd_dkdv_sm100(const BwdArgs& a, cudaStream_t s);
cudaError_t launch_bwd_dq_sm100(const BwdArgs& a, cudaStream_t s);

cudaError_t launch_decode_split(const DecodeArgs& a, cudaStream_t s);
// One CTA waiting on a barrier nothing arrives on, limit in microseconds (watchdog.cu).
cudaError_t launch_watchdog_selftest(int* status, int limit_us, cudaStream_t s);
cudaError_t launch_decode_combine(const CombineArgs& a, cudaStream_t s);

}  // namespace fa
