// fa_api.cu -- the C ABI of libfa.so (declared in include/fa.h): argument
// validation, workspace sizing, the split heuristic and kernel dispatch.
// Validation happens before anything is launched; the library allocates no
// device memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>
#include <mutex>

#include "fa.h"
#include "kernels.h"

namespace {

// Device status word written by kernels whose bounded waits run out.  Host
// code reaches it only through the address that cudaGetSymbolAddress returns
// for the current device.
__device__ int g_fa_status = 0;

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {nullptr};
std::mutex g_status_mu;

int* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fa_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

fa_status check_shape(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, fa_dtype dt) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1) return FA_ERR_INVALID;
  if (Hq % Hkv != 0) return FA_ERR_INVALID;
  if (causal && Nq > Nk) return FA_ERR_INVALID;
  if (dt != FA_FP16 && dt != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || Hq > 65535) return FA_ERR_UNSUPPORTED;
  // every element index must fit the kernels' 64-bit offsets and the grid
  if ((long long)Nq > (1ll << 30) || (long long)Nk > (1ll << 30)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

fa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FA_OK : FA_ERR_CUDA; }

// Dropout parameters: keep iff the 16-bit Philox value >= floor(p 2^16), weights scaled by 1 / (1 - p).
struct DropParams {
  float p = 0.f;
  uint32_t thr = 0;
  float inv_keep = 1.f;
  uint32_t seed_lo = 0, seed_hi = 0, offset = 0;
};
bool make_drop(float p, unsigned long long seed, uint32_t offset, DropParams* out) {
  if (!(p >= 0.f && p < 1.f)) return false;
  const double t = std::floor((double)p * 65536.0);  // 16-bit keep threshold
  out->p = p;
  out->thr = (uint32_t)(t > 65535.0 ? 65535.0 : t);
  out->inv_keep = (float)(1.0 / (1.0 - (double)p));
  out->seed_lo = (uint32_t)(seed & 0xFFFFFFFFull);
  out->seed_hi = (uint32_t)(seed >> 32);
  out->offset = offset;
  return true;
}
template <typename A>
void apply_drop(A& a, const DropParams& d) {
  a.drop_p = d.p;
  a.drop_thr = d.thr;
  a.drop_inv_keep = d.inv_keep;
  a.seed_lo = d.seed_lo;
  a.seed_hi = d.seed_hi;
  a.drop_offset = d.offset;
}

}  // namespace

extern "C" {

int fa_version(void) { return 1; }

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration";
    case FA_ERR_ALIGN: return "pointer not aligned";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "kernel wait timed out";
    case FA_ERR_BOUNDS: return "device-side index check failed";
  }
  return "unknown status";
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                 int Nk, int d, int causal, float scale, fa_dtype dt, fa_stream_t stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID;
  fa_status st = check_shape(B, Hq, Hkv, Nq, Nk, d, causal, dt);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse)) return FA_ERR_ALIGN;
  fa::AttnArgs a{q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal ? 1 : 0, scale, dt == FA_BF16 ? 1 : 0, status_ptr()};
  if (!a.status) return FA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!fa::fwd_sm100_supported(a)) return FA_ERR_CUDA;  // the driver lacks the tensor-map encoder
  return from_cuda(fa::launch_fwd_sm100(a, s));
}

fa_status fa_fp8_quantize_qk(const void* x, void* x8, float* scales, const float* signs, int B, int H, int N, int d,
                             fa_dtype dt, fa_stream_t stream) {
  if (!x || !x8 || !scales) return FA_ERR_INVALID;
  fa_status st = check_shape(B, H, H, N, N, d, 0, dt);
  if (st != FA_OK) return st;
  if (!aligned16(x) || !aligned16(x8) || !aligned4(scales) || (signs && !aligned4(signs))) return FA_ERR_ALIGN;
  fa::Fp8QuantArgs a{x, x8, scales, signs, nullptr, B, H, N, d, dt == FA_BF16 ? 1 : 0, status_ptr()};
  return from_cuda(fa::launch_fp8_quant_qk(a, static_cast<cudaStream_t>(stream)));
}

size_t fa_fp8_v_workspace_bytes(int B, int Hkv, int Nk) {
  if (B < 1 || Hkv < 1 || Nk < 1) return 0;
  return (size_t)B * Hkv * ((Nk + 127) / 128) * sizeof(float);
}

fa_status fa_fp8_quantize_v(const void* v, void* v8t, float* scale, void* workspace, int B, int Hkv, int Nk, int d,
                            fa_dtype dt, fa_stream_t stream) {
  if (!v || !v8t || !scale || !workspace) return FA_ERR_INVALID;
  fa_status st = check_shape(B, Hkv, Hkv, Nk, Nk, d, 0, dt);
  if (st != FA_OK) return st;
  if (!aligned16(v) || !aligned16(v8t) || !aligned16(workspace) || !aligned4(scale)) return FA_ERR_ALIGN;
  fa::Fp8QuantArgs a{v, v8t, scale, nullptr, static_cast<float*>(workspace), B, Hkv, Nk, d, dt == FA_BF16 ? 1 : 0,
                     status_ptr()};
  return from_cuda(fa::launch_fp8_quant_v(a, static_cast<cudaStream_t>(stream)));
}

fa_status fa_fp8_quantize_qkv(const void* q, const void* k, const void* v, void* q8, void* k8, void* v8t,
                              float* q_scale, float* k_scale, float* v_scale, const float* signs, void* workspace,
                              int B, int Hq, int Hkv, int Nq, int Nk, int d, fa_dtype dt, fa_stream_t stream) {
  if (!q || !k || !v || !q8 || !k8 || !v8t || !q_scale || !k_scale || !v_scale || !workspace) return FA_ERR_INVALID;
  fa_status st = check_shape(B, Hq, Hkv, Nq, Nk, d, 0, dt);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q8) || !aligned16(k8) || !aligned16(v8t) ||
      !aligned16(workspace) || !aligned4(q_scale) || !aligned4(k_scale) || !aligned4(v_scale) ||
      (signs && !aligned4(signs)))
    return FA_ERR_ALIGN;
  fa::Fp8QkvArgs a{q, k, v, q8, k8, v8t, q_scale, k_scale, v_scale, signs, static_cast<float*>(workspace),
                   B, Hq, Hkv, Nq, Nk, d, dt == FA_BF16 ? 1 : 0, status_ptr()};
  return from_cuda(fa::launch_fp8_quant_qkv(a, static_cast<cudaStream_t>(stream)));
}

fa_status fa_fwd_fp8(const void* q8, const float* q_scale, const void* k8, const float* k_scale, const void* v8t,
                     const float* v_scale, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                     int causal, float scale, int rotated, fa_dtype out_dt, fa_stream_t stream) {
  if (!q8 || !q_scale || !k8 || !k_scale || !v8t || !v_scale || !o || !lse) return FA_ERR_INVALID;
  fa_status st = check_shape(B, Hq, Hkv, Nq, Nk, d, causal, out_dt);
  if (st != FA_OK) return st;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8t) || !aligned16(o) || !aligned4(lse) || !aligned4(q_scale) ||
      !aligned4(k_scale) || !aligned4(v_scale))
    return FA_ERR_ALIGN;
  if (!fa::tma_available()) return FA_ERR_CUDA;
  fa::Fp8AttnArgs a{q8,  q_scale, k8, k_scale, v8t, v_scale, o, lse, B, Hq, Hkv, Nq, Nk, d, causal ? 1 : 0, scale,
                    rotated ? 1 : 0, out_dt == FA_BF16 ? 1 : 0, status_ptr()};
  if (!a.status) return FA_ERR_CUDA;
  return from_cuda(fa::launch_fwd_fp8_sm100(a, static_cast<cudaStream_t>(stream)));
}

fa_status fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                         int Nq, int Nk, int d, int causal, float scale, float p_drop, unsigned long long seed,
                         uint32_t offset, fa_dtype dt, fa_stream_t stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID;
  DropParams dp;
  if (!make_drop(p_drop, seed, offset, &dp)) return FA_ERR_INVALID;
  fa_status st = check_shape(B, Hq, Hkv, Nq, Nk, d, causal, dt);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse)) return FA_ERR_ALIGN;
  fa::AttnArgs a{q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal ? 1 : 0, scale, dt == FA_BF16 ? 1 : 0, status_ptr()};
  apply_drop(a, dp);
  if (!a.status) return FA_ERR_CUDA;
  if (!fa::fwd_sm100_supported(a)) return FA_ERR_CUDA;
  return from_cuda(fa::launch_fwd_sm100(a, static_cast<cudaStream_t>(stream)));
}

fa_status fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                             const uint8_t* block_mask, int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                             float scale, fa_dtype dt, fa_stream_t stream) {
  if (!q || !k || !v || !o || !lse || !block_mask) return FA_ERR_INVALID;
  fa_status st = check_shape(B, Hq, Hkv, Nq, Nk, d, causal, dt);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse)) return FA_ERR_ALIGN;
  fa::AttnArgs a{q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal ? 1 : 0, scale, dt == FA_BF16 ? 1 : 0, status_ptr(),
                 block_mask};
  if (!a.status) return FA_ERR_CUDA;
  if (!fa::fwd_sm100_supported(a)) return FA_ERR_CUDA;
  return from_cuda(fa::launch_fwd_sm100(a, static_cast<cudaStream_t>(stream)));
}

fa_status fa_fwd_merge(const void* q, const void* k, const void* v, void* o, float* lse, float* acc_o,
                       float* acc_lse, int mode, int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                       float scale, fa_dtype dt, fa_stream_t stream) {
  if (!q || !k || !v || !o || !lse || !acc_o || !acc_lse) return FA_ERR_INVALID;
  if (mode < 0 || mode > 2) return FA_ERR_INVALID;
  fa_status st = check_shape(B, Hq, Hkv, Nq, Nk, d, causal, dt);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(acc_o) || !aligned4(lse) ||
      !aligned4(acc_lse))
    return FA_ERR_ALIGN;
  fa::AttnArgs a{q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal ? 1 : 0, scale, dt == FA_BF16 ? 1 : 0, status_ptr()};
  a.acc_o = acc_o;
  a.acc_lse = acc_lse;
  a.acc_mode = mode;
  if (!a.status) return FA_ERR_CUDA;
  if (!fa::fwd_sm100_supported(a)) return FA_ERR_CUDA;
  return from_cuda(fa::launch_fwd_sm100(a, static_cast<cudaStream_t>(stream)));
}

fa_status fa_lse_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                       int N, int H, int d, int mode, fa_dtype dt, fa_stream_t stream) {
  if (!o_acc || !lse_acc || !o_part || !lse_part || (mode == 2 && !o_out)) return FA_ERR_INVALID;
  if (mode < 0 || mode > 2 || B < 1 || N < 1 || H < 1) return FA_ERR_INVALID;
  if (dt != FA_FP16 && dt != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned16(o_acc) || !aligned16(o_part) || (o_out && !aligned16(o_out)) || !aligned4(lse_acc) ||
      !aligned4(lse_part))
    return FA_ERR_ALIGN;
  fa::MergeArgs a{o_acc, lse_acc, o_part, lse_part, o_out, B, N, H, d, mode, dt == FA_BF16 ? 1 : 0};
  return from_cuda(fa::launch_lse_merge(a, static_cast<cudaStream_t>(stream)));
}

fa_status fa_accumulate(float* acc, const void* part, long long n, int init, fa_dtype dt, fa_stream_t stream) {
  if (!acc || !part || n < 0 || (n & 7)) return FA_ERR_INVALID;
  if (dt != FA_FP16 && dt != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (!aligned16(acc) || !aligned16(part)) return FA_ERR_ALIGN;
  return from_cuda(fa::launch_accumulate(acc, part, (long)n, init ? 1 : 0, dt == FA_BF16 ? 1 : 0,
                                         static_cast<cudaStream_t>(stream)));
}

fa_status fa_cast_f32(const float* acc, void* out, long long n, fa_dtype dt, fa_stream_t stream) {
  if (!acc || !out || n < 0 || (n & 7)) return FA_ERR_INVALID;
  if (dt != FA_FP16 && dt != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (!aligned16(acc) || !aligned16(out)) return FA_ERR_ALIGN;
  return from_cuda(fa::launch_cast(acc, out, (long)n, dt == FA_BF16 ? 1 : 0, static_cast<cudaStream_t>(stream)));
}

size_t fa_bwd_workspace_bytes(int B, int Hq, int Nq) {
  if (B < 1 || Hq < 1 || Nq < 1) return 0;
  return (size_t)B * Hq * Nq * sizeof(float);
}

// step bits for bwd_run
enum { kPre = 1, kDkdv = 2, kDq = 4 };

static fa_status bwd_run(int steps, const void* q, const void* k, const void* v, const void* o, const void* dout,
                         const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int Hq, int Hkv,
                         int Nq, int Nk, int d, int causal, float scale, fa_dtype dt, fa_stream_t stream,
                         const DropParams& drop = DropParams{}) {
  const bool pre = steps & kPre, dkdv = steps & kDkdv, dqs = steps & kDq;
  if (!workspace || !dout) return FA_ERR_INVALID;
  if (pre && !o) return FA_ERR_INVALID;
  if ((dkdv || dqs) && (!q || !k || !v || !lse)) return FA_ERR_INVALID;
  if (dkdv && (!dk || !dv)) return FA_ERR_INVALID;
  if (dqs && !dq) return FA_ERR_INVALID;
  fa_status st = check_shape(B, Hq, Hkv, Nq, Nk, d, causal, dt);
  if (st != FA_OK) return st;
  const void* p16[] = {q, k, v, o, dout, dq, dk, dv, workspace};
  for (const void* p : p16)
    if (p && !aligned16(p)) return FA_ERR_ALIGN;
  if (lse && !aligned4(lse)) return FA_ERR_ALIGN;
  if ((dkdv || dqs) && !fa::tma_available()) return FA_ERR_CUDA;  // the driver lacks the tensor-map encoder
  fa::BwdArgs a{q, k, v, o, dout, lse, dq, dk, dv, static_cast<float*>(workspace), B, Hq, Hkv, Nq, Nk, d,
                causal ? 1 : 0, scale, dt == FA_BF16 ? 1 : 0, status_ptr()};
  apply_drop(a, drop);
  if (!a.status) return FA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (pre) e = fa::launch_bwd_preprocess(a, s);
  if (e == cudaSuccess && dkdv) e = fa::launch_bwd_dkdv_sm100(a, s);
  a.after_dkdv = dkdv ? 1 : 0;
  if (e == cudaSuccess && dqs) e = fa::launch_bwd_dq_sm100(a, s);
  return from_cuda(e);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                 void* dq, void* dk, void* dv, void* workspace, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                 int causal, float scale, fa_dtype dt, fa_stream_t stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID;
  return bwd_run(kPre | kDkdv | kDq, q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, causal,
                 scale, dt, stream);
}

fa_status fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const void* dout,
                         const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int Hq, int Hkv,
                         int Nq, int Nk, int d, int causal, float scale, float p_drop, unsigned long long seed,
                         uint32_t offset, fa_dtype dt, fa_stream_t stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID;
  DropParams dp;
  if (!make_drop(p_drop, seed, offset, &dp)) return FA_ERR_INVALID;
  return bwd_run(kPre | kDkdv | kDq, q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, causal,
                 scale, dt, stream, dp);
}

fa_status fa_bwd_preprocess(const void* q, const void* k, const void* v, const void* o, const void* dout,
                            const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int Hq, int Hkv,
                            int Nq, int Nk, int d, int causal, float scale, fa_dtype dt, fa_stream_t stream) {
  return bwd_run(kPre, q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, causal, scale, dt,
                 stream);
}

fa_status fa_bwd_dkdv(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                      void* dq, void* dk, void* dv, void* workspace, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                      int causal, float scale, fa_dtype dt, fa_stream_t stream) {
  return bwd_run(kDkdv, q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, causal, scale, dt,
                 stream);
}

fa_status fa_bwd_dq(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                    void* dq, void* dk, void* dv, void* workspace, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                    int causal, float scale, fa_dtype dt, fa_stream_t stream) {
  return bwd_run(kDq, q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, causal, scale, dt,
                 stream);
}

int fa_decode_chunk(int Nk_max, int num_splits) {
  if (Nk_max < 1 || num_splits < 1) return 64;
  int c = (Nk_max + num_splits - 1) / num_splits;
  return ((c + 63) / 64) * 64;
}

int fa_decode_num_splits(int B, int Hkv, int Nk_max, int d, int num_sms) {
  (void)d;
  if (B < 1 || Hkv < 1 || Nk_max < 1) return 1;
  if (num_sms <= 0) {
    int dev = 0;
    num_sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) {
      int n = 0;
      if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0) num_sms = n;
    }
  }
  const long long units = (long long)B * Hkv;
  const int max_splits = (Nk_max + 63) / 64;
  // Aim at ~26 (b, h_kv, split) units per SM (13 waves of the two CTAs an SM
  // holds) so that the ragged lengths of a batch even out, with splits of at
  // least 256 keys.  Measured on B200 for B=64, Hkv=8, Nk_max=32768: 8 splits
  // stream the cache at 6.95 TB/s, 3 splits at 6.57 TB/s, 32 at 6.02 TB/s.
  long long want = (26ll * num_sms + units - 1) / units;
  int splits = (int)(want < 1 ? 1 : want);
  const int min_keys = 256;
  const int cap = (Nk_max + min_keys - 1) / min_keys;
  if (splits > cap) splits = cap;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  // drop trailing splits that the 64-key rounding of the chunk left empty
  const int chunk = fa_decode_chunk(Nk_max, splits);
  return (Nk_max + chunk - 1) / chunk;
}

size_t fa_decode_workspace_bytes(int B, int Hq, int num_splits, int d) {
  if (B < 1 || Hq < 1 || num_splits < 1 || d < 1) return 0;
  const size_t o = (size_t)B * Hq * num_splits * d * sizeof(float);
  const size_t l = (size_t)B * Hq * num_splits * sizeof(float);
  return o + ((l + 255) / 256) * 256;
}

static fa_status decode_check(int B, int Hq, int Hkv, int Nk_max, int d, int num_splits, fa_dtype dt) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Nk_max < 1 || num_splits < 1) return FA_ERR_INVALID;
  if (Hq % Hkv != 0) return FA_ERR_INVALID;
  if (dt != FA_FP16 && dt != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (Hq / Hkv > 16) return FA_ERR_UNSUPPORTED;  // one CTA holds a GQA group of at most 16 query heads
  if (B > 65535 || Hkv > 65535 || Hq > 65535 || num_splits > 65535) return FA_ERR_UNSUPPORTED;
  if (num_splits > (Nk_max + 63) / 64) return FA_ERR_INVALID;
  return FA_OK;
}

fa_status fa_decode_splitkv(const void* q, const void* k_cache, const void* v_cache, const int* seqlens_k, int B,
                            int Hq, int Hkv, int Nk_max, int d, float scale, int num_splits, void* workspace,
                            fa_dtype dt, fa_stream_t stream) {
  if (!q || !k_cache || !v_cache || !seqlens_k || !workspace) return FA_ERR_INVALID;
  fa_status st = decode_check(B, Hq, Hkv, Nk_max, d, num_splits, dt);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(workspace) || !aligned4(seqlens_k))
    return FA_ERR_ALIGN;
  float* o_part = static_cast<float*>(workspace);
  float* lse_part = o_part + (size_t)B * Hq * num_splits * d;
  fa::DecodeArgs a{q,     k_cache, v_cache,    seqlens_k, o_part, lse_part, B, Hq, Hkv, Nk_max, d, num_splits,
                   fa_decode_chunk(Nk_max, num_splits), scale, dt == FA_BF16 ? 1 : 0, status_ptr()};
  if (!a.status) return FA_ERR_CUDA;
  return from_cuda(fa::launch_decode_split(a, static_cast<cudaStream_t>(stream)));
}

fa_status fa_decode_combine(const void* workspace, void* o, float* lse, const int* seqlens_k, int B, int Hq,
                            int num_splits, int d, fa_dtype dt, fa_stream_t stream) {
  if (!workspace || !o || !lse || !seqlens_k) return FA_ERR_INVALID;
  if (B < 1 || Hq < 1 || num_splits < 1) return FA_ERR_INVALID;
  if (dt != FA_FP16 && dt != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || Hq > 65535) return FA_ERR_UNSUPPORTED;
  if (!aligned16(workspace) || !aligned16(o) || !aligned4(lse) || !aligned4(seqlens_k)) return FA_ERR_ALIGN;
  const float* o_part = static_cast<const float*>(workspace);
  const float* lse_part = o_part + (size_t)B * Hq * num_splits * d;
  fa::CombineArgs a{o_part, lse_part, seqlens_k, o, lse, B, Hq, d, num_splits, dt == FA_BF16 ? 1 : 0, status_ptr()};
  return from_cuda(fa::launch_decode_combine(a, static_cast<cudaStream_t>(stream)));
}

fa_status fa_watchdog_selftest(int limit_us, fa_stream_t stream) {
  if (limit_us < 1 || limit_us > 2000000) return FA_ERR_INVALID;
  int* st = status_ptr();
  if (!st) return FA_ERR_CUDA;
  return from_cuda(fa::launch_watchdog_selftest(st, limit_us, static_cast<cudaStream_t>(stream)));
}

fa_status fa_get_device_status(fa_stream_t stream) {
  int* p = status_ptr();
  if (!p) return FA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return FA_ERR_CUDA;
  }
  return static_cast<fa_status>(v);
}

}  // extern "C"

fa_status fa_bwd_accumulate(const void* q, const void* k, const void* v, const void* dout, const float* lse,
                            const void* workspace, float* dq_acc, float* dk_acc, float* dv_acc, int init, int B,
                            int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale, fa_dtype dt,
                            fa_stream_t stream) {
  if (!q || !k || !v || !dout || !lse || !workspace || !dq_acc || !dk_acc || !dv_acc) return FA_ERR_INVALID;
  if (init < 0 || init > 3) return FA_ERR_INVALID;
  fa_status st = check_shape(B, Hq, Hkv, Nq, Nk, d, causal, dt);
  if (st != FA_OK) return st;
  const void* p16[] = {q, k, v, dout, workspace, dq_acc, dk_acc, dv_acc};
  for (const void* p : p16)
    if (!aligned16(p)) return FA_ERR_ALIGN;
  if (!aligned4(lse)) return FA_ERR_ALIGN;
  if (!fa::tma_available()) return FA_ERR_CUDA;
  fa::BwdArgs a{q, k, v, nullptr, dout, lse, nullptr, nullptr, nullptr, static_cast<float*>(const_cast<void*>(workspace)),
                B, Hq, Hkv, Nq, Nk, d, causal ? 1 : 0, scale, dt == FA_BF16 ? 1 : 0, status_ptr()};
  if (!a.status) return FA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  fa::BwdArgs kv = a;
  kv.acc_k = dk_acc;
  kv.acc_v = dv_acc;
  kv.acc_init = (init & 2) ? 1 : 0;
  cudaError_t e = fa::launch_bwd_dkdv_sm100(kv, s);
  if (e != cudaSuccess) return from_cuda(e);
  fa::BwdArgs qa = a;
  qa.acc_q = dq_acc;
  qa.acc_init = (init & 1) ? 1 : 0;
  qa.after_dkdv = 1;
  return from_cuda(fa::launch_bwd_dq_sm100(qa, s));
}
