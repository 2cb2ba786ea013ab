/*
 * fa.h -- C ABI of libfa.so: exact IO-aware scaled-dot-product attention on
 * one NVIDIA B200 (sm_100a).
 *
 * What is computed.  O = softmax(scale * Q K^T + causal mask) V, the plain
 * definition of attention ("FlashAttention 심층 분석", section 1), evaluated
 * tile by tile with the online softmax of section 3 of the same page (running
 * max m, running sum l, rescaling of O) so that the N x N score matrix never
 * reaches HBM.  The forward pass keeps one fp32 log-sum-exp per query row
 * (smithlab guide to FlashAttention versions and training cost, memory table) and the
 * backward pass recomputes P from it (same analysis page, section 4).  One-token
 * decode splits the key axis and merges the splits by log-sum-exp (analysis
 * page, "Flash-Decoding").  GQA is expressed by the KV-head count, with no K/V
 * copies, and causal masking is a flag (smithlab guide, adoption checklist).
 *
 * Conventions shared by every entry point:
 *  - Layout "BSHD", contiguous, d innermost:
 *      q, o, dout, dq : [B, Nq, Hq, d]      k, v, dk, dv : [B, Nk, Hkv, d]
 *      lse, D         : [B, Hq, Nq] fp32    decode caches : [B, Nk_max, Hkv, d]
 *  - Element type of q/k/v/o/dout/dq/dk/dv: fa_dtype (IEEE fp16 or bf16).
 *  - LSE is the natural-log log-sum-exp of the scaled, masked scores of a row.
 *  - Causal keeps key j for query i iff j <= i + (Nk - Nq) (bottom-right
 *    alignment; the lower triangle when Nq == Nk).  causal requires Nq <= Nk.
 *  - GQA: Hq % Hkv == 0; query head h reads KV head h / (Hq / Hkv).
 *  - d must be 64 or 128 (FA_ERR_UNSUPPORTED otherwise).  Nq, Nk >= 1, any
 *    value (ragged tails are masked inside the kernels).
 *  - Every pointer is a DEVICE pointer; tensors and workspaces 16-byte
 *    aligned, lse and seqlens_k 4-byte aligned (FA_ERR_ALIGN otherwise).  The
 *    caller owns and allocates every buffer, workspaces included; the library
 *    allocates no device memory and keeps no per-call state (fa_decode_noalloc
 *    uses a fixed static array inside the library instead of a workspace).
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  The return value reports argument validation (checked
 *    before anything is launched) and launch errors only.  Errors raised by a
 *    running kernel (a bounded wait that ran out, see fa_get_device_status)
 *    are recorded in a device status word.
 *  - Outputs are overwritten, never accumulated into.  Results are
 *    deterministic: two calls on the same inputs give bitwise-equal outputs.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID = -1,     /* null pointer, bad size, Hq % Hkv != 0, causal with Nq > Nk */
  FA_ERR_UNSUPPORTED = -2, /* d not in {64, 128}, unknown dtype, size beyond a stated limit */
  FA_ERR_ALIGN = -3,       /* a pointer is not 16-byte aligned */
  FA_ERR_CUDA = -4,        /* a CUDA runtime/driver call or a launch failed */
  FA_ERR_TIMEOUT = -5,     /* a kernel's bounded wait ran out (device status word) */
  FA_ERR_BOUNDS = -6       /* a device-side index check failed (libfa_checks.so only; device status word) */
} fa_status;

typedef enum { FA_FP16 = 0, FA_BF16 = 1 } fa_dtype;

/* A cudaStream_t passed as an opaque pointer (keeps this header free of CUDA includes). */
typedef void* fa_stream_t;

/*
 * Forward pass.  Writes o [B,Nq,Hq,d] (dtype dt) and lse [B,Hq,Nq] (fp32).
 * Source: "FlashAttention 심층 분석", sections 1 and 3 (definition; tiling and
 * online softmax fused into one kernel: scale, mask, softmax, PV).
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                 fa_dtype dt, fa_stream_t stream);

/* Bytes of workspace fa_bwd needs: the fp32 row term D [B,Hq,Nq]. */
size_t fa_bwd_workspace_bytes(int B, int Hq, int Nq);

/*
 * Backward pass.  Given q, k, v, the forward output o, the upstream gradient
 * dout and the forward lse, writes dq, dk, dv (dtype dt), each overwritten.
 * P is recomputed from lse ("FlashAttention 심층 분석", section 4); the
 * gradients are the chain rule of the definition:
 *   D_i = sum_c dO_ic O_ic,  dS = P * (dO V^T - D),
 *   dV = P^T dO,  dQ = scale dS K,  dK = scale dS^T Q,
 * with dK, dV of a KV head summed over its Hq/Hkv query heads.  `workspace`
 * must hold fa_bwd_workspace_bytes(B, Hq, Nq) bytes (device, 16-byte aligned).
 * No atomics: dK/dV and dQ come from separate kernels, so the result is
 * bitwise reproducible (the deterministic mode of the smithlab guide's
 * recommendation table).  The dQ kernel is launched as a programmatic
 * dependent of the dK/dV kernel and may start on SMs that dK/dV has released;
 * the call still behaves as one stream operation: work enqueued after it on
 * `stream` starts only after every gradient is written.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, void* workspace,
                 int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                 fa_dtype dt, fa_stream_t stream);

/*
 * The three launches fa_bwd makes, callable one by one (same arguments, same
 * validation), so that a caller can time or schedule them separately:
 *   fa_bwd_preprocess: workspace D[b,h,i] = sum_c dout[b,i,h,c] * o[b,i,h,c] (fp32);
 *   fa_bwd_dkdv: dk, dv from q, k, v, dout, lse and D (one CTA per 128-key tile
 *     of a KV head, looping over its group's query heads and query tiles);
 *   fa_bwd_dq: dq from q, k, v, dout, lse and D (one CTA per 128-row query tile).
 * fa_bwd_dkdv and fa_bwd_dq read the D that fa_bwd_preprocess wrote, so on one
 * stream the preprocess call must come first.  Arguments a step does not read
 * may be NULL (preprocess: q, k, v, lse, dq, dk, dv; dkdv: o, dq; dq: o, dk, dv).
 */
fa_status fa_bwd_preprocess(const void* q, const void* k, const void* v, const void* o, const void* dout,
                            const float* lse, void* dq, void* dk, void* dv, void* workspace,
                            int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                            fa_dtype dt, fa_stream_t stream);
fa_status fa_bwd_dkdv(const void* q, const void* k, const void* v, const void* o, const void* dout,
                      const float* lse, void* dq, void* dk, void* dv, void* workspace,
                      int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                      fa_dtype dt, fa_stream_t stream);
fa_status fa_bwd_dq(const void* q, const void* k, const void* v, const void* o, const void* dout,
                    const float* lse, void* dq, void* dk, void* dv, void* workspace,
                    int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                    fa_dtype dt, fa_stream_t stream);

/*
 * Suggested number of key splits for fa_decode_splitkv: about 26 (b, h_kv, split)
 * units per SM so that ragged sequence lengths even out (num_sms <= 0: query
 * the current device), splits of at least 256 keys.  Always >= 1 and
 * <= ceil(Nk_max / 64).
 */
int fa_decode_num_splits(int B, int Hkv, int Nk_max, int d, int num_sms);

/* Bytes of the split partials: O_s fp32 [B,Hq,num_splits,d] + LSE_s fp32 [B,Hq,num_splits]. */
size_t fa_decode_workspace_bytes(int B, int Hq, int num_splits, int d);

/*
 * Split-KV decode, partial pass ("FlashAttention 심층 분석", Flash-Decoding).
 * q [B,1,Hq,d]; k_cache, v_cache [B,Nk_max,Hkv,d]; seqlens_k: DEVICE int32 [B],
 * 0 <= seqlens_k[b] <= Nk_max (values outside are clamped into that range).
 * Split s of sequence b covers keys [s*C, min((s+1)*C, seqlens_k[b])) with
 * C = fa_decode_chunk(Nk_max, num_splits); each split writes its normalised
 * partial output O_s and LSE_s into `workspace` (an empty split writes O_s = 0,
 * LSE_s = -inf).  Non-causal: the query is the newest token.
 */
fa_status fa_decode_splitkv(const void* q, const void* k_cache, const void* v_cache,
                            const int* seqlens_k, int B, int Hq, int Hkv, int Nk_max, int d,
                            float scale, int num_splits, void* workspace, fa_dtype dt,
                            fa_stream_t stream);

/*
 * Split-KV decode, combine pass: LSE = ln sum_s exp(LSE_s) and
 * O = sum_s exp(LSE_s - LSE) O_s, cast to dt.  o [B,1,Hq,d]; lse [B,Hq,1] fp32.
 * A sequence with seqlens_k[b] == 0 gets O = 0 and LSE = -inf.
 */
fa_status fa_decode_combine(const void* workspace, void* o, float* lse, const int* seqlens_k,
                            int B, int Hq, int num_splits, int d, fa_dtype dt,
                            fa_stream_t stream);

/* Keys per split used by fa_decode_splitkv: ceil(Nk_max / num_splits) rounded up to 64. */
int fa_decode_chunk(int Nk_max, int num_splits);

/*
 * Split-KV decode that allocates nothing and takes no workspace.  The pages
 * have no counterpart: this exists for callers that cannot allocate device
 * memory -- a serving runtime that plans all device memory up front and
 * forbids allocation on the request path, code running inside another
 * library's allocator callback (allocating would re-enter it), or a
 * latency-bound caller that cannot pay for a fresh allocation.
 *
 * Same inputs, outputs and result as fa_decode_splitkv followed by
 * fa_decode_combine (q [B,1,Hq,d], caches [B,Nk_max,Hkv,d], seqlens_k device
 * int32 [B], o [B,1,Hq,d], lse [B,Hq,1] fp32), computed by the same kernels;
 * the split partials live in a static device array of
 * FA_DECODE_NOALLOC_SCRATCH_BYTES bytes inside libfa.so, which every GPU that
 * loads the library holds until the process exits.
 *  - Size limit: the partials take B*Hq*S*d*4 bytes, rounded up to 256, plus
 *    B*Hq*S*4 bytes for S splits; a request beyond the array returns
 *    FA_ERR_UNSUPPORTED before anything is launched.  num_splits <= 0 takes the
 *    fa_decode_num_splits suggestion, reduced until the partials fit.
 *  - First call on a device: looks up the array's device address with
 *    cudaGetSymbolAddress (with that device current) and keeps it; make that
 *    first call before any stream capture on the device.
 *  - Every call on a device shares the one array, which keeps the last call's
 *    contents.  Calls whose kernels overlap on the GPU (two streams, or two host
 *    threads without ordering) race on it; issue them on one stream.  Nothing
 *    needs to start at zero: every partial the combine reads is written first
 *    by the same call.
 * Calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define FA_DECODE_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
fa_status fa_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, const int* seqlens_k,
                            void* o, float* lse, int B, int Hq, int Hkv, int Nk_max, int d, float scale,
                            int num_splits, fa_dtype dt, fa_stream_t stream);

/*
 * Dropout ("FlashAttention 심층 분석", section 2: dropout is one of the fused steps;
 * section 4: the backward pass regenerates what it needs).  The mask comes from
 * Philox4x32-10 (Salmon et al., SC 2011): one call per 2 x 4 block of (query i,
 * key j) of head (b, h), counter (j >> 2, i >> 1, b * Hq + h, offset), key =
 * (seed & 0xffffffff, seed >> 32); the call's four words are read as eight
 * 16-bit values (low half of a word first), element (i, j) takes value
 * 4 (i & 1) + (j & 3) and is kept iff that value >= floor(p_drop * 2^16)
 * (p_drop as passed, in [0, 1); FA_ERR_INVALID otherwise).  The forward computes
 * O = (P * M / (1 - p_drop)) V and the LSE of the undropped scores; the
 * backward (same seed, offset and p_drop) regenerates M and returns the
 * gradients of sum(dO * O) for that forward.  p_drop = 0 gives fa_fwd /
 * fa_bwd.  Otherwise as fa_fwd / fa_bwd (layouts, GQA, alignment, workspace).
 */
fa_status fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                         int Nq, int Nk, int d, int causal, float scale, float p_drop, unsigned long long seed,
                         uint32_t offset, fa_dtype dt, fa_stream_t stream);
fa_status fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const void* dout,
                         const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int Hq, int Hkv,
                         int Nq, int Nk, int d, int causal, float scale, float p_drop, unsigned long long seed,
                         uint32_t offset, fa_dtype dt, fa_stream_t stream);

/*
 * Block-sparse forward ("FlashAttention-2 (KO)", FA-1 results: the IO-aware
 * kernel extended with a block-sparse pattern).  block_mask: device uint8
 * [B, Hq, ceil(Nq / 128), ceil(Nk / 128)]; entry (b, h, I, J) nonzero means
 * queries 128 I .. 128 I + 127 may attend to keys 128 J .. 128 J + 127
 * (intersected with the causal rule when causal).  Blocks not marked are
 * skipped; a row with no visible key gets O = 0 and LSE = -inf.  Otherwise as
 * fa_fwd (layouts, GQA, alignment, errors).
 */
fa_status fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                             const uint8_t* block_mask, int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                             float scale, fa_dtype dt, fa_stream_t stream);

/* ------------------------------------------------------------------------------
 * FP8 forward pass ("FlashAttention-2 (KO)", FA-3 paragraph: low-precision FP8
 * with incoherent processing; smithlab guide, version table: FP8 is forward
 * only).  The pages give no formats; the library fixes them:
 *  - codes are E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
 *    largest finite 448), converted with round-to-nearest-even and saturation;
 *  - Q and K: one fp32 scale per (batch, head, 128-row block), s = amax / 448
 *    (1 for an all-zero block), code = E4M3(y / s) with a correctly rounded
 *    fp32 division;
 *  - incoherent processing (optional): before quantization the rows of Q and
 *    K are multiplied by `signs` (d values, each +1 or -1) and then by the
 *    unnormalised d x d Walsh-Hadamard matrix, in fp32 with the butterflies
 *    (a, b) -> (a + b, a - b) taken for h = 1, 2, 4, ..., d / 2; the scores
 *    become d times the original ones, which fa_fwd_fp8 undoes when `rotated`;
 *  - V: one fp32 scale per (batch, kv head) over all Nk keys, codes stored
 *    transposed as [B, Hkv, d, Nk_pad], Nk_pad = Nk rounded up to 16, zero
 *    codes in the padding.
 * d must be 128 for fa_fwd_fp8 (64 or 128 for the quantizers).
 * ---------------------------------------------------------------------------- */

/*
 * Quantize Q or K.  x: [B, N, H, d] 16-bit (dt); x8: [B, N, H, d] bytes;
 * scales: [B, H, ceil(N / 128)] fp32; signs: d fp32 values of +-1 on the device,
 * or NULL for no rotation.  x, x8 16-byte aligned, scales and signs 4-byte
 * aligned.  Writes every code and scale; FA_ERR_INVALID / _UNSUPPORTED /
 * _ALIGN on bad arguments, FA_ERR_CUDA if the launch fails.
 */
fa_status fa_fp8_quantize_qk(const void* x, void* x8, float* scales, const float* signs, int B, int H, int N, int d,
                             fa_dtype dt, fa_stream_t stream);

/* Workspace bytes of fa_fp8_quantize_v: B * Hkv * ceil(Nk / 128) fp32 block maxima (0 on bad sizes). */
size_t fa_fp8_v_workspace_bytes(int B, int Hkv, int Nk);

/*
 * Quantize V.  v: [B, Nk, Hkv, d] 16-bit; v8t: [B, Hkv, d, Nk_pad] bytes
 * (Nk_pad = Nk rounded up to 16); scale: [B, Hkv] fp32; workspace as sized by
 * fa_fp8_v_workspace_bytes.  v, v8t, workspace 16-byte aligned, scale 4-byte.
 */
fa_status fa_fp8_quantize_v(const void* v, void* v8t, float* scale, void* workspace, int B, int Hkv, int Nk,
                            int d, fa_dtype dt, fa_stream_t stream);

/*
 * Q, K and V of one FP8 forward pass quantized together, in two launches (the
 * Q and K rows with the V block maxima, then V's transposing encode): the same
 * codes and scales as fa_fp8_quantize_qk on q and on k (both with `signs`)
 * and fa_fp8_quantize_v on v.  q [B, Nq, Hq, d], k and v [B, Nk, Hkv, d]
 * 16-bit; q8 [B, Nq, Hq, d] and k8 [B, Nk, Hkv, d] bytes with q_scale
 * [B, Hq, ceil(Nq / 128)] and k_scale [B, Hkv, ceil(Nk / 128)]; v8t
 * [B, Hkv, d, Nk_pad] bytes with v_scale [B, Hkv]; workspace as sized by
 * fa_fp8_v_workspace_bytes(B, Hkv, Nk).  Tensors and workspace 16-byte
 * aligned, scales and signs 4-byte aligned.
 */
fa_status fa_fp8_quantize_qkv(const void* q, const void* k, const void* v, void* q8, void* k8, void* v8t,
                              float* q_scale, float* k_scale, float* v_scale, const float* signs, void* workspace,
                              int B, int Hq, int Hkv, int Nq, int Nk, int d, fa_dtype dt, fa_stream_t stream);

/*
 * FP8 forward.  q8 [B, Nq, Hq, 128] and k8 [B, Nk, Hkv, 128] E4M3 codes with
 * scales [B, Hq, ceil(Nq / 128)] and [B, Hkv, ceil(Nk / 128)]; v8t [B, Hkv,
 * 128, Nk_pad] with scale [B, Hkv] (as written by the quantizers above).
 * Computes S = scale * (Q K^T) (divided by d when `rotated`), the online
 * softmax of the 16-bit path with P rounded to E4M3 for the P V product, and
 * writes o [B, Nq, Hq, 128] in `out_dt` and lse [B, Hq, Nq] fp32 (natural log
 * of the scaled scores).  Same causal, GQA, alignment and error rules as fa_fwd.
 */
fa_status fa_fwd_fp8(const void* q8, const float* q_scale, const void* k8, const float* k_scale, const void* v8t,
                     const float* v_scale, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                     int causal, float scale, int rotated, fa_dtype out_dt, fa_stream_t stream);

/*
 * Log-sum-exp merge of a partial attention result over a disjoint set of keys
 * into an accumulator ("FlashAttention 심층 분석", "Flash-Decoding": partial
 * results over key ranges merge by their log-sum-exp); the step that folds each
 * key/value chunk of a context-parallel ring into the running result.
 * o_acc fp32 [B, N, H, d] and lse_acc fp32 [B, H, N] (the caller's accumulator);
 * o_part 16-bit [B, N, H, d] and lse_part [B, H, N] as written by fa_fwd.
 * mode 0: acc = part; 1: acc = merge(acc, part); 2: o_out 16-bit [B, N, H, d] =
 * merge(acc, part) and lse_acc = the merged LSE (the last chunk).  A row whose
 * LSE is -inf in both has O = 0.  o_acc, o_part, o_out 16-byte aligned.
 */
fa_status fa_lse_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                       int N, int H, int d, int mode, fa_dtype dt, fa_stream_t stream);

/*
 * Forward over one key/value chunk merged into an fp32 accumulator by
 * log-sum-exp ("FlashAttention 심층 분석", "Flash-Decoding": attention over
 * disjoint key ranges combines exactly by the ranges' log-sum-exp) -- the
 * fa_fwd kernel with the merge done in its epilogue, so the partial result is
 * never rounded to 16 bits.  acc_o fp32 [B, Nq, Hq, d] and acc_lse fp32
 * [B, Hq, Nq] are the caller's accumulator.  mode 0: acc = this chunk's result;
 * 1: acc = merge(acc, result); 2: o and lse = merge(acc, result), acc left as
 * it was (the last chunk).  o [B, Nq, Hq, d] (dt) and lse are written in every
 * mode (modes 0 and 1: the running result).  A row with no visible key in
 * either gets O = 0 and LSE = -inf.  Otherwise as fa_fwd; acc_o 16-byte
 * aligned, acc_lse 4-byte aligned.
 */
fa_status fa_fwd_merge(const void* q, const void* k, const void* v, void* o, float* lse, float* acc_o,
                       float* acc_lse, int mode, int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                       float scale, fa_dtype dt, fa_stream_t stream);

/*
 * Backward contributions of one key/value chunk added into fp32 accumulators
 * (the dK/dV and dQ kernels of fa_bwd with their epilogues adding into fp32
 * instead of writing 16-bit gradients): with P = exp(scale Q K^T - lse) over
 * this chunk's keys and D the rows' term from fa_bwd_preprocess (`workspace`,
 * over the whole rows), dq_acc [B, Nq, Hq, d] += scale dS K, and dk_acc,
 * dv_acc [B, Nk, Hkv, d] += scale dS^T Q, P^T dO (summed over each group's
 * query heads).  Summed over a partition of the keys this is the full
 * backward, since the chain rule is linear in the keys once LSE and D are
 * fixed.  init bit 0: dq_acc is set instead of added to; bit 1: dk_acc and
 * dv_acc are.  All fp32 buffers 16-byte aligned.  Otherwise as fa_bwd.
 */
fa_status fa_bwd_accumulate(const void* q, const void* k, const void* v, const void* dout, const float* lse,
                            const void* workspace, float* dq_acc, float* dk_acc, float* dv_acc, int init, int B,
                            int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale, fa_dtype dt,
                            fa_stream_t stream);

/*
 * Summation of 16-bit partial results in fp32 (the backward of the ring sums the
 * dQ, dK and dV contributions of every key/value chunk): fa_accumulate sets
 * acc[i] = (init ? 0 : acc[i]) + part[i] for n elements, fa_cast_f32 writes
 * out[i] = acc[i] rounded to the 16-bit type.  n a multiple of 8; acc, part and
 * out 16-byte aligned device pointers.
 */
fa_status fa_accumulate(float* acc, const void* part, long long n, int init, fa_dtype dt, fa_stream_t stream);
fa_status fa_cast_f32(const float* acc, void* out, long long n, fa_dtype dt, fa_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the device status word that the
 * kernels set when a bounded wait runs out (FA_ERR_TIMEOUT) or, in the checking
 * build libfa_checks.so (same ABI, compiled with FA_CHECKS), when a device-side
 * index check finds an access outside its tensor (FA_ERR_BOUNDS; the access is
 * skipped, nothing traps).  Returns FA_OK when no kernel reported an error.
 */
fa_status fa_get_device_status(fa_stream_t stream);

/*
 * Self-test of the kernels' failure detection, with no fault involved: launches
 * one CTA that waits on an mbarrier nothing ever arrives on, through the same
 * bounded-wait routine the attention kernels use, giving up after `limit_us`
 * microseconds (1 .. 2000000).  A following fa_get_device_status must return
 * FA_ERR_TIMEOUT, and the CUDA context stays usable.
 */
fa_status fa_watchdog_selftest(int limit_us, fa_stream_t stream);

/* Static, NUL-terminated description of a status code. */
const char* fa_status_string(fa_status s);

/* Library version, for the binding's sanity check. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
