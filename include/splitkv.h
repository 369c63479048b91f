/*
 * splitkv.h -- C ABI of the B200 (sm_100a) attention-with-LSE library.
 *
 * Three device operations and their host-side planning helpers:
 *
 *   attn_fwd_lse         prefill / varlen attention forward writing O and one
 *                        log2 LSE per query row;
 *   attn_splitkv_decode  split-KV decode for 1..4 query rows per head with a
 *                        stable per-split online softmax, merged on device;
 *   merge_state          combines partial (O, LSE) pairs of disjoint KV ranges.
 *
 * The quantity (all entry points): for query row i of head h and the KV range J
 * of the call, s_j = scale * q_i . k_j and
 *
 *     LSE_i = log2( sum_{j in J} exp(s_j) ),  O_i = sum_j exp(s_j) v_j / sum_j exp(s_j)
 *
 * over the ORIGINAL, unsmoothed logits: natural exponentials, reported in log2
 * units, one value per row ("ARK return_lse gives the same LSE for every 16
 * query rows", auto-round issue #2556, "Expected:" in Problem Description).
 * An empty KV range gives O_i = 0 and LSE_i = -inf.
 *
 * Conventions (SGLang PR #33840 "[XPU] Support softmax_lse in sgl_kernel::fwd
 * API", Modifications and the review thread):
 *   - outputs are written in place into caller-owned device buffers; the return
 *     value is only a status;
 *   - the LSE output is optional: a NULL lse pointer means "do not store it";
 *   - the varlen (packed TND) path writes a 2-D LSE [H, total_q]; the dense
 *     paths write a 3-D LSE [B, H, S_q].
 * Shapes that do not satisfy the contract are rejected with a status, never
 * reshaped silently (SGLang Ascend backend record "Unexpected Ascend TND
 * softmax LSE shape").  There is no fixed exponent offset ("phi"): the split
 * path uses a per-split running max (ExecuTorch PR #22133 "Prevent Voxtral
 * NaNs in CUDA split-K attention").
 *
 * Memory and ownership: every pointer named "device" must point to device
 * memory of the current CUDA device; the library never allocates device memory
 * and keeps no per-call state.  Scratch space is the caller's "workspace",
 * sized by the matching *_workspace() query.  All device entry points are
 * asynchronous on `stream` (NULL = the legacy default stream), validate every
 * argument on the host first and launch nothing if validation fails.
 *
 * Stream order: the results of a call are visible to everything the caller
 * enqueues after it on the stream, as usual.  To hide launch latency, the
 * decode's split kernel, the merge_state kernels and the smooth_k column sums
 * are launched with programmatic stream serialization (their CTAs may start
 * while the preceding kernel finishes; each waits for that kernel's completion
 * before it touches memory), and the library's kernels signal their dependents
 * early (griddepcontrol.launch_dependents).  A kernel the caller itself
 * launches right after a call WITH the programmatic-serialization attribute
 * must therefore wait for its predecessor (griddepcontrol.wait /
 * cudaGridDependencySynchronize) before it reads the call's outputs; kernels
 * launched without that attribute need nothing.
 *
 * Element types: bf16 or fp16 for q/k/v/out (q, k, v and out share one type);
 * LSE is always fp32.  Head dimension D in {64, 128, 256} (INT8 prefill: 128).
 * Pointers passed as tensors must be 16-byte aligned.
 *
 * Thread safety: entry points may be called from several host threads; calls
 * that share a workspace must not overlap on the device.
 */
#ifndef SPLITKV_H_
#define SPLITKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st* skv_stream_t;

typedef enum {
  SKV_OK = 0,
  SKV_ERR_INVALID_ARG = 1,        /* a size, pointer, alignment or layout is invalid */
  SKV_ERR_UNSUPPORTED = 2,        /* valid but not implemented (e.g. D=96, fp32 inputs) */
  SKV_ERR_WORKSPACE_TOO_SMALL = 3,/* workspace_bytes < the *_workspace() query */
  SKV_ERR_CUDA = 4                /* a CUDA runtime/driver call failed; see skv_last_cuda_error */
} skv_status;

typedef enum { SKV_BF16 = 0, SKV_FP16 = 1, SKV_FP32 = 2 } skv_dtype;

/* HND: [B, H, S, D] contiguous.  NHD: [B, S, H, D] contiguous.
 * TND: packed varlen [T, H, D] contiguous; needs cu_seqlens. */
typedef enum { SKV_HND = 0, SKV_NHD = 1, SKV_TND = 2 } skv_layout;

/* ------------------------------------------------------------------------ */
/* attn_fwd_lse: attention forward with a per-row log2 LSE (prefill/varlen). */
/*
 * Defined by the ARK return_lse issue ("Expected:" and the repro's
 * ref_lse_log2); layouts and the varlen LSE shape by the SGLang sgl_kernel::fwd
 * PR (CUDA FA: varlen LSE 2-D, dense 3-D); GQA by Hq % Hkv == 0 (SGLang Ascend
 * backend record, validationCode), query head h reading kv head h / (Hq/Hkv).
 *
 * Dense (layout HND or NHD; cu_seqlens_q = cu_seqlens_k = NULL):
 *   q [B, Hq, Sq, D] / [B, Sq, Hq, D]; k, v [B, Hkv, Sk, D] / [B, Sk, Hkv, D];
 *   out like q; lse [B, Hq, Sq] fp32 (nullable).
 * Varlen (layout TND): B = number of sequences; cu_seqlens_q, cu_seqlens_k are
 *   DEVICE int32 arrays of B+1 non-decreasing offsets starting at 0;
 *   q [total_q, Hq, D], k, v [total_k, Hkv, D] with total_q = Sq and
 *   total_k = Sk (the caller passes the packed totals); sequence b owns query
 *   rows [cu_q[b], cu_q[b+1]) and keys [cu_k[b], cu_k[b+1]); out like q;
 *   lse [Hq, total_q] (nullable).  max_seqlen_q bounds every query length
 *   (used to size the grid); max_seqlen_k is accepted for API symmetry.
 * Non-causal: every query row sees every key of its sequence.
 *
 * smooth_k (ARK issue, second issue and part 3 of the repro): K is smoothed by
 * its mean mu over the call's own KV range, taken in fp32 per (batch or
 * sequence, kv head, channel), and the LSE is corrected by adding
 * scale * (q_i . mu) / ln 2 so that it stays the LSE of the ORIGINAL logits --
 * partial LSEs of chunks with different means then lie on one scale.  O is
 * unchanged up to rounding (softmax is shift invariant).
 *   0: no smoothing.
 *   1: the smoothing is applied to the fp32 logits, s_ij - scale * q_i . mu,
 *      which is exactly K' = K - mu with no 16-bit rounding of K'.
 *   2: K' = K - mu is materialised in the input type in the workspace and used
 *      by the tensor cores.  The 16-bit rounding of K' perturbs every logit by
 *      up to scale * sum_d |q_d| |K'_d| * 2^-9, so the LSE of this mode is NOT
 *      held to the 1e-3 log2 accuracy of modes 0 and 1 against the exact
 *      unsmoothed LSE: on randn-like inputs with K offset by 0.5 (the chunked
 *      workload) its error is about 2e-3 log2, and it grows with |q| |K'|
 *      (about 2e-2 log2 with query rows scaled up to 4x).  It equals, to 1e-3,
 *      the exact LSE of the logits of the rounded K' (plus the correction).
 *      Use mode 1 where the LSE accuracy matters.
 *   Both modes need workspace (see below); for varlen, max_seqlen_k must bound
 *   every key length.
 *
 * scale: the logit scale (e.g. D^-0.5), finite and > 0.
 * k and v may be NULL only when there are no keys (Sk == 0).
 * workspace: device, >= attn_fwd_lse_workspace(...) bytes, 256-byte aligned;
 *   may be NULL when that query returns 0.  After a varlen call its first
 *   bytes hold the work order: int32 order[B] (sequences, longest kv first,
 *   ties by index) then int32 offsets[B+1] (prefix sums of
 *   Hq*ceil(len_q/rows), rows = 256 query rows per CTA for D <= 128 and 128 for
 *   D = 256).
 * Errors: SKV_ERR_INVALID_ARG for NULL q/out, NULL k/v with keys, non-positive sizes (B, Hq,
 *   Hkv, D; Sq, Sk may be 0 in the dense case), Hq % Hkv != 0, misaligned
 *   pointers, unknown layout/dtype, or missing/extra cu_seqlens;
 *   SKV_ERR_UNSUPPORTED for D not in {64,128,256} or dtype fp32.
 */
skv_status attn_fwd_lse(const void* q, const void* k, const void* v, void* out, float* lse,
                        int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                        skv_dtype dtype, skv_layout layout,
                        const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                        int max_seqlen_q, int max_seqlen_k, int smooth_k,
                        void* workspace, size_t workspace_bytes, skv_stream_t stream);

/* attn_fwd_lse_causal: attn_fwd_lse with a causal mask.
 *
 * Not on the source pages (they use full, non-causal key ranges); the plainest
 * adjacent variant, for autoregressive chunks: the len_q query rows of a
 * sequence (batch entry or varlen sequence) are the LAST len_q positions of
 * its len_k keys, so query row i sees keys j <= i + len_k - len_q
 * (bottom-right alignment; the usual lower triangle when len_q == len_k).
 * Rows i < len_q - len_k see no key: O = 0, LSE = -inf.  Arguments, layouts,
 * workspace and errors as attn_fwd_lse; smooth_k subtracts the mean of the
 * call's whole key range and still returns the unsmoothed LSE of the visible
 * keys. */
skv_status attn_fwd_lse_causal(const void* q, const void* k, const void* v, void* out, float* lse,
                               int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                               skv_dtype dtype, skv_layout layout, const int32_t* cu_seqlens_q,
                               const int32_t* cu_seqlens_k, int max_seqlen_q, int max_seqlen_k,
                               int smooth_k, void* workspace, size_t workspace_bytes,
                               skv_stream_t stream);

/* attn_fwd_lse_chunks: the partial results of one query block over several
 * KV chunks, in one launch.
 *
 * Chunk c is keys [chunk_bounds[c], chunk_bounds[c+1]) of every batch entry
 * and kv head.  Its partial (O_c, LSE_c) is exactly what attn_fwd_lse gives
 * for q against k[..., chunk c, ...], v[..., chunk c, ...] (with smooth_k,
 * the mean is chunk c's own and LSE_c is still that of the original logits,
 * so the partials lie on one scale).  These are the per-chunk partials that
 * ring / chunked attention merges (ARK issue, Problem Description: chunks
 * smoothed by their own means whose LSEs are merged; SGLang PR review thread:
 * the per-hop merge of ring attention); merge_state of the num_chunks parts gives
 * the attention over all Sk keys.  All chunks run in one grid, so the work of
 * the chunks fills the GPU together instead of each leaving a partial wave.
 *
 * Dense layouts only (HND or NHD), non-causal.  q, k, v as attn_fwd_lse;
 * out_parts [num_chunks, <q's shape>] in q's layout and type (part c starts
 * c * B*Hq*Sq*D elements in); lse_parts [num_chunks, B, Hq, Sq] fp32
 * (nullable).  chunk_bounds: HOST int32 [num_chunks + 1], chunk_bounds[0] = 0,
 * non-decreasing, chunk_bounds[num_chunks] = Sk (empty chunks are allowed:
 * O_c = 0, LSE_c = -inf).  1 <= num_chunks <= 64.  workspace: device,
 * 256-byte aligned, >= attn_fwd_lse_chunks_workspace(...) bytes (0 without
 * smooth_k).  Errors as attn_fwd_lse, and SKV_ERR_INVALID_ARG for a TND
 * layout or invalid chunk bounds. */
skv_status attn_fwd_lse_chunks(const void* q, const void* k, const void* v, void* out_parts,
                               float* lse_parts, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                               float scale, skv_dtype dtype, skv_layout layout, int num_chunks,
                               const int32_t* chunk_bounds, int smooth_k, void* workspace,
                               size_t workspace_bytes, skv_stream_t stream);
size_t attn_fwd_lse_chunks_workspace(int B, int Hq, int Hkv, int Sk, int D, skv_dtype dtype,
                                     skv_layout layout, int num_chunks, int smooth_k);

/* attn_fwd_lse_int8: attention with Q K'^T computed from INT8 codes.
 *
 * ARK issue, Problem Description: K is smoothed (its mean over the call's keys
 * subtracted) so that it quantizes well to INT8, and the LSE of the original
 * logits is restored with the q . mean(K) shift.  Here: K' = K - mean (fp32)
 * and Q are quantized per block of 128 rows (symmetric, scale = amax / 127,
 * round half to even), S is the exact s32 product of the codes on the int8
 * tensor cores times the two block scales, and the softmax and P V (V in
 * 16-bit) are those of attn_fwd_lse; LSE = log2 sum_j exp(s_ij) + the shift.
 * Results approximate attn_fwd_lse to the quantization error (logits to about
 * 1e-2 for randn-like inputs); they are exact for inputs the codes represent.
 * Dense HND only: q [B,Hq,Sq,128], k/v [B,Hkv,Sk,128], out like q, lse
 * [B,Hq,Sq] fp32 (nullable); bf16 or fp16; causal 0/1 as attn_fwd_lse_causal.
 * workspace (device, 256-byte aligned, >= attn_fwd_lse_int8_workspace bytes)
 * holds, each section 256-byte aligned and in this order: fp32 column sums
 * [ceil(Sk/256), B, Hkv, 128], fp32 mean [B, Hkv, 128], Q codes int8
 * [B, Hq, Sq, 128], K' codes int8 [B, Hkv, Sk, 128], fp32 Q block scales
 * [B, Hq, ceil(Sq/128)], fp32 K' block scales [B, Hkv, ceil(Sk/128)], fp32
 * shift [B, Hq, Sq].  Errors as attn_fwd_lse; SKV_ERR_UNSUPPORTED for D != 128,
 * fp32, or B*Hq > 65535. */
skv_status attn_fwd_lse_int8(const void* q, const void* k, const void* v, void* out, float* lse,
                             int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                             skv_dtype dtype, int causal, void* workspace, size_t workspace_bytes,
                             skv_stream_t stream);
size_t attn_fwd_lse_int8_workspace(int B, int Hq, int Hkv, int Sq, int Sk, int D);

/* Workspace bytes attn_fwd_lse needs for these arguments (0 if none).
 * Sk is the per-batch key length (dense) or total_k (TND). Host-only, pure. */
size_t attn_fwd_lse_workspace(int B, int Hq, int Hkv, int Sk, int D, skv_dtype dtype,
                              skv_layout layout, int smooth_k);

/* Host restatement of the varlen work order the device builds (for tests and
 * inspection).  cu_seqlens_q/k are HOST arrays of B+1 entries; writes order[B]
 * and offsets[B+1] as documented under attn_fwd_lse, for head dimension D
 * (rows per CTA: 256 for D <= 128, 128 for D = 256). */
skv_status attn_varlen_plan(const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B,
                            int Hq, int D, int32_t* order, int32_t* offsets);

/* ------------------------------------------------------------------------ */
/* attn_splitkv_decode: split-KV decode with a stable online softmax.        */
/*
 * ExecuTorch PR #22133 (split-K decode kernel, small-query split-K kernel and
 * cross-split reduce; review items 1-3): each split keeps its own running max
 * and writes rescaled partials; the partials are merged against the global
 * max.  Empty trailing splits are allowed and write O = 0, LSE = -inf.
 *
 * q [B, Hq, Lq, D]; k, v [B, Hkv, Lkv, D] (HND, contiguous); out [B, Hq, Lq, D];
 * lse [B, Hq, Lq] fp32 (nullable).  1 <= Lq (any Lq works; 1..4 is the target).
 * Non-causal: all Lq rows see keys [0, kv_len[b]).
 * kv_len: DEVICE int32 [B] or NULL (= Lkv for every batch).  It is read on the
 *   device, so a captured CUDA graph follows its current value; values are
 *   clamped to [0, Lkv].
 * num_splits: 0 = automatic (attn_splitkv_plan with the device's SM count);
 *   otherwise the number of splits, 1..256.
 * workspace: device, >= attn_splitkv_workspace(B, Hq, Lq, D, num_splits) bytes
 *   for the split count actually used (0 bytes when it is 1).
 * Errors as for attn_fwd_lse; SKV_ERR_UNSUPPORTED for D not in {64,128,256}.
 */
skv_status attn_splitkv_decode(const void* q, const void* k, const void* v, void* out,
                               float* lse, int B, int Hq, int Hkv, int Lq, int Lkv, int D,
                               float scale, skv_dtype dtype, const int32_t* kv_len,
                               int num_splits, void* workspace, size_t workspace_bytes,
                               skv_stream_t stream);

/* attn_splitkv_decode_causal: attn_splitkv_decode with a causal mask over the
 * Lq query rows (not on the source pages; the reading of attn_fwd_lse_causal):
 * with n = kv_len[b] (or Lkv), query row i of [0, Lq) sees keys
 * [0, n - Lq + 1 + i), so the last row sees the whole cache and Lq = 1 is the
 * non-causal decode.  Arguments, workspace and errors as attn_splitkv_decode. */
skv_status attn_splitkv_decode_causal(const void* q, const void* k, const void* v, void* out,
                                      float* lse, int B, int Hq, int Hkv, int Lq, int Lkv, int D,
                                      float scale, skv_dtype dtype, const int32_t* kv_len,
                                      int num_splits, void* workspace, size_t workspace_bytes,
                                      skv_stream_t stream);

/* Split plan (host, pure integer).  For n keys, split s covers
 *   [s*C, min((s+1)*C, n)),  C = 64 * ceil(ceil(n / num_splits) / 64).
 * If requested_splits > 0 it is used as is (1..256).  Otherwise, with
 * G = Hq/Hkv and units = B * Hkv * ceil(G*Lq/16) (the decode CTAs of one
 * split), the count is
 *   S0 = max(1, ceil(T / units)),  T = ceil(num_sms * 1 / 1)  for D <= 128,
 *                                  T = ceil(num_sms * 2 / 3)  for D = 256,
 *   S1 = min(S0, max(1, ceil(n / 128)), 256)   (>= 128 keys per split),
 *   num_splits = ceil(n / C(S1))  (n > 0; drops splits the rounding of C
 *                                  would leave empty), else S1,
 * i.e. about one decode CTA per SM for D <= 128 and two per three SMs for
 * D = 256 (whose CTA keeps twice the bytes in flight).  The targets were
 * chosen by measurement; the pages only ask for "splits sized to fill the
 * SMs".  Examples with num_sms = 148: B=1, Hq=32, Hkv=8, Lq=1, D=128 gives 16
 * splits at n = 4096 and 19 at n = 32768; B=1, Hq=16, Hkv=4, Lq=1, D=256
 * gives 25 at n = 32768.
 * Writes *num_splits and, if bounds != NULL, bounds[0..num_splits] (host) with
 * split s = [bounds[s], bounds[s+1]). */
skv_status attn_splitkv_plan(int B, int Hq, int Hkv, int Lq, int n, int D, int num_sms,
                             int requested_splits, int* num_splits, int32_t* bounds);

/* Workspace bytes for a decode with this many splits: fp32 partial O and LSE
 * plus the arrival counters attn_splitkv_decode_fused uses (0 for one split). */
size_t attn_splitkv_workspace(int B, int Hq, int Lq, int D, int num_splits);

/* attn_splitkv_decode_fused: the same decode in ONE kernel launch.
 *
 * The single-launch variant of the split-KV decode: the cross-split reduce of
 * the ExecuTorch split-K PR (and the merge formula of merge_state) runs inside
 * the decode kernel.  Each CTA writes its split's partial (O, LSE) and then
 * increments the arrival counter of its (batch, kv head, row group); the CTA
 * that brings the counter to num_splits merges the group's partials, writes
 * out and lse, and sets the counter back to zero.  No CTA waits for another.
 * Results equal attn_splitkv_decode's up to fp32 rounding order.
 *
 * Arguments as attn_splitkv_decode.  The workspace's counter region must be
 * zero before the first call on a workspace: zero the whole workspace once
 * (attn_splitkv_workspace_init, or any memset).  Every call that completes
 * without a device error leaves it zero again, so one zeroed workspace serves
 * any number of calls and CUDA-graph replays on one stream.  After a device
 * error (skv_device_error), zero it again.  A counter found non-zero on
 * arrival records device error 0x103.  Calls that overlap on the GPU must use
 * different workspaces. */
skv_status attn_splitkv_decode_fused(const void* q, const void* k, const void* v, void* out,
                                     float* lse, int B, int Hq, int Hkv, int Lq, int Lkv, int D,
                                     float scale, skv_dtype dtype, const int32_t* kv_len,
                                     int num_splits, void* workspace, size_t workspace_bytes,
                                     skv_stream_t stream);

/* Zeroes `workspace_bytes` bytes of a decode workspace on `stream`
 * (cudaMemsetAsync): the one-time preparation attn_splitkv_decode_fused needs.
 * NULL with 0 bytes is a no-op. */
skv_status attn_splitkv_workspace_init(void* workspace, size_t workspace_bytes, skv_stream_t stream);

/* attn_splitkv_decode_static: the same decode for callers that cannot
 * allocate device memory (code running under an allocator that owns all device
 * memory, plugins handed only their input and output buffers, hosts that
 * forbid allocation after start-up).  The source pages describe no such entry
 * point; it exists for those callers.
 *
 * Arguments and results are those of attn_splitkv_decode without the
 * workspace: the per-split partials go to a fixed 8 MiB array in device global
 * memory that the library defines (every GPU that loads the library holds it
 * until the process exits).  Nothing is allocated: no cudaMalloc, cudaFree or
 * allocating library call.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *   - A problem whose partials need more than 8 MiB
 *     (attn_splitkv_workspace(B, Hq, Lq, D, splits) > 8 MiB) is refused with
 *     SKV_ERR_WORKSPACE_TOO_SMALL before anything is launched.
 *   - Every call shares the one array and it keeps the last call's contents;
 *     nothing in it needs to start at zero (each call writes every partial
 *     slot it reads).  Calls that overlap on the GPU (other streams, other host
 *     threads) race on it and must be serialised by the caller.
 * Errors: the size, dtype, head-dimension and scale checks of
 * attn_splitkv_decode come first and give its statuses; then the 8 MiB
 * refusal; then attn_splitkv_decode's pointer checks.  A failing CUDA call
 * (device query, address lookup) returns SKV_ERR_CUDA with the error kept for
 * skv_last_cuda_error. */
skv_status attn_splitkv_decode_static(const void* q, const void* k, const void* v, void* out,
                                      float* lse, int B, int Hq, int Hkv, int Lq, int Lkv, int D,
                                      float scale, skv_dtype dtype, const int32_t* kv_len,
                                      int num_splits, skv_stream_t stream);

/* ------------------------------------------------------------------------ */
/* merge_state: combine P partial (O, LSE) results of disjoint KV ranges.    */
/*
 * The per-hop merge of ring attention (merge_state_v2 / _merge_attention_partials
 * in the SGLang PR thread) and the cross-split reduce of the ExecuTorch split-K
 * PR: per row, M = max_p L_p, w_p = 2^(L_p - M) (0 for -inf),
 *   O = sum_p w_p O_p / sum_p w_p,  LSE = M + log2(sum_p w_p);
 * if every part is -inf: O = 0, LSE = -inf.  Parts of weight 0 are not read.
 *
 * o_parts: device, P parts each laid out like an attention output of shape
 *   (B, H, S, D) in `layout` (HND: [B,H,S,D]; NHD/TND: [B,S,H,D], for TND pass
 *   B = 1 and S = total_q); part p starts part_stride_o ELEMENTS after part p-1
 *   (0 = B*H*S*D, i.e. packed).
 * lse_parts: device fp32, P parts of [B, H, S] (for TND: [H, total_q]);
 *   part stride part_stride_lse elements (0 = B*H*S).
 * out: device, one part's layout, type out_dtype; lse: device [B,H,S] or NULL.
 * parts_dtype: bf16, fp16 or fp32; out_dtype: bf16, fp16 or fp32.
 * Any flattening of rows works with B = H = 1, S = rows, layout HND.
 */
skv_status merge_state(const void* o_parts, const float* lse_parts, void* out, float* lse,
                       int P, int B, int H, int S, int D, skv_layout layout,
                       skv_dtype parts_dtype, skv_dtype out_dtype,
                       int64_t part_stride_o, int64_t part_stride_lse, skv_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Diagnostics.                                                              */

/* Static text for a status code. */
const char* skv_status_string(skv_status s);

/* The cudaError_t of the last failing CUDA call made by this library on the
 * calling host thread (0 if none). */
int skv_last_cuda_error(void);

/* Reads and clears the device-side error word of the current device: nonzero if
 * a kernel gave up a bounded pipeline wait (it then returns without hanging; its
 * outputs are undefined).  Synchronises the device.  Returns SKV_ERR_CUDA if the
 * read itself fails. */
skv_status skv_device_error(int* code);

/* Number of kernels this library has launched in this process so far (all
 * devices, all threads).  Benchmarks difference it around a timed region. */
uint64_t skv_launch_count(void);

/* Library version, e.g. "0.2.0". */
const char* skv_version(void);

/* Evaluates, elementwise on the device, the exp2 that the prefill softmax
 * computes on the FMA pipe for a share of its probabilities: y[i] = 2^x[i]
 * from the degree-3 minimax polynomial of exp2_poly_fit.py (relative error
 * <= 7.5e-5 for x in [-125, 126]; x < -125 gives a value below 2^-124).  Not
 * part of the attention path (for tests of that error).  x, y: device fp32
 * arrays of n elements. */
skv_status skv_exp2_fma(const float* x, float* y, int64_t n, skv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SPLITKV_H_ */
