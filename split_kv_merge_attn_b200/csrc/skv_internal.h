// Internal interface between the host-side ABI layer (validation, planning,
// workspace layout) and the translation unit that holds the kernels and their
// launchers.  Not part of the public C ABI.
#pragma once

#include <cstddef>
#include <cstdint>

#include "splitkv.h"


namespace skv {

// Device error codes recorded when a bounded wait gives up.
enum DeviceError : int {
  kErrDecodeEmptyWait = 0x101,
  kErrDecodeFullWait = 0x102,
  kErrDecodeCounter = 0x103,   // a decode arrival counter was not zero before the call
  kErrPrefillWait = 0x201,
};

// Constants of the split planner (mirrored by the decode kernel).
constexpr int kSplitAlign = 64;
constexpr int kSplitMinKeys = 128;
constexpr int kSplitMax = 256;
// The automatic decode plan aims for ceil(num_sms * num / den) CTAs in all:
// one per SM for D <= 128 (the kernel could hold two, but fewer, longer splits
// measured faster: fewer concurrent K/V streams and a smaller merge) and two
// per three SMs for D = 256, whose CTA keeps twice the bytes in flight.
constexpr int kCtasPerSmNum = 1, kCtasPerSmDen = 1;
constexpr int kCtasPerSmD256Num = 2, kCtasPerSmD256Den = 3;
constexpr int kDecodeRowsPerCta = 16;
// Largest number of KV chunks of one multi-chunk prefill call.
constexpr int kMaxKvChunks = 64;
constexpr int kPrefillRowsPerCta = 256;      // two 128-row query tiles (D <= 128)
constexpr int kPrefillRowsPerCtaD256 = 128;  // one tile (D = 256)
inline int prefill_rows_per_cta(int D) { return D == 256 ? kPrefillRowsPerCtaD256 : kPrefillRowsPerCta; }

inline int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Launchers (kernels TU).  Return a cudaError_t value (0 = success).
int sm_count();  // SM count of the current device (cached per device)

int launch_merge_state(const void* o_parts, const float* lse_parts, void* out, float* lse, int P, int B,
                       int H, int S, int D, int layout_bsh, skv_dtype parts_dt, skv_dtype out_dt,
                       int64_t part_stride_o, int64_t part_stride_lse, skv_stream_t stream);

// counters: null = partials only (merge_state merges them); else per-group
// arrival counters, zero on entry, and the last CTA of each group merges.
int launch_decode(const void* q, const void* k, const void* v, void* out, float* lse, float* part_o,
                  float* part_lse, int* counters, const int32_t* kv_len, int B, int Hq, int Hkv, int Lq, int Lkv,
                  int D, float scale, skv_dtype dt, int num_splits, int causal, skv_stream_t stream);

struct PrefillLaunch {
  const void* q;
  const void* k;  // K, or the smoothed K' when smooth_k
  const void* v;
  void* out;
  float* lse;
  const float* kmean;      // [B(or seqs), Hkv, D] fp32 mean (materialised smooth_k), else null
  const float* kpartial;   // [chunks, B(or seqs), Hkv, D] per-256-key sums (shift smooth_k), else null
  int shift_logits;        // smooth_k == 1: apply the mean shift to the logits
  int causal;              // bottom-right aligned causal mask
  const int32_t* cu_q;     // device, varlen only
  const int32_t* cu_k;
  const int32_t* order;    // device work order (varlen)
  const int32_t* offsets;
  int B, Hq, Hkv, Sq, Sk, D;
  int max_seqlen_q;
  float scale;
  skv_dtype dt;
  skv_layout layout;
  int nchunks;               // dense: KV chunks (1 = the whole key range)
  const int32_t* kv_bounds;  // host [nchunks + 1] chunk bounds, or null when nchunks == 1
  int after_kpartial;        // 1: the kernel just launched on the stream is the one writing kpartial
};
int launch_prefill(const PrefillLaunch& p, skv_stream_t stream);

// INT8 Q K'^T prefill (dense HND, D = 128): mean of K, int8 codes of K - mean
// and of Q with their per-128-row scales and the per-row smoothing shift, then
// the prefill over the codes.  All buffers device, caller-owned.
struct Int8PrefillLaunch {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;
  float* kpartial;  // [ceil(Sk/256), B, Hkv, 128]
  float* kmean;     // [B, Hkv, 128]
  int8_t* q8;       // [B, Hq, Sq, 128]
  int8_t* k8;       // [B, Hkv, Sk, 128]
  float* qscale;    // [B, Hq, ceil(Sq/128)]
  float* kscale;    // [B, Hkv, ceil(Sk/128)]
  float* dq;        // [B, Hq, Sq]
  int B, Hq, Hkv, Sq, Sk;
  float scale;
  skv_dtype dt;
  int causal;
};
int launch_prefill_int8(const Int8PrefillLaunch& p, skv_stream_t stream);

int launch_varlen_plan(const int32_t* cu_q, const int32_t* cu_k, int B, int Hq, int rows_per_cta, int32_t* order,
                       int32_t* offsets, skv_stream_t stream);

// smooth_k prepass: fp32 per-256-key column sums of K for each (batch or
// sequence, kv head) into `partial`; if k_smoothed != null also the mean
// kmean [B, Hkv, D] and K' = K - mean rounded to the input type.
// Dense multi-chunk calls pass kv_ranges > 1 chunks per batch entry with host
// bounds kv_bounds[kv_ranges + 1]; every mean is then per (batch, chunk).
int launch_smooth_k(const void* k, void* k_smoothed, float* kmean, float* partial, const int32_t* cu_k, int B,
                    int Hkv, int Sk, int max_len, int D, skv_dtype dt, skv_layout layout, skv_stream_t stream,
                    int kv_ranges = 1, const int32_t* kv_bounds = nullptr);

int read_and_clear_device_error(int* code);

// Elementwise evaluation of the prefill's FMA-pipe exp2 (diagnostics).
int launch_exp2_fma(const float* x, float* y, int64_t n, skv_stream_t stream);

// Maps a cudaError_t value to a status: SKV_OK for 0, else SKV_ERR_CUDA with
// the error recorded for skv_last_cuda_error on the calling thread.
skv_status cuda_status(int e);

// Launch accounting (incremented by every successful kernel launch).
void count_launches(int n);
uint64_t launch_count();

}  // namespace skv
