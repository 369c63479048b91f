// Host side of the C ABI: argument validation (before any device work),
// workspace layout, split and varlen planning, and dispatch to the launchers.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <algorithm>

#include <cuda_runtime_api.h>

#include "skv_internal.h"

namespace {
thread_local int g_last_cuda_error = 0;
}  // namespace

skv_status skv::cuda_status(int e) {
  if (e == 0) return SKV_OK;
  g_last_cuda_error = e;
  return SKV_ERR_CUDA;
}

namespace {
using skv::cuda_status;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool is_half_type(skv_dtype d) { return d == SKV_BF16 || d == SKV_FP16; }

size_t dtype_bytes(skv_dtype d) { return d == SKV_FP32 ? 4 : 2; }

// ----- attn_fwd_lse workspace layout
struct FwdWorkspace {
  size_t order = 0, offsets = 0, kmean = 0, partial = 0, kprime = 0, total = 0;
};

// nranges: key ranges per batch entry with their own smoothing mean (the
// chunks of a multi-chunk call; 1 otherwise).  The per-256-key column sums
// are sized for ranges as long as Sk.
FwdWorkspace fwd_workspace(int B, int Hkv, int Sk, int D, skv_layout layout, int smooth_k, int nranges = 1) {
  FwdWorkspace w;
  size_t off = 0;
  if (layout == SKV_TND) {
    w.order = off;
    off += skv::align256(static_cast<size_t>(B) * 4);
    w.offsets = off;
    off += skv::align256(static_cast<size_t>(B + 1) * 4);
  }
  if (smooth_k) {
    const size_t nchunks = static_cast<size_t>(skv::ceil_div64(Sk, 256));
    const size_t ranges = static_cast<size_t>(B) * nranges;
    w.kmean = off;
    off += skv::align256(ranges * Hkv * D * 4);
    w.partial = off;
    off += skv::align256(nchunks * ranges * Hkv * D * 4);
    if (smooth_k == 2) {
      const size_t rows = layout == SKV_TND ? static_cast<size_t>(Sk) : static_cast<size_t>(B) * Sk;
      w.kprime = off;
      off += skv::align256(rows * Hkv * D * 2);
    }
  }
  w.total = off;
  return w;
}

// [splits][rows][D] fp32 partial O | [splits][rows] fp32 partial LSE |
// [rows] int32 arrival counters (one per (batch, kv head, row group) are used;
// rows bounds their number), each region 256-byte aligned.
struct DecodeWs {
  size_t part_o = 0, part_lse = 0, counters = 0, total = 0;
};
DecodeWs decode_ws_layout(int B, int Hq, int Lq, int D, int splits) {
  DecodeWs w;
  if (splits <= 1) return w;
  const size_t rows = static_cast<size_t>(B) * Hq * Lq;
  w.part_o = 0;
  w.part_lse = skv::align256(static_cast<size_t>(splits) * rows * D * 4);
  w.counters = w.part_lse + skv::align256(static_cast<size_t>(splits) * rows * 4);
  w.total = w.counters + skv::align256(rows * 4);
  return w;
}

size_t decode_workspace(int B, int Hq, int Lq, int D, int splits) {
  return decode_ws_layout(B, Hq, Lq, D, splits).total;
}

}  // namespace

extern "C" {

const char* skv_status_string(skv_status s) {
  switch (s) {
    case SKV_OK: return "SKV_OK";
    case SKV_ERR_INVALID_ARG: return "SKV_ERR_INVALID_ARG: invalid size, pointer, alignment, layout or value";
    case SKV_ERR_UNSUPPORTED: return "SKV_ERR_UNSUPPORTED: valid arguments outside what this library implements";
    case SKV_ERR_WORKSPACE_TOO_SMALL: return "SKV_ERR_WORKSPACE_TOO_SMALL: workspace smaller than the size query";
    case SKV_ERR_CUDA: return "SKV_ERR_CUDA: a CUDA call failed (see skv_last_cuda_error)";
  }
  return "unknown skv_status";
}

int skv_last_cuda_error(void) { return g_last_cuda_error; }

const char* skv_version(void) { return "0.2.0"; }

skv_status skv_exp2_fma(const float* x, float* y, int64_t n, skv_stream_t stream) {
  if (n < 0 || (n > 0 && (x == nullptr || y == nullptr))) return SKV_ERR_INVALID_ARG;
  return cuda_status(skv::launch_exp2_fma(x, y, n, stream));
}

uint64_t skv_launch_count(void) { return skv::launch_count(); }

skv_status skv_device_error(int* code) {
  if (code == nullptr) return SKV_ERR_INVALID_ARG;
  return cuda_status(skv::read_and_clear_device_error(code));
}

// ------------------------------------------------------------------ planning

skv_status attn_splitkv_plan(int B, int Hq, int Hkv, int Lq, int n, int D, int num_sms, int requested_splits,
                             int* num_splits, int32_t* bounds) {
  if (num_splits == nullptr || B < 1 || Hq < 1 || Hkv < 1 || Lq < 1 || n < 0 || D < 1 || Hq % Hkv != 0)
    return SKV_ERR_INVALID_ARG;
  if (requested_splits < 0 || requested_splits > skv::kSplitMax) return SKV_ERR_INVALID_ARG;
  int s;
  if (requested_splits > 0) {
    s = requested_splits;
  } else {
    if (num_sms < 1) return SKV_ERR_INVALID_ARG;
    const int64_t G = Hq / Hkv;
    const int64_t row_groups = skv::ceil_div64(G * Lq, skv::kDecodeRowsPerCta);
    const int64_t units = static_cast<int64_t>(B) * Hkv * row_groups;
    const int64_t num = D > 128 ? skv::kCtasPerSmD256Num : skv::kCtasPerSmNum;
    const int64_t den = D > 128 ? skv::kCtasPerSmD256Den : skv::kCtasPerSmDen;
    const int64_t target = skv::ceil_div64(static_cast<int64_t>(num_sms) * num, den);
    int64_t ss = std::max<int64_t>(1, skv::ceil_div64(target, units));
    ss = std::min<int64_t>(ss, std::max<int64_t>(1, skv::ceil_div64(n, skv::kSplitMinKeys)));
    ss = std::min<int64_t>(ss, skv::kSplitMax);
    if (n > 0) {
      const int64_t C = skv::ceil_div64(skv::ceil_div64(n, ss), skv::kSplitAlign) * skv::kSplitAlign;
      ss = skv::ceil_div64(n, C);
    }
    s = static_cast<int>(std::max<int64_t>(ss, 1));
  }
  *num_splits = s;
  if (bounds != nullptr) {
    if (n == 0) {
      for (int i = 0; i <= s; ++i) bounds[i] = 0;
    } else {
      const int64_t C = skv::ceil_div64(skv::ceil_div64(n, s), skv::kSplitAlign) * skv::kSplitAlign;
      for (int i = 0; i <= s; ++i) bounds[i] = static_cast<int32_t>(std::min<int64_t>(i * C, n));
    }
  }
  return SKV_OK;
}

size_t attn_splitkv_workspace(int B, int Hq, int Lq, int D, int num_splits) {
  if (B < 1 || Hq < 1 || Lq < 1 || D < 1 || num_splits < 1) return 0;
  return decode_workspace(B, Hq, Lq, D, num_splits);
}

skv_status attn_varlen_plan(const int32_t* cu_q, const int32_t* cu_k, int B, int Hq, int D, int32_t* order,
                            int32_t* offsets) {
  if (cu_q == nullptr || cu_k == nullptr || order == nullptr || offsets == nullptr || B < 1 || Hq < 1 || D < 1)
    return SKV_ERR_INVALID_ARG;
  const int rows = skv::prefill_rows_per_cta(D);
  for (int b = 0; b < B; ++b)
    if (cu_q[b + 1] < cu_q[b] || cu_k[b + 1] < cu_k[b]) return SKV_ERR_INVALID_ARG;
  std::vector<int> idx(B);
  for (int b = 0; b < B; ++b) idx[b] = b;
  std::stable_sort(idx.begin(), idx.end(), [&](int x, int y) {
    return (cu_k[x + 1] - cu_k[x]) > (cu_k[y + 1] - cu_k[y]);
  });
  int64_t run = 0;
  for (int i = 0; i < B; ++i) {
    order[i] = idx[i];
    offsets[i] = static_cast<int32_t>(run);
    const int64_t lq = cu_q[idx[i] + 1] - cu_q[idx[i]];
    run += static_cast<int64_t>(Hq) * skv::ceil_div64(lq, rows);
  }
  offsets[B] = static_cast<int32_t>(run);
  return SKV_OK;
}

// ------------------------------------------------------------------ prefill

size_t attn_fwd_lse_workspace(int B, int Hq, int Hkv, int Sk, int D, skv_dtype dtype, skv_layout layout,
                              int smooth_k) {
  (void)Hq;
  (void)dtype;
  if (B < 1 || Hkv < 1 || Sk < 0 || D < 1 || smooth_k < 0 || smooth_k > 2) return 0;
  if (layout != SKV_HND && layout != SKV_NHD && layout != SKV_TND) return 0;
  return fwd_workspace(B, Hkv, Sk, D, layout, smooth_k).total;
}

namespace {
skv_status fwd_lse_impl(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                        int Sq, int Sk, int D, float scale, skv_dtype dtype, skv_layout layout,
                        const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int max_seqlen_q,
                        int max_seqlen_k, int smooth_k, void* workspace, size_t workspace_bytes,
                        skv_stream_t stream, int causal, int nchunks = 1, const int32_t* kv_bounds = nullptr) {
  // ---- validation (no device work before it passes)
  if (q == nullptr || out == nullptr) return SKV_ERR_INVALID_ARG;
  if ((k == nullptr || v == nullptr) && Sk != 0) return SKV_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return SKV_ERR_INVALID_ARG;
  if (lse != nullptr && !aligned(lse, 4)) return SKV_ERR_INVALID_ARG;
  if (layout != SKV_HND && layout != SKV_NHD && layout != SKV_TND) return SKV_ERR_INVALID_ARG;
  if (dtype != SKV_BF16 && dtype != SKV_FP16 && dtype != SKV_FP32) return SKV_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || D < 1 || Sq < 0 || Sk < 0) return SKV_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SKV_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return SKV_ERR_INVALID_ARG;
  if (smooth_k < 0 || smooth_k > 2) return SKV_ERR_INVALID_ARG;
  const bool varlen = layout == SKV_TND;
  if (varlen) {
    if (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr) return SKV_ERR_INVALID_ARG;
    if (!aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4)) return SKV_ERR_INVALID_ARG;
    if (max_seqlen_q < 0 || max_seqlen_q > Sq || max_seqlen_k < 0 || max_seqlen_k > Sk) return SKV_ERR_INVALID_ARG;
  } else {
    if (cu_seqlens_q != nullptr || cu_seqlens_k != nullptr) return SKV_ERR_INVALID_ARG;
  }
  if (!is_half_type(dtype)) return SKV_ERR_UNSUPPORTED;
  if (D != 64 && D != 128 && D != 256) return SKV_ERR_UNSUPPORTED;
  // TMA extents and int32 coordinates
  const int64_t rows_q = varlen ? Sq : static_cast<int64_t>(Sq);
  if (rows_q > (int64_t(1) << 31) - 512 || Sk > (1 << 30)) return SKV_ERR_UNSUPPORTED;
  if (nchunks < 1 || nchunks > skv::kMaxKvChunks) return SKV_ERR_INVALID_ARG;
  int max_chunk = Sk;
  if (nchunks > 1) {
    if (varlen || causal || kv_bounds == nullptr) return SKV_ERR_INVALID_ARG;
    if (kv_bounds[0] != 0 || kv_bounds[nchunks] != Sk) return SKV_ERR_INVALID_ARG;
    max_chunk = 0;
    for (int c = 0; c < nchunks; ++c) {
      if (kv_bounds[c + 1] < kv_bounds[c]) return SKV_ERR_INVALID_ARG;
      max_chunk = std::max(max_chunk, kv_bounds[c + 1] - kv_bounds[c]);
    }
    // every chunk's partial is one output's worth of rows further
    if (static_cast<int64_t>(nchunks) * B * Hq * skv::ceil_div64(Sq, skv::prefill_rows_per_cta(D)) > 0x7fffffff)
      return SKV_ERR_UNSUPPORTED;
  }
  const FwdWorkspace ws = fwd_workspace(B, Hkv, Sk, D, layout, smooth_k, nchunks);
  if (workspace_bytes < ws.total) return SKV_ERR_WORKSPACE_TOO_SMALL;
  if (ws.total > 0 && (workspace == nullptr || !aligned(workspace, 256))) return SKV_ERR_INVALID_ARG;
  if (Sq == 0) return SKV_OK;  // nothing to compute

  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  skv::PrefillLaunch p;
  std::memset(&p, 0, sizeof(p));
  p.q = q;
  p.k = k;
  p.v = v;
  p.out = out;
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Sq = Sq;
  p.Sk = Sk;
  p.D = D;
  p.max_seqlen_q = max_seqlen_q;
  p.scale = scale;
  p.dt = dtype;
  p.layout = layout;
  p.causal = causal ? 1 : 0;
  p.nchunks = nchunks;
  p.kv_bounds = nchunks > 1 ? kv_bounds : nullptr;
  if (varlen) {
    p.cu_q = cu_seqlens_q;
    p.cu_k = cu_seqlens_k;
    p.order = reinterpret_cast<const int32_t*>(wsb + ws.order);
    p.offsets = reinterpret_cast<const int32_t*>(wsb + ws.offsets);
    int e = skv::launch_varlen_plan(cu_seqlens_q, cu_seqlens_k, B, Hq, skv::prefill_rows_per_cta(D),
                                    reinterpret_cast<int32_t*>(wsb + ws.order),
                                    reinterpret_cast<int32_t*>(wsb + ws.offsets), stream);
    if (e) return cuda_status(e);
  }
  if (smooth_k) {
    float* kmean = reinterpret_cast<float*>(wsb + ws.kmean);
    float* partial = reinterpret_cast<float*>(wsb + ws.partial);
    void* kprime = smooth_k == 2 ? static_cast<void*>(wsb + ws.kprime) : nullptr;
    const int max_len = varlen ? max_seqlen_k : max_chunk;
    int e = skv::launch_smooth_k(k, kprime, kmean, partial, varlen ? cu_seqlens_k : nullptr, B, Hkv, Sk, max_len,
                                 D, dtype, layout, stream, nchunks, nchunks > 1 ? kv_bounds : nullptr);
    if (e) return cuda_status(e);
    if (smooth_k == 1) {
      p.kpartial = partial;   // the prefill kernel sums these into the mean itself
      p.after_kpartial = max_len > 0 ? 1 : 0;  // the column-sum kernel was the last launch
    } else {
      p.kmean = kmean;
      p.k = kprime;
    }
    p.shift_logits = smooth_k == 1 ? 1 : 0;
  }
  return cuda_status(skv::launch_prefill(p, stream));
}
}  // namespace

skv_status attn_fwd_lse(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                        int Sq, int Sk, int D, float scale, skv_dtype dtype, skv_layout layout,
                        const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int max_seqlen_q,
                        int max_seqlen_k, int smooth_k, void* workspace, size_t workspace_bytes,
                        skv_stream_t stream) {
  return fwd_lse_impl(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, dtype, layout, cu_seqlens_q, cu_seqlens_k,
                      max_seqlen_q, max_seqlen_k, smooth_k, workspace, workspace_bytes, stream, 0);
}

skv_status attn_fwd_lse_causal(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                               int Hkv, int Sq, int Sk, int D, float scale, skv_dtype dtype, skv_layout layout,
                               const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int max_seqlen_q,
                               int max_seqlen_k, int smooth_k, void* workspace, size_t workspace_bytes,
                               skv_stream_t stream) {
  return fwd_lse_impl(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, dtype, layout, cu_seqlens_q, cu_seqlens_k,
                      max_seqlen_q, max_seqlen_k, smooth_k, workspace, workspace_bytes, stream, 1);
}

size_t attn_fwd_lse_chunks_workspace(int B, int Hq, int Hkv, int Sk, int D, skv_dtype dtype, skv_layout layout,
                                     int num_chunks, int smooth_k) {
  (void)Hq;
  (void)dtype;
  if (B < 1 || Hkv < 1 || Sk < 0 || D < 1 || smooth_k < 0 || smooth_k > 2) return 0;
  if (layout != SKV_HND && layout != SKV_NHD) return 0;
  if (num_chunks < 1 || num_chunks > skv::kMaxKvChunks) return 0;
  return fwd_workspace(B, Hkv, Sk, D, layout, smooth_k, num_chunks).total;
}

skv_status attn_fwd_lse_chunks(const void* q, const void* k, const void* v, void* out_parts, float* lse_parts, int B,
                               int Hq, int Hkv, int Sq, int Sk, int D, float scale, skv_dtype dtype,
                               skv_layout layout, int num_chunks, const int32_t* chunk_bounds, int smooth_k,
                               void* workspace, size_t workspace_bytes, skv_stream_t stream) {
  if (layout != SKV_HND && layout != SKV_NHD) return SKV_ERR_INVALID_ARG;
  if (num_chunks < 1 || num_chunks > skv::kMaxKvChunks || chunk_bounds == nullptr) return SKV_ERR_INVALID_ARG;
  if (chunk_bounds[0] != 0 || chunk_bounds[num_chunks] != Sk) return SKV_ERR_INVALID_ARG;
  for (int c = 0; c < num_chunks; ++c)
    if (chunk_bounds[c + 1] < chunk_bounds[c]) return SKV_ERR_INVALID_ARG;
  return fwd_lse_impl(q, k, v, out_parts, lse_parts, B, Hq, Hkv, Sq, Sk, D, scale, dtype, layout, nullptr, nullptr, 0,
                      0, smooth_k, workspace, workspace_bytes, stream, 0, num_chunks, chunk_bounds);
}

// ------------------------------------------------------------------ int8 prefill

namespace {
struct Int8Ws {
  size_t partial = 0, kmean = 0, q8 = 0, k8 = 0, qs = 0, ks = 0, dq = 0, total = 0;
};
Int8Ws int8_ws_layout(int B, int Hq, int Hkv, int Sq, int Sk) {
  Int8Ws w;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += skv::align256(bytes);
    return o;
  };
  const size_t b = static_cast<size_t>(B);
  w.partial = take(static_cast<size_t>((Sk + 255) / 256) * b * Hkv * 128 * 4);
  w.kmean = take(b * Hkv * 128 * 4);
  w.q8 = take(b * Hq * static_cast<size_t>(Sq) * 128);
  w.k8 = take(b * Hkv * static_cast<size_t>(Sk) * 128);
  w.qs = take(b * Hq * static_cast<size_t>((Sq + 127) / 128) * 4);
  w.ks = take(b * Hkv * static_cast<size_t>((Sk + 127) / 128) * 4);
  w.dq = take(b * Hq * static_cast<size_t>(Sq) * 4);
  w.total = off;
  return w;
}
}  // namespace

size_t attn_fwd_lse_int8_workspace(int B, int Hq, int Hkv, int Sq, int Sk, int D) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 0 || Sk < 0 || D != 128) return 0;
  return int8_ws_layout(B, Hq, Hkv, Sq, Sk).total;
}

skv_status attn_fwd_lse_int8(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                             int Hkv, int Sq, int Sk, int D, float scale, skv_dtype dtype, int causal,
                             void* workspace, size_t workspace_bytes, skv_stream_t stream) {
  if (q == nullptr || out == nullptr) return SKV_ERR_INVALID_ARG;
  if ((k == nullptr || v == nullptr) && Sk != 0) return SKV_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return SKV_ERR_INVALID_ARG;
  if (lse != nullptr && !aligned(lse, 4)) return SKV_ERR_INVALID_ARG;
  if (dtype != SKV_BF16 && dtype != SKV_FP16 && dtype != SKV_FP32) return SKV_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || D < 1 || Sq < 0 || Sk < 0 || Hq % Hkv != 0) return SKV_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return SKV_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SKV_ERR_INVALID_ARG;
  if (!is_half_type(dtype) || D != 128) return SKV_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * Hq > 65535) return SKV_ERR_UNSUPPORTED;  // grid.y of the code kernels
  if (static_cast<int64_t>(B) * Hq * skv::ceil_div64(Sq, skv::kPrefillRowsPerCta) > 0x7fffffff)
    return SKV_ERR_UNSUPPORTED;
  if (Sq == 0) return SKV_OK;
  if (Sk == 0) {  // no keys: O = 0, LSE = -inf, as the 16-bit path writes them
    return causal ? attn_fwd_lse_causal(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, dtype, SKV_HND, nullptr,
                                        nullptr, 0, 0, 0, nullptr, 0, stream)
                  : attn_fwd_lse(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, dtype, SKV_HND, nullptr, nullptr,
                                 0, 0, 0, nullptr, 0, stream);
  }
  const Int8Ws w = int8_ws_layout(B, Hq, Hkv, Sq, Sk);
  if (workspace_bytes < w.total) return SKV_ERR_WORKSPACE_TOO_SMALL;
  if (workspace == nullptr || !aligned(workspace, 256)) return SKV_ERR_INVALID_ARG;
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  skv::Int8PrefillLaunch p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.out = out;
  p.lse = lse;
  p.kpartial = reinterpret_cast<float*>(wsb + w.partial);
  p.kmean = reinterpret_cast<float*>(wsb + w.kmean);
  p.q8 = reinterpret_cast<int8_t*>(wsb + w.q8);
  p.k8 = reinterpret_cast<int8_t*>(wsb + w.k8);
  p.qscale = reinterpret_cast<float*>(wsb + w.qs);
  p.kscale = reinterpret_cast<float*>(wsb + w.ks);
  p.dq = reinterpret_cast<float*>(wsb + w.dq);
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Sq = Sq;
  p.Sk = Sk;
  p.scale = scale;
  p.dt = dtype;
  p.causal = causal;
  return cuda_status(skv::launch_prefill_int8(p, stream));
}

// ------------------------------------------------------------------ decode

namespace {
skv_status decode_impl(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                       int Lq, int Lkv, int D, float scale, skv_dtype dtype, const int32_t* kv_len, int num_splits,
                       void* workspace, size_t workspace_bytes, skv_stream_t stream, bool in_launch_merge,
                       int causal) {
  if (q == nullptr || out == nullptr) return SKV_ERR_INVALID_ARG;
  if ((k == nullptr || v == nullptr) && Lkv != 0) return SKV_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return SKV_ERR_INVALID_ARG;
  if (lse != nullptr && !aligned(lse, 4)) return SKV_ERR_INVALID_ARG;
  if (kv_len != nullptr && !aligned(kv_len, 4)) return SKV_ERR_INVALID_ARG;
  if (dtype != SKV_BF16 && dtype != SKV_FP16 && dtype != SKV_FP32) return SKV_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Lq < 1 || Lkv < 0 || D < 1 || Hq % Hkv != 0) return SKV_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return SKV_ERR_INVALID_ARG;
  if (num_splits < 0 || num_splits > skv::kSplitMax) return SKV_ERR_INVALID_ARG;
  if (!is_half_type(dtype)) return SKV_ERR_UNSUPPORTED;
  if (D != 64 && D != 128 && D != 256) return SKV_ERR_UNSUPPORTED;
  const int64_t G = Hq / Hkv;
  const int64_t row_groups = skv::ceil_div64(G * Lq, skv::kDecodeRowsPerCta);
  if (static_cast<int64_t>(B) * Hkv * row_groups > 65535) return SKV_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * Hkv * Lkv > (int64_t(1) << 31) - 1) return SKV_ERR_UNSUPPORTED;
  int splits = num_splits;
  if (splits == 0) {
    const int sms = skv::sm_count();
    if (sms <= 0) return cuda_status(cudaErrorNoDevice);
    skv_status s = attn_splitkv_plan(B, Hq, Hkv, Lq, Lkv, D, sms, 0, &splits, nullptr);
    if (s != SKV_OK) return s;
  }
  const size_t need = decode_workspace(B, Hq, Lq, D, splits);
  if (workspace_bytes < need) return SKV_ERR_WORKSPACE_TOO_SMALL;
  if (need > 0 && (workspace == nullptr || !aligned(workspace, 256))) return SKV_ERR_INVALID_ARG;
  float* part_o = nullptr;
  float* part_lse = nullptr;
  int* counters = nullptr;
  if (splits > 1) {
    const DecodeWs w = decode_ws_layout(B, Hq, Lq, D, splits);
    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    part_o = reinterpret_cast<float*>(wsb + w.part_o);
    part_lse = reinterpret_cast<float*>(wsb + w.part_lse);
    if (in_launch_merge) counters = reinterpret_cast<int*>(wsb + w.counters);
  }
  int e = skv::launch_decode(q, k, v, out, lse, part_o, part_lse, counters, kv_len, B, Hq, Hkv, Lq, Lkv, D, scale,
                             dtype, splits, causal, stream);
  if (e) return cuda_status(e);
  if (splits > 1 && !in_launch_merge) {
    const int64_t rows = static_cast<int64_t>(B) * Hq * Lq;
    e = skv::launch_merge_state(part_o, part_lse, out, lse, splits, 1, 1, static_cast<int>(rows), D, 0, SKV_FP32,
                                dtype, rows * D, rows, stream);
    if (e) return cuda_status(e);
  }
  return SKV_OK;
}

}  // namespace

skv_status attn_splitkv_decode(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                               int Hkv, int Lq, int Lkv, int D, float scale, skv_dtype dtype, const int32_t* kv_len,
                               int num_splits, void* workspace, size_t workspace_bytes, skv_stream_t stream) {
  return decode_impl(q, k, v, out, lse, B, Hq, Hkv, Lq, Lkv, D, scale, dtype, kv_len, num_splits, workspace,
                     workspace_bytes, stream, /*in_launch_merge=*/false, /*causal=*/0);
}

skv_status attn_splitkv_decode_fused(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                                     int Hq, int Hkv, int Lq, int Lkv, int D, float scale, skv_dtype dtype,
                                     const int32_t* kv_len, int num_splits, void* workspace, size_t workspace_bytes,
                                     skv_stream_t stream) {
  return decode_impl(q, k, v, out, lse, B, Hq, Hkv, Lq, Lkv, D, scale, dtype, kv_len, num_splits, workspace,
                     workspace_bytes, stream, /*in_launch_merge=*/true, /*causal=*/0);
}

skv_status attn_splitkv_decode_causal(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                                      int Hq, int Hkv, int Lq, int Lkv, int D, float scale, skv_dtype dtype,
                                      const int32_t* kv_len, int num_splits, void* workspace, size_t workspace_bytes,
                                      skv_stream_t stream) {
  return decode_impl(q, k, v, out, lse, B, Hq, Hkv, Lq, Lkv, D, scale, dtype, kv_len, num_splits, workspace,
                     workspace_bytes, stream, /*in_launch_merge=*/false, /*causal=*/1);
}

skv_status attn_splitkv_workspace_init(void* workspace, size_t workspace_bytes, skv_stream_t stream) {
  if (workspace_bytes == 0) return SKV_OK;
  if (workspace == nullptr) return SKV_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(workspace, 0, workspace_bytes, reinterpret_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------------ merge

skv_status merge_state(const void* o_parts, const float* lse_parts, void* out, float* lse, int P, int B, int H, int S,
                       int D, skv_layout layout, skv_dtype parts_dtype, skv_dtype out_dtype, int64_t part_stride_o,
                       int64_t part_stride_lse, skv_stream_t stream) {
  if (o_parts == nullptr || lse_parts == nullptr || out == nullptr) return SKV_ERR_INVALID_ARG;
  if (!aligned(o_parts, 16) || !aligned(out, 16) || !aligned(lse_parts, 4)) return SKV_ERR_INVALID_ARG;
  if (lse != nullptr && !aligned(lse, 4)) return SKV_ERR_INVALID_ARG;
  if (P < 1 || B < 0 || H < 0 || S < 0 || D < 8 || D % 8 != 0) return SKV_ERR_INVALID_ARG;
  if (layout != SKV_HND && layout != SKV_NHD && layout != SKV_TND) return SKV_ERR_INVALID_ARG;
  auto ok_dt = [](skv_dtype d) { return d == SKV_BF16 || d == SKV_FP16 || d == SKV_FP32; };
  if (!ok_dt(parts_dtype) || !ok_dt(out_dtype)) return SKV_ERR_INVALID_ARG;
  const int64_t rows = static_cast<int64_t>(B) * H * S;
  const int64_t so = part_stride_o == 0 ? rows * D : part_stride_o;
  const int64_t sl = part_stride_lse == 0 ? rows : part_stride_lse;
  if (P > 1 && (so < rows * D || sl < rows)) return SKV_ERR_INVALID_ARG;
  if (so % 8 != 0) return SKV_ERR_INVALID_ARG;
  if (rows == 0) return SKV_OK;
  return cuda_status(skv::launch_merge_state(o_parts, lse_parts, out, lse, P, B, H, S, D, layout == SKV_HND ? 0 : 1,
                                             parts_dtype, out_dtype, so, sl, stream));
}

}  // extern "C"
