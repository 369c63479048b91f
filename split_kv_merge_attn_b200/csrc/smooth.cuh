// smooth_k prepass: mean of K over the call's own KV range, per (batch or
// sequence, kv head, channel), in fp32 -- the "k.mean(dim=2)" of the ARK
// return_lse issue's repro (HND: mean over the keys) -- and, in the
// materialising mode, K' = K - mean rounded to the input type.
//
// Deterministic two-pass reduction: pass 1 writes one fp32 partial column sum
// per 256-key chunk, pass 2 adds the chunks in order and divides by the range
// length.  Bandwidth bound (one read of K; a second read plus a write of K'
// when it is materialised).
#pragma once

#include "skv_device.cuh"

namespace skv {

constexpr int kSmoothChunk = 256;

// A "range" is the key range one mean is taken over: a batch entry (dense), a
// varlen sequence, or, in a multi-chunk dense call, KV chunk c of batch entry
// b (range index b * nranges_per_batch + c, keys [kvb[c], kvb[c+1])).
struct SmoothArgs {
  const void* k;
  void* k_out;          // K' (materialising mode) or null
  float* partial;       // [nchunks, Bseq, Hkv, D]
  float* kmean;         // [Bseq, Hkv, D]
  const int* cu_k;      // varlen offsets or null
  int Bseq, Hkv, Sk, D; // Bseq: number of ranges
  int nchunks;          // 256-key chunks of the longest range
  int layout;           // 0 HND, 1 NHD, 2 TND
  int kv_ranges;        // dense: key ranges per batch entry (1 = all Sk keys)
  int kvb[kMaxKvChunks + 1];
};

// element offset of key s (inside its range) of kv head hkv
__device__ __forceinline__ int64_t smooth_row_off(const SmoothArgs& a, int r, int hkv, int s) {
  if (a.layout == 2) return (static_cast<int64_t>(a.cu_k[r] + s) * a.Hkv + hkv) * a.D;
  const int b = r / a.kv_ranges;
  const int key = a.kvb[r - b * a.kv_ranges] + s;
  if (a.layout == 0) return ((static_cast<int64_t>(b) * a.Hkv + hkv) * a.Sk + key) * a.D;
  return ((static_cast<int64_t>(b) * a.Sk + key) * a.Hkv + hkv) * a.D;
}

__device__ __forceinline__ int smooth_len(const SmoothArgs& a, int r) {
  if (a.layout == 2) return a.cu_k[r + 1] - a.cu_k[r];
  const int c = r % a.kv_ranges;
  return a.kvb[c + 1] - a.kvb[c];
}

// grid (nchunks, Bseq, Hkv), 256 threads: (D/8) column vectors x (256/(D/8)) row lanes.
// Every thread issues its row loads in batches of 16 before summing them (all
// of its rows of the chunk at D = 128: enough bytes in flight to stream K).
template <typename T>
__global__ void __launch_bounds__(256) kmean_partial_kernel(SmoothArgs a) {
  const int c = blockIdx.x, b = blockIdx.y, hkv = blockIdx.z;
  const int len = smooth_len(a, b);
  const int vpr = a.D / 8;
  const int lanes = 256 / vpr;
  const int cv = threadIdx.x % vpr, rl = threadIdx.x / vpr;
  const int s0 = c * kSmoothChunk, s1 = min(len, s0 + kSmoothChunk);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const T* k = static_cast<const T*>(a.k);
  // rows of this thread: s0 + rl + i * lanes; loads issued in batches of 16
  constexpr int kBatch = 16;
  for (int i0 = 0; i0 * lanes < kSmoothChunk; i0 += kBatch) {
    uint4 u[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int s = s0 + rl + (i0 + i) * lanes;
      u[i] = (s < s1) ? __ldg(reinterpret_cast<const uint4*>(k + smooth_row_off(a, b, hkv, s) + cv * 8))
                      : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = unpack2<T>(w[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
  }
  __shared__ float red[256 * 8];
#pragma unroll
  for (int e = 0; e < 8; ++e) red[(rl * vpr + cv) * 8 + e] = acc[e];
  __syncthreads();
  if (rl == 0) {
    for (int r = 1; r < lanes; ++r)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += red[(r * vpr + cv) * 8 + e];
    float* dst = a.partial + ((static_cast<int64_t>(c) * a.Bseq + b) * a.Hkv + hkv) * a.D + cv * 8;
#pragma unroll
    for (int e = 0; e < 8; ++e) dst[e] = acc[e];
  }
}

// grid (Bseq * Hkv), D threads
__global__ void kmean_finalize_kernel(SmoothArgs a) {
  const int bh = blockIdx.x;
  const int b = bh / a.Hkv;
  const int d = threadIdx.x;
  const int len = smooth_len(a, b);
  const int nch = (len + kSmoothChunk - 1) / kSmoothChunk;
  float s = 0.f;
  for (int c = 0; c < nch; ++c) s += a.partial[(static_cast<int64_t>(c) * a.Bseq * a.Hkv + bh) * a.D + d];
  a.kmean[static_cast<int64_t>(bh) * a.D + d] = len > 0 ? s / static_cast<float>(len) : 0.f;
}

// K' = K - mean, rounded to T; grid (nchunks, Bseq, Hkv), 256 threads
template <typename T>
__global__ void __launch_bounds__(256) ksmooth_write_kernel(SmoothArgs a) {
  const int c = blockIdx.x, b = blockIdx.y, hkv = blockIdx.z;
  const int len = smooth_len(a, b);
  const int vpr = a.D / 8;
  const int lanes = 256 / vpr;
  const int cv = threadIdx.x % vpr, rl = threadIdx.x / vpr;
  const int s0 = c * kSmoothChunk, s1 = min(len, s0 + kSmoothChunk);
  const float* mu = a.kmean + (static_cast<int64_t>(b) * a.Hkv + hkv) * a.D + cv * 8;
  float m[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m[e] = mu[e];
  const T* k = static_cast<const T*>(a.k);
  T* ko = static_cast<T*>(a.k_out);
  for (int s = s0 + rl; s < s1; s += lanes) {
    const int64_t off = smooth_row_off(a, b, hkv, s) + cv * 8;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(k + off));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack2<T>(w[e]);
      o[e] = pack2<T>(f.x - m[2 * e], f.y - m[2 * e + 1]);
    }
    *reinterpret_cast<uint4*>(ko + off) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace skv
