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

// row stride (elements) between consecutive keys of one range and kv head
__device__ __forceinline__ int64_t smooth_row_stride(const SmoothArgs& a) {
  return a.layout == 0 ? a.D : static_cast<int64_t>(a.Hkv) * a.D;
}

// A unit is one 256-key chunk c of range r and kv head hkv: block u of the
// 1-D grid, u = c + nchunks * (r + Bseq * hkv).
struct KmeanUnit {
  int c, r, hkv, s0, s1;
};

__device__ __forceinline__ KmeanUnit kmean_unit(const SmoothArgs& a, int u) {
  KmeanUnit w;
  w.c = u % a.nchunks;
  w.r = (u / a.nchunks) % a.Bseq;
  w.hkv = u / (a.nchunks * a.Bseq);
  w.s0 = w.c * kSmoothChunk;
  w.s1 = min(smooth_len(a, w.r), w.s0 + kSmoothChunk);
  return w;
}

// Column sums of one unit per CTA, 256 threads: (D/8) column vectors x
// (256/(D/8)) row lanes; thread (cv, rl) sums the 16-byte piece cv of rows
// s0 + rl + i * lanes, loads issued eight at a time.  The unit's base address
// is computed once and each further row is one pointer step, and 64 registers
// allow four CTAs per SM: this streams K at the rate of a plain read of it
// (row addresses recomputed per load made the kernel issue bound at a third of
// that).  The sums over the row lanes go through warp shuffles (lanes D/8 apart
// hold the same columns), then the 8 warps' sums through shared memory, added
// in warp order, so each partial is the same fp32 sum on every run.
constexpr int kKmeanBatch = 8;

template <typename T>
__global__ void __launch_bounds__(256, 4) kmean_partial_kernel(SmoothArgs a) {
  // launched as a programmatic dependent of the kernel before it (which may
  // have written K): wait for it before any load.  Then a prefill launched as
  // this grid's programmatic dependent may start: it reads these sums only
  // after its own griddepcontrol.wait, and its inputs were complete before
  // this wait returned.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int vpr = a.D / 8, lanes = 256 / vpr;
  const int cv = tid % vpr, rl = tid / vpr;
  const int rpt = kSmoothChunk / lanes;  // rows of the unit per thread: 8, 16, 32
  const KmeanUnit w = kmean_unit(a, blockIdx.x);
  const int nv = w.s1 - w.s0;            // rows of the unit (none past the range's end)
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (nv > 0) {
    const int64_t rs = smooth_row_stride(a);
    const int64_t step = lanes * rs;
    const T* p = static_cast<const T*>(a.k) + smooth_row_off(a, w.r, w.hkv, w.s0) + rl * rs + cv * 8;
    for (int i0 = 0; i0 < rpt; i0 += kKmeanBatch) {
      uint4 u[kKmeanBatch];
#pragma unroll
      for (int i = 0; i < kKmeanBatch; ++i)
        u[i] = (rl + (i0 + i) * lanes < nv) ? __ldg(reinterpret_cast<const uint4*>(p + (i0 + i) * step))
                                             : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int i = 0; i < kKmeanBatch; ++i) {
        const uint32_t x[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack2<T>(x[e]);
          acc[2 * e] += f.x;
          acc[2 * e + 1] += f.y;
        }
      }
    }
  }
  for (int o = vpr; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
  __shared__ float4 red[8][32][2];  // [warp][column vector][8 floats]
  if (lane < vpr) {
    red[warp][lane][0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    red[warp][lane][1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  __syncthreads();
  if (tid < vpr) {
    float4 s0 = red[0][tid][0], s1 = red[0][tid][1];
#pragma unroll
    for (int wi = 1; wi < 8; ++wi) {
      const float4 x0 = red[wi][tid][0], x1 = red[wi][tid][1];
      s0.x += x0.x; s0.y += x0.y; s0.z += x0.z; s0.w += x0.w;
      s1.x += x1.x; s1.y += x1.y; s1.z += x1.z; s1.w += x1.w;
    }
    float4* dst = reinterpret_cast<float4*>(
        a.partial + ((static_cast<int64_t>(w.c) * a.Bseq + w.r) * a.Hkv + w.hkv) * a.D + tid * 8);
    dst[0] = s0;
    dst[1] = s1;
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

// K' = K - mean, rounded to T; one unit per CTA (as the column sums), 256 threads
template <typename T>
__global__ void __launch_bounds__(256) ksmooth_write_kernel(SmoothArgs a) {
  const KmeanUnit w = kmean_unit(a, blockIdx.x);
  const int vpr = a.D / 8;
  const int lanes = 256 / vpr;
  const int cv = threadIdx.x % vpr, rl = threadIdx.x / vpr;
  if (w.s1 <= w.s0) return;
  const float* mu = a.kmean + (static_cast<int64_t>(w.r) * a.Hkv + w.hkv) * a.D + cv * 8;
  float m[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m[e] = mu[e];
  const int64_t rs = smooth_row_stride(a);
  const int64_t base = smooth_row_off(a, w.r, w.hkv, w.s0) + cv * 8;
  const T* k = static_cast<const T*>(a.k);
  T* ko = static_cast<T*>(a.k_out);
  for (int s = w.s0 + rl; s < w.s1; s += lanes) {
    const int64_t off = base + (s - w.s0) * rs;
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
