// merge_state kernel: combine P partial (O, LSE) results of disjoint KV ranges.
//
// Per row: M = max_p L_p; w_p = 2^(L_p - M) (0 for an empty part, which is then
// not read at all); O = sum_p w_p O_p / sum_p w_p; LSE = M + log2(sum_p w_p);
// all parts empty -> O = 0, LSE = -inf.  This is the per-hop merge of ring
// attention (merge_state_v2 in the SGLang sgl_kernel::fwd PR thread) and the
// cross-split reduce of the ExecuTorch split-K PR.  That PR's review measured a
// reduce parallel over rows only, with two exponentials on the loop-carried
// chain, as latency bound; here every thread owns one 16-byte slice of one
// row (parallel over rows x D) and requests all of its parts at once.
#pragma once

#include <type_traits>

#include "skv_device.cuh"

namespace skv {

template <typename T>
struct Vec8;  // eight elements of T loaded / stored as one 16- or 32-byte unit

template <>
struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&x)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&x)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
  }
};

template <typename H>
struct Vec8Half {
  static __device__ __forceinline__ void load(const H* p, float (&x)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    float2 f;
    f = unpack2<H>(u.x); x[0] = f.x; x[1] = f.y;
    f = unpack2<H>(u.y); x[2] = f.x; x[3] = f.y;
    f = unpack2<H>(u.z); x[4] = f.x; x[5] = f.y;
    f = unpack2<H>(u.w); x[6] = f.x; x[7] = f.y;
  }
  static __device__ __forceinline__ void store(H* p, const float (&x)[8]) {
    uint4 u;
    u.x = pack2<H>(x[0], x[1]);
    u.y = pack2<H>(x[2], x[3]);
    u.z = pack2<H>(x[4], x[5]);
    u.w = pack2<H>(x[6], x[7]);
    *reinterpret_cast<uint4*>(p) = u;
  }
};
template <>
struct Vec8<__nv_bfloat16> : Vec8Half<__nv_bfloat16> {};
template <>
struct Vec8<__half> : Vec8Half<__half> {};

// Eight elements kept as the raw 16-byte words they were loaded as (one word
// for 16-bit types, two for fp32) until they are used: fewer live registers
// than unpacked floats, so more loads can be in flight per SM.
template <typename T>
struct Raw8 {
  static constexpr int kWords = sizeof(T) == 4 ? 2 : 1;
  uint4 w[kWords];
  __device__ __forceinline__ void load(const T* p) {
#pragma unroll
    for (int i = 0; i < kWords; ++i) w[i] = __ldg(reinterpret_cast<const uint4*>(p) + i);
  }
  __device__ __forceinline__ void unpack(float (&x)[8]) const {
    if constexpr (sizeof(T) == 4) {
      const float* f0 = reinterpret_cast<const float*>(&w[0]);
      const float* f1 = reinterpret_cast<const float*>(&w[1]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[e] = f0[e];
        x[4 + e] = f1[e];
      }
    } else {
      const uint32_t u[4] = {w[0].x, w[0].y, w[0].z, w[0].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = unpack2<T>(u[e]);
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
      }
    }
  }
};

template <typename T>
__device__ __forceinline__ void store1(T* p, float x) {
  if constexpr (std::is_same<T, float>::value) *p = x;
  else if constexpr (std::is_same<T, __half>::value) *p = __float2half_rn(x);
  else *p = __float2bfloat16_rn(x);
}

struct MergeArgs {
  const void* o_parts;
  const float* lse_parts;
  void* out;
  float* lse;
  int P, B, H, S, D;
  int layout_bsh;          // 1: O rows ordered (b, s, h) (NHD/TND); 0: (b, h, s) (HND)
  int64_t part_stride_o;   // elements
  int64_t part_stride_lse; // elements
  int64_t n_vec;           // rows * D / 8
};

// Many-row merge (the ring / chunk merge) for D / 8 = VPR slices per row: one
// thread per kSlices adjacent 8-element slices of a row (kSlices * 16 or 32
// contiguous bytes per part); the LSEs and O slices of up to kBatch parts are
// all requested before any is used (one memory round trip per batch), then
// the batch's max is taken first and each part gets one approximate exp2 (no
// running-max chain inside a batch).  Two slices per thread halve the
// per-byte share of that weight arithmetic, which every thread of a row
// repeats, and double the bytes each thread has in flight.  Row arithmetic is
// 32-bit where the slice count allows it.  A part whose LSE is -inf carries no
// weight and its O slot (which may hold anything) is not used.
#ifndef SKV_MERGE_SLICES
#define SKV_MERGE_SLICES 2
#endif
template <typename TI, typename TO, int VPR, bool kWide, int kSlices = SKV_MERGE_SLICES>
__global__ void __launch_bounds__(256) merge_rows_kernel(MergeArgs a) {
  // launched as a programmatic dependent of the kernel before it (which may
  // have produced the parts): wait for it before any load
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  static_assert(VPR % kSlices == 0, "slices of a row split evenly over its threads");
  constexpr int kBatch = 4;
  constexpr int kTpr = VPR / kSlices;  // threads per row
  const TI* __restrict__ op = static_cast<const TI*>(a.o_parts);
  const float* __restrict__ lp = a.lse_parts;
  TO* __restrict__ out = static_cast<TO*>(a.out);
  using Idx = typename std::conditional<kWide, int64_t, int32_t>::type;
  const Idx g = static_cast<Idx>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= a.n_vec / kSlices) return;
  const Idx row = g / kTpr;
  const int c = static_cast<int>(g % kTpr) * kSlices;  // first slice of this thread
  Idx lrow = row;
  if (a.layout_bsh) {
    const Idx h = row % a.H;
    const Idx bs = row / a.H;
    lrow = (bs / a.S * a.H + h) * a.S + bs % a.S;
  }
  const TI* base = op + static_cast<int64_t>(row) * a.D + c * 8;
  const float* lbase = lp + lrow;
  float m = -INFINITY, W = 0.f;
  float acc[kSlices][8];
#pragma unroll
  for (int k = 0; k < kSlices; ++k)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[k][e] = 0.f;
  for (int p0 = 0; p0 < a.P; p0 += kBatch) {
    float L[kBatch];
    Raw8<TI> x[kBatch][kSlices];
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      const int p = p0 + r;
      L[r] = (p < a.P) ? __ldg(lbase + p * a.part_stride_lse) : -INFINITY;
      if (p < a.P)
#pragma unroll
        for (int k = 0; k < kSlices; ++k) x[r][k].load(base + p * a.part_stride_o + k * 8);
    }
    float mb = m;
#pragma unroll
    for (int r = 0; r < kBatch; ++r) mb = fmaxf(mb, L[r]);
    if (mb == -INFINITY) continue;          // every part so far is empty
    const float sc = ex2_approx(m - mb);    // 0 while m is -inf
    W *= sc;
#pragma unroll
    for (int k = 0; k < kSlices; ++k)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[k][e] *= sc;
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      if (L[r] == -INFINITY) continue;      // an empty part: its O slot is not used
      const float w = ex2_approx(L[r] - mb);
#pragma unroll
      for (int k = 0; k < kSlices; ++k) {
        float xf[8];
        x[r][k].unpack(xf);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[k][e] = fmaf(w, xf[e], acc[k][e]);
      }
      W += w;
    }
    m = mb;
  }
  const float inv = (m != -INFINITY && W > 0.f) ? 1.0f / W : 0.f;
#pragma unroll
  for (int k = 0; k < kSlices; ++k) {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[k][e] *= inv;
    Vec8<TO>::store(out + static_cast<int64_t>(row) * a.D + (c + k) * 8, acc[k]);
  }
  if (c == 0 && a.lse != nullptr) a.lse[lrow] = (m == -INFINITY) ? -INFINITY : m + __log2f(W);
}

// Generic many-row merge (any D that is a multiple of 8): one thread per
// 8-element slice of one row; the loads of up to kBatch parts (LSE and O
// slice) are issued together and merged with a running max, so a thread waits
// for memory once per kBatch parts, not once per part.
template <typename TI, typename TO>
__global__ void __launch_bounds__(256) merge_state_kernel(MergeArgs a) {
  // launched as a programmatic dependent of the kernel before it (which may
  // have produced the parts): wait for it before any load
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int kBatch = 4;
  const TI* __restrict__ op = static_cast<const TI*>(a.o_parts);
  const float* __restrict__ lp = a.lse_parts;
  TO* __restrict__ out = static_cast<TO*>(a.out);
  const int vpr = a.D >> 3;  // 8-element vectors per row
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= a.n_vec) return;
  const int64_t row = g / vpr;          // row in O's memory order
  const int c = static_cast<int>(g - row * vpr);
  int64_t lrow = row;                   // row in the [B, H, S] LSE order
  if (a.layout_bsh) {
    const int h = static_cast<int>(row % a.H);
    const int64_t bs = row / a.H;
    const int s = static_cast<int>(bs % a.S);
    const int64_t b = bs / a.S;
    lrow = (b * a.H + h) * a.S + s;
  }
  const TI* base = op + row * a.D + c * 8;
  float m = -INFINITY, W = 0.f;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int p0 = 0; p0 < a.P; p0 += kBatch) {
    float L[kBatch];
    Raw8<TI> x[kBatch];
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      const int p = p0 + r;
      L[r] = (p < a.P) ? __ldg(lp + p * a.part_stride_lse + lrow) : -INFINITY;
      if (p < a.P) x[r].load(base + p * a.part_stride_o);
    }
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      if (L[r] == -INFINITY) continue;   // an empty part carries no weight; its O slot is not used
      const float mn = fmaxf(m, L[r]);
      const float sc = exp2f(m - mn);    // 0 while m is -inf
      const float w = exp2f(L[r] - mn);
      float xf[8];
      x[r].unpack(xf);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, xf[e], acc[e] * sc);
      W = W * sc + w;
      m = mn;
    }
  }
  const float inv = (m != -INFINITY && W > 0.f) ? 1.0f / W : 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] *= inv;
  Vec8<TO>::store(out + row * a.D + c * 8, acc);
  if (c == 0 && a.lse != nullptr) a.lse[lrow] = (m == -INFINITY) ? -INFINITY : m + log2f(W);
}

// Variant for few rows and many parts (the cross-split reduce of a decode:
// tens of rows, tens of splits).  One CTA per row; its 256 threads split into
// (D/8) column slices x (256 / (D/8)) part lanes.  Each thread issues the
// loads of all its parts (LSE and O slice) at once and merges them with a
// running max of its own; the part lanes are then rescaled to the row max and
// summed through shared memory -- one round trip to memory instead of one per
// part.  A part of LSE -inf contributes nothing (its O slot is never used in
// arithmetic).  Launched as a programmatic dependent of the kernel before it
// (the decode's split kernel, or whatever wrote the parts), it waits for that
// grid's results with griddepcontrol.wait.
template <typename TI, typename TO>
__global__ void __launch_bounds__(256) merge_state_parts_kernel(MergeArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the next kernel on the stream, if launched as a programmatic dependent
  // (the next decode's split kernel), may become resident meanwhile
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const TI* __restrict__ op = static_cast<const TI*>(a.o_parts);
  const float* __restrict__ lp = a.lse_parts;
  TO* __restrict__ out = static_cast<TO*>(a.out);
  const int vpr = a.D >> 3;
  const int lanes = 256 / vpr;
  const int c = threadIdx.x % vpr;
  const int pl = threadIdx.x / vpr;
  const int64_t row = blockIdx.x;
  int64_t lrow = row;
  if (a.layout_bsh) {
    const int h = static_cast<int>(row % a.H);
    const int64_t bs = row / a.H;
    const int s = static_cast<int>(bs % a.S);
    const int64_t b = bs / a.S;
    lrow = (b * a.H + h) * a.S + s;
  }
  __shared__ float red[256 * 8];
  __shared__ float wmax[8];
  __shared__ float wsum[256];
  float m = -INFINITY, W = 0.f;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const TI* base = op + row * a.D + c * 8;
  constexpr int R = 4;
  if (pl < lanes) {
    for (int p0 = pl; p0 < a.P; p0 += R * lanes) {
      float L[R];
      float x[R][8];
#pragma unroll
      for (int r = 0; r < R; ++r) {  // every load of this batch is issued before any use
        const int p = p0 + r * lanes;
        L[r] = (p < a.P) ? __ldg(lp + p * a.part_stride_lse + lrow) : -INFINITY;
        if (p < a.P) Vec8<TI>::load(base + p * a.part_stride_o, x[r]);
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (L[r] == -INFINITY) continue;
        const float mn = fmaxf(m, L[r]);
        const float sc = exp2f(m - mn);  // 0 while m is -inf
        const float w = exp2f(L[r] - mn);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, x[r][e], acc[e] * sc);
        W = W * sc + w;
        m = mn;
      }
    }
  }
  // row max over all threads
  float M = m;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = M;
  __syncthreads();
  M = wmax[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) M = fmaxf(M, wmax[w]);
  const float f = (m == -INFINITY) ? 0.f : exp2f(m - M);
#pragma unroll
  for (int e = 0; e < 8; ++e) red[threadIdx.x * 8 + e] = acc[e] * f;
  wsum[threadIdx.x] = (c == 0) ? W * f : 0.f;
  __syncthreads();
  if (pl == 0) {
    float Wt = 0.f;
    for (int l = 0; l < lanes; ++l) Wt += wsum[l * vpr];
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = 0.f;
    for (int l = 0; l < lanes; ++l)
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] += red[(l * vpr + c) * 8 + e];
    const float inv = (M != -INFINITY && Wt > 0.f) ? 1.0f / Wt : 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] *= inv;
    Vec8<TO>::store(out + row * a.D + c * 8, v);
    if (c == 0 && a.lse != nullptr) a.lse[lrow] = (M == -INFINITY) ? -INFINITY : M + log2f(Wt);
  }
}

// Few rows and many parts with D / 8 = VPR in {8, 16} (instantiable for 32):
// one CTA per row; thread t takes column slice t / LANES and parts t % LANES,
// t % LANES + LANES, ... (LANES = 256 / VPR consecutive threads of one warp
// per slice, so the LANES threads of a slice hold every part once).  A thread
// requests the LSEs and O slices of up to R of its parts at once (one memory
// round trip per batch), weighs them against its own running max (one exp2
// per part, one per batch for the rescale), and the slice's threads then agree
// on the row max and add their weighted sums and weight sums with warp
// shuffles: no shared memory and no block barrier.  A part of LSE -inf has
// weight 0 and its O slot is not used.  Launched as a programmatic dependent
// of the kernel before it, whose results it waits for (griddepcontrol.wait).
template <typename TI, typename TO, int VPR>
__global__ void __launch_bounds__(256) merge_parts_shfl_kernel(MergeArgs a) {
  constexpr int kLanes = 256 / VPR;
  constexpr int R = 4;  // parts per thread in flight
  static_assert(kLanes >= 8 && kLanes <= 32, "one slice's part lanes lie inside one warp");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the next kernel on the stream, if launched as a programmatic dependent
  // (the next decode's split kernel), may become resident meanwhile
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int pl = threadIdx.x % kLanes;
  const int c = threadIdx.x / kLanes;
  const int64_t row = blockIdx.x;
  int64_t lrow = row;
  if (a.layout_bsh) {
    const int h = static_cast<int>(row % a.H);
    const int64_t bs = row / a.H;
    const int s = static_cast<int>(bs % a.S);
    const int64_t b = bs / a.S;
    lrow = (b * a.H + h) * a.S + s;
  }
  const TI* __restrict__ base = static_cast<const TI*>(a.o_parts) + row * a.D + c * 8;
  const float* __restrict__ lb = a.lse_parts + lrow;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float m = -INFINITY, W = 0.f;
  for (int p0 = pl; p0 < a.P; p0 += R * kLanes) {
    float L[R];
    Raw8<TI> x[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {  // every load of the batch is issued before any use
      const int p = p0 + r * kLanes;
      L[r] = (p < a.P) ? __ldg(lb + p * a.part_stride_lse) : -INFINITY;
      if (p < a.P) x[r].load(base + p * a.part_stride_o);
    }
    float bm = m;
#pragma unroll
    for (int r = 0; r < R; ++r) bm = fmaxf(bm, L[r]);
    if (bm == -INFINITY) continue;  // no part with weight yet
    const float sc = (m == -INFINITY) ? 0.f : ex2_approx(m - bm);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] *= sc;
    W *= sc;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (L[r] == -INFINITY) continue;
      const float w = ex2_approx(L[r] - bm);
      float xf[8];
      x[r].unpack(xf);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, xf[e], acc[e]);
      W += w;
    }
    m = bm;
  }
  float M = m;
#pragma unroll
  for (int o = kLanes / 2; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float f = (m == -INFINITY) ? 0.f : ex2_approx(m - M);
  W *= f;
#pragma unroll
  for (int o = kLanes / 2; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
  // reduce-scatter of the 8 sums over the slice's threads: at lane distance
  // 1, 2, 4 each thread keeps one half of what it holds, sends the other half
  // and adds its partner's (4 + 2 + 1 shuffles); then thread pl holds element
  // 4 (pl & 1) + 2 (pl >> 1 & 1) + (pl >> 2 & 1) summed over 8 threads, and the
  // remaining distances (8, 16) add whole values.
  float h4[4];
  {
    const bool up = pl & 1;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float send = up ? acc[e] * f : acc[e + 4] * f;
      const float keep = up ? acc[e + 4] * f : acc[e] * f;
      h4[e] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
    }
  }
  float h2[2];
  {
    const bool up = (pl >> 1) & 1;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float send = up ? h4[e] : h4[e + 2];
      const float keep = up ? h4[e + 2] : h4[e];
      h2[e] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
  }
  float v;
  {
    const bool up = (pl >> 2) & 1;
    const float send = up ? h2[0] : h2[1];
    const float keep = up ? h2[1] : h2[0];
    v = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
#pragma unroll
  for (int o = 8; o < kLanes; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (pl < 8) {
    const int e = 4 * (pl & 1) + 2 * ((pl >> 1) & 1) + ((pl >> 2) & 1);
    const float inv = (M != -INFINITY && W > 0.f) ? 1.0f / W : 0.f;
    store1<TO>(static_cast<TO*>(a.out) + row * a.D + c * 8 + e, v * inv);
    if (c == 0 && pl == 0 && a.lse != nullptr) a.lse[lrow] = (M == -INFINITY) ? -INFINITY : M + __log2f(W);
  }
}

}  // namespace skv
