// merge_state kernel: combine P partial (O, LSE) results of disjoint KV ranges.
//
// Per row: M = max_p L_p; w_p = 2^(L_p - M) (0 for an empty part, which is then
// not read at all); O = sum_p w_p O_p / sum_p w_p; LSE = M + log2(sum_p w_p);
// all parts empty -> O = 0, LSE = -inf.  This is the per-hop merge of ring
// attention (merge_state_v2 in the SGLang sgl_kernel::fwd PR thread) and the
// cross-split reduce of the ExecuTorch split-K PR.  That PR's review measured a
// reduce parallel over rows only, with two exponentials on the loop-carried
// chain, as latency bound; here every thread owns one 16-byte slice of one
// row (parallel over rows x D), the max is a separate first pass over the P
// LSE values, and the weights are independent, so no exponential sits on a
// serial dependency chain.
#pragma once

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

template <typename TI, typename TO>
__global__ void __launch_bounds__(256) merge_state_kernel(MergeArgs a) {
  const TI* __restrict__ op = static_cast<const TI*>(a.o_parts);
  const float* __restrict__ lp = a.lse_parts;
  TO* __restrict__ out = static_cast<TO*>(a.out);
  const int vpr = a.D >> 3;  // 8-element vectors per row
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < a.n_vec; g += stride) {
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
    // pass 1: the max over parts (independent loads)
    float M = -INFINITY;
    for (int p = 0; p < a.P; ++p) M = fmaxf(M, __ldg(lp + p * a.part_stride_lse + lrow));
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    float W = 0.f;
    if (M != -INFINITY) {
      // pass 2: weights and the weighted sum; parts of weight 0 are skipped
      const TI* base = op + row * a.D + c * 8;
      int p = 0;
      for (; p + 2 <= a.P; p += 2) {
        const float w0 = exp2f(__ldg(lp + p * a.part_stride_lse + lrow) - M);
        const float w1 = exp2f(__ldg(lp + (p + 1) * a.part_stride_lse + lrow) - M);
        float x0[8], x1[8];
        if (w0 > 0.f) Vec8<TI>::load(base + p * a.part_stride_o, x0);
        if (w1 > 0.f) Vec8<TI>::load(base + (p + 1) * a.part_stride_o, x1);
        if (w0 > 0.f) {
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = fmaf(w0, x0[e], acc[e]);
          W += w0;
        }
        if (w1 > 0.f) {
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = fmaf(w1, x1[e], acc[e]);
          W += w1;
        }
      }
      for (; p < a.P; ++p) {
        const float w = exp2f(__ldg(lp + p * a.part_stride_lse + lrow) - M);
        if (w > 0.f) {
          float x[8];
          Vec8<TI>::load(base + p * a.part_stride_o, x);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, x[e], acc[e]);
          W += w;
        }
      }
      const float inv = 1.0f / W;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] *= inv;
    }
    Vec8<TO>::store(out + row * a.D + c * 8, acc);
    if (c == 0 && a.lse != nullptr) a.lse[lrow] = (M == -INFINITY) ? -INFINITY : M + log2f(W);
  }
}

}  // namespace skv
