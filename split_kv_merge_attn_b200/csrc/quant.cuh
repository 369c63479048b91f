// INT8 codes for the int8 Q K^T prefill (the use the ARK issue gives for
// smooth_k: K is smoothed so that it quantizes well to INT8).
//
// One CTA per (128-row block, batch x head) of an HND [B, H, S, D] 16-bit
// tensor, D = 128: the block's values x (Q as is; K minus the fp32 mean of
// its kv head) are held in registers, amax = max |x| over the block, the
// block's scale is amax / 127 (1 for an all-zero block), and each code is
// round-half-to-even(x * (127 / amax)) clamped to [-127, 127]: one IEEE fp32
// division per block, one fp32 product per value.  For Q the same pass also writes the per-row smoothing shift
// scale * log2(e) * (q . mean K) that the prefill adds back to the LSE.
// Bandwidth bound: one read of the 16-bit tensor, one write of the codes.
#pragma once

#include "skv_device.cuh"

namespace skv {

struct QuantArgs {
  const void* x;        // [B, H, S, 128] 16-bit, HND, contiguous
  int8_t* codes;        // [B, H, S, 128]
  float* scales;        // [B, H, nblk]
  const float* kmean;   // [B, Hkv, 128] fp32 mean of K over the call's keys
  float* dq;            // Q only: [B, H, S]
  int B, H, Hkv, S, nblk;
  float scale_log2;
};

constexpr int kQuantBlock = 128;

template <typename T, bool kIsQ>
__global__ void __launch_bounds__(256) quant_int8_kernel(QuantArgs a) {
  constexpr int D = 128;
  constexpr int kVec = D / 8;                  // 16 vectors of 8 values per row
  constexpr int kRowsPerPass = 256 / kVec;     // 16
  const int blk = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int hkv = kIsQ ? h / (a.H / a.Hkv) : h;
  const int row0 = blk * kQuantBlock;
  const int rows = min(kQuantBlock, a.S - row0);
  const int cv = threadIdx.x % kVec;
  const int r0 = threadIdx.x / kVec;
  const float* mu = a.kmean + (static_cast<int64_t>(b) * a.Hkv + hkv) * D + cv * 8;
  float m8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m8[e] = mu[e];
  const T* src = static_cast<const T*>(a.x) + (static_cast<int64_t>(bh) * a.S + row0) * D + cv * 8;
  constexpr int kPasses = kQuantBlock / kRowsPerPass;
  // every row load of the block is issued before any is used
  uint4 u[kPasses];
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int r = r0 + kRowsPerPass * p;
    u[p] = r < rows ? __ldg(reinterpret_cast<const uint4*>(src + static_cast<int64_t>(r) * D)) : make_uint4(0, 0, 0, 0);
  }
  float x[kPasses][8];
  float amax = 0.f;
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int r = r0 + kRowsPerPass * p;
    const uint32_t w[4] = {u[p].x, u[p].y, u[p].z, u[p].w};
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack2<T>(w[e]);
      if constexpr (kIsQ) {
        x[p][2 * e] = f.x;
        x[p][2 * e + 1] = f.y;
        dot = fmaf(f.x, m8[2 * e], dot);
        dot = fmaf(f.y, m8[2 * e + 1], dot);
      } else {
        // rows past the end stay 0 (not 0 - mean), so they cannot raise amax
        x[p][2 * e] = r < rows ? f.x - m8[2 * e] : 0.f;
        x[p][2 * e + 1] = r < rows ? f.y - m8[2 * e + 1] : 0.f;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[p][e]));
    if constexpr (kIsQ) {
      // the 16 threads of a row are 16 consecutive lanes of one warp
#pragma unroll
      for (int o = kVec / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (cv == 0 && r < rows) a.dq[static_cast<int64_t>(bh) * a.S + row0 + r] = dot * a.scale_log2;
    }
  }
  // block max
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
  const float sc = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 1.0f;
  const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
  if (threadIdx.x == 0) a.scales[static_cast<int64_t>(bh) * a.nblk + blk] = sc;
  int8_t* dst = a.codes + (static_cast<int64_t>(bh) * a.S + row0) * D + cv * 8;
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int r = r0 + kRowsPerPass * p;
    if (r < rows) {
      uint32_t pk[2] = {0u, 0u};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int c = max(-127, min(127, __float2int_rn(__fmul_rn(x[p][e], inv))));
        pk[e >> 2] |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * (e & 3));
      }
      *reinterpret_cast<uint2*>(dst + static_cast<int64_t>(r) * D) = make_uint2(pk[0], pk[1]);
    }
  }
}

}  // namespace skv
