// Split-KV decode kernel (memory bound): per (batch, kv head, row group,
// split) one CTA streams its split of K and V from HBM exactly once.
//
// Prior art: the ExecuTorch split-K decode kernels (PR #22133, "Prevent
// Voxtral NaNs in CUDA split-K attention").  That PR replaced a fixed
// exponent offset by a per-split running max with rescaled partials; this
// kernel does the same (stable online softmax in the exp2 domain) and writes
// every partial slot (empty splits write O = 0, LSE = -inf).  The cross-split
// reduction is either the merge_state kernel, launched after it, or done in
// this launch: with an arrival counter per (batch, kv head, row group), the
// CTA that finishes last among the group's splits merges their partials
// itself (no CTA ever waits for another) and sets the counter back to zero.
//
// B200 mapping:
//  * the G*Lq query rows that share one kv head (GQA) form one 16-row M tile,
//    so each K/V byte read from HBM serves all of them;
//  * one producer warp streams 64-key K and V tiles with 2-D TMA loads
//    (128-byte swizzle, no multicast) into an NS-stage mbarrier ring;
//  * four consumer warps each take 16 keys of every tile and run
//    S = Q K^T and O += P V as m16n8k16 tensor-core MMAs (fp32 accumulate)
//    with the online softmax in registers; warp states are combined through
//    shared memory at the end.
// Tensor cores are used because at G*Lq = 16 rows the FMA work per key
// (2 * 16 * D) exceeds what the CUDA cores sustain at HBM rate; the MMA shape
// simply holds the 16 rows that share a kv head.
#pragma once

#include "skv_device.cuh"

namespace skv {

constexpr int kDecodeKeysPerTile = 64;
constexpr int kDecodeRows = 16;
constexpr int kDecodeConsumerWarps = 4;
constexpr int kDecodeThreads = (kDecodeConsumerWarps + 1) * 32;
constexpr int kSplitMaxDevice = 256;   // largest num_splits (the host planner's cap)
constexpr int kDecodeCombineHeader = 1024;  // per-warp running max and sum, before the fragments
constexpr int kMergeStageOffset = kSplitMaxDevice * kDecodeRows * 4 + 128;  // after weights + 1/sum

// Tuning switches (compile time): K/V ring depth of the decode for D = 128 and
// D = 256 (one stage holds the K and V tiles of 64 keys).
#ifndef SKV_DECODE_STAGES_D128
#define SKV_DECODE_STAGES_D128 3
#endif
#ifndef SKV_DECODE_STAGES_D256
#define SKV_DECODE_STAGES_D256 3
#endif

template <int D>
struct DecodeCfg {
  static constexpr int kBoxes = D / 64;                       // 64-element column boxes per row
  static constexpr int kTileBytes = kBoxes * kDecodeKeysPerTile * 128;  // one K or V tile
  static constexpr int kStages = (D == 64) ? 6 : (D == 128 ? SKV_DECODE_STAGES_D128 : SKV_DECODE_STAGES_D256);
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kQStride = D + 8;                      // elements; 16-byte pad per row
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kCombineBytes = kDecodeCombineHeader + kDecodeConsumerWarps * kDecodeRows * D * 4;
  static_assert(kRingBytes >= kCombineBytes, "combine area reuses the ring");
  static constexpr int kQBytes = kDecodeRows * kQStride * 2;
  static constexpr int kSmemBytes = kRingBytes + kQBytes + 2 * kStages * 8 + 16 + 1024;  // +align pad
  static constexpr bool kQInRegs = (D <= 128);
};

struct DecodeArgs {
  const void* q;
  void* out;
  float* lse;
  float* part_o;
  float* part_lse;
  int* counters;  // [grid.y] arrival counters (zero between calls), or null: merge_state merges
  const int* kv_len;
  int B, Hq, Hkv, Lq, Lkv;
  int num_splits;
  int row_groups;
  int causal;  // 1: query row i (of Lq) sees keys j < kv_len - Lq + 1 + i
  float scale_log2;
};

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// Merge of every split's partial (O, LSE) of one row group, run by the 128
// consumer threads of the CTA that finished last; `smem` is the (idle) K/V
// ring.  Per row: M = max_s L_s, w_s = 2^(L_s - M) (0 for -inf),
// O = sum_s w_s O_s / sum_s w_s, LSE = M + log2(sum_s w_s); all splits empty
// gives O = 0, LSE = -inf.  The partials of a row group are contiguous
// (rn rows x D floats per split); they are staged into shared memory with
// 16-byte cp.async copies (L2 only), as many splits per batch as fit.
template <int D, typename T>
__device__ __forceinline__ void decode_merge_group(const DecodeArgs& a, uint8_t* smem, int smem_bytes,
                                                   int64_t orow0, int rn, int64_t rows_all) {
  constexpr int kV = D / 4;                  // float4 per row
  constexpr int kJ = kDecodeRows * kV / 128; // float4 outputs per thread (at most)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = a.num_splits;
  float* wt = reinterpret_cast<float*>(smem);  // [S][16] weights
  float* rinv = wt + kSplitMaxDevice * kDecodeRows;  // [16] 1 / sum of weights
  float4* stage = reinterpret_cast<float4*>(smem + kMergeStageOffset);
  const int nv = rn * kV;
  const int cap = (smem_bytes - kMergeStageOffset) / 16;
  const int nb = max(1, cap / nv);  // splits per batch

  const float4* po = reinterpret_cast<const float4*>(a.part_o);
  const uint32_t stage_addr = smem_u32(stage);
  // copies of splits [s0, s1) into the staging area (one commit group)
  auto issue = [&](int s0, int s1) {
    for (int s = s0; s < s1; ++s) {
      const float4* src = po + (s * rows_all + orow0) * kV;
#pragma unroll
      for (int j = 0; j < kJ; ++j) {
        const int v = tid + 128 * j;
        if (v < nv) cp_async_16(stage_addr + static_cast<uint32_t>(((s - s0) * nv + v) * 16), src + v);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  issue(0, min(S, nb));  // the first batch is in flight while the weights are computed

  // ---- weights: warp w takes rows w, w+4, ...
  for (int r = warp; r < rn; r += kDecodeConsumerWarps) {
    float L[kSplitMaxDevice / 32];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < kSplitMaxDevice / 32; ++i) {
      const int s = lane + 32 * i;
      L[i] = (s < S) ? __ldcg(a.part_lse + s * rows_all + orow0 + r) : -INFINITY;
      mx = fmaxf(mx, L[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < kSplitMaxDevice / 32; ++i) {
      const int s = lane + 32 * i;
      const float w = (L[i] == -INFINITY) ? 0.f : ex2_approx(L[i] - mx);
      if (s < S) wt[s * kDecodeRows + r] = w;
      sum += w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) {
      rinv[r] = sum > 0.f ? 1.0f / sum : 0.f;
      if (a.lse != nullptr) a.lse[orow0 + r] = sum > 0.f ? mx + __log2f(sum) : -INFINITY;
    }
  }
  named_barrier_sync(1, kDecodeConsumerWarps * 32);

  // ---- O: thread t owns float4 outputs t, t + 128, ...
  float4 acc[kJ];
#pragma unroll
  for (int j = 0; j < kJ; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < S; s0 += nb) {
    const int s1 = min(S, s0 + nb);
    if (s0 > 0) issue(s0, s1);
    asm volatile("cp.async.wait_all;" ::: "memory");
    // each thread reads back only the slots it copied itself
    for (int s = s0; s < s1; ++s) {
#pragma unroll
      for (int j = 0; j < kJ; ++j) {
        const int v = tid + 128 * j;
        if (v < nv) {
          const float w = wt[s * kDecodeRows + v / kV];
          const float4 x = stage[(s - s0) * nv + v];
          acc[j].x = fmaf(w, x.x, acc[j].x);
          acc[j].y = fmaf(w, x.y, acc[j].y);
          acc[j].z = fmaf(w, x.z, acc[j].z);
          acc[j].w = fmaf(w, x.w, acc[j].w);
        }
      }
    }
  }
  T* out = static_cast<T*>(a.out) + orow0 * D;
#pragma unroll
  for (int j = 0; j < kJ; ++j) {
    const int v = tid + 128 * j;
    if (v < nv) {
      const float inv = rinv[v / kV];
      uint2 u;
      u.x = pack2<T>(acc[j].x * inv, acc[j].y * inv);
      u.y = pack2<T>(acc[j].z * inv, acc[j].w * inv);
      *reinterpret_cast<uint2*>(out + static_cast<int64_t>(v) * 4) = u;
    }
  }
}

template <int D, typename T>
__global__ void __launch_bounds__(kDecodeThreads) decode_split_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                      const __grid_constant__ CUtensorMap tmV,
                                                                      const DecodeArgs a) {
  using Cfg = DecodeCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  T* qs = reinterpret_cast<T*>(smem + Cfg::kRingBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kRingBytes + Cfg::kQBytes);
  uint64_t* empty = full + Cfg::kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + Cfg::kStages);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int split = blockIdx.x;
  const int G = a.Hq / a.Hkv;
  const int rows_total = G * a.Lq;
  const int rg = blockIdx.y % a.row_groups;
  const int hkv = (blockIdx.y / a.row_groups) % a.Hkv;
  const int b = blockIdx.y / (a.row_groups * a.Hkv);

  if (tid == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecodeConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();  // barriers initialised
  // This grid is launched as a programmatic dependent of the kernel before it
  // on the stream, so its CTAs can be resident before that kernel ends: every
  // thread waits here for that kernel's completion (and its memory) before it
  // reads an input (kv_len, Q, K, V) or writes anything.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // let a programmatically dependent merge launch be scheduled; it still waits
  // for this whole grid to finish before it reads the partials
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- split bounds (same rule as the host planner)
  int n = a.Lkv;
  if (a.kv_len != nullptr) n = min(max(a.kv_len[b], 0), a.Lkv);
  int s0 = 0, s1 = 0;
  if (n > 0) {
    const int per = (n + a.num_splits - 1) / a.num_splits;
    const int C = ((per + 63) / 64) * 64;
    s0 = min(split * C, n);
    s1 = min(s0 + C, n);
  }
  const int ntiles = (s1 - s0 + kDecodeKeysPerTile - 1) / kDecodeKeysPerTile;

  const int64_t row0 = (static_cast<int64_t>(b) * a.Hkv + hkv) * a.Lkv;

  if (warp == kDecodeConsumerWarps) {
    // ================= producer warp: TMA ring
    if (lane == 0 && ntiles > 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int st = t % Cfg::kStages;
        if (t >= Cfg::kStages) {
          if (!mbar_wait(&empty[st], ((t / Cfg::kStages) & 1) ^ 1, abort_flag, 0x101)) break;
        }
        mbar_arrive_expect_tx(&full[st], Cfg::kStageBytes);
        uint8_t* kt = ring + st * Cfg::kStageBytes;
        uint8_t* vt = kt + Cfg::kTileBytes;
        const int row = static_cast<int>(row0 + s0 + t * kDecodeKeysPerTile);
#pragma unroll
        for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
          tma_load_2d(kt + bx * kDecodeKeysPerTile * 128, &tmK, &full[st], bx * 64, row);
          tma_load_2d(vt + bx * kDecodeKeysPerTile * 128, &tmV, &full[st], bx * 64, row);
        }
        issued = t + 1;
      }
      if (*abort_flag) {
        // let every load already issued land before the CTA's shared memory goes away
        for (int t = max(0, issued - Cfg::kStages); t < issued; ++t)
          mbar_drain(&full[t % Cfg::kStages], (t / Cfg::kStages) & 1, 20000000ull);
      }
    }
    return;
  }

  // ================= consumer warps
  // Q rows of this group into shared memory (zero rows pad the tile); the
  // producer's first K/V loads are already in flight meanwhile.  Every load of
  // a thread is issued before its first shared-memory store (one round trip:
  // the stores could alias the loads' addresses for the compiler, which would
  // otherwise keep each load behind the previous store).
  {
    constexpr int vpr = D / 8;
    constexpr int kQv = kDecodeRows * vpr / (kDecodeConsumerWarps * 32);  // 16-byte pieces per thread
    static_assert(kDecodeRows * vpr % (kDecodeConsumerWarps * 32) == 0, "Q pieces divide over the consumers");
    uint4 qv[kQv];
#pragma unroll
    for (int u = 0; u < kQv; ++u) {
      const int v = tid + kDecodeConsumerWarps * 32 * u;
      const int r = v / vpr, c = v % vpr;
      const int rglob = rg * kDecodeRows + r;
      qv[u] = make_uint4(0, 0, 0, 0);
      if (rglob < rows_total) {
        const int h = hkv * G + rglob / a.Lq;
        const int i = rglob % a.Lq;
        const T* src = static_cast<const T*>(a.q) + ((static_cast<int64_t>(b) * a.Hq + h) * a.Lq + i) * D + c * 8;
        qv[u] = __ldg(reinterpret_cast<const uint4*>(src));
      }
    }
#pragma unroll
    for (int u = 0; u < kQv; ++u) {
      const int v = tid + kDecodeConsumerWarps * 32 * u;
      *reinterpret_cast<uint4*>(qs + (v / vpr) * Cfg::kQStride + (v % vpr) * 8) = qv[u];
    }
  }
  named_barrier_sync(1, kDecodeConsumerWarps * 32);
  const int g = lane >> 2, tq = lane & 3;
  const uint32_t qs_addr = smem_u32(qs);
  uint32_t qa[Cfg::kQInRegs ? D / 16 : 1][4];
  if constexpr (Cfg::kQInRegs) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int r = (lane & 7) + ((lane >> 3) & 1) * 8;
      const int c = kk * 16 + (lane >> 4) * 8;
      ldmatrix_x4(qs_addr + (r * Cfg::kQStride + c) * 2, qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
    }
  }
  // keys each of this thread's two tile rows (g, g + 8) may see: all of the
  // split, or under the causal mask the first n - Lq + 1 + i keys of row i
  int row_end[2] = {s1, s1};
  if (a.causal) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int i = (rg * kDecodeRows + g + 8 * hr) % a.Lq;
      row_end[hr] = min(s1, max(n - a.Lq + 1 + i, 0));
    }
  }
  float m[2] = {-INFINITY, -INFINITY};
  float lsum[2] = {0.f, 0.f};
  float o[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;

  bool ok = true;
  for (int t = 0; t < ntiles; ++t) {
    const int st = t % Cfg::kStages;
    if (!mbar_wait(&full[st], (t / Cfg::kStages) & 1, abort_flag, 0x102)) { ok = false; break; }
    const uint32_t kt = smem_u32(ring + st * Cfg::kStageBytes);
    const uint32_t vt = kt + Cfg::kTileBytes;
    const int key0 = s0 + t * kDecodeKeysPerTile + warp * 16;  // first key of this warp
    const int nvalid = min(16, s1 - key0);                     // may be <= 0

    // ---- S = Q K^T for 16 rows x 16 keys
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t aq[4];
      if constexpr (Cfg::kQInRegs) {
        aq[0] = qa[kk][0]; aq[1] = qa[kk][1]; aq[2] = qa[kk][2]; aq[3] = qa[kk][3];
      } else {
        const int r = (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = kk * 16 + (lane >> 4) * 8;
        ldmatrix_x4(qs_addr + (r * Cfg::kQStride + c) * 2, aq[0], aq[1], aq[2], aq[3]);
      }
      const int bx = kk >> 2;
      const int chunk = (kk & 3) * 2 + ((lane >> 3) & 1);
      const int krow = warp * 16 + (lane & 7) + (lane >> 4) * 8;
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(kt + bx * kDecodeKeysPerTile * 128 + sw128(krow, chunk), b0, b1, b2, b3);
      mma_16816<T>(sc[0], aq, b0, b1);
      mma_16816<T>(sc[1], aq, b2, b3);
    }

    // ---- online softmax (exp2 domain), rows g and g+8 of the tile
    float x[2][4];
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kidx = nt * 8 + 2 * tq + (e & 1);
        const float val = (key0 + kidx < row_end[e >> 1]) ? sc[nt][e] * a.scale_log2 : -INFINITY;
        x[nt][e] = val;
      }
      mx0 = fmaxf(mx0, fmaxf(x[nt][0], x[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(x[nt][2], x[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m[0], mx0), mn1 = fmaxf(m[1], mx1);
    const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0;
    const float mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
    const float al0 = ex2_approx(m[0] - mu0), al1 = ex2_approx(m[1] - mu1);
    m[0] = mn0;
    m[1] = mn1;
    float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      x[nt][0] = ex2_approx(x[nt][0] - mu0);
      x[nt][1] = ex2_approx(x[nt][1] - mu0);
      x[nt][2] = ex2_approx(x[nt][2] - mu1);
      x[nt][3] = ex2_approx(x[nt][3] - mu1);
      ps0 += x[nt][0] + x[nt][1];
      ps1 += x[nt][2] + x[nt][3];
    }
    lsum[0] = lsum[0] * al0 + ps0;
    lsum[1] = lsum[1] * al1 + ps1;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      o[j][0] *= al0; o[j][1] *= al0;
      o[j][2] *= al1; o[j][3] *= al1;
    }
    uint32_t pa[4];
    pa[0] = pack2<T>(x[0][0], x[0][1]);
    pa[1] = pack2<T>(x[0][2], x[0][3]);
    pa[2] = pack2<T>(x[1][0], x[1][1]);
    pa[3] = pack2<T>(x[1][2], x[1][3]);

    // keys past the end of the split: their P is 0, and their V rows (which
    // may hold anything, e.g. unfilled cache) are zeroed so 0 * V stays 0
    if (nvalid < 16) {
      const int nz = 16 - max(nvalid, 0);
      uint8_t* vgen = ring + st * Cfg::kStageBytes + Cfg::kTileBytes;
      for (int idx = lane; idx < nz * Cfg::kBoxes * 8; idx += 32) {
        const int rr = 16 - nz + idx / (Cfg::kBoxes * 8);
        const int rem = idx % (Cfg::kBoxes * 8);
        const int bx = rem / 8, ch = rem % 8;
        *reinterpret_cast<uint4*>(vgen + bx * kDecodeKeysPerTile * 128 + (warp * 16 + rr) * 128 + ch * 16) =
            make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }

    // ---- O += P V
#pragma unroll
    for (int nd = 0; nd < D / 16; ++nd) {
      const int bx = nd >> 2;
      const int chunk = (nd & 3) * 2 + (lane >> 4);
      const int vrow = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      uint32_t v0, v1, v2, v3;
      ldmatrix_x4_trans(vt + bx * kDecodeKeysPerTile * 128 + sw128(vrow, chunk), v0, v1, v2, v3);
      mma_16816<T>(o[2 * nd], pa, v0, v1);
      mma_16816<T>(o[2 * nd + 1], pa, v2, v3);
    }
    if (nvalid < 16) fence_proxy_async_smem();  // generic writes before the async proxy reuses the stage
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }

  // ---- combine the four warps' states
  named_barrier_sync(1, kDecodeConsumerWarps * 32);
  (void)ok;  // a failed wait has set the abort flag, which every consumer thread sees after the barrier
  const bool aborted = *abort_flag != 0;
  if (aborted && (a.counters == nullptr || a.num_splits == 1)) return;
  lsum[0] += __shfl_xor_sync(0xffffffffu, lsum[0], 1);
  lsum[0] += __shfl_xor_sync(0xffffffffu, lsum[0], 2);
  lsum[1] += __shfl_xor_sync(0xffffffffu, lsum[1], 1);
  lsum[1] += __shfl_xor_sync(0xffffffffu, lsum[1], 2);
  // Each warp stores its accumulator fragments in fragment order: per 8-column
  // block j one float4 per lane (rows g and g + 8, columns 2tq and 2tq + 1),
  // so every store and every load below is a contiguous 512-byte run per warp
  // instruction (no shared-memory bank conflicts).
  float* cm = reinterpret_cast<float*>(ring);                    // [4][16] running max
  float* cl = cm + kDecodeConsumerWarps * kDecodeRows;            // [4][16] sums
  float4* co4 = reinterpret_cast<float4*>(ring + kDecodeCombineHeader);  // [4][D/8][32]
  if (tq == 0) {
    cm[warp * 16 + g] = m[0];
    cm[warp * 16 + g + 8] = m[1];
    cl[warp * 16 + g] = lsum[0];
    cl[warp * 16 + g + 8] = lsum[1];
  }
#pragma unroll
  for (int j = 0; j < D / 8; ++j) co4[(warp * (D / 8) + j) * 32 + lane] = make_float4(o[j][0], o[j][1], o[j][2], o[j][3]);
  named_barrier_sync(1, kDecodeConsumerWarps * 32);

  // Thread t combines fragment slots t, t + 128, ...: blocks j = warp + 4k of
  // lane `lane`, i.e. always rows g and g + 8, whose weights it computes
  // itself.  Per row: M = max_w m_w, L = sum_w 2^(m_w - M) l_w, weight of warp
  // w 2^(m_w - M) / L (0 for a warp that saw no key), LSE = M + log2 L.
  const int rows_here = min(kDecodeRows, rows_total - rg * kDecodeRows);
  const int64_t rows_all = static_cast<int64_t>(a.B) * a.Hq * a.Lq;
  const int64_t orow0 = (static_cast<int64_t>(b) * a.Hq + static_cast<int64_t>(hkv) * G) * a.Lq +
                        static_cast<int64_t>(rg) * kDecodeRows;
  if (!aborted && g < rows_here) {
    float wt[2][kDecodeConsumerWarps];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int r = g + 8 * hr;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kDecodeConsumerWarps; ++w) M = fmaxf(M, cm[w * 16 + r]);
      float L = 0.f;
#pragma unroll
      for (int w = 0; w < kDecodeConsumerWarps; ++w) {
        const float mw = cm[w * 16 + r];
        wt[hr][w] = (mw == -INFINITY) ? 0.f : ex2_approx(mw - M);
        L += wt[hr][w] * cl[w * 16 + r];
      }
      const float inv = (L > 0.f) ? 1.0f / L : 0.f;
#pragma unroll
      for (int w = 0; w < kDecodeConsumerWarps; ++w) wt[hr][w] *= inv;
      if (warp == 0 && tq == 0 && r < rows_here) {
        const float lse_val = (L > 0.f) ? M + __log2f(L) : -INFINITY;
        if (a.num_splits == 1) {
          if (a.lse != nullptr) a.lse[orow0 + r] = lse_val;
        } else {
          a.part_lse[static_cast<int64_t>(split) * rows_all + orow0 + r] = lse_val;
        }
      }
    }
    const bool hi = g + 8 < rows_here;
#pragma unroll
    for (int k = 0; k < D / 32; ++k) {
      const int j = warp + 4 * k;
      const int col = j * 8 + 2 * tq;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < kDecodeConsumerWarps; ++w) {
        const float4 x = co4[(w * (D / 8) + j) * 32 + lane];
        acc.x = fmaf(wt[0][w], x.x, acc.x);
        acc.y = fmaf(wt[0][w], x.y, acc.y);
        acc.z = fmaf(wt[1][w], x.z, acc.z);
        acc.w = fmaf(wt[1][w], x.w, acc.w);
      }
      if (a.num_splits == 1) {
        T* dst = static_cast<T*>(a.out) + (orow0 + g) * D + col;
        *reinterpret_cast<uint32_t*>(dst) = pack2<T>(acc.x, acc.y);
        if (hi) *reinterpret_cast<uint32_t*>(dst + 8 * D) = pack2<T>(acc.z, acc.w);
      } else {
        float* dst = a.part_o + (static_cast<int64_t>(split) * rows_all + orow0 + g) * D + col;
        *reinterpret_cast<float2*>(dst) = make_float2(acc.x, acc.y);
        if (hi) *reinterpret_cast<float2*>(dst + 8 * D) = make_float2(acc.z, acc.w);
      }
    }
  }
  if (a.counters == nullptr || a.num_splits == 1) return;

  // ---- in-launch merge: the last CTA of this row group to arrive merges.
  // The barrier orders every consumer thread's partial stores before thread
  // 0's arrival, whose release (cumulative) publishes them; its acquire, with
  // the next barrier, orders the last CTA's loads after every other split's
  // release.
  named_barrier_sync(1, kDecodeConsumerWarps * 32);
  volatile int* last_flag = abort_flag + 1;
  if (tid == 0) {
    int old;
    asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], 1;" : "=r"(old) : "l"(a.counters + blockIdx.y) : "memory");
    if (old < 0 || old >= a.num_splits) record_error(kErrDecodeCounter);  // counter was not zero before the call
    *last_flag = (old == a.num_splits - 1) ? 1 : 0;
  }
  named_barrier_sync(1, kDecodeConsumerWarps * 32);
  if (*last_flag == 0) return;
  decode_merge_group<D, T>(a, ring, Cfg::kRingBytes, orow0, rows_here, rows_all);
  if (tid == 0) a.counters[blockIdx.y] = 0;  // ready for the next call on this workspace
}

}  // namespace skv
