// Prefill / varlen attention forward with a per-row log2 LSE on sm_100a.
//
// Defines O_i = softmax_j(scale * q_i . k_j) V and LSE_i = log2 sum_j exp(scale *
// q_i . k_j) over the original logits, one LSE per row (ARK return_lse issue,
// "Expected:").  The ARK kernel the issue describes stored one value per
// 16-row group; here the softmax thread that owns TMEM lane i (= query row i
// of its 128-row tile) computes and stores row i's LSE itself.
//
// CTA = up to two 128-row query tiles of one (sequence, head) that share every
// K/V tile (one tile at D = 256).  Warp roles (320 threads):
//   warps 0-3  softmax + epilogue for query tile 0 (thread t owns row t)
//   warps 4-7  softmax + epilogue for query tile 1
//   warp  8    TMA producer: Q tiles once, then K_j, V_j into a ring of
//              NS shared-memory buffers (128-byte swizzle, no multicast)
//   warp  9    TMEM allocator and (one elected thread) tcgen05.mma issuer
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+D),
// O_1 [256+D, 256+2D) for D <= 128.  S_a holds fp32 logits; the softmax
// writes P_a as packed 16-bit pairs into S_a's first 64 columns, and
// O_a += P_a V_j reads P_a straight from TMEM (A operand in tensor memory).
//
// The MMA thread alternates between the tiles (S_0(j), PV_1(j-1), S_1(j),
// PV_0(j)), so while the softmax warps of one tile exponentiate, the tensor
// core works on the other tile.  At D = 256 (one tile; O_0 fills [256,512))
// the two S buffers hold the logits of consecutive KV steps instead, in the
// order S(0) | S(j+1), PV(j): the tensor core computes the next step's
// logits while the softmax of step j runs.
//
// Online softmax in the exp2 domain with a lazily updated running max: the
// max is only raised (and O_a rescaled in TMEM) when it grows by more than 8
// (log2 units); otherwise the stale max is kept, which bounds P by 2^8 and is
// exact once O and the row sum are divided at the end.  No fixed exponent
// offset is used anywhere (ExecuTorch split-K PR).
#pragma once

#include <type_traits>

#include "skv_device.cuh"
#include "tcgen05.cuh"

namespace skv {

constexpr int kPfBM = 128;          // rows per query tile
constexpr int kPfBN = 128;          // keys per KV tile
constexpr int kPfThreads = 320;
constexpr float kPfRescaleThreshold = 8.0f;

// Tuning switches (compile time) of the softmax's exponent pass, whose 64
// ex2 per row half occupy the special-function unit (about 8 cycles per warp
// instruction on B200, against 2.3 for a packed fp32 FMA):
//   SKV_PF_POLY_PAIRS  of every 16 pairs of probabilities, this many are
//                      computed on the FMA pipe (poly_exp2_pair) instead of ex2;
//   SKV_PF_INT_PACK    1: round the probabilities to 16 bits with integer
//                      operations instead of the conversion instruction.
#ifndef SKV_PF_POLY_PAIRS
#define SKV_PF_POLY_PAIRS 6   // measured best of 0, 4, 6, 8, 10 (varlen workload: 960 -> 1000 TFLOP/s)
#endif
#ifndef SKV_PF_INT_PACK
#define SKV_PF_INT_PACK 0
#endif

// 2^x on the FMA pipe for x in [-126, 2^22): x = n + f with n = round(x) (the
// 1.5 * 2^23 addition) and f in [-1/2, 1/2]; 2^f by the degree-3 polynomial
// of least maximum relative error on [-1/2, 1/2] (7.5e-5; the coefficients
// are those printed by exp2_poly_fit.py in this directory, a Remez exchange);
// 2^n is an addition to the exponent field.  Arguments below -126 are clamped
// there; below -125 the results are only known to be < 2^-124 (no row sum
// notices them: the row's largest probability is >= 1).
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;

__device__ __forceinline__ void poly_exp2_pair(uint64_t x2, float& p0, float& p1) {
  float2 x = f2_unpack(x2);
  const uint64_t xc = f2_pack(fmaxf(x.x, -126.f), fmaxf(x.y, -126.f));
  const uint64_t y = fadd2(xc, f2_pack(12582912.f, 12582912.f));    // round(x) in the low mantissa bits
  const uint64_t n = fadd2(y, f2_pack(-12582912.f, -12582912.f));   // round(x) as a float
  const uint64_t f = ffma2(n, f2_pack(-1.f, -1.f), xc);              // x - round(x), exact
  uint64_t q = ffma2(f2_pack(kExp2C3, kExp2C3), f, f2_pack(kExp2C2, kExp2C2));
  q = ffma2(q, f, f2_pack(kExp2C1, kExp2C1));
  q = ffma2(q, f, f2_pack(kExp2C0, kExp2C0));
  const float2 qf = f2_unpack(q), yf = f2_unpack(y);
  p0 = __uint_as_float(__float_as_uint(qf.x) + (__float_as_uint(yf.x) << 23));
  p1 = __uint_as_float(__float_as_uint(qf.y) + (__float_as_uint(yf.y) << 23));
}

// Two non-negative finite floats rounded to nearest-even 16-bit pairs with
// integer operations (bf16: the upper half after adding 0x7FFF plus the lowest
// kept bit; fp16 goes through the conversion instruction).
template <typename T>
__device__ __forceinline__ uint32_t pack2_p(float lo, float hi) {
  if constexpr (SKV_PF_INT_PACK && std::is_same<T, __nv_bfloat16>::value) {
    uint32_t a = __float_as_uint(lo), b = __float_as_uint(hi);
    a += 0x7FFFu + ((a >> 16) & 1u);
    b += 0x7FFFu + ((b >> 16) & 1u);
    return __byte_perm(a, b, 0x7632);
  } else {
    return pack2<T>(lo, hi);
  }
}

// Exponentiates 64 logits (32 pairs) of one row: p = 2^(s * scale_log2 + nb),
// packs them as 16-bit pairs and accumulates the row sum in packed fp32 pairs.
// kPoly: a tile without masked keys, where SKV_PF_POLY_PAIRS of every 16 pairs
// go to the FMA pipe (a masked key must give exactly 0, which ex2 does).
template <bool kPoly, typename T>
__device__ __forceinline__ void exp_pack_64(const float (&sv)[64], uint64_t sc2, uint64_t nb2, uint32_t (&pk)[32],
                                            uint64_t (&ps2)[2]) {
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const uint64_t x2 = ffma2(f2_pack(sv[2 * e], sv[2 * e + 1]), sc2, nb2);
    float p0, p1;
    if (kPoly && ((e % 16) * SKV_PF_POLY_PAIRS) % 16 < SKV_PF_POLY_PAIRS) {
      poly_exp2_pair(x2, p0, p1);
    } else {
      const float2 x = f2_unpack(x2);
      p0 = ex2_approx(x.x);
      p1 = ex2_approx(x.y);
    }
    ps2[e & 1] = fadd2(ps2[e & 1], f2_pack(p0, p1));
    pk[e] = pack2_p<T>(p0, p1);
  }
}

// kI8: Q and K arrive as int8 codes (one 128-byte box per row at D = 128)
// and S = Q K^T is an s32 .kind::i8 product; V stays 16-bit.
// s32 logits read from TMEM (bit patterns in float registers) as the floats
// kMagic + s: |s| < 2^22 for int8 codes at D <= 128, so adding the bits of
// kMagic = 1.5 * 2^23 to the integer gives that float exactly.  The kernel
// keeps the offset and folds -kMagic * scale into the bias of its FMA, so a
// logit costs one integer add more than in the 16-bit path.
constexpr float kMagic = 12582912.0f;
__device__ __forceinline__ void s32_to_magic_64(float (&v)[64]) {
#pragma unroll
  for (int c = 0; c < 64; ++c) v[c] = __int_as_float(__float_as_int(v[c]) + 0x4B400000);
}

// Query tiles per CTA: two (the MMA ping-pongs between them) for D <= 128; one
// for D = 256, whose O accumulator takes the 256 TMEM columns the second tile
// would need.
__host__ __device__ constexpr int prefill_tiles(int D) { return D == 256 ? 1 : 2; }

template <int D, bool kI8 = false>
struct PrefillCfg {
  static constexpr int kTiles = prefill_tiles(D);
  static constexpr int kRows = kTiles * kPfBM;       // query rows per CTA
  static constexpr int kBoxes = D / 64;              // 64-element boxes of a 16-bit row (V, and Q/K)
  static constexpr int kQKBoxes = kI8 ? D / 128 : kBoxes;  // boxes of a Q or K row
  static constexpr int kQKBoxElems = kI8 ? 128 : 64;
  static constexpr int kBoxBytes = 128 * 128;       // 128 rows x 128 bytes
  static constexpr int kQTileBytes = kQKBoxes * kBoxBytes;
  static constexpr int kKTileBytes = kQKBoxes * kBoxBytes;
  static constexpr int kKVTileBytes = kBoxes * kBoxBytes;   // one ring buffer (a V tile; a K tile fits)
  // D = 256: K_j and V_j only; K_{j+1} loads once S(j) is done (while the
  // softmax of step j runs), V_{j+1} once PV(j) is done (while S(j+2) runs)
  static constexpr int kStages = (D == 64) ? 8 : (D == 256 ? 2 : 5);
  static constexpr int kRingBytes = kStages * kKVTileBytes;
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = kTiles * kQTileBytes;
  static constexpr int kOffBar = kOffRing + kRingBytes;
  // barriers: q_full, kv_full[NS], kv_empty[NS], s_full[2], p_half[2][2], o_full[2], drain
  static constexpr int kNumBars = 1 + 2 * kStages + 2 + 4 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffMu = kOffMisc + 16;             // [2][D] fp32 mean of K (smooth_k)
  static constexpr int kSmemBytes = kOffMu + 2 * D * 4 + 1024;  // + alignment pad
  static constexpr int kSCol0 = 0, kSCol1 = 128, kOCol0 = 256, kOCol1 = 256 + D;  // O_1 only when kTiles = 2
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kOCol0 + kTiles * D <= 512, "TMEM columns");
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

struct PrefillArgs {
  void* out;
  float* lse;
  const float* qscale;  // int8: [B, Hq, ceil(Sq/128)] scale of each 128-row block of Q codes
  const float* kscale;  // int8: [B, Hkv, ceil(Sk/128)] scale of each 128-key block of K' codes
  const float* dq;      // int8: [B, Hq, Sq] smoothing shift scale*log2(e)*(q . mean K), added to the LSE
  const float* kmean;   // smooth (materialised K'): [Bseq, Hkv, D] fp32 mean, else null
  const float* kpartial;  // smooth (logit shift): [chunks, Bseq, Hkv, D] per-256-key column sums, else null
  int shift_logits;     // smooth: 1 = subtract the mean term from the fp32 logits (K unsmoothed),
                        //         0 = K was replaced by K' = K - mean (already smoothed)
  const int* cu_q;
  const int* cu_k;
  const int* order;
  const int* offsets;
  int B, Hq, Hkv, Sq, Sk;
  int nqb;              // dense: 256-row query blocks per (b, h)
  int layout;           // 0 HND, 1 NHD, 2 TND
  int causal;           // 1: row i of a sequence sees keys j <= i + len_k - len_q
  float scale_log2;
  // Multi-chunk dense call: KV chunk c is keys [kvb[c], kvb[c+1]) of every
  // batch entry; its partial O and LSE go to out / lse + c * the size of one
  // output (nchunks = 1: the whole key range, one output).
  int nchunks;
  int kvb[kMaxKvChunks + 1];
};

template <int D, typename T, bool kI8 = false>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const PrefillArgs a) {
  using Cfg = PrefillCfg<D, kI8>;
  static_assert(!kI8 || D == 128, "the int8 path has one 128-byte box per row");
  constexpr int kIsBf16 = std::is_same<T, __nv_bfloat16>::value ? 1 : 0;
  constexpr uint32_t kIdescQK = kI8 ? tc5::idesc_i8(kPfBM, kPfBN) : tc5::idesc_f16(kIsBf16, 0, kPfBM, kPfBN);
  constexpr uint32_t kIdescPV = tc5::idesc_f16(kIsBf16, 1, kPfBM, D);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + Cfg::kStages;
  uint64_t* s_full = kv_empty + Cfg::kStages;
  uint64_t* p_half = s_full + 2;     // [tile][half]: P of keys [64h, 64h+64) is in TMEM (half 1 first)
  uint64_t* o_full = p_half + 4;
  uint64_t* drain = o_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kOffMisc + 8);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = a.Hq / a.Hkv;

  // ---------------- work item
  int b, h, qblk, len_q, len_k, q_row0, k_row0, bcoord;
  int chunk = 0;  // KV chunk of a multi-chunk call
  if (a.layout == 2) {
    const int item = blockIdx.x;
    if (item >= a.offsets[a.B]) return;
    int lo = 0, hi = a.B - 1;  // last p with offsets[p] <= item
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.offsets[mid] <= item) lo = mid; else hi = mid - 1;
    }
    b = a.order[lo];
    const int rem = item - a.offsets[lo];
    len_q = a.cu_q[b + 1] - a.cu_q[b];
    len_k = a.cu_k[b + 1] - a.cu_k[b];
    const int nblk = (len_q + Cfg::kRows - 1) / Cfg::kRows;
    if (a.causal) {
      // causal work grows with the block index: the sequence's last (longest)
      // blocks of every head start first
      qblk = nblk - 1 - rem / a.Hq;
      h = rem % a.Hq;
    } else {
      h = rem / nblk;
      qblk = rem % nblk;
    }
    q_row0 = a.cu_q[b] + qblk * Cfg::kRows;
    k_row0 = a.cu_k[b];
    bcoord = 0;
  } else {
    int item = blockIdx.x;
    if (a.nchunks > 1) {  // chunk-major: the CTAs running together share one chunk's K/V
      const int per = a.B * a.Hq * a.nqb;
      chunk = item / per;
      item -= chunk * per;
    }
    if (a.causal) {
      // causal work grows with the block index: longest blocks (of every
      // batch and head) first, so the grid runs longest-processing-time first
      const int bh = item % (a.B * a.Hq);
      qblk = a.nqb - 1 - item / (a.B * a.Hq);
      h = bh % a.Hq;
      b = bh / a.Hq;
    } else {
      qblk = item % a.nqb;
      h = (item / a.nqb) % a.Hq;
      b = item / (a.nqb * a.Hq);
    }
    len_q = a.Sq;
    len_k = a.kvb[chunk + 1] - a.kvb[chunk];
    q_row0 = qblk * Cfg::kRows;
    k_row0 = a.kvb[chunk];
    bcoord = b;
  }
  // smooth_k statistics are per (batch or sequence, chunk): index `seq` of
  // nseq such ranges
  const int seq = b * a.nchunks + chunk;
  const int nseq = a.B * a.nchunks;
  const int hkv = h / G;
  const int rows_here = min(Cfg::kRows, len_q - qblk * Cfg::kRows);
  const int nt = rows_here > kPfBM ? 2 : 1;
  // causal: rows are the last len_q positions of the key range (bottom-right
  // alignment); the block stops at the KV tile holding its last row's last
  // key, and both query tiles run over the same tiles (the first tile's rows
  // simply see more masked keys)
  const int causal_off = len_k - len_q;
  const int kv_end = a.causal ? min(max(qblk * Cfg::kRows + rows_here + causal_off, 0), len_k) : len_k;
  const int nkv = (kv_end + kPfBN - 1) / kPfBN;

  // output addressing for query row qi (index inside the sequence); the rows
  // of chunk c start c outputs further
  const int64_t chunk_rows = static_cast<int64_t>(chunk) * a.B * a.Hq * a.Sq;
  auto out_row = [&](int qi) -> T* {
    int64_t r;
    if (a.layout == 0) r = (static_cast<int64_t>(b) * a.Hq + h) * a.Sq + qi;
    else if (a.layout == 1) r = (static_cast<int64_t>(b) * a.Sq + qi) * a.Hq + h;
    else r = static_cast<int64_t>(a.cu_q[b] + qi) * a.Hq + h;
    return static_cast<T*>(a.out) + (chunk_rows + r) * D;
  };
  auto lse_idx = [&](int qi) -> int64_t {
    if (a.layout == 2) return static_cast<int64_t>(h) * a.Sq + a.cu_q[b] + qi;
    return chunk_rows + (static_cast<int64_t>(b) * a.Hq + h) * a.Sq + qi;
  };

  if (nkv == 0) {
    // no keys: O = 0, LSE = -inf for every valid row of this block
    for (int r = tid; r < rows_here; r += kPfThreads) {
      const int qi = qblk * Cfg::kRows + r;
      uint4* dst = reinterpret_cast<uint4*>(out_row(qi));
#pragma unroll
      for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
      if (a.lse != nullptr) a.lse[lse_idx(qi)] = -INFINITY;
    }
    return;
  }

  // ---------------- setup
  if (tid == 0) {
    for (int i = 0; i < Cfg::kNumBars; ++i) {
      const bool per_thread = &bars[i] >= &p_half[0] && &bars[i] < &p_half[4];
      mbar_init(&bars[i], per_thread ? 128u : 1u);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tc5::alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tc5::relinquish();
  }
  tc5::fence_before();
  __syncthreads();
  tc5::fence_after();
  const uint32_t tmem = *tmem_slot;
  // a kernel launched as this grid's programmatic dependent (a merge_state of
  // these partials) may become resident on SMs this grid's last wave leaves
  // idle; it waits for this grid to finish before it reads anything
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  uint8_t* qtile[2] = {smem + Cfg::kOffQ, smem + Cfg::kOffQ + Cfg::kQTileBytes};
  uint8_t* ring = smem + Cfg::kOffRing;

  if (warp == 8) {
    // ======================= TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const bool hnd = (a.layout == 0);
      mbar_arrive_expect_tx(q_full, nt * Cfg::kQTileBytes);
      for (int t = 0; t < nt; ++t) {
        const int s = q_row0 + t * kPfBM;
#pragma unroll
        for (int bx = 0; bx < Cfg::kQKBoxes; ++bx) {
          const int x = bx * Cfg::kQKBoxElems;
          if (hnd) tma_load_4d(qtile[t] + bx * Cfg::kBoxBytes, &tmQ, q_full, x, s, h, bcoord);
          else tma_load_4d(qtile[t] + bx * Cfg::kBoxBytes, &tmQ, q_full, x, h, s, bcoord);
        }
      }
      int last_u[Cfg::kStages];  // last load issued into each ring buffer (-1: none)
#pragma unroll
      for (int i = 0; i < Cfg::kStages; ++i) last_u[i] = -1;
      bool ok = true;
      // Load order: K_0 V_0 K_1 V_1 ... for two query tiles.  With one tile
      // (D = 256: two ring buffers, K in buffer 0 and V in buffer 1) the MMA
      // order is S(0) S(1) PV(0) S(2) PV(1) ..., so the buffers free up (and
      // are refilled) in the order K_0 V_0 K_1 | K_2 V_1 | K_3 V_2 | ...
      // (n -> u: 3 -> 4, 4 -> 3, 5 -> 6, ...; the one u past the end is skipped)
      const int n_end = 2 * nkv + (Cfg::kTiles == 1 ? 1 : 0);
      for (int n = 0; n < n_end && ok; ++n) {
        int u = n;
        if (Cfg::kTiles == 1 && n >= 3) u = (n & 1) ? n + 1 : n - 1;
        if (u >= 2 * nkv) continue;
        const int j = u >> 1;
        const int s = k_row0 + j * kPfBN;
        {
          const int which = u & 1;
          const int buf = u % Cfg::kStages;
          if (u >= Cfg::kStages) {
            if (!mbar_wait(&kv_empty[buf], ((u / Cfg::kStages) & 1) ^ 1, abort_flag, kErrPrefillWait)) {
              ok = false;
              break;
            }
          }
          const CUtensorMap* m = which ? &tmV : &tmK;
          const int nbox = which ? Cfg::kBoxes : Cfg::kQKBoxes;
          const int bxe = which ? 64 : Cfg::kQKBoxElems;
          mbar_arrive_expect_tx(&kv_full[buf], which ? Cfg::kKVTileBytes : Cfg::kKTileBytes);
#pragma unroll
          for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
            if (bx >= nbox) break;
            uint8_t* dst = ring + buf * Cfg::kKVTileBytes + bx * Cfg::kBoxBytes;
            if (hnd) tma_load_4d(dst, m, &kv_full[buf], bx * bxe, s, hkv, bcoord);
            else tma_load_4d(dst, m, &kv_full[buf], bx * bxe, hkv, s, bcoord);
          }
          last_u[buf] = u;
        }
      }
      if (*abort_flag) {
        // every load issued lands before the CTA's shared memory goes away: a
        // buffer is refilled only after its previous load was consumed, so only
        // the last load into each buffer can still be in flight
        mbar_drain(q_full, 0, 20000000ull);
#pragma unroll
        for (int i = 0; i < Cfg::kStages; ++i)
          if (last_u[i] >= 0) mbar_drain(&kv_full[i], (last_u[i] / Cfg::kStages) & 1, 20000000ull);
      }
    }
  } else if (warp == 9) {
    // ======================= MMA issuer
    // Issue order (ping-pong between the two query tiles, so their softmax
    // phases alternate on the exp units):
    //   S_0(0) S_1(0) PV_0(0) | S_0(j) PV_1(j-1) S_1(j) PV_0(j) | PV_1(last)
    // S_t(j) overwrites the TMEM columns that PV_t(j-1) reads P_t from; the two
    // are issued back to back by one thread and executed in issue order, the
    // ordering NVIDIA's CUTLASS Blackwell FMHA also relies on.
    // The whole warp runs this role in step (waits, descriptor arithmetic),
    // and one elected lane issues each group of MMAs and every commit: the
    // operands stay warp-uniform, so they need no per-MMA move from a
    // thread's registers into the uniform ones tcgen05.mma reads.
    {
      const uint32_t ring_addr = smem_u32(ring);
      const uint32_t q0 = smem_u32(qtile[0]), q1 = smem_u32(qtile[1]);
      const uint32_t s0c = tmem + Cfg::kSCol0, s1c = tmem + Cfg::kSCol1;
      const uint32_t o0c = tmem + Cfg::kOCol0, o1c = tmem + Cfg::kOCol1;
      // Shared-memory descriptors are built once; every MMA then only adds a
      // constant to the start-address field (shared addresses are < 256 KB, so
      // the 14-bit field never carries).
      const uint64_t dq0 = tc5::smem_desc(q0, 16, 1024), dq1 = tc5::smem_desc(q1, 16, 1024);
      const uint64_t dk_base = tc5::smem_desc(ring_addr, 16, 1024);
      const uint64_t dv_base = tc5::smem_desc(ring_addr, Cfg::kBoxBytes, 1024);
      auto issue_s = [&](uint64_t dq, uint32_t sc, int u) {
        const uint64_t dk = dk_base + static_cast<uint64_t>(((u % Cfg::kStages) * Cfg::kKVTileBytes) >> 4);
        if (elect_one()) {
          // one MMA per 32 bytes of a Q/K row (K = 16 for 16-bit, 32 for int8)
#pragma unroll
          for (int kk = 0; kk < (kI8 ? D / 32 : D / 16); ++kk) {
            const uint64_t o = static_cast<uint64_t>(((kk >> 2) * Cfg::kBoxBytes + (kk & 3) * 32) >> 4);
            if constexpr (kI8) tc5::mma_ss_i8(sc, dq + o, dk + o, kIdescQK, kk > 0 ? 1u : 0u);
            else tc5::mma_ss(sc, dq + o, dk + o, kIdescQK, kk > 0 ? 1u : 0u);
          }
        }
        __syncwarp();
      };
      // PV over the 64 keys of half hf: key block kk (16 keys) reads P from
      // columns kk * 8 (half 0) or 64 + (kk - 4) * 8 (half 1), where the
      // softmax writes them; half 1 is issued first, so its first MMA is the
      // one that overwrites O when `acc` is false
      auto issue_pv_half = [&](uint32_t sc, uint32_t oc, int u, bool acc, int hf) {
        const uint64_t dv = dv_base + static_cast<uint64_t>(((u % Cfg::kStages) * Cfg::kKVTileBytes) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int k4 = 0; k4 < kPfBN / 32; ++k4) {
            const int kk = hf * (kPfBN / 32) + k4;
            tc5::mma_ts(oc, sc + kk * 8 + hf * 32, dv + static_cast<uint64_t>((kk * 2048) >> 4), kIdescPV,
                        (acc || hf == 0 || k4 > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
      };
      auto commit = [&](uint64_t* bar) {
        if (elect_one()) tc5::commit(smem_u32(bar));
        __syncwarp();
      };
      // every lane waits; the warp proceeds only on a decision common to all lanes
      auto wait_bar = [&](uint64_t* bar, uint32_t parity) -> bool {
        const bool r = __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, kErrPrefillWait));
        tc5::fence_after();
        return r;
      };
      auto wait_kv = [&](int u) -> bool { return wait_bar(&kv_full[u % Cfg::kStages], (u / Cfg::kStages) & 1); };
      auto wait_p = [&](int t, int hf, int j) -> bool { return wait_bar(&p_half[2 * t + hf], j & 1); };
      // PV of tile t for KV tile j, started on keys [64, 128) of P while the
      // softmax still exponentiates keys [0, 64)
      auto issue_pv = [&](int t, int u, bool acc, int j) -> bool {
        const uint32_t sc = t ? s1c : s0c, oc = t ? o1c : o0c;
        if (!wait_p(t, 1, j)) return false;
        issue_pv_half(sc, oc, u, acc, 1);
        if (!wait_p(t, 0, j)) return false;
        issue_pv_half(sc, oc, u, acc, 0);
        return true;
      };
      auto release = [&](int u) { commit(&kv_empty[u % Cfg::kStages]); };
      const bool two = nt == 2;

      if constexpr (Cfg::kTiles == 1) {
        // One query tile (D = 256): S is double-buffered in TMEM columns
        // [0, 128) and [128, 256), and the order S(0) | S(j+1) PV(j) lets the
        // tensor core compute the next logits while the softmax of step j
        // runs.  S(j+1) overwrites the buffer PV(j-1) read P from, issued
        // before it.  After each PV, o_full[1] tracks its completion: the
        // softmax of step j+1 waits for it before it rescales O.
        auto sbuf = [&](int j) { return (j & 1) ? s1c : s0c; };
        auto wait_p1 = [&](int j, int hf) { return wait_bar(&p_half[2 * (j & 1) + hf], (j >> 1) & 1); };
        bool ok = wait_bar(q_full, 0) && wait_kv(0);
        if (ok) {
          issue_s(dq0, s0c, 0);
          commit(&s_full[0]);
          release(0);
        }
        for (int j = 0; j < nkv && ok; ++j) {
          if (j + 1 < nkv) {
            const int uk = 2 * (j + 1);
            if (!wait_kv(uk)) { ok = false; break; }
            issue_s(dq0, sbuf(j + 1), uk);
            commit(&s_full[(j + 1) & 1]);
            release(uk);
          }
          const int uv = 2 * j + 1;
          if (!wait_kv(uv) || !wait_p1(j, 1)) { ok = false; break; }
          issue_pv_half(sbuf(j), o0c, uv, j > 0, 1);
          if (!wait_p1(j, 0)) { ok = false; break; }
          issue_pv_half(sbuf(j), o0c, uv, j > 0, 0);
          commit(&o_full[1]);
          release(uv);
          if (j == nkv - 1) commit(&o_full[0]);
        }
      } else {
        bool ok = wait_bar(q_full, 0) && wait_kv(0);
        if (ok) {
          issue_s(dq0, s0c, 0);
          commit(&s_full[0]);
          if (two) {
            issue_s(dq1, s1c, 0);
            commit(&s_full[1]);
          }
          release(0);
          ok = wait_kv(1) && issue_pv(0, 1, false, 0);
          if (ok && nkv == 1) commit(&o_full[0]);
        }
        for (int j = 1; j < nkv && ok; ++j) {
          const int uk = 2 * j, uv = 2 * j + 1;
          if (!wait_kv(uk)) { ok = false; break; }
          issue_s(dq0, s0c, uk);
          commit(&s_full[0]);
          if (two && !issue_pv(1, uv - 2, j - 1 > 0, j - 1)) { ok = false; break; }
          release(uv - 2);              // V_{j-1}: both of its PV products are issued
          if (two) {
            issue_s(dq1, s1c, uk);
            commit(&s_full[1]);
          }
          release(uk);                  // K_j: both S products are issued
          if (!wait_kv(uv)) { ok = false; break; }
          if (!issue_pv(0, uv, true, j)) { ok = false; break; }
          if (j == nkv - 1) commit(&o_full[0]);
        }
        if (ok && two && issue_pv(1, 2 * nkv - 1, nkv - 1 > 0, nkv - 1)) commit(&o_full[1]);
      }
      // every MMA the elected lane issued has completed before TMEM is released
      commit(drain);
      mbar_drain(drain, 0, 20000000ull);
    }
  } else {
    // ======================= softmax + epilogue (warps 0-7)
    const int t = warp >> 2;           // query tile
    const int lg = warp & 3;           // TMEM lane group
    const int row = lg * 32 + lane;    // row inside the tile
    if (t < nt) {
      const uint32_t lane_base = static_cast<uint32_t>(lg * 32) << 16;
      // one query tile: S of step j in buffer j & 1 (columns [0,128) / [128,256))
      constexpr bool kSDouble = Cfg::kTiles == 1;
      const uint32_t s_base = tmem + lane_base + (t == 0 ? Cfg::kSCol0 : Cfg::kSCol1);
      const uint32_t o_addr = tmem + lane_base + (t == 0 ? Cfg::kOCol0 : Cfg::kOCol1);
      const int qi = qblk * Cfg::kRows + t * kPfBM + row;  // row index inside the sequence
      const bool row_valid = qi < len_q;
      const int row_keys = a.causal ? min(max(qi + causal_off + 1, 0), len_k) : len_k;  // keys this row sees
      bool ok = true;

      // smooth_k: delta = scale*log2(e) * (q_i . mean(K)), the shift smoothing removes
      float delta = 0.f;
      if (a.kmean != nullptr || a.kpartial != nullptr) {
        const float* mu;
        if (a.kpartial != nullptr) {
          // mean over this call's KV range from the per-256-key column sums.
          // The column-sum kernel may still be running (this grid can be its
          // programmatic dependent): wait for its completion first (a no-op
          // otherwise).  Loads go out sixteen at a time (all of them for a 4096-key
          // range: one round trip); the sum keeps chunk order.
          asm volatile("griddepcontrol.wait;" ::: "memory");
          float* mu_s = reinterpret_cast<float*>(smem + Cfg::kOffMu) + t * D;
          const int nch = (len_k + 255) / 256;
          const int64_t cstride = static_cast<int64_t>(nseq) * a.Hkv * D;
          for (int d = row; d < D; d += kPfBM) {
            const float* pp = a.kpartial + (static_cast<int64_t>(seq) * a.Hkv + hkv) * D + d;
            float sum = 0.f;
            int c = 0;
            for (; c + 16 <= nch; c += 16) {
              float x[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) x[i] = pp[(c + i) * cstride];
#pragma unroll
              for (int i = 0; i < 16; ++i) sum += x[i];
            }
            for (; c < nch; ++c) sum += pp[c * cstride];
            mu_s[d] = sum / static_cast<float>(len_k);
          }
          named_barrier_sync(1 + t, kPfBM);
          mu = mu_s;
        } else {
          mu = a.kmean + (static_cast<int64_t>(seq) * a.Hkv + hkv) * D;
        }
        ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, abort_flag, kErrPrefillWait));
        if (ok) {
          float acc = 0.f;
#pragma unroll
          for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
            const uint8_t* qrow = qtile[t] + bx * Cfg::kBoxBytes;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 u = *reinterpret_cast<const uint4*>(qrow + sw128(row, c));
              const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = unpack2<T>(w[e]);
                const int d = bx * 64 + c * 8 + 2 * e;
                acc = fmaf(f.x, mu[d], acc);
                acc = fmaf(f.y, mu[d + 1], acc);
              }
            }
          }
          delta = acc * a.scale_log2;
        }
      }

      // logits seen by the softmax are the smoothed ones: K' = K - mean either
      // materialised (K' in the MMA) or applied here as a per-row fp32 shift
      const float bias_shift = a.shift_logits ? delta : 0.f;
      // int8: a logit is s32 codes-product x (Q block scale x K block scale);
      // the K scale of the next KV tile is fetched one tile ahead
      float qsc = 1.f, ks_next = 1.f;
      const float* ksc = nullptr;
      if constexpr (kI8) {
        qsc = __ldg(a.qscale + (static_cast<int64_t>(b) * a.Hq + h) * ((a.Sq + 127) / 128) + qblk * 2 + t);
        ksc = a.kscale + (static_cast<int64_t>(b) * a.Hkv + hkv) * ((a.Sk + 127) / 128);
        ks_next = __ldg(ksc);
        if (row_valid) delta = __ldg(a.dq + (static_cast<int64_t>(b) * a.Hq + h) * a.Sq + qi);
      }
      float m_run = -INFINITY;  // running max of the (smoothed) log2-domain logits, possibly stale
      float l_run = 0.f;
      for (int j = 0; j < nkv && ok; ++j) {
        const int sb = kSDouble ? (j & 1) : t;  // S buffer, and index of its S and P barriers
        const uint32_t s_addr = kSDouble ? tmem + lane_base + (sb ? Cfg::kSCol1 : Cfg::kSCol0) : s_base;
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], kSDouble ? (j >> 1) & 1 : j & 1, abort_flag,
                                               kErrPrefillWait));
        if (!ok) break;
        tc5::fence_after();
        float sl2 = a.scale_log2;  // log2 units per logit unit of this tile
        if constexpr (kI8) {
          sl2 = a.scale_log2 * qsc * ks_next;
          if (j + 1 < nkv) ks_next = __ldg(ksc + j + 1);
        }
        // pass 1 over S (two halves of 64 columns read from TMEM): the row max;
        // the second half's logits stay in sh for the exponent pass
        const int n_valid = row_keys - j * kPfBN;
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = -INFINITY;
        float sh[64];
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {
          tc5::ld32(s_addr + hf * 64, *reinterpret_cast<float(*)[32]>(&sh[0]));
          tc5::ld32(s_addr + hf * 64 + 32, *reinterpret_cast<float(*)[32]>(&sh[32]));
          tc5::wait_ld();
          if constexpr (kI8) s32_to_magic_64(sh);
          if (n_valid < kPfBN) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (hf * 64 + c >= n_valid) sh[c] = -INFINITY;
          }
#pragma unroll
          for (int c = 0; c < 64; c += 16)
#pragma unroll
            for (int e = 0; e < 8; ++e) mx8[e] = fmax3(mx8[e], sh[c + e], sh[c + 8 + e]);
        }
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
        const float t_max = fmaf(mx, sl2, kI8 ? -fmaf(kMagic, sl2, bias_shift) : -bias_shift);
        const float m_new = fmaxf(m_run, t_max);
        const bool rescale = m_new > m_run + kPfRescaleThreshold;
        float alpha = 1.f;
        if (rescale) {
          alpha = ex2_approx(m_run - m_new);
          m_run = m_new;
        }
        l_run *= alpha;
        if (j > 0 && __any_sync(0xffffffffu, rescale)) {
          // correction before this tile's P is published: O_t holds the PV
          // products of tiles < j, complete since S_t(j) was issued after them
          // (one query tile: S(j) is issued before PV(j-1), whose completion
          // o_full[1] reports; PV(j-2) completed before S(j), so that wait is at
          // most one phase behind)
          if constexpr (kSDouble) {
            ok = __all_sync(0xffffffffu, mbar_wait(&o_full[1], (j - 1) & 1, abort_flag, kErrPrefillWait));
            if (!ok) break;
            tc5::fence_after();
          }
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tc5::ld32(o_addr + c * 32, o);
            tc5::wait_ld();
            const uint64_t al2 = f2_pack(alpha, alpha);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 r = f2_unpack(fmul2(f2_pack(o[e], o[e + 1]), al2));
              o[e] = r.x;
              o[e + 1] = r.y;
            }
            tc5::st32(o_addr + c * 32, o);
          }
          tc5::wait_st();
        }
        // p = 2^(s * scale*log2(e) - max), packed as 16-bit pairs into TMEM and
        // published per 64-key half on its own barrier, so PV starts on one half
        // while the other is exponentiated.  Keys [64, 128) go first, from the
        // registers of the max pass; their P lands in columns [64, 96) (logits
        // already read).  Keys [0, 64) are then reloaded (the load is issued
        // before the first half's store is waited for) and their P lands in
        // columns [0, 32).
        // A row that has seen no key yet (causal rows before the first key)
        // keeps m = -inf: exponentiate its masked logits against 0 instead.
        float neg_bias = -((m_run == -INFINITY ? 0.f : m_run) + bias_shift);
        if constexpr (kI8) neg_bias = fmaf(-kMagic, sl2, neg_bias);  // the logits carry +kMagic
        const uint64_t sc2 = f2_pack(sl2, sl2);
        const uint64_t nb2 = f2_pack(neg_bias, neg_bias);
        uint64_t ps2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
        const bool full_tile = n_valid >= kPfBN;
        uint32_t pk[32];
        if (full_tile) exp_pack_64<true, T>(sh, sc2, nb2, pk, ps2);
        else exp_pack_64<false, T>(sh, sc2, nb2, pk, ps2);
        tc5::st16(s_addr + 64, *reinterpret_cast<const uint32_t(*)[16]>(&pk[0]));
        tc5::st16(s_addr + 80, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16]));
        tc5::ld32(s_addr, *reinterpret_cast<float(*)[32]>(&sh[0]));
        tc5::ld32(s_addr + 32, *reinterpret_cast<float(*)[32]>(&sh[32]));
        tc5::wait_st();
        tc5::fence_before();
        mbar_arrive(&p_half[2 * sb + 1]);
        tc5::wait_ld();
        if constexpr (kI8) s32_to_magic_64(sh);
        if (!full_tile) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= n_valid) sh[c] = -INFINITY;
        }
        if (full_tile) exp_pack_64<true, T>(sh, sc2, nb2, pk, ps2);
        else exp_pack_64<false, T>(sh, sc2, nb2, pk, ps2);
        tc5::st16(s_addr, *reinterpret_cast<const uint32_t(*)[16]>(&pk[0]));
        tc5::st16(s_addr + 16, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16]));
        tc5::wait_st();
        tc5::fence_before();
        mbar_arrive(&p_half[2 * sb + 0]);
        const float2 psa = f2_unpack(ps2[0]), psb = f2_unpack(ps2[1]);
        l_run += (psa.x + psa.y) + (psb.x + psb.y);
      }

      // ---------------- epilogue: O / l and LSE for this thread's row
      // O rows are staged in an idle K/V ring buffer (this tile's last K tile
      // for tile 0, the last V tile for tile 1: both consumed once o_full
      // fires) in the layout of the TMA's 128-byte-swizzled 64-column boxes
      // (16-byte chunk ch of row r in box ch / 8 at position (ch mod 8) ^ (r mod
      // 8): no shared-memory bank conflicts), then one thread writes the tile
      // with bulk tensor stores and waits only until they have read shared
      // memory, so the CTA can retire while the writes drain.  A varlen tile
      // whose last rows belong to the next sequence is written row by row
      // instead (coalesced 16-byte stores).
      constexpr int kChunks = D / 8;  // 16-byte chunks per row
      uint8_t* stg = ring + ((2 * nkv - 2 + t) % Cfg::kStages) * Cfg::kKVTileBytes;
      auto stg_off = [](int r, int ch) -> uint32_t {
        return static_cast<uint32_t>(ch >> 3) * Cfg::kBoxBytes + sw128(static_cast<uint32_t>(r), static_cast<uint32_t>(ch & 7));
      };
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_full[t], 0, abort_flag, kErrPrefillWait));
      if (ok) {
        tc5::fence_after();
        const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;  // no key: O = 0, LSE = -inf
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tc5::ld32(o_addr + c * 32, o);
          tc5::wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack2<T>(o[2 * e] * inv_l, o[2 * e + 1] * inv_l);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int ch = c * 4 + i;
            *reinterpret_cast<uint4*>(stg + stg_off(row, ch)) =
                make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
        if (row_valid && a.lse != nullptr) a.lse[lse_idx(qi)] = m_run + __log2f(l_run) + delta;
        fence_proxy_async_smem();  // the staged rows become visible to the bulk stores
      }
      // every warp of the tile arrives here (an aborted one too, so none waits
      // forever); after an abort the copied rows are garbage and the device
      // error word says so
      named_barrier_sync(1 + t, kPfBM);
      if (ok) {
        const int row0 = qblk * Cfg::kRows + t * kPfBM;
        // dense rows past S_q lie outside the map and are not written
        if (a.layout != 2 || row0 + kPfBM <= len_q) {
          if (row == 0) {
            const int s = q_row0 + t * kPfBM;
            const int bo = a.layout == 2 ? 0 : chunk * a.B + b;
#pragma unroll
            for (int bx = 0; bx < D / 64; ++bx) {
              if (a.layout == 0) tma_store_4d(&tmO, stg + bx * Cfg::kBoxBytes, bx * 64, s, h, bo);
              else tma_store_4d(&tmO, stg + bx * Cfg::kBoxBytes, bx * 64, h, s, bo);
            }
            bulk_commit_group();
            bulk_wait_read_all();
          }
        } else {
#pragma unroll 4
          for (int i = 0; i < kChunks; ++i) {
            const int idx = i * kPfBM + row;
            const int r = idx / kChunks, ch = idx % kChunks;
            if (row0 + r < len_q) {
              const uint4 val = *reinterpret_cast<const uint4*>(stg + stg_off(r, ch));
              *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(out_row(row0 + r)) + ch * 16) = val;
            }
          }
        }
      }
    }
  }

  tc5::fence_before();
  __syncthreads();
  if (warp == 9) {
    tc5::fence_after();
    tc5::dealloc(tmem, Cfg::kTmemCols);
  }
}

// Device-side varlen planner (one block): orders sequences by kv length,
// longest first (ties by index), and writes prefix sums of their work items
// (Hq * ceil(len_q / rows_per_cta)).  order[B], offsets[B+1].
__global__ void __launch_bounds__(1024) varlen_plan_kernel(const int* __restrict__ cu_q, const int* __restrict__ cu_k,
                                                            int B, int Hq, int rows_per_cta, int* __restrict__ order,
                                                            int* __restrict__ offsets) {
  for (int bb = threadIdx.x; bb < B; bb += blockDim.x) {
    const int lk = cu_k[bb + 1] - cu_k[bb];
    int rank = 0;
    for (int o = 0; o < B; ++o) {
      const int lo = cu_k[o + 1] - cu_k[o];
      rank += (lo > lk) || (lo == lk && o < bb);
    }
    order[rank] = bb;
  }
  __syncthreads();
  // block-wide exclusive scan of item counts in `order`
  __shared__ int part[1024];
  const int per = (B + blockDim.x - 1) / blockDim.x;
  const int beg = min(B, static_cast<int>(threadIdx.x) * per);
  const int end = min(B, beg + per);
  int local = 0;
  for (int i = beg; i < end; ++i) {
    const int bb = order[i];
    const int lq = cu_q[bb + 1] - cu_q[bb];
    local += Hq * ((lq + rows_per_cta - 1) / rows_per_cta);
  }
  part[threadIdx.x] = local;
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int i = 0; i < static_cast<int>(blockDim.x); ++i) {
      const int v = part[i];
      part[i] = run;
      run += v;
    }
    offsets[B] = run;
  }
  __syncthreads();
  int run = part[threadIdx.x];
  for (int i = beg; i < end; ++i) {
    offsets[i] = run;
    const int bb = order[i];
    const int lq = cu_q[bb + 1] - cu_q[bb];
    run += Hq * ((lq + rows_per_cta - 1) / rows_per_cta);
  }
}

}  // namespace skv
