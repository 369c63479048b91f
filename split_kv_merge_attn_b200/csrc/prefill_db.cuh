// Prefill / varlen attention forward with a per-row log2 LSE on sm_100a, for
// head dimensions 64 and 128, with the S tiles double-buffered in TMEM.
//
// Same quantity, inputs and outputs as prefill_kernel (prefill.cuh): O_i =
// softmax_j(scale q_i . k_j) V and LSE_i = log2 sum_j exp(scale q_i . k_j)
// over the original logits, one LSE per row written by the thread that owns
// the row's TMEM lane (ARK return_lse issue, "Expected:").
//
// What differs is the pipeline.  In prefill_kernel, P_t(j) overwrites S_t(j)
// in TMEM, so S_t(j+1) can only be computed after PV_t(j) is issued, and each
// query tile's chain S -> softmax -> PV -> S runs in series.  Here a KV step
// is 64 keys and each tile owns two 64-column S buffers:
//   TMEM: O_0 [0, D), O_1 [D, 2D), S_t^b at 256 + (2t + b) * 64 (b = j mod 2)
// so the MMA warp issues S_t(j+1) into the other buffer while the softmax
// warps work on S_t(j); the softmax warps never wait for an S product after
// the first, and the tensor pipe has S work queued while P is being made.
// Issue order of step j (one elected lane of the MMA warp):
//   S_0(j+1)  PV_0(j)  S_1(j+1)  PV_1(j)
// S_t(j+1) reuses the buffer of P_t(j-1), whose PV_t(j-1) was issued in the
// previous step (tcgen05 MMAs of one thread execute in issue order).
// The softmax of step j raises the running max lazily (by more than 8 log2
// units, as in prefill_kernel); before it rescales O_t it waits for PV_t(j-1)
// to complete (pv_done), since that product is not ordered before S_t(j).
//
// Warp roles (320 threads): warps 0-3 softmax/epilogue of query tile 0,
// warps 4-7 of tile 1, warp 8 TMA producer (Q once; K_j and V_j as 64-key
// tiles into a ring of NS buffers, 128-byte swizzle, no multicast), warp 9
// TMEM allocation and the MMAs.  All waits are bounded.
#pragma once

#include "prefill.cuh"

namespace skv {

constexpr int kDbBN = 64;  // keys per KV step

template <int D>
struct PfDbCfg {
  static constexpr int kBoxes = D / 64;                    // 64-element column boxes per row
  static constexpr int kQBoxBytes = kPfBM * 128;           // 128 rows x 128 bytes
  static constexpr int kKVBoxBytes = kDbBN * 128;          // 64 keys x 128 bytes
  static constexpr int kQTileBytes = kBoxes * kQBoxBytes;
  static constexpr int kKVTileBytes = kBoxes * kKVBoxBytes;  // one ring buffer: a K or a V tile
  static constexpr int kStages = (D == 64) ? 16 : 10;
  static constexpr int kRingBytes = kStages * kKVTileBytes;
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = 2 * kQTileBytes;
  static constexpr int kOffBar = kOffRing + kRingBytes;
  // q_full, kv_full[NS], kv_empty[NS], s_full[2][2], p_full[2][2], pv_done[2], drain
  static constexpr int kNumBars = 1 + 2 * kStages + 4 + 4 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffMu = kOffMisc + 16;           // [2][D] fp32 mean of K (smooth_k)
  static constexpr int kSmemBytes = kOffMu + 2 * D * 4 + 1024;
  static constexpr int kSCol = 256;                      // S_t^b at kSCol + (2t + b) * 64
  static constexpr uint32_t kTmemCols = 512;
  static_assert(2 * D <= kSCol, "TMEM columns");
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  // the epilogue stages a tile's O rows in two ring buffers no load reaches
  static_assert(kStages >= 5 && 2 * kKVTileBytes >= kPfBM * D * 2, "epilogue staging");
};

template <int D, typename T>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_db_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const PrefillArgs a) {
  using Cfg = PfDbCfg<D>;
  static_assert(D == 64 || D == 128, "two query tiles and two S buffers each fit TMEM for D <= 128");
  constexpr int kIsBf16 = std::is_same<T, __nv_bfloat16>::value ? 1 : 0;
  constexpr uint32_t kIdescQK = tc5::idesc_f16(kIsBf16, 0, kPfBM, kDbBN);
  constexpr uint32_t kIdescPV = tc5::idesc_f16(kIsBf16, 1, kPfBM, D);
  constexpr int kRowsPerCta = 2 * kPfBM;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + Cfg::kStages;
  uint64_t* s_full = kv_empty + Cfg::kStages;  // [tile][buffer]
  uint64_t* p_full = s_full + 4;               // [tile][buffer], 128 arrivals
  uint64_t* pv_done = p_full + 4;              // [tile]: committed after every PV_t
  uint64_t* drain = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kOffMisc + 8);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = a.Hq / a.Hkv;

  // ---------------- work item (the same decomposition as prefill_kernel, 256 rows per CTA)
  int b, h, qblk, len_q, len_k, q_row0, k_row0, bcoord;
  int chunk = 0;
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
    const int nblk = (len_q + kRowsPerCta - 1) / kRowsPerCta;
    if (a.causal) {
      qblk = nblk - 1 - rem / a.Hq;
      h = rem % a.Hq;
    } else {
      h = rem / nblk;
      qblk = rem % nblk;
    }
    q_row0 = a.cu_q[b] + qblk * kRowsPerCta;
    k_row0 = a.cu_k[b];
    bcoord = 0;
  } else {
    int item = blockIdx.x;
    if (a.nchunks > 1) {
      const int per = a.B * a.Hq * a.nqb;
      chunk = item / per;
      item -= chunk * per;
    }
    if (a.causal) {
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
    q_row0 = qblk * kRowsPerCta;
    k_row0 = a.kvb[chunk];
    bcoord = b;
  }
  const int seq = b * a.nchunks + chunk;
  const int nseq = a.B * a.nchunks;
  const int hkv = h / G;
  const int rows_here = min(kRowsPerCta, len_q - qblk * kRowsPerCta);
  const int nt = rows_here > kPfBM ? 2 : 1;
  const int causal_off = len_k - len_q;
  const int kv_end = a.causal ? min(max(qblk * kRowsPerCta + rows_here + causal_off, 0), len_k) : len_k;
  const int nkv = (kv_end + kDbBN - 1) / kDbBN;

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
    for (int r = tid; r < rows_here; r += kPfThreads) {
      const int qi = qblk * kRowsPerCta + r;
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
      const bool per_thread = &bars[i] >= &p_full[0] && &bars[i] < &p_full[4];
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

  uint8_t* qtile[2] = {smem + Cfg::kOffQ, smem + Cfg::kOffQ + Cfg::kQTileBytes};
  uint8_t* ring = smem + Cfg::kOffRing;

  if (warp == 8) {
    // ======================= TMA producer: Q, then K_j (u = 2j) and V_j (u = 2j + 1)
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const bool hnd = (a.layout == 0);
      mbar_arrive_expect_tx(q_full, nt * Cfg::kQTileBytes);
      for (int t = 0; t < nt; ++t) {
        const int s = q_row0 + t * kPfBM;
#pragma unroll
        for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
          if (hnd) tma_load_4d(qtile[t] + bx * Cfg::kQBoxBytes, &tmQ, q_full, bx * 64, s, h, bcoord);
          else tma_load_4d(qtile[t] + bx * Cfg::kQBoxBytes, &tmQ, q_full, bx * 64, h, s, bcoord);
        }
      }
      int issued = 0;
      bool ok = true;
      for (int u = 0; u < 2 * nkv && ok; ++u) {
        const int buf = u % Cfg::kStages;
        if (u >= Cfg::kStages &&
            !mbar_wait(&kv_empty[buf], ((u / Cfg::kStages) & 1) ^ 1, abort_flag, kErrPrefillWait)) {
          ok = false;
          break;
        }
        const CUtensorMap* m = (u & 1) ? &tmV : &tmK;
        const int s = k_row0 + (u >> 1) * kDbBN;
        mbar_arrive_expect_tx(&kv_full[buf], Cfg::kKVTileBytes);
#pragma unroll
        for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
          uint8_t* dst = ring + buf * Cfg::kKVTileBytes + bx * Cfg::kKVBoxBytes;
          if (hnd) tma_load_4d(dst, m, &kv_full[buf], bx * 64, s, hkv, bcoord);
          else tma_load_4d(dst, m, &kv_full[buf], bx * 64, hkv, s, bcoord);
        }
        issued = u + 1;
      }
      if (*abort_flag) {
        mbar_drain(q_full, 0, 20000000ull);
        for (int u = max(0, issued - Cfg::kStages); u < issued; ++u)
          mbar_drain(&kv_full[u % Cfg::kStages], (u / Cfg::kStages) & 1, 20000000ull);
      }
    }
  } else if (warp == 9) {
    // ======================= MMA issuer (whole warp in step, one elected lane issues)
    const uint32_t ring_addr = smem_u32(ring);
    const uint64_t dq0 = tc5::smem_desc(smem_u32(qtile[0]), 16, 1024);
    const uint64_t dq1 = tc5::smem_desc(smem_u32(qtile[1]), 16, 1024);
    const uint64_t dk_base = tc5::smem_desc(ring_addr, 16, 1024);
    const uint64_t dv_base = tc5::smem_desc(ring_addr, Cfg::kKVBoxBytes, 1024);
    const bool two = nt == 2;
    auto s_col = [&](int t, int bb) -> uint32_t { return tmem + Cfg::kSCol + (2 * t + bb) * 64; };
    // S_t(j) = Q_t K_j^T into buffer j mod 2: D / 16 MMAs of M = 128, N = 64, K = 16
    auto issue_s = [&](int t, int j) {
      const uint64_t dk = dk_base + static_cast<uint64_t>((((2 * j) % Cfg::kStages) * Cfg::kKVTileBytes) >> 4);
      const uint32_t sc = s_col(t, j & 1);
      const uint64_t dq = t ? dq1 : dq0;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t oq = static_cast<uint64_t>(((kk >> 2) * Cfg::kQBoxBytes + (kk & 3) * 32) >> 4);
          const uint64_t ok_ = static_cast<uint64_t>(((kk >> 2) * Cfg::kKVBoxBytes + (kk & 3) * 32) >> 4);
          tc5::mma_ss(sc, dq + oq, dk + ok_, kIdescQK, kk > 0 ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    // O_t (+)= P_t(j) V_j: P of key block kk (16 keys) in columns kk * 8 of S_t's buffer
    auto issue_pv = [&](int t, int j) {
      const uint64_t dv = dv_base + static_cast<uint64_t>((((2 * j + 1) % Cfg::kStages) * Cfg::kKVTileBytes) >> 4);
      const uint32_t sc = s_col(t, j & 1);
      const uint32_t oc = tmem + t * D;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kDbBN / 16; ++kk)
          tc5::mma_ts(oc, sc + kk * 8, dv + static_cast<uint64_t>((kk * 2048) >> 4), kIdescPV,
                      (j > 0 || kk > 0) ? 1u : 0u);
      }
      __syncwarp();
    };
    auto commit = [&](uint64_t* bar) {
      if (elect_one()) tc5::commit(smem_u32(bar));
      __syncwarp();
    };
    auto wait_bar = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool r = __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, kErrPrefillWait));
      tc5::fence_after();
      return r;
    };
    auto wait_kv = [&](int u) -> bool { return wait_bar(&kv_full[u % Cfg::kStages], (u / Cfg::kStages) & 1); };

    bool ok = wait_bar(q_full, 0) && wait_kv(0);
    if (ok) {
      for (int t = 0; t < nt; ++t) {
        issue_s(t, 0);
        commit(&s_full[2 * t]);
      }
      commit(&kv_empty[0]);  // K_0: both S products issued
    }
    for (int j = 0; j < nkv && ok; ++j) {
      const int bb = j & 1;
      const bool more = j + 1 < nkv;
      if (more) {
        if (!wait_kv(2 * j + 2)) { ok = false; break; }
        issue_s(0, j + 1);
        commit(&s_full[0 * 2 + (bb ^ 1)]);
      }
      if (!wait_kv(2 * j + 1)) { ok = false; break; }
      if (!wait_bar(&p_full[0 * 2 + bb], (j >> 1) & 1)) { ok = false; break; }
      issue_pv(0, j);
      commit(&pv_done[0]);
      if (two) {
        if (more) {
          issue_s(1, j + 1);
          commit(&s_full[1 * 2 + (bb ^ 1)]);
        }
        if (!wait_bar(&p_full[1 * 2 + bb], (j >> 1) & 1)) { ok = false; break; }
        issue_pv(1, j);
        commit(&pv_done[1]);
      }
      if (more) commit(&kv_empty[(2 * j + 2) % Cfg::kStages]);  // K_{j+1}: its S products issued
      commit(&kv_empty[(2 * j + 1) % Cfg::kStages]);             // V_j: its PV products issued
    }
    // every MMA the elected lane issued has completed before TMEM is released
    commit(drain);
    mbar_drain(drain, 0, 20000000ull);
  } else {
    // ======================= softmax + epilogue (warps 0-7)
    const int t = warp >> 2;
    const int lg = warp & 3;
    const int row = lg * 32 + lane;
    if (t < nt) {
      const uint32_t lane_base = static_cast<uint32_t>(lg * 32) << 16;
      const uint32_t o_addr = tmem + lane_base + t * D;
      const int qi = qblk * kRowsPerCta + t * kPfBM + row;
      const bool row_valid = qi < len_q;
      const int row_keys = a.causal ? min(max(qi + causal_off + 1, 0), len_k) : len_k;
      bool ok = true;

      // smooth_k: delta = scale*log2(e) * (q_i . mean(K))
      float delta = 0.f;
      if (a.kmean != nullptr || a.kpartial != nullptr) {
        const float* mu;
        if (a.kpartial != nullptr) {
          float* mu_s = reinterpret_cast<float*>(smem + Cfg::kOffMu) + t * D;
          for (int d = row; d < D; d += kPfBM) {
            const int nch = (len_k + 255) / 256;
            float sum = 0.f;
            for (int c = 0; c < nch; ++c)
              sum += __ldg(a.kpartial + ((static_cast<int64_t>(c) * nseq + seq) * a.Hkv + hkv) * D + d);
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
            const uint8_t* qrow = qtile[t] + bx * Cfg::kQBoxBytes;
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
      const float bias_shift = a.shift_logits ? delta : 0.f;
      const float sl2 = a.scale_log2;
      const uint64_t sc2 = f2_pack(sl2, sl2);
      float m_run = -INFINITY;
      float l_run = 0.f;
      for (int j = 0; j < nkv && ok; ++j) {
        const int bb = j & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[2 * t + bb], (j >> 1) & 1, abort_flag, kErrPrefillWait));
        if (!ok) break;
        tc5::fence_after();
        const uint32_t s_addr = tmem + lane_base + Cfg::kSCol + (2 * t + bb) * 64;
        float sh[64];
        tc5::ld32(s_addr, *reinterpret_cast<float(*)[32]>(&sh[0]));
        tc5::ld32(s_addr + 32, *reinterpret_cast<float(*)[32]>(&sh[32]));
        tc5::wait_ld();
        const int n_valid = row_keys - j * kDbBN;
        const bool full_tile = n_valid >= kDbBN;
        if (!full_tile) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= n_valid) sh[c] = -INFINITY;
        }
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; c += 16)
#pragma unroll
          for (int e = 0; e < 8; ++e) mx8[e] = fmax3(mx8[e], sh[c + e], sh[c + 8 + e]);
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
        const float t_max = fmaf(mx, sl2, -bias_shift);
        const float m_new = fmaxf(m_run, t_max);
        const bool rescale = m_new > m_run + kPfRescaleThreshold;
        float alpha = 1.f;
        if (rescale) {
          alpha = ex2_approx(m_run - m_new);
          m_run = m_new;
        }
        l_run *= alpha;
        if (j > 0 && __any_sync(0xffffffffu, rescale)) {
          // O_t holds the PV products of steps < j once PV_t(j-1) completes
          // (it is issued after S_t(j), so it may still be running)
          ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[t], (j - 1) & 1, abort_flag, kErrPrefillWait));
          if (!ok) break;
          tc5::fence_after();
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
        // p = 2^(s * scale*log2(e) - max) into columns [0, 32) of this buffer;
        // a row that has seen no key yet keeps m = -inf: exponentiate against 0
        const float neg_bias = -((m_run == -INFINITY ? 0.f : m_run) + bias_shift);
        const uint64_t nb2 = f2_pack(neg_bias, neg_bias);
        uint64_t ps2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
        uint32_t pk[32];
        if (full_tile) exp_pack_64<true, T>(sh, sc2, nb2, pk, ps2);
        else exp_pack_64<false, T>(sh, sc2, nb2, pk, ps2);
        tc5::st16(s_addr, *reinterpret_cast<const uint32_t(*)[16]>(&pk[0]));
        tc5::st16(s_addr + 16, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16]));
        // pv_done[t] is waited on by parity, which is only unambiguous while
        // the barrier is at most one phase past the awaited one: the last
        // step observes PV_t(nkv-2) here, before PV_t(nkv-1) can be issued,
        // so that the epilogue's wait for PV_t(nkv-1) is unambiguous too
        if (j == nkv - 1 && j > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[t], (j - 1) & 1, abort_flag, kErrPrefillWait));
          if (!ok) break;
        }
        tc5::wait_st();
        tc5::fence_before();
        mbar_arrive(&p_full[2 * t + bb]);
        const float2 psa = f2_unpack(ps2[0]), psb = f2_unpack(ps2[1]);
        l_run += (psa.x + psa.y) + (psb.x + psb.y);
      }

      // ---------------- epilogue: O / l and LSE for this thread's row.
      // O rows are staged in two ring buffers no load reaches any more (the
      // two after the last one loaded for tile 0, the next two for tile 1;
      // their previous tiles were consumed long before) and written with
      // coalesced 16-byte stores; chunk c of row r sits at c ^ (r mod chunks).
      constexpr int kRowBytes = D * 2;
      constexpr int kChunks = kRowBytes / 16;
      constexpr int kRowsPerBuf = Cfg::kKVTileBytes / kRowBytes;
      uint8_t* stg0 = ring + ((2 * nkv + 2 * t) % Cfg::kStages) * Cfg::kKVTileBytes;
      uint8_t* stg1 = ring + ((2 * nkv + 2 * t + 1) % Cfg::kStages) * Cfg::kKVTileBytes;
      auto stg_row = [&](int r) -> uint8_t* {
        return (r < kRowsPerBuf ? stg0 + r * kRowBytes : stg1 + (r - kRowsPerBuf) * kRowBytes);
      };
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[t], (nkv - 1) & 1, abort_flag, kErrPrefillWait));
      if (ok) {
        tc5::fence_after();
        const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
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
            *reinterpret_cast<uint4*>(stg_row(row) + ((ch ^ (row % kChunks)) * 16)) =
                make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
        if (row_valid && a.lse != nullptr) a.lse[lse_idx(qi)] = m_run + __log2f(l_run) + delta;
      }
      named_barrier_sync(1 + t, kPfBM);
      if (ok) {
        const int row0 = qblk * kRowsPerCta + t * kPfBM;
#pragma unroll 4
        for (int i = 0; i < kChunks; ++i) {
          const int idx = i * kPfBM + row;
          const int r = idx / kChunks, ch = idx % kChunks;
          if (row0 + r < len_q) {
            const uint4 val = *reinterpret_cast<const uint4*>(stg_row(r) + ((ch ^ (r % kChunks)) * 16));
            *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(out_row(row0 + r)) + ch * 16) = val;
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

}  // namespace skv
