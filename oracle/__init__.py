"""FP64 CPU oracle for attention forward with a per-row log2 log-sum-exp.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
baseline leg of the benchmark may import this package.  It shares no code,
headers, tables or helpers with the CUDA library and imports nothing from it.

What it computes is the plain definition of the quantity, not the split /
online-softmax algorithm the kernels use (those are exact rewrites of it):

* For a query row q_i and the keys of the call's KV range J, the scaled logits
  are s_j = scale * q_i . k_j, and the row's LSE is reported in log2 units over
  the natural-exponential sum of the ORIGINAL (unsmoothed) logits,
  LSE_i = log2(sum_j exp(s_j)).  (ARK return_lse issue, "Problem Description",
  "Expected:" sentence, and the repro's ``ref_lse_log2``, which divides
  ``torch.logsumexp(scale * q @ k^T)`` by ln 2.)
* O_i = sum_j exp(s_j) v_j / sum_j exp(s_j).
* An empty KV range gives O_i = 0 and LSE_i = -inf (reading of the ExecuTorch
  split-K PR review, item 3: every partial slot is written, also for empty
  splits).

All arithmetic is float64 on inputs widened exactly from their storage dtype.
The matrix products use numpy's matmul (a library primitive); everything else
is written out step by step.

Functions whose results have no independent pin say so in their docstring;
every other function is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

LN2 = math.log(2.0)

__all__ = [
    "to_f64", "attention_rows", "dense", "varlen", "decode", "merge",
    "kv_mean", "smooth_shift", "smoothed_attention_rows", "chunked",
    "split_bounds", "auto_num_splits", "varlen_schedule", "lse_varlen_to_dense",
    "causal_key_counts", "quantize_int8_blocks", "int8_attention_rows", "INT8_BLOCK",
]


def to_f64(x) -> np.ndarray:
    """Exact widening of a torch tensor (bf16/fp16/fp32) or array to float64."""
    try:
        import torch  # local import: the oracle itself needs only numpy
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").double().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                   key_counts: Optional[Sequence[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """O and log2-LSE for query rows q [n, D] over keys k [m, D], values v [m, D].

    Definition: ARK return_lse issue, "Expected:" (one LSE per query row, log2
    units, original logits, LSE = log2(sum_j exp(scale * q . k_j))).  The max is
    subtracted before exponentiating only to keep float64 finite; it cancels
    exactly in both O and LSE.

    key_counts (optional, one per row): row r sees only keys [0, key_counts[r])
    -- the causal mask, see ``causal_key_counts``.  A row that sees no key gets
    O = 0 and LSE = -inf, like an empty range.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n, m = q.shape[0], k.shape[0]
    if key_counts is not None:
        o = np.zeros((n, v.shape[1]))
        lse2 = np.full(n, -np.inf)
        for r in range(n):
            c = int(key_counts[r])
            if c > 0:
                orow, lrow = attention_rows(q[r:r + 1], k[:c], v[:c], scale)
                o[r], lse2[r] = orow[0], lrow[0]
        return o, lse2
    if m == 0:
        return np.zeros((n, v.shape[1])), np.full(n, -np.inf)
    s = scale * (q @ k.T)                       # [n, m] scaled logits
    mx = s.max(axis=1, keepdims=True)           # row max
    e = np.exp(s - mx)                          # exp(s_j - max)
    z = e.sum(axis=1, keepdims=True)            # sum_j exp(s_j - max)
    lse2 = (mx[:, 0] + np.log(z[:, 0])) / LN2   # natural LSE reported in log2
    o = (e @ v) / z
    return o, lse2


def causal_key_counts(n_q: int, n_k: int) -> List[int]:
    """Keys visible to each query row under the causal mask.

    Not on the pages (they describe only full, non-causal ranges); the plainest
    adjacent reading, taken for the causal variant: the n_q query rows are the
    LAST n_q positions of a sequence whose n_k keys are positions 0..n_k-1
    (bottom-right alignment, as in an autoregressive chunk whose queries follow
    the cached keys), so row i sees keys j <= i + n_k - n_q, i.e. the first
    clamp(i + n_k - n_q + 1, 0, n_k) keys.  With n_q = n_k this is the usual
    lower-triangular mask; rows i < n_q - n_k see no key.
    """
    return [min(max(i + n_k - n_q + 1, 0), n_k) for i in range(n_q)]


def _hnd(x: np.ndarray, layout: str) -> np.ndarray:
    """View a 4-D array given in ``layout`` as [B, H, S, D]."""
    if layout == "HND":
        return x
    if layout == "NHD":
        return x.transpose(0, 2, 1, 3)
    raise ValueError(layout)


def dense(q, k, v, scale: float, layout: str = "HND", rows: Optional[Sequence[Tuple[int, int, int]]] = None,
          causal: bool = False):
    """Dense attention, q [B,Hq,Sq,D] / k,v [B,Hkv,Sk,D] in HND or NHD layout.

    Returns (O in the input layout, LSE [B, Hq, Sq]) -- the 3-D dense LSE layout
    of the SGLang ``sgl_kernel::fwd`` discussion (CUDA FA: dense path 3-D).
    GQA maps query head h to kv head h // (Hq / Hkv) (reading: contiguous head
    groups; the pages only fix ``Hq % Hkv == 0``, Ascend backend record,
    ``validationCode``).

    If ``rows`` is given (a list of (b, h, i)), only those query rows are
    computed and (O rows [len, D], LSE [len]) is returned.
    causal: the mask of ``causal_key_counts`` (per row of each (b, h)).
    """
    q4, k4, v4 = _hnd(to_f64(q), layout), _hnd(to_f64(k), layout), _hnd(to_f64(v), layout)
    B, Hq, Sq, D = q4.shape
    Hkv = k4.shape[1]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    counts = causal_key_counts(Sq, k4.shape[2]) if causal else None
    if rows is not None:
        o_out = np.zeros((len(rows), D))
        l_out = np.zeros(len(rows))
        for r, (b, h, i) in enumerate(rows):
            kc = None if counts is None else [counts[i]]
            o, l = attention_rows(q4[b, h, i:i + 1], k4[b, h // G], v4[b, h // G], scale, kc)
            o_out[r], l_out[r] = o[0], l[0]
        return o_out, l_out
    o4 = np.zeros((B, Hq, Sq, D))
    lse = np.zeros((B, Hq, Sq))
    for b in range(B):
        for h in range(Hq):
            o4[b, h], lse[b, h] = attention_rows(q4[b, h], k4[b, h // G], v4[b, h // G], scale, counts)
    if layout == "NHD":
        return np.ascontiguousarray(o4.transpose(0, 2, 1, 3)), lse
    return o4, lse


def varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, scale: float, causal: bool = False):
    """Packed TND attention: q [T, Hq, D], k/v [T_k, Hkv, D].

    Sequence b owns query rows [cu_q[b], cu_q[b+1]) and keys
    [cu_k[b], cu_k[b+1]).  The LSE comes back 2-D, [Hq, T], indexed by the
    global packed row (SGLang sgl_kernel::fwd PR: the varlen path returns
    (num_heads, total_q); the Ascend backend record squeezes [T, H, 1] and
    transposes it to the same [H, T]).
    causal: the mask of ``causal_key_counts`` within each sequence.
    """
    q3, k3, v3 = to_f64(q), to_f64(k), to_f64(v)
    cq = [int(x) for x in np.asarray(cu_seqlens_q).tolist()]
    ck = [int(x) for x in np.asarray(cu_seqlens_k).tolist()]
    T, Hq, D = q3.shape
    Hkv = k3.shape[1]
    G = Hq // Hkv
    o = np.zeros((T, Hq, D))
    lse = np.full((Hq, T), -np.inf)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        counts = causal_key_counts(q1 - q0, k1 - k0) if causal else None
        for h in range(Hq):
            ob, lb = attention_rows(q3[q0:q1, h], k3[k0:k1, h // G], v3[k0:k1, h // G], scale, counts)
            o[q0:q1, h] = ob
            lse[h, q0:q1] = lb
    return o, lse


def decode(q, k, v, scale: float, kv_len: Optional[Sequence[int]] = None, causal: bool = False):
    """Decode: q [B,Hq,Lq,D], k/v [B,Hkv,Lkv,D] (HND), keys [0, kv_len[b]).

    Non-causal: all Lq rows see every key of the range (reading; the pages
    route Lq 2..4 to a split-K kernel without naming a mask).  kv_len=None
    means the full Lkv (ExecuTorch split-K PR, the kv_len docstring).
    causal: the Lq rows are the last Lq positions, row i sees the first
    kv_len - Lq + 1 + i keys (``causal_key_counts``; not on the pages).
    Returns (O [B,Hq,Lq,D], LSE [B,Hq,Lq]).
    """
    q4, k4, v4 = to_f64(q), to_f64(k), to_f64(v)
    B, Hq, Lq, D = q4.shape
    Hkv, Lkv = k4.shape[1], k4.shape[2]
    G = Hq // Hkv
    o = np.zeros((B, Hq, Lq, D))
    lse = np.zeros((B, Hq, Lq))
    for b in range(B):
        n = Lkv if kv_len is None else int(kv_len[b])
        counts = causal_key_counts(Lq, n) if causal else None
        for h in range(Hq):
            o[b, h], lse[b, h] = attention_rows(q4[b, h], k4[b, h // G, :n], v4[b, h // G, :n], scale, counts)
    return o, lse


def merge(o_parts, lse_parts) -> Tuple[np.ndarray, np.ndarray]:
    """Combine partial results of disjoint KV ranges.

    o_parts [P, ..., D] (each part normalised over its own range), lse_parts
    [P, ...] (log2).  The merged LSE is log2(sum_p 2^{L_p}) and the merged O is
    sum_p 2^{L_p - L} O_p -- the per-hop merge of ring attention
    (merge_state_v2 / _merge_attention_partials in the SGLang PR thread) and
    the cross-split reduce of the ExecuTorch split-K PR (global max, rescale
    partials).  Parts with LSE = -inf carry no weight; if every part is -inf
    the result is O = 0, LSE = -inf.
    """
    op = to_f64(o_parts)
    lp = to_f64(lse_parts)
    M = lp.max(axis=0)                                       # [...]
    all_empty = ~np.isfinite(M)
    Ms = np.where(all_empty, 0.0, M)
    w = np.where(np.isneginf(lp), 0.0, np.exp2(lp - Ms[None]))   # [P, ...]
    W = w.sum(axis=0)
    Wsafe = np.where(all_empty, 1.0, W)
    o = (w[..., None] * op).sum(axis=0) / Wsafe[..., None]
    lse = np.where(all_empty, -np.inf, Ms + np.log2(Wsafe))
    o = np.where(all_empty[..., None], 0.0, o)
    return o, lse


def kv_mean(k_rows: np.ndarray) -> np.ndarray:
    """mean over the KV axis of k rows [m, D] -> [D] (smooth_k; ARK issue repro
    ``k.mean(dim=2)`` in HND, i.e. over the keys, per channel, per (b, h))."""
    k_rows = np.asarray(k_rows, dtype=np.float64)
    return k_rows.mean(axis=0)


def smooth_shift(q_rows: np.ndarray, mu: np.ndarray, scale: float) -> np.ndarray:
    """The term smoothing removes from each row's LSE, in log2 units:
    scale * (q_i . mean(k)) / ln 2 (ARK issue, part 3 of the repro, ``shift``)."""
    return scale * (np.asarray(q_rows, dtype=np.float64) @ np.asarray(mu, dtype=np.float64)) / LN2


def smoothed_attention_rows(q, k, v, scale: float, k_smoothed: Optional[np.ndarray] = None):
    """Attention over mean-subtracted keys K' = K - mean(K) (smooth_k).

    Returns (O', LSE' + shift, LSE') where adding the shift gives back the LSE
    of the original logits (ARK issue: the smooth_k=True LSE lacks
    q . mean(k) * scale; adding it back fixes it).  ``k_smoothed`` may supply
    K' already rounded to a storage dtype (the kernel's reading); by default
    K' is exact.  Both paths are pinned: the exact one by the smoothing
    invariants, the stored-K' one against PyTorch's float64 attention over the
    same keys and the LSE bound of the K' rounding.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    mu = kv_mean(k) if k.shape[0] else np.zeros(k.shape[1])
    kp = (k - mu[None]) if k_smoothed is None else np.asarray(k_smoothed, dtype=np.float64)
    o, lse_s = attention_rows(q, kp, v, scale)
    return o, lse_s + smooth_shift(q, mu, scale), lse_s


# ---------------------------------------------------------------------------
# INT8 QK^T with smooth_k (the variant smoothing exists for).
# ---------------------------------------------------------------------------

INT8_BLOCK = 128   # rows (query rows or keys) per quantization block


def quantize_int8_blocks(x_rows, block: int = INT8_BLOCK) -> Tuple[np.ndarray, np.ndarray]:
    """Symmetric int8 quantization with one scale per block of `block` rows.

    ARK issue, Problem Description: smoothing K (subtracting its mean) is done
    so that K quantizes well to INT8 in SageAttention-style kernels, with the
    LSE of the original logits restored afterwards.  The pages give no
    quantizer; the plainest reading, taken here: for the rows of one block,
    amax = max |x| over the block, scale = amax / 127 (a block of zeros gets
    scale 1), code = round-half-to-even(x * (127 / amax)) clamped to
    [-127, 127] -- one fp32 reciprocal per block and one fp32 product per
    value (a block of zeros gets codes 0).  All of it in fp32 (the values are
    fp32: 16-bit inputs widened, or K - mean in fp32), so that the integer
    codes are decided in the kernel's precision.
    Returns (codes int8 [n, D], scales fp32 [ceil(n / block)]).
    """
    x32 = np.asarray(x_rows, dtype=np.float32)
    n = x32.shape[0]
    nb = (n + block - 1) // block
    codes = np.zeros(x32.shape, dtype=np.int8)
    scales = np.ones(nb, dtype=np.float32)
    for b in range(nb):
        blk = x32[b * block:(b + 1) * block]
        amax = np.float32(np.abs(blk).max()) if blk.size else np.float32(0.0)
        sc = np.float32(amax / np.float32(127.0)) if amax > 0 else np.float32(1.0)
        inv = np.float32(np.float32(127.0) / amax) if amax > 0 else np.float32(0.0)
        c = np.rint(blk * inv)                      # fp32 product, ties to even
        codes[b * block:(b + 1) * block] = np.clip(c, -127, 127).astype(np.int8)
        scales[b] = sc
    return codes, scales


def int8_attention_rows(q, k, v, scale: float, smooth: bool = True, mu: Optional[np.ndarray] = None,
                        block: int = INT8_BLOCK) -> Tuple[np.ndarray, np.ndarray]:
    """O and log2-LSE of query rows q [n, D] (one head) over keys k [m, D] with
    Q K'^T taken from int8 codes.

    K' = K - mean(K) over the call's keys (fp32; ``smooth=False`` quantizes K
    itself), Q and K' quantized per block of rows (``quantize_int8_blocks``),
    logits from the exact integer dot products,
    s_ij = scale * sq_{block(i)} * sk_{block(j)} * (qc_i . kc_j), then the
    plain definition (``attention_rows`` on those logits, via scaled codes) with
    the 16-bit V, and the smoothing shift scale * (q_i . mean) / ln 2 added back
    to the LSE (ARK issue, repro part 3).  ``mu`` may supply the fp32 mean.
    """
    q32 = np.asarray(q, dtype=np.float32)
    k32 = np.asarray(k, dtype=np.float32)
    n, m = q32.shape[0], k32.shape[0]
    if m == 0:
        return np.zeros((n, np.asarray(v).shape[1])), np.full(n, -np.inf)
    if smooth:
        mu32 = np.float32(kv_mean(k32)) if mu is None else np.asarray(mu, dtype=np.float32)
    else:
        mu32 = np.zeros(k32.shape[1], dtype=np.float32)
    kp = (k32 - mu32[None]).astype(np.float32)
    qc, qs = quantize_int8_blocks(q32, block)
    kc, ks = quantize_int8_blocks(kp, block)
    qd = qc.astype(np.float64) * np.repeat(qs.astype(np.float64), block)[:n, None]
    kd = kc.astype(np.float64) * np.repeat(ks.astype(np.float64), block)[:m, None]
    o, lse = attention_rows(qd, kd, v, scale)
    return o, lse + smooth_shift(q32, mu32.astype(np.float64), scale)


def chunked(q, k, v, scale: float, bounds: Sequence[int], layout: str = "HND"):
    """Per-chunk partial results of dense attention over KV chunks
    [bounds[c], bounds[c+1]) -- the inputs a ring-attention per-hop merge
    combines.  Returns (O_parts [C, ...layout...], LSE_parts [C, B, Hq, Sq])."""
    q4, k4, v4 = _hnd(to_f64(q), layout), _hnd(to_f64(k), layout), _hnd(to_f64(v), layout)
    outs, lses = [], []
    for c in range(len(bounds) - 1):
        a, e = bounds[c], bounds[c + 1]
        o, l = dense(q4, k4[:, :, a:e], v4[:, :, a:e], scale, "HND")
        if layout == "NHD":
            o = np.ascontiguousarray(o.transpose(0, 2, 1, 3))
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


def lse_varlen_to_dense(lse_ht: np.ndarray, B: int, S: int) -> np.ndarray:
    """[H, B*S] varlen LSE of equal-length sequences -> [B, H, S] dense layout
    (the reshape(H, B, S).transpose(0, 1) adapter in the SGLang PR thread)."""
    H = lse_ht.shape[0]
    return lse_ht.reshape(H, B, S).transpose(1, 0, 2)


# ---------------------------------------------------------------------------
# Integer planning, restated from its specification (bit-exact comparisons).
# ---------------------------------------------------------------------------

SPLIT_ALIGN = 64          # split chunk is a multiple of this many keys
SPLIT_MIN_KEYS = 128      # the automatic plan keeps at least this many keys per split
SPLIT_MAX = 256           # upper limit on the number of splits
CTAS_PER_SM = (1, 1)      # the automatic plan aims for num/den decode CTAs per SM (D <= 128) ...
CTAS_PER_SM_D256 = (2, 3) # ... and for D = 256 (whose CTA holds twice the bytes in flight)
DECODE_ROWS_PER_CTA = 16  # query rows (G * Lq) one decode CTA handles
PREFILL_ROWS_PER_CTA = 256


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def split_bounds(n: int, num_splits: int) -> List[int]:
    """Bounds of split s: [s*C, min((s+1)*C, n)) with C = roundup(ceil(n/S), 64).

    Every split index 0..S-1 exists; trailing ones may be empty (begin == end
    == n), which the split-K PR allows ("empty trailing splits").  Returns the
    S+1 begin offsets clipped to n, so split s is [out[s], out[s+1]).
    """
    if num_splits < 1:
        raise ValueError("num_splits >= 1")
    if n <= 0:
        return [0] * (num_splits + 1)
    C = _ceil_div(_ceil_div(n, num_splits), SPLIT_ALIGN) * SPLIT_ALIGN
    return [min(s * C, n) for s in range(num_splits + 1)]


def auto_num_splits(B: int, Hkv: int, Hq: int, Lq: int, n: int, num_sms: int, D: int = 128) -> int:
    """Automatic split count: ceil(num_sms * num / den) CTAs in all, with
    (num, den) = CTAS_PER_SM (CTAS_PER_SM_D256 for D = 256), no split shorter
    than SPLIT_MIN_KEYS keys, at most SPLIT_MAX, and no split that the chunk
    rounding would leave empty.  (Reading of "num_splits sized to fill the
    SMs": the pages give no formula.)"""
    G = Hq // Hkv
    row_groups = _ceil_div(G * Lq, DECODE_ROWS_PER_CTA)
    units = B * Hkv * row_groups
    num, den = CTAS_PER_SM_D256 if D > 128 else CTAS_PER_SM
    target = _ceil_div(num_sms * num, den)
    s = max(1, _ceil_div(target, max(units, 1)))
    s = min(s, max(1, _ceil_div(n, SPLIT_MIN_KEYS)), SPLIT_MAX)
    if n > 0:
        C = _ceil_div(_ceil_div(n, s), SPLIT_ALIGN) * SPLIT_ALIGN
        s = _ceil_div(n, C)
    return max(s, 1)


def varlen_schedule(cu_seqlens_q, cu_seqlens_k, H: int, rows_per_cta: int = PREFILL_ROWS_PER_CTA):
    """Longest-first work list for varlen prefill.

    Sequences are ordered by kv length, longest first, ties by index; each
    contributes H * ceil(len_q / rows_per_cta) work items ordered (head, q block).
    Returns (order [B], offsets [B+1]) where offsets are prefix sums of the item
    counts in that order, and the explicit item list [(b, h, block), ...].
    """
    cq = [int(x) for x in np.asarray(cu_seqlens_q).tolist()]
    ck = [int(x) for x in np.asarray(cu_seqlens_k).tolist()]
    B = len(cq) - 1
    lq = [cq[b + 1] - cq[b] for b in range(B)]
    lk = [ck[b + 1] - ck[b] for b in range(B)]
    order = sorted(range(B), key=lambda b: (-lk[b], b))
    offsets = [0]
    items = []
    for b in order:
        nblk = _ceil_div(lq[b], rows_per_cta)
        offsets.append(offsets[-1] + H * nblk)
        for h in range(H):
            for i in range(nblk):
                items.append((b, h, i))
    return order, offsets, items
