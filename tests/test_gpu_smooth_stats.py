"""GPU parity of the smooth_k statistics themselves, read back from the
documented workspace sections: the per-256-key column sums of K, the fp32 mean
of K over each key range (ARK return_lse issue, part 3 of the repro: the mean
of K over the keys, per channel and head) and the materialised K' = K - mean,
for dense HND/NHD, varlen TND (with empty and one-key sequences) and
multi-chunk calls, at D = 64, 128 and 256.

Mode 1's O and LSE cannot show a wrong mean: the shift it applies to the logits
is added back to the LSE, and the softmax does not see a per-row shift.  So the
statistics are compared with the oracle's mean directly, within the error bound
of an fp32 sum of n 16-bit values (n * 2^-24 * sum |k|, doubled)."""
import numpy as np
import pytest
import torch

import oracle as O
import split_kv_merge_attn_b200 as skv
import workloads as W
from tests._gpu_helpers import check_lse, check_o, vmax

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24


def _a256(x):
    return (x + 255) // 256 * 256


def fwd_sections(B, Hkv, Sk, D, tnd, smooth_k, nranges=1):
    """Byte offsets of the prefill workspace sections (include/splitkv.h):
    [order, offsets] (varlen), fp32 mean [ranges, Hkv, D], fp32 column sums
    [ceil(Sk / 256), ranges, Hkv, D], K' (smooth_k = 2) in K's layout."""
    off = 0
    if tnd:
        off += _a256(B * 4) + _a256((B + 1) * 4)
    ranges = B * nranges
    kmean = off
    off += _a256(ranges * Hkv * D * 4)
    partial = off
    nch = (Sk + 255) // 256
    off += _a256(nch * ranges * Hkv * D * 4)
    kprime = None
    if smooth_k == 2:
        kprime = off
        rows = Sk if tnd else B * Sk
        off += _a256(rows * Hkv * D * 2)
    return dict(kmean=kmean, partial=partial, kprime=kprime, nch=nch, ranges=ranges, total=off)


def _f32(ws, off, count):
    return ws[off:off + 4 * count].view(torch.float32).cpu().numpy().astype(np.float64)


def check_sums(got, rows):
    """got [D] fp32 column sum of rows [n, D] (any order of fp32 additions)."""
    rows = np.asarray(rows, dtype=np.float64)
    n = rows.shape[0]
    exact = O.kv_mean(rows) * n if n else np.zeros(rows.shape[1])
    bound = 2.0 * max(n, 1) * U32 * np.abs(rows).sum(axis=0) + 1e-30
    assert np.all(np.abs(got - exact) <= bound), float(np.max(np.abs(got - exact) / bound))


def check_mean(got, rows):
    rows = np.asarray(rows, dtype=np.float64)
    n = rows.shape[0]
    if n == 0:
        assert np.all(got == 0.0)
        return
    exact = O.kv_mean(rows)
    bound = 2.0 * (n + 1) * U32 * np.abs(rows).sum(axis=0) / n + 1e-30
    assert np.all(np.abs(got - exact) <= bound), float(np.max(np.abs(got - exact) / bound))


def check_ranges(ws, sec, ranges_rows, Hkv, D, smooth_k):
    """ranges_rows[r][h]: the [n, D] float64 keys of range r, kv head h."""
    R = sec["ranges"]
    part = _f32(ws, sec["partial"], sec["nch"] * R * Hkv * D).reshape(sec["nch"], R, Hkv, D)
    mean = _f32(ws, sec["kmean"], R * Hkv * D).reshape(R, Hkv, D)
    max_len = max(ranges_rows[r][0].shape[0] for r in range(R))
    for r in range(R):
        for h in range(Hkv):
            rows = ranges_rows[r][h]
            n = rows.shape[0]
            for c in range((max_len + 255) // 256):
                check_sums(part[c, r, h], rows[256 * c:min(n, 256 * c + 256)])
            if smooth_k == 2:
                check_mean(mean[r, h], rows)


def check_kprime(ws, sec, k_gpu, mean_of_row, shape):
    """K' = round16(K - mean) in K's layout, bit for bit from the kernel's own
    fp32 mean: an fp32 subtraction and one round-to-nearest conversion."""
    kp = ws[sec["kprime"]:sec["kprime"] + 2 * k_gpu.numel()].view(k_gpu.dtype).reshape(shape)
    ref = (k_gpu.float() - mean_of_row).to(k_gpu.dtype)
    assert torch.equal(kp.view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("layout", ["HND", "NHD"])
@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("smooth_k", [1, 2])
def test_dense_column_sums_and_mean(layout, D, smooth_k):
    B, Hq, Hkv, Sq, Sk = 2, 4, 2, 130, 700
    d = W.dense_case(B, Hq, Hkv, Sq, Sk, D, seed=D + smooth_k, k_offset=0.5)
    q, k, v = (W.to_layout(x, layout).cuda() for x in (d["q"], d["k"], d["v"]))
    sec = fwd_sections(B, Hkv, Sk, D, False, smooth_k)
    nbytes = skv.attn_fwd_lse_workspace(B, Hq, Hkv, Sk, D, layout=layout, smooth_k=smooth_k)
    assert nbytes == sec["total"]
    ws = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device="cuda")
    skv.attn_fwd_lse(q, k, v, d["scale"], layout=layout, smooth_k=smooth_k, workspace=ws)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    k64 = O.to_f64(d["k"])
    check_ranges(ws, sec, [[k64[b, h] for h in range(Hkv)] for b in range(B)], Hkv, D, smooth_k)
    if smooth_k == 2:
        mean = torch.from_numpy(_f32(ws, sec["kmean"], B * Hkv * D).astype(np.float32)).cuda().view(B, Hkv, 1, D)
        if layout == "NHD":
            mean = mean.permute(0, 2, 1, 3)
        check_kprime(ws, sec, k, mean, k.shape)


def test_varlen_column_sums_and_mean():
    lens = [300, 0, 1, 257, 1024]
    Hkv, D = 3, 128
    d = W.varlen_case([64] * len(lens), lens, 6, Hkv, D, seed=5, k_offset=0.5)
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    Tk = k.shape[0]
    for smooth_k in (1, 2):
        sec = fwd_sections(len(lens), Hkv, Tk, D, True, smooth_k)
        nbytes = skv.attn_fwd_lse_workspace(len(lens), 6, Hkv, Tk, D, layout="TND", smooth_k=smooth_k)
        assert nbytes == sec["total"]
        ws = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device="cuda")
        out, lse = skv.attn_fwd_lse(q, k, v, d["scale"], layout="TND", cu_seqlens_q=d["cu_seqlens_q"].cuda(),
                                    cu_seqlens_k=d["cu_seqlens_k"].cuda(), max_seqlen_q=d["max_seqlen_q"],
                                    max_seqlen_k=d["max_seqlen_k"], smooth_k=smooth_k, workspace=ws)
        torch.cuda.synchronize()
        assert skv.device_error() == 0
        # and the call's own result: the unsmoothed attention of each sequence;
        # smooth_k = 2 attends over K' = K - mean rounded to 16 bits, so its LSE
        # is held to the oracle's model of that problem (the same rounding of
        # each sequence's K', done in float64) instead
        o_ref, l_ref = O.varlen(d["q"], d["k"], d["v"], d["cu_seqlens_q"], d["cu_seqlens_k"], d["scale"])
        check_o(out, o_ref, vmax(d["v"]))
        if smooth_k == 1:
            check_lse(lse, l_ref)
        else:
            q64, k64, v64 = O.to_f64(d["q"]), O.to_f64(d["k"]), O.to_f64(d["v"])
            cq, ck = d["cu_seqlens_q"].tolist(), d["cu_seqlens_k"].tolist()
            ref2 = l_ref.copy()
            for bseq in range(len(lens)):
                if ck[bseq + 1] == ck[bseq]:
                    continue  # no keys: LSE -inf in both
                for hq in range(6):
                    kk = k64[ck[bseq]:ck[bseq + 1], hq // 2]
                    kp = torch.from_numpy(kk - kk.mean(0)[None]).float().bfloat16().double().numpy()
                    _, ref2[hq, cq[bseq]:cq[bseq + 1]], _ = O.smoothed_attention_rows(
                        q64[cq[bseq]:cq[bseq + 1], hq], kk, v64[ck[bseq]:ck[bseq + 1], hq // 2], d["scale"],
                        k_smoothed=kp)
            check_lse(lse, ref2)
        k64 = O.to_f64(d["k"])
        cu = d["cu_seqlens_k"].tolist()
        rows = [[k64[cu[r]:cu[r + 1], h] for h in range(Hkv)] for r in range(len(lens))]
        check_ranges(ws, sec, rows, Hkv, D, smooth_k)
        if smooth_k == 2:
            mean = _f32(ws, sec["kmean"], len(lens) * Hkv * D).reshape(len(lens), Hkv, D).astype(np.float32)
            seq_of_row = np.repeat(np.arange(len(lens)), lens)
            check_kprime(ws, sec, k, torch.from_numpy(mean[seq_of_row]).cuda(), k.shape)


@pytest.mark.parametrize("layout,D", [("HND", 128), ("NHD", 256), ("HND", 64)])
@pytest.mark.parametrize("smooth_k", [1, 2])
def test_chunk_ranges_column_sums_and_mean(layout, D, smooth_k):
    """One mean per (batch, KV chunk): ranges r = b * chunks + c."""
    B, H, Sq, Sk = 2, 2, 64, 1000
    bounds = [0, 1, 300, 300, 813, 1000]  # includes a one-key and an empty chunk
    C = len(bounds) - 1
    d = W.dense_case(B, H, H, Sq, Sk, D, seed=3 * D + smooth_k, k_offset=0.5)
    q, k, v = (W.to_layout(x, layout).cuda() for x in (d["q"], d["k"], d["v"]))
    sec = fwd_sections(B, H, Sk, D, False, smooth_k, nranges=C)
    nbytes = skv.attn_fwd_lse_chunks_workspace(B, H, H, Sk, D, C, layout=layout, smooth_k=smooth_k)
    assert nbytes == sec["total"]
    ws = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device="cuda")
    skv.attn_fwd_lse_chunks(q, k, v, bounds, d["scale"], layout=layout, smooth_k=smooth_k, workspace=ws)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    k64 = O.to_f64(d["k"])
    rows = [[k64[b, h, bounds[c]:bounds[c + 1]] for h in range(H)] for b in range(B) for c in range(C)]
    check_ranges(ws, sec, rows, H, D, smooth_k)
