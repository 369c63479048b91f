"""GPU parity of attn_fwd_lse (dense HND/NHD, varlen TND, smooth_k) and of the
chunked ring-style path (attn_fwd_lse per KV chunk + merge_state) against the
FP64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
import split_kv_merge_attn_b200 as skv
import workloads as W
from tests._gpu_helpers import check_lse, check_o, nan_empty, vmax

pytestmark = pytest.mark.gpu


def run_dense(d, layout="HND", smooth_k=0):
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    if layout == "HND":
        B, Hq, Sq, D = q.shape
    else:
        B, Sq, Hq, D = q.shape
    out = nan_empty(q.shape, q.dtype)
    lse = nan_empty((B, Hq, Sq), torch.float32)
    out, lse = skv.attn_fwd_lse(q, k, v, d["scale"], layout=layout, smooth_k=smooth_k, out=out, lse=lse)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    return out, lse


def run_varlen(d, smooth_k=0):
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    out = nan_empty(q.shape, q.dtype)
    lse = nan_empty((q.shape[1], q.shape[0]), torch.float32)
    out, lse = skv.attn_fwd_lse(q, k, v, d["scale"], layout="TND", cu_seqlens_q=d["cu_seqlens_q"].cuda(),
                                cu_seqlens_k=d["cu_seqlens_k"].cuda(), max_seqlen_q=d["max_seqlen_q"],
                                max_seqlen_k=d["max_seqlen_k"], smooth_k=smooth_k, out=out, lse=lse)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    return out, lse


# ------------------------------------------------------------ workload 1

@pytest.mark.parametrize("variant", ["rows", "blocks"])
def test_config1(variant):
    d = W.config1(variant)
    out, lse = run_dense(d)
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"])
    check_o(out, o_ref, vmax(d["v"]))
    err = check_lse(lse, l_ref)
    l = lse.cpu()
    if variant == "blocks":
        blocks = l.view(1, 4, 4, 16)
        assert torch.equal(blocks, blocks[..., :1].expand_as(blocks)), "16 identical rows -> 16 identical LSEs"
    else:
        # every row carries its own LSE: a per-16-row store would be off by several units
        bug = l.view(1, 4, 4, 16)[..., -1:].expand(1, 4, 4, 16).reshape(1, 4, 64)
        assert float((bug.double() - torch.from_numpy(l_ref)).abs().max()) > 1.0
    assert err < 1e-3


@pytest.mark.parametrize("smooth_k", [1, 2])
def test_config1_smooth_k(smooth_k):
    """K + 0.5 with 16 equal rows per block (the ARK issue's third case): the
    returned LSE is that of the ORIGINAL logits."""
    d = W.config1("koff")
    out, lse = run_dense(d, smooth_k=smooth_k)
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"])
    check_o(out, o_ref, vmax(d["v"]))
    if smooth_k == 1:
        check_lse(lse, l_ref)
    else:
        # K' = K - mean rounded to bf16 (the same rounding, done by the oracle
        # in float64): match that problem to 1e-3, and the unsmoothed LSE to the
        # size of the rounding error
        q, k, v = (O.to_f64(d[x])[0] for x in "qkv")
        ref2 = np.zeros_like(l_ref)
        for h in range(4):
            mu = k[h].mean(0)
            kp = torch.from_numpy(k[h] - mu[None]).float().bfloat16().double().numpy()
            _, ref2[0, h], _ = O.smoothed_attention_rows(q[h], k[h], v[h], d["scale"], k_smoothed=kp)
        check_lse(lse, ref2)
        check_lse(lse, l_ref, tol=2e-2)


# ------------------------------------------------------------ dense shapes

@pytest.mark.parametrize("layout", ["HND", "NHD"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_dense_ragged_gqa(layout, D, dtype):
    d = W.dense_case(2, 8, 2, 300, 333, D, seed=4, dtype=dtype, q_mult=2.0)
    if layout == "NHD":
        d = dict(d, q=W.to_layout(d["q"], "NHD"), k=W.to_layout(d["k"], "NHD"), v=W.to_layout(d["v"], "NHD"))
    out, lse = run_dense(d, layout=layout)
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"], layout=layout)
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


@pytest.mark.parametrize("Sq,Sk", [(1, 1), (1, 129), (129, 1), (128, 128), (256, 256), (257, 383), (64, 0)])
def test_dense_edge_sizes(Sq, Sk):
    d = W.dense_case(1, 2, 1, Sq, Sk, 128, seed=Sq + Sk, q_mult=3.0)
    out, lse = run_dense(d)
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"])
    check_o(out, o_ref, vmax(d["v"]) if Sk else 1.0)
    check_lse(lse, l_ref)


def test_dense_large_logits():
    """Row scale 30: logits of several hundred; the lazy running max rescales."""
    d = W.dense_case(1, 2, 2, 200, 700, 128, seed=8, q_mult=30.0)
    out, lse = run_dense(d)
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"])
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


def test_dense_increasing_logits_force_rescales():
    """Keys whose logits grow along the sequence make the running max rise in
    every tile, so O is rescaled in tensor memory many times."""
    d = W.dense_case(1, 1, 1, 130, 1000, 128, seed=3)
    ramp = torch.linspace(0.0, 12.0, 1000).view(1, 1, 1000, 1)
    d["k"] = (d["k"].float() + ramp * d["q"].float()[:, :, :1].sign()).bfloat16()
    out, lse = run_dense(d)
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"])
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_dense_max_jumps_inside_tiles(dtype):
    """Planted keys raise the running max by far more than the lazy-rescale
    threshold at chosen places: in the second half of a 128-key tile (its first
    half already published to the PV products), in the first half of a later
    tile, and in a tile's last key.  Even rows see the jumps, odd rows see the
    same keys as large negative logits, so warps mix rows that rescale with
    rows that do not."""
    B, H, Sq, Sk, D = 1, 2, 256, 1024, 128
    d = W.dense_case(B, H, H, Sq, Sk, D, seed=12, dtype=dtype)
    scale = d["scale"]
    q = d["q"].float()
    k = d["k"].float()
    sign = torch.tensor([4.0, -4.0]).repeat(Sq // 2)
    q[:, :, :, 0] = sign                              # q . e0 = +-4
    for pos, logit in [(3 * 128 + 64 + 7, 20.0), (5 * 128 + 3, 40.0), (6 * 128 + 100, 60.0), (7 * 128 + 127, 75.0)]:
        k[:, :, pos, :] = 0.0
        k[:, :, pos, 0] = logit / (4.0 * scale)       # natural-log logit +-logit
    t = d["q"].dtype
    d["q"], d["k"] = q.to(t), k.to(t)
    out, lse = run_dense(d)
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"])
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


# ------------------------------------------------------------ varlen

def test_varlen_small_ragged():
    lens_q = [3, 0, 300, 129, 1, 256]
    lens_k = [5, 7, 0, 600, 1, 300]
    d = W.varlen_case(lens_q, lens_k, 8, 4, 128, seed=6)
    out, lse = run_varlen(d)
    o_ref, l_ref = O.varlen(d["q"], d["k"], d["v"], d["cu_seqlens_q"], d["cu_seqlens_k"], d["scale"])
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


def test_varlen_work_order_on_device_matches_oracle():
    d = W.varlen_case([100, 900, 40, 700, 513], [50, 900, 900, 10, 0], 3, 3, 64, seed=2)
    B = 5
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    nbytes = skv.attn_fwd_lse_workspace(B, 3, 3, k.shape[0], 64, "bf16", "TND", 0)
    ws = torch.full((nbytes,), 0xFF, dtype=torch.uint8, device="cuda")
    skv.attn_fwd_lse(q, k, v, d["scale"], layout="TND", cu_seqlens_q=d["cu_seqlens_q"].cuda(),
                     cu_seqlens_k=d["cu_seqlens_k"].cuda(), max_seqlen_q=900, max_seqlen_k=900, workspace=ws)
    torch.cuda.synchronize()
    w = ws.cpu().numpy()
    order = np.frombuffer(w[:4 * B].tobytes(), dtype=np.int32).tolist()
    offsets = np.frombuffer(w[256:256 + 4 * (B + 1)].tobytes(), dtype=np.int32).tolist()
    o_order, o_offsets, _ = O.varlen_schedule(d["cu_seqlens_q"], d["cu_seqlens_k"], 3)
    assert order == o_order and offsets == o_offsets


def _sample_varlen_rows(d, n, seed):
    rng = np.random.default_rng(seed)
    T, Hq, _ = d["q"].shape
    cu = d["cu_seqlens_q"].tolist()
    rows = [(int(t), int(h)) for t, h in zip(rng.integers(0, T, n), rng.integers(0, Hq, n))]
    # always include the first and last row of every sequence
    for b in range(len(cu) - 1):
        if cu[b + 1] > cu[b]:
            rows += [(cu[b], 0), (cu[b + 1] - 1, Hq - 1)]
    return rows


def _varlen_oracle_rows(d, rows):
    q, k, v = O.to_f64(d["q"]), O.to_f64(d["k"]), O.to_f64(d["v"])
    cq, ck = d["cu_seqlens_q"].tolist(), d["cu_seqlens_k"].tolist()
    G = q.shape[1] // k.shape[1]
    o_ref, l_ref = [], []
    for t, h in rows:
        b = max(i for i in range(len(cq) - 1) if cq[i] <= t)
        o, l = O.attention_rows(q[t:t + 1, h], k[ck[b]:ck[b + 1], h // G], v[ck[b]:ck[b + 1], h // G], d["scale"])
        o_ref.append(o[0])
        l_ref.append(l[0])
    return np.array(o_ref), np.array(l_ref)


def test_config4_full_size_sampled():
    d = W.config4()
    out, lse = run_varlen(d)
    rows = _sample_varlen_rows(d, 300, seed=0)
    o_ref, l_ref = _varlen_oracle_rows(d, rows)
    got_o = torch.stack([out[t, h] for t, h in rows])
    got_l = torch.stack([lse[h, t] for t, h in rows])
    check_o(got_o, o_ref, vmax(d["v"]))
    check_lse(got_l, l_ref)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


# ------------------------------------------------------------ chunked (workload 5)

def run_chunked(d, smooth_k=1):
    """Ring-style: attn_fwd_lse over each KV chunk (each smoothed by its own
    mean), then merge_state of the partial (O, LSE) pairs."""
    layout = d["layout"]
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    bounds = d["chunk_bounds"]
    if layout == "HND":
        B, H, Sq, D = q.shape
        sl = lambda t, a, b: t[:, :, a:b].contiguous()
    else:
        B, Sq, H, D = q.shape
        sl = lambda t, a, b: t[:, a:b].contiguous()
    P = len(bounds) - 1
    o_parts = nan_empty((P,) + tuple(q.shape), q.dtype)
    l_parts = nan_empty((P, B, H, Sq), torch.float32)
    for c in range(P):
        skv.attn_fwd_lse(q, sl(k, bounds[c], bounds[c + 1]), sl(v, bounds[c], bounds[c + 1]), d["scale"],
                         layout=layout, smooth_k=smooth_k, out=o_parts[c], lse=l_parts[c])
    out = nan_empty(tuple(q.shape), q.dtype)
    lse = nan_empty((B, H, Sq), torch.float32)
    skv.merge_state(o_parts, l_parts, layout, out=out, lse=lse)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    return out, lse, o_parts, l_parts


@pytest.mark.parametrize("dtype,layout", [("bf16", "HND"), ("fp16", "HND"), ("bf16", "NHD")])
def test_config5_small(dtype, layout):
    d = W.config5(dtype=dtype, layout=layout, Sq=512, Sk=2048, H=4)
    out, lse, _, _ = run_chunked(d)
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"], layout=layout)
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


def test_config5_full_size_sampled():
    d = W.config5()
    out, lse, o_parts, l_parts = run_chunked(d)
    rng = np.random.default_rng(1)
    rows = [(0, int(h), int(i)) for h, i in zip(rng.integers(0, 16, 160), rng.integers(0, 4096, 160))]
    rows += [(0, 0, 0), (0, 15, 4095)]
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"], rows=rows)
    check_o(torch.stack([out[b, h, i] for b, h, i in rows]), o_ref, vmax(d["v"]))
    check_lse(torch.stack([lse[b, h, i] for b, h, i in rows]), l_ref)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    # each chunk's LSE is the LSE of the original logits of that chunk
    c = 2
    a, e = d["chunk_bounds"][c], d["chunk_bounds"][c + 1]
    oc, lc = O.dense(d["q"], d["k"][:, :, a:e], d["v"][:, :, a:e], d["scale"], rows=rows[:40])
    check_lse(torch.stack([l_parts[c, b, h, i] for b, h, i in rows[:40]]), lc)


@pytest.mark.parametrize("D", [128, 256])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_first_half_raises_max_after_second_half_published(D, dtype):
    """The softmax exponentiates keys [64, 128) of a KV tile first, against the
    max of those keys; a key in [0, 64) of the same tile that lies far above
    them (here in the first tile, where O holds only that step's products, and
    in a later one) makes it wait for the first half's PV products and rescale
    O before the second half is exponentiated.  Rows alternate between seeing
    the planted keys as large positive and large negative logits."""
    B, H, Sq, Sk = 1, 2, 256, 512
    d = W.dense_case(B, H, H, Sq, Sk, D, seed=21, dtype=dtype)
    scale = d["scale"]
    q = d["q"].float()
    k = d["k"].float()
    q[:, :, :, 0] = torch.tensor([4.0, -4.0]).repeat(Sq // 2)
    for pos, logit in [(5, 30.0), (2 * 128 + 40, 70.0)]:
        k[:, :, pos, :] = 0.0
        k[:, :, pos, 0] = logit / (4.0 * scale)
    t = d["q"].dtype
    d["q"], d["k"] = q.to(t), k.to(t)
    out, lse = run_dense(d)
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"])
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)
