"""GPU parity of the causal variants (attn_fwd_lse_causal,
attn_splitkv_decode_causal) against the FP64 oracle's causal mask
(bottom-right aligned: query row i of a sequence sees keys j <= i + len_k - len_q),
through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
import split_kv_merge_attn_b200 as skv
import workloads as W
from tests._gpu_helpers import check_lse, check_o, nan_empty, vmax

pytestmark = pytest.mark.gpu


def run_dense_causal(d, layout="HND", smooth_k=0):
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    B, Hq, Sq = (q.shape[0], q.shape[1], q.shape[2]) if layout == "HND" else (q.shape[0], q.shape[2], q.shape[1])
    out = nan_empty(q.shape, q.dtype)
    lse = nan_empty((B, Hq, Sq), torch.float32)
    out, lse = skv.attn_fwd_lse(q, k, v, d["scale"], layout=layout, smooth_k=smooth_k, out=out, lse=lse,
                                causal=True)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    return out, lse


def check_dense(d, out, lse, layout="HND"):
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"], layout=layout, causal=True)
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


@pytest.mark.parametrize("Sq,Sk", [(1000, 1000), (300, 1000), (700, 300), (256, 256), (129, 383), (1, 500),
                                   (500, 1), (383, 129)])
def test_dense_shapes(Sq, Sk):
    """Square, queries after a cache (Sq < Sk), rows before the first key
    (Sq > Sk), tile-aligned and ragged sizes."""
    d = W.dense_case(1, 4, 2, Sq, Sk, 128, seed=Sq * 7 + Sk, q_mult=2.0)
    out, lse = run_dense_causal(d)
    check_dense(d, out, lse)


@pytest.mark.parametrize("layout,D,dtype", [("NHD", 128, "bf16"), ("HND", 64, "fp16"), ("NHD", 64, "bf16")])
def test_dense_layouts_dims_dtypes(layout, D, dtype):
    d = W.dense_case(2, 6, 2, 333, 611, D, seed=5, dtype=dtype, q_mult=2.0)
    if layout == "NHD":
        for x in ("q", "k", "v"):
            d[x] = d[x].transpose(1, 2).contiguous()
    out, lse = run_dense_causal(d, layout=layout)
    check_dense(d, out, lse, layout=layout)


@pytest.mark.parametrize("smooth_k", [1, 2])
def test_dense_smooth_k(smooth_k):
    d = W.dense_case(1, 2, 2, 400, 900, 128, seed=9, k_offset=0.5)
    out, lse = run_dense_causal(d, smooth_k=smooth_k)
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"], causal=True)
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref, tol=1e-3 if smooth_k == 1 else 2e-2)


def test_varlen_ragged():
    lens_q = [300, 0, 77, 512, 200, 1]
    lens_k = [300, 5, 400, 128, 50, 9]
    d = W.varlen_case(lens_q, lens_k, 8, 4, 128, seed=13)
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    out = nan_empty(q.shape, q.dtype)
    lse = nan_empty((q.shape[1], q.shape[0]), torch.float32)
    out, lse = skv.attn_fwd_lse(q, k, v, d["scale"], layout="TND", cu_seqlens_q=d["cu_seqlens_q"].cuda(),
                                cu_seqlens_k=d["cu_seqlens_k"].cuda(), max_seqlen_q=d["max_seqlen_q"],
                                max_seqlen_k=d["max_seqlen_k"], out=out, lse=lse, causal=True)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    o_ref, l_ref = O.varlen(d["q"], d["k"], d["v"], d["cu_seqlens_q"], d["cu_seqlens_k"], d["scale"], causal=True)
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


def test_full_size_chunk_sampled():
    """B=1, H=16, Sq=Sk=4096, D=128 (one KV chunk of the chunked workload,
    causal): every row of two heads and sampled rows of the rest."""
    c = W.config5(Sk=4096, n_chunks=1)
    q, k, v = c["q"].cuda(), c["k"].cuda(), c["v"].cuda()
    out, lse = skv.attn_fwd_lse(q, k, v, c["scale"], causal=True)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    rng = np.random.default_rng(0)
    rows = [(0, h, i) for h in (0, 15) for i in range(0, 4096, 3)]
    rows += [(0, int(h), int(i)) for h, i in zip(rng.integers(0, 16, 300), rng.integers(0, 4096, 300))]
    rows += [(0, 3, i) for i in (0, 1, 127, 128, 255, 256, 4095)]
    o_ref, l_ref = O.dense(c["q"], c["k"], c["v"], c["scale"], rows=rows, causal=True)
    o = torch.stack([out[b, h, i] for b, h, i in rows])
    l = torch.stack([lse[b, h, i] for b, h, i in rows])
    check_o(o, o_ref, vmax(c["v"]))
    check_lse(l, l_ref)


# ------------------------------------------------------------ decode

def run_decode_causal(d, num_splits=0, kv_len=None):
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    out = nan_empty(q.shape, q.dtype)
    lse = nan_empty(q.shape[:3], torch.float32)
    B, Hq, Lq, D = q.shape
    splits = num_splits
    if splits == 0:
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        splits, _ = skv.attn_splitkv_plan(B, Hq, k.shape[1], Lq, k.shape[2], D, sms, 0)
    ws = torch.full((max(skv.attn_splitkv_workspace(B, Hq, Lq, D, splits), 1),), 0xFF, dtype=torch.uint8,
                    device="cuda")
    kl = None if kv_len is None else torch.tensor(kv_len, dtype=torch.int32, device="cuda")
    out, lse = skv.attn_splitkv_decode(q, k, v, d["scale"], kv_len=kl, num_splits=splits, out=out, lse=lse,
                                       workspace=ws, causal=True)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    return out, lse


@pytest.mark.parametrize("Lkv", [4096, 32768])
def test_decode_config2_lq4(Lkv):
    d = W.config2(4, Lkv)
    out, lse = run_decode_causal(d)
    o_ref, l_ref = O.decode(d["q"], d["k"], d["v"], d["scale"], causal=True)
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


def test_decode_config3_lq4():
    d = W.config3(4, 16384)
    out, lse = run_decode_causal(d)
    o_ref, l_ref = O.decode(d["q"], d["k"], d["v"], d["scale"], causal=True)
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


@pytest.mark.parametrize("splits", [1, 7, 64])
def test_decode_kv_len_and_masked_splits(splits):
    """Device kv_len (NaN past it), kv_len shorter than Lq (rows with no key),
    and split counts where the last split is masked for the earlier rows."""
    d = W.decode_case(8, 2, 128, 3, 700, B=4, seed=6, q_mult=2.0)
    kv_len = [700, 2, 0, 130]
    for b, n in enumerate(kv_len):
        d["k"][b, :, n:] = float("nan")
        d["v"][b, :, n:] = float("nan")
    out, lse = run_decode_causal(d, num_splits=splits, kv_len=kv_len)
    d_ref = dict(d)
    d_ref["k"] = torch.nan_to_num(d["k"])
    d_ref["v"] = torch.nan_to_num(d["v"])
    o_ref, l_ref = O.decode(d_ref["q"], d_ref["k"], d_ref["v"], d["scale"], kv_len=kv_len, causal=True)
    check_o(out, o_ref, vmax(d_ref["v"]))
    check_lse(lse, l_ref)


def test_decode_lq1_equals_noncausal():
    d = W.config2(1, 8192, seed=3)
    o1, l1 = run_decode_causal(d)
    o2, l2 = skv.attn_splitkv_decode(d["q"].cuda(), d["k"].cuda(), d["v"].cuda(), d["scale"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
