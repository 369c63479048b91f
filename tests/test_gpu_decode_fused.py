"""GPU parity of attn_splitkv_decode_fused (one launch: the last CTA of each
(batch, kv head, row group) merges the splits' partials) against the FP64
oracle, through the C ABI.

Beyond the cases the two-kernel decode is tested on, this checks what the
arrival counters add: the counters return to zero after every call, so one
workspace serves repeated calls and CUDA-graph replays, and a workspace whose
counters were not zeroed is reported (device error 0x103) instead of merging.
"""
import pytest
import torch

import oracle as O
import split_kv_merge_attn_b200 as skv
import workloads as W
from tests._gpu_helpers import check_lse, check_o, nan_empty, vmax

pytestmark = pytest.mark.gpu

ERR_COUNTER = 0x103


def _align256(x):
    return (x + 255) // 256 * 256


def fused_workspace(B, Hq, Lq, D, splits):
    """A workspace with the partial regions poisoned (0xFF bytes: NaN) and the
    counter region zeroed.  Region order: partial O [splits, rows, D] fp32,
    partial LSE [splits, rows] fp32, counters [rows] int32, each 256-byte aligned."""
    n = skv.attn_splitkv_workspace(B, Hq, Lq, D, splits)
    ws = torch.full((max(n, 1),), 0xFF, dtype=torch.uint8, device="cuda")
    if n:
        rows = B * Hq * Lq
        off = _align256(splits * rows * D * 4) + _align256(splits * rows * 4)
        assert n == off + _align256(rows * 4)
        ws[off:].zero_()
    return ws


def splits_for(q, k, num_splits):
    if num_splits:
        return num_splits
    B, Hq, Lq, D = q.shape
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return skv.attn_splitkv_plan(B, Hq, k.shape[1], Lq, k.shape[2], D, sms, 0)[0]


def run_fused(d, num_splits=0, kv_len=None, workspace=None):
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    out = nan_empty(q.shape, q.dtype)
    lse = nan_empty(q.shape[:3], torch.float32)
    B, Hq, Lq, D = q.shape
    splits = splits_for(q, k, num_splits)
    if workspace is None:
        workspace = fused_workspace(B, Hq, Lq, D, splits)
    kl = None if kv_len is None else torch.tensor(kv_len, dtype=torch.int32, device="cuda")
    out, lse = skv.attn_splitkv_decode(q, k, v, d["scale"], kv_len=kl, num_splits=splits, out=out, lse=lse,
                                       workspace=workspace, fused=True)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    return out, lse


def check_against_oracle(d, out, lse, kv_len=None):
    o_ref, l_ref = O.decode(d["q"], d["k"], d["v"], d["scale"], kv_len=kv_len)
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


@pytest.mark.parametrize("Lq", [1, 4])
@pytest.mark.parametrize("Lkv", [4096, 32768])
def test_config2_full_size(Lq, Lkv):
    d = W.config2(Lq, Lkv)
    out, lse = run_fused(d)
    check_against_oracle(d, out, lse)


@pytest.mark.parametrize("Lq", [1, 4])
@pytest.mark.parametrize("Lkv", [4096, 32768])
def test_config3_full_size(Lq, Lkv):
    d = W.config3(Lq, Lkv)
    out, lse = run_fused(d)
    check_against_oracle(d, out, lse)


@pytest.mark.parametrize("planted", ["pos", "allpos", "allneg"])
def test_large_logits_stable(planted):
    d = W.config2(4, 4096, planted=planted)
    out, lse = run_fused(d)
    check_against_oracle(d, out, lse)


@pytest.mark.parametrize("splits", [1, 2, 3, 37, 64, 256])
def test_explicit_split_counts_including_empty_splits(splits):
    # 1000 keys over 256 splits: C = 64, so splits 16..255 are empty
    d = W.config2(4, 1000, seed=3)
    out, lse = run_fused(d, num_splits=splits)
    check_against_oracle(d, out, lse)


def test_device_kv_len_with_empty_batches():
    d = W.decode_case(8, 2, 128, 3, 3000, B=4, seed=5, q_mult=2.0)
    kv_len = [3000, 1, 0, 1234]
    for b, n in enumerate(kv_len):
        d["k"][b, :, n:] = float("nan")
        d["v"][b, :, n:] = float("nan")
    d_ref = dict(d)
    d_ref["k"] = torch.nan_to_num(d["k"])
    d_ref["v"] = torch.nan_to_num(d["v"])
    for splits in (0, 5, 40):
        out, lse = run_fused(d, num_splits=splits, kv_len=kv_len)
        check_against_oracle(d_ref, out, lse, kv_len=kv_len)
        assert torch.all(out[2].float() == 0) and torch.all(torch.isneginf(lse[2]))


@pytest.mark.parametrize("Hq,Hkv,Lq", [(32, 2, 4), (8, 8, 1), (12, 4, 3), (64, 4, 2)])
def test_gqa_row_groups(Hq, Hkv, Lq):
    d = W.decode_case(Hq, Hkv, 128, Lq, 700, B=2, seed=7, q_mult=4.0)
    out, lse = run_fused(d)
    check_against_oracle(d, out, lse)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_head_dims_and_dtypes(D, dtype):
    d = W.decode_case(8, 2, D, 4, 1500, B=1, seed=9, q_mult=2.0, dtype=dtype)
    out, lse = run_fused(d, num_splits=7)
    check_against_oracle(d, out, lse)


def test_matches_two_kernel_decode():
    d = W.config3(4, 16384, seed=4)
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    o2, l2 = skv.attn_splitkv_decode(q, k, v, d["scale"])
    o1, l1 = run_fused(d)
    assert float((o1.float() - o2.float()).abs().max()) <= 2e-2 * vmax(d["v"])
    assert float((l1 - l2).abs().max()) <= 1e-4


def test_counters_return_to_zero_across_calls_and_graph_replays():
    """One zeroed workspace, many calls: eager calls with different inputs,
    then a captured graph replayed with new inputs copied into its buffers."""
    d0 = W.config2(4, 8192, seed=21)
    q, k, v = d0["q"].cuda(), d0["k"].cuda(), d0["v"].cuda()
    B, Hq, Lq, D = q.shape
    splits = splits_for(q, k, 0)
    ws = fused_workspace(B, Hq, Lq, D, splits)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    for seed in (22, 23):
        d = W.config2(4, 8192, seed=seed)
        q.copy_(d["q"]), k.copy_(d["k"]), v.copy_(d["v"])
        skv.attn_splitkv_decode(q, k, v, d["scale"], num_splits=splits, out=out, lse=lse, workspace=ws, fused=True)
        torch.cuda.synchronize()
        assert skv.device_error() == 0
        check_against_oracle(d, out, lse)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            skv.attn_splitkv_decode(q, k, v, d0["scale"], num_splits=splits, out=out, lse=lse, workspace=ws,
                                    fused=True, stream=s)
    torch.cuda.synchronize()
    for seed in (24, 25, 26):
        d = W.config2(4, 8192, seed=seed)
        q.copy_(d["q"]), k.copy_(d["k"]), v.copy_(d["v"])
        g.replay()
        torch.cuda.synchronize()
        assert skv.device_error() == 0
        check_against_oracle(d, out, lse)
    del g
    rows = B * Hq * Lq
    off = _align256(splits * rows * D * 4) + _align256(splits * rows * 4)
    assert int(ws[off:].count_nonzero()) == 0, "arrival counters must be zero after every call"


def test_workspace_not_zeroed_is_reported():
    """Counters that did not start at zero (here 0x7F7F7F7F and -1) record
    device error 0x103; no CTA merges, so the outputs are left as they were."""
    d = W.config2(1, 4096, seed=31)
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    B, Hq, Lq, D = q.shape
    splits = 8
    n = skv.attn_splitkv_workspace(B, Hq, Lq, D, splits)
    for fill in (0x7F, 0xFF):
        ws = torch.full((n,), fill, dtype=torch.uint8, device="cuda")
        out = torch.zeros_like(q)
        skv.attn_splitkv_decode(q, k, v, d["scale"], num_splits=splits, out=out, workspace=ws, fused=True)
        torch.cuda.synchronize()
        assert skv.device_error() == ERR_COUNTER
        assert torch.all(out == 0)
