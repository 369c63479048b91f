"""GPU parity of attn_splitkv_decode against the FP64 oracle (through the C ABI).

Decode problems are small in rows, so the oracle runs every row in full even
at the benchmark's sizes (Lkv up to 32768)."""
import numpy as np
import pytest
import torch

import oracle as O
import split_kv_merge_attn_b200 as skv
import workloads as W
from tests._gpu_helpers import check_lse, check_o, nan_empty, vmax

pytestmark = pytest.mark.gpu


def run_decode(d, num_splits=0, kv_len=None, poison=True):
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    out = nan_empty(q.shape, q.dtype) if poison else None
    lse = nan_empty(q.shape[:3], torch.float32) if poison else None
    B, Hq, Lq, D = q.shape
    splits = num_splits
    if splits == 0:
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        splits, _ = skv.attn_splitkv_plan(B, Hq, k.shape[1], Lq, k.shape[2], D, sms, 0)
    ws = skv.attn_splitkv_workspace(B, Hq, Lq, D, splits)
    workspace = torch.full((max(ws, 1),), 0xFF, dtype=torch.uint8, device="cuda")  # NaN bit patterns
    kl = None if kv_len is None else torch.tensor(kv_len, dtype=torch.int32, device="cuda")
    out, lse = skv.attn_splitkv_decode(q, k, v, d["scale"], kv_len=kl, num_splits=splits, out=out, lse=lse,
                                       workspace=workspace)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    return out, lse


def check_against_oracle(d, out, lse, kv_len=None):
    o_ref, l_ref = O.decode(d["q"], d["k"], d["v"], d["scale"], kv_len=kv_len)
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


@pytest.mark.parametrize("Lq", [1, 4])
@pytest.mark.parametrize("Lkv", [4096, 8192, 32768])
def test_config2_full_size(Lq, Lkv):
    d = W.config2(Lq, Lkv)
    out, lse = run_decode(d)
    check_against_oracle(d, out, lse)


@pytest.mark.parametrize("Lq", [1, 4])
@pytest.mark.parametrize("Lkv", [4096, 16384, 32768])
def test_config3_full_size(Lq, Lkv):
    d = W.config3(Lq, Lkv)
    out, lse = run_decode(d)
    check_against_oracle(d, out, lse)


@pytest.mark.parametrize("planted", ["pos", "allpos", "allneg"])
@pytest.mark.parametrize("Lq", [1, 2, 4])
def test_large_logits_stable(planted, Lq):
    """Scaled logits of +-150: a fixed exponent offset overflows or underflows
    here (ExecuTorch split-K PR); the per-split max keeps everything finite."""
    d = W.config2(Lq, 4096, planted=planted)
    out, lse = run_decode(d)
    check_against_oracle(d, out, lse)


@pytest.mark.parametrize("splits", [1, 2, 3, 37, 64, 256])
def test_explicit_split_counts_including_empty_splits(splits):
    # 1000 keys over 256 splits: C = 64, so splits 16..255 are empty
    d = W.config2(4, 1000, seed=3)
    out, lse = run_decode(d, num_splits=splits)
    check_against_oracle(d, out, lse)


def test_device_kv_len_ignores_trailing_positions():
    """kv_len read on the device: keys >= kv_len[b] (here NaN, like an unfilled
    cache) never reach the result; batches with kv_len 0 give O = 0, LSE = -inf."""
    d = W.decode_case(8, 2, 128, 3, 3000, B=4, seed=5, q_mult=2.0)
    kv_len = [3000, 1, 0, 1234]
    for b, n in enumerate(kv_len):
        d["k"][b, :, n:] = float("nan")
        d["v"][b, :, n:] = float("nan")
    for splits in (0, 1, 5, 40):
        out, lse = run_decode(d, num_splits=splits, kv_len=kv_len)
        d_ref = dict(d)
        d_ref["k"] = torch.nan_to_num(d["k"])  # the oracle only reads [0, kv_len) anyway
        d_ref["v"] = torch.nan_to_num(d["v"])
        check_against_oracle(d_ref, out, lse, kv_len=kv_len)


@pytest.mark.parametrize("Hq,Hkv,Lq", [(32, 2, 4), (8, 8, 1), (12, 4, 3), (64, 4, 2)])
def test_gqa_row_groups(Hq, Hkv, Lq):
    """G*Lq above 16 rows takes several row groups per kv head; G*Lq below 16
    leaves padding rows in the tile."""
    d = W.decode_case(Hq, Hkv, 128, Lq, 700, B=2, seed=7, q_mult=4.0)
    out, lse = run_decode(d)
    check_against_oracle(d, out, lse)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_head_dims_and_dtypes(D, dtype):
    d = W.decode_case(8, 2, D, 2, 1500, B=1, seed=9, q_mult=2.0, dtype=dtype)
    out, lse = run_decode(d)
    check_against_oracle(d, out, lse)


def test_identical_rows_identical_lse():
    d = W.config2(4, 4096, seed=1)
    d["q"][:, :, 1:] = d["q"][:, :, :1]         # 4 identical query rows per head
    out, lse = run_decode(d)
    l = lse.cpu()
    assert torch.equal(l[:, :, 1:], l[:, :, :1].expand_as(l[:, :, 1:])), "identical rows must give identical LSE"
    check_against_oracle(d, out, lse)


def test_lkv_zero():
    d = W.decode_case(4, 2, 128, 1, 0, seed=2)
    out, lse = run_decode(d, num_splits=1)
    assert torch.all(out.float() == 0) and torch.all(torch.isneginf(lse))
