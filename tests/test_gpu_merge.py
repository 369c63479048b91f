"""GPU parity of merge_state against the oracle's merge (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle as O
import split_kv_merge_attn_b200 as skv
from tests._gpu_helpers import check_lse, check_o, nan_empty

pytestmark = pytest.mark.gpu

DT = {"fp32": torch.float32, "bf16": torch.bfloat16, "fp16": torch.float16}


def make_parts(P, shape_o, shape_l, seed, pdt, empty_frac=0.2, spread=40.0):
    g = torch.Generator().manual_seed(seed)
    o = torch.randn(P, *shape_o, generator=g).to(DT[pdt])
    l = (torch.randn(P, *shape_l, generator=g) * spread).float()
    m = torch.rand(P, *shape_l, generator=g) < empty_frac
    l[m] = float("-inf")
    return o, l


@pytest.mark.parametrize("P", [1, 2, 4, 7, 37])
@pytest.mark.parametrize("pdt,odt", [("fp32", "bf16"), ("bf16", "bf16"), ("fp16", "fp16"), ("fp32", "fp32")])
def test_merge_hnd(P, pdt, odt):
    B, H, S, D = 2, 3, 50, 128
    o, l = make_parts(P, (B, H, S, D), (B, H, S), seed=P, pdt=pdt)
    if P > 1:
        l[:, 0, 0, :5] = float("-inf")       # rows with no part at all
    o_ref, l_ref = O.merge(O.to_f64(o), O.to_f64(l))
    out = nan_empty((B, H, S, D), DT[odt])
    lse = nan_empty((B, H, S), torch.float32)
    skv.merge_state(o.cuda(), l.cuda(), "HND", out=out, lse=lse)
    torch.cuda.synchronize()
    tol = 1e-5 if odt == "fp32" else 8e-3       # one rounding of the output to 16 bits
    check_o(out, o_ref, float(o.float().abs().max()), tol=tol)
    check_lse(lse, l_ref, tol=1e-4)


@pytest.mark.parametrize("layout", ["NHD", "TND"])
def test_merge_token_major_layouts(layout):
    P, B, H, S, D = 4, (2 if layout == "NHD" else 1), 5, 33, 64
    o_bhsd, l = make_parts(P, (B, H, S, D), (B, H, S), seed=11, pdt="bf16")
    o_ref, l_ref = O.merge(O.to_f64(o_bhsd), O.to_f64(l))
    if layout == "NHD":
        o_in = o_bhsd.permute(0, 1, 3, 2, 4).contiguous()          # [P,B,S,H,D]
        l_in = l
        out = nan_empty((B, S, H, D), torch.bfloat16)
        skv.merge_state(o_in.cuda(), l_in.cuda(), "NHD", out=out, lse=nan_empty((B, H, S), torch.float32))
        got = out.permute(0, 2, 1, 3)
    else:
        o_in = o_bhsd[:, 0].permute(0, 2, 1, 3).contiguous()         # [P,T,H,D]
        l_in = l[:, 0]                                              # [P,H,T]
        out = nan_empty((S, H, D), torch.bfloat16)
        lse = nan_empty((H, S), torch.float32)
        skv.merge_state(o_in.cuda(), l_in.cuda(), "TND", out=out, lse=lse)
        check_lse(lse, l_ref[0], tol=1e-4)
        got = out.permute(1, 0, 2)[None]
    torch.cuda.synchronize()
    check_o(got.contiguous(), o_ref, float(o_bhsd.float().abs().max()), tol=8e-3)


def test_merge_extreme_lse_and_ignored_garbage():
    """LSE parts spanning +-150 log2 units, and a -inf part whose O slot holds
    NaN: it carries no weight and is never read."""
    B, H, S, D = 1, 2, 16, 128
    o = torch.randn(3, B, H, S, D, dtype=torch.float32)
    l = torch.empty(3, B, H, S)
    l[0] = 150.0
    l[1] = -150.0
    l[2] = float("-inf")
    o[2] = float("nan")
    out = nan_empty((B, H, S, D), torch.bfloat16)
    lse = nan_empty((B, H, S), torch.float32)
    skv.merge_state(o.cuda(), l.cuda(), "HND", out=out, lse=lse)
    o_ref, l_ref = O.merge(O.to_f64(o[:2]), O.to_f64(l[:2]))
    check_o(out, o_ref, float(o[:2].abs().max()), tol=8e-3)
    check_lse(lse, l_ref, tol=1e-4)


def test_merge_of_splits_reproduces_full_attention():
    """Split the keys of a dense problem, take the oracle's per-split results
    as parts, merge on the GPU, compare with the full oracle run."""
    import workloads as W
    d = W.dense_case(1, 4, 4, 40, 300, 128, seed=2, q_mult=3.0)
    bounds = [0, 64, 65, 200, 300]
    o_parts, l_parts = O.chunked(d["q"], d["k"], d["v"], d["scale"], bounds)
    o_full, l_full = O.dense(d["q"], d["k"], d["v"], d["scale"])
    out = nan_empty((1, 4, 40, 128), torch.bfloat16)
    lse = nan_empty((1, 4, 40), torch.float32)
    skv.merge_state(torch.from_numpy(o_parts).float().cuda(), torch.from_numpy(l_parts).float().cuda(),
                    "HND", out=out, lse=lse)
    check_o(out, o_full, float(d["v"].float().abs().max()))
    check_lse(lse, l_full)


@pytest.mark.parametrize("D", [64, 96, 256])
@pytest.mark.parametrize("P", [8, 40, 200])
@pytest.mark.parametrize("layout", ["HND", "NHD"])
def test_merge_few_rows_many_parts(D, P, layout):
    """The per-row kernels (few rows, P >= 8 parts): several batches of parts
    per thread at P = 200, empty parts, rows without any part, the
    slice-by-shuffle variant (D = 64, 256) and the general one (D = 96)."""
    B, H, S = 1, 3, 5
    o, l = make_parts(P, (B, H, S, D), (B, H, S), seed=D + P, pdt="fp32", empty_frac=0.3)
    l[:, 0, 1, 2] = float("-inf")
    o_ref, l_ref = O.merge(O.to_f64(o), O.to_f64(l))
    lse = nan_empty((B, H, S), torch.float32)
    if layout == "HND":
        out = nan_empty((B, H, S, D), torch.bfloat16)
        skv.merge_state(o.cuda(), l.cuda(), "HND", out=out, lse=lse)
        got = out
    else:
        out = nan_empty((B, S, H, D), torch.bfloat16)
        skv.merge_state(o.permute(0, 1, 3, 2, 4).contiguous().cuda(), l.cuda(), "NHD", out=out, lse=lse)
        got = out.permute(0, 2, 1, 3)
    torch.cuda.synchronize()
    check_o(got.contiguous(), o_ref, float(o.abs().max()), tol=8e-3)
    check_lse(lse, l_ref, tol=1e-4)
    assert torch.all(lse[0, 1, 2] == float("-inf")) and torch.all(got[0, 1, 2] == 0)
