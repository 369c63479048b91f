"""Host-only checks of the C ABI (no GPU needed).

* the shared library loads and exports every function include/splitkv.h declares;
* every entry point rejects invalid arguments with the documented status
  before touching the device (only invalid argument sets are passed here, so
  no call can reach a launch);
* the integer planners (split plan, varlen work order) match the oracle's
  independent restatement bit for bit.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
import split_kv_merge_attn_b200 as skv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "splitkv.h")

INVALID, UNSUPPORTED, WS_SMALL = skv.SKV_ERR_INVALID_ARG, skv.SKV_ERR_UNSUPPORTED, skv.SKV_ERR_WORKSPACE_TOO_SMALL
P16 = 0x10000  # an aligned, never-dereferenced address: only used with otherwise INVALID arguments
BAD = 0x10001  # misaligned


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[\w\*\s]+?\b(\w+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "defined")))


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert {"attn_fwd_lse", "attn_splitkv_decode", "merge_state"} <= set(names)
    L = skv.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(skv.SIGNATURES), "binding signatures cover exactly the header"


def test_status_strings():
    for s in range(5):
        assert skv.status_string(s).startswith("SKV_")
    assert skv.lib().skv_version().decode().count(".") == 2


def fwd(**kw):
    a = dict(q=P16, k=P16, v=P16, out=P16, lse=None, B=1, Hq=4, Hkv=4, Sq=64, Sk=64, D=128, scale=0.1, dt=0,
             layout=0, cq=None, ck=None, mq=0, mk=0, smooth=0, ws=None, wsb=0)
    a.update(kw)
    return skv.lib().attn_fwd_lse(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Sq"],
                                  a["Sk"], a["D"], a["scale"], a["dt"], a["layout"], a["cq"], a["ck"], a["mq"],
                                  a["mk"], a["smooth"], a["ws"], a["wsb"], None)


def test_attn_fwd_lse_rejects_invalid_arguments():
    # each case breaks exactly one rule and also keeps q = NULL or another error
    # in front of any launch: the expected status is what validation returns
    assert fwd(q=None) == INVALID
    assert fwd(out=None) == INVALID
    assert fwd(k=BAD) == INVALID
    assert fwd(lse=0x10002) == INVALID
    assert fwd(Hq=6, Hkv=4) == INVALID                 # Hq % Hkv != 0
    assert fwd(B=0) == INVALID
    assert fwd(Sq=-1) == INVALID
    assert fwd(scale=float("nan")) == INVALID
    assert fwd(scale=-1.0) == INVALID
    assert fwd(layout=7) == INVALID
    assert fwd(dt=9) == INVALID
    assert fwd(smooth=3) == INVALID
    assert fwd(cq=P16, ck=P16) == INVALID              # cu_seqlens with a dense layout
    assert fwd(layout=2) == INVALID                    # varlen without cu_seqlens
    assert fwd(layout=2, cq=P16, ck=P16, mq=65, Sq=64) == INVALID   # max_seqlen_q > total_q
    assert fwd(D=96) == UNSUPPORTED
    assert fwd(dt=2) == UNSUPPORTED
    need = skv.attn_fwd_lse_workspace(1, 4, 4, 64, 128, "bf16", "HND", 1)
    assert need > 0
    assert fwd(smooth=1, ws=P16, wsb=need - 1) == WS_SMALL
    assert fwd(smooth=1, ws=None, wsb=need) == INVALID   # claims bytes but no pointer
    assert fwd(smooth=1, ws=0x10010, wsb=need) == INVALID  # not 256-byte aligned


def dec(**kw):
    a = dict(q=P16, k=P16, v=P16, out=P16, lse=None, B=1, Hq=32, Hkv=8, Lq=1, Lkv=4096, D=128, scale=0.1, dt=0,
             kv_len=None, splits=1, ws=None, wsb=0)
    a.update(kw)
    return skv.lib().attn_splitkv_decode(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                                         a["Lq"], a["Lkv"], a["D"], a["scale"], a["dt"], a["kv_len"], a["splits"],
                                         a["ws"], a["wsb"], None)


def test_attn_splitkv_decode_rejects_invalid_arguments():
    assert dec(q=None) == INVALID
    assert dec(v=BAD) == INVALID
    assert dec(kv_len=0x10002) == INVALID
    assert dec(Hq=30) == INVALID
    assert dec(Lq=0) == INVALID
    assert dec(Lkv=-1) == INVALID
    assert dec(splits=257) == INVALID
    assert dec(splits=-1) == INVALID
    assert dec(scale=0.0) == INVALID
    assert dec(D=96) == UNSUPPORTED
    assert dec(dt=2) == UNSUPPORTED
    assert dec(B=70000, Hkv=1, Hq=1) == UNSUPPORTED    # grid.y limit
    need = skv.attn_splitkv_workspace(1, 32, 1, 128, 8)
    assert need == O_ws(1, 32, 1, 128, 8)
    assert dec(splits=8, ws=P16, wsb=need - 1) == WS_SMALL
    assert dec(splits=8, ws=None, wsb=need) == INVALID


def dec_fused(**kw):
    a = dict(q=P16, k=P16, v=P16, out=P16, lse=None, B=1, Hq=32, Hkv=8, Lq=1, Lkv=4096, D=128, scale=0.1, dt=0,
             kv_len=None, splits=1, ws=None, wsb=0)
    a.update(kw)
    return skv.lib().attn_splitkv_decode_fused(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["Hq"],
                                               a["Hkv"], a["Lq"], a["Lkv"], a["D"], a["scale"], a["dt"], a["kv_len"],
                                               a["splits"], a["ws"], a["wsb"], None)


def test_attn_splitkv_decode_fused_validates_like_the_two_kernel_decode():
    assert dec_fused(q=None) == INVALID
    assert dec_fused(Hq=30) == INVALID
    assert dec_fused(splits=257) == INVALID
    assert dec_fused(D=96) == UNSUPPORTED
    need = skv.attn_splitkv_workspace(1, 32, 1, 128, 8)
    assert dec_fused(splits=8, ws=P16, wsb=need - 1) == WS_SMALL
    assert dec_fused(splits=8, ws=None, wsb=need) == INVALID


def test_workspace_init_arguments():
    assert skv.lib().attn_splitkv_workspace_init(None, 0, None) == skv.SKV_OK
    assert skv.lib().attn_splitkv_workspace_init(None, 256, None) == INVALID


def O_ws(B, Hq, Lq, D, S):
    """Workspace of S splits: fp32 partial O, fp32 partial LSE, then one int32
    arrival counter per row (the fused decode's), each 256-byte aligned."""
    a = lambda x: (x + 255) // 256 * 256
    rows = B * Hq * Lq
    return a(S * rows * D * 4) + a(S * rows * 4) + a(rows * 4) if S > 1 else 0


def test_decode_workspace_sizes():
    for args in [(1, 32, 1, 128, 37), (1, 16, 4, 256, 64), (2, 8, 3, 64, 1), (1, 1, 1, 64, 2)]:
        assert skv.attn_splitkv_workspace(*args) == O_ws(*args)


def mrg(**kw):
    a = dict(o=P16, l=P16, out=P16, lse=None, P=2, B=1, H=4, S=8, D=128, layout=0, pdt=2, odt=0, so=0, sl=0)
    a.update(kw)
    return skv.lib().merge_state(a["o"], a["l"], a["out"], a["lse"], a["P"], a["B"], a["H"], a["S"], a["D"],
                                 a["layout"], a["pdt"], a["odt"], a["so"], a["sl"], None)


def test_merge_state_rejects_invalid_arguments():
    assert mrg(o=None) == INVALID
    assert mrg(out=BAD) == INVALID
    assert mrg(l=0x10002) == INVALID
    assert mrg(P=0) == INVALID
    assert mrg(D=12) == INVALID
    assert mrg(layout=5) == INVALID
    assert mrg(pdt=7) == INVALID
    assert mrg(so=100) == INVALID         # part stride smaller than one part
    assert mrg(sl=3) == INVALID
    assert mrg(B=0) == skv.SKV_OK         # zero rows: valid no-op, nothing launched


def test_split_plan_matches_oracle_bit_exact():
    rng = np.random.default_rng(0)
    cases = [(1, 32, 8, 1, n, 148) for n in (0, 1, 63, 64, 100, 4096, 8192, 32768)]
    cases += [(1, 32, 8, 4, n, 148) for n in (4096, 32768)]
    cases += [(1, 16, 4, lq, n, 148) for lq in (1, 4) for n in (4096, 16384, 32768)]
    for _ in range(200):
        hkv = int(rng.integers(1, 9))
        cases.append((int(rng.integers(1, 9)), hkv * int(rng.integers(1, 9)), hkv, int(rng.integers(1, 9)),
                      int(rng.integers(0, 70000)), int(rng.integers(1, 200))))
    for (B, Hq, Hkv, Lq, n, sms) in cases:
        for D in (64, 128, 256):
            s, bounds = skv.attn_splitkv_plan(B, Hq, Hkv, Lq, n, D, sms, 0)
            assert s == O.auto_num_splits(B, Hkv, Hq, Lq, n, sms, D=D), (B, Hq, Hkv, Lq, n, sms, D)
            assert bounds == O.split_bounds(n, s)
        for req in (1, 3, 37, 256):
            s2, b2 = skv.attn_splitkv_plan(B, Hq, Hkv, Lq, n, 128, sms, req)
            assert s2 == req and b2 == O.split_bounds(n, req)


def test_split_plan_examples_quoted_in_the_header():
    """include/splitkv.h quotes the automatic plan on the decode workloads'
    shapes with 148 SMs; the library must give exactly those counts."""
    assert skv.attn_splitkv_plan(1, 32, 8, 1, 4096, 128, 148, 0)[0] == 16
    assert skv.attn_splitkv_plan(1, 32, 8, 1, 32768, 128, 148, 0)[0] == 19
    assert skv.attn_splitkv_plan(1, 16, 4, 1, 32768, 256, 148, 0)[0] == 25


def test_varlen_plan_matches_oracle_bit_exact():
    rng = np.random.default_rng(1)
    cu = [0, 512, 1536, 3584, 7680]
    assert skv.attn_varlen_plan(cu, cu, 24) == O.varlen_schedule(cu, cu, 24)[:2]
    for _ in range(100):
        B = int(rng.integers(1, 40))
        lq = rng.integers(0, 1200, size=B)
        lk = rng.integers(0, 5, size=B) * int(rng.integers(1, 400))   # many ties
        cq = [0] + list(np.cumsum(lq).astype(int))
        ck = [0] + list(np.cumsum(lk).astype(int))
        H = int(rng.integers(1, 33))
        order, offsets, _ = O.varlen_schedule(cq, ck, H)
        assert skv.attn_varlen_plan(cq, ck, H) == (order, offsets)
        # D = 256 runs one 128-row query tile per CTA
        order, offsets, _ = O.varlen_schedule(cq, ck, H, rows_per_cta=128)
        assert skv.attn_varlen_plan(cq, ck, H, D=256) == (order, offsets)


def test_fwd_workspace_sizes():
    a = lambda x: (x + 255) // 256 * 256
    assert skv.attn_fwd_lse_workspace(1, 16, 16, 4096, 128, "bf16", "HND", 0) == 0
    # varlen: order[B] and offsets[B+1]
    assert skv.attn_fwd_lse_workspace(4, 24, 24, 7680, 128, "bf16", "TND", 0) == a(16) + a(20)
    # smooth (shift): mean [B,Hkv,D] + per-256-key partial sums
    assert skv.attn_fwd_lse_workspace(1, 16, 16, 4096, 128, "bf16", "HND", 1) == a(16 * 128 * 4) + a(16 * 16 * 128 * 4)
    # materialised K' adds one copy of K
    assert skv.attn_fwd_lse_workspace(1, 16, 16, 4096, 128, "bf16", "NHD", 2) == (
        a(16 * 128 * 4) + a(16 * 16 * 128 * 4) + a(4096 * 16 * 128 * 2))


def test_binding_rejects_inconsistent_tensors():
    """The Python binding checks the tensors of one call against each other
    before anything reaches the library (which sees only q's dtype and the
    sizes read off q and k): mismatched K/V shapes, a wrong-size output, LSE or
    kv_len buffer, mixed dtypes.  CPU tensors suffice: these checks come before
    the device check."""
    import torch
    bf = torch.bfloat16
    q = torch.zeros(1, 4, 64, 128, dtype=bf)
    k = torch.zeros(1, 2, 100, 128, dtype=bf)
    v = k.clone()
    with pytest.raises(ValueError, match="v has shape"):
        skv.attn_fwd_lse(q, k, v[:, :, :99].contiguous(), 0.1)
    with pytest.raises(ValueError, match="dtype"):
        skv.attn_fwd_lse(q, k, v.half(), 0.1)
    with pytest.raises(ValueError, match="out has shape"):
        skv.attn_fwd_lse(q, k, v, 0.1, out=torch.zeros(1, 4, 63, 128, dtype=bf))
    with pytest.raises(ValueError, match="lse must be float32"):
        skv.attn_fwd_lse(q, k, v, 0.1, lse=torch.zeros(1, 4, 64, dtype=torch.float64))
    with pytest.raises(ValueError, match="k has shape"):
        skv.attn_fwd_lse(q, torch.zeros(1, 2, 100, 64, dtype=bf), v, 0.1)
    # varlen
    qt, kt = torch.zeros(10, 4, 128, dtype=bf), torch.zeros(12, 2, 128, dtype=bf)
    cu = torch.tensor([0, 4, 10], dtype=torch.int32)
    with pytest.raises(ValueError, match="cu_seqlens_q must be int32"):
        skv.attn_fwd_lse(qt, kt, kt, 0.1, layout="TND", cu_seqlens_q=cu.long(), cu_seqlens_k=cu,
                         max_seqlen_q=6, max_seqlen_k=8)
    with pytest.raises(ValueError, match="same length"):
        skv.attn_fwd_lse(qt, kt, kt, 0.1, layout="TND", cu_seqlens_q=cu, cu_seqlens_k=cu[:2],
                         max_seqlen_q=6, max_seqlen_k=8)
    with pytest.raises(ValueError, match="lse has shape"):
        skv.attn_fwd_lse(qt, kt, kt, 0.1, layout="TND", cu_seqlens_q=cu, cu_seqlens_k=cu, max_seqlen_q=6,
                         max_seqlen_k=8, lse=torch.zeros(10, 4))
    # decode
    qd = torch.zeros(1, 4, 1, 128, dtype=bf)
    with pytest.raises(ValueError, match="kv_len has shape"):
        skv.attn_splitkv_decode(qd, k, v, 0.1, kv_len=torch.zeros(2, dtype=torch.int32))
    with pytest.raises(ValueError, match="kv_len must be int32"):
        skv.attn_splitkv_decode(qd, k, v, 0.1, kv_len=torch.zeros(1, dtype=torch.int64))
    with pytest.raises(ValueError, match="k has shape"):
        skv.attn_splitkv_decode(qd, torch.zeros(1, 2, 100, 64, dtype=bf), v, 0.1)
    with pytest.raises(ValueError, match="no causal variant"):
        skv.attn_splitkv_decode(qd, k, v, 0.1, fused=True, causal=True)
    # int8 prefill
    with pytest.raises(ValueError, match="v has shape"):
        skv.attn_fwd_lse_int8(q, k, v[:, :1].contiguous(), 0.1)
    # merge
    o = torch.zeros(2, 1, 4, 64, 128, dtype=bf)
    lp = torch.zeros(2, 1, 4, 64)
    with pytest.raises(ValueError, match="lse_parts has shape"):
        skv.merge_state(o, lp[:, :, :, :63].contiguous())
    with pytest.raises(ValueError, match="lse_parts must be float32"):
        skv.merge_state(o, lp.double())
    with pytest.raises(ValueError, match="out has shape"):
        skv.merge_state(o, lp, out=torch.zeros(1, 4, 64, 64, dtype=bf))
    with pytest.raises(ValueError, match="lse_parts has shape"):
        skv.merge_state(o[:, 0].contiguous(), lp, layout="TND")
    # a consistent call made of CPU tensors stops at the device check
    with pytest.raises(ValueError, match="CUDA"):
        skv.attn_fwd_lse(q, k, v, 0.1)
    with pytest.raises(ValueError, match="CUDA"):
        skv.merge_state(o, lp)
