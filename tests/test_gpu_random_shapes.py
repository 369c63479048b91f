"""Seeded sweeps of small, irregular problems against the FP64 oracle: every
entry point on shapes the fixed-shape tests do not pick (ragged lengths on
both sides of the 128-row/128-key tiles, one-key and empty key ranges, GQA
ratios, all head dimensions, both layouts and 16-bit types, causal masks,
smoothing, explicit split counts and device kv_len)."""
import numpy as np
import pytest
import torch

import oracle as O
import split_kv_merge_attn_b200 as skv
import workloads as W
from tests._gpu_helpers import check_lse, check_o, nan_empty, vmax

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "fp16": torch.float16}


def _prefill_cases(n=40, seed=101):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        D = int(rng.choice([64, 128, 256]))
        Hkv = int(rng.integers(1, 4))
        G = int(rng.choice([1, 2, 4]))
        Sq = int(rng.choice([1, 7, 127, 128, 129, 255, 256, 257, int(rng.integers(1, 400))]))
        Sk = int(rng.choice([0, 1, 63, 64, 65, 128, 129, int(rng.integers(1, 500))]))
        causal = bool(rng.integers(0, 2))
        smooth = 0 if causal else int(rng.integers(0, 2))
        cases.append(dict(B=int(rng.integers(1, 3)), Hkv=Hkv, Hq=Hkv * G, Sq=Sq, Sk=Sk, D=D,
                          layout=str(rng.choice(["HND", "NHD"])), dtype=str(rng.choice(["bf16", "fp16"])),
                          causal=causal, smooth=smooth, seed=seed + i))
    return cases


@pytest.mark.parametrize("c", _prefill_cases(), ids=lambda c: "D{D}_H{Hq}x{Hkv}_Sq{Sq}_Sk{Sk}_{layout}_{dtype}"
                         "_c{causal}_s{smooth}".format(**c))
def test_dense_prefill_random(c):
    d = W.dense_case(c["B"], c["Hq"], c["Hkv"], c["Sq"], c["Sk"], c["D"], seed=c["seed"], dtype=c["dtype"])
    q, k, v = d["q"], d["k"], d["v"]
    if c["layout"] == "NHD":
        q, k, v = (x.permute(0, 2, 1, 3).contiguous() for x in (q, k, v))
    out = nan_empty(q.shape, q.dtype)
    lse = nan_empty((c["B"], c["Hq"], c["Sq"]), torch.float32)
    skv.attn_fwd_lse(q.cuda(), k.cuda(), v.cuda(), d["scale"], layout=c["layout"], smooth_k=c["smooth"],
                     causal=c["causal"], out=out, lse=lse)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"], causal=c["causal"])
    got = out.permute(0, 2, 1, 3) if c["layout"] == "NHD" else out
    check_o(got.contiguous(), o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


def _varlen_cases(n=20, seed=202):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        B = int(rng.integers(1, 6))
        lq = [int(rng.choice([0, 1, 100, 128, 129, 256, 300, int(rng.integers(1, 600))])) for _ in range(B)]
        lk = [int(rng.choice([0, 1, 64, 128, 257, int(rng.integers(1, 700))])) for _ in range(B)]
        if sum(lq) == 0:
            lq[0] = 5
        Hkv = int(rng.integers(1, 3))
        cases.append(dict(lq=lq, lk=lk, Hkv=Hkv, Hq=Hkv * int(rng.choice([1, 3])), D=int(rng.choice([64, 128, 256])),
                          dtype=str(rng.choice(["bf16", "fp16"])), causal=bool(rng.integers(0, 2)), seed=seed + i))
    return cases


@pytest.mark.parametrize("c", _varlen_cases(), ids=lambda c: "D{D}_B{n}_c{causal}_{dtype}".format(n=len(c["lq"]), **c))
def test_varlen_prefill_random(c):
    d = W.varlen_case(c["lq"], c["lk"], c["Hq"], c["Hkv"], c["D"], seed=c["seed"], dtype=c["dtype"])
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    out = nan_empty(q.shape, q.dtype)
    lse = nan_empty((c["Hq"], q.shape[0]), torch.float32)
    skv.attn_fwd_lse(q, k, v, d["scale"], layout="TND", cu_seqlens_q=d["cu_seqlens_q"].cuda(),
                     cu_seqlens_k=d["cu_seqlens_k"].cuda(), max_seqlen_q=d["max_seqlen_q"],
                     max_seqlen_k=d["max_seqlen_k"], causal=c["causal"], out=out, lse=lse)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    o_ref, l_ref = O.varlen(d["q"], d["k"], d["v"], d["cu_seqlens_q"], d["cu_seqlens_k"], d["scale"],
                            causal=c["causal"])
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


def _decode_cases(n=32, seed=303):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        Hkv = int(rng.integers(1, 5))
        Lkv = int(rng.choice([1, 63, 64, 65, 500, 1000, int(rng.integers(1, 3000))]))
        causal = bool(rng.integers(0, 2))
        cases.append(dict(B=int(rng.integers(1, 4)), Hkv=Hkv, Hq=Hkv * int(rng.choice([1, 2, 4, 8])),
                          Lq=int(rng.integers(1, 5)), Lkv=Lkv, D=int(rng.choice([64, 128, 256])),
                          dtype=str(rng.choice(["bf16", "fp16"])), causal=causal,
                          splits=int(rng.choice([0, 0, 1, 3, 17])), kv_len=bool(rng.integers(0, 2)),
                          fused=(not causal) and bool(rng.integers(0, 2)), seed=seed + i))
    return cases


@pytest.mark.parametrize("c", _decode_cases(), ids=lambda c: "D{D}_H{Hq}x{Hkv}_Lq{Lq}_Lkv{Lkv}_s{splits}_c{causal}"
                         "_f{fused}_kl{kv_len}".format(**c))
def test_decode_random(c):
    d = W.dense_case(c["B"], c["Hq"], c["Hkv"], c["Lq"], c["Lkv"], c["D"], seed=c["seed"], dtype=c["dtype"], q_mult=3.0)
    rng = np.random.default_rng(c["seed"])
    kl = [int(rng.integers(0, c["Lkv"] + 1)) for _ in range(c["B"])] if c["kv_len"] else None
    kv_len = torch.tensor(kl, dtype=torch.int32, device="cuda") if kl is not None else None
    out, lse = skv.attn_splitkv_decode(d["q"].cuda(), d["k"].cuda(), d["v"].cuda(), d["scale"], kv_len=kv_len,
                                       num_splits=c["splits"], fused=c["fused"], causal=c["causal"])
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    o_ref, l_ref = O.decode(d["q"], d["k"], d["v"], d["scale"], kv_len=kl, causal=c["causal"])
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


def _merge_cases(n=20, seed=404):
    rng = np.random.default_rng(seed)
    return [dict(P=int(rng.choice([1, 2, 3, 5, 8, 13, 40])), B=int(rng.integers(1, 3)), H=int(rng.integers(1, 5)),
                 S=int(rng.choice([1, 17, 130, int(rng.integers(1, 700))])), D=int(rng.choice([8, 64, 96, 128, 256])),
                 pdt=str(rng.choice(["fp32", "bf16", "fp16"])), odt=str(rng.choice(["fp32", "bf16", "fp16"])),
                 layout=str(rng.choice(["HND", "NHD"])), seed=seed + i) for i in range(n)]


@pytest.mark.parametrize("c", _merge_cases(), ids=lambda c: "P{P}_S{S}_D{D}_{pdt}_{odt}_{layout}".format(**c))
def test_merge_random(c):
    g = torch.Generator().manual_seed(c["seed"])
    dts = {"fp32": torch.float32, "bf16": torch.bfloat16, "fp16": torch.float16}
    P, B, H, S, D = c["P"], c["B"], c["H"], c["S"], c["D"]
    o = torch.randn(P, B, H, S, D, generator=g).to(dts[c["pdt"]])
    l = (torch.randn(P, B, H, S, generator=g) * 30).float()
    l[torch.rand(P, B, H, S, generator=g) < 0.25] = float("-inf")
    o_ref, l_ref = O.merge(O.to_f64(o), O.to_f64(l))
    o_in = o if c["layout"] == "HND" else o.permute(0, 1, 3, 2, 4).contiguous()
    out = nan_empty(o_in.shape[1:], dts[c["odt"]])
    lse = nan_empty((B, H, S), torch.float32)
    skv.merge_state(o_in.cuda(), l.cuda(), c["layout"], out=out, lse=lse)
    torch.cuda.synchronize()
    got = out if c["layout"] == "HND" else out.permute(0, 2, 1, 3)
    tol = 1e-5 if c["odt"] == "fp32" else 8e-3
    check_o(got.contiguous(), o_ref, float(o.float().abs().max()), tol=tol)
    check_lse(lse, l_ref, tol=1e-4)
