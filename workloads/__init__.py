"""Seeded synthetic inputs for the attention-with-LSE workloads.

This module only draws random tensors and arranges them in the shapes and
value distributions of the five workloads; it holds none of the attention,
softmax, log-sum-exp or merge arithmetic.  Both the oracle-based tests and the
CUDA path take their inputs from here, so every comparison runs on identical
values.  Everything is generated on the CPU from ``torch.Generator`` with an
explicit seed (fp32 ``randn``, then a cast to the storage dtype), which keeps
inputs reproducible on any machine.

Workloads (all non-causal):

1. dense HND, B=1, H=4, S_q=64, S_k=1000, D=128.  q rows are scaled by
   linspace(0.25, 4.0, 64) so each row has its own LSE ("rows"); the "blocks"
   variant repeats every 16th row 16 times; "koff" adds 0.5 to K (the
   smooth_k case).  Recipe from the ARK return_lse issue, "Reproduction Steps".
2. split-KV decode, D=128, H_q=32, H_kv=8, B=1, Lq in {1,4},
   Lkv in {4096, 8192, 32768}; k, v ~ randn, q ~ 8*randn.  Variants plant
   keys whose scaled logits reach +150, or make every logit strongly positive
   ("allpos", > +88.7 so a fixed exponent offset overflows fp32) or strongly
   negative ("allneg", < -110 so it underflows), after the ExecuTorch split-K
   PR's overflow / underflow regression tests.
3. split-KV decode, D=256, H_q=16, H_kv=4, B=1, Lq in {1,4},
   Lkv in {4096, 16384, 32768}; q scaled per query head by U[0.5, 4].
4. varlen packed TND, H=24, D=128, sequence lengths {512,1024,2048,4096}
   (q length = kv length), q rows of each sequence scaled by
   linspace(0.25, 4) over that sequence's rows.
5. chunked ring-style: B=1, H=16, S_q=4096, S_k=16384, D=128;
   K ~ randn + 0.5, q, v ~ randn; four KV chunks of 4096.
"""
from __future__ import annotations

from typing import Dict, List, Optional

import torch

_DT = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(int(seed))
    return g


def _randn(g: torch.Generator, *shape) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def to_layout(x_hnd: torch.Tensor, layout: str) -> torch.Tensor:
    """Re-arrange a [B, H, S, D] tensor into HND or NHD, contiguous."""
    if layout == "HND":
        return x_hnd.contiguous()
    if layout == "NHD":
        return x_hnd.permute(0, 2, 1, 3).contiguous()
    raise ValueError(layout)


def dense_case(B: int, Hq: int, Hkv: int, Sq: int, Sk: int, D: int, seed: int = 0,
               dtype: str = "bf16", q_mult: float = 1.0, k_offset: float = 0.0,
               row_scale: Optional[tuple] = None) -> Dict[str, torch.Tensor]:
    """Generic dense problem in HND layout: q [B,Hq,Sq,D], k/v [B,Hkv,Sk,D]."""
    g = _gen(seed)
    q = _randn(g, B, Hq, Sq, D) * q_mult
    k = _randn(g, B, Hkv, Sk, D) + k_offset
    v = _randn(g, B, Hkv, Sk, D)
    if row_scale is not None and Sq > 0:
        q = q * torch.linspace(row_scale[0], row_scale[1], Sq).view(1, 1, Sq, 1)
    t = _DT[dtype]
    return {"q": q.to(t), "k": k.to(t), "v": v.to(t), "scale": D ** -0.5}


def config1(variant: str = "rows", seed: int = 0, dtype: str = "bf16") -> Dict[str, torch.Tensor]:
    """Workload 1: B=1, H=4, S_q=64, S_k=1000, D=128, HND."""
    B, H, SQ, SK, D = 1, 4, 64, 1000, 128
    g = _gen(seed)
    t = _DT[dtype]
    q = _randn(g, B, H, SQ, D).to(t)
    k = _randn(g, B, H, SK, D).to(t)
    v = _randn(g, B, H, SK, D).to(t)
    row_scale = torch.linspace(0.25, 4.0, SQ).view(1, 1, SQ, 1)
    q_rows = (q.float() * row_scale).to(t)
    out = {"k": k, "v": v, "scale": D ** -0.5}
    if variant == "rows":
        out["q"] = q_rows
    elif variant in ("blocks", "koff"):
        out["q"] = q_rows[:, :, ::16].repeat_interleave(16, dim=2).contiguous()
        if variant == "koff":
            out["k"] = (k.float() + 0.5).to(t)
    else:
        raise ValueError(variant)
    return out


def decode_case(Hq: int, Hkv: int, D: int, Lq: int, Lkv: int, B: int = 1, seed: int = 0,
                q_mult: float = 1.0, head_scale: Optional[tuple] = None,
                planted: Optional[str] = None, dtype: str = "bf16") -> Dict[str, torch.Tensor]:
    """Decode problem: q [B,Hq,Lq,D], k/v [B,Hkv,Lkv,D] (HND)."""
    g = _gen(seed)
    t = _DT[dtype]
    scale = D ** -0.5
    q = _randn(g, B, Hq, Lq, D) * q_mult
    k = _randn(g, B, Hkv, Lkv, D)
    v = _randn(g, B, Hkv, Lkv, D)
    if head_scale is not None:
        lo, hi = head_scale
        hs = lo + (hi - lo) * torch.rand(Hq, generator=g)
        q = q * hs.view(1, Hq, 1, 1)
    if planted == "allpos":
        # every logit strongly positive: |q| . (|k| + 1.5) / sqrt(D)
        q = q.abs()
        k = k.abs() + 1.5
    elif planted == "allneg":
        q = q.abs()
        k = -(k.abs() + 1.5)
    elif planted == "pos":
        # a few keys per kv head aligned with the first query row of the group's
        # first head, scaled so that row's scaled logit is about +150
        G = Hq // Hkv
        n_plant = min(5, Lkv)
        for b in range(B):
            for hk in range(Hkv):
                qrow = q[b, hk * G, 0]
                idx = torch.randperm(Lkv, generator=g)[:n_plant]
                c = 150.0 / (scale * float(qrow.double().pow(2).sum()))
                k[b, hk, idx] = (qrow * c).unsqueeze(0)
    elif planted is not None:
        raise ValueError(planted)
    return {"q": q.to(t).contiguous(), "k": k.to(t).contiguous(), "v": v.to(t).contiguous(),
            "scale": scale}


def config2(Lq: int, Lkv: int, seed: int = 0, planted: Optional[str] = None,
            dtype: str = "bf16") -> Dict[str, torch.Tensor]:
    """Workload 2: decode D=128, H_q=32, H_kv=8, B=1, q ~ 8*randn."""
    return decode_case(32, 8, 128, Lq, Lkv, seed=seed, q_mult=8.0, planted=planted, dtype=dtype)


def config3(Lq: int, Lkv: int, seed: int = 0, dtype: str = "bf16") -> Dict[str, torch.Tensor]:
    """Workload 3: decode D=256, H_q=16, H_kv=4, B=1, per-head q scale ~ U[0.5, 4]."""
    return decode_case(16, 4, 256, Lq, Lkv, seed=seed, head_scale=(0.5, 4.0), dtype=dtype)


def varlen_case(seqlens_q: List[int], seqlens_k: List[int], Hq: int, Hkv: int, D: int,
                seed: int = 0, dtype: str = "bf16", row_scale: Optional[tuple] = (0.25, 4.0),
                k_offset: float = 0.0) -> Dict[str, object]:
    """Packed TND problem: q [T,Hq,D], k/v [T_k,Hkv,D], int32 cu_seqlens."""
    g = _gen(seed)
    t = _DT[dtype]
    Tq, Tk = sum(seqlens_q), sum(seqlens_k)
    q = _randn(g, Tq, Hq, D)
    k = _randn(g, Tk, Hkv, D) + k_offset
    v = _randn(g, Tk, Hkv, D)
    if row_scale is not None:
        off = 0
        for s in seqlens_q:
            if s > 0:
                q[off:off + s] *= torch.linspace(row_scale[0], row_scale[1], s).view(s, 1, 1)
            off += s
    cu_q = torch.tensor([0] + list(_cumsum(seqlens_q)), dtype=torch.int32)
    cu_k = torch.tensor([0] + list(_cumsum(seqlens_k)), dtype=torch.int32)
    return {"q": q.to(t), "k": k.to(t), "v": v.to(t), "cu_seqlens_q": cu_q,
            "cu_seqlens_k": cu_k, "max_seqlen_q": max(seqlens_q) if seqlens_q else 0,
            "max_seqlen_k": max(seqlens_k) if seqlens_k else 0, "scale": D ** -0.5}


def _cumsum(xs):
    s = 0
    for x in xs:
        s += x
        yield s


CONFIG4_SEQLENS = [512, 1024, 2048, 4096]


def config4(seed: int = 0, dtype: str = "bf16") -> Dict[str, object]:
    """Workload 4: varlen TND, H=24, D=128, seqlens {512,1024,2048,4096}."""
    return varlen_case(CONFIG4_SEQLENS, CONFIG4_SEQLENS, 24, 24, 128, seed=seed, dtype=dtype)


def config5(seed: int = 0, dtype: str = "bf16", layout: str = "HND", Sq: int = 4096,
            Sk: int = 16384, H: int = 16, D: int = 128, n_chunks: int = 4) -> Dict[str, object]:
    """Workload 5: B=1, H=16, S_q=4096, S_k=16384, D=128; K ~ randn + 0.5.

    Returns full q/k/v in the requested layout plus the chunk boundaries along
    the KV axis (equal chunks)."""
    d = dense_case(1, H, H, Sq, Sk, D, seed=seed, dtype=dtype, k_offset=0.5)
    C = Sk // n_chunks
    bounds = [i * C for i in range(n_chunks)] + [Sk]
    return {"q": to_layout(d["q"], layout), "k": to_layout(d["k"], layout),
            "v": to_layout(d["v"], layout), "scale": d["scale"], "chunk_bounds": bounds,
            "layout": layout}
