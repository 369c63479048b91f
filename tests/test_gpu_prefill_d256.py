"""GPU parity of attn_fwd_lse at head dimension D = 256 (one 128-row query
tile per CTA) against the FP64 oracle, through the C ABI: dense HND and NHD
with GQA and ragged sizes, fp16, varlen with its device work order, smooth_k
in both modes, the causal variant and the multi-chunk call."""
import numpy as np
import pytest
import torch

import oracle as O
import split_kv_merge_attn_b200 as skv
import workloads as W
from tests._gpu_helpers import check_lse, check_o, nan_empty, vmax
from tests.test_gpu_prefill import run_dense, run_varlen

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("layout", ["HND", "NHD"])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_d256_dense_ragged_gqa(layout, dtype):
    d = W.dense_case(2, 8, 2, 300, 333, 256, seed=41, dtype=dtype, q_mult=2.0)
    if layout == "NHD":
        d = dict(d, q=W.to_layout(d["q"], "NHD"), k=W.to_layout(d["k"], "NHD"), v=W.to_layout(d["v"], "NHD"))
    out, lse = run_dense(d, layout=layout)
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"], layout=layout)
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


@pytest.mark.parametrize("Sq,Sk", [(1, 1), (129, 1), (128, 128), (257, 383), (64, 0), (700, 1100)])
def test_d256_edge_sizes(Sq, Sk):
    d = W.dense_case(1, 2, 1, Sq, Sk, 256, seed=Sq + 3 * Sk, q_mult=3.0)
    out, lse = run_dense(d)
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"])
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


def test_d256_large_logits_and_rescales():
    """Logits that rise from tile to tile (the lazy running max is raised and
    O rescaled in TMEM) and one planted key at +150."""
    d = W.dense_case(1, 2, 2, 256, 1024, 256, seed=5)
    k = d["k"].float()
    k = k * torch.linspace(0.1, 3.0, 1024).view(1, 1, 1024, 1)
    q = d["q"].float() * 2.0
    qn = q[0, 0, 7] / q[0, 0, 7].norm()
    k[0, 0, 900] = qn * 150.0 / d["scale"] / q[0, 0, 7].norm()
    d = dict(d, q=q.bfloat16(), k=k.bfloat16())
    out, lse = run_dense(d)
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"])
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


def test_d256_varlen_and_work_order():
    d = W.varlen_case([100, 900, 40, 700, 513], [50, 900, 900, 10, 0], 4, 2, 256, seed=2)
    out, lse = run_varlen(d)
    o_ref, l_ref = O.varlen(d["q"], d["k"], d["v"], d["cu_seqlens_q"], d["cu_seqlens_k"], d["scale"])
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)
    B = 5
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    nbytes = skv.attn_fwd_lse_workspace(B, 4, 2, k.shape[0], 256, "bf16", "TND", 0)
    ws = torch.full((nbytes,), 0xFF, dtype=torch.uint8, device="cuda")
    skv.attn_fwd_lse(q, k, v, d["scale"], layout="TND", cu_seqlens_q=d["cu_seqlens_q"].cuda(),
                     cu_seqlens_k=d["cu_seqlens_k"].cuda(), max_seqlen_q=900, max_seqlen_k=900, workspace=ws)
    torch.cuda.synchronize()
    w = ws.cpu().numpy()
    order = np.frombuffer(w[:4 * B].tobytes(), dtype=np.int32).tolist()
    offsets = np.frombuffer(w[256:256 + 4 * (B + 1)].tobytes(), dtype=np.int32).tolist()
    o_order, o_offsets, _ = O.varlen_schedule(d["cu_seqlens_q"], d["cu_seqlens_k"], 4, rows_per_cta=128)
    assert order == o_order and offsets == o_offsets


@pytest.mark.parametrize("smooth_k", [1, 2])
def test_d256_smooth_k(smooth_k):
    d = W.dense_case(1, 4, 2, 200, 700, 256, seed=8, k_offset=0.5)
    out, lse = run_dense(d, smooth_k=smooth_k)
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"])
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref, tol=1e-3 if smooth_k == 1 else 2e-2)


def test_d256_causal():
    d = W.dense_case(1, 4, 2, 300, 500, 256, seed=9, q_mult=1.5)
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    out, lse = skv.attn_fwd_lse(q, k, v, d["scale"], causal=True, out=nan_empty(q.shape, q.dtype),
                                lse=nan_empty((1, 4, 300), torch.float32))
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"], causal=True)
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


def test_d256_chunks():
    d = W.dense_case(1, 4, 4, 256, 900, 256, seed=12, k_offset=0.5)
    bounds = [0, 128, 129, 600, 900]
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    o_parts, l_parts = skv.attn_fwd_lse_chunks(q, k, v, bounds, d["scale"], smooth_k=1)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    o_ref, l_ref = O.chunked(d["q"], d["k"], d["v"], d["scale"], bounds)
    for c in range(4):
        check_o(o_parts[c], o_ref[c], vmax(d["v"]))
        check_lse(l_parts[c], l_ref[c])
