"""GPU parity of attn_fwd_lse_chunks (the partials of several KV chunks of one
query block, in one launch) against the FP64 oracle, through the C ABI.

Each chunk's partial must be the oracle's attention of q over that chunk's keys
alone (O and the LSE of the original logits, smoothed or not), and the
merge_state of the partials the attention over all keys."""
import numpy as np
import pytest
import torch

import oracle as O
import split_kv_merge_attn_b200 as skv
import workloads as W
from tests._gpu_helpers import check_lse, check_o, nan_empty, vmax

pytestmark = pytest.mark.gpu


def run_chunks(d, bounds, smooth_k=0):
    layout = d.get("layout", "HND")
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    if layout == "HND":
        B, H, Sq, D = q.shape
    else:
        B, Sq, H, D = q.shape
    C = len(bounds) - 1
    o_parts = nan_empty((C,) + tuple(q.shape), q.dtype)
    l_parts = nan_empty((C, B, H, Sq), torch.float32)
    skv.attn_fwd_lse_chunks(q, k, v, bounds, d["scale"], layout=layout, smooth_k=smooth_k, out=o_parts, lse=l_parts)
    out = nan_empty(tuple(q.shape), q.dtype)
    lse = nan_empty((B, H, Sq), torch.float32)
    skv.merge_state(o_parts, l_parts, layout, out=out, lse=lse)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    return out, lse, o_parts, l_parts


@pytest.mark.parametrize("dtype,layout", [("bf16", "HND"), ("fp16", "HND"), ("bf16", "NHD")])
@pytest.mark.parametrize("smooth_k", [0, 1])
def test_chunks_partials_and_merge(dtype, layout, smooth_k):
    d = W.config5(dtype=dtype, layout=layout, Sq=384, Sk=1500, H=4)
    bounds = [0, 100, 100, 613, 1280, 1500]     # an empty chunk, ragged ends, a chunk longer than 512
    out, lse, o_parts, l_parts = run_chunks(d, bounds, smooth_k)
    o_ref, l_ref = O.chunked(d["q"], d["k"], d["v"], d["scale"], bounds, layout=layout)
    vm = vmax(d["v"])
    for c in range(len(bounds) - 1):
        if bounds[c + 1] == bounds[c]:
            assert torch.all(o_parts[c] == 0) and torch.all(torch.isneginf(l_parts[c])), f"empty chunk {c}"
            continue
        check_o(o_parts[c], o_ref[c], vm, what=f"O chunk {c}")
        check_lse(l_parts[c], l_ref[c], what=f"LSE chunk {c}")
    o_full, l_full = O.dense(d["q"], d["k"], d["v"], d["scale"], layout=layout)
    check_o(out, o_full, vm)
    check_lse(lse, l_full)


def test_chunks_gqa_and_batches_materialised_smoothing():
    d = W.dense_case(2, 8, 2, 200, 700, 128, seed=9, k_offset=0.5, q_mult=2.0)
    bounds = [0, 256, 300, 700]
    out, lse, o_parts, l_parts = run_chunks(d, bounds, smooth_k=2)
    o_ref, l_ref = O.chunked(d["q"], d["k"], d["v"], d["scale"], bounds)
    for c in range(3):
        check_o(o_parts[c], o_ref[c], vmax(d["v"]))
        check_lse(l_parts[c], l_ref[c], tol=2e-2)   # K' rounded to 16 bits (smooth_k = 2)
    o_full, _ = O.dense(d["q"], d["k"], d["v"], d["scale"])
    check_o(out, o_full, vmax(d["v"]))


def test_chunks_equal_separate_calls_bitwise():
    """One launch over the chunks gives the same bits as one attn_fwd_lse per
    chunk (the same kernel does the same arithmetic per work item)."""
    d = W.config5(Sq=512, Sk=2048, H=4)
    bounds = d["chunk_bounds"]
    _, _, o_parts, l_parts = run_chunks(d, bounds, smooth_k=1)
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    for c in range(len(bounds) - 1):
        a, e = bounds[c], bounds[c + 1]
        o1, l1 = skv.attn_fwd_lse(q, k[:, :, a:e].contiguous(), v[:, :, a:e].contiguous(), d["scale"], smooth_k=1)
        assert torch.equal(o1, o_parts[c]) and torch.equal(l1, l_parts[c]), f"chunk {c}"


def test_chunks_workload5_full_size_sampled():
    d = W.config5()
    out, lse, o_parts, l_parts = run_chunks(d, d["chunk_bounds"], smooth_k=1)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    rng = np.random.default_rng(3)
    rows = [(0, int(h), int(i)) for h, i in zip(rng.integers(0, 16, 120), rng.integers(0, 4096, 120))]
    rows += [(0, 0, 0), (0, 15, 4095)]
    o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"], rows=rows)
    check_o(torch.stack([out[b, h, i] for b, h, i in rows]), o_ref, vmax(d["v"]))
    check_lse(torch.stack([lse[b, h, i] for b, h, i in rows]), l_ref)
    c = 3
    a, e = d["chunk_bounds"][c], d["chunk_bounds"][c + 1]
    _, lc = O.dense(d["q"], d["k"][:, :, a:e], d["v"][:, :, a:e], d["scale"], rows=rows[:40])
    check_lse(torch.stack([l_parts[c, b, h, i] for b, h, i in rows[:40]]), lc)


def test_chunks_rejects_bad_bounds_without_launching():
    lib = skv.lib()
    st = torch.cuda.current_stream().cuda_stream
    import ctypes
    def call(bounds, layout=0, n=None):
        n = len(bounds) - 1 if n is None else n
        arr = (ctypes.c_int32 * len(bounds))(*bounds)
        return lib.attn_fwd_lse_chunks(None, None, None, None, None, 1, 2, 2, 8, 100, 128, 0.1, 0, layout, n, arr, 0,
                                       None, 0, st)
    assert call([0, 50, 100], n=2) == skv.SKV_ERR_INVALID_ARG        # null tensors
    q = torch.zeros(1, 2, 8, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 2, 100, 128, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros(2, 1, 2, 8, 128, dtype=torch.bfloat16, device="cuda")
    def call2(bounds, layout=0):
        arr = (ctypes.c_int32 * len(bounds))(*bounds)
        return lib.attn_fwd_lse_chunks(q.data_ptr(), k.data_ptr(), k.data_ptr(), o.data_ptr(), None, 1, 2, 2, 8, 100,
                                       128, 0.1, 0, layout, len(bounds) - 1, arr, 0, None, 0, st)
    assert call2([1, 50, 100]) == skv.SKV_ERR_INVALID_ARG     # does not start at 0
    assert call2([0, 50, 99]) == skv.SKV_ERR_INVALID_ARG      # does not end at Sk
    assert call2([0, 60, 50, 100]) == skv.SKV_ERR_INVALID_ARG # decreasing
    assert call2([0, 50, 100], layout=2) == skv.SKV_ERR_INVALID_ARG  # TND
    assert call2([0, 50, 100]) == skv.SKV_OK
    torch.cuda.synchronize()
