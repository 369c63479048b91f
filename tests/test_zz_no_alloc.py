"""GPU test of attn_splitkv_decode_static, the decode entry point for callers
that cannot allocate device memory (its scratch is a fixed device array inside
the library instead of a caller workspace).

It is called directly through the C ABI and compared with the regular
attn_splitkv_decode, on two calls in a row with different inputs (the second
call must not see anything of the first one's scratch contents), with the
parity tolerances the other GPU tests use.  The file name sorts last so that a
run that stops at the first failure has run every other test already; the test
also works alone in a fresh process, where its first call sets the scratch
array up.
"""
import pytest
import torch

import split_kv_merge_attn_b200 as skv
import workloads as W
from tests._gpu_helpers import LSE_TOL, O_TOL, nan_empty

pytestmark = pytest.mark.gpu


def _static_call(d, num_splits=0):
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    B, Hq, Lq, D = q.shape
    _, Hkv, Lkv, _ = k.shape
    out = nan_empty(q.shape, q.dtype)
    lse = nan_empty((B, Hq, Lq), torch.float32)
    st = skv.lib().attn_splitkv_decode_static(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Lq, Lkv, D,
        float(d["scale"]), 0 if q.dtype == torch.bfloat16 else 1, None, num_splits,
        torch.cuda.current_stream().cuda_stream)
    assert st == skv.SKV_OK, skv.status_string(st)
    return out, lse


def test_static_scratch_decode_matches_workspace_decode():
    for call, (d, splits) in enumerate([(W.config2(4, 8192, seed=11), 0), (W.config3(1, 16384, seed=12), 0)]):
        out_s, lse_s = _static_call(d, splits)
        out_w, lse_w = skv.attn_splitkv_decode(d["q"].cuda(), d["k"].cuda(), d["v"].cuda(), d["scale"])
        torch.cuda.synchronize()
        vmax = float(d["v"].float().abs().max())
        assert torch.isfinite(out_s.float()).all() and torch.isfinite(lse_s).all(), f"call {call}"
        assert float((out_s.float() - out_w.float()).abs().max()) <= O_TOL * vmax, f"call {call}"
        assert float((lse_s - lse_w).abs().max()) <= LSE_TOL, f"call {call}"
    assert skv.device_error() == 0


def test_static_scratch_refuses_oversized_problems():
    # 256 splits of a [1, 64, 4, 256] decode need 256 * 256 rows * 1 KB of partials (> 8 MiB)
    st = skv.lib().attn_splitkv_decode_static(
        0x10000, 0x10000, 0x10000, 0x10000, None, 1, 64, 4, 4, 65536, 256, 0.0625, 0, None, 256,
        torch.cuda.current_stream().cuda_stream)
    assert st == skv.SKV_ERR_WORKSPACE_TOO_SMALL
