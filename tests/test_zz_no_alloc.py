"""GPU test of attn_splitkv_decode_static, the decode entry point for callers
that cannot allocate device memory (code under an allocator that owns every
device byte, plugins handed only their inputs and outputs, hosts that forbid
allocation after start-up).  Its per-split scratch is a fixed 8 MiB device
array inside the library instead of a caller workspace.

Every call goes directly through the C ABI.  Each result is compared with the
FP64 oracle at the tolerances of the other parity tests, and with the regular
attn_splitkv_decode, on calls made back to back: a large problem first, then
others whose partials are fewer and smaller, one with a device kv_len shorter
than Lkv and an explicit split count, so a later call would show anything it
read from the array's stale contents.  The file name sorts last, so a run that
stops at the first failure has run every other test already; the test also
works alone in a fresh process, where its first call sets the array up.
"""

import pytest
import torch

import oracle as O
import split_kv_merge_attn_b200 as skv
import workloads as W
from tests._gpu_helpers import LSE_TOL, O_TOL, check_lse, check_o, nan_empty, vmax

pytestmark = pytest.mark.gpu


def _static_call(d, num_splits=0, kv_len=None):
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    B, Hq, Lq, D = q.shape
    _, Hkv, Lkv, _ = k.shape
    out = nan_empty(q.shape, q.dtype)
    lse = nan_empty((B, Hq, Lq), torch.float32)
    kl = None if kv_len is None else torch.tensor(kv_len, dtype=torch.int32, device="cuda")
    st = skv.lib().attn_splitkv_decode_static(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Lq, Lkv, D,
        float(d["scale"]), 0 if q.dtype == torch.bfloat16 else 1, None if kl is None else kl.data_ptr(), num_splits,
        torch.cuda.current_stream().cuda_stream)
    assert st == skv.SKV_OK, skv.status_string(st)
    return out, lse, kl


def test_static_scratch_decode_matches_oracle_and_workspace_decode():
    calls = [
        (W.config2(4, 8192, seed=11), 0, None),            # 16 rows per kv head, automatic splits
        (W.config3(1, 16384, seed=12), 0, None),           # D = 256
        (W.config2(1, 4096, seed=13), 5, [2500]),          # explicit splits, device kv_len < Lkv
    ]
    for call, (d, splits, kv_len) in enumerate(calls):
        out_s, lse_s, kl = _static_call(d, splits, kv_len)
        out_w, lse_w = skv.attn_splitkv_decode(d["q"].cuda(), d["k"].cuda(), d["v"].cuda(), d["scale"], kv_len=kl,
                                               num_splits=splits)
        torch.cuda.synchronize()
        o_ref, l_ref = O.decode(d["q"], d["k"], d["v"], d["scale"], kv_len=kv_len)
        check_o(out_s, o_ref, vmax(d["v"]), what=f"call {call} O vs oracle")
        check_lse(lse_s, l_ref, what=f"call {call} LSE vs oracle")
        vm = vmax(d["v"])
        assert float((out_s.float() - out_w.float()).abs().max()) <= O_TOL * vm, f"call {call} O vs workspace decode"
        assert float((lse_s - lse_w).abs().max()) <= LSE_TOL, f"call {call} LSE vs workspace decode"
    assert skv.device_error() == 0


def test_static_scratch_refuses_oversized_problems():
    # 256 splits of a [1, 64, 4, 256] decode need 256 * 256 rows * 1 KB of
    # partials (> 8 MiB).  Null tensors: the size refusal comes before the
    # pointer checks, and if it ever did not, the null pointers are refused
    # too, so nothing is launched either way.
    st = skv.lib().attn_splitkv_decode_static(
        None, None, None, None, None, 1, 64, 4, 4, 65536, 256, 0.0625, 0, None, 256,
        torch.cuda.current_stream().cuda_stream)
    assert st == skv.SKV_ERR_WORKSPACE_TOO_SMALL
    # an unsupported head dimension is reported as such, not as a size problem
    st = skv.lib().attn_splitkv_decode_static(
        None, None, None, None, None, 1, 64, 4, 4, 65536, 96, 0.1, 0, None, 256,
        torch.cuda.current_stream().cuda_stream)
    assert st == skv.SKV_ERR_UNSUPPORTED
