"""The ring (context-parallel) schedule of split_kv_merge_attn_b200.ring on CPU:
world-size 2 and 3 `gloo` process groups exchange float64 key/value shards
with the module's point-to-point ring exchange, and the per-hop attention and
the final merge are the FP64 oracle's.  Each rank's result must equal the
oracle's attention of its query rows over the whole sequence, causal or not."""
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, causal, q_res):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    import oracle as O
    from split_kv_merge_attn_b200.ring import ring_attn_fwd_lse

    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        g = torch.Generator().manual_seed(7)
        B, Hq, Hkv, S, D = 1, 4, 2, 6, 8        # S rows per rank
        q = torch.randn(B, Hq, S * world, D, generator=g, dtype=torch.float64)
        k = torch.randn(B, Hkv, S * world, D, generator=g, dtype=torch.float64)
        v = torch.randn(B, Hkv, S * world, D, generator=g, dtype=torch.float64)
        sl = slice(rank * S, (rank + 1) * S)
        calls = []

        def attn(qs, ks, vs, scale, causal=False, smooth_k=0):
            calls.append(bool(causal))
            o, l = O.dense(qs, ks, vs, scale, causal=causal)
            return torch.from_numpy(o), torch.from_numpy(l)

        def merge(op, lp):
            o, l = O.merge(op.numpy(), lp.numpy())
            return torch.from_numpy(o), torch.from_numpy(l)

        o, l = ring_attn_fwd_lse(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous(),
                                 0.35, causal=causal, attn=attn, merge=merge)
        o_ref, l_ref = O.dense(q, k, v, 0.35, causal=causal)
        err_o = float(np.abs(o.numpy() - o_ref[:, :, sl]).max())
        l_ok = np.allclose(l.numpy(), l_ref[:, :, sl], rtol=0, atol=1e-12)
        q_res.put((rank, err_o, bool(l_ok), calls))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_schedule_matches_full_attention(world, causal):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_rank_main, args=(r, world, port, causal, q)) for r in range(world)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=240)
    codes = [p.exitcode for p in ps]
    for p in ps:
        if p.is_alive():
            p.kill()
    assert codes == [0] * world, codes
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, err_o, l_ok, calls in res:
        assert err_o < 1e-12 and l_ok, (rank, err_o)
        if causal:
            # earlier ranks' shards in full, its own with the diagonal, later ones skipped
            assert len(calls) == rank + 1 and calls[0] is True and not any(calls[1:])
        else:
            assert calls == [False] * world
