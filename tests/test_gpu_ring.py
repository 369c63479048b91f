"""Ring attention with the library's kernels on the GPU: two ranks (processes)
share the one GPU of the test machine and pass their key/value shards through
a `gloo` group (staged through host memory, since gloo moves CPU tensors; on a
multi-GPU node NCCL moves them directly).  No kernel waits for another rank:
the ranks only meet in the host-side exchange.  Each rank's (O, LSE) is checked
against the FP64 oracle's attention of its rows over the whole sequence."""
import multiprocessing as mp
import os
import socket
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, causal, smooth_k, q_res):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime
    import numpy as np
    import torch
    import torch.distributed as dist
    import oracle as O
    import split_kv_merge_attn_b200 as skv
    import workloads as W
    from split_kv_merge_attn_b200.ring import p2p_ring_exchange, ring_attn_fwd_lse

    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    try:
        S = 640                                  # rows per rank: several tiles and a ragged one
        d = W.dense_case(1, 8, 2, S * world, S * world, 128, seed=21, q_mult=2.0, k_offset=0.5 if smooth_k else 0.0)
        sl = slice(rank * S, (rank + 1) * S)
        q, k, v = (d[x][:, :, sl].contiguous().cuda() for x in ("q", "k", "v"))

        def exchange(ts):
            wait = p2p_ring_exchange([t.cpu() for t in ts])   # gloo moves host tensors
            return lambda: [r.cuda() for r in wait()]

        o, l = ring_attn_fwd_lse(q, k, v, d["scale"], causal=causal, smooth_k=smooth_k, exchange=exchange)
        torch.cuda.synchronize()
        err = skv.device_error()
        o_ref, l_ref = O.dense(d["q"], d["k"], d["v"], d["scale"], causal=causal)
        vmax = float(d["v"].float().abs().max())
        e_o = float(np.abs(o.double().cpu().numpy() - o_ref[:, :, sl]).max())
        lr = l_ref[:, :, sl]
        lg = l.double().cpu().numpy()
        e_l = float(np.abs(lg - lr).max())
        q_res.put((rank, err, e_o / vmax, e_l, bool(np.isfinite(lg).all())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("causal,smooth_k", [(False, 0), (True, 0), (False, 1)])
def test_two_rank_ring_on_one_gpu(causal, smooth_k):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_rank_main, args=(r, world, port, causal, smooth_k, q)) for r in range(world)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=300)
    codes = [p.exitcode for p in ps]
    for p in ps:
        if p.is_alive():
            p.kill()
    assert codes == [0] * world, codes
    for rank, err, e_o, e_l, finite in sorted(q.get(timeout=5) for _ in range(world)):
        assert err == 0 and finite, rank
        assert e_o <= 2e-2, (rank, e_o)
        assert e_l <= 1e-3, (rank, e_l)
