"""bench.py --ring on CPU: two `gloo` ranks run the bench's ring job end to
end (shard inputs, warm-up, timed steps, max-over-ranks time, job value) with
the ring module's point-to-point exchange, while the per-hop attention and the
final merge are the FP64 oracle's (the exchange hook the ring module takes).
Each rank's result must equal the oracle's attention of its query rows over the
whole sequence, and both ranks must report the same (slowest-rank) time."""
import multiprocessing as mp
import os
import socket
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    import bench
    import oracle as O

    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        def attn(qs, ks, vs, scale, causal=False, smooth_k=0):
            o, l = O.dense(qs, ks, vs, scale)
            return torch.from_numpy(o), torch.from_numpy(l)

        def merge(op, lp):
            o, l = O.merge(op.numpy(), lp.numpy())
            return torch.from_numpy(o), torch.from_numpy(l)

        shard, H, D = 5, 2, 8
        r = bench.ring_job(dist, rank, world, "cpu", steps=2, warmup=1, shard=shard, H=H, D=D, seed=3,
                           dtype=torch.float64, attn=attn, merge=merge)
        # the whole sequence, rebuilt from every rank's seeded shard
        parts = []
        for rr in range(world):
            g = torch.Generator().manual_seed(3 * 1000 + rr)
            parts.append([torch.randn(1, H, shard, D, generator=g, dtype=torch.float32).double() for _ in range(3)])
        q, k, v = (torch.cat([p[i] for p in parts], dim=2) for i in range(3))
        o_ref, l_ref = O.dense(q, k, v, D ** -0.5)
        sl = slice(rank * shard, (rank + 1) * shard)
        o, l = r["result"]
        err_o = float(np.abs(o.numpy() - o_ref[:, :, sl]).max())
        err_l = float(np.abs(l.numpy() - l_ref[:, :, sl]).max())
        out.put((rank, err_o, err_l, r["ms"], r["value"], r["flops_per_rank"]))
    finally:
        dist.destroy_process_group()


def test_bench_ring_job_on_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
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
    for rank, err_o, err_l, ms, value, flops in res:
        assert err_o < 1e-10 and err_l < 1e-10, (rank, err_o, err_l)
        # every rank does 4*D*H*shard*(shard*world) FLOPs
        assert flops == 4 * 8 * 2 * 5 * 5 * world
    assert res[0][3] == res[1][3], "both ranks report the slowest rank's time"
    assert abs(res[0][4] - res[0][5] * world / (res[0][3] * 1e-3) / 1e12) < 1e-9
