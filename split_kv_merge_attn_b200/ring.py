"""Context-parallel (ring) attention across the ranks of a process group.

The multi-GPU consumer of the per-row LSE that the source pages motivate: ring
attention computes each query shard's attention over the key/value shards of
all ranks one hop at a time and combines the partial (O, LSE) pairs (SGLang PR
#33840, the motivation of returning the LSE: ring attention's per-hop
`merge_state`; ARK issue, the smooth_k paragraph: every KV chunk may carry its
own smoothing because the LSE is corrected).  One exchange step per hop: each
rank passes the key/value shard it holds to the next rank while it computes on
it, so the transfer of hop s+1 overlaps the attention of hop s.

Rank r of N holds shard r of one sequence split in rank order: queries
q [B, Hq, S_r, D] and keys/values k, v [B, Hkv, S_r, D] (HND).  At hop s it
holds the key/value shard of rank (r - s) mod N.  Every step of the attention
and of the merge runs in the library's kernels (`attn_fwd_lse`,
`attn_fwd_lse_causal`, `merge_state`); this module only schedules the hops and
the transfers (torch.distributed point-to-point operations: NCCL over NVLink on
GPUs).

Causal (bottom-right aligned inside each call, see `attn_fwd_lse_causal`):
with equal shards, rank r's queries are global positions [r S, (r+1) S), so the
shard of an earlier rank is seen in full, its own shard with the causal
diagonal, and later ranks' shards not at all (no partial is computed for them).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence


def p2p_ring_exchange(tensors: Sequence, group=None) -> Callable[[], List]:
    """Starts sending `tensors` to the next rank and receiving the previous
    rank's into new buffers; returns wait(), which completes the transfer and
    returns the received tensors.  The sent tensors must stay unmodified until
    wait() returns."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    if group is not None:
        nxt, prv = dist.get_global_rank(group, nxt), dist.get_global_rank(group, prv)
    recv = [torch.empty_like(t) for t in tensors]
    ops = [dist.P2POp(dist.isend, t, nxt, group) for t in tensors]
    ops += [dist.P2POp(dist.irecv, r, prv, group) for r in recv]
    reqs = dist.batch_isend_irecv(ops)

    def wait():
        for r in reqs:
            r.wait()
        return recv
    return wait


def ring_attn_fwd_lse(q, k, v, scale: Optional[float] = None, group=None, causal: bool = False,
                      smooth_k: int = 0, attn=None, merge=None, exchange=None):
    """Attention of this rank's query shard over every rank's key/value shard.

    Returns (O [B, Hq, S_r, D], LSE [B, Hq, S_r]) of this rank's queries, equal
    (up to the rounding of the 16-bit partials) to one attention call over the
    whole sequence.  `attn`, `merge` and `exchange` default to the library's
    kernels and `p2p_ring_exchange` (exchange(tensors) starts the transfer and
    returns a wait() that yields the received tensors); they can be replaced,
    e.g. to run the same schedule on CPU tensors.
    """
    import torch
    import torch.distributed as dist
    if attn is None or merge is None:
        from . import attn_fwd_lse, merge_state
        attn = attn or attn_fwd_lse
        merge = merge or merge_state
    if exchange is None:
        exchange = lambda ts: p2p_ring_exchange(ts, group)
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if scale is None:
        scale = q.shape[-1] ** -0.5
    o_parts, l_parts = [], []
    kv = [k, v]
    for s in range(world):
        src = (rank - s) % world
        pending = None
        if s + 1 < world:
            pending = exchange(kv)      # the next hop's shard travels while this one is used
        if not (causal and src > rank):
            o, l = attn(q, kv[0], kv[1], scale, causal=causal and src == rank, smooth_k=smooth_k)
            o_parts.append(o)
            l_parts.append(l)
        if pending is not None:
            kv = list(pending())
    return merge(torch.stack(o_parts), torch.stack(l_parts))
