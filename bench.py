#!/usr/bin/env python
"""Benchmark of the attention-with-LSE hot path on B200.

One step = one pass over every operation of the path at the workloads' full
sizes, inputs resident in HBM:
  * varlen TND prefill, H=24, D=128, seqlens {512,1024,2048,4096}   (attn_fwd_lse)
  * ring-style chunked prefill, B=1, H=16, S_q=4096, S_k=16384, D=128: the
    partials of four KV chunks of 4096, each smoothed by its own mean, in one
    attn_fwd_lse_chunks launch, then merge_state of the four partials
  * split-KV decode D=128 (H_q=32, H_kv=8) and D=256 (H_q=16, H_kv=4),
    Lkv=32768, Lq in {1, 4}                                      (attn_splitkv_decode)
The headline value is prefill-dominated TFLOP/s (algorithmic FLOPs of the
step / device time); the decode calls are also timed alone as complete
CUDA-graph-captured operators (microseconds and HBM GB/s), as is merge_state.

L2 (126 MB) is flushed before every timed step and every timed replay, outside
the timed span: a 256 MB buffer is written, then another 256 MB is read, so the
timed kernels start with clean (not dirty) L2 lines.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs the same per-GPU work (independent
heads / sequences / batches: weak scaling, no data-path collective); rank 0
prints one JSON line with the max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fwd+LSE TFLOP/s (prefill); split-KV decode µs & HBM GB/s vs B200 peak"
D128 = 128
CFG4_SEQ = [512, 1024, 2048, 4096]
DECODE_SHAPES = [  # (name, Hq, Hkv, D, Lq, Lkv)
    ("decode_d128_lq1_lkv32768", 32, 8, 128, 1, 32768),
    ("decode_d128_lq4_lkv32768", 32, 8, 128, 4, 32768),
    ("decode_d256_lq1_lkv32768", 16, 4, 256, 1, 32768),
    ("decode_d256_lq4_lkv32768", 16, 4, 256, 4, 32768),
]


# The other decode shapes of the ExecuTorch split-K PR's A100 table (complete
# graph-captured operator; D, Lq, Lkv and that table's microseconds, other
# hardware, head counts not given there).  Timed here with workload 2's heads
# (D128: Hq32/Hkv8) and workload 3's (D256: Hq16/Hkv4) as context lines.
PAGES_A100_US = {("decode", 128, 1, 4096): 16.6, ("decode", 128, 1, 8192): 26.8, ("decode", 128, 1, 32768): 93.8,
                 ("decode", 128, 4, 4096): 18.9, ("decode", 128, 4, 32768): 103.5,
                 ("decode", 256, 1, 4096): 15.7, ("decode", 256, 1, 8192): 17.6, ("decode", 256, 1, 16384): 31.7,
                 ("decode", 256, 1, 32768): 59.4, ("decode", 256, 4, 16384): 44.9, ("decode", 256, 4, 32768): 69.7}


def attn_flops(rows_x_keys: int, D: int) -> int:
    """2*D FLOPs for q.k and 2*D for p*v per (query row, key) pair."""
    return 4 * D * rows_x_keys


FLOPS_CFG4 = attn_flops(24 * sum(s * s for s in CFG4_SEQ), D128)
FLOPS_CFG5 = attn_flops(16 * 4096 * 16384, D128)
FLOPS_CFG5_CHUNK = attn_flops(16 * 4096 * 4096, D128)


def decode_flops(Hq, D, Lq, Lkv):
    return attn_flops(Hq * Lq * Lkv, D)


def decode_kv_bytes(Hkv, D, Lkv):
    return 2 * Hkv * Lkv * D * 2


MERGE5_BYTES = 4 * 16 * 4096 * (128 * 2 + 4) + 16 * 4096 * (128 * 2 + 4)
# causal prefill of one workload-5 KV chunk (Sq = Sk = 4096, H = 16): the
# visible (row, key) pairs are sum_i (i + 1)
FLOPS_CAUSAL_CHUNK = attn_flops(16 * (4096 * 4097 // 2), D128)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.f = None

    def start(self):
        try:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.strip().split(", ") for r in self.f.read().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
                for n, val in zip(names, r[5:9]):
                    if val.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- our arm

def init_distributed(world: int, backend: str = "nccl", timeout_s: int = 120):
    """One process per GPU under torchrun: binds LOCAL_RANK's device (nccl)
    and joins the process group with a short timeout, so ranks that wait for
    a lost peer end with an error.  Returns torch.distributed, or None at N=1."""
    if world <= 1:
        return None
    import datetime
    import torch
    import torch.distributed as tdist
    if backend == "nccl":
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    tdist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return tdist


def max_over_ranks(ms: float, dist, device) -> float:
    """The step time the job reports: the slowest rank's (identity at N=1)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(flops_per_rank_step: float, world: int, ms: float) -> float:
    """Whole-job TFLOP/s: the units every rank processed / the max-over-ranks time."""
    return flops_per_rank_step * world / (ms * 1e-3) / 1e12


def run_ours(args, rank, world, dist):
    import torch
    import split_kv_merge_attn_b200 as skv
    import workloads as W

    dev = torch.device("cuda", torch.cuda.current_device())
    torch.manual_seed(0)
    peaks = load_peaks()

    # ---------------- inputs (seeded, generated on the host, copied once)
    c4 = W.config4(seed=rank)
    c5 = W.config5(seed=rank)
    host = {"c4": c4, "c5": c5}
    q4, k4, v4 = c4["q"].to(dev), c4["k"].to(dev), c4["v"].to(dev)
    cuq4, cuk4 = c4["cu_seqlens_q"].to(dev), c4["cu_seqlens_k"].to(dev)
    q5 = c5["q"].to(dev)
    b5 = c5["chunk_bounds"]
    k5, v5 = c5["k"].to(dev), c5["v"].to(dev)   # the whole key range; the chunks are bounds into it
    dec_in = []
    for (name, Hq, Hkv, D, Lq, Lkv) in DECODE_SHAPES:
        if D == 128:
            d = W.config2(Lq, Lkv, seed=rank)
        else:
            d = W.config3(Lq, Lkv, seed=rank)
        host[name] = d
        dec_in.append((name, d["q"].to(dev), d["k"].to(dev), d["v"].to(dev), d["scale"]))
    scale = D128 ** -0.5

    # ---------------- outputs and workspaces
    out4 = torch.empty_like(q4)
    lse4 = torch.empty(24, q4.shape[0], dtype=torch.float32, device=dev)
    ws4 = torch.empty(max(skv.attn_fwd_lse_workspace(4, 24, 24, q4.shape[0], 128, "bf16", "TND", 0), 1),
                      dtype=torch.uint8, device=dev)
    o5p = torch.empty((4,) + tuple(q5.shape), dtype=q5.dtype, device=dev)
    l5p = torch.empty(4, 1, 16, 4096, dtype=torch.float32, device=dev)
    ws5 = torch.empty(skv.attn_fwd_lse_chunks_workspace(1, 16, 16, 16384, 128, 4, "bf16", "HND", 1),
                      dtype=torch.uint8, device=dev)
    out5 = torch.empty_like(q5)
    lse5 = torch.empty(1, 16, 4096, dtype=torch.float32, device=dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    dec_buf = []
    for (name, q, k, v, sc) in dec_in:
        B, Hq, Lq, D = q.shape
        splits, _ = skv.attn_splitkv_plan(B, Hq, k.shape[1], Lq, k.shape[2], D, sms, 0)
        ws = torch.empty(max(skv.attn_splitkv_workspace(B, Hq, Lq, D, splits), 1), dtype=torch.uint8, device=dev)
        dec_buf.append((torch.empty_like(q), torch.empty(B, Hq, Lq, dtype=torch.float32, device=dev), ws, splits))
    flush_w = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        # write 256 MB (> 2x L2), then read another 256 MB so L2 is left holding
        # clean lines: dirty lines would otherwise be written back during the
        # next timed kernel
        flush_w.zero_()
        flush_r.sum()

    def call_cfg4():
        skv.attn_fwd_lse(q4, k4, v4, scale, layout="TND", cu_seqlens_q=cuq4, cu_seqlens_k=cuk4,
                         max_seqlen_q=4096, max_seqlen_k=4096, out=out4, lse=lse4, workspace=ws4)

    def call_cfg5():
        # the four chunks' partials (each smoothed by its own mean) in one launch, then their merge
        skv.attn_fwd_lse_chunks(q5, k5, v5, b5, scale, layout="HND", smooth_k=1, out=o5p, lse=l5p, workspace=ws5)
        skv.merge_state(o5p, l5p, "HND", out=out5, lse=lse5)

    def call_decode(i):
        name, q, k, v, sc = dec_in[i]
        o, l, ws, splits = dec_buf[i]
        skv.attn_splitkv_decode(q, k, v, sc, num_splits=splits, out=o, lse=l, workspace=ws)

    step_flops = FLOPS_CFG4 + FLOPS_CFG5 + sum(decode_flops(Hq, D, Lq, Lkv) for (_, Hq, _, D, Lq, Lkv) in DECODE_SHAPES)

    # events around each call inside the timed step
    parts = ["cfg4_varlen_prefill", "cfg5_chunked_prefill_merge"] + [s[0] for s in DECODE_SHAPES]

    def step(evs=None):
        if evs is not None:
            evs[0].record()
        call_cfg4()
        if evs is not None:
            evs[1].record()
        call_cfg5()
        if evs is not None:
            evs[2].record()
        for i in range(len(DECODE_SHAPES)):
            call_decode(i)
            if evs is not None:
                evs[3 + i].record()

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert skv.device_error() == 0

    # One step is replayed as a CUDA graph, captured once with timing events
    # between its parts ("external" events: they become event-record nodes of
    # the graph), so the device times are those of the kernels, free of the
    # host's launch overhead.
    n_ev = 3 + len(DECODE_SHAPES)
    cap_evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n_ev)]
    cap_stream = torch.cuda.Stream()
    cap_stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap_stream):
        step()
    torch.cuda.current_stream().wait_stream(cap_stream)
    torch.cuda.synchronize()
    step_graph = torch.cuda.CUDAGraph()
    launches_c0 = skv.launch_count()
    with torch.cuda.graph(step_graph):
        step(cap_evs)
    launches_per_step = skv.launch_count() - launches_c0
    torch.cuda.synchronize()

    # ---------------- timed region
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.5)
    step_ms, part_ms = [], {p: [] for p in parts}
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush_l2()
        step_graph.replay()
        torch.cuda.synchronize()   # the events of this replay are read before the next one records them
        step_ms.append(cap_evs[0].elapsed_time(cap_evs[n_ev - 1]))
        for j, p in enumerate(parts):
            part_ms[p].append(cap_evs[j].elapsed_time(cap_evs[j + 1]))
    torch.cuda.synchronize()
    barrier()
    launches = launches_per_step * args.steps   # kernels of the library in each replayed step
    clocks = sampler.stop() if sampler else None
    ms = max_over_ranks(sum(step_ms) / len(step_ms), dist, dev)
    value = job_value(step_flops, world, ms)
    assert skv.device_error() == 0
    del step_graph

    # ---------------- dominant kernel roofline: the varlen prefill launch
    pf_us = 1e3 * sum(part_ms["cfg4_varlen_prefill"]) / args.steps
    pf_tflops = FLOPS_CFG4 / (pf_us * 1e-6) / 1e12
    traffic = None
    tp = os.path.join(ROOT, "profiles", "prefill_kernel_traffic.json")
    if os.path.exists(tp):
        tj = json.load(open(tp))
        if tj.get("kernel_source_sha256") == kernel_source_hash():
            traffic = tj.get("dram_bytes_per_launch")
    roofline = {"bound": "tensor", "achieved": round(pf_tflops, 1), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(pf_tflops / peaks["bf16_tflops"], 4), "traffic": traffic,
                "kernel": "prefill_kernel<128,bf16> (varlen TND, H=24, seqlens 512..4096)",
                "peak_source": peaks["source"] + " bf16 burst (kernel timed as one launch)",
                "launch_us": round(pf_us, 1)}

    # ---------------- per-operation detail (graph-captured decode, merge)
    detail = {}
    if args.quick:  # the timed steps only (the command the profiler's launch list uses)
        if rank == 0:
            print(json.dumps({"quick": True, "ms_per_step": round(ms, 4), "value": round(value, 2),
                              "varlen_prefill_us": round(pf_us, 1), "gpu_launches": int(launches)}), flush=True)
        return
    for p in parts:
        detail[p] = {"us_in_step": round(1e3 * sum(part_ms[p]) / args.steps, 2)}
    detail["cfg5_chunked_prefill_merge"]["tflops"] = round(
        FLOPS_CFG5 / (detail["cfg5_chunked_prefill_merge"]["us_in_step"] * 1e-6) / 1e12, 1)
    detail["cfg4_varlen_prefill"]["tflops"] = round(pf_tflops, 1)

    def time_graph(fn, reps, per_replay=1, flush=True):
        """Mean of the middle 60% of `reps` graph replays of fn (captured once),
        divided by `per_replay` (the calls one replay makes); L2 flushed before
        each replay unless the replay's own inputs exceed it."""
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for _ in range(3):
                fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            if flush:
                flush_l2()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3 / per_replay)
        ts.sort()
        del g
        # mean of the middle 60%: event times come in ~2 us ticks here, so a
        # median snaps to a tick while the trimmed mean resolves below it
        k = len(ts) // 5
        return sum(ts[k:len(ts) - k]) / (len(ts) - 2 * k)

    # The fixed cost of one isolated replay (graph launch, one tiny kernel,
    # events): a floor under every "graph_us" below.
    tiny = torch.zeros(1, device=dev)
    floor_us = time_graph(lambda: tiny.add_(1.0), 50)
    detail["graph_floor_us"] = {"graph_us": round(floor_us, 2),
                                "what": "one graph replay of a one-element kernel, timed like the operators below"}
    N_B2B = 6

    def back_to_back(make_call, sets):
        """Per-call time of N_B2B calls replayed in one graph, call i on input
        set i: the sets together exceed L2, so each call reads its inputs from
        HBM, and the launch cost of one call overlaps the previous call."""
        calls = [make_call(x) for x in sets]

        def run():
            for c in calls:
                c()
        return time_graph(run, 20, per_replay=len(calls), flush=False)

    for i, (name, Hq, Hkv, D, Lq, Lkv) in enumerate(DECODE_SHAPES):
        us = time_graph(lambda i=i: call_decode(i), 50)
        gbs = decode_kv_bytes(Hkv, D, Lkv) / (us * 1e-6) / 1e9
        _, q, k, v, sc = dec_in[i]
        o, l, ws, splits = dec_buf[i]
        kv_sets = [(k, v)] + [(k.clone(), v.clone()) for _ in range(N_B2B - 1)]
        us_b = back_to_back(lambda kv: (lambda: skv.attn_splitkv_decode(q, kv[0], kv[1], sc, num_splits=splits, out=o,
                                                                        lse=l, workspace=ws)), kv_sets)
        del kv_sets
        gbs_b = decode_kv_bytes(Hkv, D, Lkv) / (us_b * 1e-6) / 1e9
        detail[name].update({"graph_us": round(us, 2), "kv_gbs": round(gbs, 1),
                             "b2b_us": round(us_b, 2), "b2b_kv_gbs": round(gbs_b, 1),
                             "hbm_frac": round(gbs_b / peaks["hbm_gbs"], 3), "splits": dec_buf[i][3],
                             "pages_a100_us": PAGES_A100_US.get(("decode", D, Lq, Lkv))})
        # the single-launch variant (in-kernel merge by the last CTA of each group)
        wsz = torch.zeros_like(ws)
        us_f = time_graph(lambda: skv.attn_splitkv_decode(q, k, v, sc, num_splits=splits, out=o, lse=l,
                                                          workspace=wsz, fused=True), 50)
        detail[name]["fused_graph_us"] = round(us_f, 2)
    # the remaining shapes of the pages' decode table, graph-timed alone
    timed = {(D, Lq, Lkv) for (_, _, _, D, Lq, Lkv) in DECODE_SHAPES}
    for (_, D, Lq, Lkv), a100 in PAGES_A100_US.items():
        if (D, Lq, Lkv) in timed:
            continue
        d = W.config2(Lq, Lkv, seed=rank) if D == 128 else W.config3(Lq, Lkv, seed=rank)
        q, k, v, sc = d["q"].to(dev), d["k"].to(dev), d["v"].to(dev), d["scale"]
        B, Hq, _, _ = q.shape
        Hkv = k.shape[1]
        splits, _ = skv.attn_splitkv_plan(B, Hq, Hkv, Lq, Lkv, D, sms, 0)
        ws = torch.empty(max(skv.attn_splitkv_workspace(B, Hq, Lq, D, splits), 1), dtype=torch.uint8, device=dev)
        o, l = torch.empty_like(q), torch.empty(B, Hq, Lq, dtype=torch.float32, device=dev)
        us = time_graph(lambda: skv.attn_splitkv_decode(q, k, v, sc, num_splits=splits, out=o, lse=l, workspace=ws), 50)
        gbs = decode_kv_bytes(Hkv, D, Lkv) / (us * 1e-6) / 1e9
        n_sets = max(N_B2B, -(-8 * 126 * 2 ** 20 // decode_kv_bytes(Hkv, D, Lkv)))  # >= 8 L2 sizes in all
        kv_sets = [(k, v)] + [(k.clone(), v.clone()) for _ in range(n_sets - 1)]
        us_b = back_to_back(lambda kv: (lambda: skv.attn_splitkv_decode(q, kv[0], kv[1], sc, num_splits=splits, out=o,
                                                                        lse=l, workspace=ws)), kv_sets)
        del kv_sets
        gbs_b = decode_kv_bytes(Hkv, D, Lkv) / (us_b * 1e-6) / 1e9
        detail[f"decode_d{D}_lq{Lq}_lkv{Lkv}"] = {"graph_us": round(us, 2), "kv_gbs": round(gbs, 1),
                                                  "b2b_us": round(us_b, 2), "b2b_kv_gbs": round(gbs_b, 1),
                                                  "hbm_frac": round(gbs_b / peaks["hbm_gbs"], 3), "splits": splits,
                                                  "pages_a100_us": a100}
        del q, k, v, o, l, ws
    # merge_state of workload 5 alone (HBM bound)
    us_m = time_graph(lambda: skv.merge_state(o5p, l5p, "HND", out=out5, lse=lse5), 50)
    m_sets = [(o5p, l5p)] + [(o5p.clone(), l5p.clone()) for _ in range(N_B2B - 1)]
    us_mb = back_to_back(lambda ol: (lambda: skv.merge_state(ol[0], ol[1], "HND", out=out5, lse=lse5)), m_sets)
    del m_sets
    detail["merge_state_cfg5"] = {"graph_us": round(us_m, 2),
                                  "gbs": round(MERGE5_BYTES / (us_m * 1e-6) / 1e9, 1),
                                  "b2b_us": round(us_mb, 2),
                                  "b2b_gbs": round(MERGE5_BYTES / (us_mb * 1e-6) / 1e9, 1),
                                  "hbm_frac": round(MERGE5_BYTES / (us_mb * 1e-6) / 1e9 / peaks["hbm_gbs"], 3)}
    # the same chunked workload as four separate attn_fwd_lse calls (context
    # for the one-launch chunks call of the step)
    k5c = [k5[:, :, a:e].contiguous() for a, e in zip(b5[:-1], b5[1:])]
    v5c = [v5[:, :, a:e].contiguous() for a, e in zip(b5[:-1], b5[1:])]
    ws5s = torch.empty(skv.attn_fwd_lse_workspace(1, 16, 16, 4096, 128, "bf16", "HND", 1), dtype=torch.uint8,
                       device=dev)

    def cfg5_four_calls():
        for c in range(4):
            skv.attn_fwd_lse(q5, k5c[c], v5c[c], scale, smooth_k=1, out=o5p[c], lse=l5p[c], workspace=ws5s)
        skv.merge_state(o5p, l5p, "HND", out=out5, lse=lse5)
    us_4 = time_graph(cfg5_four_calls, 20)
    us_1 = time_graph(call_cfg5, 20)
    detail["cfg5_chunked_prefill_merge"].update({
        "graph_us": round(us_1, 2), "graph_tflops": round(FLOPS_CFG5 / (us_1 * 1e-6) / 1e12, 1),
        "four_calls_graph_us": round(us_4, 2)})
    del k5c, v5c
    # workload 1 (B1 H4 S_q 64 S_k 1000 D128): latency bound, microseconds only;
    # also with K + 0.5 and smooth_k (the repro's third part)
    c1 = W.config1("rows")
    q1, k1, v1 = c1["q"].to(dev), c1["k"].to(dev), c1["v"].to(dev)
    k1s = (c1["k"].float() + 0.5).to(c1["k"].dtype).to(dev)
    o1 = torch.empty_like(q1)
    l1 = torch.empty(1, 4, 64, dtype=torch.float32, device=dev)
    ws1 = torch.empty(skv.attn_fwd_lse_workspace(1, 4, 4, 1000, 128, "bf16", "HND", 1), dtype=torch.uint8,
                      device=dev)
    us_1a = time_graph(lambda: skv.attn_fwd_lse(q1, k1, v1, c1["scale"], out=o1, lse=l1), 50)
    us_1b = time_graph(lambda: skv.attn_fwd_lse(q1, k1s, v1, c1["scale"], smooth_k=1, out=o1, lse=l1,
                                                workspace=ws1), 50)
    detail["cfg1_dense_h4_s64_sk1000"] = {"graph_us": round(us_1a, 2), "smooth_k_graph_us": round(us_1b, 2),
                                          "note": "latency bound (0.131 GFLOP): microseconds only, the replay floor "
                                                  "included"}
    del q1, k1, v1, k1s, o1, l1, ws1
    # causal variants: prefill of the first workload-5 chunk with its own queries
    # (Sq = Sk = 4096) and the Lq = 4 decode of workload 2 at Lkv 32768
    k5_0, v5_0 = k5[:, :, b5[0]:b5[1]].contiguous(), v5[:, :, b5[0]:b5[1]].contiguous()  # the first chunk
    oc = torch.empty_like(q5)
    lc = torch.empty(1, 16, 4096, dtype=torch.float32, device=dev)
    us_c = time_graph(lambda: skv.attn_fwd_lse(q5, k5_0, v5_0, scale, out=oc, lse=lc, causal=True), 20)
    detail["causal_prefill_h16_s4096"] = {"graph_us": round(us_c, 2),
                                          "tflops": round(FLOPS_CAUSAL_CHUNK / (us_c * 1e-6) / 1e12, 1)}
    # INT8 Q K'^T with smooth_k on the same chunk (mean, codes and prefill: the whole call)
    ws8 = torch.empty(skv.attn_fwd_lse_int8_workspace(1, 16, 16, 4096, 4096), dtype=torch.uint8, device=dev)
    us_8 = time_graph(lambda: skv.attn_fwd_lse_int8(q5, k5_0, v5_0, scale, out=oc, lse=lc, workspace=ws8), 20)
    detail["int8_smooth_prefill_h16_s4096"] = {"graph_us": round(us_8, 2),
                                               "tflops": round(FLOPS_CFG5 / 4 / (us_8 * 1e-6) / 1e12, 1)}
    # prefill at D = 256 (one 128-row query tile per CTA): H16/Hkv4 (workload 3's heads), Sq = Sk = 4096
    d256 = W.dense_case(1, 16, 4, 4096, 4096, 256, seed=rank)
    q256, k256, v256 = d256["q"].to(dev), d256["k"].to(dev), d256["v"].to(dev)
    o256 = torch.empty_like(q256)
    l256 = torch.empty(1, 16, 4096, dtype=torch.float32, device=dev)
    us_256 = time_graph(lambda: skv.attn_fwd_lse(q256, k256, v256, d256["scale"], out=o256, lse=l256), 20)
    detail["prefill_d256_h16_hkv4_s4096"] = {"graph_us": round(us_256, 2),
                                             "tflops": round(attn_flops(16 * 4096 * 4096, 256) / (us_256 * 1e-6) / 1e12, 1)}
    del q256, k256, v256, o256, l256
    i4 = [n for n, *_r in DECODE_SHAPES].index("decode_d128_lq4_lkv32768")
    _, qd, kd, vd, scd = dec_in[i4]
    od, ld, wsd, spd = dec_buf[i4]
    us_cd = time_graph(lambda: skv.attn_splitkv_decode(qd, kd, vd, scd, num_splits=spd, out=od, lse=ld, workspace=wsd,
                                                       causal=True), 50)
    detail["causal_decode_d128_lq4_lkv32768"] = {
        "graph_us": round(us_cd, 2), "kv_gbs": round(decode_kv_bytes(8, 128, 32768) / (us_cd * 1e-6) / 1e9, 1)}

    # ---------------- end to end through the public API with host buffers
    e2e = run_e2e(args, dev, host, skv, torch, step_flops, world, dist)

    # ---------------- oracle on the host cores (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(budget_s=args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded randn, workloads/)",
            "config": {"workload": "one pass over: varlen TND prefill (H24 D128 seqlens 512..4096) + chunked "
                                   "ring-style prefill with smooth_k (B1 H16 Sq4096 Sk16384 D128, 4 chunks in one launch) + "
                                   "merge_state + split-KV decode (D128 Hq32/Hkv8 and D256 Hq16/Hkv4, Lkv 32768, "
                                   "Lq 1 and 4)",
                       "algorithmic_gflop_per_step": round(step_flops / 1e9, 2),
                       "l2": "flushed (256 MB write + 256 MB read) before every timed step and replay",
                       "step_timing": "each step is one replay of a CUDA graph of all its calls, timed by events "
                                      "captured between the parts; gpu_launches = the library kernels of one "
                                      "captured step times the steps",
                       "detail_timing": "decode and merge_state alone: graph_us = one CUDA-graph replay (L2 flushed "
                                        "before each; mean of the middle 60% of 50; it includes the fixed cost in "
                                        "graph_floor_us); b2b_us = per-call time of back-to-back calls in one graph "
                                        "over input sets larger than L2 together; hbm_frac uses b2b_us",
                       "parallelism": f"replicas x{world} (independent work per GPU, no exchange)"},
            "roofline": roofline, "detail": detail, "e2e": e2e, "gpu_launches": int(launches),
            "clocks": clocks, "cpu_baseline": cpu, "peaks": peaks,
        }
        print(json.dumps(line), flush=True)


def run_e2e(args, dev, host, skv, torch, step_flops, world, dist):
    """Same step through the public API, with the step's inputs copied from
    pinned host memory and its outputs (O and LSE) read back every step."""
    c4, c5 = host["c4"], host["c5"]
    pin = lambda t: t.pin_memory()
    hq4, hk4, hv4 = pin(c4["q"]), pin(c4["k"]), pin(c4["v"])
    hcu = pin(c4["cu_seqlens_q"])
    hq5 = pin(c5["q"])
    b5 = c5["chunk_bounds"]
    hk5, hv5 = pin(c5["k"]), pin(c5["v"])
    hdec = [(pin(host[n]["q"]), pin(host[n]["k"]), pin(host[n]["v"]), host[n]["scale"]) for (n, *_r) in DECODE_SHAPES]
    sc = D128 ** -0.5
    h2d = sum(t.numel() * t.element_size() for t in [hq4, hk4, hv4, hcu, hcu, hq5, hk5, hv5])
    h2d += sum(q.numel() * q.element_size() + k.numel() * k.element_size() * 2 for q, k, v, s in hdec)
    # outputs read back: O (bf16) and LSE (fp32) of every call
    d2h_o = [torch.empty_like(hq4, device="cpu").pin_memory(), torch.empty(24, hq4.shape[0]).pin_memory(),
             torch.empty_like(hq5, device="cpu").pin_memory(), torch.empty(1, 16, 4096).pin_memory()]
    d2h_o += [torch.empty_like(q, device="cpu").pin_memory() for q, k, v, s in hdec]
    d2h_o += [torch.empty(q.shape[:3]).pin_memory() for q, k, v, s in hdec]
    d2h = sum(t.numel() * t.element_size() for t in d2h_o)

    def e2e_step():
        q4, k4, v4 = hq4.to(dev, non_blocking=True), hk4.to(dev, non_blocking=True), hv4.to(dev, non_blocking=True)
        cu = hcu.to(dev, non_blocking=True)
        o4, l4 = skv.attn_fwd_lse(q4, k4, v4, sc, layout="TND", cu_seqlens_q=cu, cu_seqlens_k=cu, max_seqlen_q=4096,
                                  max_seqlen_k=4096)
        q5 = hq5.to(dev, non_blocking=True)
        op5, lp5 = skv.attn_fwd_lse_chunks(q5, hk5.to(dev, non_blocking=True), hv5.to(dev, non_blocking=True), b5,
                                           sc, smooth_k=1)
        o5, l5 = skv.merge_state(op5, lp5)
        outs = [o4, l4, o5, l5]
        dec_o, dec_l = [], []
        for q, k, v, s in hdec:
            o, l = skv.attn_splitkv_decode(q.to(dev, non_blocking=True), k.to(dev, non_blocking=True),
                                           v.to(dev, non_blocking=True), s)
            dec_o.append(o)
            dec_l.append(l)
        for dst, src in zip(d2h_o, outs + dec_o + dec_l):
            dst.copy_(src, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    n = max(2, min(args.steps, 5))
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / n, dist, dev)
    return {"value": round(job_value(step_flops, world, ms), 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms, 3),
            "steps": n}


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ("prefill.cuh", "tcgen05.cuh", "skv_device.cuh", "skv_kernels.cu"):
        h.update(open(os.path.join(ROOT, "split_kv_merge_attn_b200", "csrc", f), "rb").read())
    return h.hexdigest()


# ---------------------------------------------------------------- oracle (CPU)

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(seconds_budget: float):
    """Runs the oracle on a bounded sample of the step's workload: whole query
    heads of the chunked workload (all 16384 keys, unsmoothed definition),
    then query rows of the longest varlen sequence, until the budget is used.
    Returns (flops, seconds, description)."""
    import numpy as np
    import oracle as O
    import workloads as W
    c5 = W.config5()
    q, k, v = (O.to_f64(c5[x])[0] for x in "qkv")
    flops, t0, heads = 0, time.perf_counter(), 0
    rows = 512
    while time.perf_counter() - t0 < seconds_budget and heads < 16:
        for r0 in range(0, 4096, rows):
            O.attention_rows(q[heads, r0:r0 + rows], k[heads], v[heads], c5["scale"])
            flops += attn_flops(rows * 16384, 128)
            if time.perf_counter() - t0 >= seconds_budget:
                break
        heads += 1
    dt = time.perf_counter() - t0
    return flops, dt, (f"oracle attention_rows (float64 numpy) on workload-5 query rows in blocks of {rows} "
                       f"x 16384 keys, D=128: {flops / 1e9:.1f} GFLOP in {dt:.1f} s")


def cpu_baseline(budget_s: float = 15.0):
    """The oracle on the host cores: on all the BLAS threads it gets, and on
    one core (BLAS limited to one thread, a shorter sample).  Each rate is also
    turned into the seconds a whole varlen (workload 4) or chunked (workload 5)
    problem would take at that rate: scaled from the sample, not measured."""
    flops, dt, desc = oracle_sample(budget_s)
    rate = flops / dt
    line = {"value": round(rate / 1e12, 5), "unit": "TFLOP/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": desc,
            "scaled_seconds": {"workload4_varlen": round(FLOPS_CFG4 / rate, 1),
                               "workload5_chunked": round(FLOPS_CFG5 / rate, 1), "how": "scaled"}}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            f1, dt1, desc1 = oracle_sample(max(2.0, budget_s / 2))
        r1 = f1 / dt1
        line["one_core"] = {"value": round(r1 / 1e12, 6), "unit": "TFLOP/s", "cores": 1, "sample": desc1,
                            "scaled_seconds": {"workload4_varlen": round(FLOPS_CFG4 / r1, 1),
                                               "workload5_chunked": round(FLOPS_CFG5 / r1, 1), "how": "scaled"}}
    except ImportError:
        line["one_core"] = None
    return line


def run_reference(args, rank, world):
    """The oracle as the reference arm: each step is a bounded sample of the
    same workload on the host cores."""
    if rank != 0:
        return
    # each step a bounded sample: the whole run stays near a minute
    per_step = max(0.2, min(args.cpu_seconds, 60.0 / max(args.steps + args.warmup, 1)))
    for _ in range(args.warmup):
        oracle_sample(per_step)
    fl, secs = 0, 0.0
    desc = ""
    for _ in range(args.steps):
        f, dt, desc = oracle_sample(per_step)
        fl += f
        secs += dt
    value = fl / secs / 1e12
    cores = _blas_threads()
    line = {"metric": METRIC, "value": round(value, 5), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * secs / args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded randn, workloads/)",
            "impl": "reference",
            "config": {"workload": "bounded sample of the same step: workload-5 query rows x all 16384 keys",
                       "parallelism": "host cores"},
            "cpu_baseline": {"value": round(value, 5), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(value, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- ring (context parallel)

RING_METRIC = "ring attention fwd+LSE TFLOP/s (context-parallel, KV shards passed rank to rank)"


def ring_job(dist, rank: int, world: int, device, steps: int, warmup: int, shard: int = 4096, H: int = 16,
             D: int = 128, seed: int = 0, dtype=None, attn=None, merge=None, exchange=None):
    """Context-parallel (ring) attention timed as a job: one sequence of
    shard * world tokens, rank r holding tokens [r*shard, (r+1)*shard) of q, k
    and v ([1, H, shard, D]).  Each step every rank computes the attention of
    its queries over all keys with split_kv_merge_attn_b200.ring (one partial
    per hop while the next key/value shard travels, then merge_state).  At
    world = 4 and shard = 4096 every rank does the work of the chunked
    workload (4096 queries over 16384 keys in four chunks).  Returns the
    job's numbers and this rank's last (O, LSE).  attn / merge / exchange
    replace the library's kernels and the point-to-point exchange (the CPU
    tests use that to run this function on gloo ranks)."""
    import torch
    from split_kv_merge_attn_b200.ring import ring_attn_fwd_lse
    dtype = dtype or torch.bfloat16
    g = torch.Generator().manual_seed(seed * 1000 + rank)   # this rank's shard of the sequence
    q = torch.randn(1, H, shard, D, generator=g).to(dtype).to(device)
    k = torch.randn(1, H, shard, D, generator=g).to(dtype).to(device)
    v = torch.randn(1, H, shard, D, generator=g).to(dtype).to(device)
    scale = D ** -0.5
    cuda = torch.device(device).type == "cuda"

    def step():
        return ring_attn_fwd_lse(q, k, v, scale, attn=attn, merge=merge, exchange=exchange)

    res = None
    for _ in range(warmup):
        res = step()
    if cuda:
        torch.cuda.synchronize()
    dist.barrier()
    if cuda:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
    t0 = time.perf_counter()
    for _ in range(steps):
        res = step()
    if cuda:
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
    else:
        ms = (time.perf_counter() - t0) * 1e3 / steps
    dist.barrier()
    ms = max_over_ranks(ms, dist if world > 1 else None, device)
    flops_rank = attn_flops(H * shard * shard * world, D)
    return {"ms": ms, "value": job_value(flops_rank, world, ms), "flops_per_rank": flops_rank,
            "result": res, "inputs": (q, k, v, scale)}


def run_ring(args, rank, world, dist):
    import torch
    import split_kv_merge_attn_b200 as skv
    dev = torch.device("cuda", torch.cuda.current_device())
    if dist is None:  # one rank: a trivial group so the ring code runs its one hop
        import datetime
        import torch.distributed as tdist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29511")
        tdist.init_process_group("gloo", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
        dist = tdist
    launches0 = skv.launch_count()
    r = ring_job(dist, rank, world, dev, args.steps, args.warmup)
    launches = skv.launch_count() - launches0
    assert skv.device_error() == 0
    if rank == 0:
        line = {"metric": RING_METRIC, "value": round(r["value"], 2), "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(r["ms"], 4),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded randn per rank)",
                "config": {"workload": f"ring attention over one sequence of {4096 * world} tokens, 4096 per rank, "
                                       "H16 D128, non-causal; per hop one attn_fwd_lse partial while the next "
                                       "K/V shard travels (torch.distributed P2P: NCCL on GPUs), then merge_state",
                           "parallelism": f"context-parallel ring x{world}",
                           "l2": "not flushed (each hop's shard is new data on the rank)"},
                "gpu_launches": int(launches)}
        print(json.dumps(line), flush=True)
    if world == 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------- main

def run_case(args):
    """Runs one operation of the step `--steps` times with nothing else around
    it (the small commands the ncu captures use)."""
    import torch
    import split_kv_merge_attn_b200 as skv
    import workloads as W
    dev = torch.device("cuda", 0)
    case = args.case
    if case == "prefill_varlen":
        c = W.config4()
        q, k, v = c["q"].to(dev), c["k"].to(dev), c["v"].to(dev)
        cu = c["cu_seqlens_q"].to(dev)
        fn = lambda: skv.attn_fwd_lse(q, k, v, c["scale"], layout="TND", cu_seqlens_q=cu, cu_seqlens_k=cu,
                                      max_seqlen_q=4096, max_seqlen_k=4096)
    elif case == "prefill_chunk":
        c = W.config5(Sk=4096, n_chunks=1)
        q, k, v = c["q"].to(dev), c["k"].to(dev), c["v"].to(dev)
        fn = lambda: skv.attn_fwd_lse(q, k, v, c["scale"], smooth_k=1)
    elif case == "prefill_chunks5":
        c = W.config5()
        q, k, v = c["q"].to(dev), c["k"].to(dev), c["v"].to(dev)
        fn = lambda: skv.attn_fwd_lse_chunks(q, k, v, c["chunk_bounds"], c["scale"], smooth_k=1)
    elif case == "prefill_d256":
        c = W.dense_case(1, 16, 4, 4096, 4096, 256, seed=0)
        q, k, v = c["q"].to(dev), c["k"].to(dev), c["v"].to(dev)
        fn = lambda: skv.attn_fwd_lse(q, k, v, c["scale"])
    elif case == "prefill_causal":
        c = W.config5(Sk=4096, n_chunks=1)
        q, k, v = c["q"].to(dev), c["k"].to(dev), c["v"].to(dev)
        fn = lambda: skv.attn_fwd_lse(q, k, v, c["scale"], causal=True)
    elif case == "prefill_int8":
        c = W.config5(Sk=4096, n_chunks=1)
        q, k, v = c["q"].to(dev), c["k"].to(dev), c["v"].to(dev)
        fn = lambda: skv.attn_fwd_lse_int8(q, k, v, c["scale"])
    elif case.startswith("decode_"):
        name = [s for s in DECODE_SHAPES if s[0] == case][0]
        _, Hq, Hkv, D, Lq, Lkv = name
        d = W.config2(Lq, Lkv) if D == 128 else W.config3(Lq, Lkv)
        q, k, v = d["q"].to(dev), d["k"].to(dev), d["v"].to(dev)
        fn = lambda: skv.attn_splitkv_decode(q, k, v, d["scale"])
    elif case == "merge5":
        g = torch.Generator().manual_seed(0)
        o = torch.randn(4, 1, 16, 4096, 128, generator=g).bfloat16().to(dev)
        l = (torch.randn(4, 1, 16, 4096, generator=g) * 10).to(dev)
        fn = lambda: skv.merge_state(o, l)
    else:
        raise SystemExit(f"unknown case {case}")
    for _ in range(args.steps):
        fn()
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    print(json.dumps({"case": case, "runs": args.steps, "ok": True}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", default=None, help="run one operation only (for profiler captures)")
    ap.add_argument("--ring", action="store_true", help="time context-parallel ring attention across the ranks")
    ap.add_argument("--quick", action="store_true", help="the timed steps only (no per-operation detail, e2e, CPU)")
    args = ap.parse_args()
    if args.case:
        run_case(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    dist = init_distributed(world, "nccl")
    try:
        if args.ring:
            run_ring(args, rank, world, dist)
            return
        run_ours(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
