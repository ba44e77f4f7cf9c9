#!/usr/bin/env python
"""Benchmark of the modality-aware permutation sparse prefill path on B200.

One step = one attention layer through the whole hot path on one batch of synthetic input:
msa_estimate -> msa_permute -> msa_sparse_prefill -> msa_unpermute.

metric: sparse-prefill attention ms/layer + effective TFLOP/s (executed 128x128 block FLOPs,
4 * 128^3 per tile) at 128K and 1M tokens.  `value` is effective TFLOP/s of the whole step,
summed over ranks (by default each rank runs its own layer: weak scaling; with --shard kv-heads
the ranks split one layer by KV-head group: strong scaling; no collective on the data path in
either).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workload  # noqa: E402

METRIC = "sparse-prefill attention ms/layer + effective TFLOP/s at 128K and 1M tokens"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# NVIDIA's B200 dense bf16 tensor peak (half of the 2:4-sparse datasheet figure): context only,
# beside the measured peaks that the fractions are taken against
DATASHEET_BF16_DENSE_TFLOPS = 2250.0


def workloads():
    W = {
        "qwen2-7b-video-128k": workload.qwen2_7b_video_128k,
        "longvila-1m": workload.longvila_1m,
        "llama3-8b-text-32k": lambda: workload.llama3_8b_text(L=32768),
        "grid-1head-4k": lambda: workload.grid_single_head(),
        "qwen2-7b-video-64f": workload.qwen2_7b_video_literal,
        "mixed-image-text-64k": lambda: workload.mixed_image_text(L=65536),
    }
    for L in workload.SWEEP_LENGTHS:
        W[f"sweep-dense-L{L}"] = (lambda L=L: workload.sweep_layer(L, None))
        for b in workload.SWEEP_BUDGETS:
            W[f"sweep-b{int(round(b * 100))}-L{L}"] = (lambda L=L, b=b: workload.sweep_layer(L, b))
    return W


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kind_summary(p):
    from collections import Counter
    c = Counter(h.kind for h in p.heads)
    return " / ".join(f"{n} {k}" for k, n in c.items())


def dense_causal_flops(p):
    return 2 * p.d * p.L * (p.L + 1) * p.Hq


# ---------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid=None):
        self.uuid = uuid
        self.proc = None

    def __enter__(self):
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits", "-lms", "200"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10:
                continue
            try:
                sm.append(float(f[2]))
                mx.append(float(f[3]))
            except ValueError:
                continue
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                 f[6:10]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------
# CPU oracle on a bounded sample (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------------------
def sample_rows(L, n, seed):
    """n query rows stratified over [0, L): one seeded uniform row per stratum of L / n rows, so
    that the sample covers the whole causal range evenly (masked-attention time per row grows
    with the row's position)."""
    rng = np.random.default_rng(seed)
    n = max(1, min(n, L))
    edges = np.linspace(0, L, n + 1).astype(np.int64)
    return np.array([rng.integers(lo, hi) for lo, hi in zip(edges[:-1], edges[1:]) if hi > lo], np.int64)


def oracle_sample(p, Q, K, V, rows_per_head=4096, seed=0):
    """Times the oracle on one head of each kind: its full index estimation plus masked
    attention of `rows_per_head` stratified seeded rows, the attention time scaled by
    L / rows (an unbiased estimate of the whole head's attention time).  Returns per-kind
    seconds for one head and the sampled heads."""
    import oracle
    heads = {}
    for h, hd in enumerate(p.heads):
        heads.setdefault(hd.kind, h)
    per_kind = {}
    for kind, h in heads.items():
        t0 = time.perf_counter()
        idx = oracle.estimate_head(p, h, Q, K)
        t1 = time.perf_counter()
        rows = sample_rows(p.L, rows_per_head, seed * 1000 + h)
        oracle.attention_head(p, h, Q, K, V, idx, rows)
        t2 = time.perf_counter()
        per_kind[kind] = {"head": h, "est_s": t1 - t0, "attn_s": (t2 - t1) * p.L / len(rows), "idx": idx,
                          "rows": len(rows), "sampled_s": t2 - t0}
    return per_kind


def oracle_layer_seconds(p, per_kind):
    from collections import Counter
    n = Counter(h.kind for h in p.heads)
    return sum(n[k] * (v["est_s"] + v["attn_s"]) for k, v in per_kind.items())


def cores():
    return len(os.sched_getaffinity(0))


def job_totals(elapsed_ms: float, flops: float, world: int, device=None):
    """Max of the timed region over ranks and the sum of executed FLOPs over ranks (each rank
    runs its own layer or its own KV-head groups).  A collective only on these two scalars."""
    if world <= 1:
        return float(elapsed_ms), float(flops)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(elapsed_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    f = torch.tensor([float(flops)], dtype=torch.float64, device=device)
    dist.all_reduce(f, op=dist.ReduceOp.SUM)
    return float(t.item()), float(f.item())


# ---------------------------------------------------------------------------------------
INPUTS_NOTE = ("rope: N(0,1) rows plus a shared seeded direction of norm 15, rotated by the rotary "
               "position embedding (base 1e6) of their position")


def make_host_inputs(p, seed, inputs="iid"):
    Q, K, V = workload.make_inputs(p, seed=seed, inputs=inputs)
    return Q, K, V


_COMMENT_OR_STRING = re.compile(r'("(?:\\.|[^"\\])*")|//[^\n]*|/\*.*?\*/', re.S)


def code_only(text: str) -> str:
    """C/C++/CUDA source without comments and with whitespace runs collapsed."""
    return " ".join(_COMMENT_OR_STRING.sub(lambda m: m.group(1) or " ", text).split())


def attn_source_hash():
    """Identity of the attention kernel's code (comments and layout excluded): the recorded DRAM
    traffic is valid only for the code it was measured on."""
    h = hashlib.sha256()
    for f in ("attn.cu", "ptx.cuh", "msa_internal.h", "plan.cu"):  # plan.cu: work-item order
        with open(os.path.join(ROOT, "dynamic_sparse_attention_head_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name):
    """DRAM bytes per launch of the attention kernel from the committed ncu summary, if the
    kernel source still matches the one the counters were taken on."""
    path = os.path.join(ROOT, "profiles", "attn_dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    ent = d.get(workload_name)
    if not ent or ent.get("attn_source_hash") != attn_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


SECONDARY = {"qwen2-7b-video-128k": "longvila-1m"}  # the metric is quoted at 128K and at 1M


def per_kind_stats(p, tiles_per_head, pairs_per_head):
    """Executed density (executed block FLOPs / dense causal FLOPs) and mask density (allowed
    pairs / dense causal pairs) of each head kind of the layer."""
    dense_head = 2 * p.d * p.L * (p.L + 1)
    out = {}
    for kind in dict.fromkeys(h.kind for h in p.heads):
        hs = [h for h, hd in enumerate(p.heads) if hd.kind == kind]
        ex = sum(4 * 128 ** 3 * int(tiles_per_head[h]) for h in hs)
        us = sum(4 * p.d * int(pairs_per_head[h]) for h in hs)
        out[kind] = {"heads": len(hs), "executed_density": ex / (dense_head * len(hs)),
                     "mask_density": us / (dense_head * len(hs)),
                     "useful_over_executed": us / ex if ex else None}
    return out


def measure_layer(args, name, rank, world, local_rank, steps, warmup, with_e2e, with_cpu, with_dense):
    """Times `steps` steps of the named layer after `warmup` untimed ones (inputs resident) and
    returns the measurement as a dict (the JSON line's fields except the header)."""
    import dataclasses

    import torch
    import dynamic_sparse_attention_head_b200 as msa
    import torch.distributed as dist

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    p = workloads()[name]()
    if args.shard == "kv-heads":
        # one layer split by KV-head group: this rank's KV heads and their query heads, inputs
        # drawn as those heads of the whole layer (one seed for all ranks)
        p, qh, kvh = workload.shard_kv_heads(p, rank, world)
        Qh, Kh, Vh = workload.make_inputs(p, seed=0, inputs=args.inputs, q_heads=qh, kv_heads=kvh)
    else:
        Qh, Kh, Vh = make_host_inputs(p, seed=rank, inputs=args.inputs)

    def dev_copy(x):
        return torch.from_numpy(x).view(torch.bfloat16).to(dev)

    q, k, v = dev_copy(Qh), dev_copy(Kh), dev_copy(Vh)
    o = torch.empty_like(q)
    plan = msa.Plan(p)
    ws = plan.alloc_workspace(indexed=args.indexed)
    stream = torch.cuda.current_stream()

    n_steps = [0]

    def prefill(bq, bk, bv, bo, events=None):
        """permute -> sparse prefill -> unpermute, or the one index-based call (--indexed; the
        permute and unpermute stages are then empty and the key gathers run inside the call)."""
        if args.indexed:
            if events is not None:
                events[2].record(stream)
            plan.sparse_prefill_indexed(bq, bk, bv, ws, bo)
            if events is not None:
                events[3].record(stream)
                events[4].record(stream)
            return
        plan.permute(bq, bk, bv, ws)
        if events is not None:
            events[2].record(stream)
        plan.sparse_prefill(bq, bk, bv, ws)
        if events is not None:
            events[3].record(stream)
        plan.unpermute(ws, bo)
        if events is not None:
            events[4].record(stream)

    def step(events=None):
        if events is not None:
            events[0].record(stream)
        # --estimate-every K > 1: the index sets and tile lists left in the workspace by the last
        # estimate are reused by the next K - 1 layers of the same layout (off by default)
        if n_steps[0] % args.estimate_every == 0:
            plan.estimate(q, k, ws)
        n_steps[0] += 1
        if events is not None:
            events[1].record(stream)
        prefill(q, k, v, o, events)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    status = plan.device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")
    tiles, items = plan.tile_stats(ws)
    tiles_head = plan.tile_stats_heads(ws)
    exec_flops = msa.executed_flops(tiles)
    # allowed (query, key) pairs under the masks, counted on the device before the timed region
    pairs_head = plan.mask_pairs(ws)
    useful_flops = 4 * p.d * int(pairs_head.sum())

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(local_rank).uuid)
    except Exception:
        uuid = None
    n0 = msa.kernel_launches()
    with ClockSampler(uuid) as clk:
        start.record(stream)
        for s in range(steps):
            step(evs[s])
        end.record(stream)
        torch.cuda.synchronize()
    launches = msa.kernel_launches() - n0
    if world > 1:
        dist.barrier()
    total_ms = start.elapsed_time(end)
    stage = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(4)] for e in evs])  # ms
    # max over ranks of the timed region; sum of executed FLOPs over ranks
    total_ms, job_flops = job_totals(total_ms, exec_flops, world, dev)
    ms_step = total_ms / steps
    value = job_flops * steps / (total_ms * 1e-3) / 1e12

    # end to end through the public API with host buffers: every step copies its Q/K/V from
    # pinned host memory, runs the path and reads its O back to pinned host memory.  The copies
    # are pipelined across steps as a caller streaming layers would: two device buffer sets, the
    # H2D copy of step s+1 and the D2H copy of step s-1 run on copy streams while step s
    # computes; the timed region spans the first H2D copy to the last D2H copy.
    e2e = None
    if with_e2e:
        qp = torch.from_numpy(Qh).view(torch.bfloat16).pin_memory()
        kp = torch.from_numpy(Kh).view(torch.bfloat16).pin_memory()
        vp = torch.from_numpy(Vh).view(torch.bfloat16).pin_memory()
        ohost = [torch.empty(o.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        bufs = [(q, k, v, o), tuple(torch.empty_like(x) for x in (q, k, v, o))]
        h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event(enable_timing=False)  # noqa: E731
        in_ready, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

        def run_e2e(n):
            for s_ in range(n):
                b = s_ % 2
                bq, bk, bv, bo = bufs[b]
                with torch.cuda.stream(h2d):
                    if s_ >= 2:
                        h2d.wait_event(comp_done[b])  # step s-2 is done with this buffer set
                    bq.copy_(qp, non_blocking=True)
                    bk.copy_(kp, non_blocking=True)
                    bv.copy_(vp, non_blocking=True)
                    in_ready[b].record(h2d)
                stream.wait_event(in_ready[b])
                if s_ >= 2:
                    stream.wait_event(out_done[b])  # O of step s-2 has reached the host
                plan.estimate(bq, bk, ws)
                prefill(bq, bk, bv, bo)
                comp_done[b].record(stream)
                with torch.cuda.stream(d2h):
                    d2h.wait_event(comp_done[b])
                    ohost[b].copy_(bo, non_blocking=True)
                    out_done[b].record(d2h)

        run_e2e(2)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        h2d.wait_event(s0)
        run_e2e(steps)
        stream.wait_stream(d2h)
        s1.record(stream)
        torch.cuda.synchronize()
        e2e_ms, _ = job_totals(s0.elapsed_time(s1), 0.0, world, dev)
        bi = (Qh.nbytes + Kh.nbytes + Vh.nbytes)
        bo = int(np.prod(o.shape)) * 2
        e2e = {"value": job_flops * steps / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": e2e_ms / steps,
               "copies": "pipelined across steps (two device buffer sets, H2D and D2H streams)"}
        del bufs, qp, kp, vp, ohost

    pk, pk_src = peaks()
    attn_ms = float(stage[:, 2].mean())
    achieved = exec_flops / (attn_ms * 1e-3) / 1e12
    peak_sus = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_burst = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    traffic = recorded_traffic(name + ("+indexed" if args.indexed else ""))
    roofline = {"kernel": "msa_attn_kernel", "bound": "tensor", "achieved": achieved, "peak": peak_sus,
                "unit": "TFLOP/s", "frac": achieved / peak_sus, "traffic": traffic,
                "peak_source": f"{pk_src} bf16_tflops_sustained (kernel inside a long step)",
                "frac_of_burst_peak": achieved / peak_burst,
                "frac_of_datasheet_dense_peak": achieved / DATASHEET_BF16_DENSE_TFLOPS,
                "flops_per_launch": exec_flops, "ms_per_launch": attn_ms,
                **({"timed": "msa_sparse_prefill_indexed: the key gathers (a few % of its bytes, "
                             "under 0.2 % of its time) and the attention kernel"} if args.indexed else {})}

    # the same layer with every head dense, through the same kernel, timed once outside the
    # timed region: what the sparse index saves against dense attention on this hardware
    dense = None
    if with_dense and not args.indexed:
        pd_ = dataclasses.replace(p, heads=[workload.Head("dense")] * p.Hq)
        plan_d = msa.Plan(pd_)
        ws_d = plan_d.alloc_workspace()
        plan_d.estimate(q, k, ws_d)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for rep in range(2):  # one untimed pass, then the timed one
            plan_d.permute(q, k, v, ws_d)
            e0.record(stream)
            plan_d.sparse_prefill(q, k, v, ws_d)
            e1.record(stream)
            plan_d.unpermute(ws_d, o)
            torch.cuda.synchronize()
        assert plan_d.device_status(ws_d) == 0
        dense_ms = e0.elapsed_time(e1)
        dtiles, _ = plan_d.tile_stats(ws_d)
        # the pages' other sparsity statistic, on the dense layer's own rows: the share of the
        # dense attention weights that 95 % of each row's softmax mass needs (stratified rows)
        from dynamic_sparse_attention_head_b200.search import weight_share_stats
        ws95 = weight_share_stats(p, q, k, rows_per_head=16, recall=0.95)
        dense = {"weights_for_95pct_recall": {"mean_share": ws95["mean_share"], "per_kind": ws95["per_kind"],
                                              "rows_per_head": ws95["rows_per_head"]},
                 "attention_ms": dense_ms, "executed_flops": msa.executed_flops(dtiles),
                 "tflops": msa.executed_flops(dtiles) / (dense_ms * 1e-3) / 1e12,
                 "speedup_vs_dense_same_kernel": dense_ms / attn_ms,
                 "layer_speedup_vs_dense_attention": dense_ms / ms_step}
        del ws_d, plan_d
        torch.cuda.empty_cache()

    cpu = None
    if with_cpu and rank == 0 and world == 1:
        per_kind = oracle_sample(p, Qh, Kh, Vh, rows_per_head=args.cpu_rows)
        layer_s = oracle_layer_seconds(p, per_kind)
        rows = max(v_["rows"] for v_ in per_kind.values())
        cpu = {"value": exec_flops / layer_s / 1e12, "unit": "TFLOP/s", "cores": cores(), "kind": "oracle",
               "ms_per_layer": layer_s * 1e3, "extrapolated": True, "sampled_rows_per_head": rows,
               "sampled_seconds": sum(v_["sampled_s"] for v_ in per_kind.values()),
               "sample": (f"oracle on one head of each kind ({', '.join(per_kind)}): full index estimation + "
                          f"masked attention of {rows} stratified seeded rows, scaled to L rows; "
                          f"layer time = sum over heads of their kind's time (extrapolated); value = this "
                          f"layer's executed block FLOPs / that time")}

    sm = clk.summary()
    dcf = dense_causal_flops(p)
    return {
        "value": value, "ms_per_step": ms_step, "ms_per_layer": ms_step, "steps": steps, "warmup": warmup,
        "config": {"workload": name, "L": p.L, "Hq": p.Hq, "Hkv": p.Hkv, "d": p.d,
                   "heads": kind_summary(p),
                   "parallelism": (f"one layer split by KV-head group over {world} ranks ({p.Hkv} KV / {p.Hq} query "
                                   f"heads per rank; per-head statistics on this line are rank 0's)"
                                   if args.shard == "kv-heads" else f"independent layer per rank x{world}"),
                   **({"inputs": INPUTS_NOTE} if args.inputs == "rope" else {}),
                   "l2": "inputs larger than L2 (no flush)" if (Qh.nbytes > 126e6) else "inputs smaller than L2",
                   "seed": "rank", **({"estimate_every": args.estimate_every} if args.estimate_every > 1 else {}),
                   **({"path": "index-based (Q rows gathered in the attention kernel, O written at "
                               "original positions)"} if args.indexed else {})},
        "stages_ms": {"estimate": float(stage[:, 0].mean()), "permute": float(stage[:, 1].mean()),
                      "attention": attn_ms, "unpermute": float(stage[:, 3].mean())},
        "executed_tiles": tiles, "work_items": items, "executed_flops": exec_flops,
        "useful_flops": useful_flops, "dense_causal_flops": dcf,
        "mask_density": useful_flops / dcf, "executed_density": exec_flops / dcf,
        "useful_over_executed": useful_flops / exec_flops if exec_flops else None,
        "dense_flops_avoided": dcf - useful_flops,
        "per_kind": per_kind_stats(p, tiles_head, pairs_head),
        "dense_same_kernel": dense,
        "attn_tflops": achieved,
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(launches),
        "clocks": sm,
    }


def run_ours(args, rank, world, local_rank):
    import torch
    main = measure_layer(args, args.workload, rank, world, local_rank, args.steps, args.warmup,
                         with_e2e=not args.no_e2e, with_cpu=not args.no_cpu_baseline,
                         with_dense=not args.no_dense)
    torch.cuda.empty_cache()
    second = None
    sec_name = SECONDARY.get(args.workload) if not args.no_secondary else None
    if sec_name:
        second = measure_layer(args, sec_name, rank, world, local_rank, args.secondary_steps,
                               max(3, min(args.warmup, 3)), with_e2e=not args.no_e2e, with_cpu=False,
                               with_dense=not args.no_dense)
        second = {"metric": METRIC, "unit": "TFLOP/s", **second}
    if rank == 0:
        line = {"metric": METRIC, "value": main.pop("value"), "unit": "TFLOP/s", "n_gpus": world,
                "steps": main.pop("steps"), "warmup": main.pop("warmup"), "higher_is_better": True,
                "scaling": "strong" if args.shard == "kv-heads" else "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic", **main}
        if second is not None:
            line["secondary"] = second
        print(json.dumps(line), flush=True)


def run_sweep(args):
    """The budget sweep on the LLaMA-3-8B-shaped layer: one JSON line per (L, budget) with the
    per-stage times, estimation against attention.  A table, not the benchmark line.  The
    text-only layers' inputs depend on L alone, so they are generated once per length; layers
    of 512K tokens and more are timed over fewer repetitions (1 warm-up, 2 timed)."""
    import torch
    import dynamic_sparse_attention_head_b200 as msa
    lengths = [int(x) for x in args.sweep_lengths.split(",")]
    budgets = [None if x == "dense" else float(x) for x in args.sweep_budgets.split(",")]
    for L in lengths:
        warm, steps = (args.warmup, args.steps) if L <= 131072 else (1, 2)
        Qh, Kh, Vh = make_host_inputs(workload.sweep_layer(L, None), seed=0)
        q, k, v = (torch.from_numpy(x).view(torch.bfloat16).cuda() for x in (Qh, Kh, Vh))
        del Qh, Kh, Vh
        o = torch.empty_like(q)
        for b in budgets:
            p = workload.sweep_layer(L, b)
            plan = msa.Plan(p)
            ws = plan.alloc_workspace()
            st = torch.cuda.current_stream()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
            stages = []
            for i in range(warm + steps):
                ev[0].record(st)
                plan.estimate(q, k, ws)
                ev[1].record(st)
                plan.permute(q, k, v, ws)
                ev[2].record(st)
                plan.sparse_prefill(q, k, v, ws)
                ev[3].record(st)
                plan.unpermute(ws, o)
                ev[4].record(st)
                torch.cuda.synchronize()
                if i >= warm:
                    stages.append([ev[j].elapsed_time(ev[j + 1]) for j in range(4)])
            assert plan.device_status(ws) == 0
            tiles, _ = plan.tile_stats(ws)
            useful = 4 * p.d * int(plan.mask_pairs(ws).sum())
            st_ms = np.mean(np.array(stages), axis=0)
            flops = msa.executed_flops(tiles)
            print(json.dumps({"sweep": "llama3-8b-text", "L": L, "budget": b, "warmup": warm, "steps": steps,
                              "ms_per_layer": float(st_ms.sum()), "estimate_ms": float(st_ms[0]),
                              "permute_ms": float(st_ms[1]), "attention_ms": float(st_ms[2]),
                              "unpermute_ms": float(st_ms[3]),
                              "estimate_over_attention": float(st_ms[0] / st_ms[2]),
                              "executed_flops": flops, "dense_causal_flops": dense_causal_flops(p),
                              "density": flops / dense_causal_flops(p),
                              "mask_density": useful / dense_causal_flops(p),
                              "attn_tflops": flops / (st_ms[2] * 1e-3) / 1e12}), flush=True)
            del ws, plan
            torch.cuda.empty_cache()
        del q, k, v, o
        torch.cuda.empty_cache()


def run_reference(args, rank, world):
    """The oracle as the reference arm: bounded samples of the same workload on host cores."""
    if rank != 0:
        return
    p = workloads()[args.workload]()
    Qh, Kh, Vh = make_host_inputs(p, seed=0, inputs=args.inputs)
    flops = None
    # executed block FLOPs of the sampled heads' oracle indices, counted by the tile builder
    # (untimed, only to express the oracle's time in the metric's unit)
    per_kind = None
    times = []
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        per_kind = oracle_sample(p, Qh, Kh, Vh, rows_per_head=args.cpu_rows, seed=s)
        t = oracle_layer_seconds(p, per_kind)
        if s >= args.warmup:
            times.append(t)
        _ = time.perf_counter() - t0
    flops = executed_flops_for(p, per_kind)
    layer_s = float(np.mean(times))
    value = flops / layer_s / 1e12 if flops else None
    rows = max(v_["rows"] for v_ in per_kind.values())
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": layer_s * 1e3, "ms_per_layer": layer_s * 1e3,
            "extrapolated": True, "sampled_rows_per_head": rows,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "value_basis": ("the layer's executed block FLOPs (the unit of the metric, counted once, untimed, "
                            "from the oracle's own index sets) / the oracle's extrapolated layer time, so "
                            "that the ratio of the two arms' values is the ratio of their layer times"),
            "config": {"workload": args.workload, "L": p.L, "Hq": p.Hq, "Hkv": p.Hkv, "d": p.d,
                       "heads": kind_summary(p), **({"inputs": INPUTS_NOTE} if args.inputs == "rope" else {})},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores(), "kind": "oracle",
                             "extrapolated": True, "sampled_rows_per_head": rows,
                             "sample": (f"per step: oracle on one head of each kind, full index estimation + "
                                        f"masked attention of {rows} stratified seeded rows, scaled to L rows; "
                                        f"layer time summed over heads by kind (extrapolated)")},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def executed_flops_for(p, per_kind):
    """Executed block FLOPs of the whole layer when each head uses its kind's sampled oracle
    index set (tile builder run on the GPU, untimed).  None without a GPU."""
    try:
        import torch
        if not torch.cuda.is_available():
            return None
        import dynamic_sparse_attention_head_b200 as msa
    except Exception:
        return None
    idx = [per_kind[h.kind]["idx"] for h in p.heads]
    plan = msa.Plan(p)
    ws = plan.alloc_workspace()
    plan.set_indices(idx, ws)
    tiles, _ = plan.tile_stats(ws)
    return msa.executed_flops(tiles)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="qwen2-7b-video-128k", choices=sorted(workloads()))
    ap.add_argument("--inputs", choices=("iid", "rope"), default="iid",
                    help="rope: Q/K rows with a shared component under the rotary position embedding, so that "
                         "attention depends on the query-key offset (the index sets then cluster)")
    ap.add_argument("--shard", choices=("layers", "kv-heads"), default="layers",
                    help="layers: an independent layer per rank (weak scaling); kv-heads: one layer split by "
                         "KV-head group over the ranks (strong scaling, no exchange)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true",
                    help="skip timing the all-dense layer through the same kernel (outside the timed region)")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the second line of the metric (the 1M layer after the 128K one)")
    ap.add_argument("--secondary-steps", type=int, default=3)
    ap.add_argument("--cpu-rows", type=int, default=4096,
                    help="query rows per sampled head in the oracle's timed sample")
    ap.add_argument("--sweep", action="store_true", help="budget sweep table instead of the benchmark line")
    ap.add_argument("--estimate-every", type=int, default=1,
                    help="estimate indices on every K-th layer only and reuse them in between (index "
                         "amortisation across layers of one layout; 1, the default, is the benchmark)")
    ap.add_argument("--indexed", action="store_true",
                    help="index-based prefill (msa_sparse_prefill_indexed) in place of permute -> "
                         "sparse prefill -> unpermute")
    ap.add_argument("--sweep-lengths", default=",".join(str(x) for x in workload.SWEEP_LENGTHS))
    ap.add_argument("--sweep-budgets", default="0.02,0.05,0.1,0.25,dense")
    args = ap.parse_args()
    if args.sweep:
        run_sweep(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
