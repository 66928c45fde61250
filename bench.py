#!/usr/bin/env python3
"""Benchmark of the KDA chunk-prefill forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference] [--workload NAME]

A step is one whole forward (normalisation, intra-chunk work and the state
carry over all chunks) over the long-prefill workload: B=1, H=HV=64,
T=65536, K=V=128, fp32 initial state (seeded synthetic inputs, resident in
HBM before the timed region).  The inputs (6.5 GB) are far larger than the
126 MB L2, so no flush is needed between steps.  Prints one JSON line on
rank 0.

Under torchrun (N > 1) every rank runs its own independent batch of the same
shape (the (sequence, head) units shard without any exchange): weak scaling,
no data-path collective; the time is the max over ranks.

``--impl reference`` times the CPU oracle (the plain float64 recurrence) on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA chunk-prefill tokens·heads/s @T=64K,HV=64,K=V=128; % of roofline"
UNIT = "tokens·heads/s"
FLUSH_BELOW_BYTES = 512 << 20  # workloads under this many bytes get an L2 flush between timed steps
FLUSH_BYTES = 256 << 20
BYTES_PER_TOKEN_HEAD = 256 + 256 + 256 + 512 + 4 + 256  # q, k, v, g, beta, o (H == HV)


def algorithmic_bytes(case) -> int:
    """Bytes the forward must move at least once: inputs read, o written, state read and written."""
    group = case.HV // case.H
    th = case.tokens * case.HV
    per = 256 * 2 / group + 256 + 512 + 4 + 256
    state = case.N * case.HV * 128 * 128 * 4 * (2 if case.state != "none" else 1)
    return int(th * per + state)


def chunk_flops(case) -> int:
    """Dense chunk-form FLOPs (C=64 tiles): 180,224 per token-head."""
    return case.tokens * case.HV * 180224


def chunk_flops_triangular(C: int = 64, K: int = 128, V: int = 128) -> float:
    """FLOPs per token-head of the chunk form counting only the triangles the method needs (C=64, K=V=128):
    L (j < i) and Aqk (j <= i) over K; the unit-triangular inverse (sum over j < i of (i - j) multiply-adds) and
    its beta scaling; W and U with lower-triangular A; the carry's three dense products (W S, Qg S, Kg^T Vnew)
    and the triangular Aqk Vnew."""
    lower_strict, lower = C * (C - 1) // 2, C * (C + 1) // 2
    inverse = sum(i - j for i in range(C) for j in range(i)) * 2 + lower
    per_chunk = (lower_strict * K * 2 + lower * K * 2 + inverse + lower * K * 2 + lower * V * 2
                 + 3 * C * K * V * 2 + lower * V * 2)
    return per_chunk / C


def kernel_split(step, steps: int = 3):
    """Device time of each of this library's kernels per step, from a CUPTI trace (torch.profiler) of `steps`
    extra steps run after the timed region: {kernel name: ms per step}.  Kernels that overlap on two streams are
    each counted in full, so the sum can exceed the step time.  An "unavailable" note if the trace fails."""
    try:
        import torch
        from torch.profiler import ProfilerActivity, profile
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            for _ in range(steps):
                step()
            torch.cuda.synchronize()
        out = {}
        for ev in prof.key_averages():
            key = ev.key
            if "kda::" not in key:
                continue
            name = key[key.index("kda::"):]
            for stop in ("(", "<"):
                if stop in name:
                    name = name[:name.index(stop)] + ("<...>" if stop == "<" else "")
            us = getattr(ev, "device_time_total", None)
            if us is None:
                us = getattr(ev, "cuda_time_total", 0.0)
            out[name] = out.get(name, 0.0) + us / 1e3 / steps
        return {k: round(v, 4) for k, v in sorted(out.items(), key=lambda kv: -kv[1])} or {"unavailable": "no kernels"}
    except Exception as e:  # the bench line stays valid without the split
        return {"unavailable": str(e)[:120]}


def sustained(step, stream, seconds: float, device_index: int):
    """Back-to-back steps for about `seconds` (the power cap engages on long runs), timed by CUDA events on the
    launching stream, with the clocks sampled meanwhile."""
    import torch
    if seconds <= 0:
        return None
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    step()
    b.record(stream)
    torch.cuda.synchronize()
    n = max(20, int(seconds * 1e3 / max(a.elapsed_time(b), 1e-3)))
    with ClockSampler(device_index) as clk:
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(n):
            step()
        b.record(stream)
        torch.cuda.synchronize()
    return {"steps": n, "ms_per_step": a.elapsed_time(b) / n, "clocks": clk.summary()}


# device and host sources of the other paths (backward, decode step): edits there leave the forward unchanged
OTHER_PATH_SOURCES = {"kda_backward.cuh", "kda_backward_api.cuh", "kda_decode.cuh"}


def kernel_source_hash() -> str:
    """Hash of the sources the forward's kernels and launches are built from."""
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "kda_gated_delta_prefill_b200", "csrc", "*"))):
        if os.path.basename(f) in OTHER_PATH_SOURCES:
            continue
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def recorded_traffic(workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        rec = json.load(fh)
    ent = rec.get(workload)
    if not ent or ent.get("source_hash") != kernel_source_hash():
        return None
    return int(ent["dram_bytes_per_launch"])


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        fd, self.path = tempfile.mkstemp(prefix="kda_bench_clocks_", suffix=".csv")
        os.close(fd)

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as fh:
            lines = fh.readlines()
        try:
            os.unlink(self.path)
        except OSError:
            pass
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5], parts[6], parts[7], parts[8]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[2 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------------------------- ranks
# One process per GPU; every rank runs its own batch of the same shape (the units shard with no exchange).

def rank_case(case, rank: int):
    """The workload of one rank: the same shape, its own inputs (seed offset by 1000 per rank)."""
    import dataclasses
    return dataclasses.replace(case, seed=case.seed + 1000 * rank)


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """The slowest rank's time (every rank calls this, in the same order)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    tt = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def weak_throughput(units_per_step: float, world: int, total_ms: float, steps: int) -> float:
    """Whole-job units per second: every rank processed units_per_step per step in total_ms / steps."""
    return units_per_step * world / (total_ms / 1e3 / steps)


# ---------------------------------------------------------------------------------------------- oracle

def cpu_sample_inputs(case, heads: int, tokens: int):
    """The first `tokens` tokens of value heads [0, heads) of the workload, on the CPU."""
    import torch
    from kda_gated_delta_prefill_b200 import inputs as gen
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = gen.make_inputs(case, device=dev)
    group = case.HV // case.H
    out = {
        "q": x["q"][:, :tokens, : max(1, heads // group)].contiguous().cpu(),
        "k": x["k"][:, :tokens, : max(1, heads // group)].contiguous().cpu(),
        "v": x["v"][:, :tokens, :heads].contiguous().cpu(),
        "g": x["g"][:, :tokens, :heads].contiguous().cpu(),
        "beta": x["beta"][:, :tokens, :heads].contiguous().cpu(),
        "initial_state": None if x["initial_state"] is None else x["initial_state"][:, :heads].contiguous().cpu(),
        "cu_seqlens": None,
    }
    del x
    if dev == "cuda":
        torch.cuda.empty_cache()
    return out


def oracle_sample(case, target_s: float):
    """A bounded CPU sample of the workload for the oracle: the first `tokens` tokens of the first `heads`
    value heads (whole GQA groups), sized from a pilot run so that one oracle forward takes about target_s."""
    import oracle
    cores = oracle.max_threads()
    heads = min(case.HV, max(1, cores))
    if case.HV // case.H > 1:
        heads -= heads % (case.HV // case.H) or 0
        heads = max(heads, case.HV // case.H)
    pilot_tok = min(case.T, 256)
    xs = cpu_sample_inputs(case, heads, pilot_tok)
    t0 = time.perf_counter()
    oracle.forward(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], xs["initial_state"])
    per_tok = (time.perf_counter() - t0) / pilot_tok
    tokens = int(min(case.T, max(min(pilot_tok, 64), target_s / max(per_tok, 1e-9))))
    xs = cpu_sample_inputs(case, heads, tokens)
    return xs, tokens, heads, min(cores, heads)


def time_oracle(case, target_s: float = 15.0, steps: int = 1, warmup: int = 0):
    """Time the oracle as it stands on the host cores: `warmup` untimed and `steps` timed forwards of one
    bounded sample (about target_s seconds each)."""
    import oracle
    xs, tokens, heads, cores = oracle_sample(case, target_s)
    run = lambda: oracle.forward(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], xs["initial_state"])
    for _ in range(warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(steps):
        run()
    dt = time.perf_counter() - t0
    return {"value": tokens * heads * steps / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"first {tokens} tokens x value heads 0..{heads - 1} of {case.name}",
            "seconds": dt / steps}


# ---------------------------------------------------------------------------------------------- decode step

DECODE_METRIC = "KDA decode step rows·heads/s @B=1024,H=HV=12,K=V=128; % of roofline"
DECODE_UNIT = "rows·heads/s"


def decode_bytes(case) -> int:
    """Algorithmic bytes of one decode step: every active (row, value head) reads and writes its 128x128 bf16
    state and reads v, g, beta, writes o; q and k once per query/key head; the slot indices."""
    per_head = 2 * 128 * 128 * 2 + 128 * 2 + 128 * 4 + 4 + 128 * 2
    return case.B * case.HV * per_head + case.B * case.H * 2 * 128 * 2 + case.B * 4


def time_oracle_decode(case, target_s: float = 10.0, steps: int = 1, warmup: int = 0):
    """The oracle's decode step, as it stands, on the first rows of the workload (about target_s per step)."""
    import oracle
    from kda_gated_delta_prefill_b200 import inputs as gen
    x = gen.make_decode_inputs(case)
    pool = x["state"].float()
    run = lambda rows: oracle.decode_step(x["q"][:rows], x["k"][:rows], x["v"][:rows], x["g"][:rows],
                                          x["beta"][:rows], pool, x["state_indices"][:rows])
    t0 = time.perf_counter()
    run(8)
    per_row = (time.perf_counter() - t0) / 8
    rows = int(min(case.B, max(8, target_s / max(per_row, 1e-9))))
    for _ in range(warmup):
        run(rows)
    t0 = time.perf_counter()
    for _ in range(steps):
        run(rows)
    dt = (time.perf_counter() - t0) / steps
    return {"value": rows * case.HV / dt, "unit": DECODE_UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"first {rows} rows of {case.name}", "seconds": dt}


def bench_decode(args, case, world, rank, dev):
    import torch
    import torch.distributed as dist
    import dataclasses
    import kda_gated_delta_prefill_b200 as kda
    from kda_gated_delta_prefill_b200 import inputs as gen
    config = {"workload": case.name, "B": case.B, "H": case.H, "HV": case.HV, "K": 128, "V": 128,
              "state_slots": case.slots, "state_dtype": "bf16",
              "l2": "state pool (%.0f MB) larger than L2; no flush" % (case.slots * case.HV * 32768 / 1e6),
              "parallelism": f"independent replicas x{args.gpus} (weak)" if args.gpus > 1 else "single GPU"}
    if args.impl == "reference":
        if rank != 0:
            return 0
        per_step = min(10.0, max(0.05, 150.0 / (args.steps + args.warmup)))
        cb = time_oracle_decode(case, per_step, steps=args.steps, warmup=args.warmup)
        line = {"metric": DECODE_METRIC, "value": cb["value"], "unit": DECODE_UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": cb["seconds"] * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config, "impl": "reference",
                "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
                "e2e": {"value": cb["value"], "unit": DECODE_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    x = gen.make_decode_inputs(rank_case(case, rank), device=dev)
    o = torch.empty(case.B, case.HV, 128, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        kda.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state"], x["state_indices"], o=o,
                        stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    total_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    active = int((x["state_indices"] >= 0).sum().item())
    value = weak_throughput(active * case.HV, world, total_ms, args.steps)
    hbm_gbs, _, peak_kind = load_peaks()
    avg_s = statistics.mean(a.elapsed_time(b) for a, b in evs) / 1e3
    achieved = decode_bytes(case) / avg_s / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s", "frac": achieved / hbm_gbs,
                "traffic": None, "peak_kind": peak_kind, "algorithmic_bytes_per_launch": decode_bytes(case),
                "avg_launch_ms": avg_s * 1e3}
    e2e = None
    if not args.no_e2e:  # per step: the step's inputs from pinned host memory in, o out; the pool stays resident
        names = ("q", "k", "v", "g", "beta", "state_indices")
        xh = {k: x[k].cpu().pin_memory() for k in names}
        xd = {k: torch.empty_like(x[k]) for k in names}
        oh = torch.empty(case.B, case.HV, 128, dtype=torch.bfloat16).pin_memory()

        def hstep():
            for k in names:
                xd[k].copy_(xh[k], non_blocking=True)
            kda.decode_step(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], x["state"], xd["state_indices"], o=o,
                            stream=stream)
            oh.copy_(o, non_blocking=True)
        for _ in range(2):
            hstep()
        torch.cuda.synchronize()
        n_e = max(3, min(args.steps, 20))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_e):
            hstep()
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b), world, dev)
        e2e = {"value": weak_throughput(active * case.HV, world, e_ms, n_e), "unit": DECODE_UNIT,
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in xh.values()),
               "d2h_bytes_per_step": oh.numel() * 2, "steps": n_e}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = time_oracle_decode(case)
        cpu = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
    line = {"metric": DECODE_METRIC, "value": value, "unit": DECODE_UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk.summary(),
            "gpu_launches": args.steps, "impl": "native", "kernel_source": kernel_source_hash()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------------------------- backward

BWD_METRIC = "KDA chunk-prefill backward tokens·heads/s @T=64K,HV=64,K=V=128; % of HBM roofline"


def backward_bytes(case) -> int:
    """Bytes the backward must move at least once: q, k, v, g, beta, dout read; dq, dk, dv, dg, dbeta written;
    dht read; with an initial state, that state read and dh0 written."""
    group = case.HV // case.H
    th = case.tokens * case.HV
    per = (256 * 2 / group) * 2 + 256 * 2 + 512 * 2 + 4 * 2 + 256
    state = case.N * case.HV * 128 * 128 * 4 * (3 if case.state != "none" else 1)
    return int(th * per + state)


def time_oracle_backward(case, target_s: float = 15.0, steps: int = 1, warmup: int = 0):
    """The oracle's backward, as it stands, on a bounded sample: the first tokens of the first value heads."""
    import oracle
    from kda_gated_delta_prefill_b200 import inputs as gen
    cores = oracle.max_threads()
    heads = min(case.HV, max(1, cores))
    gr = gen.make_backward_grads(case)

    def sample(tokens):
        xs = cpu_sample_inputs(case, heads, tokens)
        do = gr["dout"][:, :tokens, :heads].float().numpy()
        dh = gr["dht"][:, :heads].numpy()
        return lambda: oracle.backward(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], xs["initial_state"], do, dh)

    pilot = min(case.T, 128)
    run = sample(pilot)
    t0 = time.perf_counter()
    run()
    per_tok = (time.perf_counter() - t0) / pilot
    tokens = int(min(case.T, max(64, target_s / max(per_tok, 1e-9))))
    run = sample(tokens)
    for _ in range(warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(steps):
        run()
    dt = (time.perf_counter() - t0) / steps
    return {"value": tokens * heads / dt, "unit": UNIT, "cores": min(cores, heads), "kind": "oracle",
            "sample": f"first {tokens} tokens x value heads 0..{heads - 1} of {case.name}", "seconds": dt}


def bench_backward(args, case, world, rank, dev):
    import dataclasses
    import torch
    import torch.distributed as dist
    import kda_gated_delta_prefill_b200 as kda
    from kda_gated_delta_prefill_b200 import inputs as gen
    name = "backward_" + case.name
    config = {"workload": name, "B": case.B, "T": case.T, "H": case.H, "HV": case.HV, "K": case.K, "V": case.V,
              "chunk": 64, "initial_state": case.state != "none", "dht": True,
              "l2": "inputs and workspace larger than L2; no flush",
              "parallelism": f"independent replicas x{args.gpus} (weak)" if args.gpus > 1 else "single GPU"}
    if args.impl == "reference":
        if rank != 0:
            return 0
        per_step = min(15.0, max(0.05, 150.0 / (args.steps + args.warmup)))
        cb = time_oracle_backward(case, per_step, steps=args.steps, warmup=args.warmup)
        line = {"metric": BWD_METRIC, "value": cb["value"], "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": cb["seconds"] * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "impl": "reference", "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
                "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    rcase = rank_case(case, rank)
    x = gen.make_inputs(rcase, device=dev)
    gr = gen.make_backward_grads(rcase, device=dev)
    B, T, H, HV, K, V, N = case.B, case.T, case.H, case.HV, case.K, case.V, case.N
    num_seqs = N if x["cu_seqlens"] is not None else 0
    ws = torch.empty(kda.backward_workspace_size(B, T, H, HV, K, V, num_seqs), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    saved = None
    if args.saved:  # the forward that keeps the blocks and chunk states, once, outside the timed region
        _, _, saved = kda.forward_save(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"],
                                       x["cu_seqlens"], saved=ws, stream=stream)
        config["saved_forward"] = True

    def step():
        return kda.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], gr["dout"], x["initial_state"], gr["dht"],
                            x["cu_seqlens"], workspace=None if saved is not None else ws, saved=saved,
                            stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    total_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    th = case.tokens * HV
    value = weak_throughput(th, world, total_ms, args.steps)
    hbm_gbs, _, peak_kind = load_peaks()
    avg_s = statistics.mean(a.elapsed_time(b) for a, b in evs) / 1e3
    alg = backward_bytes(case)
    roofline = {"bound": "hbm", "achieved": alg / avg_s / 1e9, "peak": hbm_gbs, "unit": "GB/s",
                "frac": alg / avg_s / 1e9 / hbm_gbs, "traffic": None, "peak_kind": peak_kind,
                "algorithmic_bytes_per_launch": alg, "avg_launch_ms": avg_s * 1e3,
                "scope": "the whole backward call (forward recomputation included)"}
    e2e = None
    if not args.no_e2e:  # inputs from pinned host memory in, every gradient out, each step
        names = ("q", "k", "v", "g", "beta", "initial_state")
        xh = {k: x[k].cpu().pin_memory() for k in names}
        gh = {k: gr[k].cpu().pin_memory() for k in ("dout", "dht")}
        xd = {k: torch.empty_like(x[k]) for k in names}
        gd = {k: torch.empty_like(gr[k]) for k in ("dout", "dht")}
        outs_h = None

        def hstep():
            nonlocal outs_h
            for k in names:
                xd[k].copy_(xh[k], non_blocking=True)
            for k in gd:
                gd[k].copy_(gh[k], non_blocking=True)
            outs = kda.backward(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], gd["dout"], xd["initial_state"],
                                gd["dht"], None, workspace=None if saved is not None else ws, saved=saved,
                                stream=stream)
            if outs_h is None:
                outs_h = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
            for a, b in zip(outs_h, outs):
                a.copy_(b, non_blocking=True)
        for _ in range(2):
            hstep()
        torch.cuda.synchronize()
        n_e = max(3, min(args.steps, 5))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_e):
            hstep()
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b), world, dev)
        e2e = {"value": weak_throughput(th, world, e_ms, n_e), "unit": UNIT,
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in list(xh.values()) + list(gh.values())),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in outs_h), "steps": n_e}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = time_oracle_backward(case)
        cpu = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
    launches = kda.backward_kernel_launches(B, T, H, HV, K, V, num_seqs)
    if saved is not None:  # the recomputation is skipped: reverse carry, chunk gradients, norms
        launches = 1 + (2 if case.tokens > 0 else 0)
    line = {"metric": BWD_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": config,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk.summary(),
            "gpu_launches": launches * args.steps, "impl": "native", "kernel_source": kernel_source_hash()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="long_T65536_H64_state",
                    help="a prefill workload name, backward_<prefill workload name> for the backward, or "
                         "decode_B1024_H12 for the decode step")
    ap.add_argument("--saved", action="store_true",
                    help="prefill workloads: time the forward that saves for the backward; backward workloads: time "
                         "the backward from a saved forward (forward_save once, untimed)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--sustain-s", type=float, default=3.0,
                    help="prefill workloads: seconds of back-to-back steps after the timed region for the sustained "
                         "(power-capped) figure; 0 skips it")
    ap.add_argument("--profile-T", type=int, default=0,
                    help="only run 3 forwards of B=1, H=HV=64, T=<value>, with state, and exit: the small case "
                         "the ncu captures under profiles/ use")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    import torch
    import torch.distributed as dist
    from kda_gated_delta_prefill_b200 import inputs as gen

    decode = args.workload.startswith("decode")
    backward = args.workload.startswith("backward_")
    wname = args.workload[len("backward_"):] if backward else args.workload
    case = gen.DECODE_SERVING if decode else {c.name: c for c in gen.WORKLOADS}[wname]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if decode and args.impl == "reference":
        return bench_decode(args, case, world, rank, None)
    if backward and args.impl == "reference":
        return bench_backward(args, case, world, rank, None)
    # workloads whose bytes fit a few times in the 126 MB L2 get an L2 flush between timed steps
    flush = not decode and algorithmic_bytes(case) < FLUSH_BELOW_BYTES
    config = None if decode else {"workload": case.name, "B": case.B, "T": case.T, "H": case.H, "HV": case.HV, "K": case.K,
              "V": case.V, "chunk": 64, "initial_state": case.state != "none",
              "l2": ("L2 flushed between steps (a %d MB write outside the per-step events)" % (FLUSH_BYTES >> 20))
              if flush else "inputs (%.1f GB) larger than L2; no flush" % (algorithmic_bytes(case) / 1e9),
              "parallelism": f"independent replicas x{args.gpus} (weak)" if args.gpus > 1 else "single GPU"}

    if args.impl == "reference":
        if rank != 0:
            return 0
        # each step a bounded sample, sized so that warm-up plus timed steps stay within about 2.5 minutes
        per_step = min(15.0, max(0.05, 150.0 / (args.steps + args.warmup)))
        cb = time_oracle(case, per_step, steps=args.steps, warmup=args.warmup)
        line = {"metric": METRIC, "value": cb["value"], "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": cb["seconds"] * 1e3, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config, "impl": "reference",
                "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
                "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import kda_gated_delta_prefill_b200 as kda
    if args.profile_T > 0:
        pc = gen.Case(f"profile_T{args.profile_T}", B=1, T=args.profile_T, H=64, HV=64, state="n01", seed=5)
        x = gen.make_inputs(pc, device="cuda")
        for _ in range(3):
            kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"])
        torch.cuda.synchronize()
        print(json.dumps({"profile_case": pc.name, "forwards": 3, "kernel_launches_per_forward":
                          kda.kernel_launches(pc.B, pc.T, pc.H, pc.HV)}), flush=True)
        return 0
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    kda.lib()
    if decode:
        return bench_decode(args, case, world, rank, dev)
    if backward:
        return bench_backward(args, case, world, rank, dev)

    # ---- inputs resident in HBM (rank-specific seed: independent batches) ----
    import dataclasses
    rcase = rank_case(case, rank)
    x = gen.make_inputs(rcase, device=dev)
    B, T, H, HV, K, V, N = case.B, case.T, case.H, case.HV, case.K, case.V, case.N
    o = torch.empty(B, T, HV, V, dtype=torch.bfloat16, device=dev)
    s = torch.empty(N, HV, K, V, dtype=torch.float32, device=dev)
    num_seqs = N if x["cu_seqlens"] is not None else 0
    # packed batches: the host copy of the boundaries lets the library overlap the carry (chunk windows)
    cu_host = gen.cu_seqlens_of(case.lengths) if case.lengths is not None else None
    if cu_host is not None:
        config["cu_seqlens_host"] = True
    stream = torch.cuda.current_stream(dev)
    if args.saved:  # the forward that also keeps what the backward needs
        ws = torch.empty(max(kda.backward_workspace_size(B, T, H, HV, K, V, num_seqs), 1), dtype=torch.uint8,
                         device=dev)
        config["saves_for_backward"] = True

        def step():
            kda.forward_save(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"], x["cu_seqlens"], o=o,
                             final_state=s, saved=ws, stream=stream)
    else:
        ws = torch.empty(max(kda.workspace_size(B, T, H, HV, K, V, num_seqs), 1), dtype=torch.uint8, device=dev)

        def step():
            kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"], x["cu_seqlens"], o=o,
                        final_state=s, workspace=ws, stream=stream, cu_seqlens_host=cu_host)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- timed region: K steps; per-launch CUDA events on the launching stream ----
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    scratch = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev) if flush else None
    with ClockSampler(torch.cuda.current_device()) as clk:
        barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            if flush:
                scratch.zero_()  # evict the previous step's data from L2
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
    launch_ms = [a.elapsed_time(b) for a, b in evs]
    # with flushes the steps are timed by their own events (the flushes excluded), else by the whole bracket
    total_ms = max_over_ranks(sum(launch_ms) if flush else t0.elapsed_time(t1), world, dev)
    ms_per_step = total_ms / args.steps
    th_per_step = case.tokens * HV
    value = weak_throughput(th_per_step, world, total_ms, args.steps)

    # ---- roofline of the dominant (only) compute kernel ----
    hbm_gbs, bf16_tf, peak_kind = load_peaks()
    alg = algorithmic_bytes(case)
    avg_launch_s = statistics.mean(launch_ms) / 1e3
    achieved = alg / avg_launch_s / 1e9
    tri = chunk_flops_triangular()
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s", "frac": achieved / hbm_gbs,
                "traffic": recorded_traffic(case.name), "peak_kind": peak_kind,
                "algorithmic_bytes_per_launch": alg, "avg_launch_ms": avg_launch_s * 1e3,
                "frac_nominal_8TBps": achieved / 8000.0,
                "flops_per_token_head": {"dense": 180224, "triangular": round(tri, 1)},
                "tensor_tflops": chunk_flops(case) / avg_launch_s / 1e12,
                "tensor_tflops_triangular": case.tokens * HV * tri / avg_launch_s / 1e12}
    step_ms = {"mean": statistics.mean(launch_ms), "median": statistics.median(launch_ms), "min": min(launch_ms),
               "max": max(launch_ms)}
    split = kernel_split(step)
    sus = sustained(step, stream, args.sustain_s, torch.cuda.current_device())

    # ---- end to end through the host-buffer entry point ----
    e2e = None
    if not args.no_e2e:
        del o, s
        xh = {k: (v.cpu().pin_memory() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
        del x
        torch.cuda.empty_cache()
        oh = torch.empty(B, T, HV, V, dtype=torch.bfloat16).pin_memory()
        sh = torch.empty(N, HV, K, V, dtype=torch.float32).pin_memory()
        has_cu = xh["cu_seqlens"] is not None
        st_n = kda.host_staging_size(B, T, H, HV, K, V, N if has_cu else 0, xh["initial_state"] is not None, has_cu)
        staging = torch.empty(st_n, dtype=torch.uint8, device=dev)

        def hstep():
            kda.forward_host(xh["q"], xh["k"], xh["v"], xh["g"], xh["beta"], xh["initial_state"], xh["cu_seqlens"],
                             o=oh, final_state=sh, staging=staging, stream=stream)
        for _ in range(2):
            hstep()
        torch.cuda.synchronize()
        e_steps = max(3, min(args.steps, 5))
        barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(e_steps):
            hstep()
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_ms = max_over_ranks(a.elapsed_time(b), world, dev)
        h2d = sum(t.numel() * t.element_size() for t in xh.values() if isinstance(t, torch.Tensor))
        d2h = oh.numel() * 2 + sh.numel() * 4
        e2e = {"value": weak_throughput(th_per_step, world, e_ms, e_steps), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": e_steps}
        del xh, staging

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = time_oracle(case)
        cpu = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}

    # intra-chunk and carry kernels per part of the sequence (+ chunk-offset, order and window-offset kernels for
    # packed batches)
    if cu_host is not None and not args.saved:
        launches_per_step = kda.varlen_kernel_launches(case.T, case.H, case.HV, cu_host, case.K, case.V)
    else:
        launches_per_step = kda.kernel_launches(case.B, case.T, case.H, case.HV, case.K, case.V,
                                                len(case.lengths) if case.lengths is not None else 0)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk.summary(),
            "gpu_launches": launches_per_step * args.steps, "impl": "native",
            "kernel_source": kernel_source_hash(), "step_ms": step_ms, "kernel_ms_per_step": split,
            "sustained": sus}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
