#!/usr/bin/env python
"""Benchmark of the block-sparse landmark attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-secondary] [--detail FILE]

One step of the headline workload (long_prefill_256k: B1, Hq 32, Hkv 8,
d 128, N 262144, block 128, top-16 + sink + local, bf16, causal) is one pass
of the prefill path through the C ABI: landmarks -> selection -> gated
block-sparse prefill.  ``value`` = prefill tokens/s over all ranks (each rank
runs its own seeded sequence: weak scaling, no collective on the data path).

At N = 1 the same JSON line ends with ``secondary``: a compact summary (value,
step time, per-kernel times and roofline fractions) of the other workloads --
the decode at 128K context (gated_decode_128k: 64 sequences, the metric's own
context length), the hierarchical decode at 1M, the 32K prefills (gated,
hierarchical, per-query-head lists), the ragged and per-query-head decodes,
the backward and the flat clustered index.  ``--detail FILE`` writes their
full records.

Timing: CUDA events on the launching stream around each step and each C call,
W warm-up steps, K timed steps bracketed by barrier + synchronize, L2 flushed
before every timed step (a 256 MiB write, then a 256 MiB read, so that no
input and no dirty line is left in L2), max over ranks.  ``--impl
reference`` times the CPU oracle (a deliberately slow, plain C reference) on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse prefill tokens/s and decode queries/s at 128K ctx; % of TC/HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------
# ranks
# ----------------------------------------------------------------------------

class Ranks:
    def __init__(self, backend="nccl"):
        import torch.distributed as dist
        self.dist = dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        if self.world > 1 and not dist.is_initialized():
            import datetime
            if backend == "nccl":
                torch.cuda.set_device(self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))

    @classmethod
    def single(cls):
        r = cls.__new__(cls)
        r.world, r.rank, r.local, r.backend, r.dist = 1, 0, 0, "none", None
        return r

    def barrier(self):
        if self.world > 1:
            if self.backend == "nccl":
                self.dist.barrier(device_ids=[self.local])
            else:
                self.dist.barrier()

    def max(self, x: float) -> float:
        if self.world == 1:
            return float(x)
        dev = torch.device("cuda", self.local) if self.backend == "nccl" else torch.device("cpu")
        t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def sum(self, x: float) -> float:
        if self.world == 1:
            return float(x)
        dev = torch.device("cuda", self.local) if self.backend == "nccl" else torch.device("cpu")
        t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.world > 1 and self.dist.is_initialized():
            self.dist.destroy_process_group()


def aggregate(ranks: Ranks, elapsed_ms: float, units: float) -> tuple[float, float]:
    """Whole-job throughput: units of all ranks / the slowest rank's time.
    Returns (value per second, max elapsed ms)."""
    t = ranks.max(elapsed_ms)
    u = ranks.sum(units)
    return (u / (t / 1e3) if t > 0 else 0.0), t


# ----------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            self.uuid = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            sel = ["-i", ("GPU-" + self.uuid) if self.uuid and not self.uuid.startswith("GPU-") else self.uuid] \
                if self.uuid else []
            self.proc = subprocess.Popen(["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:8], parts[3]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2]) if v.lower() == "active"})
        loaded = [r[0] for r in rows if r[3] not in ("0", "[N/A]")] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def traffic_for(kernel: str):
    """Per-launch DRAM bytes from the committed ncu summary, if its kernel
    source is unchanged since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel)
    if not d:
        return None
    # the counters stand only while every source file of the kernel is unchanged
    if "sources" not in d or "sources_sha256" not in d:
        return None
    h = hashlib.sha256()
    for rel in d["sources"]:
        src = os.path.join(ROOT, rel)
        if not os.path.exists(src):
            return None
        h.update(open(src, "rb").read())
    if h.hexdigest() != d["sources_sha256"]:
        return None
    return d["dram_bytes_per_launch"]


class Timer:
    """Per-name CUDA-event timing of calls on the current stream."""

    def __init__(self):
        self.ev = {}

    def __call__(self, name, fn):
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        out = fn()
        e.record()
        self.ev.setdefault(name, []).append((s, e))
        return out

    def ms(self):
        return {k: statistics.fmean(s.elapsed_time(e) for s, e in v) for k, v in self.ev.items()}


def flush_l2(buf):
    """Writes a buffer larger than L2, then reads a second one: every step
    starts with none of its inputs in L2 and no dirty line left from the
    flush (otherwise the first kernel of the step pays the flush's own
    write-back to DRAM)."""
    w, r = buf
    w.fill_(1)
    r.sum(dtype=torch.int32)


def flush_buffers(device="cuda"):
    return (torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device),
            torch.zeros(L2_FLUSH_BYTES, dtype=torch.uint8, device=device))


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

def prefill_case(wl, device, seed_offset=0):
    import block_sparse_long_landmark_b200 as sa
    from block_sparse_long_landmark_b200 import inputs
    wl = wl.scaled(seed=wl.seed + 1000 * seed_offset) if seed_offset else wl
    p = sa.params_for(wl)
    Q, K, V = inputs.make_prefill(wl, device=device)
    ws = sa.workspace(p, device=device)
    nb = wl.nb
    L = torch.empty(wl.B, wl.Hkv, nb, wl.d, dtype=Q.dtype, device=device)
    sel = sa._sel_out(p, False, device)
    O = torch.empty_like(Q)
    lse = torch.empty(wl.B, wl.Hq, wl.N, dtype=torch.float32, device=device)
    return wl, p, dict(Q=Q, K=K, V=V, ws=ws, L=L, sel=sel, O=O, lse=lse)


def prefill_step(p, t, timer=None):
    import block_sparse_long_landmark_b200 as sa
    tm = timer or (lambda n, f: f())
    tm("landmarks", lambda: sa.landmarks(p, t["K"], out=t["L"]))
    tm("select", lambda: sa.select(p, t["Q"], t["L"], t["ws"], out=t["sel"]))
    tm("prefill", lambda: sa.prefill(p, t["Q"], t["K"], t["V"], *t["sel"], t["ws"], out=(t["O"], t["lse"])))


def prefill_flops(wl, cnt) -> float:
    """Gathered FLOPs of one prefill launch: QK^T and PV over every kept
    (tile, block) pair, the local block counted whole: 4 * rows * keys * d,
    where a list serves G * block query rows (block rows with one list per
    query head)."""
    rows = wl.block if wl.per_qhead else (wl.Hq // wl.Hkv) * wl.block
    pairs = float(cnt.sum().item())
    return pairs * 4.0 * rows * wl.block * wl.d


def decode_case(wl, device, lens=None):
    """Decode inputs; with `lens` a ragged batch (sequence b holds lens[b]
    keys of the cache) that runs through the varlen entry points."""
    import block_sparse_long_landmark_b200 as sa
    from block_sparse_long_landmark_b200 import inputs
    p = sa.params_for(wl)
    q, K, V = inputs.make_decode(wl, device=device)
    ws = sa.workspace(p, device=device, ops=sa.DECODE_OPS)
    t = dict(q=q, K=K, V=V, ws=ws)
    if lens is None:
        t["L"] = sa.landmarks(p, K)
    else:
        t["sl"] = torch.tensor(lens, dtype=torch.int32, device=device)
        t["L"] = torch.zeros(wl.B, wl.Hkv, wl.nb, wl.d, dtype=K.dtype, device=device)
        sa.landmarks_update(p, K, t["L"], seq_len=t["sl"])
    t["sel"] = sa._sel_out(p, True, device)
    t["o"] = torch.empty_like(q)
    t["lse"] = torch.empty(wl.B, wl.Hq, dtype=torch.float32, device=device)
    return p, t


def decode_step(p, t, timer=None):
    """One decode step.  Timed: the library's decode-step call (selection and
    decode launches overlapped); attribution (with a timer): the two calls
    one after the other, each between events."""
    import block_sparse_long_landmark_b200 as sa
    if timer is None:
        sa.decode_step(p, t["q"], t["L"], t["K"], t["V"], t["ws"], seq_len=t.get("sl"), sel=t["sel"],
                       out=(t["o"], t["lse"]))
        return
    tm = timer
    if "sl" in t:
        tm("select_decode", lambda: sa.select_decode_varlen(p, t["q"], t["L"], t["sl"], t["ws"], out=t["sel"]))
        tm("decode", lambda: sa.decode_varlen(p, t["q"], t["K"], t["V"], t["sl"], *t["sel"], t["ws"],
                                              out=(t["o"], t["lse"])))
        return
    tm("select_decode", lambda: sa.select_decode(p, t["q"], t["L"], t["ws"], out=t["sel"]))
    tm("decode", lambda: sa.decode(p, t["q"], t["K"], t["V"], *t["sel"], t["ws"], out=(t["o"], t["lse"])))


def run_timed(step, steps, warmup, ranks, flush_buf):
    """Times `steps` steps, each after an L2 flush, with one event pair
    around each step and nothing recorded inside it (so launches that may
    overlap their predecessor do).  Then a second pass of the same steps with
    events around every kernel call attributes the time to kernels."""
    for _ in range(warmup):
        step(None)
    torch.cuda.synchronize()
    ranks.barrier()
    torch.cuda.synchronize()
    import block_sparse_long_landmark_b200 as sa
    n0 = sa.sparse_attn_launch_count()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    starts, ends = [], []
    for _ in range(steps):
        flush_l2(flush_buf)
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        step(None)
        e.record()
        starts.append(s)
        ends.append(e)
    torch.cuda.synchronize()
    ranks.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    launches = sa.sparse_attn_launch_count() - n0
    elapsed = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    # attribution pass (not part of the timed steps)
    timer = Timer()
    for _ in range(steps):
        flush_l2(flush_buf)
        step(timer)
    torch.cuda.synchronize()
    return elapsed, timer.ms(), launches, clocks


# ----------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and --impl reference)
# ----------------------------------------------------------------------------

def oracle_prefill_sample(wl, Q64, K64, V64, n_units, seed=0, threads=None):
    """Times the oracle on ``n_units`` (batch, kv-head, tile) units drawn from
    the upper tiles (every one with a full top-K list).  Returns (seconds,
    token-equivalents, threads)."""
    import oracle
    rng = np.random.default_rng(seed)
    lo = min(wl.nb - 1, wl.top_k + 2)
    units = [(0, int(rng.integers(0, wl.Hkv)), int(rng.integers(lo, wl.nb))) for _ in range(n_units)]
    threads = threads or os.cpu_count() or 1
    t0 = time.perf_counter()
    oracle.prefill(Q64, K64, V64, wl.block, wl.top_k, wl.flags, round_mode=oracle.ROUND_BF16, units=units,
                   threads=threads)
    dt = time.perf_counter() - t0
    return dt, n_units * wl.block / wl.Hkv, threads


def cpu_inputs(wl):
    from block_sparse_long_landmark_b200 import inputs
    Q, K, V = inputs.make_prefill(wl, device="cpu")
    return (Q.float().numpy().astype(np.float64), K.float().numpy().astype(np.float64),
            V.float().numpy().astype(np.float64))


def calibrate_units(wl, Q64, K64, V64, target_s):
    """Units whose oracle time is about target_s: two probes fit t = a + b n
    (a: the landmarks of the touched kv-heads, b: one unit's selection and
    attention)."""
    # a first call pays one-time costs (the oracle's build and load, first
    # touch of the inputs) that must not enter the fit
    oracle_prefill_sample(wl, Q64, K64, V64, 4, seed=97)
    t1, _, _ = oracle_prefill_sample(wl, Q64, K64, V64, 16, seed=98)
    t2, _, _ = oracle_prefill_sample(wl, Q64, K64, V64, 64, seed=99)
    # per-unit cost: the slope, but never below half the larger probe's mean
    # (timing noise can flatten the slope and inflate the sample)
    b = max((t2 - t1) / 48, 0.5 * t2 / 64, 1e-6)
    a = max(t1 - 16 * b, 0.0)
    return max(16, min(50000, int((target_s - a) / b)))


def cpu_baseline(wl, target_s):
    Q64, K64, V64 = cpu_inputs(wl)
    n = calibrate_units(wl, Q64, K64, V64, target_s)
    dt, tok, threads = oracle_prefill_sample(wl, Q64, K64, V64, n, seed=1)
    # the same oracle on one host thread, on a sample about 1/threads as large
    n1 = max(4, n // max(1, threads))
    dt1, tok1, _ = oracle_prefill_sample(wl, Q64, K64, V64, n1, seed=2, threads=1)
    return {"value": tok / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} random (kv-head, tile) units of {wl.name} with full top-{wl.top_k} lists "
                      f"(landmarks of the touched kv-heads, selection and gated attention), "
                      f"{dt:.1f} s on {threads} host threads; tokens counted as block/Hkv per unit",
            "one_core": {"value": tok1 / dt1, "unit": "tokens/s", "cores": 1,
                         "sample": f"{n1} units, {dt1:.1f} s on 1 thread"}}


def run_reference(args, ranks):
    from block_sparse_long_landmark_b200 import inputs
    if ranks.rank != 0:
        return 0
    wl = inputs.WORKLOADS[args.workload]
    Q64, K64, V64 = cpu_inputs(wl)
    # a few minutes in all, each step's sample capped by --cpu-seconds
    per_step_s = min(args.cpu_seconds, max(2.0, min(15.0, 150.0 / max(1, args.steps + args.warmup))))
    n = calibrate_units(wl, Q64, K64, V64, per_step_s)
    rates, times = [], []
    threads = os.cpu_count() or 1
    for i in range(args.warmup + args.steps):
        dt, tok, threads = oracle_prefill_sample(wl, Q64, K64, V64, n, seed=10 + i)
        if i >= args.warmup:
            rates.append(tok / dt)
            times.append(dt)
    value = statistics.fmean(rates)
    sample = (f"each step: {n} random (kv-head, tile) units of {wl.name} on {threads} host threads; "
              f"tokens counted as block/Hkv per unit")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.fmean(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl, extra=None):
    c = {"workload": wl.name, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "d": wl.d, "seq_len": wl.N,
         "block": wl.block, "top_k": wl.top_k, "flags": wl.flags, "mode": "hier" if wl.hier else "gated",
         "global_batch": wl.B, "parallelism": "replicas (independent sequences per rank)",
         "l2": "flushed before every timed step (256 MiB written, then 256 MiB read: no input and no dirty "
               "line in L2)"}
    if extra:
        c.update(extra)
    return c


# ----------------------------------------------------------------------------
# main arms
# ----------------------------------------------------------------------------

def e2e_prefill(wl, p, t, steps):
    """Same metric through the public API with host buffers: pinned H2D of
    Q, K, V, the three calls, D2H of O and LSE, all inside the events."""
    hQ = t["Q"].cpu().pin_memory()
    hK = t["K"].cpu().pin_memory()
    hV = t["V"].cpu().pin_memory()
    hO = torch.empty(t["O"].shape, dtype=t["O"].dtype).pin_memory()
    hL = torch.empty(t["lse"].shape, dtype=torch.float32).pin_memory()
    times = []
    for i in range(steps + 1):
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        t["Q"].copy_(hQ, non_blocking=True)
        t["K"].copy_(hK, non_blocking=True)
        t["V"].copy_(hV, non_blocking=True)
        prefill_step(p, t)
        hO.copy_(t["O"], non_blocking=True)
        hL.copy_(t["lse"], non_blocking=True)
        e.record()
        torch.cuda.synchronize()
        if i:
            times.append(s.elapsed_time(e))
    ms = statistics.fmean(times)
    h2d = sum(x.numel() * x.element_size() for x in (hQ, hK, hV))
    d2h = hO.numel() * hO.element_size() + hL.numel() * 4
    return ms, h2d, d2h


def _wl(name, args):
    from block_sparse_long_landmark_b200 import inputs
    wl = inputs.WORKLOADS[name]
    over = {k: v for k, v in (("N", args.N), ("B", args.B)) if v}
    return wl.scaled(**over) if over else wl


def secondary_prefill(name, args, pk, psrc):
    wl, p, t = prefill_case(_wl(name, args), "cuda")
    flush = flush_buffers()
    ranks1 = Ranks.single()
    steps = max(2, min(args.steps, 5))
    el, kms, launches, clocks = run_timed(lambda tm: prefill_step(p, t, tm), steps, max(3, args.warmup),
                                          ranks1, flush)
    flops = prefill_flops(wl, t["sel"][2])
    ach = flops / (kms["prefill"] / 1e3) / 1e12
    out = {"metric": "prefill tokens/s", "value": wl.N * wl.B / (el / steps / 1e3), "unit": "tokens/s",
           "ms_per_step": el / steps, "kernels_ms": kms, "config": workload_config(wl), "gpu_launches": launches,
           "roofline": {"bound": "tensor", "achieved": ach, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                        "frac": ach / pk["bf16_tflops"], "peak_source": psrc + " bf16 burst",
                        "gathered_flops_per_launch": flops, "traffic": traffic_for("prefill_" + wl.name)},
           "clocks": clocks}
    del t
    torch.cuda.empty_cache()
    return out


# fp32 FMA peak of the CUDA cores, derived from unit counts and the clock:
# 148 SMs x 128 FP32 lanes x 2 FLOP x 1.965 GHz (no measured figure exists).
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def secondary_backward(name, args, pk, psrc):
    """One backward step (attention backward + selector backward) of the gated
    prefill, the forward's outputs and an upstream gradient resident in HBM."""
    import block_sparse_long_landmark_b200 as sa
    base = name.replace("_backward", "")
    wl, p, t = prefill_case(_wl(base, args), "cuda")
    prefill_step(p, t)
    g = torch.Generator(device="cuda").manual_seed(11)
    dO = torch.randn(t["Q"].shape, generator=g, device="cuda", dtype=torch.float32).to(t["Q"].dtype)
    f32 = dict(dtype=torch.float32, device="cuda")
    grads = (torch.empty(t["Q"].shape, **f32), torch.empty(t["K"].shape, **f32), torch.empty(t["V"].shape, **f32),
             torch.empty(t["sel"][1].shape, **f32))

    def step(tm):
        tmr = tm or (lambda n, f: f())
        tmr("prefill_backward", lambda: sa.prefill_backward(p, t["Q"], t["K"], t["V"], t["O"], t["lse"], dO,
                                                            *t["sel"], t["ws"], out=grads))
        tmr("select_backward", lambda: sa.select_backward(p, t["Q"], t["L"], t["sel"][0], grads[3], t["sel"][2],
                                                          grads[0], grads[1], t["ws"]))

    flush = flush_buffers()
    steps = 2
    el, kms, launches, clocks = run_timed(step, steps, 3, Ranks.single(), flush)
    # 10 d FLOP per kept (row, key) pair: z, dO.V, dQ, dK, dV (the tensor-core path recomputes
    # z and dO.V once more for dQ; that extra work is not counted); the forward's count is 4 d
    flops = prefill_flops(wl, t["sel"][2]) * 10 / 4
    ach = flops / (kms["prefill_backward"] / 1e3) / 1e12
    G = wl.Hq // wl.Hkv
    tensor = (wl.dtype == "bf16" and wl.d == 128 and wl.block in (64, 128) and (G * wl.block) % 128 == 0
              and not wl.hier and not wl.per_qhead)
    if tensor:
        roof = {"bound": "tensor", "peak": pk["bf16_tflops"], "peak_source": psrc + " bf16 burst"}
    else:
        roof = {"bound": "alu", "peak": FP32_ALU_TFLOPS,
                "peak_source": "derived: 148 SMs x 128 fp32 FMA x 2 x 1.965 GHz"}
    roof.update({"achieved": ach, "unit": "TFLOP/s", "frac": ach / roof["peak"], "kernel": "prefill_backward",
                 "algorithmic_flops_per_launch": flops, "traffic": None})
    out = {"metric": "prefill backward tokens/s", "value": wl.N * wl.B / (el / steps / 1e3), "unit": "tokens/s",
           "ms_per_step": el / steps, "kernels_ms": kms, "config": workload_config(wl), "gpu_launches": launches,
           "roofline": roof, "clocks": clocks}
    del t, grads, dO
    torch.cuda.empty_cache()
    return out


# flat clustered index (Latent Sparse Attention style): 8 sequences of 32K
# keys, 8 kv-heads and 32 query heads, 4-key items, 64-item segments of 16
# clusters, 64 clusters expanded per query, 64 sink and 1024 window positions
LSA_DECODE_32K = dict(B=8, Hq=32, Hkv=8, d=128, N=32768, pool=4, seg=64, clusters=16, top_clusters=64, sink=64,
                      window=1024)


def secondary_lsa(name, args, pk, psrc):
    """Decode through the flat clustered index; the index is built once,
    outside the timed region (its build time is reported beside)."""
    import block_sparse_long_landmark_b200 as sa
    c = LSA_DECODE_32K
    p = sa.make_lsa_params(**c)
    g = torch.Generator(device="cuda").manual_seed(21)
    q = torch.randn(c["B"], c["Hq"], c["d"], generator=g, device="cuda").to(torch.bfloat16)
    K = torch.randn(c["B"], c["Hkv"], c["N"], c["d"], generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn(c["B"], c["Hkv"], c["N"], c["d"], generator=g, device="cuda").to(torch.bfloat16)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    index = sa.lsa_build(p, K)
    s1.record()
    torch.cuda.synchronize()
    build_ms = s0.elapsed_time(s1)
    ws = sa.lsa_workspace(p)
    out = (torch.empty_like(q), torch.empty(c["B"], c["Hq"], dtype=torch.float32, device="cuda"))
    kept = torch.zeros(c["B"], c["Hkv"], dtype=torch.int32, device="cuda")

    def step(tm):
        (tm or (lambda n, f: f()))("lsa_decode", lambda: sa.lsa_decode(p, q, K, V, index, ws, out=out, kept=kept))

    flush = flush_buffers()
    steps = 10
    el, kms, launches, clocks = run_timed(step, steps, 3, Ranks.single(), flush)
    C = sa.sparse_attn_lsa_clusters(p)
    # algorithmic bytes: every centre (fp64) once, the chosen clusters' member
    # tables, and K and V of every kept position once
    nkept = int(kept.sum().item())
    member_bytes = c["B"] * c["Hkv"] * c["top_clusters"] * (c["seg"] + 1) * 4
    nbytes = c["B"] * c["Hkv"] * C * c["d"] * 8 + member_bytes + nkept * c["d"] * 2 * 2
    hbm = pk["hbm_gbs"]
    ach = nbytes / (kms["lsa_decode"] / 1e3) / 1e9
    return {"metric": "lsa decode queries/s", "value": c["B"] / (el / steps / 1e3), "unit": "queries/s",
            "ms_per_step": el / steps, "kernels_ms": kms, "index_build_ms": build_ms, "config": dict(c),
            "gpu_launches": launches, "kept_positions": nkept,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                         "algorithmic_bytes": nbytes, "traffic": None,
                         "peak_source": psrc + " HBM copy"},
            "clocks": clocks}


LSA_TREE = dict(fanout=4, beam=16)


def secondary_lsa_tree(name, args, pk, psrc):
    """Decode through the tree over the flat index (beam search to the
    leaves); index and tree are built once, outside the timed region."""
    import block_sparse_long_landmark_b200 as sa
    c = LSA_DECODE_32K
    p = sa.make_lsa_params(**c)
    g = torch.Generator(device="cuda").manual_seed(21)
    q = torch.randn(c["B"], c["Hq"], c["d"], generator=g, device="cuda").to(torch.bfloat16)
    K = torch.randn(c["B"], c["Hkv"], c["N"], c["d"], generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn(c["B"], c["Hkv"], c["N"], c["d"], generator=g, device="cuda").to(torch.bfloat16)
    index = sa.lsa_build(p, K)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    tree, ws = sa.lsa_tree_build(p, LSA_TREE["fanout"], index)
    s1.record()
    torch.cuda.synchronize()
    build_ms = s0.elapsed_time(s1)
    out = (torch.empty_like(q), torch.empty(c["B"], c["Hq"], dtype=torch.float32, device="cuda"))
    kept = torch.zeros(c["B"], c["Hkv"], dtype=torch.int32, device="cuda")
    comp = torch.zeros_like(kept)

    def step(tm):
        (tm or (lambda n, f: f()))("lsa_tree_decode", lambda: sa.lsa_tree_decode(
            p, LSA_TREE["fanout"], LSA_TREE["beam"], q, K, V, index, tree, ws, out=out, kept=kept, compared=comp))

    flush = flush_buffers()
    steps = 10
    el, kms, launches, clocks = run_timed(step, steps, 3, Ranks.single(), flush)
    nkept, ncomp = int(kept.sum().item()), int(comp.sum().item())
    # algorithmic bytes: every centre compared (fp64), the chosen leaves' member
    # tables, K and V of every kept position
    member_bytes = c["B"] * c["Hkv"] * c["top_clusters"] * (c["seg"] + 1) * 4
    nbytes = ncomp * c["d"] * 8 + member_bytes + nkept * c["d"] * 2 * 2
    hbm = pk["hbm_gbs"]
    ach = nbytes / (kms["lsa_tree_decode"] / 1e3) / 1e9
    return {"metric": "lsa tree decode queries/s", "value": c["B"] / (el / steps / 1e3), "unit": "queries/s",
            "ms_per_step": el / steps, "kernels_ms": kms, "tree_build_ms": build_ms,
            "config": dict(c, **LSA_TREE), "gpu_launches": launches, "kept_positions": nkept,
            "centres_compared": ncomp, "centres_total": c["B"] * c["Hkv"] * sa.sparse_attn_lsa_clusters(p),
            "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                         "algorithmic_bytes": nbytes, "traffic": None, "peak_source": psrc + " HBM copy"},
            "clocks": clocks}


def secondary_decode(name, args, pk, psrc):
    varlen = name.endswith("_varlen")
    wl = _wl(name[:-len("_varlen")] if varlen else name, args)
    lens = None
    if varlen:
        # ragged batch: lengths uniform in [N/2, N], seeded
        lens = np.random.default_rng(11).integers(wl.N // 2, wl.N + 1, size=wl.B)
    p, t = decode_case(wl, "cuda", lens)
    flush = flush_buffers()
    ranks1 = Ranks.single()
    steps = max(3, args.steps)
    el, kms, launches, clocks = run_timed(lambda tm: decode_step(p, t, tm), steps, max(3, args.warmup),
                                          ranks1, flush)
    esz = 2 if wl.dtype == "bf16" else 4
    cnt = t["sel"][2].to(torch.int64)
    if lens is None:
        scan_bytes = wl.B * wl.Hkv * ((wl.N - 1) // wl.block + 1) * wl.d * esz
    else:
        scan_bytes = sum(wl.Hkv * ((int(n) - 1) // wl.block + 1) * wl.d * esz for n in lens)
    if wl.per_qhead:
        # algorithmic bytes: each kv-head's union of the blocks its query heads keep
        G = wl.Hq // wl.Hkv
        idx = t["sel"][0].view(wl.B, wl.Hkv, G * (wl.top_k + 2)).to(torch.int64)
        hit = torch.zeros(wl.B, wl.Hkv, wl.nb + 1, dtype=torch.bool, device=idx.device)
        hit.scatter_(2, torch.where(idx < 0, wl.nb, idx), True)
        gather_bytes = float(hit[..., :wl.nb].sum().item()) * wl.block * wl.d * esz * 2
    else:
        gather_bytes = float(cnt.sum().item()) * wl.block * wl.d * esz * 2
    ach_dec = gather_bytes / (kms["decode"] / 1e3) / 1e9
    ach_sel = scan_bytes / (kms["select_decode"] / 1e3) / 1e9
    step_ach = (scan_bytes + gather_bytes) / (el / steps / 1e3) / 1e9
    hbm = pk["hbm_gbs"]
    cfg = workload_config(wl, {"seq_len_min": int(min(lens)), "seq_len_mean": float(np.mean(lens)),
                               "varlen": True} if varlen else None)
    out = {"metric": "decode queries/s", "value": wl.B / (el / steps / 1e3), "unit": "queries/s",
           "ms_per_step": el / steps, "kernels_ms": kms, "config": cfg, "gpu_launches": launches,
           "roofline": {"bound": "hbm", "achieved": step_ach, "peak": hbm, "unit": "GB/s", "frac": step_ach / hbm,
                        "peak_source": psrc, "bytes_per_step": scan_bytes + gather_bytes,
                        "traffic": None},
           "kernels_roofline": {
               "decode": {"bound": "hbm", "achieved": ach_dec, "peak": hbm, "unit": "GB/s", "frac": ach_dec / hbm,
                          "algorithmic_bytes": gather_bytes, "traffic": traffic_for("decode_" + name)},
               "select_decode": {"bound": "hbm", "achieved": ach_sel, "peak": hbm, "unit": "GB/s",
                                 "frac": ach_sel / hbm, "algorithmic_bytes": scan_bytes,
                                 "traffic": traffic_for("select_decode_" + name)}},
           "clocks": clocks}
    del t
    torch.cuda.empty_cache()
    return out


def _sig(x, n=3):
    return None if x is None else float(f"{x:.{n}g}")


def compact(rec: dict) -> dict:
    """The few fields of a secondary record that the summary keeps: value,
    step time, per-kernel mean times and roofline fractions."""
    if "error" in rec:
        return {"error": rec["error"][:120]}
    unit = {"tokens/s": "tok/s", "queries/s": "q/s"}.get(rec["unit"], rec["unit"])
    out = {"v": _sig(rec["value"]), "u": unit, "ms": _sig(rec["ms_per_step"]),
           "frac": _sig(rec["roofline"]["frac"], 2)}
    kr = rec.get("kernels_roofline", {})
    out["k"] = {k: ([_sig(v), _sig(kr[k]["frac"], 2)] if k in kr else _sig(v))
                for k, v in rec["kernels_ms"].items()}
    ck = rec.get("clocks") or {}
    out["mhz"] = ck.get("sm_mhz")
    if ck.get("reasons"):
        out["why"] = ck["reasons"]
    return out


# secondary workloads at N = 1, in the order they print: the decodes at the
# metric's 128K context and the 1M hierarchical decode come last, so that they
# stay in the tail of the line.  Summary keys: v value, u unit, ms step time,
# frac the roofline fraction of the step (decode) or of the prefill kernel,
# k per-kernel mean ms (with its own roofline fraction where one is defined),
# mhz median SM clock, why throttle reasons seen
SECONDARY = ("long_prefill_256k", "gated_prefill_32k", "hils_prefill_32k", "gated_prefill_32k_perqhead",
             "gated_prefill_32k_backward", "lsa_decode_32k", "lsa_tree_decode_32k", "gated_decode_128k_perqhead",
             "gated_decode_128k_varlen",
             "hils_decode_1m", "gated_decode_128k")


def secondary_select_only(name, args, pk, psrc):
    """Decode selection alone (profiling): the workload's query and random
    landmarks of its context, no KV cache -- the selection reads only these."""
    import block_sparse_long_landmark_b200 as sa
    wl = _wl(name[:-len("_select")], args)
    p = sa.params_for(wl)
    g = torch.Generator(device="cuda").manual_seed(wl.seed)
    q = (torch.randn(wl.B, wl.Hq, wl.d, generator=g, device="cuda") * wl.sigma).to(wl.torch_dtype)
    L = (torch.randn(wl.B, wl.Hkv, wl.nb, wl.d, generator=g, device="cuda") * wl.sigma).to(wl.torch_dtype)
    ws = sa.workspace(p, ops=sa.DECODE_OPS)
    sel = sa._sel_out(p, True, "cuda")
    flush = flush_buffers()
    steps = max(3, args.steps)
    el, kms, launches, clocks = run_timed(
        lambda tm: (tm or (lambda n, f: f()))("select_decode", lambda: sa.select_decode(p, q, L, ws, out=sel)),
        steps, max(3, args.warmup), Ranks.single(), flush)
    nbytes = wl.B * wl.Hkv * ((wl.N - 1) // wl.block + 1) * wl.d * L.element_size()
    ach = nbytes / (kms["select_decode"] / 1e3) / 1e9
    return {"metric": "decode selection queries/s", "value": wl.B / (el / steps / 1e3), "unit": "queries/s",
            "ms_per_step": el / steps, "kernels_ms": kms, "config": workload_config(wl), "gpu_launches": launches,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / pk["hbm_gbs"], "algorithmic_bytes": nbytes, "traffic": None,
                         "peak_source": psrc + " HBM copy"},
            "clocks": clocks}


def run_secondary(name, args, pk, psrc):
    from block_sparse_long_landmark_b200 import inputs
    if name == "lsa_decode_32k":
        return secondary_lsa(name, args, pk, psrc)
    if name == "lsa_tree_decode_32k":
        return secondary_lsa_tree(name, args, pk, psrc)
    if name.endswith("_select"):
        return secondary_select_only(name, args, pk, psrc)
    if name.endswith("_backward"):
        return secondary_backward(name, args, pk, psrc)
    kind = inputs.WORKLOADS[name.replace("_varlen", "")].kind
    return (secondary_decode if kind == "decode" else secondary_prefill)(name, args, pk, psrc)


def run_ours(args, ranks):
    import block_sparse_long_landmark_b200 as sa
    from block_sparse_long_landmark_b200 import inputs
    sa.lib()   # fails loudly without the built CUDA library
    dev = torch.device("cuda", ranks.local)
    torch.cuda.set_device(dev)
    pk, psrc = peaks()
    if args.only:
        # one workload alone (small profiling cases): a short report, no baselines
        print(json.dumps({"only": args.only, **run_secondary(args.only, args, pk, psrc)}), flush=True)
        return 0
    base = inputs.WORKLOADS[args.workload]
    wl, p, t = prefill_case(base, "cuda", seed_offset=ranks.rank)
    flush = flush_buffers()
    el, kms, launches, clocks = run_timed(lambda tm: prefill_step(p, t, tm), args.steps, args.warmup, ranks, flush)
    value, el_max = aggregate(ranks, el, wl.N * wl.B * args.steps)
    flops = prefill_flops(wl, t["sel"][2])
    ach = flops / (kms["prefill"] / 1e3) / 1e12
    e2e_ms, h2d, d2h = e2e_prefill(wl, p, t, min(args.steps, 5))
    e2e_value, _ = aggregate(ranks, e2e_ms, wl.N * wl.B)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ranks.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": el_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "f32",
        "data": "synthetic: seeded Gaussian Q/K/V with planted relevant blocks",
        "config": workload_config(wl),
        "roofline": {"bound": "tensor", "achieved": ach, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": ach / pk["bf16_tflops"], "traffic": traffic_for("prefill_" + wl.name),
                     "kernel": "prefill", "peak_source": psrc + " bf16 burst",
                     "gathered_flops_per_launch": flops},
        "kernels_ms": kms,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    del t
    torch.cuda.empty_cache()
    if ranks.world == 1 and ranks.rank == 0:
        if not args.no_cpu:
            line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
        if not args.no_secondary:
            full = {}
            for name in SECONDARY:
                if name == wl.name:
                    continue
                try:
                    full[name] = run_secondary(name, args, pk, psrc)
                except torch.cuda.OutOfMemoryError as e:   # pragma: no cover -- recorded, the line still prints
                    full[name] = {"error": f"out of memory: {e}"}
                except sa.SparseAttnError as e:            # pragma: no cover
                    full[name] = {"error": str(e)}
                torch.cuda.empty_cache()
            if args.detail:
                with open(args.detail, "w") as f:
                    json.dump(full, f, indent=1)
            # last key of the line: what a truncated tail still shows
            line["secondary"] = {k: compact(v) for k, v in full.items()}
    if ranks.rank == 0:
        print(json.dumps(line, separators=(",", ":")), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long_prefill_256k")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--only", default=None, help="measure this one workload alone (profiling)")
    ap.add_argument("--detail", default=None, help="write the secondary workloads' full records to this file")
    ap.add_argument("--N", type=int, default=0, help="with --only: override the sequence/context length")
    ap.add_argument("--B", type=int, default=0, help="with --only: override the batch")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        # rank 0 alone times the oracle; other ranks exit without work
        return run_reference(args, Ranks.single()) if int(os.environ.get("RANK", "0")) == 0 else 0
    ranks = Ranks(backend="nccl")
    try:
        return run_ours(args, ranks)
    finally:
        ranks.close()


if __name__ == "__main__":
    sys.exit(main())
