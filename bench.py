"""Benchmark of the Mamba-2 recurrent-state decode step on B200.

Workload (one "step" = one pass of the whole decode hot path over one batch):
the Nemotron-H-8B mixer layer (H=128, P=64, N=128, G=8, K=4, conv_dim=10240),
bf16 state (2 MiB per sequence) and activations, 64 active sequences
scattered over a 256-slot cache, one fused launch per step (slot lookup, conv
tap and roll, dt/dA, state update, C read-out, D skip, silu(z) gate).

Metric: decode seq*layer-steps/s (whole job, all ranks), with the state GB/s
and its fraction of HBM in the ``roofline`` object. Inputs are synthetic
(seeded generators; no trained weights exist for this path) and resident in
HBM when the timed region starts. By default consecutive steps rotate through
the cache's four disjoint 64-slot batches, so a slot's 2 MiB state comes back
only after 536 MB of other state traffic (L2 is 126 MB) and the steps run back
to back as a layer loop would; ``--l2 flush`` instead writes 512 MiB before
every timed step (outside the kernel's events) and always uses slot set 0.

Usage: ``python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]``.
With N > 1 the script runs under torchrun: each rank runs an independent
replica of the workload on its own GPU (the path has no exchange step), and
``value`` is the units of all ranks over the max-over-ranks device time.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode seq*layer-steps/s"
UNIT = "seq*layer-steps/s"
WORKLOAD = "nemotron_h_layer decode: H=128 P=64 N=128 G=8 K=4, bf16 state+act, batch 64 / 256 slots"
FLUSH_BYTES = 512 * 1024 * 1024
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "state_update_nemotron_h_layer.md")
KERNEL_SOURCES = ["mamba_recurrent_state_b200/csrc/m2_state_update.cu",
                  "mamba_recurrent_state_b200/csrc/m2_device.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="budget of the oracle CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--l2", choices=["rotate", "flush"], default="rotate",
                    help="rotate: disjoint slot sets, back to back; flush: 512 MiB write before each step")
    ap.add_argument("--sections", default="decode,norm,multi,prefill,longprompt,stack48,fp32_23l,t1_ab",
                    help="comma list: decode (the headline, always run), norm (decode with the "
                         "fused gated RMSNorm), multi (4 speculative draft tokens), prefill (workload 4: "
                         "prefill conv and tensor-core scan), longprompt (one 16K-token prompt: "
                         "conv and varlen scan), stack48 (workload 2: 48-layer token), fp32_23l "
                         "(workload 3: fp32 state, 23 layers, 64 steps), t1_ab (one decode token "
                         "through the prefill path, conv + chunk scan at T = 1, against the decode step)")
    return ap.parse_args()


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _peak(key: str, fallback: float) -> tuple[float, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)[key]), "measured"
    except (OSError, KeyError, ValueError):
        return fallback, "fallback"


def measured_peaks() -> tuple[float, str]:
    """HBM copy bandwidth, GB/s (measured on this machine, else the fallback)."""
    return _peak("hbm_gbs", 6650.0)


def measured_tensor_peak() -> tuple[float, str]:
    """Dense 16-bit tensor throughput, TFLOP/s (the cuBLAS bf16 burst figure;
    fp16 and bf16 share the nominal dense rate)."""
    return _peak("bf16_tflops", 1590.0)


def profiled_traffic() -> float | None:
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (null otherwise)."""
    try:
        text = open(PROFILE_SUMMARY).read()
    except OSError:
        return None
    m_src = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text)
    m_b = re.search(r"traffic_bytes_per_launch:\s*([0-9.e+]+)", text)
    if not m_src or not m_b or m_src.group(1) != kernel_source_hash():
        return None
    return float(m_b.group(1))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 50 ms while the
    benchmark runs; only samples that arrive inside the timed region count."""

    QUERY = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.samples: list[tuple[float, str]] = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        t0 = time.monotonic()  # wait for the first sample (nvidia-smi start-up)
        while not self.samples and time.monotonic() - t0 < 5.0:
            time.sleep(0.05)

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.monotonic(), line.strip()))

    def stop(self, t_begin: float, t_end: float) -> dict | None:
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        for ts, ln in self.samples:
            if not (t_begin <= ts <= t_end + 0.06):
                continue
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(self.REASONS, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "samples": 0, "reasons": [],
                    "note": "no nvidia-smi sample landed inside the timed region"}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest of every rank's ``x`` (a device time); every rank gets it."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, local_ms: float, world: int) -> tuple[float, float]:
    """Whole-job throughput of replicas: every rank's units over the slowest
    rank's device time. Returns (units per second, that time in ms)."""
    ms = max_over_ranks(local_ms, world)
    return units_per_rank * world / (ms / 1e3), ms


def oracle_sample(rows: int = 16, threads: int | None = None):
    """A bounded sample of the workload step for the oracle: ``rows`` of the 64
    sequences, inputs generated up front, run on ``threads`` host threads (all
    of them by default). Returns (step function, rows, threads)."""
    import numpy as np
    import m2synth as S
    import oracle as O
    from m2synth import workloads as W
    w = W.WORKLOADS[1]
    orc = O.default()
    p = W.layer_params(w)
    f64 = S.storage_to_f64
    idx = list(range(rows))
    slots = W.slot_indices(w)
    ssm_rows = [np.ascontiguousarray(f64(W.ssm_slot(w, int(slots[r])), w.state_dtype)) for r in idx]
    conv_rows = [np.ascontiguousarray(f64(W.conv_slot(w, int(slots[r])), w.act_dtype)) for r in idx]
    inp = {k: f64(v, w.act_dtype) for k, v in W.step_inputs(w, 0, rows=idx).items()}
    params = (f64(p.conv_w, w.act_dtype), f64(p.conv_b, w.act_dtype), p.dt_bias.astype(np.float64),
              p.A_log.astype(np.float64), p.D.astype(np.float64))
    threads = threads or os.cpu_count() or 1

    def step():
        O.decode_rows(orc, w.H, w.P, w.N, w.G, O.ROUND_BF16, ssm_rows, conv_rows, inp["xBC"],
                      inp["dt"], inp["z"], *params, threads=threads)

    return step, rows, threads


def cpu_baseline(seconds: float) -> dict:
    """The oracle, as it stands, on the host cores: one decode step over a
    sample of the workload's sequences, repeated until the time budget is used."""
    step, rows, threads = oracle_sample()
    done = 0
    t0 = time.perf_counter()
    while True:
        step()
        done += rows
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    # the same oracle on one thread, on a smaller sample (a fifth of the budget)
    step1, rows1, _ = oracle_sample(rows=4, threads=1)
    done1 = 0
    t1 = time.perf_counter()
    while True:
        step1()
        done1 += rows1
        el1 = time.perf_counter() - t1
        if el1 >= seconds / 5:
            break
    return {"value": done / el, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{rows} of the 64 sequences of the workload step, decoded "
                      f"{done // rows} times ({done} seq*layer-steps in {el:.1f} s)",
            "one_thread": {"value": done1 / el1, "unit": UNIT, "cores": 1,
                           "sample": f"{rows1} sequences, {done1 // rows1} times ({el1:.1f} s)"}}


def run_reference(args, world, rank):
    """The reference arm: the oracle as it stands on the host cores (rank 0 only)."""
    if rank != 0:
        return
    step, rows, threads = oracle_sample()
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = rows * args.steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded generators)",
        "config": {"workload": WORKLOAD, "sample_rows": rows},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{rows} of the 64 sequences per step, {args.steps} steps"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _time_us(fn, flush, reps: int) -> list[float]:
    """Device time of fn() per rep (CUDA events on the current stream), L2
    flushed before every rep, outside the events."""
    import torch
    stream = torch.cuda.current_stream()
    out = []
    for _ in range(reps):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        out.append(1e3 * a.elapsed_time(b))
    return out


def measure_prefill(flush, peak_gbs: float, peak_tflops: float, reps: int = 10) -> dict:
    """Workload 4's prefill: conv over 8 x 2048 tokens, then the tensor-core
    chunk scan (fp16 operands, fp32 accumulate, 128-token chunks)."""
    import torch
    import mamba_recurrent_state_b200 as m2
    from m2synth import torch_inputs as TI
    from m2synth import workloads as W
    w = W.WORKLOADS[4]
    shape = m2.Shape(w.H, w.P, w.N, w.G, w.K, w.state_dtype, w.act_dtype)
    cache = m2.Cache(shape, w.num_slots)
    t = TI.layer_tensors(w)
    ssm = m2.SSMParams(t["A_log"], t["dt_bias"], t["D"])
    conv = m2.ConvParams(t["conv_w"], t["conv_b"], 1)
    T = w.seqlen
    d = TI.step_tensors(w, 0, rows=w.batch * T)
    xr = d["xBC"].view(w.batch, T, -1)
    dt = d["dt"].view(w.batch, T, -1)
    z = d["z"].view(w.batch, T, -1)
    xp = torch.empty(xr.shape, dtype=torch.float16, device="cuda")  # fp16 post-conv buffer
    y = torch.empty((w.batch, T, w.H * w.P), dtype=torch.bfloat16, device="cuda")

    def conv_step():
        m2.conv1d_update(cache, conv, xr, t["slots"], out=xp)

    def scan_step():
        m2.chunk_scan(cache, ssm, xp, dt, t["slots"], z=z, chunk_size=w.chunk, y=y)

    for _ in range(3):
        conv_step()
        scan_step()
    conv_us = statistics.median(_time_us(conv_step, flush, reps))
    scan_us = statistics.median(_time_us(scan_step, flush, reps))
    # the scan again, 12 launches back to back between one pair of events (no
    # flush: 893 MB of operands per launch against a 126 MB L2); an ncu capture
    # of these launches counts each launch's DRAM traffic including the
    # write-back of its own output
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(12):
        scan_step()
    e1.record(stream)
    e1.synchronize()
    scan_b2b_us = 1e3 * e0.elapsed_time(e1) / 12
    if cache.device_error() != 0:
        raise RuntimeError("device error word set during the prefill benchmark")
    tokens = w.batch * T
    hp, cd = w.H * w.P, w.conv_dim
    # scan algorithmic bytes: post-conv xBC, dt, z in; y out; final state out
    scan_bytes = tokens * (cd + w.H + hp + hp) * 2 + w.batch * w.H * w.P * w.N * 2
    conv_bytes = tokens * cd * 2 * 2 + w.batch * (w.K - 1) * cd * 2 * 2
    # SSD form with C.B^T shared by the heads of a group, per (sequence, chunk):
    # G * 2Q^2N + H * (2Q^2P + 2QNP (C.S^T) + 2QNP (state increment))
    chunks = w.batch * (T // w.chunk)
    q = w.chunk
    alg_flops = chunks * (w.G * 2 * q * q * w.N + w.H * (2 * q * q * w.P + 4 * q * w.N * w.P))
    exec_flops = chunks * w.H * (2 * q * q * w.N + 2 * q * q * w.P + 4 * q * w.N * w.P)
    return {
        "workload": "prefill: 8 seqs x 2048 tokens, Nemotron-H layer, bf16, zero initial state",
        "conv_us": conv_us, "conv_GBs": conv_bytes / conv_us / 1e3,
        "conv_frac_hbm": conv_bytes / conv_us / 1e3 / peak_gbs,
        "scan_us": scan_us, "scan_b2b_us": scan_b2b_us, "scan_bytes": scan_bytes,
        "scan_GBs": scan_bytes / scan_us / 1e3,
        "scan_frac_hbm": scan_bytes / scan_us / 1e3 / peak_gbs,
        "scan_alg_flops": alg_flops, "scan_exec_flops": exec_flops,
        "scan_alg_TFLOPs": alg_flops / scan_us / 1e6,
        "scan_frac_fp16_tensor_peak": alg_flops / scan_us / 1e6 / peak_tflops,
        "tokens_per_s": tokens / (scan_us + conv_us) * 1e6,
    }


def measure_longprompt(flush, peak_gbs: float, reps: int = 10, T: int = 16384) -> dict:
    """One long prompt (16384 tokens, the long-prompt regime of mixed serving)
    through the Nemotron-H layer: the prefill conv (fp16 post-conv buffer),
    then the variable-length scan. Its 128 (sequence, head) pairs run one CTA
    per head: a split into segments does not pay at this head count."""
    import torch
    import mamba_recurrent_state_b200 as m2
    import m2synth as S
    from m2synth import torch_inputs as TI
    from m2synth import workloads as W
    w = W.Workload(405, "longprompt", 128, 64, 128, 8, 4, S.BF16, S.BF16, 4, 1, seqlen=T, chunk=128)
    shape = m2.Shape(w.H, w.P, w.N, w.G, w.K, w.state_dtype, w.act_dtype)
    cache = m2.Cache(shape, w.num_slots)
    t = TI.layer_tensors(w)
    ssm = m2.SSMParams(t["A_log"], t["dt_bias"], t["D"])
    conv = m2.ConvParams(t["conv_w"], t["conv_b"], 1)
    d = TI.step_tensors(w, 0, rows=T)
    xr = d["xBC"].view(1, T, -1)
    xp = torch.empty(xr.shape, dtype=torch.float16, device="cuda")
    y = torch.empty((T, w.H * w.P), dtype=torch.bfloat16, device="cuda")
    cu = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    slots = t["slots"][:1]

    def conv_step():
        m2.conv1d_update(cache, conv, xr, slots, out=xp)

    def scan_step():
        m2.chunk_scan_varlen(cache, ssm, xp.view(T, -1), d["dt"], cu, slots, max_seqlen=T, z=d["z"], y=y)

    for _ in range(3):
        conv_step()
        scan_step()
    conv_us = statistics.median(_time_us(conv_step, flush, reps))
    scan_us = statistics.median(_time_us(scan_step, flush, reps))
    if cache.device_error() != 0:
        raise RuntimeError("device error word set during the long-prompt benchmark")
    hp, cd = w.H * w.P, w.conv_dim
    scan_bytes = T * (cd + w.H + hp + hp) * 2 + w.H * w.P * w.N * 2
    return {
        "workload": f"one {T}-token prompt, Nemotron-H layer, bf16, fp16 post-conv buffer",
        "conv_us": conv_us, "scan_us": scan_us, "scan_bytes": scan_bytes,
        "scan_GBs": scan_bytes / scan_us / 1e3, "scan_frac_hbm": scan_bytes / scan_us / 1e3 / peak_gbs,
        "tokens_per_s": T / (conv_us + scan_us) * 1e6,
    }


def measure_decode_norm(peak_gbs: float, reps: int = 200) -> dict:
    """The workload-1 decode step with the gated RMSNorm fused
    (m2_state_update_norm), rotating the four disjoint slot sets back to back
    like the headline loop, against the same loop without the norm."""
    import torch
    import mamba_recurrent_state_b200 as m2
    from m2synth import torch_inputs as TI
    from m2synth import workloads as W
    w = W.WORKLOADS[1]
    shape = m2.Shape(w.H, w.P, w.N, w.G, w.K, w.state_dtype, w.act_dtype)
    cache = m2.Cache(shape, w.num_slots)
    TI.fill_caches(w, cache.ssm, cache.conv)
    t = TI.layer_tensors(w)
    ssm = m2.SSMParams(t["A_log"], t["dt_bias"], t["D"])
    conv = m2.ConvParams(t["conv_w"], t["conv_b"], 1)
    norm = m2.NormParams(TI.to_torch(W.norm_weight(w), w.act_dtype), 1e-5)
    sets = [torch.from_numpy(x).to("cuda") for x in W.slot_sets(w)]
    inputs = [TI.step_tensors(w, s) for s in range(len(sets))]
    y = torch.empty((w.batch, w.H * w.P), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()
    out = {}
    for tag, nrm in (("plain", None), ("norm", norm)):
        def step(i):
            inp = inputs[i % len(sets)]
            m2.state_update(cache, ssm, inp["xBC"], inp["dt"], sets[i % len(sets)], z=inp["z"], conv=conv,
                            y=y, norm=nrm)
        for i in range(8):
            step(i)
        a = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
        b = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
        torch.cuda.synchronize()
        for i in range(reps):
            a[i].record(stream)
            step(i)
            b[i].record(stream)
        torch.cuda.synchronize()
        out[f"{tag}_us"] = statistics.median(x.elapsed_time(e) * 1e3 for x, e in zip(a, b))
    if cache.device_error() != 0:
        raise RuntimeError("device error word set during the norm benchmark")
    bytes_ = W.bytes_per_unit(w) * w.batch + W.param_bytes_per_launch(w) + w.H * w.P * 2
    out["norm_GBs"] = bytes_ / out["norm_us"] / 1e3
    out["norm_frac_hbm"] = out["norm_GBs"] / peak_gbs
    out["workload"] = "workload-1 decode step + fused gated RMSNorm (1024-channel groups, eps 1e-5)"
    return out


def measure_multi(peak_gbs: float, reps: int = 50, T: int = 4) -> dict:
    """Multi-token decode (speculative drafts): the Nemotron-H layer, 64
    sequences x T = 4 draft tokens, every token's state stored into its own
    slot (a cache of 64 + 64 T slots)."""
    import torch
    import mamba_recurrent_state_b200 as m2
    import m2synth as S
    from m2synth import torch_inputs as TI
    from m2synth import workloads as W
    w = W.WORKLOADS[1]
    batch = w.batch
    slots_n = batch * (T + 1)
    shape = m2.Shape(w.H, w.P, w.N, w.G, w.K, w.state_dtype, w.act_dtype)
    cache = m2.Cache(shape, slots_n)
    t = TI.layer_tensors(w)
    ssm = m2.SSMParams(t["A_log"], t["dt_bias"], t["D"])
    conv = m2.ConvParams(t["conv_w"], t["conv_b"], 1)
    d = TI.step_tensors(w, 0, rows=batch * T)
    x, dt, z = (d[k].view(batch, T, -1) for k in ("xBC", "dt", "z"))
    slots = torch.arange(batch, dtype=torch.int32, device="cuda")
    dest = (batch + torch.arange(batch * T, dtype=torch.int32, device="cuda")).view(batch, T)
    y = torch.empty((batch, T, w.H * w.P), dtype=torch.bfloat16, device="cuda")
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device="cuda")
    fn = lambda: m2.state_update_multi(cache, ssm, conv, x, dt, slots, dest, z=z, y=y)
    for _ in range(3):
        fn()
    us = statistics.median(_time_us(fn, flush, reps))
    if cache.device_error() != 0:
        raise RuntimeError("device error word set during the multi-token benchmark")
    state = w.H * w.P * w.N * 2
    bytes_ = batch * (state * (1 + T) + T * (w.conv_dim * 2 * 4 + w.H * 2 + 2 * w.H * w.P * 2))
    return {"workload": f"Nemotron-H layer, {batch} sequences x {T} draft tokens, every token's state stored",
            "us": us, "GBs": bytes_ / us / 1e3, "frac_hbm": bytes_ / us / 1e3 / peak_gbs,
            "tokens_per_s": batch * T / us * 1e6}


def measure_stack48(flush, reps: int = 10) -> dict:
    """Workload 2: one decode token for 384 sequences through 48 layers
    (36 GiB of bf16 state), one CUDA graph of 48 fused launches per token."""
    import torch
    import mamba_recurrent_state_b200 as m2
    from m2synth import torch_inputs as TI
    from m2synth import workloads as W
    w = W.WORKLOADS[2]
    shape = m2.Shape(w.H, w.P, w.N, w.G, w.K, w.state_dtype, w.act_dtype)
    caches, objs, inps = [], [], []
    for layer in range(w.layers):
        c = m2.Cache(shape, w.num_slots)
        TI.fill_caches(w, c.ssm, c.conv, layer)
        caches.append(c)
        t = TI.layer_tensors(w, layer)
        objs.append((t, m2.SSMParams(t["A_log"], t["dt_bias"], t["D"]),
                     m2.ConvParams(t["conv_w"], t["conv_b"], 1)))
        inps.append(TI.step_tensors(w, 0, layer))
    ys = [torch.empty((w.batch, w.H * w.P), dtype=torch.bfloat16, device="cuda") for _ in caches]
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for layer in range(w.layers):
            t, ssm, conv = objs[layer]
            m2.state_update(caches[layer], ssm, inps[layer]["xBC"], inps[layer]["dt"], t["slots"],
                            z=inps[layer]["z"], conv=conv, y=ys[layer])
    for _ in range(3):
        g.replay()
    token_us = statistics.median(_time_us(g.replay, flush, reps))
    for c in caches:
        if c.device_error() != 0:
            raise RuntimeError("device error word set during the 48-layer benchmark")
    del g
    bytes_tok = w.layers * (W.bytes_per_unit(w) * w.batch + W.param_bytes_per_launch(w))
    return {"workload": "48 layers x 384 sequences, one token, CUDA graph of 48 launches",
            "per_token_us": token_us, "per_layer_us": token_us / w.layers,
            "bytes_per_token": bytes_tok, "GBs": bytes_tok / token_us / 1e3,
            "seq_layer_steps_per_s": w.layers * w.batch / token_us * 1e6}


def measure_fp32_23l(peak_gbs: float) -> dict:
    """Workload 3: the fp32-state mixer (H=64, P=64, N=128, G=8, 2 MiB of fp32
    state per layer per sequence), 23 layers of 512-slot caches, 128 sequences,
    64 consecutive decode steps carried in place. One step is the 23 fused
    launches of the layer loop, captured once as a CUDA graph and replayed per
    step; every step is timed with CUDA events. A layer's 128 x 2 MiB of state
    (256 MiB) exceeds L2 (126 MB), and a slot comes back only after the 22
    other layers, so no flush is needed."""
    import torch
    import mamba_recurrent_state_b200 as m2
    from m2synth import torch_inputs as TI
    from m2synth import workloads as W
    w = W.WORKLOADS[3]
    shape = m2.Shape(w.H, w.P, w.N, w.G, w.K, w.state_dtype, w.act_dtype)
    caches, objs, ys = [], [], []
    inputs = [[TI.step_tensors(w, s, layer) for layer in range(w.layers)] for s in range(2)]
    staged = {k: [torch.empty_like(inputs[0][layer][k]) for layer in range(w.layers)]
              for k in ("xBC", "dt", "z")}
    for layer in range(w.layers):
        c = m2.Cache(shape, w.num_slots)
        TI.fill_caches(w, c.ssm, c.conv, layer)
        caches.append(c)
        t = TI.layer_tensors(w, layer)
        objs.append((t, m2.SSMParams(t["A_log"], t["dt_bias"], t["D"]),
                     m2.ConvParams(t["conv_w"], t["conv_b"], 1)))
        ys.append(torch.empty((w.batch, w.H * w.P), dtype=torch.bfloat16, device="cuda"))

    def stage(step):  # the step's inputs into the graph's buffers (outside the timed region)
        for layer in range(w.layers):
            for k in ("xBC", "dt", "z"):
                staged[k][layer].copy_(inputs[step % 2][layer][k])

    stage(0)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for layer in range(w.layers):
            t, ssm, conv = objs[layer]
            m2.state_update(caches[layer], ssm, staged["xBC"][layer], staged["dt"][layer], t["slots"],
                            z=staged["z"][layer], conv=conv, y=ys[layer])
    stream = torch.cuda.current_stream()
    for i in range(3):
        stage(i)
        g.replay()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(w.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(w.steps)]
    torch.cuda.synchronize()
    for i in range(w.steps):
        stage(i)
        starts[i].record(stream)
        g.replay()
        ends[i].record(stream)
    torch.cuda.synchronize()
    step_us = [1e3 * a.elapsed_time(b) for a, b in zip(starts, ends)]
    for c in caches:
        if c.device_error() != 0:
            raise RuntimeError("device error word set during the fp32-state benchmark")
    del g
    bytes_step = w.layers * (W.bytes_per_unit(w) * w.batch + W.param_bytes_per_launch(w))
    mean_us = statistics.mean(step_us)
    return {"workload": "fp32 state (H=64 P=64 N=128 G=8, 2 MiB per layer per sequence), 23 layers x "
                        "128 sequences in 512-slot caches, 64 steps in place, one CUDA graph of 23 "
                        "launches per step",
            "steps": w.steps, "ms_per_step_mean": mean_us / 1e3,
            "ms_per_step_median": statistics.median(step_us) / 1e3,
            "bytes_per_step": bytes_step, "GBs": bytes_step / mean_us / 1e3,
            "frac_hbm": bytes_step / mean_us / 1e3 / peak_gbs,
            "seq_layer_steps_per_s": w.layers * w.batch / mean_us * 1e6}


def measure_t1_ab(reps: int = 200) -> dict:
    """One decode token of the workload-1 layer (Nemotron-H, 64 sequences,
    bf16) taken two ways from the same cache: the decode step (one fused
    launch: conv tap and roll, state update) against the prefill path at
    T = 1 (the prefill conv writing its fp16 post-conv buffer, then the chunk
    scan with the cached state as its initial state). Steps rotate over the
    four disjoint 64-slot sets like the headline loop; each way is timed as
    one region per step with CUDA events. This library's scan keeps its chunk
    state on chip and takes no scratch memory, so the prefill path here is two
    launches and no allocation, not the five launches with scratch of the
    chunk-scan-at-decode design it is compared with on the pages."""
    import torch
    import mamba_recurrent_state_b200 as m2
    from m2synth import torch_inputs as TI
    from m2synth import workloads as W
    w = W.WORKLOADS[1]
    shape = m2.Shape(w.H, w.P, w.N, w.G, w.K, w.state_dtype, w.act_dtype)
    cache = m2.Cache(shape, w.num_slots)
    TI.fill_caches(w, cache.ssm, cache.conv)
    t = TI.layer_tensors(w)
    ssm = m2.SSMParams(t["A_log"], t["dt_bias"], t["D"])
    conv = m2.ConvParams(t["conv_w"], t["conv_b"], 1)
    sets = [torch.from_numpy(x).to("cuda") for x in W.slot_sets(w)]
    inputs = [TI.step_tensors(w, s) for s in range(len(sets))]
    y = torch.empty((w.batch, w.H * w.P), dtype=torch.bfloat16, device="cuda")
    xp = torch.empty((w.batch, 1, w.conv_dim), dtype=torch.float16, device="cuda")
    ones = torch.ones(w.batch, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def decode(i):
        inp = inputs[i % len(sets)]
        m2.state_update(cache, ssm, inp["xBC"], inp["dt"], sets[i % len(sets)], z=inp["z"], conv=conv, y=y)

    def prefill_t1(i):
        inp = inputs[i % len(sets)]
        s = sets[i % len(sets)]
        m2.conv1d_update(cache, conv, inp["xBC"].view(w.batch, 1, -1), s, out=xp)
        m2.chunk_scan(cache, ssm, xp, inp["dt"].view(w.batch, 1, -1), s, z=inp["z"].view(w.batch, 1, -1),
                      chunk_size=128, has_initial_state=ones, y=y.view(w.batch, 1, -1))

    out = {}
    for tag, fn in (("decode", decode), ("prefill_path_t1", prefill_t1)):
        for i in range(8):
            fn(i)
        a = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
        b = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
        torch.cuda.synchronize()
        for i in range(reps):
            a[i].record(stream)
            fn(i)
            b[i].record(stream)
        torch.cuda.synchronize()
        out[f"{tag}_us"] = statistics.median(x.elapsed_time(e) * 1e3 for x, e in zip(a, b))
    if cache.device_error() != 0:
        raise RuntimeError("device error word set during the T = 1 comparison")
    out.update({
        "workload": "one decode token, Nemotron-H layer, 64 sequences in 256 slots, bf16",
        "decode_launches": 1, "prefill_path_launches": 2,
        "decode_scratch_bytes": 0, "prefill_path_scratch_bytes": 0,
        "prefill_path_buffer_bytes": w.batch * w.conv_dim * 2,
        "ratio": out["prefill_path_t1_us"] / out["decode_us"],
    })
    return out


def run_ours(args, world, rank, local):
    import torch
    import mamba_recurrent_state_b200 as m2
    from m2synth import torch_inputs as TI
    from m2synth import workloads as W

    w = W.WORKLOADS[1]
    shape = m2.Shape(w.H, w.P, w.N, w.G, w.K, w.state_dtype, w.act_dtype)
    cache = m2.Cache(shape, w.num_slots)
    TI.fill_caches(w, cache.ssm, cache.conv)
    t = TI.layer_tensors(w)
    ssm = m2.SSMParams(t["A_log"], t["dt_bias"], t["D"])
    conv = m2.ConvParams(t["conv_w"], t["conv_b"], 1)
    rotate = args.l2 == "rotate"
    slot_sets = [torch.from_numpy(x).to("cuda") for x in W.slot_sets(w)] if rotate else [t["slots"]]
    n_sets = 4  # distinct input sets (and, rotating, disjoint slot sets)
    inputs = [TI.step_tensors(w, s) for s in range(n_sets)]
    y = torch.empty((w.batch, w.H * w.P), dtype=torch.bfloat16, device="cuda")
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    def pre_step():
        if not rotate:
            flush.zero_()

    def step(i):
        inp = inputs[i % n_sets]
        m2.state_update(cache, ssm, inp["xBC"], inp["dt"], slot_sets[i % len(slot_sets)], z=inp["z"],
                        conv=conv, y=y)

    for i in range(max(args.warmup, n_sets)):
        pre_step()
        step(i)
    torch.cuda.synchronize()

    # ---- device-resident timed region. Rotating slot sets (the default): the K
    # steps run back to back, as a layer loop would issue them, between one pair
    # of CUDA events. With --l2 flush every step is bracketed by its own events
    # and the flush before it stays outside them.
    sampler = ClockSampler(local)
    sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    t_begin = time.monotonic()
    if rotate:
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for i in range(args.steps):
            step(i)
        ev1.record(stream)
        torch.cuda.synchronize()
        local_ms = ev0.elapsed_time(ev1)
    else:
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        for i in range(args.steps):
            pre_step()
            starts[i].record(stream)
            step(i)
            ends[i].record(stream)
        torch.cuda.synchronize()
        local_ms = sum(s_.elapsed_time(e_) for s_, e_ in zip(starts, ends))
    t_end = time.monotonic()
    barrier(world)
    clocks = sampler.stop(t_begin, t_end)
    value, total_ms = job_throughput(w.batch * args.steps, local_ms, world)
    if cache.device_error() != 0:
        raise RuntimeError("device error word set during the benchmark")
    # for context: the same step bracketed by its own pair of events (the
    # events and the launch gap between steps are then inside every figure)
    nb = min(args.steps, 200)
    sb = [torch.cuda.Event(enable_timing=True) for _ in range(nb)]
    eb = [torch.cuda.Event(enable_timing=True) for _ in range(nb)]
    for i in range(nb):
        pre_step()
        sb[i].record(stream)
        step(i)
        eb[i].record(stream)
    torch.cuda.synchronize()
    bracketed_us = statistics.median(1e3 * a_.elapsed_time(b_) for a_, b_ in zip(sb, eb))

    # ---- end to end through the C ABI with host buffers: every step copies its
    # inputs from pinned host memory to the device, runs the step and copies y
    # back to pinned host memory, all inside one C call (m2_state_update_host).
    # A step's xBC, z and dt sit back to back in one pinned buffer and cross
    # PCIe as one copy; y comes back as one copy. The library's staging ring of
    # four device buffers and two copy streams lets the inputs of later steps
    # and the y of earlier ones cross PCIe while a step computes. The timed
    # region is the whole K-step loop, from the first input copy to the last y
    # landing in host memory (CUDA events); the host's own issue time for the
    # loop is reported beside it.
    import ctypes
    ring = 4
    parts = [("xBC", inputs[0]["xBC"]), ("z", inputs[0]["z"]), ("dt", inputs[0]["dt"])]
    offs, off = {}, 0
    for k, v in parts:
        offs[k] = off
        off += (v.numel() * v.element_size() + 255) // 256 * 256
    packed_bytes = off
    host_in = []
    for inp in inputs:
        hb = torch.empty(packed_bytes, dtype=torch.uint8).pin_memory()
        for k, v in parts:
            n = v.numel() * v.element_size()
            hb[offs[k]:offs[k] + n].copy_(inp[k].contiguous().view(torch.uint8).view(-1).cpu())
        host_in.append(hb)
    host_y = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(ring)]
    h2d = sum(v.numel() * v.element_size() for _, v in parts)  # bytes of the step's inputs
    d2h = host_y[0].numel() * host_y[0].element_size()
    stage = m2.HostStage(ring, packed_bytes, d2h)
    L = m2.lib()
    step_host, join = L.m2_state_update_host, L.m2_host_stage_join
    sp, cp = ssm.c(), conv.c()
    cache_ref, sp_ref, cp_ref = ctypes.byref(cache.c), ctypes.byref(sp), ctypes.byref(cp)
    hp, cd = w.H * w.P, w.conv_dim
    set_ptrs = [ss.data_ptr() for ss in slot_sets]
    stream_ptr = stream.cuda_stream
    in_ptr = [hb.data_ptr() for hb in host_in]
    hy_ptr = [hy.data_ptr() for hy in host_y]
    off_x, off_dt, off_z = offs["xBC"], offs["dt"], offs["z"]

    def e2e_loop(n, t_start=None, t_end=None):
        if t_start is not None:
            t_start.record(stream)
        for i in range(n):
            st = step_host(stage.ptr, cache_ref, sp_ref, cp_ref, w.batch, in_ptr[i % n_sets], off_x, cd, off_dt,
                           w.H, off_z, hp, hy_ptr[i % ring], hp, set_ptrs[i % len(set_ptrs)], stream_ptr)
            if st != m2.M2_OK:
                raise m2.M2Error(st, "m2_state_update_host")
        if join(stage.ptr, stream_ptr) != m2.M2_OK:
            raise m2.M2Error(m2.M2_ERR_CUDA, "m2_host_stage_join")
        if t_end is not None:
            t_end.record(stream)

    e2e_loop(max(args.warmup, ring))
    torch.cuda.synchronize()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    h0 = time.perf_counter()
    e2e_loop(args.steps, e_start, e_end)
    host_issue_s = time.perf_counter() - h0
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = e_start.elapsed_time(e_end)
    stage.close()
    e2e_value, _ = job_throughput(w.batch * args.steps, e2e_ms, world)
    # the link itself on this machine: one step's packed inputs host -> device and
    # its y device -> host, each timed alone (CUDA events on a copy stream)
    dev_in = torch.empty(packed_bytes, dtype=torch.uint8, device="cuda")
    dev_y = torch.empty_like(y)
    s_copy = torch.cuda.Stream()

    def link_us(copy, strm, reps=20):
        with torch.cuda.stream(strm):
            for _ in range(3):
                copy()
            a_ = torch.cuda.Event(enable_timing=True)
            b_ = torch.cuda.Event(enable_timing=True)
            a_.record(strm)
            for _ in range(reps):
                copy()
            b_.record(strm)
        torch.cuda.synchronize()
        return 1e3 * a_.elapsed_time(b_) / reps
    h2d_us = link_us(lambda: dev_in.copy_(host_in[0], non_blocking=True), s_copy)
    d2h_us = link_us(lambda: host_y[0].copy_(dev_y, non_blocking=True), s_copy)
    bytes_per_launch = W.bytes_per_unit(w) * w.batch + W.param_bytes_per_launch(w)
    avg_s = local_ms / args.steps / 1e3
    achieved = bytes_per_launch / avg_s / 1e9
    peak, peak_kind = measured_peaks()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded generators, random-init mixer parameters)",
        "config": {"workload": WORKLOAD, "batch_per_gpu": w.batch, "num_slots": w.num_slots,
                   "state_bytes_per_seq": w.state_bytes_per_slot(),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": ("not flushed: steps rotate over 4 disjoint 64-slot sets, 536 MB of state "
                          "between reuses of a slot (L2 126 MB), back to back") if rotate
                         else "flushed (512 MiB write) before every timed step, slot set 0"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": profiled_traffic(),
                     "peak_source": f"{peak_kind} hbm_gbs", "kernel": "m2 state_update (fused)",
                     "algorithmic_bytes_per_launch": bytes_per_launch,
                     "kernel_us_avg": 1e6 * avg_s,
                     "timing": ("K launches back to back between one pair of CUDA events" if rotate
                                else "every launch between its own pair of CUDA events"),
                     "event_bracketed_us_median": bracketed_us},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "us_per_step": 1e3 * e2e_ms / args.steps,
                "host_issue_us_per_step": 1e6 * host_issue_s / args.steps,
                "link": {"h2d_us_per_step": h2d_us, "h2d_GBs": packed_bytes / h2d_us / 1e3,
                         "d2h_us_per_step": d2h_us, "d2h_GBs": d2h / d2h_us / 1e3,
                         "note": "each direction timed alone on this box; the steps overlap them with "
                                 "the kernel, so the slowest of the three bounds us_per_step"},
                "how": "m2_state_update_host through the C ABI, one call per step: pinned host "
                       "buffer (xBC|z|dt packed) -> device, one copy; the fused step; y -> pinned "
                       "host, one copy; the library's staging ring of 4 device buffers and two copy "
                       "streams overlaps the copies with the steps"},
        "gpu_launches": args.steps,  # one fused decode launch per timed step (device-resident loop)
        "clocks": clocks,
    }
    sections = set(args.sections.split(","))
    del cache, inputs, host_in
    torch.cuda.empty_cache()
    if "prefill" in sections:
        tpeak, tkind = measured_tensor_peak()
        line["prefill"] = measure_prefill(flush, peak, tpeak)
        line["prefill"]["tensor_peak"] = f"{tpeak} TFLOP/s ({tkind} bf16_tflops)"
    if "norm" in sections:
        line["decode_norm"] = measure_decode_norm(peak)
    if "multi" in sections:
        line["multi_token"] = measure_multi(peak)
    if "longprompt" in sections:
        line["longprompt"] = measure_longprompt(flush, peak)
    if "stack48" in sections:
        line["stack48"] = measure_stack48(flush)
    if "fp32_23l" in sections:
        line["fp32_state_23l"] = measure_fp32_23l(peak)
    if "t1_ab" in sections:
        line["t1_ab"] = measure_t1_ab()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup()
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
