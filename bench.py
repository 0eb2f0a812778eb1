#!/usr/bin/env python
"""Benchmark of the YaRN-RoPE attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl yarn|reference]

One step is one prefill of the Llama-3-8B-shaped GQA workload at 128K (B=1, Hq=32,
Hkv=8, d=128, T=131072, causal, YaRN base 5e5, L_train 8192, s=16): the
rotated-key pass plus the attention kernel, inputs resident in HBM.  It is the
largest single-GPU prefill configuration; the headline is prefill TFLOP/s with
causal FLOPs counted (4 d Hq B sum_m |visible(m)|).  The same run times the other
workloads and puts them at the end of the line: the method/structure sweep at
64K, the chunked prefill, ring attention over emulated ranks, the 16K MHA
prefill, and last the single-token decode workload (B=8, Hq=32, Hkv=8, d=128,
cache lengths U[32768,131072]) as KV-read GB/s.

For N > 1 (launched with torch.distributed.run) every rank runs the same
workload as an independent replica; NCCL carries only the barrier and the
max-over-ranks of the timings.  --impl reference times the fp64 CPU oracle on
a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
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

from yarn_position_scaling_b200 import metrics, synth  # noqa: E402

L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["yarn", "reference"], default="yarn")
    ap.add_argument("--decode-steps", type=int, default=None)
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the sweep, chunk, ring and 16K prefill workloads")
    ap.add_argument("--headline", default="llama3_8b_128k_gqa_prefill",
                    help="prefill workload of the headline (a name from synth.ALL)")
    ap.add_argument("--other-steps", type=int, default=3)
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="sequences in the decode workload (default 8; smaller for profiling)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {
    "prefill_attn_kernel<128, false>": ["prefill_sm100.cuh"],
    "kv_prep_kernel<false>": ["kvprep_sm100.cuh"],
    "decode_split_kernel<128, 1>": ["decode_sm100.cuh"],
}


def kernel_source_sha(kernel: str) -> str:
    """Hash of the sources that define `kernel` (its own header plus the shared PTX and
    status helpers)."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel] + ["sm100_ptx.cuh", "yr_status.cuh"]:
        with open(os.path.join(ROOT, "yarn_position_scaling_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the last ncu capture of it, or None when its
    sources changed since that capture (profiles/traffic.json keeps their hash)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        rec = t[kernel]
        if rec["source_sha"] != kernel_source_sha(kernel):
            return None
        return float(rec["dram_read"] + rec["dram_write"])
    except Exception:
        return None


class Dist:
    """One process per GPU (torch.distributed.run).  The collective carries only the
    barrier and the max of the timings: the replicas share no data."""

    def __init__(self, n_gpus: int, backend: str = "nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        if self.world != n_gpus:
            raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={self.world}: launch N>1 with "
                             "torch.distributed.run")
        self.pg = None
        self.device = "cuda" if backend == "nccl" else "cpu"
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {}
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                kw["device_id"] = torch.device("cuda", self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.dist = dist
            self.pg = True

    def barrier(self):
        if self.pg:
            self.dist.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.dist.barrier()
            self.dist.destroy_process_group()
            self.pg = None


def throughput(units_per_step: float, steps: int, max_ms: float, world: int, scale: float):
    """Whole-job rate: the units every rank processed over the slowest rank's time."""
    return world * units_per_step * steps / (max_ms * 1e-3) / scale


class Clocks:
    """nvidia-smi samples of this GPU during a timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None

    def start(self):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        self.file.close()
        os.unlink(self.file.name)
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                power.append(float(r[3]))
            except (ValueError, IndexError):
                continue
            for name, val in zip(names, r[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        loaded = [s for s, p in zip(sm, power) if p > 300.0] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


def time_events(fn, steps, stream):
    """Run fn(step) `steps` times; fn returns a list of (start, end) event pairs per kernel."""
    starts = torch.cuda.Event(enable_timing=True)
    ends = torch.cuda.Event(enable_timing=True)
    per_kernel = []
    torch.cuda.synchronize()
    starts.record(stream)
    for i in range(steps):
        per_kernel.append(fn(i))
    ends.record(stream)
    torch.cuda.synchronize()
    total = starts.elapsed_time(ends)
    kernel_ms = [sum(a.elapsed_time(b) for a, b in ev) for ev in zip(*per_kernel)]
    return total, kernel_ms


# ------------------------------------------------------------------ CPU oracle
_CPU_INPUTS = {}


def _cpu_inputs(w):
    if w.name not in _CPU_INPUTS:
        q, k, v = synth.prefill_inputs(w, "cpu")
        _CPU_INPUTS[w.name] = tuple(t.view(torch.int16).numpy().view(np.uint16) for t in (q, k, v))
    return _CPU_INPUTS[w.name]


def oracle_sample(w, seconds: float, seed: int = 0):
    """Time the fp64 oracle on query rows of workload w drawn until ~`seconds` of CPU work;
    returns (flops_done, wall_s, threads, description)."""
    import oracle
    rng = np.random.default_rng(seed)
    T, d = w.T, w.d
    qb, kb, vb = _cpu_inputs(w)
    th, _, ss = oracle.rope_theta(d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    counts = metrics.visible_counts(T, w.causal, w.window, w.n_sink)
    done_flops, done_rows, wall = 0.0, 0, 0.0
    batch = 16
    while wall < seconds:
        h = int(rng.integers(0, w.Hq))
        ms = rng.integers(0, T, size=batch)
        rows = (h * T + ms).astype(np.int64)
        t0 = time.perf_counter()
        oracle.attn_rows(qb, kb, vb, th, ss, w.causal, w.window, w.n_sink, rows=rows)
        wall += time.perf_counter() - t0
        done_flops += float(4.0 * d * counts[ms].sum())
        done_rows += batch
        batch = min(batch * 2, 256)
    threads = int(os.environ.get("OMP_NUM_THREADS", len(os.sched_getaffinity(0))))
    desc = (f"{done_rows} query rows of {w.name} drawn uniformly over positions, "
            f"one head per batch of rows; keys rotated on the fly by the oracle; "
            f"FLOPs counted as 4*d*|visible(m)| per row")
    return done_flops, wall, threads, desc


def workload_config(w, n: int) -> dict:
    """The `config` of the JSON line for prefill workload w on n GPUs (both arms)."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "T": w.T,
            "method": w.method, "base": w.base, "L_train": w.L_train, "scale": w.scale,
            "causal": w.causal, "window": w.window, "n_sink": w.n_sink, "io_dtype": "bf16",
            "mma_operands": "fp16", "accumulate": "fp32", "parallelism": f"replicas x{n}",
            "l2": "no flush: q+k+v+o = %.0f MB per step > 126 MB L2" %
                  ((2 * w.B * w.Hq + 2 * w.B * w.Hkv) * w.T * w.d * 2 / 2 ** 20),
            "step": "yr_prefill_prepare_kv + yr_prefill_attend (= yr_attn_prefill)"}


def reference_arm(args, dist: Dist):
    w = synth.ALL[args.headline]
    line = {"impl": "reference"}
    if dist.rank != 0:
        return None
    steps, warm = args.steps, args.warmup
    per_step = min(max(0.2, 120.0 / max(1, steps + warm)), 20.0)
    for _ in range(warm):
        oracle_sample(w, min(per_step, 2.0), seed=1)
    flops, wall = 0.0, 0.0
    desc, threads = "", 0
    for s in range(steps):
        f, t, threads, desc = oracle_sample(w, per_step, seed=100 + s)
        flops += f
        wall += t
    value = flops / wall / 1e12
    line.update({
        "metric": "causal YaRN-RoPE attention prefill TFLOP/s", "value": value, "unit": "TFLOP/s",
        "n_gpus": 1, "steps": steps, "warmup": warm, "ms_per_step": wall / steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic N(0,1) bf16 inputs, seeded",
        "config": workload_config(w, 1),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"each step ~{per_step:.1f}s of oracle work: {desc}"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    })
    return line


# ------------------------------------------------------------------- GPU arm
def prefill_bench(w, steps, warmup, stream, pairs="interleaved"):
    from yarn_position_scaling_b200 import api
    q, k, v = synth.prefill_inputs(w, "cuda")
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta,
                              pairs=pairs)
    ws = torch.empty(api.attn_prefill_workspace_bytes(w.B, w.Hkv, w.T, w.d), dtype=torch.uint8,
                     device="cuda")
    o = torch.empty_like(q)

    def step(_):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        api.prefill_prepare_kv(k, v, tab, ws, stream=stream)
        e[1].record(stream)
        api.prefill_attend(q, w.Hkv, tab, ws, w.causal, w.window, w.n_sink, out=o, stream=stream)
        e[2].record(stream)
        return [(e[0], e[1]), (e[1], e[2])]

    for i in range(warmup):
        step(i)
    api.device_status(stream)
    return step, (q, k, v, o, ws, tab)


def decode_bench(w, steps, warmup, stream):
    from yarn_position_scaling_b200 import api
    qn, kn, vn, kc, vc, lens = synth.decode_inputs(w, "cuda")
    cl = lens.cuda()
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    ws = torch.empty(api.attn_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.d, w.T),
                     dtype=torch.uint8, device="cuda")
    o = torch.empty_like(qn)

    def step(_):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record(stream)
        api.attn_decode(qn, kn, vn, kc, vc, cl, tab, out=o, workspace=ws, stream=stream)
        e[1].record(stream)
        return [(e[0], e[1])]

    for i in range(warmup):
        step(i)
    api.device_status(stream)
    return step, lens.tolist()


def workload_prefill(w, steps, stream, dist, peak_t, warmup=2, pairs="interleaved"):
    """Prefill of one more workload: attention-kernel TFLOP/s with causal (and window/sink)
    FLOPs counted, and the whole step (rotated-key pass + attention)."""
    step, keep = prefill_bench(w, steps, warmup, stream, pairs)
    flops = metrics.prefill_flops(w.B, w.Hq, w.T, w.d, w.causal, w.window, w.n_sink)
    dist.barrier()
    total_ms, (prep_ms, attn_ms) = time_events(step, steps, stream)
    dist.barrier()
    from yarn_position_scaling_b200 import api
    api.device_status(stream)
    total_ms, attn_ms = dist.max(total_ms), dist.max(attn_ms)
    attn = flops / (attn_ms / steps * 1e-3) / 1e12
    del keep, step
    return {"method": w.method, "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv, "window": w.window,
            "n_sink": w.n_sink, "flops_per_step": flops, "steps": steps,
            "step_tflops": throughput(flops, steps, total_ms, dist.world, 1e12),
            "attn_kernel_tflops": attn, "attn_kernel_ms": attn_ms / steps,
            "frac_of_peak": attn / peak_t}


def chunk_bench(w, steps, stream, dist, peak_t):
    """Chunked prefill after a cached prefix: the whole yr_attn_prefill_chunk call (prefix
    and chunk laid out as fp16, chunk keys rotated and appended, attention) as causal
    TFLOP/s."""
    from yarn_position_scaling_b200 import api
    q, kn, vn, kc, vc = synth.chunk_inputs(w, "cuda")
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    ws = torch.empty(api.attn_prefill_workspace_bytes(w.B, w.Hkv, w.P0 + w.Tq, w.d),
                     dtype=torch.uint8, device="cuda")
    o = torch.empty_like(q)

    def step(_):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record(stream)
        api.attn_prefill_chunk(q, kn, vn, kc, vc, w.P0, tab, out=o, workspace=ws, stream=stream)
        e[1].record(stream)
        return [(e[0], e[1])]

    for i in range(2):
        step(i)
    api.device_status(stream)
    dist.barrier()
    total_ms, (call_ms,) = time_events(step, steps, stream)
    dist.barrier()
    api.device_status(stream)
    call_ms = dist.max(call_ms)
    flops = metrics.chunk_flops(w.B, w.Hq, w.d, w.P0, w.Tq)
    tf = flops / (call_ms / steps * 1e-3) / 1e12
    return {"P0": w.P0, "Tq": w.Tq, "Hq": w.Hq, "Hkv": w.Hkv, "T_max": w.T, "method": w.method,
            "flops_per_step": flops, "steps": steps, "call_ms": call_ms / steps,
            "call_tflops": tf, "frac_of_peak": tf / peak_t,
            "timed_over": "the whole call (prefix/chunk layout + attention launches)"}


def chunk_fp16cache_bench(w, Tq, steps, stream, dist, peak_t):
    """A short chunk after a long cached prefix, the serving loop's steady state: the fp16
    copy of the cache already holds the prefix, so a call writes only its own Tq rows,
    cuts each query block's keys into shares (split-KV) and merges them.  The whole
    yr_attn_prefill_chunk_fp16cache call, as causal TFLOP/s."""
    from yarn_position_scaling_b200 import api
    q, kn, vn, kc, vc = synth.chunk_inputs(w, "cuda", Tq=Tq, T_max=w.P0 + Tq)
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    k16, v16 = kc.to(torch.float16), vc.to(torch.float16)
    ws = torch.empty(api.attn_prefill_chunk_split_bytes(w.B, w.Hq, Tq, w.d), dtype=torch.uint8,
                     device="cuda")
    o = torch.empty_like(q)

    def step(_):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record(stream)
        api.attn_prefill_chunk_fp16cache(q, kn, vn, kc, vc, k16, v16, w.P0, w.P0, tab, out=o,
                                         workspace=ws, stream=stream)
        e[1].record(stream)
        return [(e[0], e[1])]

    for i in range(3):
        step(i)
    api.device_status(stream)
    dist.barrier()
    total_ms, (call_ms,) = time_events(step, steps, stream)
    dist.barrier()
    api.device_status(stream)
    call_ms = dist.max(call_ms)
    flops = metrics.chunk_flops(w.B, w.Hq, w.d, w.P0, Tq)
    tf = flops / (call_ms / steps * 1e-3) / 1e12
    return {"tflops": tf, "frac": tf / peak_t, "ms": call_ms / steps}


def ring_bench(w, world, steps, stream, dist, peak_t, layout="contiguous"):
    """Ring attention over `world` ranks emulated in one process on this GPU: every rank's
    block kernels (keys prepared at their positions, one attention call per visible
    block, fp32 partials folded by the log-sum-exp merge) run in turn, without the
    exchange.  Causal TFLOP/s of the whole sequence over the sum of all ranks' work, i.e.
    the single-GPU cost of the ring's compute."""
    from yarn_position_scaling_b200 import api, ring
    q, k, v = synth.prefill_inputs(w, "cuda")
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)

    def step(_):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        with torch.cuda.stream(stream):
            e[0].record(stream)
            ring.ring_prefill_emulated(q, k, v, tab, world, w.causal, w.window, w.n_sink,
                                       layout=layout)
            e[1].record(stream)
        return [(e[0], e[1])]

    for i in range(2):
        step(i)
    api.device_status(stream)
    dist.barrier()
    total_ms, (call_ms,) = time_events(step, steps, stream)
    dist.barrier()
    api.device_status(stream)
    call_ms = dist.max(call_ms)
    flops = metrics.prefill_flops(w.B, w.Hq, w.T, w.d, w.causal, w.window, w.n_sink)
    tf = flops / (call_ms / steps * 1e-3) / 1e12
    # causal work per rank in (query chunk, key chunk) pairs: the multi-GPU balance
    work = [len(ring.rank_pairs(r, world, layout, w.causal)) for r in range(world)]
    return {"ranks_emulated": world, "layout": layout,
            "rank_work_max_over_mean": max(work) / (sum(work) / world), "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv, "method": w.method,
            "flops_per_step": flops, "steps": steps, "call_ms": call_ms / steps,
            "call_tflops": tf, "frac_of_peak": tf / peak_t,
            "timed_over": "all ranks' block preparation, block attention and merge launches, "
                          "run in turn on one GPU (no exchange)"}


def e2e_prefill(w, steps, warmup, stream):
    """Through the C ABI's host-buffer entry point (yr_host_prefill_run, wrapped by
    `api.HostPrefill`): pinned host q, k, v in, the pinned host output out; the H2D copies,
    the kernels and the D2H copy of each (batch, KV-head group) unit overlap those of the
    other units."""
    from yarn_position_scaling_b200 import api
    qh, kh, vh = [t.pin_memory() for t in synth.prefill_inputs(w, "cpu")]
    oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    hp = api.HostPrefill(w.B, w.Hq, w.Hkv, w.T, w.d)

    def step(_):
        hp(qh, kh, vh, tab, w.causal, w.window, w.n_sink, out=oh)
        return []

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size()
    return step, h2d, d2h


def _r(x, nd=4):
    """Round for the JSON line (keeps it short enough for its tail to carry the
    per-workload results)."""
    if isinstance(x, float):
        return float(f"{x:.{nd}g}")
    if isinstance(x, dict):
        return {k: _r(v, nd) for k, v in x.items()}
    if isinstance(x, list):
        return [_r(v, nd) for v in x]
    return x


def main():
    args = parse()
    if args.impl == "reference":
        # CPU only: rank 0 runs the oracle, the other ranks exit at once without a
        # process group (nothing to synchronise).
        if int(os.environ.get("RANK", "0")) != 0:
            return

        class _Solo:
            rank = 0
        line = reference_arm(args, _Solo())
        print(json.dumps(line), flush=True)
        return
    dist = Dist(args.gpus)
    if not torch.cuda.is_available():
        raise SystemExit("no CUDA device: the benchmark needs a B200")
    from yarn_position_scaling_b200 import api
    api.load()
    torch.cuda.set_device(dist.local)
    stream = torch.cuda.current_stream()
    peaks, peak_src = load_peaks()
    n = dist.world
    wp, wd = synth.ALL[args.headline], synth.DECODE
    if args.decode_batch:
        import dataclasses
        wd = dataclasses.replace(wd, B=args.decode_batch)
    steps, warm = args.steps, max(3, args.warmup)
    dsteps = args.decode_steps or max(steps, 20)
    esteps = args.e2e_steps or steps

    # ---------------- prefill (headline)
    pstep, keep = prefill_bench(wp, steps, warm, stream)
    flops_step = metrics.prefill_flops(wp.B, wp.Hq, wp.T, wp.d, wp.causal, wp.window, wp.n_sink)
    clocks = Clocks(torch.cuda.current_device())
    clocks.start()
    dist.barrier()
    total_ms, (prep_ms, attn_ms) = time_events(pstep, steps, stream)
    dist.barrier()
    clk = clocks.stop()
    api.device_status(stream)
    total_ms = dist.max(total_ms)
    attn_ms_max = dist.max(attn_ms)
    prep_ms_max = dist.max(prep_ms)
    ms_per_step = total_ms / steps
    value = throughput(flops_step, steps, total_ms, n, 1e12)
    attn_tflops = flops_step / (attn_ms_max / steps * 1e-3) / 1e12
    # Each attention launch runs for a large part of a second inside a seconds-long
    # loop: the sustained (power-capped) tensor peak is its denominator.
    long_step = attn_ms_max / steps > 20.0
    peak_t = peaks["bf16_tflops_sustained"] if long_step else peaks["bf16_tflops"]
    peak_burst = peaks["bf16_tflops"]
    del keep, pstep
    torch.cuda.empty_cache()

    # ---------------- the other prefill workloads
    others = {}
    if not args.no_other_workloads:
        for w in synth.SWEEP:
            # at least ~0.1 s of work per variant (the windowed ones take ~4 ms a launch)
            flops_w = metrics.prefill_flops(w.B, w.Hq, w.T, w.d, w.causal, w.window, w.n_sink)
            r = workload_prefill(w, max(args.other_steps, int(1e14 / flops_w)), stream, dist,
                                 peak_burst)
            others[w.name.replace("sweep_", "")] = {
                "tflops": r["attn_kernel_tflops"], "step_tflops": r["step_tflops"],
                "frac": r["frac_of_peak"]}
            torch.cuda.empty_cache()
        # the half-split pair layout (i, i + d/2), a kernel instantiation of its own
        w = synth.sweep("yarn", False)
        flops_w = metrics.prefill_flops(w.B, w.Hq, w.T, w.d, w.causal, w.window, w.n_sink)
        r = workload_prefill(w, max(args.other_steps, int(1e14 / flops_w)), stream, dist,
                             peak_burst, pairs="half")
        others["yarn_dense_half_pairs"] = {"tflops": r["attn_kernel_tflops"],
                                           "step_tflops": r["step_tflops"],
                                           "frac": r["frac_of_peak"]}
        torch.cuda.empty_cache()
        r = chunk_bench(synth.CHUNK, args.other_steps, stream, dist, peak_burst)
        others["chunk_124k_plus_4k"] = {"tflops": r["call_tflops"], "frac": r["frac_of_peak"],
                                        "ms": r["call_ms"]}
        torch.cuda.empty_cache()
        others["chunk_124k_plus_256_fp16cache"] = chunk_fp16cache_bench(
            synth.CHUNK, 256, max(args.other_steps, 10), stream, dist, peak_burst)
        torch.cuda.empty_cache()
        wr = synth.LLAMA3_128K
        for layout in ("contiguous", "zigzag"):
            r = ring_bench(wr, 8, args.other_steps, stream, dist, peak_burst, layout)
            others[f"ring_128k_8_emulated_{layout}"] = {
                "tflops": r["call_tflops"], "frac": r["frac_of_peak"],
                "rank_work_max_over_mean": r["rank_work_max_over_mean"]}
            torch.cuda.empty_cache()
        # the largest single-GPU prefill: 2^20 tokens, ~8 s a step, against the sustained peak
        w1m = synth.LLAMA3_1M
        r = workload_prefill(w1m, 1, stream, dist, peaks["bf16_tflops_sustained"], warmup=1)
        others["prefill_1m"] = {"tflops": r["attn_kernel_tflops"], "step_tflops": r["step_tflops"],
                                "frac_of_sustained": r["frac_of_peak"],
                                "ms": r["attn_kernel_ms"]}
        torch.cuda.empty_cache()
        w16 = synth.LLAMA2_16K
        r = workload_prefill(w16, max(args.other_steps, 20), stream, dist, peak_burst)
        prefill_16k = {"workload": w16.name, "step_tflops": r["step_tflops"],
                       "attn_kernel_tflops": r["attn_kernel_tflops"],
                       "attn_kernel_ms": r["attn_kernel_ms"], "frac_of_burst": r["frac_of_peak"],
                       "steps": r["steps"]}
        torch.cuda.empty_cache()
    else:
        prefill_16k = None

    # ---------------- decode
    dstep, lens = decode_bench(wd, dsteps, warm, stream)
    dbytes = metrics.decode_kv_bytes(lens, wd.Hkv, wd.d)
    dist.barrier()
    dtotal_ms, (dcall_ms,) = time_events(dstep, dsteps, stream)
    dist.barrier()
    api.device_status(stream)
    dtotal_ms = dist.max(dtotal_ms)
    dcall_ms = dist.max(dcall_ms)
    d_gbs = throughput(dbytes, dsteps, dtotal_ms, n, 1e9)
    d_call_gbs = dbytes / (dcall_ms / dsteps * 1e-3) / 1e9
    del dstep
    torch.cuda.empty_cache()

    # ---------------- end to end through the API with host buffers
    estep, h2d, d2h = e2e_prefill(wp, esteps, 2, stream)
    dist.barrier()
    etotal_ms, _ = time_events(estep, esteps, stream)
    dist.barrier()
    etotal_ms = dist.max(etotal_ms)
    e2e_value = throughput(flops_step, esteps, etotal_ms, n, 1e12)
    del estep
    torch.cuda.empty_cache()

    # ---------------- CPU oracle baseline (rank 0, N=1 only)
    cpu = None
    if dist.rank == 0 and n == 1 and not args.no_cpu_baseline:
        f, t, threads, desc = oracle_sample(wp, args.cpu_seconds)
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": desc}

    line = {
        "metric": "causal YaRN-RoPE attention prefill TFLOP/s", "value": value,
        "unit": "TFLOP/s", "n_gpus": n, "steps": steps, "warmup": warm,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp16",
        "data": "synthetic: seeded i.i.d. N(0,1) inputs rounded to bf16",
        "config": workload_config(wp, n),
        "roofline": {"bound": "tensor", "kernel": "prefill_attn_kernel<128, false>",
                     "achieved": attn_tflops, "peak": peak_t, "unit": "TFLOP/s",
                     "frac": attn_tflops / peak_t,
                     "peak_source": f"{peak_src} bf16 "
                                    f"{'sustained' if long_step else 'burst'} (of {peak_src}; "
                                    "the fp16 tensor rate equals bf16)",
                     "frac_of_burst": attn_tflops / peak_burst, "peak_burst": peak_burst,
                     "traffic": ncu_traffic("prefill_attn_kernel<128, false>"),
                     "algorithmic_flops_per_launch": flops_step,
                     "kernel_ms": attn_ms_max / steps,
                     "kv_prep_ms": prep_ms_max / steps},
        "cpu_baseline": cpu,
        "gpu_launches": 2 * steps,
        "clocks": clk,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": esteps,
                "path": "yr_host_prefill_run (C ABI, through api.HostPrefill): pinned host "
                        "q/k/v in, pinned host o out, copies and kernels overlapped per "
                        "(batch, KV-head group)"},
        "other_workloads": _r(others, 4),
        "prefill_16k": _r(prefill_16k, 5),
        "decode": _r({
            "metric": "decode KV-read GB/s", "value": d_gbs, "unit": "GB/s", "steps": dsteps,
            "ms_per_step": dtotal_ms / dsteps, "workload": wd.name,
            "cache_len": lens,
            "roofline": {"bound": "hbm", "kernel": "decode_split_kernel<128, 1> + merge",
                         "achieved": d_call_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": d_call_gbs / peaks["hbm_gbs"],
                         "peak_source": f"{peak_src} HBM copy",
                         "traffic": ncu_traffic("decode_split_kernel<128, 1>"),
                         "algorithmic_bytes_per_launch": dbytes}}, 5),
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()


if __name__ == "__main__":
    main()
