"""Throughput benchmark of Reformer LSH self-attention on B200.

One step = the whole hot path over one batch of synthetic input already in
HBM: lsh_hash -> lsh_sort -> lsh_attn_fwd (chunk attention + round combine)
-> lsh_attn_bwd, all through the C ABI on one stream. Metric: tokens/s
(B*L per step, summed over ranks). Prints one JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the float64 CPU oracle, timed on host cores
For N > 1 launch with torchrun; each rank runs its own independent problem
(weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from efficient_transformer_lsh_b200.workloads import (BLOCK_FF, HEADLINE, WORKLOADS,  # noqa: E402
                                                      generate, generate_block, generate_slices)

METRIC = "LSH-attn fwd+bwd tokens/s at L=64K, 8 heads, 4 rounds; % of roofline"
UNIT = "tokens/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------
# Algorithmic bytes and FLOPs (stage by stage; their sum over a step is the
# compulsory traffic of the whole path: each stage reads its inputs once and
# writes its outputs once).
# ----------------------------------------------------------------------------

def stage_models(w):
    N = w.B * w.H * w.L
    d, nr, m = w.d, w.n_rounds, w.chunk
    e = 4 if w.dtype == "f32" else 2
    de = d * e
    hash_b = N * (de + 4 * nr)
    sort_b = N * 12 * nr
    if nr >= 2:
        fwd_b = N * (de * (1 + 4 * nr) + 12 * nr + 4)
    else:
        fwd_b = N * (3 * de + 8)
    bwd_b = N * (2 * de + 4 + nr * (3 * de + 12) + 8 * d)
    attn_fwd_flops = w.B * w.H * nr * 4 * m * m * d * (2 * w.L / m - 1)
    return {
        "hash": {"bytes": hash_b, "flops": N * nr * d * w.n_buckets},
        "sort": {"bytes": sort_b, "flops": 0},
        "fwd": {"bytes": fwd_b, "flops": attn_fwd_flops},
        "bwd": {"bytes": bwd_b if w.backward else 0,
                "flops": 2.5 * attn_fwd_flops if w.backward else 0},
    }


def bench_block(w, dev, stream, steps, warmup, peaks):
    """One Reformer layer around this workload's attention: the reversible
    block forward (hash, sort, y1 = x1 + F(x2), y2 = x2 + G(y1)) and backward
    (x2 = y2 - G(y1), x1 = y1 - F(x2), all gradients), timed with CUDA events
    on `stream`; then the chunked feed-forward alone (lsh_ff_fwd, and
    lsh_ff_bwd with the reconstruction) against the tensor-core peak.
    Every step touches well over the L2's 126 MB (ten 64 MB activations)."""
    import torch

    from efficient_transformer_lsh_b200 import _lib
    from efficient_transformer_lsh_b200.attention import ReversibleLSHBlock

    cfg = BLOCK_FF[w.name]
    d_ff, ff_chunk = cfg["d_ff"], cfg["ff_chunk"]
    inp = generate_block(w, d_ff)
    t = {k: torch.from_numpy(a).to(dev).to(torch.float32 if k in ("b1", "b2") else torch.bfloat16)
         for k, a in inp.items()}
    blk = ReversibleLSHBlock(w.B, w.H, w.L, w.n_buckets, w.n_rounds, w.chunk, w.causal, d_ff,
                             ff_chunk, w.scale, dev)
    W = (t["W1"], t["b1"], t["W2"], t["b2"])

    def fwd():
        blk.forward(t["x1"], t["x2"], t["R"], *W, stream)

    def bwd():
        blk.backward(blk.y1, blk.y2, t["dy1"], t["dy2"], *W, stream)

    f = blk.f
    nff = _lib.lsh_ff_workspace_size(f)
    wsff = torch.empty(nff, dtype=torch.uint8, device=dev)
    y, rec, dx = (torch.empty_like(t["x1"]) for _ in range(3))
    g = (blk.dW1, blk.db1, blk.dW2, blk.db2)

    def ff_fwd():
        _lib.lsh_ff_fwd(f, t["x1"], *W, t["x2"], y, wsff, nff, stream)

    def ff_bwd():
        _lib.lsh_ff_bwd(f, t["x1"], *W, t["dy2"], t["dy1"], y, rec, dx, *g, wsff, nff, stream)

    def timed(fns):
        for _ in range(warmup):
            for fn in fns:
                fn()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
               for _ in range(steps)]
        torch.cuda.synchronize(dev)
        for k in range(steps):
            for i, fn in enumerate(fns):
                evs[k][i].record(stream)
                fn()
            evs[k][-1].record(stream)
        torch.cuda.synchronize(dev)
        return [statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(steps))
                for i in range(len(fns))]

    launches0 = _lib.lsh_launch_count()
    ms_fwd, ms_bwd = timed([fwd, bwd])
    ff_ms_fwd, ff_ms_bwd = timed([ff_fwd, ff_bwd])
    launches = (_lib.lsh_launch_count() - launches0) // (2 * (warmup + steps))
    assert _lib.lsh_device_status(stream) == 0
    T, D = w.B * w.L, w.H * w.d
    gemm = 2.0 * T * D * d_ff            # FLOPs of one feed-forward product
    tf_fwd = 2 * gemm / (ff_ms_fwd / 1e3) / 1e12
    tf_bwd = 6 * gemm / (ff_ms_bwd / 1e3) / 1e12
    peak = peaks["bf16_tflops"]
    return {
        "what": "reversible block y1 = x1 + LSHAttn(x2), y2 = x2 + FF(y1), forward + backward "
                "from the outputs; the feed-forward alone below",
        "d_model": D, "d_ff": d_ff, "ff_chunk": ff_chunk, "steps": steps,
        "ms_fwd": ms_fwd, "ms_bwd": ms_bwd, "ms_per_step": ms_fwd + ms_bwd,
        "tokens_per_s": T / ((ms_fwd + ms_bwd) / 1e3),
        "launches_per_step": launches,
        "ff": {"ms_fwd": ff_ms_fwd, "ms_bwd": ff_ms_bwd,
               "flops_fwd": 2 * gemm, "flops_bwd": 6 * gemm,
               "tflops_fwd": tf_fwd, "tflops_bwd": tf_bwd, "peak_tflops": peak,
               "frac_fwd": tf_fwd / peak, "frac_bwd": tf_bwd / peak,
               "peak_source": peaks["source"],
               "note": "fwd: h = relu(x W1 + b1), y = res + h W2 + b2; bwd: h again, "
                       "the reconstruction, dh, dW2, dW1, dx (six products)"},
    }


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, source="fallback")


# ----------------------------------------------------------------------------
# Clock sampling during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.rows = []
        self.proc = None
        self.gpu_index = gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        threading.Thread(target=self._read, daemon=True).start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 8:
                self.rows.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        win = [p for t, p in self.rows if t0 - 0.15 <= t <= t1 + 0.15]
        note = "in timed window"
        if not win:
            near = sorted(self.rows, key=lambda r: min(abs(r[0] - t0), abs(r[0] - t1)))[:3]
            win = [p for _, p in near]
            note = "nearest samples (timed window shorter than the sampling period)"
        sm = [float(p[1]) for p in win if p[1].replace(".", "").isdigit()]
        mx = [float(p[2]) for p in win if p[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for p in win for i in range(4) if p[4 + i] == "Active"})
        pw = [float(p[3]) for p in win if p[3].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "power_w_max": max(pw) if pw else None, "samples": len(win), "note": note}


# ----------------------------------------------------------------------------
# CPU oracle timing (baseline leg and the reference arm)
# ----------------------------------------------------------------------------

def _pool_init():
    # one BLAS thread per worker process: the pool's size is the core count used
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


def _oracle_slice(task):
    """hash + sort + forward (+ backward) of the oracle on one (batch, head)
    slice at full L (runs in a pool worker)."""
    import numpy as np
    from oracle import lsh_oracle as orc
    qk, v, dO, R, chunk, causal, scale, backward = task
    qk = qk.astype(np.float64)[None, None]
    v = v.astype(np.float64)[None, None]
    bucket, _ = orc.hash_buckets(qk, R.astype(np.float64))
    perm = orc.sort_positions(bucket)
    O, LSE = orc.forward(qk, v, perm, chunk, causal, scale)
    if backward:
        orc.backward(qk, v, perm, chunk, causal, scale, O, LSE, dO.astype(np.float64)[None, None])
    return True


class OracleTimer:
    """Times the float64 oracle on the host cores: one (batch, head) slice per
    worker of a spawn-started process pool, all slices at once."""

    def __init__(self, w):
        import multiprocessing as mp
        self.w = w
        inp = generate(w)
        n_slices = w.B * w.H
        self.cores = max(1, min(n_slices, len(os.sched_getaffinity(0))))
        self.tasks = []
        for k in range(self.cores):
            b, h = divmod(k, w.H)
            dO = inp["dO"][b, h] if w.backward else None
            self.tasks.append((inp["qk"][b, h], inp["v"][b, h], dO, inp["R"], w.chunk, w.causal,
                               w.scale, w.backward))
        self.frac = self.cores / n_slices
        self.pool = mp.get_context("spawn").Pool(self.cores, initializer=_pool_init)

    def run(self):
        t = time.perf_counter()
        self.pool.map(_oracle_slice, self.tasks, chunksize=1)
        return time.perf_counter() - t

    def sample(self):
        w = self.w
        return (f"{self.cores} of {w.B * w.H} (batch, head) slices at full L={w.L}, one per worker "
                f"process, all {w.n_rounds} rounds, hash+sort+fwd{'+bwd' if w.backward else ''}; "
                f"tokens/s scaled by the slice fraction {self.frac:.4f}")

    def close(self):
        self.pool.close()
        self.pool.join()


def cpu_baseline(w):
    timer = OracleTimer(w)
    try:
        timer.run()                      # workers start and import numpy
        dt = timer.run()
    finally:
        timer.close()
    return {"value": w.tokens * timer.frac / dt, "unit": UNIT, "cores": timer.cores,
            "kind": "oracle", "seconds": dt, "sample": timer.sample()}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", 0))
    if rank != 0:
        return 0
    timer = OracleTimer(w)
    try:
        for _ in range(args.warmup):
            timer.run()
        times = [timer.run() for _ in range(args.steps)]
    finally:
        timer.close()
    per_step = sum(times) / len(times)
    value = w.tokens * timer.frac / per_step
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3 / timer.frac,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": timer.cores, "kind": "oracle",
                         "sample": "each step: " + timer.sample()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def source_digest(files):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload, stage):
    """DRAM bytes per launch of a stage's kernels from the committed ncu
    summary (profiles/traffic.json), or None when there is none or when the
    kernel sources changed since the counters were taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            e = json.load(f).get(workload, {}).get(stage)
        if not e or source_digest(e["sources"]) != e["digest"]:
            return None
        return e["bytes"]
    except Exception:
        return None


def config_of(w):
    c = w.describe()
    c["l2"] = "no flush: each step streams >1 GB (inputs, partials, gradients), 10x the 126 MB L2"
    return c


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE, choices=list(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--heads", type=int, default=None,
                    help="override H (smaller cases of the same kernels, e.g. for profiler captures)")
    ap.add_argument("--seq-len", type=int, default=None, help="override L")
    ap.add_argument("--no-block", action="store_true",
                    help="skip the reversible-block (attention + chunked feed-forward) timing")
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    if args.heads is not None:
        w = w.with_sizes(H=args.heads)
    if args.seq_len is not None:
        w = w.with_sizes(L=args.seq_len)
    if args.impl == "reference":
        return run_reference(args, w)
    args.warmup = max(3, args.warmup)

    import numpy as np
    import torch

    from efficient_transformer_lsh_b200 import _lib, dist
    from efficient_transformer_lsh_b200.attention import LSHAttention

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    rank, local, world = dist.init("nccl")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    _lib.lib()

    # one global problem of world x B batches; this rank runs its shard of
    # B*H slices (weak scaling: the per-rank work is fixed)
    gw = w.with_sizes(B=w.B * world)
    lo, hi = dist.shard(gw.B * gw.H, rank, world)
    inp = generate_slices(gw, lo, hi)
    for k in ("qk", "v", "dO"):
        if k in inp:
            inp[k] = inp[k].reshape(w.B, w.H, w.L, w.d)
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    host = {k: torch.from_numpy(a).to(td).pin_memory() for k, a in inp.items()}
    d_in = {k: t.to(dev, non_blocking=True) for k, t in host.items()}
    run = LSHAttention(w.B, w.H, w.L, w.n_buckets, w.n_rounds, w.chunk, w.causal, w.dtype, w.d,
                       w.scale, dev)
    stream = torch.cuda.current_stream(dev)
    names = ["hash", "sort", "fwd", "bwd"] if w.backward else ["hash", "sort", "fwd"]

    def step(evs=None):
        if evs is not None:
            evs[0].record(stream)
        run.hash(d_in["qk"], d_in["R"], stream)
        if evs is not None:
            evs[1].record(stream)
        run.sort(None, stream)
        if evs is not None:
            evs[2].record(stream)
        run.attend(d_in["qk"], d_in["v"], None, stream)
        if evs is not None:
            evs[3].record(stream)
        if w.backward:
            run.backward(d_in["qk"], d_in["v"], d_in["dO"], None, stream)
            if evs is not None:
                evs[4].record(stream)

    torch.cuda.synchronize(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert _lib.lsh_device_status(stream) == 0
    memory = {"peak_bytes": int(torch.cuda.max_memory_allocated(dev)),
              "workspace_bytes": int(run.ws_sort_bytes + run.ws_fwd_bytes + run.ws_bwd_bytes),
              "note": "device memory torch allocated for one problem: inputs, outputs, "
                      "bucket/perm and the three workspaces"}

    # timed region: K whole steps, device time, max over ranks
    gpu_index = os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local if world > 1 else 0]
    sampler = ClockSampler(gpu_index.strip() or local)
    sampler.start()
    time.sleep(0.3)
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(K)]
    launches0 = _lib.lsh_launch_count()
    dist.barrier(dev)
    torch.cuda.synchronize(dev)
    t_host0 = time.time()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for k in range(K):
        step(evs[k])
    end.record(stream)
    torch.cuda.synchronize(dev)
    t_host1 = time.time()
    dist.barrier(dev)
    launches = _lib.lsh_launch_count() - launches0
    time.sleep(0.2)
    sampler.stop()
    assert _lib.lsh_device_status(stream) == 0
    t_ms = start.elapsed_time(end)
    t_ms_max = dist.max_over_ranks(t_ms, dev)
    ms_per_step = t_ms_max / K
    value = world * w.tokens * K / (t_ms_max / 1e3)

    stage_ms = {n: statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(K))
                for i, n in enumerate(names)}
    models = stage_models(w)
    peaks = load_peaks()
    stages = {}
    for n in names:
        t = stage_ms[n] / 1e3
        b, f = models[n]["bytes"], models[n]["flops"]
        t_b = b / (peaks["hbm_gbs"] * 1e9)
        t_f = f / (peaks["bf16_tflops"] * 1e12)
        bound = "hbm" if t_b >= t_f else "tensor"
        if w.dtype == "f32" and bound == "tensor":
            bound = "alu"
        stages[n] = {"ms": stage_ms[n], "bytes": b, "flops": f, "bound": bound,
                     "gbs": b / t / 1e9, "tflops": f / t / 1e12,
                     "frac": max(t_b, t_f) / t}
    dom = max(names, key=lambda n: stage_ms[n])
    ds = stages[dom]
    traffic = measured_traffic(w.name, dom)
    if ds["bound"] == "hbm":
        roof = {"bound": "hbm", "achieved": ds["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        roof = {"bound": ds["bound"], "achieved": ds["tflops"], "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic
    roof["kernel"] = f"lsh_{'attn_' if dom in ('fwd', 'bwd') else ''}{dom} stage"
    roof["peak_source"] = peaks["source"]
    t_b = sum(models[n]["bytes"] for n in names) / (peaks["hbm_gbs"] * 1e9)
    t_f = sum(models[n]["flops"] for n in names if n != "hash") / (peaks["bf16_tflops"] * 1e12)
    t_star = max(t_b, t_f)
    step_roof = {"t_star_us": t_star * 1e6, "t_step_us": ms_per_step * 1e3,
                 "frac": t_star / (ms_per_step / 1e3),
                 "definition": "max(algorithmic bytes / HBM peak, chunk-attention FLOPs / bf16 "
                               "peak) over the whole step, divided by the measured step time"}

    # end to end through the public API with host buffers: every step copies
    # its inputs in from pinned host memory and its outputs (out, lse, dqk, dv)
    # back. Two sets of device buffers alternate, so that step i's host->device
    # copy, step i-1's compute and step i-2's device->host copy overlap on
    # three streams (PCIe is full duplex).
    E = max(1, args.e2e_steps)
    runs = [run, LSHAttention(w.B, w.H, w.L, w.n_buckets, w.n_rounds, w.chunk, w.causal, w.dtype,
                              w.d, w.scale, dev)]
    ins = [d_in, {k: torch.empty_like(t) for k, t in d_in.items()}]
    out_names = ["out", "lse"] + (["dqk", "dv"] if w.backward else [])
    outs_h = [{k: torch.empty(getattr(r, k).shape, dtype=getattr(r, k).dtype).pin_memory()
               for k in out_names} for r in runs]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs_h[0].values())
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    in_ready, done, out_read = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def e2e_step(i):
        k = i & 1
        r, d = runs[k], ins[k]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(done[k])              # step i-2 no longer reads d
            for name in host:
                d[name].copy_(host[name], non_blocking=True)
            in_ready[k].record(s_in)
        stream.wait_event(in_ready[k])
        if i >= 2:
            stream.wait_event(out_read[k])            # step i-2's outputs copied out
        r.hash(d["qk"], d["R"], stream)
        r.sort(None, stream)
        r.attend(d["qk"], d["v"], None, stream)
        if w.backward:
            r.backward(d["qk"], d["v"], d["dO"], None, stream)
        done[k].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done[k])
            for name in out_names:
                outs_h[k][name].copy_(getattr(r, name), non_blocking=True)
            out_read[k].record(s_out)

    dist.barrier(dev)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(E):
        e2e_step(i)
    for k in range(min(E, 2)):
        stream.wait_event(out_read[k])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    assert _lib.lsh_device_status(stream) == 0
    e2e_ms = dist.max_over_ranks(e0.elapsed_time(e1), dev)
    e2e = {"value": world * w.tokens * E / (e2e_ms / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": E,
           "note": "copies on their own streams, overlapping the neighbouring steps' compute"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": config_of(w), "roofline": roof, "step_roofline": step_roof, "stages": stages,
        "e2e": e2e, "gpu_launches": launches, "clocks": sampler.summary(t_host0, t_host1),
        "memory": memory,
    }
    if rank == 0 and world == 1 and not args.no_block and w.name in BLOCK_FF and \
            args.heads is None and args.seq_len is None:
        line["rev_block"] = bench_block(w, dev, stream, min(K, 10), args.warmup, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.finish()
    return 0


if __name__ == "__main__":
    sys.exit(main())
