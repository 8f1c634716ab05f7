#!/usr/bin/env python3
"""Benchmark: batch-1 greedy decode tokens/s of the ~1.9B (2B-class) bf16 decoder at a
4096-token context on one B200, and the fraction of the HBM roofline it reaches.

A step is one whole decode run of the workload (kd_reset + one kd_decode launch that
generates n_gen tokens, i.e. every row of the hot path, n_gen times). Weights, KV cache and
the start token are resident in HBM before timing starts; timing uses CUDA events on the
decode stream, max over ranks. The model streams 3.65 GB of weights per token, far above
the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

With --gpus N > 1 (launched under torch.distributed.run) each rank runs an independent
replica of the request on its own GPU: batch-1 decode has no data-parallel split, so the
aggregate is N replicas ("weak" scaling), with no collective on the data path.
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
sys.path.insert(0, ROOT)

METRIC = "batch-1 decode tokens/s on 1 B200 (2B bf16) and % of HBM-bandwidth roofline"
SPEC_HBM_GBS = 8000.0          # B200 HBM3e specification
# DRAM bytes per algorithmic byte of the monokernel, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum of one launch decoding 8 tokens of the 2B model
# at a 4k context, `--workload 2b-4k --n-gen 8`). It holds for the kernel source it was taken on
# only: when csrc/kd_kernel.cu + csrc/kd_layout.h no longer hash to this SHA-256, traffic is
# null.
TRAFFIC_CAPTURE = {"kernel_sha256": "c23556280ff148b3c55673ca72c3471862dbd97e66f81a4b6d581d338a152f88",
                   "dram_bytes": 32999673000.0 + 163582976.0, "algorithmic_bytes": 32998424576.0}
FALLBACK_HBM_GBS = 6650.0       # an earlier B200 copy measurement, used without a measured peaks file


def kernel_source_sha256() -> str:
    """SHA-256 of the kernel source and its launch-shape header, concatenated."""
    import hashlib
    h = hashlib.sha256()
    for name in ("kd_kernel.cu", "kd_layout.h"):
        with open(os.path.join(ROOT, "persistent_monokernel_sm_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def launch_traffic(bytes_launch: float):
    """DRAM bytes of one timed launch: the captured DRAM/algorithmic ratio times this launch's
    algorithmic bytes, or None when the kernel changed since the capture."""
    cap = TRAFFIC_CAPTURE
    if not cap["kernel_sha256"] or cap["kernel_sha256"] != kernel_source_sha256():
        return None
    return cap["dram_bytes"] / cap["algorithmic_bytes"] * bytes_launch


def max_over_ranks(values, device):
    """Element-wise maximum of `values` over all ranks of the default process group (the
    values themselves with one rank). Used for every time the benchmark reports."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def replica_throughput(tokens_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job tokens/s of `world` independent replicas: all tokens over the slowest rank's time."""
    return tokens_per_rank * world / (max_ms * 1e-3)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="2b-4k")
    ap.add_argument("--n-gen", type=int, default=None, help="override generated tokens per step")
    ap.add_argument("--impl", default="kernel", choices=["kernel", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-tokens", type=int, default=8)
    ap.add_argument("--phase-trace", action="store_true",
                    help="instead of the benchmark line, print where one launch spends its time (per-phase trace)")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi SM clock and throttle reasons, sampled every 200 ms while timing."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_cores():
    return os.cpu_count() or 1


def run_oracle_sample(w, weights_h, K, V, start, n_tokens):
    """Time the oracle (single-threaded) generating n_tokens of workload w; tokens/s."""
    import oracle
    o = oracle.Oracle(w.dims(), weights_h, capacity=w.start_pos + w.n_pending + n_tokens, n_threads=1)
    if K is not None:
        o.set_kv(K, V)
    t0 = time.perf_counter()
    o.greedy(start, w.start_pos, n_tokens, keep_logits=False)
    dt = time.perf_counter() - t0
    o.close()
    return n_tokens / dt, dt


def lscpu_model():
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for ln in out.splitlines():
            if ln.startswith("Model name"):
                return ln.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def reference_arm(args, w):
    """The oracle, as it stands, timed on the host cores; rank 0 only."""
    import torch
    import synth
    rank, world, local = dist_env()
    if rank != 0:
        return
    n_tok = 1  # tokens per step: one decode step of the full workload is ~2 s on one core
    weights = synth.make_weights(w)
    wh = {k: v.cpu() for k, v in weights.items()}
    del weights
    K = V = None
    if w.kv_len:
        K, V = synth.make_kv(w)
        K, V = K.cpu(), V.cpu()
    start = synth.make_prompt(w).numpy()
    for _ in range(args.warmup):
        run_oracle_sample(w, wh, K, V, start, n_tok)
    total = 0.0
    for _ in range(args.steps):
        _, dt = run_oracle_sample(w, wh, K, V, start, n_tok)
        total += dt
    value = args.steps * n_tok / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": workload_config(w, n_tok),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": "%d decode token(s) per step of workload %s (start token at position %d), "
                                   "single-threaded oracle; host %s, %d cores present"
                                   % (n_tok, w.name, w.start_pos, lscpu_model(), cpu_cores())},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


PHASES = ["qkv", "attention", "o_proj", "gate_up", "down", "lm_head"]


def phase_trace(dec, w, d_start, warmup):
    """Where one launch spends its time, from the kernel's per-phase trace (kd_set_trace):
    one traced launch of the workload with every CTA recording, next to the median of three
    untraced ones. Returns a dict (printed as one JSON line); see summarize_trace."""
    import torch
    import persistent_monokernel_sm_b200 as kd
    L, steps = w.dims()["n_layers"], w.n_steps
    rows = 5 * L * steps + steps + 2
    grid = dec.info().grid
    buf = torch.zeros(grid * rows * 8, dtype=torch.int64, device=d_start.device)

    def launch(traced):
        kd.kd_set_trace(dec.h, buf.data_ptr() if traced else None, buf.numel(), 1)
        dec.reset(d_start, w.start_pos)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(dec.stream)
        dec.decode(w.n_gen)
        e1.record(dec.stream)
        dec.sync()
        return e0.elapsed_time(e1)

    for _ in range(max(1, warmup)):
        launch(False)
    plain_ms = statistics.median(launch(False) for _ in range(3))
    traced_ms = launch(True)
    kd.kd_set_trace(dec.h, None, 0, 1)
    tr = buf.cpu().numpy().reshape(grid, rows, 8)
    out = summarize_trace(tr, traced_ms)
    out.update({"workload": w.name, "tokens": w.n_gen, "grid": grid, "launch_ms": plain_ms,
                "traced_launch_ms": traced_ms, "launches_per_token": 1.0 / w.n_gen})
    return {"phase_trace": out}


def summarize_trace(tr, traced_ms):
    """Per-phase times and time fractions of one traced launch.

    tr: [grid][rows][8] int64, the kernel's trace rows (per phase: id = step << 16 | layer << 4
    | phase, begin, inputs ready, compute done, end, cycles waiting for stages, first and last
    stage ready), the producer's row last. Inputs ready ends the cross-CTA wait of a phase that
    follows a sync (Q/K/V after layer 0, gate/up, LM head: the wait for the counter plus the
    fold of the summed delta into the residual and its norm) or the poll on the kv head's
    exchange words (attention: the step's q/k/v; output projection: the attention records). A
    CTA without an attention piece stamps neither mark in that phase (all of it counts as
    compute). The step boundary (the wait for the previous step's argmax, the embedding
    gather) lies between a step's last phase and the next step's first and counts as sync
    wait. Steps >= 1 are averaged; SM cycles become time by the launch's measured duration."""
    import numpy as np
    grid, rows = tr.shape[0], tr.shape[1]
    body = tr[:, :rows - 1, :].astype(np.int64)
    live = []
    for c in range(grid):
        b = body[c][body[c][:, 1] != 0].copy()
        b[:, 2] = np.where(b[:, 2] == 0, b[:, 1], b[:, 2])
        b[:, 3] = np.where(b[:, 3] == 0, b[:, 4], b[:, 3])
        live.append(b)
    span_cyc = [b[:, 4].max() - b[:, 1].min() for b in live if len(b)]
    mhz = float(np.median(span_cyc)) / (traced_ms * 1e3)  # SM cycles per microsecond
    keys = ("wait", "compute", "tail", "stage_wait", "total", "first_stage", "stage_span", "after_last_stage",
            "gap_before")
    per = {n: {k: [] for k in keys} for n in PHASES}
    spans, boundary, other_gaps, sync_wait, xchg_wait, stage_wait, tails = [], [], [], [], [], [], []
    for b in live:
        ids = b[:, 0]
        step, layer, ph = ids >> 16, (ids >> 4) & 0xfff, ids & 15
        sel = step >= 1
        if not sel.any():
            continue
        bs, phs, lays, sts = b[sel], ph[sel], layer[sel], step[sel]
        spans.append((bs[:, 4].max() - bs[:, 1].min()) / mhz)
        for k, n in enumerate(PHASES):
            x = bs[phs == k]
            if not len(x):
                continue
            d = per[n]
            d["wait"].append(((x[:, 2] - x[:, 1]) / mhz).mean())
            d["compute"].append(((x[:, 3] - x[:, 2]) / mhz).mean())
            d["tail"].append(((x[:, 4] - x[:, 3]) / mhz).mean())
            d["stage_wait"].append((x[:, 5] / mhz).mean())
            d["total"].append(((x[:, 4] - x[:, 1]) / mhz).mean())
            hs = x[x[:, 6] != 0]
            if len(hs):
                d["first_stage"].append(((hs[:, 6] - hs[:, 2]) / mhz).mean())
                d["stage_span"].append(((hs[:, 7] - hs[:, 6]) / mhz).mean())
                d["after_last_stage"].append(((hs[:, 3] - hs[:, 7]) / mhz).mean())
        w_in = (bs[:, 2] - bs[:, 1]) / mhz
        after_sync = ((phs == 0) & (lays > 0)) | (phs == 3) | (phs == 5)
        gaps = (bs[1:, 1] - bs[:-1, 4]) / mhz
        new_step = sts[1:] != sts[:-1]
        for k, n in enumerate(PHASES):  # the gap from the previous phase of the same step
            m = (phs[1:] == k) & ~new_step
            if m.any():
                per[n]["gap_before"].append(gaps[m].mean())
        nsteps = max(1, len(set(sts.tolist())) - 1)
        boundary.append(gaps[new_step].sum() / nsteps)
        other_gaps.append(gaps[~new_step].sum() / nsteps)
        sync_wait.append(w_in[after_sync].sum() + gaps[new_step].sum())
        xchg_wait.append(w_in[(phs == 1) | (phs == 2)].sum())
        stage_wait.append((bs[:, 5] / mhz).sum())
        tails.append(((bs[:, 4] - bs[:, 3]) / mhz).sum())
    span = float(np.mean(spans))
    return {
        "sm_cycles_per_us": mhz,
        "us_per_phase": {n: {k: float(np.mean(v)) for k, v in d.items() if v} for n, d in per.items() if d["total"]},
        "fraction_of_time": {
            "cross_cta_sync_wait": float(np.mean(sync_wait)) / span,
            "kv_head_exchange_wait": float(np.mean(xchg_wait)) / span,
            "stage_wait_in_compute": float(np.mean(stage_wait)) / span,
            "phase_tails": float(np.mean(tails)) / span,
        },
        "step_boundary_us": float(np.mean(boundary)),
        "between_phases_us_per_step": float(np.mean(other_gaps)),
        "step_boundary_us_max_over_ctas": float(np.max(boundary)),
    }


def read_stream_gbs(device, gib: int = 4, reps: int = 3) -> float:
    """Read-only HBM bandwidth for context beside the copy-based peak: the best of `reps`
    timed sums over a `gib` GiB bf16 buffer (a library reduction, outside the timed region of
    the decode)."""
    import torch
    buf = torch.ones(gib << 29, dtype=torch.bfloat16, device=device)  # gib GiB
    torch.cuda.synchronize(device)
    best = float("inf")
    for _ in range(reps + 1):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        s = buf.sum(dtype=torch.float32)
        e1.record()
        torch.cuda.synchronize(device)
        best = min(best, e0.elapsed_time(e1))
    del buf, s
    torch.cuda.empty_cache()
    return (gib << 30) / (best * 1e-3) / 1e9


def workload_config(w, n_gen):
    return {"workload": w.name, "n_layers": w.n_layers, "d_model": w.d_model, "n_heads": w.n_heads,
            "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim, "ffn_dim": w.ffn_dim, "vocab": w.vocab,
            "kv_len": w.kv_len, "prompt_len": w.prompt_len, "n_gen": n_gen, "batch": 1,
            "parallelism": "replicas", "l2": "inputs larger than L2 (weights streamed every token)"}


def main():
    args = parse()
    import synth
    w = synth.get(args.workload)
    if args.n_gen:
        w = w.replace(n_gen=args.n_gen)
    if args.impl == "reference":
        return reference_arm(args, w)

    import torch
    import torch.distributed as dist
    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    from persistent_monokernel_sm_b200 import build
    build.build()
    import persistent_monokernel_sm_b200 as kd

    weights = synth.make_weights(w, device="cuda")
    K = V = None
    if w.kv_len:
        K, V = synth.make_kv(w, device="cuda")
    start = synth.make_prompt(w)
    dec = kd.Decoder(w.dims(), w.capacity, device=dev)
    dec.load_weights(weights)
    if K is not None:
        dec.set_kv(K, V)
    weights_h = None
    if rank == 0 and not args.no_cpu_baseline:
        weights_h = {k: v.cpu() for k, v in weights.items()}
        Kh, Vh = (K.cpu(), V.cpu()) if K is not None else (None, None)
    del weights
    torch.cuda.empty_cache()
    stream = dec.stream
    d_start = start.to(dev)
    tok_out = torch.empty(w.n_gen, dtype=torch.int32, device=dev)

    def step():
        dec.reset(d_start, w.start_pos)
        dec.decode(w.n_gen, out=tok_out)

    if args.phase_trace:
        if rank == 0:
            print(json.dumps(phase_trace(dec, w, d_start, args.warmup)), flush=True)
        dec.close()
        if world > 1:
            dist.destroy_process_group()
        return

    for _ in range(args.warmup):
        step()
    dec.sync()
    launches0 = dec.info().launches

    # ---- device-timed region
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            dec.reset(d_start, w.start_pos)
            ev[i][0].record(stream)
            dec.decode(w.n_gen, out=tok_out)
            ev[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize(dev)
    dec.sync()
    total_ms = t0.elapsed_time(t1)
    kern_ms = [a.elapsed_time(b) for a, b in ev]
    launches = dec.info().launches - launches0
    total_ms, kern_max = max_over_ranks([total_ms, max(kern_ms)], dev)
    if world > 1:
        dist.barrier()

    # ---- end to end through the public host-memory call
    h_in = start.pin_memory()
    h_out = torch.empty(w.n_gen, dtype=torch.int32).pin_memory()
    dec.generate(h_in, w.start_pos, w.n_gen, h_out)  # warm
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        dec.generate(h_in, w.start_pos, w.n_gen, h_out)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks([e0.elapsed_time(e1)], dev)[0]

    # ---- roofline of the monokernel: algorithmic bytes per launch / launch time
    cfg = dec.cfg
    bytes_launch = sum(kd.kd_step_bytes(cfg, w.start_pos + i + 1, True) for i in range(w.n_steps))
    mean_kern_ms = statistics.mean(kern_ms)
    achieved = bytes_launch / (mean_kern_ms * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    traffic = launch_traffic(bytes_launch)

    line = None
    if rank == 0:
        value = replica_throughput(args.steps * w.n_gen, world, total_ms)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "storage": "bf16 weights and KV cache",
            "data": "synthetic", "config": workload_config(w, w.n_gen),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": "%s copy bandwidth (MEASURED_PEAKS.json hbm_gbs)" % peak_kind
                         if peak_kind == "measured" else "fallback 6.65 TB/s",
                         "frac_of_8tbs_spec": achieved / SPEC_HBM_GBS,
                         "bytes_per_launch": bytes_launch, "kernel": "kd::monokernel",
                         "launch_ms": mean_kern_ms},
            "tokens_per_s_per_launch": w.n_gen / (mean_kern_ms * 1e-3),
            "roofline_tokens_per_s": w.n_gen / (bytes_launch / (peak * 1e9)),
            "e2e": {"value": replica_throughput(args.steps * w.n_gen, world, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": 4 * w.n_pending, "d2h_bytes_per_step": 4 * w.n_gen},
            "gpu_launches": launches, "launches_per_token": launches / (args.steps * w.n_gen),
            "clocks": clk.summary(),
            "stream_read_gbs": read_stream_gbs(dev),
        }
    if rank == 0 and not args.no_cpu_baseline:
        n = max(1, args.cpu_sample_tokens)
        tps, dt = run_oracle_sample(w, weights_h, Kh, Vh, start.numpy(), n)
        line["cpu_baseline"] = {
            "value": tps, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "effective_gbs": tps * bytes_launch / w.n_gen / 1e9,
            "sample": "first %d greedy tokens of workload %s, single-threaded oracle, %.1f s; host %s, %d cores"
                      % (n, w.name, dt, lscpu_model(), cpu_cores())}
    if rank == 0:
        print(json.dumps(line), flush=True)
    dec.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
