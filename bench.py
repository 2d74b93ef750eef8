#!/usr/bin/env python
"""Benchmark of the ReHyAt hybrid attention forward on B200.

One step = one whole-sequence forward of the 480x832 5 s workload (B=1, 12 heads, D=128,
21 frames x 1560 tokens, Tc=3, To=1, P=2, F=128, G=8, bf16): the state folds with phi_k, their
prefix scan, and the fused softmax + linear attention with phi_q, through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

N > 1 runs under torchrun: every rank runs its own replica of the workload (weak scaling, no
collective on the data path; NCCL only for the timing barrier and the max over ranks).
Prints one JSON line (rank 0).  `--impl reference` times the float64 CPU oracle on the same
workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hybrid_softmax_linear_chunked_b200 import binding as rb  # noqa: E402
from hybrid_softmax_linear_chunked_b200 import configs as C  # noqa: E402
from hybrid_softmax_linear_chunked_b200.inputs import make_inputs  # noqa: E402
from hybrid_softmax_linear_chunked_b200.replicas import Replicas, job_throughput  # noqa: E402

METRIC = "hybrid-attn query tokens/s (12 heads, D=128); % of dense BF16 tensor peak"
UNIT = "tokens/s"
WORKLOAD = C.WAN_480P_5S
L2_BYTES = 126 * 1024 * 1024
ATTN_SOURCES = ["hybrid_softmax_linear_chunked_b200/csrc/attn_bf16.cuh",
                "hybrid_softmax_linear_chunked_b200/csrc/sm100.cuh",
                "hybrid_softmax_linear_chunked_b200/csrc/featmap.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_traffic.txt")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def attn_source_hash() -> str:
    h = hashlib.sha256()
    for rel in ATTN_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def read_traffic():
    """DRAM bytes per attention launch from the committed ncu summary, if it was taken on the
    current attention source (hash match); else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    want = attn_source_hash()
    with open(TRAFFIC_FILE) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 2 and parts[0] == want:
                return float(parts[1])
    return None


class ClockSampler:
    """nvidia-smi samples (every 200 ms) while the timed region runs."""

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        self.cmd = ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms",
                    "200", "-i", str(device_index)]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

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
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        loaded = [x for x in sm if x > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def device_index_for_smi(dev: torch.device) -> str:
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:  # noqa: BLE001
        return str(dev.index)


# ---------------------------------------------------------------------------------------------
# CPU oracle timings (the baseline, and the reference arm)
# ---------------------------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:  # noqa: BLE001
        pass
    return len(os.sched_getaffinity(0))


def f64(t):
    return t.to(torch.float64).numpy()


def cpu_baseline(inp, w: C.Workload, budget_s: float = 12.0):
    """The oracle's recurrent (linear-cost) form, head by head, until `budget_s` has passed or all
    heads are done; tokens/s scaled to the whole workload (a token = one query position across
    all heads)."""
    import oracle.rehyat_oracle as O
    t0 = time.perf_counter()
    heads = 0
    for h in range(w.H):
        q, k, v = f64(inp.q[0, h]), f64(inp.k[0, h]), f64(inp.v[0, h])
        pq = O.feature_map(q, f64(inp.Wq[h]), f64(inp.bq[h]), w.P)
        pk = O.feature_map(k, f64(inp.Wk[h]), f64(inp.bk[h]), w.P)
        O.hybrid_attention_recurrent(q, k, v, pq, pk, w.frame_tokens, w.Tc, w.To)
        heads += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    tokens = w.B * w.N * heads / w.H
    return {"value": tokens / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"float64 recurrent form, batch 0 heads 0-{heads - 1} of {w.H} (all "
                      f"{w.N} query rows each), {dt:.1f} s; scaled to query tokens of all heads"}


def run_reference(args, rank: int):
    """Reference arm: the oracle as it stands, on host cores, one bounded sample per step."""
    if rank != 0:
        return
    import oracle.rehyat_oracle as O
    w = WORKLOAD
    inp = make_inputs(w)
    rng = np.random.default_rng(0)
    cache = {}

    def step(i, n_rows):
        h = i % w.H
        if h not in cache:
            cache[h] = [f64(x) for x in (inp.q[0, h], inp.k[0, h], inp.v[0, h], inp.Wq[h],
                                         inp.bq[h], inp.Wk[h], inp.bk[h])]
        q, k, v, Wq, bq, Wk, bk = cache[h]
        rows = rng.integers(0, w.N, size=n_rows)
        O.hybrid_attention_rows(q, k, v, Wq, bq, Wk, bk, w.P, w.frame_tokens, w.Tc, w.To, rows)

    # size a step so that warm-up + timed steps take about two minutes in all
    t = time.perf_counter()
    step(0, 64)
    per64 = time.perf_counter() - t
    budget = min(0.5, 120.0 / max(1, args.steps + args.warmup))
    n_rows = int(max(8, min(4096, 64 * budget / max(per64, 1e-6))))
    for i in range(args.warmup):
        step(i, n_rows)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i, n_rows)
    dt = time.perf_counter() - t0
    tokens = args.steps * n_rows / w.H
    value = tokens / dt
    sample = (f"float64 oracle (row form), {n_rows} random query rows of one head per step, "
              f"heads cycled; a token = one query position across all {w.H} heads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(w: C.Workload, n_gpus: int):
    return {"workload": w.name, "B": w.B, "H": w.H, "D": w.D, "T": w.T,
            "frame_tokens": w.frame_tokens, "seq_len": w.N, "Tc": w.Tc, "To": w.To, "P": w.P,
            "F": w.F, "G": w.G, "global_batch": w.B * n_gpus,
            "parallelism": f"dp{n_gpus} (independent replicas, no collective)",
            "l2": "inputs larger than L2 (q, k, v = %.0f MB > 126 MB), no flush"
                  % (3 * w.B * w.H * w.N * w.D * 2 / 1e6)}


# ---------------------------------------------------------------------------------------------
# native arm
# ---------------------------------------------------------------------------------------------

def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args, int(os.environ.get("RANK", "0")))
        return

    rep = Replicas.from_env("nccl")
    rank, world, local = rep.rank, rep.world, rep.local_rank
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    rb.load()
    w = WORKLOAD
    inp = make_inputs(w, seed=rep.seed(w.seed))
    q, k, v = (x.to(dev) for x in (inp.q, inp.k, inp.v))
    Wq, bq, Wk, bk = (x.to(dev) for x in (inp.Wq, inp.bq, inp.Wk, inp.bk))
    kw = dict(P=w.P, frame_tokens=w.frame_tokens, Tc=w.Tc, To=w.To)
    d = rb.dims_of(q, Wq, w.P)
    ws = torch.empty(rb.forward_workspace_size(d, rb.REHYAT_BF16, w.T, w.frame_tokens, w.Tc,
                                               w.To), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)

    def step(ev_mid=None, ev_end=None):
        rb.forward_states(k, v, Wk, bk, workspace=ws, **kw)
        rb.forward_phiq(q, Wq, bq, workspace=ws, **kw)
        if ev_mid is not None:
            ev_mid.record(stream)
        rb.forward_attend(q, k, v, dims=d, frame_tokens=w.frame_tokens, Tc=w.Tc, To=w.To,
                          workspace=ws, out=out)
        if ev_end is not None:
            ev_end.record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    rb.sync_status(dev)

    K = args.steps
    mids = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(device_index_for_smi(dev))
    with sampler:
        rep.barrier()
        torch.cuda.synchronize(dev)
        start.record(stream)
        for i in range(K):
            step(mids[i], ends[i])
        stop.record(stream)
        torch.cuda.synchronize(dev)
        rep.barrier()
    rb.sync_status(dev)
    elapsed_ms = start.elapsed_time(stop)
    attn_ms = statistics.mean(mids[i].elapsed_time(ends[i]) for i in range(K))
    # states + phi_q phases of step i run between the end of step i-1 (or start) and mid of step i
    state_ms = statistics.mean((ends[i - 1].elapsed_time(mids[i]) if i else
                                start.elapsed_time(mids[0])) for i in range(K))
    elapsed_ms = rep.max(elapsed_ms, dev)

    # ---- end to end through the public API: pinned host inputs in, result out ----
    host = [x.pin_memory() for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk, inp.bk)]
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in host)
    d2h = out_h.numel() * out_h.element_size()

    def e2e_step():
        qd, kd, vd, Wqd, bqd, Wkd, bkd = (x.to(dev, non_blocking=True) for x in host)
        o = rb.forward(qd, kd, vd, Wqd, bqd, Wkd, bkd, workspace=ws, **kw)
        out_h.copy_(o, non_blocking=True)

    for _ in range(3):
        e2e_step()
    E = args.e2e_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    rep.barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    rep.barrier()
    rb.sync_status(dev)
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = rep.max(e2e_ms, dev)

    if rank == 0:
        peaks = read_peaks()
        ms_per_step = elapsed_ms / K
        flops_attn = w.attn_tensor_flops()
        achieved = flops_attn / (attn_ms * 1e-3) / 1e12
        line = {
            "metric": METRIC,
            "value": job_throughput(w.B * w.N, world, ms_per_step),
            "unit": UNIT,
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": ms_per_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": workload_config(w, world),
            "tflops": w.flops() * world / (ms_per_step * 1e-3) / 1e12,
            "frac_of_bf16_peak_step": w.flops() / (ms_per_step * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "kernel_ms": {"attention": attn_ms, "states_and_phiq": state_ms},
            "roofline": {"kernel": "hybrid_attn_bf16_kernel", "bound": "tensor",
                         "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"],
                         "peak_source": f"{peaks['source']} bf16 dense (burst)",
                         "frac_of_sustained": (achieved / peaks["bf16_tflops_sustained"]
                                               if peaks.get("bf16_tflops_sustained") else None),
                         "traffic": read_traffic()},
            "e2e": {"value": job_throughput(w.B * w.N, world, e2e_ms / E), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": 6 * K,  # per step: 2 weight preps, fold, scan, phi_q, attention
            "clocks": sampler.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(inp, w)
        print(json.dumps(line), flush=True)
    rep.close()


if __name__ == "__main__":
    main()
