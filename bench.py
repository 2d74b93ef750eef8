#!/usr/bin/env python
"""Benchmark of the ReHyAt hybrid attention forward on B200.

One step = one whole-sequence forward of the 480x832 5 s workload (B=1, 12 heads, D=128,
21 frames x 1560 tokens, Tc=3, To=1, P=2, F=128, G=8, bf16): the state folds with phi_k, their
prefix scan, phi_q, and the fused softmax + linear attention, through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload 480p5s|480p10s|720p5s|480p20s-stream] [--phi poly|elu1]
                    [--schedule FRAMES/OVERLAP,...] [--tc TC] [--to TO] [--p P]

The other workloads and options measure the remaining configurations: the streaming workload's
step is the whole chunk-by-chunk pass (27 calls per sequence, both sequences of the batch at
once) through the streaming session; --schedule gives it a variable chunk schedule (the first
entry once, the others cyclically, e.g. 5/0,3/1,3/2); --phi elu1 swaps the feature map;
--tc/--to/--p change the chunk length, overlap or part count (the ablation sweep).

N > 1 runs under torchrun: every rank runs its own replica of the workload (weak scaling, no
collective on the data path; NCCL only for the timing barrier and the max over ranks).
Prints one JSON line (rank 0).  `--impl reference` times the float64 CPU oracle on the same
workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
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
from hybrid_softmax_linear_chunked_b200.context_parallel import (  # noqa: E402
    ContextParallel, split_chunks)
from hybrid_softmax_linear_chunked_b200.head_parallel import HeadSharded  # noqa: E402
from hybrid_softmax_linear_chunked_b200.host_pipeline import HostPipeline  # noqa: E402
from hybrid_softmax_linear_chunked_b200.inputs import make_inputs  # noqa: E402
from hybrid_softmax_linear_chunked_b200.replicas import Replicas, job_throughput  # noqa: E402
from hybrid_softmax_linear_chunked_b200.streaming import ChunkStream  # noqa: E402

METRIC = "hybrid-attn query tokens/s (12 heads, D=128); % of dense BF16 tensor peak"
UNIT = "tokens/s"
WORKLOADS = {"480p5s": C.WAN_480P_5S, "480p10s": C.WAN_480P_10S, "720p5s": C.WAN_720P_5S,
             "480p20s-stream": C.WAN_480P_20S_STREAM}
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
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="480p5s")
    ap.add_argument("--phi", choices=["poly", "elu1"], default="poly")
    ap.add_argument("--pass", dest="which", choices=["forward", "backward"], default="forward",
                    help="backward: time the backward pass (the forward's out and row statistics "
                         "are computed before the timed region)")
    ap.add_argument("--schedule", default=None,
                    help="streaming only: FRAMES/OVERLAP entries, first once, rest cyclic")
    ap.add_argument("--tc", type=int, default=None, help="chunk length in frames (ablation)")
    ap.add_argument("--to", type=int, default=None, help="overlap frames (ablation)")
    ap.add_argument("--p", type=int, default=None, help="polynomial parts of phi (ablation)")
    ap.add_argument("--parallel", choices=["replicas", "context", "heads"], default="replicas",
                    help="replicas: every rank runs its own batch (weak scaling); context: the "
                         "ranks split one sequence into chunk ranges; heads: the ranks split the "
                         "(batch, head) problems of one batch and all-gather the outputs (both "
                         "strong scaling)")
    return ap.parse_args()


def pick_workload(args) -> C.Workload:
    w = WORKLOADS[args.workload]
    if args.phi != "poly":
        w = dataclasses.replace(w, phi=args.phi, P=1, name=w.name + ", elu+1 feature map")
    over = {k: v for k, v in (("Tc", args.tc), ("To", args.to), ("P", args.p)) if v is not None}
    if over:
        w = dataclasses.replace(w, name=w.name + ", " + " ".join(f"{k}={v}" for k, v in
                                                                  over.items()), **over)
    return w


def parse_schedule(spec: str | None, w: C.Workload):
    """(chunk_frames, overlap) per chunk covering w.T frames; None -> the uniform Tc / To."""
    if not spec:
        return [(e - s, w.To) for (_, s, e) in w.chunk_bounds()]
    items = [tuple(int(x) for x in it.split("/")) for it in spec.split(",")]
    out, t, i = [], 0, 0
    while t < w.T:
        cf, ov = items[i] if i == 0 or len(items) == 1 else items[1 + (i - 1) % (len(items) - 1)]
        cf = min(cf, w.T - t)
        out.append((cf, ov))
        t += cf
        i += 1
    return out


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


# ---------------------------------------------------------------------------------------------
# Launch counts: the library kernels each call enqueues, following the library's own decisions
# (which kernels a call needs, and when a chunk's lone last query tile is cut into parts)
# ---------------------------------------------------------------------------------------------

def _tiles(rows: int) -> int:
    return -(-rows // 128)


def lone_parts(L: int, Tc: int, To: int, frames_before: int, T: int, n_chunks: int) -> int:
    """Parts a whole-sequence or segment attention launch cuts its chunks' lone last query tiles
    into (1: no chunk has an odd tile count): up to 4, at most the fewest key tiles of a window
    that has one."""
    min_key = None
    for c in range(n_chunks):
        gs = frames_before + c * Tc
        ge = min(gs + Tc, frames_before + T)
        if _tiles((ge - gs) * L) % 2:
            k = _tiles((ge - max(0, gs - To)) * L)
            min_key = k if min_key is None else min(min_key, k)
    return 1 if min_key is None else max(1, min(4, min_key))


def forward_launches(w: C.Workload) -> int:
    """One whole-sequence bf16 forward (in one call or its three phases): the fold (when a chunk
    folds), the state scan, phi_q (when a chunk reads a state), the attention, and the lone-tile
    combine (when a lone tile is cut into parts)."""
    row_lin = (w.To // w.Tc + 1) * w.Tc * w.frame_tokens
    parts = lone_parts(w.frame_tokens, w.Tc, w.To, 0, w.T, w.n_chunks)
    return ((1 if w.n_chunks > 1 else 0) + 1 + (1 if row_lin < w.N else 0) + 1
            + (1 if parts > 1 else 0))


def segment_launches(w: C.Workload, c0: int, c1: int) -> int:
    """The two context-parallel calls of the chunk range [c0, c1): the fold (when the range folds)
    and the segment sum; then the scan, phi_q (when a chunk reads a state), the attention and
    the lone-tile combine."""
    L = w.frame_tokens
    n_fold = max(0, min(c1, w.n_chunks - 1) - c0)
    s0, s1 = c0 * w.Tc, min(c1 * w.Tc, w.T)
    row_lin = (max(w.To // w.Tc + 1, c0) - c0) * w.Tc * L
    parts = lone_parts(L, w.Tc, w.To, s0, s1 - s0, c1 - c0)
    return ((1 if n_fold else 0) + 1 + 1 + (1 if row_lin < (s1 - s0) * L else 0) + 1
            + (1 if parts > 1 else 0))


def backward_launches(w: C.Workload) -> int:
    """One bf16 backward pass: per chunk the dK/dV and dQ kernels (and, for a chunk with a
    linear region, a GEMM, the phi_q gradient, a GEMM and the r partial sums); the row
    statistics, the r reduction and the suffix sums; two GEMMs per group of folded frames; two
    feature-map backwards (per batch three GEMMs: U, dx, dW; then the feature gradient, the
    block-diagonal gradient, the column sums and the bias gradient); and the recomputed states
    and feature maps (two block-diagonal weight preparations, phi_q and phi_k, fold, scan)."""
    b = w.chunk_bounds()
    C_ = len(b)
    lin = sum(1 for (wf, _, _) in b if wf > 0)
    groups = sum(1 for c in range(C_ - 1) if b[c + 1][0] > b[c][0])
    return 2 * C_ + 4 * lin + 3 + 2 * groups + 2 * (3 * w.B + 4) + 6


def stream_call_launches(L: int, s: int, e: int, ov: int, nxt: int, cap: int) -> int:
    """One bf16 streaming call on frames [s, e) with overlap ov, next overlap nxt and a carry of
    cap frames: the S^T copy, phi_q (when the chunk reads a state), the attention, the fold (when
    frames leave the window), the lone-tile combine (odd query tile count), then the closing
    state add with the next carry copied in the same launch, or, for a chunk shorter than the
    carry, the state add (when it folded) and two carry gathers."""
    o = min(ov, s)
    wf = s - o
    fold = max(0, max(0, e - nxt) - wf) > 0
    q_tiles = _tiles((e - s) * L)
    key_tiles = _tiles(o * L) + _tiles((e - s) * L)
    n = 1 + (1 if wf > 0 else 0) + 1 + (1 if fold else 0)
    n += 1 if (q_tiles % 2 and min(4, key_tiles) > 1) else 0
    if e - s >= cap:
        n += 1 if (cap > 0 or fold) else 0
    else:
        n += (1 if fold else 0) + 2
    return n


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


def cpu_baseline(inp, w: C.Workload, out=None, budget_s: float = 28.0):
    """The oracle's recurrent (linear-cost) form, head by head, until `budget_s` has passed or all
    heads are done; tokens/s scaled to the whole workload (a token = one query position across
    all heads).  With `out` (the timed run's output, [B, H, N, D] on the device) the oracle's rows
    are also compared with it: relative L2 and max-abs per head and per chunk.  The row-sampled
    quadratic form (the check form) is timed on 64 rows as well."""
    import oracle.rehyat_oracle as O
    kind = O.PHI_ELU1 if w.phi == "elu1" else O.PHI_POLY
    t0 = time.perf_counter()
    heads, per_head, per_chunk, max_abs = 0, [], {}, 0.0
    L = w.frame_tokens
    for h in range(w.H):
        q, k, v = f64(inp.q[0, h]), f64(inp.k[0, h]), f64(inp.v[0, h])
        pq = O.feature_map(q, f64(inp.Wq[h]), f64(inp.bq[h]), w.P, kind)
        pk = O.feature_map(k, f64(inp.Wk[h]), f64(inp.bk[h]), w.P, kind)
        want = O.hybrid_attention_recurrent(q, k, v, pq, pk, L, w.Tc, w.To)
        heads += 1
        if out is not None:
            got = f64(out[0, h].cpu())
            per_head.append(float(np.linalg.norm(got - want) / np.linalg.norm(want)))
            max_abs = max(max_abs, float(np.abs(got - want).max()))
            for c, (_, s, e) in enumerate(w.chunk_bounds()):
                a, b = got[s * L:e * L], want[s * L:e * L]
                r = float(np.linalg.norm(a - b) / np.linalg.norm(b))
                per_chunk[c] = max(per_chunk.get(c, 0.0), r)
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    tokens = w.B * w.N * heads / w.H
    res = {"value": tokens / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
           "sample": f"float64 recurrent form, batch 0 heads 0-{heads - 1} of {w.H} (all "
                     f"{w.N} query rows each), {dt:.1f} s; scaled to query tokens of all heads"}
    rows = np.random.default_rng(0).integers(0, w.N, size=64)
    args_h = [f64(x) for x in (inp.q[0, 0], inp.k[0, 0], inp.v[0, 0], inp.Wq[0], inp.bq[0],
                               inp.Wk[0], inp.bk[0])]
    t1 = time.perf_counter()
    O.hybrid_attention_rows(*args_h, w.P, L, w.Tc, w.To, rows, kind)
    res["check_form"] = {"value": 64 / w.H / (time.perf_counter() - t1), "unit": UNIT,
                         "what": "quadratic form (explicit weight of every key), 64 random "
                                 "rows of head 0; a correctness tool, not a baseline"}
    if out is not None:
        res["parity_vs_timed_output"] = {
            "heads": heads, "rel_l2_per_head": per_head, "max_abs": max_abs,
            "rel_l2_per_chunk_worst_head": [per_chunk[c] for c in sorted(per_chunk)],
            "bounds": "rel-L2 <= 5e-3, max-abs <= 2e-2"}
    return res


def run_reference(args, rank: int):
    """Reference arm: the oracle as it stands, on host cores, one bounded sample per step."""
    if rank != 0:
        return
    import oracle.rehyat_oracle as O
    w = pick_workload(args)
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
        O.hybrid_attention_rows(q, k, v, Wq, bq, Wk, bk, w.P, w.frame_tokens, w.Tc, w.To, rows,
                                O.PHI_ELU1 if w.phi == "elu1" else O.PHI_POLY)

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
    w = pick_workload(args)
    context = args.parallel in ("context", "heads")
    if context and (args.which != "forward" or w.mode == "stream"):
        raise SystemExit(f"--parallel {args.parallel} times the whole-sequence forward")
    # context and head parallelism split one problem: every rank draws the same one
    inp = make_inputs(w, seed=w.seed if context else rep.seed(w.seed))
    if args.parallel == "heads":
        run = heads_runner(w, inp, dev, args, rep)
    elif context:
        run = context_runner(w, inp, dev, args, rep)
    elif args.which == "backward":
        run = backward_runner(w, inp, dev, args)
    else:
        run = (stream_runner if w.mode == "stream" else full_runner)(w, inp, dev, args)
    stream = torch.cuda.current_stream(dev)

    for _ in range(max(3, args.warmup)):
        run.step()
    rb.sync_status(dev)

    K = args.steps
    mids = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    sts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(device_index_for_smi(dev))
    with sampler:
        rep.barrier()
        torch.cuda.synchronize(dev)
        start.record(stream)
        for i in range(K):
            run.step(mids[i], ends[i], sts[i])
        stop.record(stream)
        torch.cuda.synchronize(dev)
        rep.barrier()
    rb.sync_status(dev)
    elapsed_ms = start.elapsed_time(stop)
    # the attention launch of step i runs between its mid and end events; the phases before it
    # between the end of step i-1 (or start) and the mid of step i
    attn_ms = statistics.mean(mids[i].elapsed_time(ends[i]) for i in range(K))
    pre_ms = statistics.mean((ends[i - 1].elapsed_time(mids[i]) if i else
                              start.elapsed_time(mids[0])) for i in range(K))
    phases = None
    if run.attn_isolated:
        # states (weight preps, fold, scan) from the end of step i-1 to its states event; phi_q
        # from there to the attention's start
        st_ms = statistics.mean((ends[i - 1].elapsed_time(sts[i]) if i else
                                 start.elapsed_time(sts[0])) for i in range(K))
        phi_ms = statistics.mean(sts[i].elapsed_time(mids[i]) for i in range(K))
        phases = {"states_ms": st_ms, "phiq_ms": phi_ms,
                  "states_gbs": run.states_bytes / (st_ms * 1e-3) / 1e9,
                  "phiq_gbs": run.phiq_bytes / (phi_ms * 1e-3) / 1e9,
                  "bytes": "algorithmic: states = K and V of the folded tokens (bf16); phi_q = "
                           "q rows in and phi_q rows out (bf16) of the chunks with a linear "
                           "region"}
    peak_mem = torch.cuda.max_memory_allocated(dev)
    elapsed_ms = rep.max(elapsed_ms, dev)

    # ---- end to end through the public API: pinned host inputs in, result out ----
    run.e2e_run(3)
    E = args.e2e_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    rep.barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    run.e2e_run(E)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    rep.barrier()
    rb.sync_status(dev)
    e2e_ms = rep.max(e0.elapsed_time(e1), dev)

    if rank == 0:
        peaks = read_peaks()
        ms_per_step = elapsed_ms / K
        kernel_time = attn_ms if run.attn_isolated else ms_per_step
        achieved = run.attn_flops / (kernel_time * 1e-3) / 1e12
        cfg = workload_config(w, world)
        cfg.update(run.config)
        # replicas: every rank processed its own batch; context: the ranks shared one
        units, ranks = (w.B * w.N, 1) if context else (w.B * w.N, world)
        if context:
            cfg["global_batch"] = w.B
        line = {
            "metric": METRIC,
            "value": job_throughput(units, ranks, ms_per_step),
            "unit": UNIT,
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": ms_per_step,
            "higher_is_better": True,
            "scaling": "strong" if context else "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": cfg,
            "tflops": run.step_flops * ranks / (ms_per_step * 1e-3) / 1e12,
            "frac_of_bf16_peak_step": run.step_flops / (ms_per_step * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "kernel_ms": ({"attention": attn_ms, "states_and_phiq": pre_ms} if run.attn_isolated
                          else {"step": ms_per_step}),
            "hbm_phases": phases,
            "peak_device_bytes": peak_mem,
            "roofline": {"kernel": run.roofline_kernel, "bound": "tensor",
                         "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"],
                         "peak_source": f"{peaks['source']} bf16 dense (burst)",
                         "frac_of_sustained": (achieved / peaks["bf16_tflops_sustained"]
                                               if peaks.get("bf16_tflops_sustained") else None),
                         "traffic": read_traffic() if run.attn_isolated and args.workload == "480p5s"
                                    and w.phi == "poly" else None},
            "e2e": {"value": job_throughput(units, ranks, e2e_ms / E), "unit": UNIT,
                    "h2d_bytes_per_step": run.h2d, "d2h_bytes_per_step": run.d2h},
            "gpu_launches": run.launches_per_step * K,
            "clocks": sampler.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            out_fn = getattr(run, "output", None)
            line["cpu_baseline"] = cpu_baseline(inp, w, out_fn() if out_fn else None)
        print(json.dumps(line), flush=True)
    rep.close()


class _Run:
    """What one timed step does, for one workload mode."""
    attn_isolated = True
    roofline_kernel = "hybrid_attn_bf16_kernel"
    config: dict = {}

    def e2e_run(self, n: int) -> None:
        """n end-to-end steps from host buffers (one after another unless a runner overlaps
        their copies)."""
        for _ in range(n):
            self.e2e_step()


def full_runner(w: C.Workload, inp, dev, args) -> _Run:
    """One whole-sequence forward: states, phi_q, then the attention (events around it)."""
    r = _Run()
    q, k, v = (x.to(dev) for x in (inp.q, inp.k, inp.v))
    Wq, bq, Wk, bk = (x.to(dev) for x in (inp.Wq, inp.bq, inp.Wk, inp.bk))
    kw = dict(P=w.P, phi=w.phi_code, frame_tokens=w.frame_tokens, Tc=w.Tc, To=w.To)
    d = rb.dims_of(q, Wq, w.P, w.phi_code)
    ws = torch.empty(rb.forward_workspace_size(d, rb.REHYAT_BF16, w.T, w.frame_tokens, w.Tc,
                                               w.To), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)

    def step(ev_mid=None, ev_end=None, ev_states=None):
        rb.forward_states(k, v, Wk, bk, workspace=ws, **kw)
        if ev_states is not None:
            ev_states.record(stream)
        rb.forward_phiq(q, Wq, bq, workspace=ws, **kw)
        if ev_mid is not None:
            ev_mid.record(stream)
        rb.forward_attend(q, k, v, dims=d, frame_tokens=w.frame_tokens, Tc=w.Tc, To=w.To,
                          workspace=ws, out=out)
        if ev_end is not None:
            ev_end.record(stream)

    host = [x.pin_memory() for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk, inp.bk)]
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    # end to end: every step uploads its inputs (q, k, v and the weights) from pinned host memory
    # and downloads its output; the upload of step i+1 and the download of step i-1 overlap the
    # forward of step i (HostPipeline)
    def e2e_compute(i, ins, o):
        rb.forward(*ins, workspace=ws, out=o, **kw)

    pipe = HostPipeline(e2e_compute, host, out, dev)
    r.step = step
    r.output = lambda: out
    r.e2e_run = lambda n: pipe.run([host] * n, [out_h] * n)
    r.h2d = sum(x.numel() * x.element_size() for x in host)
    r.d2h = out_h.numel() * out_h.element_size()
    r.attn_flops = w.attn_tensor_flops()
    r.step_flops = w.flops(streaming=False)
    r.launches_per_step = forward_launches(w)
    bnd = w.chunk_bounds()
    folded = bnd[-1][0] * w.frame_tokens                       # tokens folded (frames < w_{C-1})
    phiq_rows = sum((e - s) * w.frame_tokens for (wf, s, e) in bnd if wf > 0)
    r.states_bytes = w.B * w.H * folded * 2 * w.D * 2
    r.phiq_bytes = w.B * w.H * phiq_rows * (w.D + w.F) * 2
    return r


def backward_runner(w: C.Workload, inp, dev, args) -> _Run:
    """One backward pass over the whole sequence (dq, dk, dv, dW, db); the forward's output and
    row statistics and a seeded dL/dout are in HBM before the timed region."""
    r = _Run()
    r.attn_isolated = False
    q, k, v = (x.to(dev) for x in (inp.q, inp.k, inp.v))
    Wq, bq, Wk, bk = (x.to(dev) for x in (inp.Wq, inp.bq, inp.Wk, inp.bk))
    kw = dict(P=w.P, phi=w.phi_code, frame_tokens=w.frame_tokens, Tc=w.Tc, To=w.To)
    out, lse = rb.forward_train(q, k, v, Wq, bq, Wk, bk, **kw)
    dout = torch.randn(out.shape, generator=torch.Generator().manual_seed(w.seed + 1)).to(
        torch.bfloat16).to(dev)
    d = rb.dims_of(q, Wq, w.P, w.phi_code)
    ws = torch.empty(rb.backward_workspace_size(d, rb.REHYAT_BF16, w.T, w.frame_tokens, w.Tc,
                                                w.To), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev_mid=None, ev_end=None, ev_states=None):
        if ev_mid is not None:
            ev_mid.record(stream)
        rb.backward(q, k, v, Wq, bq, Wk, bk, out, lse, dout, workspace=ws, **kw)
        if ev_end is not None:
            ev_end.record(stream)

    host = [x.pin_memory() for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk, inp.bk)]
    host += [out.cpu().pin_memory(), lse.cpu().pin_memory(), dout.cpu().pin_memory()]
    # end to end: every step uploads q, k, v, the weights, out, the row statistics and dL/dout
    # and downloads the seven gradients; copies overlap the computation (HostPipeline)
    shapes = {"dq": q.shape, "dk": q.shape, "dv": q.shape, "dWq": Wq.shape, "dWk": Wk.shape,
              "dbq": (w.H, w.F), "dbk": (w.H, w.F)}
    grad_like = [torch.empty(shapes[n], dtype=torch.float32, device=dev) for n in rb.GRAD_NAMES]
    grads_h = [torch.empty(g.shape, dtype=g.dtype).pin_memory() for g in grad_like]

    def e2e_compute(i, ins, outs):
        rb.backward(*ins, workspace=ws, grads=dict(zip(rb.GRAD_NAMES, outs)), **kw)

    pipe = HostPipeline(e2e_compute, host, grad_like, dev)
    r.step = step
    r.e2e_run = lambda n: pipe.run([host] * n, [grads_h] * n)
    r.h2d = sum(x.numel() * x.element_size() for x in host)
    r.d2h = 3 * q.numel() * 4 + 2 * Wq.numel() * 4 + 2 * w.H * w.F * 4
    r.attn_flops = w.backward_flops()
    r.step_flops = w.backward_flops()
    r.launches_per_step = backward_launches(w)
    r.roofline_kernel = "backward pass (all launches; algorithmic FLOPs / time)"
    r.config = {"pass": "backward"}
    return r


def context_runner(w: C.Workload, inp, dev, args, rep) -> _Run:
    """The whole-sequence forward split into chunk ranges over the ranks (context parallelism):
    each rank holds its own frames of q, k, v; per step the halo frames go point to point, the
    segment sums are all-gathered, and each rank computes its chunks' outputs."""
    r = _Run()
    r.attn_isolated = False
    L = w.frame_tokens
    Wq, bq, Wk, bk = (x.to(dev) for x in (inp.Wq, inp.bq, inp.Wk, inp.bk))
    cp = ContextParallel(Wq, bq, Wk, bk, T=w.T, frame_tokens=L, Tc=w.Tc, To=w.To, P=w.P,
                         phi=w.phi_code)
    own = slice(cp.s0 * L, cp.s1 * L)
    q_own = inp.q[:, :, own].contiguous().to(dev)
    k_buf, v_buf = cp.kv_buffer(q_own), cp.kv_buffer(q_own)
    cp.own(k_buf).copy_(inp.k[:, :, own])
    cp.own(v_buf).copy_(inp.v[:, :, own])
    out = torch.empty_like(q_own)
    stream = torch.cuda.current_stream(dev)

    def step(ev_mid=None, ev_end=None, ev_states=None):
        if ev_mid is not None:
            ev_mid.record(stream)
        cp.forward(q_own, k_buf, v_buf, out=out)
        if ev_end is not None:
            ev_end.record(stream)

    host = [inp.q[:, :, own].contiguous().pin_memory(), inp.k[:, :, own].contiguous().pin_memory(),
            inp.v[:, :, own].contiguous().pin_memory()]
    host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def e2e_step():
        q_own.copy_(host[0], non_blocking=True)
        cp.own(k_buf).copy_(host[1], non_blocking=True)
        cp.own(v_buf).copy_(host[2], non_blocking=True)
        cp.forward(q_own, k_buf, v_buf, out=out)
        host_out.copy_(out, non_blocking=True)

    r.step, r.e2e_step = step, e2e_step
    r.h2d = sum(x.numel() * x.element_size() for x in host)
    r.d2h = host_out.numel() * host_out.element_size()
    r.step_flops = w.flops(streaming=False)
    r.attn_flops = w.flops(streaming=False)
    r.launches_per_step = segment_launches(w, cp.c0, cp.c1)  # this rank's
    r.roofline_kernel = "context-parallel forward step (whole-sequence FLOPs / step time)"
    r.config = {"parallelism": f"cp{rep.world} (chunk ranges [c0, c1) per rank: "
                               f"{split_chunks(w.n_chunks, rep.world)}; halo point to point, "
                               "segment sums all-gathered)"}
    return r


def heads_runner(w: C.Workload, inp, dev, args, rep) -> _Run:
    """The whole-sequence forward with the B*H (batch, head) problems split over the ranks: each
    rank holds its units' q, k, v, runs the library forward on them, and the output slices are
    all-gathered so that every rank ends with the whole output."""
    r = _Run()
    r.attn_isolated = False
    Wq, bq, Wk, bk = (x.to(dev) for x in (inp.Wq, inp.bq, inp.Wk, inp.bk))
    hs = HeadSharded(Wq, bq, Wk, bk, B=w.B, H=w.H, frame_tokens=w.frame_tokens, Tc=w.Tc,
                     To=w.To, P=w.P, phi=w.phi_code)
    host = [hs.shard(x).contiguous().pin_memory() for x in (inp.q, inp.k, inp.v)]
    q_s, k_s, v_s = (x.to(dev) for x in host)
    out_s = torch.empty_like(q_s)
    stream = torch.cuda.current_stream(dev)
    full = [None]

    def step(ev_mid=None, ev_end=None, ev_states=None):
        if ev_mid is not None:
            ev_mid.record(stream)
        hs.forward(q_s, k_s, v_s, out=out_s)
        full[0] = hs.gather(out_s)
        if ev_end is not None:
            ev_end.record(stream)

    host_out = torch.empty((w.B, w.H, w.N, w.D), dtype=q_s.dtype).pin_memory()

    def e2e_step():
        for d_, h_ in zip((q_s, k_s, v_s), host):
            d_.copy_(h_, non_blocking=True)
        hs.forward(q_s, k_s, v_s, out=out_s)
        host_out.copy_(hs.gather(out_s), non_blocking=True)

    r.step, r.e2e_step = step, e2e_step
    r.output = lambda: full[0]
    r.h2d = sum(x.numel() * x.element_size() for x in host)
    r.d2h = host_out.numel() * host_out.element_size()
    r.step_flops = w.flops(streaming=False)
    r.attn_flops = w.flops(streaming=False)
    r.launches_per_step = forward_launches(w)  # this rank's forward (the all-gather is NCCL's)
    r.roofline_kernel = "head-sharded forward step (whole-problem FLOPs / step time)"
    r.config = {"parallelism": f"heads{rep.world} ((batch, head) units per rank: "
                               f"{hs.ranges}; output slices all-gathered)"}
    return r


def sched_bounds(sched):
    """(w, s, e, overlap, next overlap) per chunk of a (frames, overlap) schedule."""
    out, s = [], 0
    for c, (cf, ov) in enumerate(sched):
        nxt = sched[c + 1][1] if c + 1 < len(sched) else ov
        out.append((max(0, s - ov), s, s + cf, ov, nxt))
        s += cf
    return out


def stream_runner(w: C.Workload, inp, dev, args) -> _Run:
    """The whole sequence fed chunk by chunk through the streaming session (every sequence of
    the batch at once); the inputs sit in HBM already split into chunks."""
    r = _Run()
    r.attn_isolated = False
    sched = parse_schedule(args.schedule, w)
    bounds = sched_bounds(sched)
    L = w.frame_tokens
    Wq, bq, Wk, bk = (x.to(dev) for x in (inp.Wq, inp.bq, inp.Wk, inp.bk))
    chunks = [[x[:, :, s * L:e * L].contiguous().to(dev) for x in (inp.q, inp.k, inp.v)]
              for (_, s, e, _, _) in bounds]
    outs = [torch.empty_like(c[0]) for c in chunks]
    sess = ChunkStream(Wq, bq, Wk, bk, B=w.B, P=w.P, phi=w.phi_code, frame_tokens=L,
                       Tc=max(cf for cf, _ in sched), To=max(ov for _, ov in sched))
    stream = torch.cuda.current_stream(dev)

    def step(ev_mid=None, ev_end=None, ev_states=None):
        if ev_mid is not None:
            ev_mid.record(stream)
        sess.reset()
        for c, (_, _, _, ov, nxt) in enumerate(bounds):
            sess.step(*chunks[c], out=outs[c], To=ov, To_next=nxt)
        if ev_end is not None:
            ev_end.record(stream)

    host = [[x[:, :, s * L:e * L].contiguous().pin_memory() for x in (inp.q, inp.k, inp.v)]
            for (_, s, e, _, _) in bounds]
    host_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]

    def e2e_step():
        sess.reset()
        for c, (_, _, _, ov, nxt) in enumerate(bounds):
            qd, kd, vd = (x.to(dev, non_blocking=True) for x in host[c])
            o = sess.step(qd, kd, vd, To=ov, To_next=nxt)
            host_out[c].copy_(o, non_blocking=True)

    # with equal chunk shapes the calls' uploads and downloads overlap the computation
    # (HostPipeline, one step per call; the session restarts at every sequence)
    same_shape = all(h[0].shape == host[0][0].shape for h in host)
    if same_shape:
        n_calls = len(bounds)

        def e2e_compute(i, ins, o):
            c = i % n_calls
            if c == 0:
                sess.reset()
            _, _, _, ov, nxt = bounds[c]
            sess.step(*ins, out=o, To=ov, To_next=nxt)

        pipe = HostPipeline(e2e_compute, host[0], outs[0], dev)
        r.e2e_run = lambda n: pipe.run(host * n, host_out * n)

    # algorithmic work of the schedule: softmax over each window, readout of chunks with a linear
    # region, every fold (the streaming calls fold after every chunk), and the feature maps
    D, F = w.D, w.F
    attn = step_f = 0.0
    launches = 0
    cap = max(ov_ for _, ov_ in sched)  # the session's carry
    for (wf, s, e, ov, nxt) in bounds:
        nq, nw = (e - s) * L, (e - wf) * L
        attn += 4.0 * nq * nw * D + (2.0 * nq * F * D if wf > 0 else 0.0)
        fold = max(0, max(0, e - nxt) - wf) * L
        step_f += (2.0 * nq * F + (2.0 * nq * D * F / w.G) if wf > 0 else 0.0)
        step_f += fold * (2.0 * F * D + F + 2.0 * D * F / w.G)
        launches += stream_call_launches(L, s, e, ov, nxt, cap)
    r.attn_flops = attn * w.B * w.H
    r.step_flops = (attn + step_f) * w.B * w.H
    r.step, r.e2e_step = step, e2e_step
    if not args.schedule:
        r.output = lambda: torch.cat(outs, dim=2)
    r.h2d = sum(x.numel() * x.element_size() for c in host for x in c)
    r.d2h = sum(o.numel() * o.element_size() for o in host_out)
    r.launches_per_step = launches
    r.roofline_kernel = "whole streaming step (attention FLOPs / step time)"
    r.config = {"mode": "stream", "calls_per_step": len(bounds),
                "schedule": [[cf, ov] for cf, ov in sched]}
    return r


if __name__ == "__main__":
    main()
