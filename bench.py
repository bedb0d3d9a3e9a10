"""Benchmark of one Matryoshka-suite hot-path step on B200.

A step is one pass of the whole path over one batch of synthetic input:
    junction fwd (block m -> m+1, for m < M)
    multi-exit loss fwd (per-exit CE + distillation from the largest exit)
    multi-exit loss bwd (dh_m, dW^m)
    junction bwd (do_m, de rows, deterministic dE scatter), fed with dh_{m+1}
    as the incoming gradient of block m+1's input (the blocks themselves are
    not part of this path).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload main3] [--impl ours|reference]

Prints one JSON line (rank 0).  Under torchrun every rank runs its own batch
(weak scaling, no collective on the data path) and the reported time is the
max over ranks.  ``--impl reference`` times the fp64 CPU oracle on a bounded
sample of the same workload instead.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from lm_head_loss_junction_b200 import workloads as wl  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK), "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.thread = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            if self.thread is not None:
                self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def cublas_calibration(step, run_loss_fwd, run_loss_bwd, stream, device, seconds=1.0):
    """cuBLAS GEMMs of the loss's shapes (torch.matmul: the same bf16 operands,
    fp32 accumulation, bf16 out) against the library's calls, each repeated
    for about `seconds` (a sustained load under the power cap, like the
    step), interleaved twice, with the SM clock sampled during each.
    Forward: the logits GEMM of every exit against mls_multiexit_loss_fwd.
    Backward: per exit the logits GEMM, G W (dh) and G^T h (dW), with the
    logits standing in for G, against mls_multiexit_loss_bwd.  A same-box,
    same-clock denominator; cuBLAS is timed here only, never on the path."""
    c = step.cfg
    outs = [torch.empty(c.T, c.V, dtype=torch.bfloat16, device=device) for _ in range(c.M)]
    dh = [torch.empty(c.T, d, dtype=torch.bfloat16, device=device) for d in c.D]
    dW = [torch.empty(c.V, d, dtype=torch.bfloat16, device=device) for d in c.D]

    def cublas():
        for m in range(c.M):
            torch.matmul(step.o[m], step.W[m].t(), out=outs[m])

    def cublas_bwd():
        for m in range(c.M):
            torch.matmul(step.o[m], step.W[m].t(), out=outs[m])
            torch.matmul(outs[m], step.W[m], out=dh[m])
            torch.matmul(outs[m].t(), step.o[m], out=dW[m])

    flops = 2.0 * c.T * c.V * sum(c.D)

    def sustained(fn):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize(device)
        n = max(3, int(seconds * 1000.0 / max(e0.elapsed_time(e1), 1e-3)))
        with ClockSampler(device.index) as clk:
            e0.record(stream)
            for _ in range(n):
                fn()
            e1.record(stream)
            torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) / n, clk.summary()["sm_mhz"]

    arms = {"cublas": [], "loss_fwd": [], "cublas_bwd": [], "loss_bwd": []}
    for _ in range(2):
        arms["cublas"].append(sustained(cublas))
        arms["loss_fwd"].append(sustained(run_loss_fwd))
        arms["cublas_bwd"].append(sustained(cublas_bwd))
        arms["loss_bwd"].append(sustained(run_loss_bwd))
    del outs, dh, dW
    out = {"what": "cuBLAS bf16 GEMMs of the loss's shapes (forward: the logits of every exit; backward: "
                   "logits, dh and dW of every exit) against mls_multiexit_loss_fwd / _bwd, each sustained "
                   "for ~1 s, interleaved twice"}
    for k, v in arms.items():
        ms = statistics.mean(t for t, _ in v)
        mhz = [f for _, f in v if f is not None]
        n = 3.0 if k.endswith("bwd") else 1.0
        out[k] = {"ms": ms, "tflops": n * flops / (ms / 1000.0) / 1e12,
                  "sm_mhz": statistics.mean(mhz) if mhz else None}
    out["loss_fwd_vs_cublas"] = out["cublas"]["ms"] / out["loss_fwd"]["ms"]
    out["loss_bwd_vs_cublas"] = out["cublas_bwd"]["ms"] / out["loss_bwd"]["ms"]
    return out


# ---------------------------------------------------------------- the step
class Step:
    """Device-resident inputs, outputs and workspaces of one hot-path step."""

    def __init__(self, cfg: wl.SuiteConfig, device, seed_offset: int = 0, bwd_ws_bytes: int = 0):
        import dataclasses
        from lm_head_loss_junction_b200 import api
        self.api = api
        self.cfg = dataclasses.replace(cfg, seed=cfg.seed + seed_offset)
        c = self.cfg
        d = wl.make_inputs(c)
        self.host = d
        self.dev = device
        self.x = torch.from_numpy(d.x).to(device)
        self.y = torch.from_numpy(d.y).to(device)
        self.o = [t.to(device) for t in d.o]
        self.E = [t.to(device) for t in d.E]
        self.W = [t.to(device) for t in d.W]
        dt = self.o[0].dtype
        T, V, M = c.T, c.V, c.M
        self.jy = [torch.empty((T, c.D[j + 1]), dtype=dt, device=device) for j in range(M - 1)]
        self.jscale = [torch.empty(T, dtype=torch.float32, device=device) for _ in range(M - 1)]
        self.losses = torch.empty(2 * M, dtype=torch.float32, device=device)
        self.stats = torch.empty((3 * M - 1, T), dtype=torch.float32, device=device)
        self.dh = [torch.empty_like(t) for t in self.o]
        self.dW = [torch.empty((V, c.D[m]), dtype=torch.float32, device=device) for m in range(M)]
        self.do = [torch.empty_like(self.o[j]) for j in range(M - 1)]
        self.de = [torch.empty((T, c.deltas[j + 1]), dtype=dt, device=device) for j in range(M - 1)]
        self.dE = [torch.empty((V, c.deltas[j + 1]), dtype=torch.float32, device=device) for j in range(M - 1)]
        fb, bb = api.multiexit_loss_workspace(T, list(c.D), V, dt)
        bb = bwd_ws_bytes or bb               # the query's bounded size unless asked otherwise
        self.ws_loss = torch.empty(max(fb, bb), dtype=torch.uint8, device=device)
        self.bwd_plan = api.multiexit_loss_bwd_plan(T, list(c.D), V, dt, max(fb, bb))
        self.ws_j = torch.empty(api.junction_bwd_multi_workspace(T, V, M - 1) if M > 1 else 1, dtype=torch.uint8,
                                device=device)
        self.status = api.new_status(device)

    def phases(self):
        """The step as four stream-ordered callables f(stream): junction fwd,
        loss fwd, loss bwd, junction bwd (fed with dh_{m+1})."""
        a, c = self.api, self.cfg
        M = c.M

        def junction_fwd(stream):
            if M > 1:    # every junction of the suite in one call (one launch for bf16)
                a.junction_fwd_multi(self.x, self.o[:M - 1], self.E[1:], out=self.jy, scale_out=self.jscale,
                                     status=self.status, stream=stream)

        def loss_fwd(stream):
            a.multiexit_loss_fwd(self.y, self.o, self.W, c.alpha_d, losses=self.losses, stats=self.stats,
                                 workspace=self.ws_loss, status=self.status, stream=stream)

        def loss_bwd(stream):
            a.multiexit_loss_bwd(self.y, self.o, self.W, self.stats, c.alpha_d, 1.0, dh=self.dh, dW=self.dW,
                                 workspace=self.ws_loss, status=self.status, stream=stream)

        def junction_bwd(stream):
            if M > 1:    # every junction in one call: one id grouping for all table gradients
                a.junction_bwd_multi(self.x, self.o[:M - 1], self.E[1:], self.dh[1:], do_out=self.do,
                                     de_out=self.de, dE=self.dE, accumulate_dE=False, workspace=self.ws_j,
                                     status=self.status, stream=stream)

        return [junction_fwd, loss_fwd, loss_bwd, junction_bwd]

    def run(self, stream=None):
        for f in self.phases():
            f(stream)

    def working_set_gb(self):
        ts = [self.x, self.y] + self.o + self.E[1:] + self.W + self.dh + self.dW + self.jy + self.do + self.de + \
            self.dE
        return (sum(t.numel() * t.element_size() for t in ts) + self.ws_loss.numel()) / 1e9

    # algorithmic work
    def loss_flops_algorithmic(self):
        c = self.cfg
        return 6.0 * c.T * c.V * sum(c.D)

    def loss_flops_executed(self):
        c = self.cfg
        return 8.0 * c.T * c.V * sum(c.D)

    def junction_bytes(self):
        """(forward, backward) algorithmic HBM bytes over all junctions of the step.

        Backward: the row pass (dy, o, e row in; do, de rows, coefficient out;
        id) plus the table gradient in overwrite mode: every row of each fp32
        table dE written once, and the g_e part of dy and the coefficients
        read again by the id-grouped sums.  (The embedding rows of the ids
        present are read again too; not counted, so the rate is a lower bound.)"""
        c = self.cfg
        b = 2 if c.dtype == "bf16" else 4
        fwd = bwd = 0
        for j in range(c.M - 1):
            D, dl, Dn = c.D[j], c.deltas[j + 1], c.D[j + 1]
            fwd += c.T * ((D + dl + Dn) * b + 4 + 4)                 # o, e row, y; id; scale
            bwd += c.T * ((Dn + D + dl + D + dl) * b + 4 + 4)        # dy, o, e row, do, de; id; coef
            bwd += c.V * dl * 4 + c.T * (dl * b + 4)                 # dE table; g_e and coef re-read
        return fwd, bwd


def measured_traffic(cfg):
    """DRAM bytes per launch of the forward loss tile kernel from the committed
    ncu capture, or None when the capture is for another workload or the kernel
    source has changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic_loss_tile_stats_main3_T8192.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        src = os.path.join(ROOT, rec["source"])
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except Exception:
        return None
    if sha != rec["source_sha256_16"] or cfg.name != wl.CONFIGS["main3"].name:
        return None
    return rec["dram_bytes_read_per_launch"] + rec["dram_bytes_write_per_launch"]


def _dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def grad_sync(tensors, mode: str, ws: int, shards=None):
    """Data-parallel exchange of the step's parameter gradients (dW^m of every
    head, dE of every residual table) over the process group: "allreduce" sums
    them on every rank; "reduce_scatter" leaves rank r the sum of its 1/ws
    slice of each flattened gradient (a sharded optimizer's input) in
    shards[i].  Every rank issues the same collectives in the same order."""
    if ws == 1 or mode == "none":
        return
    import torch.distributed as dist
    for i, t in enumerate(tensors):
        if mode == "allreduce":
            dist.all_reduce(t)
        else:
            dist.reduce_scatter_tensor(shards[i], t.view(-1))


def grad_shards(tensors, ws: int):
    """Output buffers of the reduce-scatter (each flattened gradient must split evenly)."""
    for t in tensors:
        if t.numel() % ws:
            raise ValueError(f"gradient of {t.numel()} elements does not split over {ws} ranks")
    return [torch.empty(t.numel() // ws, dtype=t.dtype, device=t.device) for t in tensors]


def _max_over_ranks(v: float, ws: int, device) -> float:
    if ws == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_oracle_sample(d: wl.SuiteInputs, n_tokens: int):
    """Times the fp64 oracle on the first n_tokens tokens of the workload (full
    V and full dW work for those tokens, both junctions).  Returns (seconds, tokens)."""
    import oracle
    c = d.cfg
    rows = np.arange(n_tokens)
    sub_o = [t[:n_tokens] for t in d.o]
    t0 = time.perf_counter()
    for j in range(c.M - 1):
        oracle.junction_fwd(d.x[rows], sub_o[j], d.E[j + 1])
    r = oracle.multiexit_loss(d.y[:n_tokens], sub_o, d.W, alpha_d=c.alpha_d, grad_scale=1.0)
    for j in range(c.M - 1):
        oracle.junction_bwd(d.x[rows], sub_o[j], d.E[j + 1], r["dh"][j + 1])
    return time.perf_counter() - t0, n_tokens


def measure_workload(name, device, stream, peaks, K, eager, cpu_tokens):
    """One of the other workloads at its full size: the same step (junctions
    fwd, loss fwd, loss bwd, junctions bwd), captured and replayed the same way,
    K timed steps with CUDA events between phases; its loss-forward roofline
    fraction; and the fp64 oracle timed on the first cpu_tokens tokens on the
    host cores.  Returns a dict for the bench line's extras."""
    cfg = wl.CONFIGS[name]
    step = Step(cfg, device)
    for _ in range(3):
        step.run(stream)
    torch.cuda.synchronize(device)
    code, word = step.api.status_read(step.status, stream)
    if code != 0:
        raise RuntimeError(f"{name}: device status after warm-up: {code} ({word})")
    fns = step.phases()
    if eager:
        runners = [lambda f=f: f(stream) for f in fns]
        graphs = []
    else:
        graphs = []
        for f in fns:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="relaxed"):
                f(None)
            graphs.append(g)
        runners = [g.replay for g in graphs]
    for _ in range(2):
        for r in runners:
            r()
    torch.cuda.synchronize(device)
    marks = [[torch.cuda.Event(enable_timing=True) for _ in range(len(runners) + 1)] for _ in range(K)]
    with ClockSampler(device.index) as clocks:
        for k in range(K):
            for i, r in enumerate(runners):
                marks[k][i].record(stream)
                r()
            marks[k][-1].record(stream)
        torch.cuda.synchronize(device)
    ms = [statistics.mean(marks[k][i].elapsed_time(marks[k][i + 1]) for k in range(K)) for i in range(len(runners))]
    code, word = step.api.status_read(step.status, stream)
    if code != 0:
        raise RuntimeError(f"{name}: device status after timing: {code} ({word})")
    c = step.cfg
    ms_step = sum(ms)
    fl_fwd = 2.0 * c.T * c.V * sum(c.D)
    out = {"workload": c.name, "T": c.T, "steps": K, "ms_per_step": ms_step,
           "tokens_per_s": c.T / (ms_step / 1000.0),
           "phases_ms": {"junction_fwd": ms[0], "loss_fwd": ms[1], "loss_bwd": ms[2], "junction_bwd": ms[3]},
           "loss_bwd_pieces": {"token_block": step.bwd_plan[0], "vocab_chunk": step.bwd_plan[1]}}
    if c.dtype == "bf16":
        peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
        out["roofline"] = {"bound": "tensor", "kernel": "loss_tile_kernel<stats> (mls_multiexit_loss_fwd call)",
                           "achieved": fl_fwd / (ms[1] / 1000.0) / 1e12, "peak": peak, "unit": "TFLOP/s",
                           "frac": fl_fwd / (ms[1] / 1000.0) / 1e12 / peak}
        out["loss_executed_frac_of_peak"] = step.loss_flops_executed() / ((ms[1] + ms[2]) / 1000.0) / 1e12 / peak
    else:
        peak_fma = 148 * 128 * 2 * 1.965e9 / 1e12
        out["roofline"] = {"bound": "alu", "kernel": "simt_stats_kernel (fp32 CUDA-core path)",
                           "achieved": fl_fwd / (ms[1] / 1000.0) / 1e12, "peak": peak_fma, "unit": "TFLOP/s",
                           "frac": fl_fwd / (ms[1] / 1000.0) / 1e12 / peak_fma}
    if c.M > 1:
        jf, jb = step.junction_bytes()
        out["junction_fwd_frac_of_hbm"] = jf / (ms[0] / 1000.0) / 1e9 / peaks["hbm_gbs"]
        out["junction_bwd_frac_of_hbm"] = jb / (ms[3] / 1000.0) / 1e9 / peaks["hbm_gbs"]
    out["clocks"] = clocks.summary()
    n = min(cpu_tokens, c.T)
    sec, n = cpu_oracle_sample(step.host, n)
    out["cpu_baseline"] = {"value": n / sec, "unit": "tokens/s", "cores": _cores(), "kind": "oracle",
                           "sample": f"first {n} tokens: junctions fwd+bwd and the {c.M}-exit loss fwd+bwd over "
                                     f"the full vocabulary, fp64 numpy ({sec:.1f} s)"}
    del graphs, runners, step
    torch.cuda.empty_cache()
    return out


def _cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 1) for i in info if i.get("internal_api") in ("openblas", "mkl", "blis")),
                default=None)
        if n:
            return int(n)
    except Exception:
        pass
    return os.cpu_count()


def run_reference(args, cfg):
    ws, rank, _ = _dist_env()
    if rank != 0:
        return
    n = args.ref_tokens
    d = wl.make_inputs(cfg)
    times = []
    for i in range(args.warmup + args.steps):
        sec, _ = cpu_oracle_sample(d, n)
        if i >= args.warmup:
            times.append(sec)
    tot = sum(times)
    value = n * len(times) / tot
    line = {
        "impl": "reference", "metric": "multi-exit head-loss fwd+bwd tokens/s (1 B200) and % bf16 tensor peak; "
        "junction GB/s", "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * tot / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, **cfg.describe(), "sample_tokens_per_step": n},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": _cores(), "kind": "oracle",
                         "sample": f"first {n} tokens of {cfg.name} per step: both junctions fwd+bwd and the "
                                   f"{cfg.M}-exit loss fwd+bwd over the full vocabulary, fp64 numpy"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="main3", choices=wl.CONFIG_ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-tokens", type=int, default=64)
    ap.add_argument("--cpu-tokens", type=int, default=256)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--tokens", type=int, default=0,
                    help="run the workload with this many tokens per GPU instead of its own batch")
    ap.add_argument("--eager", action="store_true",
                    help="launch every step from Python instead of replaying a captured CUDA graph")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other four workloads (measured after the headline on one GPU by default)")
    ap.add_argument("--bwd-ws-gb", type=float, default=0.0,
                    help="workspace of the loss backward call in GB (default: the size the workspace query "
                         "returns); a larger one lets the call use fewer token blocks and vocabulary chunks")
    ap.add_argument("--grad-sync", default="none", choices=["none", "allreduce", "reduce_scatter"],
                    help="with more than one rank, exchange dW and dE over NCCL inside every step")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    cfg = wl.CONFIGS[args.workload]
    if args.tokens:
        seq = min(cfg.seq, args.tokens)
        cfg = wl.small_variant(cfg, batch=max(1, args.tokens // seq), seq=seq, name_suffix=f"T{args.tokens}")

    if args.impl == "reference":
        run_reference(args, cfg)
        return

    ws, rank, local = _dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    from lm_head_loss_junction_b200 import _lib
    step = Step(cfg, device, seed_offset=rank, bwd_ws_bytes=int(args.bwd_ws_gb * 1e9))
    stream = torch.cuda.current_stream(device)
    peaks, peak_kind = load_peaks()

    def barrier():
        if ws > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(device)

    for _ in range(args.warmup):
        step.run(stream)
    barrier()
    code, word = step.api.status_read(step.status, stream)
    if code != 0:
        raise RuntimeError(f"device status after warm-up: {code} ({word})")
    l0 = _lib.lib().mls_kernel_launches()
    step.run(stream)
    launches_per_step = _lib.lib().mls_kernel_launches() - l0

    # The four phases of a step, each captured once as a CUDA graph and
    # replayed (the library launches only stream-ordered work), so the timed
    # region carries no Python launch overhead.  --eager launches from Python.
    phase_fns = step.phases()
    if args.eager:
        runners = [lambda f=f: f(stream) for f in phase_fns]
    else:
        graphs = []
        for f in phase_fns:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="relaxed"):
                f(None)
            graphs.append(g)
        runners = [g.replay for g in graphs]
    # the data-parallel gradient exchange (eager NCCL calls), when asked for
    sync_on = ws > 1 and args.grad_sync != "none"
    grads = step.dW + step.dE
    shards = grad_shards(grads, ws) if sync_on and args.grad_sync == "reduce_scatter" else None
    if sync_on:
        runners.append(lambda: grad_sync(grads, args.grad_sync, ws, shards))
    for _ in range(2):
        for r in runners:
            r()
    barrier()

    # ---------------- timed region: K steps, events between phases
    K = args.steps
    NP = len(runners)
    marks = [[torch.cuda.Event(enable_timing=True) for _ in range(NP + 1)] for _ in range(K)]
    barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        start.record(stream)
        for k in range(K):
            for i, r in enumerate(runners):
                marks[k][i].record(stream)
                r()
            marks[k][NP].record(stream)
        end.record(stream)
        barrier()
    launches = launches_per_step * K
    ms_total = start.elapsed_time(end)
    ms_total = _max_over_ranks(ms_total, ws, device)
    ms_step = ms_total / K
    phase_ms = [statistics.mean(marks[k][i].elapsed_time(marks[k][i + 1]) for k in range(K)) for i in range(NP)]
    code, word = step.api.status_read(step.status, stream)
    if code != 0:
        raise RuntimeError(f"device status after timing: {code} ({word})")

    c = step.cfg
    tokens_all = c.T * ws
    value = tokens_all * K / (ms_total / 1000.0)

    # ---------------- end to end through the public API with host buffers
    # Every step's inputs (x, y, o_m) come from pinned host memory and its losses
    # go back to pinned host memory.  The host-to-device copy of step k+1 runs on
    # a copy stream into a staging buffer while step k computes (as a training
    # loop would prefetch its next batch); each step starts with a device-side
    # copy from the staging buffer into the step's input buffers.  The first
    # copy is not overlapped; exactly K copies are made.
    e2e = None
    if not args.no_e2e:
        host_in = [torch.from_numpy(step.host.x).pin_memory(), torch.from_numpy(step.host.y).pin_memory()] + \
                  [t.pin_memory() for t in step.host.o]
        dev_in = [step.x, step.y] + step.o
        stage = [torch.empty_like(t) for t in dev_in]
        host_out = torch.empty(step.losses.shape, dtype=torch.float32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host_in)
        d2h = host_out.numel() * host_out.element_size()
        copy_stream = torch.cuda.Stream(device)
        ev_staged = torch.cuda.Event()
        ev_consumed = torch.cuda.Event()

        def h2d_to_stage():
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(ev_consumed)          # the staging buffer is free
                for hsrc, sdst in zip(host_in, stage):
                    sdst.copy_(hsrc, non_blocking=True)
                ev_staged.record(copy_stream)

        def e2e_step(prefetch):
            stream.wait_event(ev_staged)
            for ssrc, ddst in zip(stage, dev_in):
                ddst.copy_(ssrc, non_blocking=True)
            ev_consumed.record(stream)
            if prefetch:
                h2d_to_stage()                               # inputs of the next step
            for r in runners:                                # the step (and gradient exchange, if on)
                r()
            host_out.copy_(step.losses, non_blocking=True)

        ev_consumed.record(stream)
        for _ in range(2):
            h2d_to_stage()
            e2e_step(False)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        ev_consumed.record(stream)                           # the first copy starts after e0
        h2d_to_stage()
        for k in range(K):
            e2e_step(k + 1 < K)
        e1.record(stream)
        barrier()
        ms_e2e = _max_over_ranks(e0.elapsed_time(e1), ws, device)
        e2e = {"value": tokens_all * K / (ms_e2e / 1000.0), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h,
               "how": "pinned host -> device copy of step k+1 overlapped with step k on a copy stream"}

    # ---------------- inter-exit agreement pass (a measurement, outside the step)
    extras = {}
    if c.M > 1:
        def agree_run(s):
            return step.api.exit_agreement(step.o, step.W, step.stats, workspace=step.ws_loss, stream=s)[0]
        am = agree_run(stream)
        if args.eager:
            arun = lambda: agree_run(stream)  # noqa: E731
        else:
            ga = torch.cuda.CUDAGraph()
            with torch.cuda.graph(ga, capture_error_mode="relaxed"):
                am = agree_run(None)
            arun = ga.replay
        for _ in range(2):
            arun()
        barrier()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        ka = max(3, K // 5)
        a0.record(stream)
        for _ in range(ka):
            arun()
        a1.record(stream)
        barrier()
        ms_a = a0.elapsed_time(a1) / ka
        vals = am.float().cpu().tolist()
        S = c.M - 1
        extras["exit_agreement"] = {
            "ms": ms_a, "tflops": 2.0 * c.T * c.V * sum(c.D) / (ms_a / 1000.0) / 1e12,
            "beta_mean": vals[:S], "kl_mean": vals[S:2 * S], "top1_agree_mean": vals[2 * S:],
            "what": "each smaller exit vs the largest: acceptance sum_v min(q,p), KL(p||q), top-1 agreement"}

    # ---------------- the forward against cuBLAS GEMMs of the same shapes, same box
    if ws == 1 and c.dtype == "bf16":
        extras["cublas_calibration"] = cublas_calibration(step, runners[1], runners[2], stream, device)
        barrier()

    # ---------------- each junction kernel alone: 24 back-to-back launches rotating
    # over enough copies of the streamed rows (o, dy in; y, do, de out) that they
    # span at least 3x the 126 MB L2, captured as one CUDA graph, CUDA events
    # around its replay
    if c.M > 1:
        b = 2 if c.dtype == "bf16" else 4
        alone = []
        for j in range(c.M - 1):
            D, dl, Dn = c.D[j], c.deltas[j + 1], c.D[j + 1]
            fwd_bytes = c.T * ((D + dl + Dn) * b + 8)
            bwd_bytes = c.T * ((Dn + 2 * D + 2 * dl) * b + 4)
            copies = max(2, -(-3 * (126 << 20) // fwd_bytes))
            o_c = [step.o[j]] + [step.o[j].clone() for _ in range(copies - 1)]
            y_c = [torch.empty_like(step.jy[j]) for _ in range(copies)]
            dy_c = [step.dh[j + 1]] + [step.dh[j + 1].clone() for _ in range(copies - 1)]
            do_c = [torch.empty_like(step.do[j]) for _ in range(copies)]
            de_c = [torch.empty_like(step.de[j]) for _ in range(copies)]
            calls = {
                "fwd": (lambda i, s, j=j: step.api.junction_fwd(step.x, o_c[i], step.E[j + 1], out=y_c[i],
                                                                scale_out=step.jscale[j], status=step.status,
                                                                stream=s), fwd_bytes),
                "bwd_rows": (lambda i, s, j=j: step.api.junction_bwd(step.x, o_c[i], step.E[j + 1], dy_c[i],
                                                                     do_out=do_c[i], de_out=de_c[i], dE=None,
                                                                     workspace=step.ws_j, status=step.status,
                                                                     stream=s), bwd_bytes),
            }
            for kind, (fn, nbytes) in calls.items():
                n = 24
                for i in range(copies):
                    fn(i, stream)
                if args.eager:
                    batch = lambda fn=fn: [fn(i % copies, stream) for i in range(n)]  # noqa: E731
                else:
                    gj = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(gj, capture_error_mode="relaxed"):
                        for i in range(n):
                            fn(i % copies, None)
                    batch = gj.replay
                batch()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                batch()
                e1.record(stream)
                e1.synchronize()
                us = e0.elapsed_time(e1) * 1000.0 / n
                alone.append({"junction": f"{D}->{Dn}", "pass": kind, "us": us, "bytes": nbytes,
                              "gbs": nbytes / us / 1e3, "frac_of_hbm": nbytes / us / 1e3 / peaks.get("hbm_gbs"),
                              "copies": copies})
            del o_c, y_c, dy_c, do_c, de_c
        extras["junction_alone"] = alone

    # ---------------- roofline of the dominant kernel and phase rates
    ms_fwd, ms_bwd = phase_ms[1], phase_ms[2]
    flops_fwd = 2.0 * c.T * c.V * sum(c.D)
    peak_tc = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    ach_fwd = flops_fwd / (ms_fwd / 1000.0) / 1e12
    jf_bytes, jb_bytes = step.junction_bytes()
    hbm = peaks.get("hbm_gbs")
    phases = {
        "junction_fwd_ms": phase_ms[0], "loss_fwd_ms": ms_fwd, "loss_bwd_ms": ms_bwd, "junction_bwd_ms": phase_ms[3],
        "loss_fwd_bwd_tokens_per_s": c.T / ((ms_fwd + ms_bwd) / 1000.0),
        "loss_executed_tflops": step.loss_flops_executed() / ((ms_fwd + ms_bwd) / 1000.0) / 1e12,
        "loss_executed_frac_of_peak": step.loss_flops_executed() / ((ms_fwd + ms_bwd) / 1000.0) / 1e12 / peak_tc,
        "loss_algorithmic_frac_of_peak": step.loss_flops_algorithmic() / ((ms_fwd + ms_bwd) / 1000.0) / 1e12 / peak_tc,
        "junction_fwd_gbs": jf_bytes / (phase_ms[0] / 1000.0) / 1e9 if c.M > 1 else None,
        "junction_fwd_frac_of_hbm": jf_bytes / (phase_ms[0] / 1000.0) / 1e9 / hbm if c.M > 1 else None,
        "junction_bwd_gbs": jb_bytes / (phase_ms[3] / 1000.0) / 1e9 if c.M > 1 else None,
        "junction_bwd_frac_of_hbm": jb_bytes / (phase_ms[3] / 1000.0) / 1e9 / hbm if c.M > 1 else None,
        "junction_bytes": {"fwd": jf_bytes, "bwd_rows_and_tables": jb_bytes},
    }
    if sync_on:
        gbytes = sum(t.numel() * t.element_size() for t in grads)
        phases["grad_sync_ms"] = phase_ms[4]
        phases["grad_sync_bytes"] = gbytes
    if c.dtype == "bf16":
        roofline = {"bound": "tensor", "achieved": ach_fwd, "peak": peak_tc, "unit": "TFLOP/s",
                    "frac": ach_fwd / peak_tc, "traffic": measured_traffic(c),
                    "kernel": "loss_tile_kernel<stats> (mls_multiexit_loss_fwd call: tile kernel + merge + reduce)",
                    "algorithmic_per_launch": f"2*T*V*sum(D) = {flops_fwd:.4g} flop",
                    "peak_source": f"{peak_kind} bf16_tflops_sustained"}
    else:
        # fp32 inputs take the CUDA-core path: 148 SMs x 128 fp32 FMA lanes x 2 flop x 1.965 GHz
        peak_fma = 148 * 128 * 2 * 1.965e9 / 1e12
        roofline = {"bound": "alu", "achieved": ach_fwd, "peak": peak_fma, "unit": "TFLOP/s",
                    "frac": ach_fwd / peak_fma, "traffic": None,
                    "kernel": "simt_stats_kernel (mls_multiexit_loss_fwd call, fp32 CUDA-core path)",
                    "algorithmic_per_launch": f"2*T*V*sum(D) = {flops_fwd:.4g} flop",
                    "peak_source": "nominal fp32 FMA rate at the maximum SM clock (no measured fp32 figure)"}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        sec, n = cpu_oracle_sample(step.host, args.cpu_tokens)
        cpu = {"value": n / sec, "unit": "tokens/s", "cores": _cores(), "kind": "oracle",
               "sample": f"first {n} tokens of {cfg.name}: both junctions fwd+bwd and the {c.M}-exit loss "
                         f"fwd+bwd over the full vocabulary, fp64 numpy ({sec:.1f} s)"}

    if rank == 0 and ws == 1 and not args.no_workloads and not args.tokens:
        # the other workloads, each at its full size with the oracle beside it
        others = []
        for name in wl.CONFIG_ORDER:
            if wl.CONFIGS[name].name == c.name:
                continue
            others.append(measure_workload(name, device, stream, peaks, max(5, min(K, 20)), args.eager,
                                           256 if name == "tiny3" else 64))
        extras["workloads"] = others

    if rank == 0:
        line = {
            "metric": "multi-exit head-loss fwd+bwd tokens/s (1 B200) and % bf16 tensor peak; junction GB/s",
            "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if c.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": c.name, "global_batch": c.batch * ws, "seq_len": c.seq, "tokens_per_gpu": c.T,
                       "M": c.M, "D": list(c.D), "V": c.V, "alpha_d": c.alpha_d,
                       "parallelism": f"dp{ws} (independent batches)" if not sync_on else
                                      f"dp{ws} (dW and dE {args.grad_sync} over NCCL every step)",
                       "l2": f"no flush; per-step working set {step.working_set_gb():.2f} GB > 126 MB L2",
                       "loss_bwd_pieces": {"token_block": step.bwd_plan[0], "vocab_chunk": step.bwd_plan[1],
                                           "workspace_bytes": step.ws_loss.numel()}},
            "e2e": e2e, "gpu_launches": int(launches), "launch_mode": "eager" if args.eager else "cuda_graph",
            "roofline": roofline, "cpu_baseline": cpu,
            "phases": phases, "extras": extras, "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
