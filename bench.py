#!/usr/bin/env python
"""Throughput of the theta-bundle hot path on B200.

One step is one pass of every stage of the path over one synthetic workload,
Gemma-3-1B-shaped: 26 layers, the seven projection families (q [1024,1152],
k/v [256,1152], o [1152,1024], gate/up [6912,1152], down [1152,6912]), bf16
weights drawn as a common N(0,0.02) base plus per-layer N(0,0.005) noise,
rank-32 factors U, V ~ N(0,0.01), activations X ~ N(0,1). For each of
G = 26 (passthrough) and G = 1 the step runs, per family:

  prelude      band means W0, row scales s and residuals R  (theta_decompose_prelude)
  reconstruct  diag(s).W0 + U.V^T for every layer           (theta_reconstruct)
  frob         ||W - W_rec||_F / ||W||_F for every layer     (theta_frob_error)
  forward      s*(X.W0^T) + (X.V).U^T for every layer at M = 1, 16, 256
                                                             (theta_linear_forward)

Throughput is algorithmic bytes per second: the bytes each call must move at
minimum (inputs read once, outputs written once; W0 counted once per forward
call), summed over the step, divided by the device time of the step. Each
stage is captured as a CUDA graph; the step replays them back to back with
CUDA events between stages. The step touches > 10 GB, far more than the 126 MB
L2, so no explicit flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun each rank runs the whole workload on its own GPU (independent
problems, weak scaling); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synthetic as syn  # noqa: E402

METRIC = "theta-forward TFLOP/s (prefill) & GB/s (decode) vs B200 roofline; decompose GB/s"
WORKLOAD = "gemma3-1b-shaped theta path: 26 layers x 7 families, bf16, G in {26,1}, rank 32, M in {1,16,256}"
MODEL = syn.GEMMA3_1B
RANK = 32
M_VALUES = (1, 16, 256)
G_VALUES = (26, 1)
BF16 = 2  # bytes


# --------------------------------------------------------------- accounting
def bytes_prelude(L, G, O, I, b=BF16):
    """Minimum traffic of the whole prelude of one family: read every W once,
    write the G shared blocks, the L residuals and the L fp32 scales."""
    return L * O * I * b + G * O * I * b + L * O * I * b + 4 * L * O


def bytes_reconstruct(O, I, r, b=BF16):
    return O * I * b + 4 * O + r * (O + I) * b + O * I * b


def bytes_frob(O, I, b=BF16):
    return 2 * O * I * b


def bytes_forward(M, O, I, r, b=BF16):
    return O * I * b + 4 * O + r * (O + I) * b + M * I * b + M * O * b


def flops_forward(M, O, I, r):
    return 2 * M * (O * I + r * (I + O))


def prelude_launches(L, G, I, b=BF16, num_sms=148):
    """Kernel launches of one theta_decompose_prelude call, following the
    library's dispatch: one pipeline launch for bands of <= 4 layers; one
    two-pass launch for longer bands whose rows for one CTA per SM fit the
    kernel's 64 MB L2 budget (threads per row: the fewest of 32..256 giving
    <= 4 vectors per thread within a 32 KB item); else a band-mean launch per
    band and one row-pass launch."""
    nmax = -(-L // G)
    if nmax <= 4:
        return 1
    nv, row_bytes = I * b // 16, I * b
    for cap in (4, 8):
        tpr = next((t for t in (32, 64, 128, 256) if -(-nv // t) <= cap and (256 // t) * row_bytes <= 32 * 1024), None)
        if tpr:
            break
    if tpr and nmax * (256 // tpr) * row_bytes * num_sms <= (64 << 20):
        return 1
    return G + 1


def step_accounting(model=MODEL, r=RANK, m_values=M_VALUES, g_values=G_VALUES, grouped=True):
    """Per-stage algorithmic bytes / flops / kernel launches of one step.
    With `grouped`, a stage of one or two tokens is one grouped call (T = X.V
    slices, their sums, one sweep: 3 launches, 1 at rank 0)."""
    L = model.num_layers
    stages = []
    for G in g_values:
        pre = rec = fro = 0
        fwd = {m: [0, 0] for m in m_values}
        for fam, (O, I) in model.shapes.items():
            pre += bytes_prelude(L, G, O, I)
            rec += L * bytes_reconstruct(O, I, r)
            fro += L * bytes_frob(O, I)
            for m in m_values:
                fwd[m][0] += L * bytes_forward(m, O, I, r)
                fwd[m][1] += L * flops_forward(m, O, I, r)
        nf = len(model.shapes)
        stages.append(dict(name=f"prelude_G{G}", kind="prelude", bytes=pre, flops=0,
                           launches=sum(prelude_launches(L, G, I) for (_, I) in model.shapes.values())))
        stages.append(dict(name=f"reconstruct_G{G}", kind="reconstruct", bytes=rec, flops=0, launches=nf * L))
        stages.append(dict(name=f"frob_G{G}", kind="frob", bytes=fro, flops=0, launches=nf * L * 2))
        for m in m_values:
            launches = (3 if r > 0 else 1) if grouped and m <= 2 else nf * L * (2 if r > 0 else 1)
            stages.append(dict(name=f"forward_m{m}_G{G}", kind=f"forward_m{m}", bytes=fwd[m][0],
                               flops=fwd[m][1], launches=launches))
    return stages


# --------------------------------------------------------------- environment
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank number over all ranks (identity for one process)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def result_line(*, value, unit, n_gpus, steps, warmup, ms_per_step, extra):
    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": n_gpus, "steps": steps, "warmup": warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded; weights, factors and activations drawn on the device)"}
    line.update(extra)
    return line


# --------------------------------------------------------------- workload
class Workload:
    """All device tensors of one step, and the stage call lists."""

    def __init__(self, theta, torch, seed=0, model=MODEL, r=RANK, streams=1, grouped=True):
        self.theta, self.torch = theta, torch
        # independent calls of a stage (layers, families) spread round-robin
        # over this many streams; each stream has its own workspaces
        self.nstreams = streams
        self.side = [torch.cuda.Stream() for _ in range(streams)] if streams > 1 else []
        self.model, self.r, self.L = model, r, model.num_layers
        dev = "cuda"
        bf = torch.bfloat16
        L = self.L
        self.W, self.W0, self.s, self.R, self.rec, self.U, self.V = {}, {}, {}, {}, {}, {}, {}
        for fam, (O, I) in model.shapes.items():
            self.W[fam] = syn.device_family_weights(L, O, I, seed=seed, family=fam, dtype="bf16")
            self.W0[fam] = [torch.empty(O, I, dtype=bf, device=dev) for _ in range(max(G_VALUES))]
            self.s[fam] = [torch.empty(O, dtype=torch.float32, device=dev) for _ in range(L)]
            self.R[fam] = [torch.empty(O, I, dtype=bf, device=dev) for _ in range(L)]
            self.rec[fam] = [torch.empty(O, I, dtype=bf, device=dev) for _ in range(L)]
            self.U[fam] = [syn.device_normal((O, r), 0.01, seed, "U", fam, l) for l in range(L)]
            self.V[fam] = [syn.device_normal((I, r), 0.01, seed, "V", fam, l) for l in range(L)]
        in_dims = sorted({I for (_, I) in model.shapes.values()})
        self.X = {(m, I): syn.device_normal((m, I), 1.0, seed, "X", m, I) for m in M_VALUES for I in in_dims}
        self.Y = {(m, fam, l): torch.empty(m, O, dtype=bf, device=dev)
                  for m in M_VALUES for fam, (O, _) in model.shapes.items() for l in range(L)}
        self.frob_out = torch.zeros(len(G_VALUES), len(model.shapes), L, dtype=torch.float64, device=dev)
        fb = theta.theta_workspace_size(theta.THETA_OP_FROB_ERROR, 1, 1, 1, 0, theta.THETA_BF16)
        self.frob_ws = [torch.empty(fb, dtype=torch.uint8, device=dev) for _ in range(streams)]
        wb = max(theta.theta_workspace_size(theta.THETA_OP_LINEAR_FORWARD, m, O, I, r, theta.THETA_BF16)
                 for m in M_VALUES for (O, I) in model.shapes.values())
        self.fwd_ws = [torch.empty(max(wb, 256), dtype=torch.uint8, device=dev) for _ in range(streams)]
        self.bands = {G: theta.theta_band_index(L, G)[0] for G in G_VALUES}
        # one or two tokens: every family of every layer in one grouped call
        self.groups = {}
        if grouped:
            for G in G_VALUES:
                for m in M_VALUES:
                    if m <= 2:
                        band = self.bands[G]
                        self.groups[(G, m)] = theta.ForwardGroup([
                            (self.X[(m, I)], self.W0[fam][band[l]], self.s[fam][l], self.U[fam][l], self.V[fam][l],
                             self.Y[(m, fam, l)]) for fam, (O, I) in model.shapes.items() for l in range(L)])
        gb = max([g.workspace_size() for g in self.groups.values()] + [256])
        self.grp_ws = torch.empty(gb, dtype=torch.uint8, device=dev)

    # stage bodies ------------------------------------------------------
    def _fan_out(self, calls):
        """Runs calls(k) with k the stream slot: all on the current stream,
        or forked round-robin over the side streams and joined back."""
        if not self.side:
            for c in calls:
                c(0)
            return
        torch = self.torch
        main = torch.cuda.current_stream()
        for st in self.side:
            st.wait_stream(main)
        for i, c in enumerate(calls):
            k = i % len(self.side)
            with torch.cuda.stream(self.side[k]):
                c(k)
        for st in self.side:
            main.wait_stream(st)

    def prelude(self, G):
        t = self.theta
        self._fan_out([lambda k, fam=fam: t.theta_decompose_prelude(self.W[fam], G, self.W0[fam][:G], self.s[fam],
                                                                     self.R[fam])
                       for fam in self.model.shapes])

    def reconstruct(self, G):
        t = self.theta
        band = self.bands[G]
        self._fan_out([lambda k, fam=fam, l=l: t.theta_reconstruct(self.s[fam][l], self.W0[fam][band[l]],
                                                                    self.U[fam][l], self.V[fam][l],
                                                                    self.rec[fam][l])
                       for fam in self.model.shapes for l in range(self.L)])

    def frob(self, G):
        t = self.theta
        gi = G_VALUES.index(G)
        self._fan_out([lambda k, fi=fi, fam=fam, l=l: t.theta_frob_error(self.W[fam][l], self.rec[fam][l],
                                                                          self.frob_out[gi, fi, l:l + 1],
                                                                          self.frob_ws[k])
                       for fi, fam in enumerate(self.model.shapes) for l in range(self.L)])

    def forward(self, G, m):
        t = self.theta
        if (G, m) in self.groups:
            t.theta_linear_forward_grouped(self.groups[(G, m)], self.grp_ws)
            return
        band = self.bands[G]
        self._fan_out([lambda k, fam=fam, I=I, l=l: t.theta_linear_forward(
            self.X[(m, I)], self.W0[fam][band[l]], self.s[fam][l], self.U[fam][l], self.V[fam][l],
            self.Y[(m, fam, l)], self.fwd_ws[k])
            for fam, (O, I) in self.model.shapes.items() for l in range(self.L)])

    def stage_fns(self):
        fns = []
        for G in G_VALUES:
            fns.append(lambda G=G: self.prelude(G))
            fns.append(lambda G=G: self.reconstruct(G))
            fns.append(lambda G=G: self.frob(G))
            for m in M_VALUES:
                fns.append(lambda G=G, m=m: self.forward(G, m))
        return fns

    # host side of the end-to-end run -----------------------------------
    def input_tensors(self):
        ins = []
        for fam in self.model.shapes:
            ins += self.W[fam] + self.U[fam] + self.V[fam]
        ins += list(self.X.values())
        return ins

    def output_tensors(self):
        return [self.frob_out] + list(self.Y.values()) + [s for fam in self.model.shapes for s in self.s[fam]]


# The sources that define each stage's kernels and their launch code (the
# shared device helpers included): a recorded ncu traffic figure stands only
# while these files hash to the value recorded beside it.
KIND_SOURCES = {
    "prelude": ["prelude_kernels.cu", "stream_kernels.cu", "common.cuh", "umma_ptx.cuh"],
    "reconstruct": ["umma_kernels.cu", "umma_ptx.cuh", "common.cuh"],
    "frob": ["stream_kernels.cu", "common.cuh"],
    "forward_m1": ["gemv_kernels.cu", "common.cuh"],
    "forward_m16": ["umma_kernels.cu", "umma_ptx.cuh", "common.cuh"],
    "forward_m256": ["umma_kernels.cu", "umma_ptx.cuh", "common.cuh"],
}


def kernel_source_hash(kind=None):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_theta_forward_b200", "csrc")
    names = KIND_SOURCES.get(kind) or sorted(os.listdir(csrc))
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kind):
    """DRAM bytes per launch of a stage's main kernel from a committed ncu
    capture, or None when that stage's kernel sources changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    entry = rec.get(kind)
    if not entry or entry.get("source_hash") != kernel_source_hash(kind):
        return None
    return entry.get("dram_bytes_per_launch")


# --------------------------------------------------------------- CPU oracle
def oracle_sample_step(rows=64, seed=0, model=MODEL, r=RANK):
    """One bounded sample of the step on the host CPU with the fp64 oracle:
    the first `rows` output rows of every family, all layers, both G values.
    Inputs are drawn before the clock starts. Returns (algorithmic bytes of
    the sample, seconds)."""
    import oracle
    L = model.num_layers
    inputs = {}
    for fam, (O, I) in model.shapes.items():
        n = min(rows, O)
        w = syn.host_family_weights(L, n, I, seed=seed, family=f"cpu-{fam}", dtype="bf16")
        U = [syn.host_normal((n, r), 0.01, seed, "U", fam, l, dtype="bf16") for l in range(L)]
        V = [syn.host_normal((I, r), 0.01, seed, "V", fam, l, dtype="bf16") for l in range(L)]
        X = {m: syn.host_activations(m, I, seed=seed, tag=f"cpu-{m}", dtype="bf16") for m in M_VALUES}
        inputs[fam] = (n, I, w, U, V, X)
    total_bytes = 0
    t0 = time.perf_counter()
    for fam, (n, I, w, U, V, X) in inputs.items():
        for G in G_VALUES:
            band, _ = oracle.band_index(L, G)
            W0 = oracle.band_mean(w, G, "bf16")
            for l in range(L):
                w0 = W0[band[l]]
                s = oracle.row_scale(w[l], w0)
                oracle.residual(w[l], w0, s, "bf16")
                s32 = oracle.round_to(s, "f32")
                rec = oracle.reconstruct(s32, w0, U[l], V[l], "bf16")
                oracle.frob_error(w[l], rec)
                for m in M_VALUES:
                    oracle.linear_forward(X[m], w0, s32, U[l], V[l], "bf16")
            total_bytes += bytes_prelude(L, G, n, I)
            total_bytes += L * (bytes_reconstruct(n, I, r) + bytes_frob(n, I))
            total_bytes += L * sum(bytes_forward(m, n, I, r) for m in M_VALUES)
    return total_bytes, time.perf_counter() - t0


def cpu_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((d.get("num_threads", 1) for d in info), default=1)
        return int(n)
    except Exception:
        return len(os.sched_getaffinity(0))


def cpu_baseline(target_s=12.0, rows=64):
    np.ones((64, 64)) @ np.ones((64, 64))  # load BLAS so its threads are visible
    done_bytes, spent, reps = 0, 0.0, 0
    while spent < target_s and reps < 50:
        b, s = oracle_sample_step(rows=rows, seed=reps)
        done_bytes += b
        spent += s
        reps += 1
    return {"value": done_bytes / spent / 1e9, "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{reps} x (first {rows} output rows of each of the 7 families, all 26 layers, "
                      f"G in {{26,1}}, every stage incl. forward at M in {{1,16,256}}); {spent:.1f} s"}


def run_reference(args):
    """The oracle as the reference arm: each step is one bounded row sample."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    oracle_sample_step(rows=16)  # warm the imports and BLAS
    for _ in range(args.warmup):
        oracle_sample_step(rows=args.ref_rows)
    times, nbytes = [], 0
    for i in range(args.steps):
        b, s = oracle_sample_step(rows=args.ref_rows, seed=i)
        times.append(s)
        nbytes = b
    per_step = sum(times) / len(times)
    value = nbytes / per_step / 1e9
    line = result_line(value=value, unit="GB/s", n_gpus=args.gpus, steps=args.steps, warmup=args.warmup,
                       ms_per_step=per_step * 1e3, extra={
                           "impl": "reference", "dtype": "f64",
                           "data": "synthetic (seeded; weights, factors and activations drawn on the host)",
                           "config": {"workload": WORKLOAD, "sample_rows_per_family": args.ref_rows,
                                      "l2": "n/a (CPU)"},
                           "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle",
                                            "sample": f"first {args.ref_rows} output rows of each family per step"},
                           "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                       })
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------- GPU arm
def run_gpu(args):
    import torch
    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    import linear_theta_forward_b200 as theta

    peaks = measured_peaks()
    # many independent calls in flight at once: no split-K
    policy = theta.THETA_POLICY_THROUGHPUT if args.streams > 1 else theta.THETA_POLICY_LATENCY
    theta.theta_set_policy(policy)
    wl = Workload(theta, torch, seed=rank, streams=args.streams, grouped=not args.per_call_decode)
    stages = step_accounting(grouped=not args.per_call_decode)
    fns = wl.stage_fns()
    assert len(fns) == len(stages)
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()

    # one eager pass (initialises the library), then capture every stage
    with torch.cuda.stream(stream):
        for fn in fns:
            fn()
    theta.theta_device_status(stream)
    graphs = []
    if not args.no_graph:
        for fn in fns:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fn()
            graphs.append(g)
    run = [g.replay for g in graphs] if graphs else fns

    def one_step(events=None):
        with torch.cuda.stream(stream):
            for i, f in enumerate(run):
                if events is not None:
                    events[i].record(stream)
                f()
            if events is not None:
                events[-1].record(stream)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    theta.theta_device_status(stream)

    n_st = len(stages)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_st + 1)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        start = torch.cuda.Event(enable_timing=True)
        stop = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for k in range(args.steps):
            one_step(ev[k])
        stop.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    theta.theta_device_status(stream)
    total_ms = max_over_ranks(start.elapsed_time(stop), world, device="cuda")
    stage_ms = [sum(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(args.steps)) / args.steps
                for i in range(n_st)]

    step_bytes = sum(s["bytes"] for s in stages)
    ms_per_step = total_ms / args.steps
    value = world * step_bytes / (ms_per_step * 1e-3) / 1e9
    launches = sum(s["launches"] for s in stages) * args.steps

    # per-kind aggregates; the dominant kind gives the roofline entry
    kinds = {}
    for st, ms in zip(stages, stage_ms):
        k = kinds.setdefault(st["kind"], {"ms": 0.0, "bytes": 0, "flops": 0, "launches": 0})
        k["ms"] += ms
        k["bytes"] += st["bytes"]
        k["flops"] += st["flops"]
        k["launches"] += st["launches"]
    parts = {}
    for name, k in kinds.items():
        parts[name] = {"ms": round(k["ms"], 4), "GB/s": round(k["bytes"] / (k["ms"] * 1e-3) / 1e9, 1),
                       "frac_hbm": round(k["bytes"] / (k["ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)}
        if k["flops"]:
            parts[name]["TFLOP/s"] = round(k["flops"] / (k["ms"] * 1e-3) / 1e12, 2)
    dom_name, dom = max(kinds.items(), key=lambda kv: kv[1]["ms"])
    per_launch_bytes = dom["bytes"] / dom["launches"]
    per_launch_s = dom["ms"] * 1e-3 / dom["launches"]
    achieved = per_launch_bytes / per_launch_s / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": recorded_traffic(dom_name),
                "kernel": dom_name, "peak_source": peaks["source"],
                "bytes_per_launch": round(per_launch_bytes), "launches_per_step": dom["launches"]}

    e2e = None
    if not args.skip_e2e:
        e2e = run_e2e(torch, theta, wl, run, stream, step_bytes, min(args.steps, args.e2e_steps), world)

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        cpu = cpu_baseline(target_s=args.cpu_seconds)

    if rank == 0:
        line = result_line(value=round(value, 2), unit="GB/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
                           ms_per_step=round(ms_per_step, 4), extra={
                               "config": {"workload": WORKLOAD, "model": "gemma3-1b-shaped (random init)",
                                          "layers": MODEL.num_layers, "families": list(MODEL.shapes),
                                          "G": list(G_VALUES), "rank": RANK, "M": list(M_VALUES),
                                          "global_batch": max(M_VALUES), "seq_len": 1,
                                          "parallelism": f"independent replicas x{world}",
                                          "graphs": not args.no_graph, "streams": args.streams,
                                          "policy": "throughput" if policy else "latency",
                                          "decode": "per call" if args.per_call_decode else "grouped",
                                          "l2": "inputs larger than L2 (>10 GB touched per step); no flush"},
                               "parts": parts,
                               "roofline": roofline,
                               "cpu_baseline": cpu,
                               "e2e": e2e,
                               "gpu_launches": launches,
                               "clocks": clocks.summary(),
                           })
        print(json.dumps(line), flush=True)
    for g in graphs:
        del g
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def run_e2e(torch, theta, wl, run, stream, step_bytes, steps, world):
    """The same step through the public API with HOST buffers: every step copies
    its inputs from pinned host memory, runs, and reads its results back."""
    ins = wl.input_tensors()
    outs = wl.output_tensors()
    h_in = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in ins]
    for h, t in zip(h_in, ins):
        h.copy_(t)
    h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
    h2d = sum(t.numel() * t.element_size() for t in ins)
    d2h = sum(t.numel() * t.element_size() for t in outs)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(steps):
            for h, t in zip(h_in, ins):
                t.copy_(h, non_blocking=True)
            for f in run:
                f()
            for h, t in zip(h_out, outs):
                h.copy_(t, non_blocking=True)
        stop.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(stop), world, device="cuda") / steps
    return {"value": round(world * step_bytes / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3), "steps": steps}


def run_op(args):
    """One entry point on one synthetic problem, timed per call with CUDA
    events (median of --iters calls, L2 flushed before each). Prints a JSON
    line with the achieved rate and its fraction of the measured roofline."""
    import torch
    torch.cuda.set_device(0)
    import linear_theta_forward_b200 as theta
    peaks = measured_peaks()
    M, O, I, r, L, G = args.M, args.O, args.I, args.rank, args.layers, args.G
    seed = 0
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    if args.op == "forward":
        # --b2b: calls cycle over --bufs independent problems (like the layers
        # of a model), so no call finds its W0 in L2
        nbuf = args.bufs if args.b2b else 1
        X = syn.device_normal((M, I), 1.0, seed, "X", M, I)
        probs = []
        for k in range(nbuf):
            W0 = syn.device_normal((O, I), 0.02, seed + k, "W0", O, I)
            s = 1.0 + syn.device_normal((O,), 0.05, seed + k, "s", O, dtype="f32")
            U = syn.device_normal((O, r), 0.01, seed + k, "U", O, r) if r else None
            V = syn.device_normal((I, r), 0.01, seed + k, "V", I, r) if r else None
            probs.append((W0, s, U, V, torch.empty(M, O, dtype=torch.bfloat16, device="cuda")))
        nb = theta.theta_workspace_size(theta.THETA_OP_LINEAR_FORWARD, M, O, I, r, theta.THETA_BF16)
        ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
        turn = [0]

        def call():
            W0, s, U, V, Y = probs[turn[0] % nbuf]
            turn[0] += 1
            theta.theta_linear_forward(X, W0, s, U, V, Y, ws)
        nbytes, nflops = bytes_forward(M, O, I, r), flops_forward(M, O, I, r)
    elif args.op == "gate_up":
        nbuf = args.bufs if args.b2b else 1
        X = syn.device_normal((M, I), 1.0, seed, "X", M, I)

        def proj(k, tag):
            return (syn.device_normal((O, I), 0.02, seed + k, "W0", tag, O, I),
                    1.0 + syn.device_normal((O,), 0.05, seed + k, "s", tag, O, dtype="f32"),
                    syn.device_normal((O, r), 0.01, seed + k, "U", tag, O, r) if r else None,
                    syn.device_normal((I, r), 0.01, seed + k, "V", tag, I, r) if r else None)
        probs = [(proj(k, "gate"), proj(k, "up"), torch.empty(M, O, dtype=torch.bfloat16, device="cuda"))
                 for k in range(nbuf)]
        nb = theta.theta_workspace_size(theta.THETA_OP_GATE_UP_FORWARD, M, O, I, r, theta.THETA_BF16)
        ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
        turn = [0]

        def call():
            gate, up, Y = probs[turn[0] % nbuf]
            turn[0] += 1
            theta.theta_linear_gate_up_forward(X, gate, up, Y, ws)
        # both weights streamed once, X read once, one output written
        nbytes = 2 * bytes_forward(M, O, I, r) - M * I * BF16 - M * O * BF16
        nflops = 2 * flops_forward(M, O, I, r)
    elif args.op == "forward_nvfp4":
        nbuf = args.bufs if args.b2b else 1
        X = syn.device_normal((M, I), 1.0, seed, "X", M, I)
        qws = torch.empty(16, dtype=torch.uint8, device="cuda")
        probs = []
        for k in range(nbuf):
            W0 = syn.device_normal((O, I), 0.02, seed + k, "W0", O, I)
            codes = torch.empty(O, I // 2, dtype=torch.uint8, device="cuda")
            scales = torch.empty(O, I // 16, dtype=torch.uint8, device="cuda")
            g = torch.empty(1, dtype=torch.float32, device="cuda")
            theta.theta_nvfp4_quantize(W0, codes, scales, g, qws)
            del W0
            s = 1.0 + syn.device_normal((O,), 0.05, seed + k, "s", O, dtype="f32")
            U = syn.device_normal((O, r), 0.01, seed + k, "U", O, r) if r else None
            V = syn.device_normal((I, r), 0.01, seed + k, "V", I, r) if r else None
            probs.append((codes, scales, g, s, U, V, torch.empty(M, O, dtype=torch.bfloat16, device="cuda")))
        nb = theta.theta_workspace_size(theta.THETA_OP_LINEAR_FORWARD_NVFP4, M, O, I, r, theta.THETA_BF16)
        ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
        turn = [0]

        def call():
            codes, scales, g, s, U, V, Y = probs[turn[0] % nbuf]
            turn[0] += 1
            theta.theta_linear_forward_nvfp4(X, codes, scales, g, s, U, V, Y, ws)
        # the NVFP4 block (0.5625 bytes per weight) instead of bf16 W0
        nbytes = bytes_forward(M, O, I, r) - O * I * BF16 + O * I * 9 // 16
        nflops = flops_forward(M, O, I, r)
    elif args.op == "grouped":
        # every family of --layers Gemma-3-1B-shaped layers in one grouped call
        # (or, with --per-call-decode, one theta_linear_forward per problem)
        xs = {I_: syn.device_normal((M, I_), 1.0, seed, "X", M, I_) for (_, I_) in MODEL.shapes.values()}
        probs = []
        for fam, (O_, I_) in MODEL.shapes.items():
            for l in range(L):
                probs.append((xs[I_], syn.device_normal((O_, I_), 0.02, seed + l, "W0", fam),
                              1.0 + syn.device_normal((O_,), 0.05, seed + l, "s", fam, dtype="f32"),
                              syn.device_normal((O_, r), 0.01, seed + l, "U", fam) if r else None,
                              syn.device_normal((I_, r), 0.01, seed + l, "V", fam) if r else None,
                              torch.empty(M, O_, dtype=torch.bfloat16, device="cuda")))
        if args.per_call_decode:
            nb = max(theta.theta_workspace_size(theta.THETA_OP_LINEAR_FORWARD, M, O_, I_, r, theta.THETA_BF16)
                     for (O_, I_) in MODEL.shapes.values())
            ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")

            def call():
                for X_, W0, s, U, V, Y in probs:
                    theta.theta_linear_forward(X_, W0, s, U, V, Y, ws)
        else:
            group = theta.ForwardGroup(probs)
            ws = torch.empty(max(group.workspace_size(), 256), dtype=torch.uint8, device="cuda")
            call = lambda: theta.theta_linear_forward_grouped(group, ws)  # noqa: E731
        nbytes = sum(bytes_forward(M, p[1].shape[0], p[1].shape[1], r) for p in probs)
        nflops = sum(flops_forward(M, p[1].shape[0], p[1].shape[1], r) for p in probs)
    elif args.op == "svd":
        # randomized SVD of one residual: rank r, r + 10 samples, 2 subspace iterations
        k, q = min(r + 10, O, I), 2
        R = syn.device_normal((O, I), 0.005, seed, "R", O, I)
        omega = syn.device_normal((k, I), 1.0, seed, "omega", k, I, dtype="f32")
        Ud = torch.empty(O, r, dtype=torch.bfloat16, device="cuda")
        Vd = torch.empty(I, r, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(theta.theta_workspace_size(theta.THETA_OP_RESIDUAL_SVD, k, O, I, r, theta.THETA_BF16),
                         dtype=torch.uint8, device="cuda")
        call = lambda: theta.theta_residual_svd(R, r, omega, Ud, Vd, ws, power_iters=q)  # noqa: E731
        # R is read by 2 + 2q products (R.Omega^T, 2 per iteration, Q^T.R)
        nbytes, nflops = (2 + 2 * q) * O * I * BF16, (2 + 2 * q) * 2 * O * I * k
    elif args.op == "reconstruct":
        W0 = syn.device_normal((O, I), 0.02, seed, "W0", O, I)
        s = 1.0 + syn.device_normal((O,), 0.05, seed, "s", O, dtype="f32")
        U = syn.device_normal((O, r), 0.01, seed, "U", O, r) if r else None
        V = syn.device_normal((I, r), 0.01, seed, "V", I, r) if r else None
        out = torch.empty(O, I, dtype=torch.bfloat16, device="cuda")
        call = lambda: theta.theta_reconstruct(s, W0, U, V, out)  # noqa: E731
        nbytes, nflops = bytes_reconstruct(O, I, r), 2 * O * I * r
    elif args.op == "prelude":
        W = syn.device_family_weights(L, O, I, seed=seed, family="op")
        W0 = [torch.empty(O, I, dtype=torch.bfloat16, device="cuda") for _ in range(G)]
        sl = [torch.empty(O, dtype=torch.float32, device="cuda") for _ in range(L)]
        R = None if args.no_residual else [torch.empty(O, I, dtype=torch.bfloat16, device="cuda") for _ in range(L)]
        call = lambda: theta.theta_decompose_prelude(W, G, W0, sl, R)  # noqa: E731
        nbytes, nflops = bytes_prelude(L, G, O, I) - (L * O * I * BF16 if args.no_residual else 0), 0
    elif args.op == "frob":
        A = syn.device_normal((O, I), 0.02, seed, "A", O, I)
        B = syn.device_normal((O, I), 0.02, seed, "B", O, I)
        out = torch.empty(1, dtype=torch.float64, device="cuda")
        ws = torch.empty(theta.theta_workspace_size(theta.THETA_OP_FROB_ERROR, 1, 1, 1, 0, 1), dtype=torch.uint8,
                         device="cuda")
        call = lambda: theta.theta_frob_error(A, B, out, ws)  # noqa: E731
        nbytes, nflops = bytes_frob(O, I), 0
    else:
        raise ValueError(args.op)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    theta.theta_device_status()
    if args.b2b:
        # calls back to back between one pair of events; only meaningful
        # for HBM when one call moves well over the 126 MB L2
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.iters):
            call()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / args.iters
        l2 = "calls back to back, no flush (mean of %d)" % args.iters
        if args.op in ("forward", "forward_nvfp4", "gate_up"):
            l2 += ", cycling over %d independent problems" % args.bufs
    else:
        times = []
        for _ in range(args.iters):
            flush.fill_(1)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            call()
            b.record()
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        ms = statistics.median(times)
        l2 = "flushed (256 MiB write) before every call"
    theta.theta_device_status()
    line = {"op": args.op, "shape": {"M": M, "O": O, "I": I, "rank": r, "layers": L, "G": G}, "dtype": "bf16",
            "ms": round(ms, 5), "iters": args.iters, "l2": l2,
            "GB/s": round(nbytes / (ms * 1e-3) / 1e9, 1),
            "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4), "algorithmic_bytes": nbytes}
    if nflops:
        line["TFLOP/s"] = round(nflops / (ms * 1e-3) / 1e12, 2)
        line["frac_tensor_burst"] = round(nflops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of replaying CUDA graphs")
    ap.add_argument("--streams", type=int, default=32, help="streams the independent calls of a stage spread over")
    ap.add_argument("--per-call-decode", action="store_true",
                    help="one theta_linear_forward per problem for one or two tokens instead of a grouped call")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-rows", type=int, default=32)
    ap.add_argument("--op", choices=["forward", "forward_nvfp4", "gate_up", "grouped", "reconstruct", "prelude", "frob",
                                     "svd"],
                    help="time one entry point on one problem instead of the whole step")
    ap.add_argument("--M", type=int, default=256)
    ap.add_argument("--O", type=int, default=21504)
    ap.add_argument("--I", type=int, default=5376)
    ap.add_argument("--rank", type=int, default=64)
    ap.add_argument("--layers", type=int, default=4)
    ap.add_argument("--G", type=int, default=1)
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--b2b", action="store_true", help="--op: time --iters calls back to back (no L2 flush)")
    ap.add_argument("--bufs", type=int, default=4, help="--op forward --b2b: independent problems cycled over")
    ap.add_argument("--no-residual", action="store_true", help="--op prelude: skip the residual output")
    args = ap.parse_args(argv)
    if args.op:
        return run_op(args)
    if args.warmup < 3 and args.impl == "native":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
