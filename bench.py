#!/usr/bin/env python
"""Throughput of the theta-bundle hot path on B200, against its roofline.

One step is one pass of every stage of the path over four synthetic
workloads, all resident in device memory at once (bf16 weights drawn as a
common N(0,0.02) base plus per-layer N(0,0.005) noise, factors U, V ~
N(0,0.01), activations X ~ N(0,1)):

  C1  Gemma-3-1B shapes (26 layers; q [1024,1152], k/v [256,1152],
      o [1152,1024], gate/up [6912,1152], down [1152,6912]), rank 32,
      G in {26, 1}: prelude, reconstruct, frob, forward at M in {1, 16, 256}
  C2  the same shapes at G = 4 (bands of 7,7,6,6 layers), rank 64: the
      decode forward of every family of every layer at M in {1,2,4,8,16,32}
  C3  Gemma-4-31B shapes (60 layers; q [8192,5376], k/v [2048,5376],
      o [5376,8192], gate/up [21504,5376], down [5376,21504]), rank 64,
      G in {1, 15, 60}: the forward of every family of every layer at
      M in {1, 64, 2048} (M = 2048 is the tensor-bound prefill)
  C4  the decomposition sweep: 60 layers of the 31B gate family
      [21504,5376], G in {1, 4, 15, 60}, rank 64: prelude (band mean, row
      scale, residual), reconstruct and relative Frobenius error per layer

The stages are (entry points of libtheta):
  prelude      theta_decompose_prelude      W0 per band, s and R per layer
  reconstruct  theta_reconstruct_band       diag(s).W0 + U.V^T for the layers of a band
  frob         theta_frob_error             ||W - W_rec||_F / ||W||_F per layer
  forward      theta_linear_forward (one or two tokens on Gemma-3-1B shapes:
               theta_linear_forward_grouped, one call for all 182 problems)

Accounting. Each call's algorithmic bytes are the minimum it must move
(inputs read once, outputs written once). Within one stage, calls that share
a tensor (the layers of a band read the same W0; every call of a stage reads
the same X) find it in L2, so the HBM-honest count ("unique" bytes) takes
each shared tensor once per stage; the per-call count is reported next to it
where they differ. L2 (126 MB) is flushed by a 256 MiB write before every
stage, so no stage reads what the previous one left in L2; the flushes are
in the step time, not in the stage times. A stage's roofline time is
max(unique bytes / HBM copy bandwidth, flops / sustained bf16 tensor
throughput) from MEASURED_PEAKS.json; its fraction is that time over the
measured time. The value is HBM-honest GB/s over the whole step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
  python bench.py --op forward|gate_up|forward_nvfp4|grouped|prelude|... (one entry point)

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
from dataclasses import dataclass, field

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synthetic as syn  # noqa: E402

METRIC = "theta-forward TFLOP/s (prefill) & GB/s (decode) vs B200 roofline; decompose GB/s"
BF16 = 2  # bytes
PREFILL_M = 1024  # forwards of at least this many tokens are the prefill regime
RIDGE_M = 128     # between RIDGE_M and PREFILL_M: near the ridge point


@dataclass(frozen=True)
class Config:
    key: str
    model: syn.Model
    G: tuple
    rank: int
    M: tuple
    decompose: bool
    forward: bool
    desc: str


GATE31 = syn.Model("gemma4-31b-gate", 60, {"gate": (21504, 5376)})

CONFIGS = {
    "C1": Config("C1", syn.GEMMA3_1B, (26, 1), 32, (1, 16, 256), True, True,
                 "gemma3-1b-shaped, 26 layers x 7 families, G in {26,1}, rank 32: prelude + reconstruct + frob + "
                 "forward at M in {1,16,256}"),
    "C2": Config("C2", syn.GEMMA3_1B, (4,), 64, (1, 2, 4, 8, 16, 32), False, True,
                 "gemma3-1b-shaped decode sweep, G=4 (7,7,6,6), rank 64: forward of 7 families x 26 layers at "
                 "M in {1,2,4,8,16,32}"),
    "C3": Config("C3", syn.GEMMA4_31B, (1, 15, 60), 64, (1, 64, 2048), False, True,
                 "gemma4-31b-shaped, 60 layers x 7 families, G in {1,15,60}, rank 64: forward at M in "
                 "{1,64,2048}"),
    "C4": Config("C4", GATE31, (1, 4, 15, 60), 64, (), True, False,
                 "decomposition sweep, 60 x [21504,5376] bf16, G in {1,4,15,60}, rank 64: prelude + reconstruct + "
                 "frob"),
}
DEFAULT_CONFIGS = ("C1", "C2", "C3", "C4")


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


def reconstruct_band_launches(L, G, r):
    """Kernel launches of the theta_reconstruct_band calls of one family, one
    call per band: one launch per 64 layers of a band, or one per layer for
    one-layer bands, rank 0 or rank above 128."""
    sizes = [L // G + (1 if b < L % G else 0) for b in range(G)]
    if r == 0 or r > 128:
        return L
    return sum(1 if n == 1 else -(-n // 64) for n in sizes)


def grouped_stage(cfg, M):
    """One or two tokens on Gemma-3-1B shapes: one grouped call per stage."""
    return M <= 2 and cfg.model.name == syn.GEMMA3_1B.name


def forward_streams(M, streams):
    """Streams a forward stage fans out over: the tensor-bound prefill calls
    fill the GPU on their own, so four streams only overlap their tails."""
    return min(streams, 4) if M >= PREFILL_M else streams


def regime_of(kind, M):
    if kind != "forward":
        return "decompose"
    return "prefill" if M >= PREFILL_M else "ridge" if M >= RIDGE_M else "decode"


def plan_stages(cfg: Config, grouped=True):
    """Host-side plan of one config's stages in step order: per stage its
    algorithmic bytes (per call, summed), HBM-honest unique bytes, flops,
    kernel launches and calls."""
    model, L, r = cfg.model, cfg.model.num_layers, cfg.rank
    fams = model.shapes
    nf = len(fams)
    out = []
    for G in cfg.G:
        if cfg.decompose:
            b = sum(bytes_prelude(L, G, O, I) for (O, I) in fams.values())
            out.append(dict(cfg=cfg.key, kind="prelude", G=G, M=0, bytes=b, unique=b, flops=0, calls=nf,
                            launches=sum(prelude_launches(L, G, I) for (_, I) in fams.values())))
            b = L * sum(bytes_reconstruct(O, I, r) for (O, I) in fams.values())
            # the layers of a band read one W0: once per band from HBM
            u = b - (L - G) * sum(O * I * BF16 for (O, I) in fams.values())
            out.append(dict(cfg=cfg.key, kind="reconstruct", G=G, M=0, bytes=b, unique=u,
                            flops=L * sum(2 * O * I * r for (O, I) in fams.values()), calls=nf * G,
                            launches=nf * reconstruct_band_launches(L, G, r)))
            b = L * sum(bytes_frob(O, I) for (O, I) in fams.values())
            out.append(dict(cfg=cfg.key, kind="frob", G=G, M=0, bytes=b, unique=b, flops=0, calls=nf * L,
                            launches=2 * nf * L))
        if cfg.forward:
            for M in cfg.M:
                b = L * sum(bytes_forward(M, O, I, r) for (O, I) in fams.values())
                f = L * sum(flops_forward(M, O, I, r) for (O, I) in fams.values())
                # W0 once per band; X once per distinct input width
                u = b - (L - G) * sum(O * I * BF16 for (O, I) in fams.values())
                in_dims = {I for (_, I) in fams.values()}
                u -= sum(M * I * BF16 for (_, I) in fams.values()) * L - sum(M * I * BF16 for I in in_dims)
                grp = grouped and grouped_stage(cfg, M)
                launches = (3 if r > 0 else 1) if grp else nf * L * (2 if r > 0 else 1)
                out.append(dict(cfg=cfg.key, kind="forward", G=G, M=M, bytes=b, unique=u, flops=f, calls=nf * L,
                                launches=launches, grouped=grp))
    for st in out:
        st["name"] = f"{st['cfg']}.{st['kind']}.G{st['G']}" + (f".M{st['M']}" if st["kind"] == "forward" else "")
        st["regime"] = regime_of(st["kind"], st["M"])
        st["L"] = L
    return out


def plan_all(keys=DEFAULT_CONFIGS, grouped=True):
    return [st for k in keys for st in plan_stages(CONFIGS[k], grouped)]


def roofline_time(st, peaks):
    """Seconds the stage would take at the measured HBM copy bandwidth or the
    sustained bf16 tensor throughput, whichever bounds it."""
    t_hbm = st["unique"] / (peaks["hbm_gbs"] * 1e9)
    t_tc = st["flops"] / (peaks["bf16_tflops_sustained"] * 1e12)
    return max(t_hbm, t_tc), ("tensor" if t_tc > t_hbm else "hbm")


def summarize(stages, stage_ms, step_ms, peaks):
    """Per-stage parts, per-regime totals and the step's roofline-time
    fraction from measured stage times (ms per step)."""
    parts, regimes = {}, {}
    for st, ms in zip(stages, stage_ms):
        s = ms * 1e-3
        t_id, bound = roofline_time(st, peaks)
        p = {"ms": round(ms, 4), "bound": bound, "frac": round(t_id / s, 4),
             "GB/s": round(st["unique"] / s / 1e9, 1),
             "frac_hbm": round(st["unique"] / s / 1e9 / peaks["hbm_gbs"], 4)}
        if st["unique"] != st["bytes"]:
            p["GB/s_per_call"] = round(st["bytes"] / s / 1e9, 1)
            p["frac_hbm_per_call"] = round(st["bytes"] / s / 1e9 / peaks["hbm_gbs"], 4)
        if st["flops"]:
            p["TFLOP/s"] = round(st["flops"] / s / 1e12, 2)
            p["frac_tensor"] = round(st["flops"] / s / 1e12 / peaks["bf16_tflops_sustained"], 4)
        parts[st["name"]] = p
        r = regimes.setdefault(st["regime"], {"ms": 0.0, "ideal_ms": 0.0, "bytes": 0, "flops": 0, "stages": 0})
        r["ms"] += ms
        r["ideal_ms"] += t_id * 1e3
        r["bytes"] += st["unique"]
        r["flops"] += st["flops"]
        r["stages"] += 1
    for name, r in regimes.items():
        s = r["ms"] * 1e-3
        r["frac"] = round(r["ideal_ms"] / r["ms"], 4)
        r["GB/s"] = round(r["bytes"] / s / 1e9, 1)
        r["frac_hbm"] = round(r["bytes"] / s / 1e9 / peaks["hbm_gbs"], 4)
        if r["flops"]:
            r["TFLOP/s"] = round(r["flops"] / s / 1e12, 2)
            r["frac_tensor"] = round(r["flops"] / s / 1e12 / peaks["bf16_tflops_sustained"], 4)
        r["ms"] = round(r["ms"], 3)
        r["ideal_ms"] = round(r["ideal_ms"], 3)
    ideal = sum(roofline_time(st, peaks)[0] for st in stages) * 1e3
    return parts, regimes, round(ideal / step_ms, 4)


# The main kernel behind each group of stages, and the sources that define it
# and its launch code (shared device helpers included): a recorded ncu traffic
# figure stands only while these files hash to the value recorded beside it.
KIND_SOURCES = {
    "prelude": ["prelude_kernels.cu", "stream_kernels.cu", "common.cuh", "umma_ptx.cuh"],
    "reconstruct": ["umma_kernels.cu", "umma_ptx.cuh", "common.cuh"],
    "frob": ["stream_kernels.cu", "common.cuh"],
    "forward_decode": ["gemv_kernels.cu", "umma_kernels.cu", "umma_ptx.cuh", "common.cuh"],
    "forward_ridge": ["umma_kernels.cu", "umma_ptx.cuh", "common.cuh"],
    "forward_prefill": ["umma_kernels.cu", "umma_ptx.cuh", "common.cuh"],
}
KERNEL_NAMES = {
    "prelude": "prelude_pipe_kernel / prelude_band2_kernel (+ band_mean_kernel)",
    "reconstruct": "recon_kernel",
    "frob": "frob_partial_kernel + frob_final_kernel",
    "forward_decode": "gemv_rows_kernel / grouped_rows_kernel / umma_kernel<16..64,FORWARD>",
    "forward_ridge": "pair_kernel<FORWARD> (+ umma_kernel<64,XV>)",
    "forward_prefill": "pair_kernel<FORWARD> (+ umma_kernel<64,XV>)",
}


def group_key(st):
    return st["kind"] if st["kind"] != "forward" else f"forward_{st['regime']}"


def dominant_group(stages, stage_ms):
    """The (config, kernel group) with the most time per step."""
    groups = {}
    for st, ms in zip(stages, stage_ms):
        g = groups.setdefault((st["cfg"], group_key(st)), {"ms": 0.0, "bytes": 0, "unique": 0, "flops": 0,
                                                            "calls": 0, "names": []})
        g["ms"] += ms
        g["bytes"] += st["bytes"]
        g["unique"] += st["unique"]
        g["flops"] += st["flops"]
        g["calls"] += st["calls"]
        g["names"].append(st["name"])
    return max(groups.items(), key=lambda kv: kv[1]["ms"])


def roofline_entry(stages, stage_ms, peaks):
    (cfg, kind), g = dominant_group(stages, stage_ms)
    per_call_s = g["ms"] * 1e-3 / g["calls"]
    t_hbm = g["unique"] / (peaks["hbm_gbs"] * 1e9)
    t_tc = g["flops"] / (peaks["bf16_tflops_sustained"] * 1e12)
    if t_tc > t_hbm:
        achieved = g["flops"] / g["calls"] / per_call_s / 1e12
        ent = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peaks["bf16_tflops_sustained"],
               "unit": "TFLOP/s", "peak_kind": "bf16 dense, sustained (kernel timed inside a seconds-long step)"}
    else:
        achieved = g["unique"] / g["calls"] / per_call_s / 1e9
        ent = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
               "peak_kind": "HBM copy bandwidth"}
    ent["frac"] = round(achieved / ent["peak"], 4)
    ent["traffic"] = recorded_traffic(kind, cfg)
    ent.update({"kernel": KERNEL_NAMES[kind], "stages": g["names"], "peak_source": peaks["source"],
                "launches_per_step": g["calls"], "bytes_per_launch": round(g["unique"] / g["calls"]),
                "flops_per_launch": round(g["flops"] / g["calls"])})
    return ent


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

    def __init__(self, gpu_index: int, period_ms: int = 50):
        self.gpu = gpu_index
        self.period = period_ms
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
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
        sm, mx, power, reasons = [], [], [], set()
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
            try:
                power.append(float(parts[3]))
            except ValueError:
                pass
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        out = {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
               "samples": len(sm), "sm_mhz_min": min(sm)}
        if power:
            out["power_w_max"] = max(power)
        return out


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


def workload_name(keys):
    return "theta path, one step = " + "; ".join(f"{k}: {CONFIGS[k].desc}" for k in keys)


# --------------------------------------------------------------- workload
class Workload:
    """All device tensors of one step and the callables of its stages."""

    def __init__(self, theta, torch, keys=DEFAULT_CONFIGS, seed=0, streams=32, grouped=True):
        self.theta, self.torch = theta, torch
        self.keys = tuple(keys)
        self.nstreams = streams
        self.side = [torch.cuda.Stream() for _ in range(streams)]
        self.grouped = grouped
        self.stages = plan_all(self.keys, grouped)
        self.seed = seed
        self.t = {}  # per config: dict of tensors
        dev, bf = "cuda", torch.bfloat16
        fwd_ws = 256
        for k in self.keys:
            cfg = CONFIGS[k]
            d = self.t[k] = {}
            L, r = cfg.model.num_layers, cfg.rank
            fams = cfg.model.shapes
            d["U"] = {f: [syn.device_normal((O, r), 0.01, seed, k, "U", f, l) for l in range(L)]
                      for f, (O, I) in fams.items()}
            d["V"] = {f: [syn.device_normal((I, r), 0.01, seed, k, "V", f, l) for l in range(L)]
                      for f, (O, I) in fams.items()}
            d["bands"] = {G: theta.theta_band_index(L, G)[0] for G in cfg.G}
            if cfg.decompose:
                d["W"] = {f: syn.device_family_weights(L, O, I, seed=seed, family=f"{k}-{f}")
                          for f, (O, I) in fams.items()}
                d["W0"] = {f: [torch.empty(O, I, dtype=bf, device=dev) for _ in range(max(cfg.G))]
                           for f, (O, I) in fams.items()}
                d["s"] = {f: [torch.empty(O, dtype=torch.float32, device=dev) for _ in range(L)]
                          for f, (O, I) in fams.items()}
                d["R"] = {f: [torch.empty(O, I, dtype=bf, device=dev) for _ in range(L)] for f, (O, I) in fams.items()}
                d["rec"] = {f: [torch.empty(O, I, dtype=bf, device=dev) for _ in range(L)]
                            for f, (O, I) in fams.items()}
                d["frob"] = torch.zeros(len(cfg.G), len(fams), L, dtype=torch.float64, device=dev)
            elif len(cfg.G) == 1 and cfg.model.name == syn.GEMMA3_1B.name:
                # forward only at one G: the shared blocks and scales of a real
                # prelude of freshly drawn weights (set-up, untimed)
                G = cfg.G[0]
                d["W0"], d["s"] = {}, {}
                for f, (O, I) in fams.items():
                    w = syn.device_family_weights(L, O, I, seed=seed, family=f"{k}-{f}")
                    d["W0"][f] = [torch.empty(O, I, dtype=bf, device=dev) for _ in range(G)]
                    d["s"][f] = [torch.empty(O, dtype=torch.float32, device=dev) for _ in range(L)]
                    theta.theta_decompose_prelude(w, G, d["W0"][f], d["s"][f], None)
                    del w
                torch.cuda.synchronize()
            else:
                # forward only over several G: one block per band of the finest
                # banding; a coarser banding reads the first G of them
                d["W0"] = {f: [syn.device_normal((O, I), 0.02, seed, k, "W0", f, b) for b in range(max(cfg.G))]
                           for f, (O, I) in fams.items()}
                d["s"] = {f: [torch.add(syn.device_normal((O,), 0.02, seed, k, "s", f, l, dtype="f32"), 1.0)
                              for l in range(L)] for f, (O, I) in fams.items()}
            if cfg.forward:
                in_dims = sorted({I for (_, I) in fams.values()})
                d["X"] = {(M, I): syn.device_normal((M, I), 1.0, seed, k, "X", M, I) for M in cfg.M for I in in_dims}
                d["Y"] = {}
                for M in cfg.M:
                    for f, (O, I) in fams.items():
                        for slot in range(forward_streams(M, streams)):
                            d["Y"][(M, f, slot)] = torch.empty(M, O, dtype=bf, device=dev)
                    for (O, I) in fams.values():
                        fwd_ws = max(fwd_ws, theta.theta_workspace_size(theta.THETA_OP_LINEAR_FORWARD, M, O, I, r,
                                                                        theta.THETA_BF16))
        self.fwd_ws = [torch.empty(fwd_ws, dtype=torch.uint8, device=dev) for _ in range(streams)]
        fb = theta.theta_workspace_size(theta.THETA_OP_FROB_ERROR, 1, 1, 1, 0, theta.THETA_BF16)
        self.frob_ws = [torch.empty(fb, dtype=torch.uint8, device=dev) for _ in range(streams)]
        # one or two tokens on the small model: every problem of a stage in one grouped call
        self.groups = {}
        for st in self.stages:
            if st["kind"] == "forward" and st.get("grouped"):
                self.groups[st["name"]] = theta.ForwardGroup(self._forward_problems(st))
        gb = max([g.workspace_size() for g in self.groups.values()] + [256])
        self.grp_ws = torch.empty(gb, dtype=torch.uint8, device=dev)
        l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
        self.flush_buf = torch.empty(max(256 << 20, 2 * l2), dtype=torch.uint8, device=dev)

    # ------------------------------------------------------------------
    def _forward_problems(self, st):
        """(X, W0, s, U, V, Y) of every call of a forward stage, layer-major;
        call i writes the Y slot i mod the stage's stream count."""
        cfg, d = CONFIGS[st["cfg"]], self.t[st["cfg"]]
        G, M = st["G"], st["M"]
        band = d["bands"][G]
        nslot = forward_streams(M, self.nstreams)
        probs = []
        for l in range(cfg.model.num_layers):
            for f, (O, I) in cfg.model.shapes.items():
                i = len(probs)
                probs.append((d["X"][(M, I)], d["W0"][f][band[l]], d["s"][f][l], d["U"][f][l], d["V"][f][l],
                              d["Y"][(M, f, i % nslot)]))
        return probs

    def _fan_out(self, calls, nstreams=None):
        """Runs calls(k), k the stream slot, round-robin over the side streams
        (forked from and joined back to the current stream)."""
        torch = self.torch
        side = self.side[:nstreams or self.nstreams]
        main = torch.cuda.current_stream()
        for st in side:
            st.wait_stream(main)
        for i, c in enumerate(calls):
            k = i % len(side)
            with torch.cuda.stream(side[k]):
                c(k)
        for st in side:
            main.wait_stream(st)

    def stage_fn(self, st):
        t, k, G = self.theta, st["cfg"], st["G"]
        cfg, d = CONFIGS[k], self.t[k]
        fams = cfg.model.shapes
        L = cfg.model.num_layers
        if st["kind"] == "prelude":
            return lambda: self._fan_out([lambda s, f=f: t.theta_decompose_prelude(d["W"][f], G, d["W0"][f][:G],
                                                                                   d["s"][f], d["R"][f])
                                          for f in fams])
        band = d["bands"][G]
        if st["kind"] == "reconstruct":
            # one call per band: each W0 tile read once for all the band's layers
            calls = []
            for f in fams:
                for b in range(G):
                    ls = [l for l in range(L) if band[l] == b]
                    calls.append(lambda s, f=f, b=b, ls=ls: t.theta_reconstruct_band(
                        [d["s"][f][l] for l in ls], d["W0"][f][b], [d["U"][f][l] for l in ls],
                        [d["V"][f][l] for l in ls], [d["rec"][f][l] for l in ls]))
            return lambda: self._fan_out(calls)
        if st["kind"] == "frob":
            gi = cfg.G.index(G)
            fi = {f: i for i, f in enumerate(fams)}
            return lambda: self._fan_out([lambda s, f=f, l=l: t.theta_frob_error(d["W"][f][l], d["rec"][f][l],
                                                                                d["frob"][gi, fi[f], l:l + 1],
                                                                                self.frob_ws[s])
                                          for l in range(L) for f in fams])
        if st["name"] in self.groups:
            grp = self.groups[st["name"]]
            return lambda: t.theta_linear_forward_grouped(grp, self.grp_ws)
        probs = self._forward_problems(st)
        n = forward_streams(st["M"], self.nstreams)
        return lambda: self._fan_out([lambda s, p=p: t.theta_linear_forward(*p, self.fwd_ws[s]) for p in probs], n)

    def flush_l2(self):
        self.flush_buf.fill_(1)

    # host side of the end-to-end run -----------------------------------
    def input_tensors(self, keys=None):
        """Every tensor a step reads that no stage of it writes (of the given
        configs, default all)."""
        ins = []
        for k in (self.keys if keys is None else keys):
            cfg, d = CONFIGS[k], self.t[k]
            for f in cfg.model.shapes:
                ins += d["U"][f] + d["V"][f]
                if cfg.decompose:
                    ins += d["W"][f]
                else:
                    ins += d["W0"][f] + d["s"][f]
            if cfg.forward:
                ins += list(d["X"].values())
        return ins

    def output_tensors(self):
        """The step's results read back: Frobenius errors, row scales, and the
        last forward output of every (stage token count, family, stream slot)."""
        outs = []
        for k in self.keys:
            cfg, d = CONFIGS[k], self.t[k]
            if cfg.decompose:
                outs.append(d["frob"])
                for f in cfg.model.shapes:
                    outs += d["s"][f]
            if cfg.forward:
                outs += list(d["Y"].values())
        return outs


# --------------------------------------------------------------- CPU oracle
# Bounded row samples of each config for the oracle on the host: the first
# `rows` output rows of every family (scaled per config), and for the 31B
# forward one layer per G (its T = X.V costs the same whatever the rows).
SAMPLE_ROWS = {"C1": 1.0, "C2": 1.0, "C3": 0.125, "C4": 0.125}


def oracle_sample_inputs(rows=64, seed=0, keys=DEFAULT_CONFIGS):
    """Host inputs of one bounded sample of the step (drawn once, outside any
    timing): per config and family the first rows of every layer's weight,
    the factors and the activations; for a forward-only config also the
    shared blocks and row scales its forward consumes."""
    import oracle
    jobs = []
    for k in keys:
        cfg = CONFIGS[k]
        n_rows = max(1, int(rows * SAMPLE_ROWS[k]))
        L, r = cfg.model.num_layers, cfg.rank
        layers = list(range(L)) if (cfg.decompose or cfg.model.name == syn.GEMMA3_1B.name) else [0]
        X_by_I = {}
        for fam, (O, I) in cfg.model.shapes.items():
            n = min(n_rows, O)
            w = syn.host_family_weights(L, n, I, seed=seed, family=f"cpu-{k}-{fam}", dtype="bf16")
            U = {l: syn.host_normal((n, r), 0.01, seed, k, "U", fam, l, dtype="bf16") for l in layers}
            V = {l: syn.host_normal((I, r), 0.01, seed, k, "V", fam, l, dtype="bf16") for l in layers}
            if I not in X_by_I:
                X_by_I[I] = {m: syn.host_activations(m, I, seed=seed, tag=f"cpu-{k}-{m}", dtype="bf16")
                             for m in cfg.M}
            fwd_in = {}
            if not cfg.decompose:
                for G in cfg.G:
                    band, _ = oracle.band_index(L, G)
                    W0 = oracle.band_mean(w, G, "bf16")
                    fwd_in[G] = [(W0[band[l]], oracle.round_to(oracle.row_scale(w[l], W0[band[l]]), "f32"))
                                 for l in layers]
            jobs.append((k, cfg, fam, n, I, w, U, V, X_by_I[I], layers, fwd_in))
    return jobs


def oracle_sample_run(jobs):
    """The fp64 oracle over one sample (every stage of each config, as in the
    step). Returns (HBM-honest algorithmic bytes of the sample, seconds,
    per-config seconds)."""
    import oracle
    total, per = 0, {}
    t_all = time.perf_counter()
    for k, cfg, fam, n, I, w, U, V, X, layers, fwd_in in jobs:
        t0 = time.perf_counter()
        L, r = cfg.model.num_layers, cfg.rank
        for G in cfg.G:
            if cfg.decompose:
                band, _ = oracle.band_index(L, G)
                W0 = oracle.band_mean(w, G, "bf16")
                for l in layers:
                    w0 = W0[band[l]]
                    s = oracle.row_scale(w[l], w0)
                    oracle.residual(w[l], w0, s, "bf16")
                    rec = oracle.reconstruct(oracle.round_to(s, "f32"), w0, U[l], V[l], "bf16")
                    oracle.frob_error(w[l], rec)
                    if cfg.forward:
                        s32 = oracle.round_to(s, "f32")
                        for m in cfg.M:
                            oracle.linear_forward(X[m], w0, s32, U[l], V[l], "bf16")
                total += bytes_prelude(L, G, n, I) + L * (bytes_reconstruct(n, I, r) + bytes_frob(n, I))
                if cfg.forward:
                    total += L * sum(bytes_forward(m, n, I, r) for m in cfg.M)
            else:
                for j, l in enumerate(layers):
                    w0, s32 = fwd_in[G][j]
                    for m in cfg.M:
                        oracle.linear_forward(X[m], w0, s32, U[l], V[l], "bf16")
                        total += bytes_forward(m, n, I, r)
        per[k] = per.get(k, 0.0) + time.perf_counter() - t0
    return total, time.perf_counter() - t_all, per


def oracle_sample_step(rows=64, seed=0, keys=DEFAULT_CONFIGS):
    """Inputs, then one timed run of the sample."""
    return oracle_sample_run(oracle_sample_inputs(rows, seed, keys))


def cpu_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((d.get("num_threads", 1) for d in info), default=1)
        return int(n)
    except Exception:
        return len(os.sched_getaffinity(0))


def _cpu_leg(target_s, jobs):
    done, spent, reps, per = 0, 0.0, 0, {}
    while spent < target_s and reps < 50:
        b, s, p = oracle_sample_run(jobs)
        done += b
        spent += s
        reps += 1
        for k, v in p.items():
            per[k] = per.get(k, 0.0) + v
    return done / spent / 1e9, reps, spent, per


def sample_text(rows, keys):
    parts = []
    for k in keys:
        n = max(1, int(rows * SAMPLE_ROWS[k]))
        cfg = CONFIGS[k]
        lay = "all layers" if (cfg.decompose or cfg.model.name == syn.GEMMA3_1B.name) else "layer 0 of each G"
        parts.append(f"{k}: first {n} output rows of each family, {lay}")
    return "; ".join(parts)


def cpu_baseline(target_s=12.0, rows=16, keys=DEFAULT_CONFIGS):
    """The oracle on the host: all threads, then one thread, on row samples."""
    np.ones((64, 64)) @ np.ones((64, 64))  # load BLAS so its threads are visible
    cores = cpu_threads()
    jobs = oracle_sample_inputs(rows, 0, keys)
    v_all, reps, spent, per = _cpu_leg(target_s / 2, jobs)
    out = {"value": v_all, "unit": "GB/s", "cores": cores, "kind": "oracle",
           "sample": f"{reps} x ({sample_text(rows, keys)}); every stage of each config; {spent:.1f} s",
           "seconds_per_config": {k: round(v / reps, 3) for k, v in per.items()}}
    try:
        import threadpoolctl
        with threadpoolctl.threadpool_limits(1):
            v1, reps1, spent1, _ = _cpu_leg(target_s / 2, jobs)
        out["single_thread"] = {"value": v1, "unit": "GB/s", "cores": 1, "reps": reps1,
                                "seconds": round(spent1, 1)}
    except ImportError:
        pass
    return out


def run_reference(args):
    """The oracle as the reference arm: each step is one bounded row sample."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    keys = tuple(args.configs.split(","))
    jobs = oracle_sample_inputs(args.ref_rows, 0, keys)  # host inputs, drawn once
    for _ in range(args.warmup):
        oracle_sample_run(jobs)
    times, nbytes = [], 0
    for i in range(args.steps):
        b, s, _ = oracle_sample_run(jobs)
        times.append(s)
        nbytes = b
    per_step = sum(times) / len(times)
    value = nbytes / per_step / 1e9
    line = result_line(value=value, unit="GB/s", n_gpus=args.gpus, steps=args.steps, warmup=args.warmup,
                       ms_per_step=per_step * 1e3, extra={
                           "impl": "reference", "dtype": "f64",
                           "data": "synthetic (seeded; weights, factors and activations drawn on the host)",
                           "config": {"workload": workload_name(keys), "sample": sample_text(args.ref_rows, keys),
                                      "l2": "n/a (CPU)"},
                           "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle",
                                            "sample": sample_text(args.ref_rows, keys)},
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

    keys = tuple(args.configs.split(","))
    peaks = measured_peaks()
    # many independent calls in flight at once: whole tiles per CTA
    theta.theta_set_policy(theta.THETA_POLICY_THROUGHPUT)
    wl = Workload(theta, torch, keys=keys, seed=rank, streams=args.streams, grouped=not args.per_call_decode)
    stages = wl.stages
    fns = [wl.stage_fn(st) for st in stages]
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
                wl.flush_l2()
                if events is not None:
                    events[2 * i].record(stream)
                f()
                if events is not None:
                    events[2 * i + 1].record(stream)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    theta.theta_device_status(stream)

    n_st = len(stages)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * n_st)] for _ in range(args.steps)]
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
    stage_ms = [sum(ev[k][2 * i].elapsed_time(ev[k][2 * i + 1]) for k in range(args.steps)) / args.steps
                for i in range(n_st)]
    ms_per_step = total_ms / args.steps
    unique = sum(st["unique"] for st in stages)
    value = world * unique / (ms_per_step * 1e-3) / 1e9
    launches = sum(st["launches"] for st in stages) * args.steps
    parts, regimes, roof_frac = summarize(stages, stage_ms, ms_per_step, peaks)
    roofline = roofline_entry(stages, stage_ms, peaks)
    flush_ms = ms_per_step - sum(stage_ms)

    e2e = None
    if not args.skip_e2e:
        e2e = run_e2e(torch, wl, run, stream, unique, min(args.steps, args.e2e_steps), world)
    del graphs, run

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        cpu = cpu_baseline(target_s=args.cpu_seconds, keys=keys)

    if rank == 0:
        line = result_line(value=round(value, 2), unit="GB/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
                           ms_per_step=round(ms_per_step, 4), extra={
                               "config": {"workload": workload_name(keys), "configs": list(keys),
                                          "global_batch": max(m for k in keys for m in CONFIGS[k].M or (0,)),
                                          "seq_len": 1, "parallelism": f"independent replicas x{world}",
                                          "graphs": not args.no_graph, "streams": args.streams,
                                          "policy": "throughput", "decode": "per call" if args.per_call_decode
                                          else "grouped (one- and two-token stages of the 1B shapes)",
                                          "value_counts": "HBM-honest algorithmic bytes: every input read once "
                                                          "per call, except that a tensor several calls of one "
                                                          "stage share (a band's W0, the stage's X) counts once "
                                                          "per stage",
                                          "l2": f"flushed before every stage by a {wl.flush_buf.numel() >> 20} MiB "
                                                f"write ({flush_ms:.3f} ms per step, in the step time, not in "
                                                f"the stage times)"},
                               "regimes": regimes,
                               "roofline_time_frac": roof_frac,
                               "parts": parts,
                               "roofline": roofline,
                               "cpu_baseline": cpu,
                               "e2e": e2e,
                               "gpu_launches": launches,
                               "clocks": clocks.summary(),
                           })
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def run_e2e(torch, wl, run, stream, step_bytes, steps, world):
    """The same step through the public API with HOST buffers: every step
    copies every input tensor's bytes from pinned host memory, runs, and
    reads its results back into pinned host memory. The host inputs come
    from pinned pools of pre-drawn values (bf16 ~ N(0, 0.02); fp32 near 1),
    sliced to each tensor's size, so that tens of GB of inputs need no copy
    of their own in host memory.

    The copies of each config's inputs run on a second stream, so that they
    overlap the stages of the configs before it: a config's stages wait for
    its own copies, and a config's copies of the next step wait until its
    stages of this step are done with the tensors they overwrite."""
    ins = wl.input_tensors()
    outs = wl.output_tensors()
    # consecutive stages of one config, in step order
    segments = []
    for st, f in zip(wl.stages, run):
        if not segments or segments[-1][0] != st["cfg"]:
            segments.append((st["cfg"], []))
        segments[-1][1].append(f)
    seg_ins = [wl.input_tensors([k]) for k, _ in segments]
    assert sum(len(x) for x in seg_ins) == len(ins)
    copy_stream = torch.cuda.Stream()
    pools = {}
    for t in ins:
        pools.setdefault(t.dtype, 0)
        pools[t.dtype] = max(pools[t.dtype], t.numel())
    host = {}
    for dt, n in pools.items():
        h = torch.empty(n, dtype=dt, pin_memory=True)
        h.copy_(torch.randn(n, dtype=torch.float32).mul_(0.02).add_(1.0 if dt == torch.float32 else 0.0).to(dt))
        host[dt] = h
    h_out = torch.empty(max(t.numel() * t.element_size() for t in outs), dtype=torch.uint8, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in ins)
    d2h = sum(t.numel() * t.element_size() for t in outs)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    done = [None] * len(segments)  # a config's stages of the previous step finished
    start.record(stream)
    copy_stream.wait_stream(stream)
    for _ in range(steps):
        copied = []
        with torch.cuda.stream(copy_stream):
            for i, tensors in enumerate(seg_ins):
                if done[i] is not None:
                    copy_stream.wait_event(done[i])
                for t in tensors:
                    t.view(-1).copy_(host[t.dtype][:t.numel()], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(copy_stream)
                copied.append(ev)
        with torch.cuda.stream(stream):
            for i, (_, fns) in enumerate(segments):
                stream.wait_event(copied[i])
                for f in fns:
                    wl.flush_l2()
                    f()
                ev = torch.cuda.Event()
                ev.record(stream)
                done[i] = ev
            for t in outs:
                nb = t.numel() * t.element_size()
                h_out[:nb].copy_(t.reshape(-1).view(torch.uint8), non_blocking=True)
    stream.wait_stream(copy_stream)
    stop.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(stop), world, device="cuda") / steps
    return {"value": round(world * step_bytes / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3), "steps": steps,
            "copies": "each config's inputs on a second stream, overlapping the stages of the configs before it"}


# The sources that define each --op's kernels, for the recorded-traffic gate
def kernel_source_hash(kind=None):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_theta_forward_b200", "csrc")
    names = KIND_SOURCES.get(kind) or sorted(os.listdir(csrc))
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kind, cfg=None):
    """DRAM bytes per launch of a kernel group's main kernel from a committed
    ncu capture, or None when none is recorded for it or its sources changed
    since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    entry = rec.get(f"{cfg}.{kind}") or rec.get(kind)
    if not entry or entry.get("source_hash") != kernel_source_hash(kind):
        return None
    return entry.get("dram_bytes_per_launch")


def run_op(args):
    """One entry point on one synthetic problem, timed per call with CUDA
    events (median of --iters calls, L2 flushed before each, or --b2b calls
    back to back). Prints a JSON line with the achieved rate, its fraction of
    the measured roofline and the SM clocks sampled meanwhile."""
    import torch
    torch.cuda.set_device(0)
    import linear_theta_forward_b200 as theta
    peaks = measured_peaks()
    # the step runs under the throughput policy; single ops default to latency
    theta.theta_set_policy(theta.THETA_POLICY_THROUGHPUT if args.policy == "throughput"
                           else theta.THETA_POLICY_LATENCY)
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
    elif args.op == "layer_forward":
        # one layer of a model (--model 1b|31b): the forward of each of its 7
        # families in turn (layer-major order, as in the step)
        model = syn.GEMMA4_31B if args.model == "31b" else syn.GEMMA3_1B
        probs = []
        xs = {I_: syn.device_normal((M, I_), 1.0, seed, "X", M, I_) for (_, I_) in model.shapes.values()}
        for f, (O_, I_) in model.shapes.items():
            probs.append((xs[I_], syn.device_normal((O_, I_), 0.02, seed, "W0", f),
                          1.0 + syn.device_normal((O_,), 0.05, seed, "s", f, dtype="f32"),
                          syn.device_normal((O_, r), 0.01, seed, "U", f) if r else None,
                          syn.device_normal((I_, r), 0.01, seed, "V", f) if r else None,
                          torch.empty(M, O_, dtype=torch.bfloat16, device="cuda")))
        nb = max(theta.theta_workspace_size(theta.THETA_OP_LINEAR_FORWARD, M, O_, I_, r, theta.THETA_BF16)
                 for (O_, I_) in model.shapes.values())
        ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")

        def call():
            for X_, W0, s, U, V, Y in probs:
                theta.theta_linear_forward(X_, W0, s, U, V, Y, ws)
        nbytes = sum(bytes_forward(M, O_, I_, r) for (O_, I_) in model.shapes.values())
        nflops = sum(flops_forward(M, O_, I_, r) for (O_, I_) in model.shapes.values())
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
        model = syn.GEMMA3_1B
        xs = {I_: syn.device_normal((M, I_), 1.0, seed, "X", M, I_) for (_, I_) in model.shapes.values()}
        probs = []
        for fam, (O_, I_) in model.shapes.items():
            for l in range(L):
                probs.append((xs[I_], syn.device_normal((O_, I_), 0.02, seed + l, "W0", fam),
                              1.0 + syn.device_normal((O_,), 0.05, seed + l, "s", fam, dtype="f32"),
                              syn.device_normal((O_, r), 0.01, seed + l, "U", fam) if r else None,
                              syn.device_normal((I_, r), 0.01, seed + l, "V", fam) if r else None,
                              torch.empty(M, O_, dtype=torch.bfloat16, device="cuda")))
        if args.per_call_decode:
            nb = max(theta.theta_workspace_size(theta.THETA_OP_LINEAR_FORWARD, M, O_, I_, r, theta.THETA_BF16)
                     for (O_, I_) in model.shapes.values())
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
    elif args.op == "reconstruct_band":
        # the --layers layers of one band: one shared W0, each layer's s, U, V
        W0 = syn.device_normal((O, I), 0.02, seed, "W0", O, I)
        sl = [1.0 + syn.device_normal((O,), 0.05, seed + l, "s", O, dtype="f32") for l in range(L)]
        Ul = [syn.device_normal((O, r), 0.01, seed + l, "U", O, r) for l in range(L)] if r else None
        Vl = [syn.device_normal((I, r), 0.01, seed + l, "V", I, r) for l in range(L)] if r else None
        outs = [torch.empty(O, I, dtype=torch.bfloat16, device="cuda") for _ in range(L)]
        call = lambda: theta.theta_reconstruct_band(sl, W0, Ul, Vl, outs)  # noqa: E731
        # W0 read once for the band; every layer's s, U, V read and W written
        nbytes = O * I * BF16 + L * (bytes_reconstruct(O, I, r) - O * I * BF16)
        nflops = L * 2 * O * I * r
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
    # the sampler starts first (nvidia-smi needs a moment), and the timed
    # region repeats until it spans at least 0.6 s, so that the clocks seen
    # while it ran are on record
    with ClockSampler(0, period_ms=20) as clocks:
        time.sleep(0.3)
        t_end = time.perf_counter() + 0.6
        rounds, per_call = 0, []
        while rounds == 0 or time.perf_counter() < t_end:
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
                per_call.append(a.elapsed_time(b) / args.iters)
            else:
                for _ in range(args.iters):
                    flush.fill_(1)
                    a = torch.cuda.Event(enable_timing=True)
                    b = torch.cuda.Event(enable_timing=True)
                    a.record()
                    call()
                    b.record()
                    torch.cuda.synchronize()
                    per_call.append(a.elapsed_time(b))
            rounds += 1
    ms = statistics.median(per_call)
    if args.b2b:
        l2 = "calls back to back, no flush (median over %d rounds of %d calls)" % (rounds, args.iters)
        if args.op in ("forward", "forward_nvfp4", "gate_up"):
            l2 += ", cycling over %d independent problems" % args.bufs
    else:
        l2 = "flushed (256 MiB write) before every call (median of %d)" % len(per_call)
    theta.theta_device_status()
    line = {"op": args.op, "shape": {"M": M, "O": O, "I": I, "rank": r, "layers": L, "G": G}, "dtype": "bf16",
            "ms": round(ms, 5), "iters": args.iters, "l2": l2, "policy": args.policy,
            "GB/s": round(nbytes / (ms * 1e-3) / 1e9, 1),
            "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4), "algorithmic_bytes": nbytes,
            "clocks": clocks.summary()}
    if args.op == "layer_forward":
        line["shape"]["model"] = args.model
    if nflops:
        line["TFLOP/s"] = round(nflops / (ms * 1e-3) / 1e12, 2)
        line["frac_tensor_burst"] = round(nflops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--configs", default=",".join(DEFAULT_CONFIGS),
                    help="comma-separated subset of C1,C2,C3,C4 making up the step")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of replaying CUDA graphs")
    ap.add_argument("--streams", type=int, default=32, help="streams the independent calls of a stage spread over")
    ap.add_argument("--per-call-decode", action="store_true",
                    help="one theta_linear_forward per problem for one or two tokens instead of a grouped call")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-rows", type=int, default=8)
    ap.add_argument("--op", choices=["forward", "layer_forward", "forward_nvfp4", "gate_up", "grouped", "reconstruct",
                                     "reconstruct_band", "prelude", "frob", "svd"],
                    help="time one entry point on one problem instead of the whole step")
    ap.add_argument("--model", choices=["1b", "31b"], default="31b", help="--op layer_forward: the model's shapes")
    ap.add_argument("--policy", choices=["latency", "throughput"], default="latency",
                    help="--op: the library's launch policy (the step uses throughput)")
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
    for k in args.configs.split(","):
        if k not in CONFIGS:
            ap.error(f"unknown config {k!r}")
    if args.op:
        return run_op(args)
    if args.warmup < 3 and args.impl == "native":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
