"""bench.py's host-side bookkeeping on the CPU: the launch counts it claims
per step follow the library's dispatch (grouped or per-call decode), the
HBM-honest byte counts match a call-by-call recount, the stage summary
divides what it should, the per-group source lists behind recorded ncu
traffic name files that exist, and a recorded traffic figure is used only
while its sources are unchanged."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synthetic as syn  # noqa: E402


def _band_of(L, G):
    q, m = divmod(L, G)
    out = []
    for b in range(G):
        out += [b] * (q + (1 if b < m else 0))
    return out


def test_launch_counts_per_step():
    per_call = bench.plan_all(grouped=False)
    grouped = bench.plan_all(grouped=True)
    assert [s["name"] for s in per_call] == [s["name"] for s in grouped]
    n_grouped = 0
    for a, b in zip(per_call, grouped):
        assert a["bytes"] == b["bytes"] and a["flops"] == b["flops"] and a["unique"] == b["unique"]
        if b.get("grouped"):
            n_grouped += 1
            assert a["launches"] == 2 * a["calls"]  # T = X.V kernel + sweep per problem
            assert b["launches"] == 3               # T slices, their sums, one sweep
            assert b["M"] <= 2 and b["cfg"] in ("C1", "C2")
        else:
            assert a["launches"] == b["launches"]
    assert n_grouped == 4  # C1 M=1 at G=26 and G=1; C2 M=1 and M=2
    # prelude: one launch per family except the 60-layer single band of the
    # 31B gate family (band mean, then the row pass)
    pre = {s["name"]: s["launches"] for s in grouped if s["kind"] == "prelude"}
    assert pre == {"C1.prelude.G26": 7, "C1.prelude.G1": 7, "C4.prelude.G1": 2, "C4.prelude.G4": 1,
                   "C4.prelude.G15": 1, "C4.prelude.G60": 1}
    # reconstruct: one band call per (family, band); a one-layer band is one
    # per-layer launch (C1 at G = 26: 182; G = 1: 7; C4: 1 + 4 + 15 + 60)
    rec = {s["name"]: s["launches"] for s in grouped if s["kind"] == "reconstruct"}
    assert rec == {"C1.reconstruct.G26": 182, "C1.reconstruct.G1": 7, "C4.reconstruct.G1": 1,
                   "C4.reconstruct.G4": 4, "C4.reconstruct.G15": 15, "C4.reconstruct.G60": 60}
    assert bench.reconstruct_band_launches(130, 1, 64) == 3 and bench.reconstruct_band_launches(10, 2, 0) == 10
    assert sum(s["launches"] for s in grouped) == 11980
    assert sum(s["launches"] for s in per_call) == 11980 + 4 * (364 - 3)


@pytest.mark.parametrize("key", ["C1", "C2", "C3", "C4"])
def test_unique_bytes_match_a_call_by_call_recount(key):
    cfg = bench.CONFIGS[key]
    L, r = cfg.model.num_layers, cfg.rank
    for st in bench.plan_stages(cfg):
        G, M = st["G"], st["M"]
        band = _band_of(L, G)
        seen, total, per_call = set(), 0, 0
        for l in range(L):
            for f, (O, I) in cfg.model.shapes.items():
                if st["kind"] == "forward":
                    per_call += bench.bytes_forward(M, O, I, r)
                    reads = {("W0", f, band[l]): O * I * 2, ("X", M, I): M * I * 2}
                    total += 4 * O + r * (O + I) * 2 + M * O * 2  # s, U, V read; Y written
                elif st["kind"] == "reconstruct":
                    per_call += bench.bytes_reconstruct(O, I, r)
                    reads = {("W0", f, band[l]): O * I * 2}
                    total += 4 * O + r * (O + I) * 2 + O * I * 2
                else:
                    continue
                for key_, nb in reads.items():
                    if key_ not in seen:
                        seen.add(key_)
                        total += nb
        if st["kind"] in ("forward", "reconstruct"):
            assert st["bytes"] == per_call, st["name"]
            assert st["unique"] == total, st["name"]
        else:
            assert st["unique"] == st["bytes"], st["name"]
        assert st["unique"] <= st["bytes"]


def test_summary_fractions():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 2000.0, "bf16_tflops_sustained": 1000.0, "source": "test"}
    stages = [dict(name="a", cfg="C9", kind="frob", regime="decompose", bytes=2e9, unique=2e9, flops=0, calls=1),
              dict(name="b", cfg="C9", kind="forward", regime="prefill", bytes=1e9, unique=5e8, flops=4e12, calls=2)]
    parts, regimes, frac = bench.summarize(stages, [4.0, 8.0], 12.5, peaks)
    # a: 2 GB in 4 ms = 500 GB/s = half the 1000 GB/s roofline
    assert parts["a"]["frac"] == 0.5 and parts["a"]["bound"] == "hbm"
    # b: 4 TFLOP in 8 ms = 500 TFLOP/s of 1000 sustained; bytes alone need 0.5 ms
    assert parts["b"]["bound"] == "tensor" and parts["b"]["frac"] == 0.5
    assert parts["b"]["GB/s_per_call"] == 125.0 and parts["b"]["GB/s"] == 62.5
    assert regimes["prefill"]["TFLOP/s"] == 500.0
    assert frac == round((2.0 + 4.0) / 12.5, 4)
    (cfg, kind), g = bench.dominant_group(stages, [4.0, 8.0])
    assert (cfg, kind) == ("C9", "forward_prefill")
    ent = bench.roofline_entry(stages, [4.0, 8.0], peaks)
    assert ent["bound"] == "tensor" and ent["unit"] == "TFLOP/s" and ent["frac"] == 0.5
    assert ent["launches_per_step"] == 2 and ent["flops_per_launch"] == 2e12


def test_workload_fits_one_gpu():
    """Every tensor of the four configs resident at once stays well inside
    one B200's 180 GB."""
    total = 0
    for key in bench.DEFAULT_CONFIGS:
        cfg = bench.CONFIGS[key]
        L, r = cfg.model.num_layers, cfg.rank
        for (O, I) in cfg.model.shapes.values():
            total += L * r * (O + I) * 2 + L * O * 4          # U, V, s
            if cfg.decompose:
                total += 3 * L * O * I * 2 + max(cfg.G) * O * I * 2  # W, R, rec; W0 blocks
            else:
                total += max(cfg.G) * O * I * 2
            for M in cfg.M:
                total += bench.forward_streams(M, 32) * M * O * 2 + M * I * 2
    assert total < 140e9, total / 1e9


def test_traffic_sources_exist_and_gate_the_figure(tmp_path, monkeypatch):
    csrc = os.path.join(ROOT, "linear_theta_forward_b200", "csrc")
    for kind, files in bench.KIND_SOURCES.items():
        for f in files:
            assert os.path.exists(os.path.join(csrc, f)), (kind, f)
    assert set(bench.KERNEL_NAMES) == set(bench.KIND_SOURCES)
    path = os.path.join(ROOT, "profiles", "traffic.json")
    rec = json.load(open(path)) if os.path.exists(path) else {}
    for key, entry in rec.items():
        kind = key.split(".")[-1]
        assert entry["source_files"] == bench.KIND_SOURCES[kind]
        assert entry["dram_bytes_per_launch"] > 0
    # a figure recorded at another hash of the sources is not reported
    now = bench.kernel_source_hash("prelude")
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kind=None: now)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    entry = {"source_files": bench.KIND_SOURCES["prelude"], "dram_bytes_per_launch": 123}
    for stamp, expect in (("0" * 16, None), (now, 123)):
        fake = {"C4.prelude": dict(entry, source_hash=stamp)}
        (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(fake))
        assert bench.recorded_traffic("prelude", "C4") == expect
        assert bench.recorded_traffic("prelude", "C1") is None or stamp == now


def test_oracle_sample_is_bounded_and_counts_bytes():
    """The CPU baseline's sample runs every config's stages on a few rows and
    reports the bytes of exactly what it ran."""
    b, s, per = bench.oracle_sample_step(rows=8, keys=("C1", "C4"))
    assert set(per) == {"C1", "C4"} and s > 0
    expect = 0
    for key in ("C1", "C4"):
        cfg = bench.CONFIGS[key]
        n = max(1, int(8 * bench.SAMPLE_ROWS[key]))
        L, r = cfg.model.num_layers, cfg.rank
        for (O, I) in cfg.model.shapes.values():
            n_ = min(n, O)
            for G in cfg.G:
                expect += bench.bytes_prelude(L, G, n_, I) + L * (bench.bytes_reconstruct(n_, I, r)
                                                                  + bench.bytes_frob(n_, I))
                expect += L * sum(bench.bytes_forward(m, n_, I, r) for m in cfg.M)
    assert b == expect
    assert syn.GEMMA3_1B.num_layers == bench.CONFIGS["C1"].model.num_layers
