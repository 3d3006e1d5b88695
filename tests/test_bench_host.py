"""bench.py's host-side bookkeeping on the CPU: the launch counts it claims
per step follow the library's dispatch (grouped or per-call decode), the
per-stage source lists behind recorded ncu traffic name files that exist,
and a recorded traffic figure is used only while its sources are unchanged."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_launch_counts_per_step():
    L, nf = bench.MODEL.num_layers, len(bench.MODEL.shapes)
    per_call = bench.step_accounting(grouped=False)
    grouped = bench.step_accounting(grouped=True)
    assert [s["name"] for s in per_call] == [s["name"] for s in grouped]
    for a, b in zip(per_call, grouped):
        assert a["bytes"] == b["bytes"] and a["flops"] == b["flops"]
        if a["kind"] == "forward_m1":
            assert a["launches"] == 2 * nf * L  # T = X.V kernel + sweep per problem
            assert b["launches"] == 3  # T slices, their sums, one sweep
        else:
            assert a["launches"] == b["launches"]
    assert sum(s["launches"] for s in per_call) == 3290
    assert sum(s["launches"] for s in grouped) == 3290 - 2 * (2 * nf * L - 3)


def test_traffic_sources_exist_and_gate_the_figure(tmp_path, monkeypatch):
    csrc = os.path.join(ROOT, "linear_theta_forward_b200", "csrc")
    for kind, files in bench.KIND_SOURCES.items():
        for f in files:
            assert os.path.exists(os.path.join(csrc, f)), (kind, f)
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for kind, entry in rec.items():
        assert entry["source_files"] == bench.KIND_SOURCES[kind]
        assert entry["dram_bytes_per_launch"] > 0
    # a figure recorded at another hash of the prelude's sources is not reported
    now = bench.kernel_source_hash("prelude")
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kind=None: now)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    for stamp, expect in (("0" * 16, None), (now, rec["prelude"]["dram_bytes_per_launch"])):
        fake = {"prelude": dict(rec["prelude"], source_hash=stamp)}
        (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(fake))
        assert bench.recorded_traffic("prelude") == expect
