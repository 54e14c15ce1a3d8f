"""bench.py's host-side contract without a GPU: the reference arm's JSON line
(the oracle timed on the host), the algorithmic byte counts against the sizes
of the arrays one launch must touch, and the measured-traffic record that
stays valid only for the kernel sources it was captured on."""
import json
import os
import shutil
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] >= 3
    assert d["metric"] == bench.METRIC and d["unit"] == "edges/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "edges/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in d["config"]


def test_conv_bytes_are_the_arrays_a_launch_touches():
    n, E, P, u, ni, ns, no = 7, 40, 19, 128, 9, 25, 9
    fwd, bwd = bench.conv_bytes(n, E, P, u, ni, ns, no)
    f32 = 4
    # forward: W, x, out, edge vectors, col, row_ptr
    W, x, out = E * P * u, n * ni * u, n * no * u
    assert fwd == f32 * (W + x + out + 3 * E + E + (n + 1))
    # backward: W read and grad_W written, x read and grad_x written, grad_out
    # read, edge vectors read and their gradients written, the CSC edge and
    # destination lists, and both offset arrays; no workspace partials
    assert bwd == f32 * (2 * W + 2 * x + out + 3 * E + 3 * E + 2 * E + 2 * (n + 1))
    assert bench.partials_bytes(E, ns, 4) == f32 * 2 * 4 * E * ns


def test_measured_traffic_tracks_the_sources(tmp_path, monkeypatch):
    import hashlib
    rec = dict(bench.MEASURED_TRAFFIC["conv_bwd"])
    # a record taken on the current sources scales with the edge count
    m = hashlib.sha256()
    for name in rec["sources"]:
        with open(os.path.join(ROOT, "equivariant_mlip_tensor_b200", "csrc", name), "rb") as f:
            m.update(f.read())
    rec["sha256_16"] = m.hexdigest()[:16]
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, "conv_bwd", rec)
    assert bench.measured_traffic("conv_bwd", rec["n_edges"]) == rec["bytes"]
    assert bench.measured_traffic("conv_bwd", 2 * rec["n_edges"]) == 2 * rec["bytes"]
    assert bench.measured_traffic("no_such_kernel", 10) is None
    # a copy of the sources with one kernel file changed no longer matches
    src = os.path.join(ROOT, "equivariant_mlip_tensor_b200", "csrc")
    dst = tmp_path / "equivariant_mlip_tensor_b200" / "csrc"
    shutil.copytree(src, dst)
    with open(dst / "conv_bwd_kernel.cuh", "a") as f:
        f.write("\n// changed\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("conv_bwd", rec["n_edges"]) is None
