"""The backward's compile-time chunk plans (CPU): a host-only probe built with
nvcc prints the plans of several shapes, and these checks pin what the
kernels rely on:
  - every path is in exactly one chunk;
  - a chunk's paths belong to its keys key..key_hi, and each key is covered by
    consecutive chunks;
  - the first chunk covering a key starts its rows (first_of_key), every later
    one continues them, follows its predecessor directly and shares its chain
    (lane), and a chain is a run of consecutive chunks;
  - a chunk's estimated instructions stay within the budget unless it holds a
    single path;
  - a key's paths after the first chunk that holds some of them are the same
    key (no block is split across chains)."""
import json
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "equivariant_mlip_tensor_b200", "csrc")


def _nvcc():
    return os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"


@pytest.fixture(scope="module")
def plans():
    nvcc = _nvcc()
    if not os.path.exists(nvcc) and shutil.which(nvcc) is None:
        pytest.skip("nvcc not available")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "plan_probe")
        cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O1", "-std=c++17", "--expt-relaxed-constexpr",
               "-I", CSRC, "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "plan_probe.cu"),
               "-o", exe]
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr[-3000:]
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    return [json.loads(line) for line in out.splitlines() if line.strip()]


def test_every_path_in_exactly_one_chunk(plans):
    for pl in plans:
        paths = [tuple(p[:3]) for c in pl["chunks"] for p in c["paths"]]
        assert len(paths) == pl["n_paths"] == len(set(paths)), pl


def test_chunks_cover_their_keys_in_order(plans):
    for pl in plans:
        prev_hi = -1
        for c in pl["chunks"]:
            keys = [p[0] for p in c["paths"]]
            assert c["key"] == min(keys) and c["key_hi"] == max(keys), c
            assert c["key"] >= prev_hi, pl  # keys never go back
            prev_hi = c["key_hi"]


def test_continuations_follow_their_predecessor_on_its_chain(plans):
    for pl in plans:
        ch = pl["chunks"]
        for i, c in enumerate(ch):
            if i == 0:
                assert c["first_of_key"] and c["chain"] == 0
                continue
            if c["first_of_key"]:
                assert c["key"] > ch[i - 1]["key_hi"] and c["chain"] == ch[i - 1]["chain"] + 1, pl
            else:
                # continues the rows its predecessor started or continued
                assert c["key"] == c["key_hi"] == ch[i - 1]["key_hi"] and c["chain"] == ch[i - 1]["chain"], pl
        assert pl["chains"] == ch[-1]["chain"] + 1


def test_chunks_within_budget(plans):
    for pl in plans:
        for c in pl["chunks"]:
            cost = sum(p[3] for p in c["paths"])
            assert cost <= pl["budget"] or len(c["paths"]) == 1, (pl["shape"], pl["variant"], c)


def test_known_plans(plans):
    by = {(tuple(p["shape"]), p["variant"]): p for p in plans}
    # the molecules shape: l1 = 0 and 1 merged in one launch, l1 = 2 in two on their own lane
    mol = by[((2, 4, 2), "backward")]
    assert [(c["key"], c["key_hi"], len(c["paths"])) for c in mol["chunks"]] == [(0, 1, 10), (2, 2, 7), (2, 2, 2)]
    assert mol["chains"] == 2
    # its fused double-backward pass: the l1 = 1 block's last chunk rides with the l1 = 0 block
    dd = by[((2, 4, 2), "double_backward")]
    assert len(dd["chunks"]) == 5 and dd["chunks"][0]["key_hi"] == 1 and dd["chains"] == 2
