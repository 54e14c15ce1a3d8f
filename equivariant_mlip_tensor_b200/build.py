"""Build libcgtp.so (sm_100a) in-tree.

Every per-shape kernel family (conv forward, conv backward, edge-free tensor
product) is compiled once per shape listed in csrc/configs.h, each as its
own translation unit so that the compiles run in parallel; the shape-free
parts (graph, radial network, forces, harmonics, C ABI, host CG tables) are
one unit each.  Objects go to _build/, the library to the package directory.
Objects newer than their sources and headers are reused.
"""
import os
import re
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libcgtp.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
                     "-Xcompiler", "-fPIC", "-I", CSRC, "-I", INCLUDE]
PER_SHAPE = ["conv_fwd.cu", "conv_bwd.cu", "conv_paths.cu", "conv_shared.cu", "tp.cu", "cp.cu"]
SHAPE_FREE = ["graph.cu", "radial.cu", "misc.cu", "abi.cu", "cg_table.cpp", "uvw.cu"]


def cutlass_include():
    """Include directories of a CUTLASS (>= 4) header tree for the tensor-core
    GEMM of the fully connected convolution: $CUTLASS_HOME, else the trees
    vendored in this Python environment's packages.  None if there is none
    (uvw.cu then builds without it and its entry point reports unsupported)."""
    import site
    cands = []
    if os.environ.get("CUTLASS_HOME"):
        cands.append(os.environ["CUTLASS_HOME"])
    for sp in site.getsitepackages():
        cands += [os.path.join(sp, "flashinfer", "data", "cutlass"), os.path.join(sp, "tilelang", "3rdparty", "cutlass")]
    for c in cands:
        inc = os.path.join(c, "include")
        if os.path.exists(os.path.join(inc, "cutlass", "gemm", "collective", "builders", "sm100_9xBF16_umma_builder.inl")):
            util = os.path.join(c, "tools", "util", "include")
            return [inc] + ([util] if os.path.isdir(util) else [])
    return None


def nvcc():
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    return cand


def shapes():
    text = open(os.path.join(CSRC, "configs.h")).read()
    return [tuple(int(v) for v in m) for m in re.findall(r"X\((\d+),\s*(\d+),\s*(\d+)\)", text)]


def _headers():
    return [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))] + \
        [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]


def _stale(obj, src, deps):
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(p) > t for p in [src] + deps)


def _jobs():
    jobs = []
    for src in PER_SHAPE:
        for li, ls, lo in shapes():
            obj = os.path.join(BUILD, f"{src.split('.')[0]}_{li}{ls}{lo}.o")
            defs = [f"-DCGTP_CFG_LI={li}", f"-DCGTP_CFG_LS={ls}", f"-DCGTP_CFG_LO={lo}"]
            jobs.append((os.path.join(CSRC, src), obj, defs))
    for src in SHAPE_FREE:
        obj = os.path.join(BUILD, src.rsplit(".", 1)[0] + ".o")
        defs = []
        if src == "uvw.cu":
            inc = cutlass_include()
            defs = (sum((["-I", d] for d in inc), []) + ["-diag-suppress", "20012,177"]) if inc else ["-DCGTP_NO_CUTLASS"]
        jobs.append((os.path.join(CSRC, src), obj, defs))
    return jobs


def _compile(job, verbose):
    src, obj, defs = job
    cmd = [nvcc()] + NVCC_FLAGS + defs + ["-c", src, "-o", obj]
    if src.endswith(".cpp"):
        cmd = [nvcc(), "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-I", CSRC, "-x", "c++", "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"compile failed: {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    if verbose:
        print("built", os.path.basename(obj), flush=True)
    return obj


def build(verbose=False, jobs=None):
    os.makedirs(BUILD, exist_ok=True)
    deps = _headers()
    todo = [j for j in _jobs() if _stale(j[1], j[0], deps)]
    workers = jobs or max(1, min(len(todo), os.cpu_count() or 4))
    if todo:
        with ThreadPoolExecutor(max_workers=workers) as ex:
            list(ex.map(lambda j: _compile(j, verbose), todo))
    objs = [j[1] for j in _jobs()]
    if todo or not os.path.exists(LIB) or any(os.path.getmtime(o) > os.path.getmtime(LIB) for o in objs):
        tmp = LIB + ".tmp"
        cmd = [nvcc()] + ARCH + ["-shared", "-o", tmp] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed: {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
        if verbose:
            print("linked", LIB, flush=True)
    return LIB


if __name__ == "__main__":
    build(verbose=True)
    sys.exit(0)
