"""Build libcgtp.so (sm_100a) in-tree.

Every per-shape kernel family (convolution forward, backward, the double
backward's fused passes, edge-free tensor product, CP product) is compiled
once per shape of CGTP_CONFIGS in csrc/configs.h, and the weight-structure
variants (path-shared weights, fully connected convolution) once per shape of
CGTP_VARIANT_CONFIGS, each as its own translation unit so that the compiles
run in parallel; the shape-free parts (graph, radial network, forces,
harmonics, C ABI, host CG tables, tensor-core GEMMs, side streams) are one
unit each.  Objects go to _build/, the library to the package directory.
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
# Line information (for profiler source views) is compiled into the
# shape-free units and the units of the standard workloads' shapes; the
# fully unrolled kernels of the other policy shapes omit it, since their line
# tables would be about 8x their code and the library several hundred MB.
BASE_FLAGS = ARCH + ["-O3", "-std=c++17", "--expt-relaxed-constexpr",
                     "-Xcompiler", "-fPIC", "-I", CSRC, "-I", INCLUDE]
NVCC_FLAGS = BASE_FLAGS + ["-lineinfo"]
# per-shape units: every shape of CGTP_CONFIGS, and the weight-structure
# variants for the shapes of CGTP_VARIANT_CONFIGS
PER_SHAPE = ["conv_fwd.cu", "conv_bwd.cu", "conv_dd.cu", "tp.cu", "cp.cu"]
PER_VARIANT_SHAPE = ["conv_paths.cu", "conv_shared.cu"]
SHAPE_FREE = ["graph.cu", "radial.cu", "misc.cu", "abi.cu", "cg_table.cpp", "uvw.cu", "lanes.cu"]


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


def shapes(macro="CGTP_CONFIGS"):
    """(lmax_in, lmax_sh, lmax_out) entries of one list of csrc/configs.h."""
    text = open(os.path.join(CSRC, "configs.h")).read()
    body = text.split("#define " + macro + "(X)", 1)[1].split("\n\n", 1)[0]
    return [tuple(int(v) for v in m) for m in re.findall(r"X\((\d+),\s*(\d+),\s*(\d+)\)", body)]


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
    for src in SHAPE_FREE:
        obj = os.path.join(BUILD, src.rsplit(".", 1)[0] + ".o")
        defs = []
        if src == "uvw.cu":
            inc = cutlass_include()
            defs = (sum((["-I", d] for d in inc), []) + ["-diag-suppress", "20012,177"]) if inc else ["-DCGTP_NO_CUTLASS"]
        jobs.append((os.path.join(CSRC, src), obj, defs))
    units = [(src, shp) for src in PER_SHAPE for shp in shapes()]
    units += [(src, shp) for src in PER_VARIANT_SHAPE for shp in shapes("CGTP_VARIANT_CONFIGS")]
    # the largest shapes first, so that the long compiles start early
    units.sort(key=lambda u: -(u[1][0] + 1) * (u[1][1] + 1) * (u[1][2] + 1))
    lined = set(shapes("CGTP_VARIANT_CONFIGS"))
    for src, (li, ls, lo) in units:
        obj = os.path.join(BUILD, f"{src.split('.')[0]}_{li}{ls}{lo}.o")
        defs = [f"-DCGTP_CFG_LI={li}", f"-DCGTP_CFG_LS={ls}", f"-DCGTP_CFG_LO={lo}"]
        if (li, ls, lo) not in lined:
            defs.append("--no-lineinfo")
        jobs.append((os.path.join(CSRC, src), obj, defs))
    return jobs


def _compile(job, verbose):
    src, obj, defs = job
    flags = BASE_FLAGS if "--no-lineinfo" in defs else NVCC_FLAGS
    cmd = [nvcc()] + flags + [d for d in defs if d != "--no-lineinfo"] + ["-c", src, "-o", obj]
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
