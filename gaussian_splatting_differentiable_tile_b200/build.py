"""Builds libgs.so (the C-ABI CUDA library) in-tree for sm_100a.

    python -m gaussian_splatting_differentiable_tile_b200.build [--force] [--verbose] [--check]

--check builds libgs_check.so instead: the same sources compiled with
GS_CHECK, whose kernels test every gather and scatter index of the blend,
binning and sort stages and record GS_ERR_BOUNDS in the bins' status word
instead of accessing out of range (the binding loads it when GS_LIBRARY is
libgs_check.so).  GS_EXTRA_NVCC_FLAGS in the environment adds compiler flags
(tuning builds).

Each translation unit under csrc/ is compiled to an object in _build/ (in
parallel), then linked into libgs.so beside this file.  --verbose passes
-Xptxas -v so the register, spill and shared-memory figures of every kernel
are printed.
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libgs.so")
LIB_CHECK = os.path.join(HERE, "libgs_check.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or put the CUDA toolkit on PATH")


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps():
    files = _sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    files.append(os.path.join(INCLUDE, "gs.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _deps())


def build(force: bool = False, verbose: bool = False, check: bool = False) -> str:
    lib = LIB_CHECK if check else LIB
    if not force and not verbose and not os.environ.get("GS_EXTRA_NVCC_FLAGS") and up_to_date(lib):
        return lib
    nvcc = _nvcc()
    build_dir = os.path.join(BUILD, "check") if check else BUILD
    os.makedirs(build_dir, exist_ok=True)
    extra = ["-Xptxas", "-v"] if verbose else []
    if check:
        extra.append("-DGS_CHECK")
    # extra compiler flags, e.g. GS_EXTRA_NVCC_FLAGS="-DGS_ROWS_PER_LANE=2" for
    # a variant of the blend's pixels-per-lane layout
    extra += os.environ.get("GS_EXTRA_NVCC_FLAGS", "").split()

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        cmd = [nvcc, *ARCH, *FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stderr

    with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1)) as ex:
        results = list(ex.map(compile_one, _sources()))
    if verbose:
        for _, log in results:
            sys.stderr.write(log)
    objs = [o for o, _ in results]
    tmp = lib + ".tmp"
    cmd = [nvcc, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, check="--check" in sys.argv))
