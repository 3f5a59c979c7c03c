"""Build libbitmoe.so (sm_100a) in-tree from bit_moe_b200/csrc/*.cu.

    python -m bit_moe_b200.build [--force]

Compiles for sm_100a only (-gencode arch=compute_100a,code=sm_100a), with
-lineinfo for profiling and without fast-math (the kernels rely on IEEE
division and explicit rounding intrinsics).
"""
import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OUT = os.path.join(HERE, "libbitmoe.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(out=None):
    out = OUT if out is None else out
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


CHECKED_OUT = os.path.join(HERE, "libbitmoe_checked.so")


def build_checked(force=False, verbose=False):
    """The bounds-checked build (-DMOE_CHECKED): every guarded index that
    falls outside its buffer records MOE_ERR_BOUNDS and the access is skipped.
    The tests load it beside the normal build (no memory checker runs on this
    pool's GPUs)."""
    return build(force=force, verbose=verbose, extra=("-DMOE_CHECKED",), out=CHECKED_OUT)


def build(force=False, verbose=False, extra=(), out=None):
    """Compile every source to an object file (in parallel, one nvcc per
    source) and link them into libbitmoe.so (or `out`)."""
    out = OUT if out is None else out
    if not force and not _stale(out):
        return out
    tag = ".tmp.%d.%d" % (os.getpid(), len(extra))
    flags = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
             "--expt-relaxed-constexpr", *extra]
    srcs = sources()
    objs = [os.path.join(CSRC, os.path.basename(s)[:-3] + tag + ".o") for s in srcs]

    def compile_one(pair):
        src, obj = pair
        cmd = [nvcc_path(), *flags, "-c", "-o", obj, src]
        if verbose:
            print(" ".join(cmd), flush=True)
        return subprocess.run(cmd).returncode

    try:
        with ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
            rcs = list(ex.map(compile_one, zip(srcs, objs)))
        bad = [s for s, rc in zip(srcs, rcs) if rc != 0]
        if bad:
            raise subprocess.CalledProcessError(1, "nvcc " + " ".join(os.path.basename(b) for b in bad))
        tmp = out + tag
        cmd = [nvcc_path(), *ARCH, "-shared", "-o", tmp, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        os.replace(tmp, out)
    finally:
        for o in objs:
            if os.path.exists(o):
                os.remove(o)
    return out


if __name__ == "__main__":
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []
    print(build(force="--force" in sys.argv or bool(extra), verbose=True, extra=extra))
    if "--checked" in sys.argv:
        print(build_checked(force="--force" in sys.argv, verbose=True))
