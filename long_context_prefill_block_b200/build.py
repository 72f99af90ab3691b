"""Build libmoba.so in-tree: every csrc/*.cu compiled by nvcc for sm_100a.

    python -m long_context_prefill_block_b200.build [--force] [--trace | --checked]

--trace builds libmoba_trace.so instead: the same sources with MOBA_TRACE
defined, which adds the phase-trace entry points of include/moba_trace.h
(a measuring aid; the ordinary library carries none of it).
--checked builds libmoba_checked.so: the same sources with MOBA_CHECKED
defined, whose device index and bounds checks record MOBA_ERR_CHECK in the
status word and skip the access instead of trapping (a debugging aid).
"""
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libmoba.so")
OBJ_TRACE = os.path.join(HERE, "_build_trace")
LIB_TRACE = os.path.join(HERE, "libmoba_trace.so")
OBJ_CHECKED = os.path.join(HERE, "_build_checked")
LIB_CHECKED = os.path.join(HERE, "libmoba_checked.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-I", CSRC]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


def _compile(src, force, extra, objdir=OBJ):
    obj = os.path.join(objdir, os.path.basename(src) + ".o")
    newest = max([os.path.getmtime(src)] + [os.path.getmtime(h) for h in _headers()])
    if not force and os.path.exists(obj) and os.path.getmtime(obj) >= newest:
        return obj, False
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
    if "-Xptxas" in extra and r.stderr:
        sys.stderr.write(r.stderr)
    return obj, True


def build(force: bool = False, verbose_ptxas: bool = False, trace: bool = False,
          checked: bool = False) -> str:
    objdir, lib = ((OBJ_TRACE, LIB_TRACE) if trace else
                   (OBJ_CHECKED, LIB_CHECKED) if checked else (OBJ, LIB))
    os.makedirs(objdir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    if trace:
        extra = extra + ["-DMOBA_TRACE"]
    if checked:
        extra = extra + ["-DMOBA_CHECKED"]
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(lambda s: _compile(s, force, extra, objdir), srcs))
    objs = [o for o, _ in results]
    changed = any(c for _, c in results)
    if changed or force or not os.path.exists(lib):
        cmd = [NVCC, *ARCH, "-shared", "-o", lib, *objs, "-Xcompiler", "-fPIC"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode:
            raise RuntimeError(f"link failed:\n{r.stderr}")
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--ptxas" in sys.argv,
                trace="--trace" in sys.argv, checked="--checked" in sys.argv))
