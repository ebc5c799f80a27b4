"""Builds the CUDA library ``libspffn.so`` in-tree for sm_100a (nvcc, no JIT)."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
SO = os.path.join(HERE, "libspffn.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
SOURCES = ["spffn_api.cu", "spffn_kernels.cu", "spffn_fused.cu", "spffn_union.cu", "spffn_ustack.cu",
           "spffn_attn.cu", "spffn_noalloc.cu"]
FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall", "--expt-relaxed-constexpr"]


def _deps():
    out = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh"))]
    out += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return out


def stale():
    if not os.path.exists(SO):
        return True
    t = os.path.getmtime(SO)
    return any(os.path.getmtime(p) > t for p in _deps())


def build(force=False, verbose=False):
    """Compile every source to an object in parallel (one nvcc per file), then link."""
    if not force and not stale():
        return SO
    import concurrent.futures
    import shutil
    import tempfile
    objdir = tempfile.mkdtemp(prefix="spffn_build_")
    try:
        def compile_one(src):
            obj = os.path.join(objdir, src.replace(".cu", ".o"))
            cmd = [NVCC] + FLAGS + (["-Xptxas", "-v"] if verbose else []) + ["-c", os.path.join(CSRC, src), "-o", obj]
            subprocess.check_call(cmd)
            return obj
        with concurrent.futures.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
            objs = list(ex.map(compile_one, SOURCES))
        tmp = SO + ".tmp%d" % os.getpid()
        subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp] + objs + ["-lcuda"])
        os.replace(tmp, SO)
    finally:
        shutil.rmtree(objdir, ignore_errors=True)
    return SO


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv))
