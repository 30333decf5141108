"""Build libsas.so in-tree with nvcc for sm_100a (B200).

    python -m gated_block_sparse_token_b200.build

The library is a plain C-ABI shared object (include/sas.h); CUDA runtime is
linked statically, the driver's tensor-map encoder is looked up at run time,
so loading the library needs no GPU and no libcuda.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsas.so")
TRACE_LIB = os.path.join(PKG, "libsas_trace.so")  # phase-trace build (-DSAS_PHASE_TRACE)
SOURCES = ["sas_api.cu", "sas_decode.cu", "sas_pool.cu", "sas_prefill.cu", "sas_static.cu", "sas_backward.cu",
           "sas_prefill_backward.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-I" + INCLUDE]


def _stale(lib=LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "sas.h"), __file__]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, trace: bool = False) -> str:
    lib = TRACE_LIB if trace else LIB
    if not force and not _stale(lib):
        return lib
    bdir = os.path.join(ROOT, "_build", "trace" if trace else "release")
    os.makedirs(bdir, exist_ok=True)
    objs, cmds = [], []
    for src in SOURCES:
        obj = os.path.join(bdir, src.replace(".cu", ".o"))
        cmd = [NVCC] + FLAGS + (["-DSAS_PHASE_TRACE"] if trace else []) + ["-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        cmds.append(cmd)
        objs.append(obj)
    # the translation units compile independently: run them side by side
    with ThreadPoolExecutor(max_workers=min(len(cmds), os.cpu_count() or 1)) as ex:
        for r in ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), cmds):
            if verbose or r.returncode != 0:
                sys.stderr.write(r.stdout + r.stderr)
            if r.returncode != 0:
                raise subprocess.CalledProcessError(r.returncode, r.args)
    tmp = lib + ".tmp"
    subprocess.run([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp] + objs
                   + ["-cudart", "static"], check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, trace="--trace" in sys.argv))
