"""Build libpc.so (the CUDA key-switching library) in-tree with nvcc for sm_100a.

    python -m key_switching_b200.build [--force]

Produces key_switching_b200/libpc.so from key_switching_b200/csrc/*.cu (the
kernel file once per ring degree, -DPC_LOGN=10..17, all in parallel).  With
--timeline it builds key_switching_b200/libpc_timeline.so instead: the same
library compiled with -DPC_TIMELINE, whose kernels record the per-CTA timeline
that pc_timeline_read returns (loaded by the binding when PC_TIMELINE=1).  No
GPU is needed to build (nvcc cross-compiles).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libpc.so")
LIB_TIMELINE = os.path.join(HERE, "libpc_timeline.so")
ROOT = os.path.dirname(HERE)

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr",
]


LOGNS = range(10, 18)  # ring degrees 2^10 .. 2^17


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + glob.glob(os.path.join(CSRC, "*.inc"))
    deps.append(os.path.join(ROOT, "include", "pc.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, timeline: bool = False) -> str:
    """Compile every csrc/*.cu to an object (in parallel, one nvcc per file)
    and link them into libpc.so (libpc_timeline.so with timeline=True); a
    no-op when the library is newer than every source."""
    lib = LIB_TIMELINE if timeline else LIB
    if not force and not needs_build(lib):
        return lib
    from concurrent.futures import ThreadPoolExecutor
    objdir = os.path.join(HERE, "_build", "timeline" if timeline else "default")
    extra = ["-DPC_TIMELINE"] if timeline else []
    os.makedirs(objdir, exist_ok=True)
    inc = ["-I", os.path.join(ROOT, "include")]

    def compile_one(src, name, defs):
        obj = os.path.join(objdir, name + ".o")
        cmd = [nvcc(), *NVCC_FLAGS, *extra, *defs, *inc, "-c", "-o", obj, src]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        return obj

    # kernels.cu holds every kernel template; it is compiled once per ring
    # degree (its launchers for degree 2^k live in namespace pc::n<k>)
    jobs = []
    for src in sources():
        if os.path.basename(src) == "kernels.cu":
            jobs += [(src, f"kernels_n{k}", [f"-DPC_LOGN={k}"]) for k in LOGNS]
        else:
            jobs.append((src, os.path.basename(src)[:-3], []))
    with ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 4)) as ex:
        objs = list(ex.map(lambda j: compile_one(*j), jobs))
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", lib + ".tmp", *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, timeline="--timeline" in sys.argv))
