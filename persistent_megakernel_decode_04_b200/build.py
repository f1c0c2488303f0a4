"""Build libmk.so (the C-ABI library) in place with nvcc for sm_100a.

Usage: python -m persistent_megakernel_decode_04_b200.build [--force]
The ptxas resource report (-Xptxas -v: registers, spills, shared memory per kernel)
is written next to the library as libmk.ptxas.txt.
"""
from __future__ import annotations

import glob
import time
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SO = os.path.join(HERE, "libmk.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _stale() -> bool:
    if not os.path.exists(SO):
        return True
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        [os.path.join(ROOT, "include", "mk.h")]
    so_t = os.path.getmtime(SO)
    return any(os.path.getmtime(d) > so_t for d in deps)


def build(force: bool = False, verbose: bool = False, csrc: str | None = None, out: str | None = None,
          defines=()) -> str:
    """Compile every .cu/.cpp of `csrc` (default: this package's csrc/) into `out`
    (default: libmk.so next to this file).  `defines`: extra -D macros."""
    so = out or SO
    if not force and out is None and not _stale():
        return SO
    src_dir = csrc or CSRC
    objdir = os.path.join(os.path.dirname(so), "_build")
    os.makedirs(objdir, exist_ok=True)
    objs, report = [], []
    t_start = time.time()  # sources edited while this build runs must leave the library stale
    common = ["-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"), "-I", src_dir]
    common += [f"-D{d}" for d in defines]
    srcs = sorted(glob.glob(os.path.join(src_dir, "*.cu")) + glob.glob(os.path.join(src_dir, "*.cpp")))
    for src in srcs:
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [NVCC, *ARCH, *common, "-lineinfo", "-c", src, "-o", obj]
        if src.endswith(".cu"):
            cmd += ["-Xptxas", "-v"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        report.append(f"== {os.path.basename(src)}\n{r.stderr}")
        if r.returncode != 0:
            sys.stderr.write(r.stderr)
            raise RuntimeError(f"nvcc failed on {src}")
        objs.append(obj)
    tmp = so + ".tmp"
    subprocess.check_call([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static", "-ldl", "-lrt", "-lpthread"])
    os.replace(tmp, so)
    os.utime(so, (t_start, t_start))
    with open(os.path.join(os.path.dirname(so), "libmk.ptxas.txt"), "w") as f:
        f.write("\n".join(report))
    if verbose:
        print("\n".join(report))
    return so


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
