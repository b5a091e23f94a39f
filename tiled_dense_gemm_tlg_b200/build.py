"""Build libtlg.so in-tree with nvcc for sm_100a (B200).

    python tiled_dense_gemm_tlg_b200/build.py [--force]

(Run it as a script: importing the package loads the library this builds.)

The library is plain CUDA C++ behind the C interface in include/tlg.h; it does
not link against torch.  The CUDA runtime is linked statically and the one
driver call it needs (tensor-map encoding) is looked up at run time, so the
library builds on a machine without a GPU or driver.
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libtlg.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-O2", "--expt-relaxed-constexpr",
         "-Xptxas", "-v"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libtlg")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def inputs():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [os.path.join(INCLUDE, "tlg.h"),
                                                                         os.path.abspath(__file__)]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in inputs())


def _compile(src: str, obj: str):
    cmd = [nvcc(), *ARCH, *FLAGS, "-I", INCLUDE, "-I", CSRC, "-Xcompiler", "-fPIC", "-c", "-o", obj, src]
    res = subprocess.run(cmd, capture_output=True, text=True)
    return cmd, res


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every .cu (one translation unit per operand layout, in parallel) and link libtlg.so."""
    if not (force or needs_build()):
        return LIB
    import concurrent.futures

    import shutil
    import tempfile

    obj_dir = tempfile.mkdtemp(prefix="tlg_build_")  # objects are intermediates: not kept in the tree
    srcs = sources()
    objs = [os.path.join(obj_dir, os.path.basename(s)[:-3] + ".o") for s in srcs]
    log_lines = []
    failed = False
    with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        for (cmd, res) in ex.map(_compile, srcs, objs):
            log_lines.append(" ".join(cmd) + "\n" + res.stdout + res.stderr)
            failed = failed or res.returncode != 0
    tmp = LIB + f".tmp{os.getpid()}"
    if not failed:
        cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs]
        res = subprocess.run(cmd, capture_output=True, text=True)
        log_lines.append(" ".join(cmd) + "\n" + res.stdout + res.stderr)
        failed = res.returncode != 0
    shutil.rmtree(obj_dir, ignore_errors=True)
    log = os.path.join(PKG, "_build_log.txt")
    with open(log, "w") as f:
        f.write("\n".join(log_lines))
    if failed:
        sys.stderr.write("\n".join(l for l in log_lines if "error" in l)[-20000:])
        raise RuntimeError(f"nvcc failed; see {log}")
    if verbose:
        sys.stderr.write("\n".join(log_lines))
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
