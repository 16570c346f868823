"""Build ``libbsgemm.so`` in-tree for sm_100a with nvcc.

The C ABI unit (``csrc/bsgemm_api.cu``), the allocation-free entry point
(``csrc/bsgemm_noalloc.cu``), the quantiser (``csrc/bsgemm_quant.cu``) and
one kernel-instance unit per
(granularity, layout) pair (``csrc/bsgemm_inst.cu`` compiled twelve times with
-DBSG_GRAN / -DBSG_LAYOUT) are compiled in parallel and linked into one shared
library next to this file.  Objects are rebuilt only when a source under
``csrc/`` or ``include/`` is newer than they are.

    python -m fp8_block_scaled_bsgemm_b200.build [--force] [-j N]
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libbsgemm.so")

GRANS = (64, 128, 256)
LAYOUTS = ("nt", "tn", "nn", "tt")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-v",
         "-I" + INCLUDE, "-I" + CSRC]


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libbsgemm.so")
    return exe


def _newest_source() -> float:
    files = glob.glob(os.path.join(CSRC, "*")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return max(os.path.getmtime(f) for f in files)


def _compile(src: str, obj: str, defines: list[str]) -> str:
    cmd = [nvcc()] + ARCH + FLAGS + defines + ["-c", src, "-o", obj + ".tmp"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    log = obj + ".log"
    with open(log, "w") as f:
        f.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {os.path.basename(obj)}:\n{r.stderr[-4000:]}")
    os.replace(obj + ".tmp", obj)
    return obj


def build(force: bool = False, jobs: int | None = None, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    newest = _newest_source()
    units = [(os.path.join(CSRC, "bsgemm_api.cu"), os.path.join(BUILD, "bsgemm_api.o"), []),
             (os.path.join(CSRC, "bsgemm_noalloc.cu"), os.path.join(BUILD, "bsgemm_noalloc.o"), []),
             (os.path.join(CSRC, "bsgemm_quant.cu"), os.path.join(BUILD, "bsgemm_quant.o"), [])]
    for g in GRANS:
        for lay in LAYOUTS:
            units.append((os.path.join(CSRC, "bsgemm_inst.cu"),
                          os.path.join(BUILD, f"bsgemm_inst_g{g}_{lay}.o"),
                          [f"-DBSG_GRAN={g}", f"-DBSG_LAYOUT={lay}"]))
    todo = [u for u in units if force or not os.path.exists(u[1]) or os.path.getmtime(u[1]) < newest]
    if todo:
        jobs = jobs or max(1, min(len(todo), os.cpu_count() or 1))
        with cf.ThreadPoolExecutor(jobs) as ex:
            for obj in ex.map(lambda u: _compile(*u), todo):
                if verbose:
                    print("built", os.path.basename(obj), flush=True)
    objs = [u[1] for u in units]
    if force or todo or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(map(os.path.getmtime, objs)):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [nvcc()] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-o", tmp] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n" + r.stderr[-4000:])
        os.replace(tmp, LIB)
    return LIB


def ptxas_report() -> str:
    """Registers / spills / shared memory per kernel, from the last build logs."""
    lines = []
    for log in sorted(glob.glob(os.path.join(BUILD, "*.log"))):
        cur = None
        for ln in open(log):
            if "Compiling entry function" in ln:
                cur = ln.split("'")[1]
            elif cur and ("Used" in ln or "spill" in ln):
                lines.append(f"{os.path.basename(log)[:-6]} {cur}: {ln.strip()}")
    return "\n".join(lines)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-j", type=int, default=None)
    ap.add_argument("--report", action="store_true", help="print ptxas register/spill lines")
    a = ap.parse_args(argv)
    print(build(a.force, a.j, verbose=True))
    if a.report:
        print(ptxas_report())


if __name__ == "__main__":
    sys.exit(main())
