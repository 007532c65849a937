"""Builds libsparseattn.so in-tree from csrc/*.cu for sm_100a with nvcc.

    python -m block_sparse_approximate_b200.build [--force] [-v]

Each .cu file is compiled to an object under _build/ (skipped when the object
is newer than every source and header), then linked into
block_sparse_approximate_b200/libsparseattn.so.  nvcc cross-compiles, so this
runs on a machine without a GPU.
"""

from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsparseattn.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", INCLUDE]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h")))


# attn_tc_kernel and attn_tc_linmix_kernel reallocate registers with
# setmaxnreg: their launch register count times 384 threads must cover the
# split (256 x 216 + 128 x 40, and 128 x 216 + 128 x 96 + 128 x 56; see
# attn_tc.cu), or setmaxnreg.inc would wait for registers that never come.
TC_MIN_LAUNCH_REGS = 158


def _check_tc_registers(ptxas_log: str):
    import re
    lines = ptxas_log.splitlines()
    for k, line in enumerate(lines):
        if "Compiling entry function" in line and ("attn_tc_kernel" in line or "attn_tc_linmix_kernel" in line):
            for nxt in lines[k + 1:k + 4]:
                m = re.search(r"Used (\d+) registers", nxt)
                if m:
                    regs = int(m.group(1))
                    if regs < TC_MIN_LAUNCH_REGS:
                        raise RuntimeError(f"attn_tc_kernel launches with {regs} registers per thread; "
                                           f"the setmaxnreg split needs >= {TC_MIN_LAUNCH_REGS}")
                    break


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    os.makedirs(BUILD, exist_ok=True)
    headers = _headers()
    objs, jobs = [], []
    for src in _sources():
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or _stale(obj, [src] + headers):
            extra = list(extra_flags)
            if os.path.basename(src) == "attn_tc.cu" and "-v" not in extra:
                extra += ["-Xptxas", "-v"]
            cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
            jobs.append(cmd)

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, r

    with ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        for cmd, r in ex.map(run, jobs):
            if verbose and (r.stdout or r.stderr):
                print(r.stdout + r.stderr, flush=True)
            if r.returncode != 0:
                raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
            if cmd[-3].endswith("attn_tc.cu"):
                _check_tc_registers(r.stdout + r.stderr)
    if force or jobs or _stale(LIB, objs):
        cmd = [NVCC, *ARCH, "-shared", "-o", LIB, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    return LIB


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / spills per kernel")
    a = ap.parse_args(argv)
    extra = ["-Xptxas", "-v"] if a.ptxas_info else []
    print(build(force=a.force or a.ptxas_info, verbose=a.verbose or a.ptxas_info, extra_flags=extra))


if __name__ == "__main__":
    sys.exit(main())
