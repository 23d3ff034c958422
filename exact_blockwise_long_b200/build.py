"""Build libringattn.so in-tree with nvcc for sm_100a.

    python -m exact_blockwise_long_b200.build [--force] [--checked]

Each .cu under csrc/ is compiled to an object under _build/ (in parallel),
then linked into exact_blockwise_long_b200/libringattn.so.  A rebuild happens
when the library is missing or older than any source or header.

--checked builds libringattn_checked.so instead (objects under
_build/checked/): the same sources with -DRA_CHECKED, whose kernels check
every tile and row index against its tensor before the access and latch
RA_ERR_BOUNDS in the device status word instead of making it.
"""

from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import re
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libringattn.so")
LIB_CHECKED = os.path.join(PKG, "libringattn_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
                "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
                "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


# Kernels whose warp roles re-split the launch's registers (setmaxnreg): the
# split is sized for this many registers per thread at launch, so a compile
# that lands on another count is a build error (the library also refuses to
# launch such a kernel at run time).
LAUNCH_REGS = {"fwd_tc.cu": {"fwd_tc2_kernel": 168}, "bwd_tc.cu": {"bwd_fused_kernel": 128}}


def kernel_registers(ptxas_log: str) -> dict:
    """{mangled entry name: registers} from `ptxas -v` output."""
    regs, cur = {}, None
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            cur = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and cur:
            regs[cur] = int(m.group(1))
            cur = None
    return regs


def check_launch_registers(src: str, ptxas_log: str) -> None:
    want = LAUNCH_REGS.get(os.path.basename(src), {})
    regs = kernel_registers(ptxas_log)
    for kernel, n in want.items():
        found = {name: r for name, r in regs.items() if kernel in name}
        if not found:
            raise RuntimeError(f"{src}: ptxas reported no registers for {kernel}")
        bad = {name: r for name, r in found.items() if r != n}
        if bad:
            raise RuntimeError(f"{src}: {kernel} compiled to {sorted(set(bad.values()))} registers per thread; "
                               f"its register split needs exactly {n}")


def _compile(src: str, extra, out_dir: str = BUILD) -> str:
    obj = os.path.join(out_dir, os.path.basename(src)[:-3] + ".o")
    checked = os.path.basename(src) in LAUNCH_REGS
    flags = list(extra) + (["-Xptxas", "-v"] if checked and "-v" not in extra else [])
    cmd = [nvcc()] + FLAGS + flags + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if checked:
        check_launch_registers(src, r.stdout + r.stderr)
    if r.stderr.strip() and (not checked or "-v" in extra):
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, verbose_ptxas: bool = False, checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    out_dir = os.path.join(BUILD, "checked") if checked else BUILD
    if not force and not needs_build(lib):
        return lib
    os.makedirs(out_dir, exist_ok=True)
    extra = (["-Xptxas", "-v"] if verbose_ptxas else []) + (["-DRA_CHECKED"] if checked else [])
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, out_dir), _sources()))
    tmp = lib + ".tmp"
    cmd = [nvcc()] + ARCH + ["-shared", "-o", tmp] + objs + ["-lcudart_static", "-lrt", "-ldl", "-lpthread"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print register/smem usage per kernel")
    ap.add_argument("--checked", action="store_true", help="build the bounds-checked library (-DRA_CHECKED)")
    a = ap.parse_args()
    print(build(force=a.force or a.ptxas_v, verbose_ptxas=a.ptxas_v, checked=a.checked))


if __name__ == "__main__":
    main()
