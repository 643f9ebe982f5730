"""Build libfp8bs.so in-tree with nvcc for sm_100a.

    python -m fp8_block_scaled_a8w8_b200.build [--force] [--verbose-ptxas]

Objects go to fp8_block_scaled_a8w8_b200/_build/, the library to
fp8_block_scaled_a8w8_b200/libfp8bs.so. A source is recompiled when it or any
header is newer than its object. The CUDA runtime is linked statically and
only the fp8bs_* symbols are exported.
"""

from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import re
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libfp8bs.so")
INCLUDE = os.path.join(ROOT, "include")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

SOURCES = ["api.cu", "dispatch.cpp", "quant.cu", "gemv.cu", "gemv_tma.cu", "gemv_umma.cu", "gemm_tc.cu", "gemm_fp8.cu", "gemm_mx.cu", "tma_host.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC]


def _headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh", ".inc"))]
    hs.append(os.path.join(INCLUDE, "fp8bs.h"))
    return hs


# Kernels that move registers between warpgroups with setmaxnreg: the split is only valid if
# ptxas gives every thread exactly this many registers at launch (otherwise setmaxnreg.inc
# would wait for registers that do not exist), so the build checks it.
REGISTER_CONTRACTS = {"gemm_tc.cu": ("gemm_tc_kernel", 168), "gemm_fp8.cu": ("gemm_fp8_kernel", 96)}

# Hot kernels that must compile without register spills (mangled-name patterns): the
# decode kernels, the one-split tensor-core kernel and the mma.sync decode kernel with
# staged scales. The split-K tensor-core instantiations and rare fallbacks may spill a few
# bytes and are not listed.
SPILL_FREE = {"gemv_umma.cu": [r"gemv_umma_kernel"], "gemm_tc.cu": [r"gemm_tc_kernel.*Lb0EEEv"],
              "gemv_tma.cu": [r"gemv_tma_kernel.*Lb1EEEv"], "gemm_fp8.cu": [r"gemm_fp8_kernel.*Lb0EEEv"], "gemm_mx.cu": [r"gemm_mx_kernel"]}


def _check_spill_free(src: str, log: str) -> None:
    pats = [re.compile(p) for p in SPILL_FREE.get(src, [])]
    if not pats:
        return
    lines = log.splitlines()
    seen = 0
    for i, line in enumerate(lines):
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if not m or not any(p.search(m.group(1)) for p in pats):
            continue
        for nxt in lines[i + 1:i + 6]:
            sm = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", nxt)
            if sm:
                seen += 1
                if int(sm.group(1)) or int(sm.group(2)):
                    raise RuntimeError(f"{src}: {m.group(1)} spills ({nxt.strip()})")
                break
    if seen == 0:
        raise RuntimeError(f"{src}: no ptxas spill report for {SPILL_FREE[src]}")


def _check_register_contract(src: str, log: str) -> None:
    if src not in REGISTER_CONTRACTS:
        return
    needle, regs = REGISTER_CONTRACTS[src]
    lines = log.splitlines()
    seen = 0
    for i, line in enumerate(lines):
        if "Compiling entry function" in line and needle in line:
            for nxt in lines[i + 1:i + 6]:
                m = re.search(r"Used (\d+) registers", nxt)
                if m:
                    seen += 1
                    if int(m.group(1)) != regs:
                        raise RuntimeError(f"{src}: {line.strip()} uses {m.group(1)} registers, the setmaxnreg split "
                                           f"needs exactly {regs}")
                    break
    if seen == 0:
        raise RuntimeError(f"{src}: no ptxas register report for {needle}")


def _compile(src: str, force: bool, ptxas_verbose: bool) -> tuple[str, str]:
    path = os.path.join(CSRC, src)
    obj = os.path.join(BUILD, src + ".o")
    newest = max(os.path.getmtime(h) for h in _headers() + [path])
    if not force and os.path.exists(obj) and os.path.getmtime(obj) >= newest:
        return obj, ""
    cmd = [NVCC, *ARCH, *COMMON, "-c", path, "-o", obj]
    if src.endswith(".cpp"):
        cmd[1:1] = ["-x", "cu"]
    if (ptxas_verbose and src.endswith(".cu")) or src in REGISTER_CONTRACTS or src in SPILL_FREE:
        cmd.append("-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    try:
        _check_register_contract(src, r.stderr)
        _check_spill_free(src, r.stderr)
    except RuntimeError:
        os.remove(obj)
        raise
    return obj, r.stderr if ptxas_verbose else ""


def build(force: bool = False, ptxas_verbose: bool = False, quiet: bool = True) -> str:
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        futs = [ex.submit(_compile, s, force, ptxas_verbose) for s in SOURCES]
        results = [f.result() for f in futs]
    objs = [o for o, _ in results]
    if ptxas_verbose:
        for _, log in results:
            if log:
                print(log, file=sys.stderr)
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs):
        tmp = LIB + ".tmp"
        cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-Xlinker", "--exclude-libs,ALL"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
    if not quiet:
        print(LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    a = ap.parse_args()
    build(force=a.force, ptxas_verbose=a.verbose_ptxas, quiet=False)
