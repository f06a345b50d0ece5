"""Build libpa.so in-tree with nvcc for sm_100a (B200).

    python -m paged_kv_attention_token_b200.build [--verbose-ptxas]

Objects go to paged_kv_attention_token_b200/_build/, the library to
paged_kv_attention_token_b200/libpa.so.  Sources are rebuilt when they, or any
header under csrc/ or include/, are newer than their object.
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
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libpa.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
              "-I" + os.path.join(ROOT, "include"), "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))


def _stale(obj: str, src: str, newest_header: float) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return t < os.path.getmtime(src) or t < newest_header


# Kernels that move registers between warpgroups with setmaxnreg: a split
# whose sum exceeds what the CTA was launched with would wait forever, so the
# register count ptxas gives the kernel is checked against the split the
# source assumes before the library is linked.
REG_SPLIT_SOURCES = {"prefill.cu": {"prefill_kernel": "PrefillCfg", "prefill_pair_kernel": "PairCfg"}}


def check_register_split(src: str, ptxas_log: str) -> None:
    text = open(src).read()
    for kernel, cfg in REG_SPLIT_SOURCES[os.path.basename(src)].items():
        # the kernel's constants, from the body of its configuration struct
        m = re.search(rf"struct {cfg} {{(.*?)\n}};", text, re.S)
        if not m:
            raise RuntimeError(f"{os.path.basename(src)}: no struct {cfg}")
        body = m.group(1)
        want = {k: int(re.search(rf"{k} = (\d+);", body).group(1))
                for k in ("kThreads", "kLaunchRegs", "kRegsLow", "kRegsHigh")}
        hits = re.findall(rf"Compiling entry function '([^']*\d{kernel}[IE][^']*)'.*?Used (\d+) registers", ptxas_log, re.S)
        if not hits:
            raise RuntimeError(f"{os.path.basename(src)}: no ptxas register report for {kernel}")
        threads = want["kThreads"]
        for name, regs in hits:
            regs = int(regs)
            low_threads = 128
            need = low_threads * want["kRegsLow"] + (threads - low_threads) * want["kRegsHigh"]
            if regs != want["kLaunchRegs"] or need > threads * regs:
                raise RuntimeError(f"{name}: ptxas gives {regs} registers per thread at launch; the source assumes "
                                   f"{want['kLaunchRegs']} and a split needing {need} of {threads * regs}")


def build(force: bool = False, verbose_ptxas: bool = False, quiet: bool = True) -> str:
    os.makedirs(BUILD, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))
    hdr = max([os.path.getmtime(h) for h in _headers()] + [0.0])
    cc = nvcc()
    jobs = []
    objs = []
    for src in sources:
        obj = os.path.join(BUILD, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or _stale(obj, src, hdr):
            cmd = [cc, *ARCH, *NVCC_FLAGS, "-c", src, "-o", obj]
            if (verbose_ptxas and src.endswith(".cu")) or os.path.basename(src) in REG_SPLIT_SOURCES:
                cmd.insert(1, "-Xptxas=-v")
            jobs.append((src, cmd))

    def run(job):
        src, cmd = job
        r = subprocess.run(cmd, capture_output=True, text=True)
        return src, cmd, r

    failed = False
    with cf.ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        for src, cmd, r in ex.map(run, jobs):
            if r.returncode == 0 and os.path.basename(src) in REG_SPLIT_SOURCES:
                try:
                    check_register_split(src, r.stderr)
                except RuntimeError as e:
                    os.remove(os.path.join(BUILD, os.path.basename(src) + ".o"))
                    failed = True
                    sys.stderr.write(f"[build] FAILED register check: {e}\n")
                    continue
            if r.returncode != 0:
                failed = True
                sys.stderr.write(f"[build] FAILED {os.path.basename(src)}\n{' '.join(cmd)}\n{r.stdout}{r.stderr}\n")
            elif not quiet or verbose_ptxas:
                sys.stderr.write(f"[build] {os.path.basename(src)}\n{r.stderr}")
    if failed:
        raise RuntimeError("libpa build failed")
    if jobs or not os.path.exists(LIB):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [cc, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static", "-lrt", "-ldl", "-lpthread"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{' '.join(cmd)}\n{r.stdout}{r.stderr}")
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas, quiet=False))
