"""Builds libmla_b200.so (the C-ABI library) from csrc/*.cu for sm_100a.

nvcc -gencode arch=compute_100a,code=sm_100a, static CUDA runtime, position-
independent shared object next to this file. After compiling, the ptxas
resource report is checked for register spills: a kernel that spills fails
the build unless MLA_SKIP_REG_SPILL_CHECK=1 is set (the same safeguard the
FlashMLA build applies, per the deepseek-ai/FlashMLA project page, technical
details).

Usage: python -m head_latent_attention_get_b200.build [-v]
"""
from __future__ import annotations

import os
import re
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB_NAME = "libmla_b200.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _newest_input_mtime() -> float:
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(HERE, "..", "include", "mla.h"))
    files.append(os.path.abspath(__file__))
    return max(os.path.getmtime(f) for f in files if os.path.exists(f))


def up_to_date() -> bool:
    return os.path.exists(LIB_PATH) and os.path.getmtime(LIB_PATH) >= _newest_input_mtime()


def check_spills(ptxas_log: str) -> list:
    bad = []
    func = None
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            func = m.group(1)
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and (int(m.group(1)) or int(m.group(2))):
            bad.append((func, line.strip()))
    return bad


def build(verbose: bool = False, force: bool = False) -> str:
    if not force and up_to_date():
        return LIB_PATH
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xptxas", "-v", "-cudart", "static", "-I", os.path.join(HERE, "..", "include"),
           "-o", LIB_PATH + ".tmp", *sources()]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    log = proc.stdout + proc.stderr
    if proc.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + log)
    spills = check_spills(log)
    if spills and os.environ.get("MLA_SKIP_REG_SPILL_CHECK") != "1":
        os.remove(LIB_PATH + ".tmp")
        raise RuntimeError("register spills (set MLA_SKIP_REG_SPILL_CHECK=1 to allow):\n" +
                           "\n".join(f"{f}: {l}" for f, l in spills))
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    if verbose:
        print(log)
    with open(os.path.join(HERE, "ptxas_report.txt"), "w") as f:
        f.write(log)
    return LIB_PATH


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force=True))
