"""Build libforge_attn.so in-tree with nvcc for sm_100a.

    python -m causal_flash_attention_attn_b200.build [--force]

One translation unit (csrc/api.cu includes every kernel header); the shared
library exports the C ABI declared in include/forge_attn.h.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libforge_attn.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-v",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  [os.path.join(INCLUDE, "forge_attn.h")])


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-o", LIB + ".tmp",
           os.path.join(CSRC, "api.cu")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    log = os.path.join(PKG, "build.log")
    with open(log, "w") as f:
        # paths relative to the repository root, so the log reads the same on every machine
        f.write((" ".join(cmd) + "\n" + res.stdout + res.stderr).replace(ROOT + os.sep, ""))
    if res.returncode != 0:
        sys.stderr.write(res.stderr[-20000:])
        raise RuntimeError(f"nvcc failed (see {log})")
    os.replace(LIB + ".tmp", LIB)
    if verbose:
        sys.stdout.write(res.stderr)
    return LIB


def resource_summary(log: str = os.path.join(PKG, "build.log")) -> str:
    """Markdown table of ptxas's per-kernel resource lines in the build log:
    registers a thread, spill stores / loads (bytes), static shared memory."""
    import re
    import shutil
    text = open(log).read()
    rows = []
    for m in re.finditer(r"Compiling entry function '([^']+)'.*?(\d+) bytes stack frame, (\d+) bytes spill stores, "
                         r"(\d+) bytes spill loads\s*\n[^\n]*Used (\d+) registers[^\n]*?(?:(\d+) bytes smem)?\n",
                         text, flags=re.S):
        rows.append(list(m.groups()))
    names = [r[0] for r in rows]
    if shutil.which("c++filt"):
        out = subprocess.run(["c++filt"], input="\n".join(names), capture_output=True, text=True).stdout.split("\n")
        names = [re.sub(r"\(anonymous namespace\)::", "", n) for n in out[:len(names)]]
    lines = ["| kernel | registers | stack B | spill stores B | spill loads B | static smem B |",
             "|---|---:|---:|---:|---:|---:|"]
    for n, r in sorted(zip(names, rows)):
        lines.append(f"| `{n}` | {r[4]} | {r[1]} | {r[2]} | {r[3]} | {r[5] or 0} |")
    return "\n".join(lines) + "\n"


if __name__ == "__main__":
    if "--resources" in sys.argv:
        sys.stdout.write(resource_summary())
    else:
        print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
