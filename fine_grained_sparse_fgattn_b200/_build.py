"""Build libfgattn.so in-tree with nvcc for sm_100a (B200)."""
from __future__ import annotations

import hashlib
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfgattn.so")
STAMP = LIB + ".srchash"
# Microbenchmarks of the rooflines (row loads from L2, tcgen05 issue rate, MUFU):
# a separate library; the attention path never loads it.
PROBES_SRC = os.path.join(CSRC, "probes", "probes.cu")
PROBES_LIB = os.path.join(PKG, "libfgattn_probes.so")


def _sources():
    files = [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cu", ".cuh"))]
    files.append(os.path.join(INCLUDE, "fgattn.h"))
    return files


def source_hash() -> str:
    h = hashlib.sha256()
    for f in _sources():
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _code_only(text: bytes) -> bytes:
    """Source text without comments and trailing blanks: an edit to a comment does not
    change the compiled kernel, so it does not change the kernel's hash."""
    import re
    t = text.decode()
    t = re.sub(r"/\*.*?\*/", "", t, flags=re.S)
    t = re.sub(r"//[^\n]*", "", t)
    return "\n".join(line.rstrip() for line in t.splitlines() if line.strip()).encode()


def kernel_hash(kernel: str) -> str:
    """Hash of the code (comments removed) of the sources one kernel is built from
    (ties a profile to a kernel version)."""
    files = {"fwd": ["attention_fwd.cuh", "mask_row.cuh", "sm100_ptx.cuh"],
             "fwd_qm": ["attention_fwd.cuh", "attention_fwd_qm.cuh", "mask_row.cuh", "sm100_ptx.cuh"],
             "compact": ["compact_mask.cuh"],
             "bwd": ["attention_fwd.cuh", "attention_bwd.cuh", "mask_row.cuh", "sm100_ptx.cuh"]}[kernel]
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(_code_only(fh.read()))
    return h.hexdigest()[:16]


def is_current() -> bool:
    if not os.path.exists(LIB) or not os.path.exists(STAMP):
        return False
    with open(STAMP) as f:
        return f.read().strip() == source_hash()


def nvcc_path() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found; cannot build libfgattn.so")
    return p


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and is_current():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, os.path.join(CSRC, "fgattn.cu"), "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(source_hash())
    return LIB


def _probe_deps():
    return [PROBES_SRC] + [os.path.join(CSRC, f) for f in ("attention_fwd.cuh", "sm100_ptx.cuh")]


def build_probes(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(PROBES_LIB) and \
            os.path.getmtime(PROBES_LIB) >= max(os.path.getmtime(f) for f in _probe_deps()):
        return PROBES_LIB
    tmp = PROBES_LIB + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, PROBES_SRC, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, PROBES_LIB)
    return PROBES_LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True))
    print(build_probes(force=True))
