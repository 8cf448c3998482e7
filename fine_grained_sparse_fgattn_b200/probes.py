"""Roofline microbenchmarks for the tile-sparse forward kernels (B200, sm_100a).

Runs the probes of csrc/probes/probes.cu (library libfgattn_probes.so, which
the attention path never loads) and prints one JSON object:

  rows   L2 -> shared-memory row loads with no math, for the three ways the
         forward kernels move a K/V row: 16-row TMA boxes (16-key runs), TMA
         gather4 rows and 16-byte cp.async rows (row-by-row lists).  Buffers of
         one head's K and V at the Wan-480p-like shape (65520 rows x 256 B =
         16.8 MB, L2-resident) and of the whole layer (40 heads, 671 MB, from HBM).
  mma    tcgen05.mma kind::f16 with the key-major kernel's operand layouts,
         M = 128 and N in {64, 128, 256}: the score product alone, the P.V
         product alone, both one group after the other, both interleaved MMA by
         MMA, and the score product split over two accumulators; one commit per
         8-MMA chunk.  Reported as TFLOP/s over the whole GPU and SM clocks per
         MMA.  The last two separate the tensor pipe's throughput from the
         latency of a chain of dependent accumulations.
  ex2    MUFU ex2 results per SM clock per SM.

  python -m fine_grained_sparse_fgattn_b200.probes [--out FILE]
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import sys

import torch

from . import _build

ROWB = 256


def _lib():
    path = _build.build_probes()
    lib = ctypes.CDLL(path)
    p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    fp, dp, up = ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_ulonglong)
    lib.fgprobe_rows.argtypes = [i32, p, i64, i32, i32, p, fp, dp]
    lib.fgprobe_rows.restype = i32
    lib.fgprobe_mma.argtypes = [i32, i32, i32, i32, p, fp, dp, p, up]
    lib.fgprobe_mma.restype = i32
    lib.fgprobe_ex2.argtypes = [i32, i32, p, p, p, fp, dp, dp]
    lib.fgprobe_ex2.restype = i32
    return lib


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def row_loads(lib, rows: int, chunks: int = 4096, reps: int = 5) -> dict:
    buf = torch.randint(0, 255, (rows * ROWB,), dtype=torch.uint8, device="cuda")
    res = {}
    for mode, name in ((0, "tma_box16"), (1, "tma_gather4"), (2, "cp_async16")):
        ms, by = ctypes.c_float(), ctypes.c_double()
        st = lib.fgprobe_rows(mode, ctypes.c_void_p(buf.data_ptr()), rows, chunks, reps, _stream(),
                              ctypes.byref(ms), ctypes.byref(by))
        if st != 0:
            raise RuntimeError(f"fgprobe_rows({name}) failed with status {st}")
        res[name] = {"tb_per_s": by.value / (ms.value * 1e-3) / 1e12, "ms": ms.value, "bytes": by.value}
    del buf
    return res


def mma_rates(lib, chunks: int = 2048, reps: int = 5) -> dict:
    dev = torch.zeros(1, dtype=torch.int64, device="cuda")
    res = {}
    for n in (64, 128, 256):
        for which, name in ((1, "scores"), (2, "pv"), (3, "both"), (4, "both_interleaved"),
                            (5, "scores_two_accumulators")):
            ms, fl, cyc = ctypes.c_float(), ctypes.c_double(), ctypes.c_ulonglong()
            st = lib.fgprobe_mma(which, n, chunks, reps, _stream(), ctypes.byref(ms), ctypes.byref(fl),
                                 ctypes.c_void_p(dev.data_ptr()), ctypes.byref(cyc))
            if st != 0:
                raise RuntimeError(f"fgprobe_mma({name}, N={n}) failed with status {st}")
            mmas = chunks * 8 * (2 if which in (3, 4) else 1)
            res[f"N{n}_{name}"] = {"tflops": fl.value / (ms.value * 1e-3) / 1e12, "ms": ms.value,
                                   "clocks_per_mma": cyc.value / mmas,
                                   "ideal_clocks_per_mma": 2.0 * 128 * n * 16 / 8192.0}
    return res


def ex2_rate(lib, iters: int = 4096) -> dict:
    sink = torch.zeros(256, dtype=torch.float32, device="cuda")
    dev = torch.zeros(2, dtype=torch.int64, device="cuda")
    ms, per, mhz = ctypes.c_float(), ctypes.c_double(), ctypes.c_double()
    st = lib.fgprobe_ex2(iters, 4, _stream(), ctypes.c_void_p(sink.data_ptr()), ctypes.c_void_p(dev.data_ptr()),
                         ctypes.byref(ms), ctypes.byref(per), ctypes.byref(mhz))
    if st != 0:
        raise RuntimeError(f"fgprobe_ex2 failed with status {st}")
    return {"ex2_per_clk_per_sm": per.value, "sm_mhz": mhz.value, "ms": ms.value}


def run() -> dict:
    lib = _lib()
    out = {"device": torch.cuda.get_device_name(), "sms": torch.cuda.get_device_properties(0).multi_processor_count}
    out["rows_one_head_16.8MB"] = row_loads(lib, 65520)
    out["rows_whole_layer_671MB"] = row_loads(lib, 40 * 65520, chunks=2048)
    out["mma"] = mma_rates(lib)
    out["ex2"] = ex2_rate(lib)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=None, help="also write the JSON here")
    a = ap.parse_args(argv)
    res = run()
    s = json.dumps(res, indent=1)
    print(s)
    if a.out:
        os.makedirs(os.path.dirname(os.path.abspath(a.out)), exist_ok=True)
        with open(a.out, "w") as f:
            f.write(s + "\n")
    return 0


if __name__ == "__main__":
    sys.exit(main())
