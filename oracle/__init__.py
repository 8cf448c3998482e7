"""Python handle on the plain CPU oracle (oracle/fgattn_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the tests, by the package's smoke check
and by the benchmark's CPU-baseline leg, never by the product path.

The oracle evaluates tile-sparse softmax attention by its definition in double
precision ("FG-Attn: Leveraging Fine-Grained Sparse Attention in Video
Diffusion Models", Abstract: skipped M x N score tiles count as -inf), and the
gradients of that definition with respect to q, k and v (backward).
Parity of every function here is pinned by tests/test_oracle.py against
library routines (torch float64 softmax), brute force and closed forms.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "fgattn_oracle.c")


def lib_path(mutant: int = 0) -> str:
    name = "liboracle.so" if mutant == 0 else f"liboracle_mutant{mutant}.so"
    return os.path.join(_HERE, "_build", name)


def build(mutant: int = 0, force: bool = False) -> str:
    """Compile the oracle with the host C compiler (gcc/cc); returns the .so path."""
    out = lib_path(mutant)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(SRC):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    cc = os.environ.get("CC", "gcc")
    tmp = out + f".tmp{os.getpid()}"
    cmd = [cc, "-O2", "-std=c99", "-shared", "-fPIC", "-pthread", f"-DORACLE_MUTANT={mutant}",
           SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


class Oracle:
    def __init__(self, mutant: int = 0):
        self.mutant = mutant
        self._lib = ctypes.CDLL(build(mutant))
        i64, p = ctypes.c_int64, ctypes.c_void_p
        self._lib.oracle_compact.argtypes = [p, i64, i64, i64, i64, i64, p, p, i64]
        self._lib.oracle_compact.restype = ctypes.c_int
        self._lib.oracle_attention.argtypes = [p, p, p, p, i64, i64, i64, i64, i64, i64,
                                               ctypes.c_double, p, i64, p, p, ctypes.c_int]
        self._lib.oracle_attention.restype = ctypes.c_int
        self._lib.oracle_attention_backward.argtypes = [p, p, p, p, p, i64, i64, i64, i64, i64, i64,
                                                        ctypes.c_double, p, p, p, ctypes.c_int]
        self._lib.oracle_attention_backward.restype = ctypes.c_int

    # ------------------------------------------------------------------
    def compact(self, mask: np.ndarray, B: int, H: int, L: int, M: int, N: int, cap: Optional[int] = None):
        """Return (kept_idx int32 [B,H,QB,cap], kept_cnt int32 [B,H,QB])."""
        QB = -(-L // M)
        cap = L if cap is None else cap
        mask = np.ascontiguousarray(mask, dtype=np.uint32)
        G = -(-L // N)
        assert mask.size == B * H * QB * (-(-G // 32)), "mask has the wrong size"
        idx = np.full((B, H, QB, cap), -1, dtype=np.int32)
        cnt = np.zeros((B, H, QB), dtype=np.int32)
        st = self._lib.oracle_compact(mask.ctypes.data, B, H, L, M, N, idx.ctypes.data, cnt.ctypes.data, cap)
        if st != 0:
            raise RuntimeError(f"oracle_compact failed ({st})")
        return idx, cnt

    def attention(self, q, k, v, mask: np.ndarray, M: int, N: int, scale: float,
                  blocks: Optional[Sequence[int]] = None, nthreads: int = 0):
        """q, k, v: bf16 torch tensors (or uint16 arrays of bf16 bits) [B,H,L,d].

        blocks: flat ids (b*H + h)*QB + qb; default all.  Returns float64 arrays
        out [nblocks, M, d] and lse [nblocks, M] (NaN for rows >= L)."""
        qb16, kb16, vb16 = (_bits(x) for x in (q, k, v))
        B, H, L, d = qb16.shape
        QB = -(-L // M)
        if blocks is None:
            blocks = np.arange(B * H * QB, dtype=np.int64)
        blocks = np.ascontiguousarray(np.asarray(blocks, dtype=np.int64))
        mask = np.ascontiguousarray(mask, dtype=np.uint32)
        G = -(-L // N)
        assert mask.size == B * H * QB * (-(-G // 32)), "mask has the wrong size"
        nb = blocks.size
        out = np.empty((nb, M, d), dtype=np.float64)
        lse = np.empty((nb, M), dtype=np.float64)
        if nthreads <= 0:
            nthreads = os.cpu_count() or 1
        st = self._lib.oracle_attention(qb16.ctypes.data, kb16.ctypes.data, vb16.ctypes.data, mask.ctypes.data,
                                        B, H, L, d, M, N, float(scale), blocks.ctypes.data, nb,
                                        out.ctypes.data, lse.ctypes.data, int(nthreads))
        if st != 0:
            raise RuntimeError(f"oracle_attention failed ({st})")
        return out, lse


    def backward(self, q, k, v, dout, mask: np.ndarray, M: int, N: int, scale: float, nthreads: int = 0):
        """Gradients of the forward with respect to q, k and v for the upstream gradient
        dout (bf16 like q, k, v) of out, every head.  Returns float64 arrays
        (dq, dk, dv), each [B, H, L, d]."""
        qb16, kb16, vb16, db16 = (_bits(x) for x in (q, k, v, dout))
        B, H, L, d = qb16.shape
        mask = np.ascontiguousarray(mask, dtype=np.uint32)
        QB, G = -(-L // M), -(-L // N)
        assert mask.size == B * H * QB * (-(-G // 32)), "mask has the wrong size"
        dq = np.empty((B, H, L, d), dtype=np.float64)
        dk = np.empty_like(dq)
        dv = np.empty_like(dq)
        if nthreads <= 0:
            nthreads = os.cpu_count() or 1
        st = self._lib.oracle_attention_backward(qb16.ctypes.data, kb16.ctypes.data, vb16.ctypes.data,
                                                 db16.ctypes.data, mask.ctypes.data, B, H, L, d, M, N,
                                                 float(scale), dq.ctypes.data, dk.ctypes.data, dv.ctypes.data,
                                                 int(nthreads))
        if st != 0:
            raise RuntimeError(f"oracle_attention_backward failed ({st})")
        return dq, dk, dv


def _bits(x) -> np.ndarray:
    """bf16 torch tensor -> contiguous uint16 numpy array of its bit patterns."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16, "oracle inputs are bf16"
            return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x)
    assert x.dtype == np.uint16, "pass bf16 bit patterns as uint16"
    return np.ascontiguousarray(x)


_default: Optional[Oracle] = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
