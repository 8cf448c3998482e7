"""Tile-sparse softmax attention (FG-Attn style) on NVIDIA B200, sm_100a.

A thin ctypes binding over the C ABI in include/fgattn.h.  Every step of the
computation runs in the library's CUDA kernels; this module only checks
tensors, passes their device pointers and the current CUDA stream, and turns
status codes into exceptions.  PyTorch supplies device memory and streams.
There is no CPU path: if libfgattn.so cannot be loaded, importing this package
fails.

Method: "FG-Attn: Leveraging Fine-Grained Sparse Attention in Video Diffusion
Models", Abstract -- score computations are skipped for whole M x N tiles
(M >= 16 queries, N >= 1 keys); skipped scores count as -inf.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

from . import _build

__all__ = ["kept_capacity", "compact_mask", "forward", "backward", "masked_forward", "masked_forward_noalloc", "attention_from_host",
           "device_error", "status_string", "num_sms", "FUSED_MAX_WORDS",
           "FgattnError", "LIB_PATH", "DEVERR_BAD_INDEX", "DEVERR_BAD_COUNT", "DEVERR_TIMEOUT"]

LIB_PATH = _build.LIB

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CAPACITY, ERR_CUDA, ERR_DEVICE = range(6)
FUSED_MAX_WORDS = 256  # mask words per query block that fgattn_masked_forward reads in place
DEVERR_BAD_INDEX, DEVERR_BAD_COUNT, DEVERR_TIMEOUT = 0x1, 0x2, 0x4


def _load() -> ctypes.CDLL:
    if not _build.is_current():
        try:
            _build.build()
        except Exception as e:  # no silent fallback: the CUDA library is the product
            raise ImportError(f"libfgattn.so is missing or stale and could not be built: {e}") from e
    lib = ctypes.CDLL(LIB_PATH)
    i64, p, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
    lib.fgattn_kept_capacity.argtypes = [i64]
    lib.fgattn_kept_capacity.restype = i64
    lib.fgattn_compact_mask.argtypes = [p, i64, i64, i64, i64, i64, p, p, i64, p]
    lib.fgattn_compact_mask.restype = i32
    lib.fgattn_forward.argtypes = [p, p, p, p, p, i64, i64, i64, i64, i64, i64, i64, ctypes.c_float, p, p, p]
    lib.fgattn_forward.restype = i32
    lib.fgattn_forward_strided.argtypes = [p, p, p, p, p, p, p, p, i64, i64, i64, i64, i64, i64, i64,
                                           ctypes.c_float, p, p, p, p]
    lib.fgattn_forward_strided.restype = i32
    lib.fgattn_attention_from_host.argtypes = [p, p, p, p, p, p, p, p, p, p, i64, i64, i64, i64, i64, i64, i64,
                                               ctypes.c_float, p, p, p, p, i64, p]
    lib.fgattn_attention_from_host.restype = i32
    lib.fgattn_masked_forward.argtypes = [p, p, p, p, i64, i64, i64, i64, i64, i64, ctypes.c_float, p, p, p]
    lib.fgattn_masked_forward.restype = i32
    lib.fgattn_masked_forward_noalloc.argtypes = [p, p, p, p, i64, i64, i64, i64, i64, i64, ctypes.c_float, p, p, p]
    lib.fgattn_masked_forward_noalloc.restype = i32
    lib.fgattn_backward.argtypes = [p, p, p, p, p, p, p, p, i64, i64, i64, i64, i64, i64, i64, ctypes.c_float,
                                    p, p, p, p, p]
    lib.fgattn_backward.restype = i32
    lib.fgattn_device_error.argtypes = [p, i32, ctypes.POINTER(ctypes.c_uint32)]
    lib.fgattn_device_error.restype = i32
    lib.fgattn_num_sms.argtypes = []
    lib.fgattn_num_sms.restype = i32
    lib.fgattn_status_string.argtypes = [i32]
    lib.fgattn_status_string.restype = ctypes.c_char_p
    return lib


_lib = _load()


class FgattnError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


def status_string(status: int) -> str:
    return _lib.fgattn_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise FgattnError(status, where)


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    if stream is not None:
        _require_current_device([("stream", s.device.index)])
    return int(s.cuda_stream)


def _current_device() -> int:
    return torch.cuda.current_device()


def _require_current_device(named_indices) -> None:
    """The C ABI launches on the current device and cannot see where a pointer lives:
    every device tensor of a call must be on the current device (a pointer into another
    GPU's memory would reach the kernels as an invalid address)."""
    cur = _current_device()
    for name, index in named_indices:
        if index != cur:
            raise ValueError(f"{name} is on cuda:{index} but the current device is cuda:{cur}; "
                             f"call under torch.cuda.device({index}) or move the tensor")


def _dev(t: torch.Tensor, name: str, dtypes) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    _require_current_device([(name, t.device.index)])
    return t.data_ptr()


def _geometry(L: int, M: int, N: int) -> Tuple[int, int]:
    """(QB, W): query blocks and mask words per block (the C ABI's layout)."""
    QB = -(-L // M)
    G = -(-L // min(N, L))
    return QB, -(-G // 32)


def _numel(t: torch.Tensor, n: int, name: str) -> None:
    """The C ABI takes plain pointers and cannot see extents: check them here."""
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a tensor")
    if t.numel() != n:
        raise ValueError(f"{name} has {t.numel()} elements, expected {n}")


def _dev_rows(t: torch.Tensor, name: str):
    """A [B, H, L, d] bf16 view whose last dimension is contiguous: (pointer, host int64[3] strides)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} has dtype {t.dtype}, expected torch.bfloat16")
    if t.dim() != 4 or (t.shape[-1] > 1 and t.stride(-1) != 1):
        raise ValueError(f"{name} must be a [B, H, L, d] view with a contiguous last dimension")
    _require_current_device([(name, t.device.index)])
    st = (ctypes.c_int64 * 3)(*t.stride()[:3])
    return t.data_ptr(), st


def kept_capacity(L: int) -> int:
    """Per-row stride of kept_idx: L rounded up to 16."""
    return int(_lib.fgattn_kept_capacity(int(L)))


def num_sms() -> int:
    return int(_lib.fgattn_num_sms())


def compact_mask(mask: torch.Tensor, B: int, H: int, L: int, M: int, N: int,
                 kept_idx: Optional[torch.Tensor] = None, kept_cnt: Optional[torch.Tensor] = None,
                 cap: Optional[int] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Packed tile mask uint32/int32 [B,H,QB,W] -> (kept_idx int32 [B,H,QB,cap], kept_cnt int32 [B,H,QB])."""
    QB = -(-L // M) if M >= 1 else 0
    cap = kept_capacity(L) if cap is None else int(cap)
    if min(B, H, L, M, N) >= 1:
        QB, W = _geometry(L, M, N)
        _numel(mask, B * H * QB * W, "mask")
        if kept_idx is not None:
            _numel(kept_idx, B * H * QB * cap, "kept_idx")
        if kept_cnt is not None:
            _numel(kept_cnt, B * H * QB, "kept_cnt")
    dev = mask.device
    if kept_idx is None:
        kept_idx = torch.empty((B, H, QB, cap), dtype=torch.int32, device=dev)
    if kept_cnt is None:
        kept_cnt = torch.empty((B, H, QB), dtype=torch.int32, device=dev)
    st = _lib.fgattn_compact_mask(_dev(mask, "mask", (torch.int32, torch.uint32)), B, H, L, M, N,
                                  _dev(kept_idx, "kept_idx", (torch.int32,)),
                                  _dev(kept_cnt, "kept_cnt", (torch.int32,)), cap, _stream_ptr(stream))
    _check(st, "fgattn_compact_mask")
    return kept_idx, kept_cnt


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, kept_idx: Optional[torch.Tensor],
            kept_cnt: Optional[torch.Tensor], M: int, N: int, scale: Optional[float] = None,
            out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, want_lse: bool = True,
            stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Tile-sparse attention forward.  q, k, v: bf16 [B,H,L,d].  kept_idx None = dense run.

    q, k, v and out may be any [B,H,L,d] views with a contiguous last dimension
    (e.g. x.transpose(1, 2) of a [B,L,H,d] tensor, or slices of a packed
    [B,L,3,H,d] projection); out defaults to the layout of q.
    Returns (out bf16 [B,H,L,d], lse fp32 [B,H,L] natural-log, or None)."""
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [B, H, L, d] shape")
    B, H, L, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if out.shape != q.shape:
        raise ValueError("out must have the shape of q")
    if lse is None and want_lse:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    if lse is not None:
        _numel(lse, B * H * L, "lse")
    if kept_idx is not None and min(L, M, N) >= 1:
        QB = _geometry(L, M, N)[0]
        if kept_idx.dim() < 1 or kept_idx.shape[-1] < L:
            raise ValueError("kept_idx must be [B, H, QB, cap] with cap >= L")
        _numel(kept_idx, B * H * QB * kept_idx.shape[-1], "kept_idx")
        _numel(kept_cnt, B * H * QB, "kept_cnt")
    lp = _dev(lse, "lse", (torch.float32,)) if lse is not None else None
    strided = not all(t.is_contiguous() for t in (q, k, v, out))
    if strided:
        (qp, qs), (kp, ks), (vp, vs), (op, os_) = (_dev_rows(t, n) for t, n in
                                                   ((q, "q"), (k, "k"), (v, "v"), (out, "out")))
    else:
        bf = (torch.bfloat16,)
        qp, kp, vp = _dev(q, "q", bf), _dev(k, "k", bf), _dev(v, "v", bf)
        op = _dev(out, "out", bf)
    if kept_idx is not None:
        ip = _dev(kept_idx, "kept_idx", (torch.int32,))
        cp = _dev(kept_cnt, "kept_cnt", (torch.int32,))
        cap = kept_idx.shape[-1]
    else:
        ip = cp = None
        cap = L
    if strided:
        st = _lib.fgattn_forward_strided(qp, qs, kp, ks, vp, vs, ip, cp, cap, B, H, L, d, M, N, scale, op, os_, lp,
                                         _stream_ptr(stream))
        _check(st, "fgattn_forward_strided")
    else:
        st = _lib.fgattn_forward(qp, kp, vp, ip, cp, cap, B, H, L, d, M, N, scale, op, lp, _stream_ptr(stream))
        _check(st, "fgattn_forward")
    return out, lse


def _host(t: torch.Tensor, name: str, dtypes) -> int:
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def attention_from_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, mask: torch.Tensor, M: int, N: int,
                        scale: Optional[float] = None, buffers: Optional[dict] = None, out: Optional[torch.Tensor] = None,
                        lse: Optional[torch.Tensor] = None, heads_per_group: int = 4, device=None, stream=None):
    """Host tensors in, host tensors out: copy-in, compaction, forward and copy-out pipelined by head groups.

    q, k, v: bf16 [B,H,L,d] and mask int32/uint32 [B,H,QB,W] on the host (pinned for overlap).
    `buffers` holds the device tensors q, k, v, mask, kept_idx, kept_cnt, out, lse (allocated here
    when not given).  Returns (out, lse) host tensors, complete once `stream` is synchronised."""
    B, H, L, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [B, H, L, d] shape")
    QB = -(-L // M)
    cap = kept_capacity(L)
    if min(L, M, N) >= 1:
        QB, W = _geometry(L, M, N)
        _numel(mask, B * H * QB * W, "mask")
        if buffers is not None:
            for name in ("q", "k", "v", "out"):
                if buffers[name].shape != q.shape:
                    raise ValueError(f"buffers['{name}'] must have the shape of q")
            _numel(buffers["mask"], B * H * QB * W, "buffers['mask']")
            _numel(buffers["kept_idx"], B * H * QB * cap, "buffers['kept_idx']")
            _numel(buffers["kept_cnt"], B * H * QB, "buffers['kept_cnt']")
            _numel(buffers["lse"], B * H * L, "buffers['lse']")
        if out is not None and out.shape != q.shape:
            raise ValueError("out must have the shape of q")
        if lse is not None:
            _numel(lse, B * H * L, "lse")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if buffers is None:
        buffers = {"q": torch.empty(q.shape, dtype=q.dtype, device=dev),
                   "k": torch.empty(q.shape, dtype=q.dtype, device=dev),
                   "v": torch.empty(q.shape, dtype=q.dtype, device=dev),
                   "mask": torch.empty(mask.shape, dtype=mask.dtype, device=dev),
                   "kept_idx": torch.empty((B, H, QB, cap), dtype=torch.int32, device=dev),
                   "kept_cnt": torch.empty((B, H, QB), dtype=torch.int32, device=dev),
                   "out": torch.empty(q.shape, dtype=q.dtype, device=dev),
                   "lse": torch.empty((B, H, L), dtype=torch.float32, device=dev)}
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, pin_memory=True)
    bf = (torch.bfloat16,)
    mk = (torch.int32, torch.uint32)
    b = buffers
    if b["kept_idx"].shape[-1] != cap:
        raise ValueError("buffers['kept_idx'] must have a last dimension of kept_capacity(L)")
    st = _lib.fgattn_attention_from_host(
        _host(q, "q", bf), _host(k, "k", bf), _host(v, "v", bf), _host(mask, "mask", mk),
        _dev(b["q"], "q buffer", bf), _dev(b["k"], "k buffer", bf), _dev(b["v"], "v buffer", bf),
        _dev(b["mask"], "mask buffer", mk), _dev(b["kept_idx"], "kept_idx", (torch.int32,)),
        _dev(b["kept_cnt"], "kept_cnt", (torch.int32,)), cap, B, H, L, d, M, N, scale,
        _dev(b["out"], "out buffer", bf), _dev(b["lse"], "lse buffer", (torch.float32,)),
        _host(out, "out", bf), _host(lse, "lse", (torch.float32,)), int(heads_per_group), _stream_ptr(stream))
    _check(st, "fgattn_attention_from_host")
    return out, lse


def masked_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, mask: torch.Tensor, M: int, N: int,
                   scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                   lse: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Mask -> (out, lse) in one kernel: the forward reads the packed tile mask in place of
    kept lists (each warp expands its query block's row itself), so no list is written or
    read and nothing is allocated beyond out and lse.  q, k, v: contiguous bf16 [B,H,L,d];
    mask: int32/uint32 [B,H,QB,W] with W <= FUSED_MAX_WORDS (else FgattnError UNSUPPORTED:
    use compact_mask + forward).  Results equal compact_mask + forward bit for bit."""
    B, H, L, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [B, H, L, d] shape")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if min(L, M, N) >= 1:
        QB, W = _geometry(L, M, N)
        _numel(mask, B * H * QB * W, "mask")
    if out is None:
        out = torch.empty_like(q)
    if out.shape != q.shape:
        raise ValueError("out must have the shape of q")
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    _numel(lse, B * H * L, "lse")
    bf = (torch.bfloat16,)
    st = _lib.fgattn_masked_forward(_dev(q, "q", bf), _dev(k, "k", bf), _dev(v, "v", bf),
                                    _dev(mask, "mask", (torch.int32, torch.uint32)), B, H, L, d, M, N, scale,
                                    _dev(out, "out", bf), _dev(lse, "lse", (torch.float32,)), _stream_ptr(stream))
    _check(st, "fgattn_masked_forward")
    return out, lse


def masked_forward_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, mask: torch.Tensor, M: int, N: int,
                           scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                           lse: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Mask -> (out, lse) with the kept lists in the library's fixed scratch array.

    For callers that cannot allocate device memory: pass preallocated out and
    lse and nothing is allocated (the library's array is at most
    FGATTN_NOALLOC_SCRATCH_BYTES; larger problems raise FgattnError CAPACITY).
    Calls that can overlap on the GPU share that array and race."""
    B, H, L, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [B, H, L, d] shape")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if min(L, M, N) >= 1:
        QB, W = _geometry(L, M, N)
        _numel(mask, B * H * QB * W, "mask")
    if out is None:
        out = torch.empty_like(q)
    if out.shape != q.shape:
        raise ValueError("out must have the shape of q")
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    _numel(lse, B * H * L, "lse")
    bf = (torch.bfloat16,)
    st = _lib.fgattn_masked_forward_noalloc(_dev(q, "q", bf), _dev(k, "k", bf), _dev(v, "v", bf),
                                            _dev(mask, "mask", (torch.int32, torch.uint32)), B, H, L, d, M, N,
                                            scale, _dev(out, "out", bf), _dev(lse, "lse", (torch.float32,)),
                                            _stream_ptr(stream))
    _check(st, "fgattn_masked_forward_noalloc")
    return out, lse


def backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, dout: torch.Tensor,
             lse: torch.Tensor, kept_idx: Optional[torch.Tensor], kept_cnt: Optional[torch.Tensor], M: int, N: int,
             scale: Optional[float] = None, dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None,
             dv: Optional[torch.Tensor] = None, delta: Optional[torch.Tensor] = None,
             stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Gradients of the tile-sparse forward over the same kept lists (None = dense).

    q, k, v, out (the forward's output), dout: contiguous bf16 [B,H,L,d]; lse: the
    forward's fp32 [B,H,L].  Returns (dq, dk, dv), fp32 [B,H,L,d].  delta (fp32
    [B,H,L], dO_i . O_i on return) is a workspace, allocated here when not given.
    dk and dv are sums of float atomics: their last bits depend on the order."""
    if q.dim() != 4 or any(t.shape != q.shape for t in (k, v, out, dout)):
        raise ValueError("q, k, v, out, dout must share one [B, H, L, d] shape")
    B, H, L, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _numel(lse, B * H * L, "lse")
    if kept_idx is not None and min(L, M, N) >= 1:
        QB = _geometry(L, M, N)[0]
        if kept_idx.dim() < 1 or kept_idx.shape[-1] < L:
            raise ValueError("kept_idx must be [B, H, QB, cap] with cap >= L")
        _numel(kept_idx, B * H * QB * kept_idx.shape[-1], "kept_idx")
        _numel(kept_cnt, B * H * QB, "kept_cnt")
    f32 = (torch.float32,)
    grads = []
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        if g is None:
            g = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        _numel(g, B * H * L * d, name)
        grads.append(g)
    if delta is None:
        delta = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    _numel(delta, B * H * L, "delta")
    bf = (torch.bfloat16,)
    if kept_idx is not None:
        ip, cp, cap = _dev(kept_idx, "kept_idx", (torch.int32,)), _dev(kept_cnt, "kept_cnt", (torch.int32,)), \
            kept_idx.shape[-1]
    else:
        ip = cp = None
        cap = L
    st = _lib.fgattn_backward(_dev(q, "q", bf), _dev(k, "k", bf), _dev(v, "v", bf), _dev(out, "out", bf),
                              _dev(dout, "dout", bf), _dev(lse, "lse", f32), ip, cp, cap, B, H, L, d, M, N, scale,
                              _dev(grads[0], "dq", f32), _dev(grads[1], "dk", f32), _dev(grads[2], "dv", f32),
                              _dev(delta, "delta", f32), _stream_ptr(stream))
    _check(st, "fgattn_backward")
    return grads[0], grads[1], grads[2]


def device_error(clear: bool = True, stream=None) -> int:
    """Synchronise the stream and return the kernels' device error bits (DEVERR_*)."""
    bits = ctypes.c_uint32(0)
    st = _lib.fgattn_device_error(_stream_ptr(stream), 1 if clear else 0, ctypes.byref(bits))
    if st not in (OK, ERR_DEVICE):
        _check(st, "fgattn_device_error")
    return int(bits.value)
