"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before enqueuing anything (no GPU needed).

The rejection cases pass at least one argument that validation refuses, so no
kernel is ever launched; they are skipped on a machine with a GPU anyway.
"""
import ctypes
import os
import re

import pytest
import torch

import fine_grained_sparse_fgattn_b200 as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fgattn.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fgattn_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["fgattn_compact_mask", "fgattn_forward", "fgattn_kept_capacity", "fgattn_status_string",
              "fgattn_device_error", "fgattn_num_sms"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(F.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} not exported"


def test_kept_capacity():
    assert F.kept_capacity(1) == 16
    assert F.kept_capacity(16) == 16
    assert F.kept_capacity(32760) == 32768
    assert F.kept_capacity(118800) == 118800
    assert F.kept_capacity(0) == -1


def test_status_strings():
    for s in range(6):
        assert isinstance(F.status_string(s), str) and F.status_string(s)
    assert F.status_string(99) == "unknown status"


no_gpu = pytest.mark.skipif(torch.cuda.is_available(), reason="host-validation cases only run without a GPU")

P = 1 << 20  # a 16-byte-aligned stand-in address; every case below is refused before use


def _fwd(**kw):
    a = dict(q=P, k=P, v=P, idx=P, cnt=P, cap=64, B=1, H=1, L=64, d=128, M=64, N=16, scale=0.1, out=P, lse=P)
    a.update(kw)
    return F._lib.fgattn_forward(a["q"], a["k"], a["v"], a["idx"], a["cnt"], a["cap"], a["B"], a["H"], a["L"],
                                 a["d"], a["M"], a["N"], a["scale"], a["out"], a["lse"], None)


def _cmp(**kw):
    a = dict(mask=P, B=1, H=1, L=64, M=64, N=16, idx=P, cnt=P, cap=64)
    a.update(kw)
    return F._lib.fgattn_compact_mask(a["mask"], a["B"], a["H"], a["L"], a["M"], a["N"], a["idx"], a["cnt"],
                                      a["cap"], None)


@no_gpu
@pytest.mark.parametrize("kw,status", [
    (dict(q=None), F.ERR_INVALID_ARG),
    (dict(out=None), F.ERR_INVALID_ARG),
    (dict(cnt=None), F.ERR_INVALID_ARG),
    (dict(L=0), F.ERR_INVALID_ARG),
    (dict(B=0), F.ERR_INVALID_ARG),
    (dict(N=0), F.ERR_INVALID_ARG),
    (dict(scale=float("nan")), F.ERR_INVALID_ARG),
    (dict(q=P + 8), F.ERR_INVALID_ARG),
    (dict(lse=P + 2), F.ERR_INVALID_ARG),
    (dict(cap=63), F.ERR_CAPACITY),
    (dict(cap=66), F.ERR_CAPACITY),
    (dict(idx=P + 4), F.ERR_INVALID_ARG),
    (dict(d=80), F.ERR_UNSUPPORTED),
    (dict(d=256), F.ERR_UNSUPPORTED),
    (dict(M=48), F.ERR_UNSUPPORTED),
    (dict(M=8), F.ERR_UNSUPPORTED),
    (dict(M=256), F.ERR_UNSUPPORTED),
])
def test_forward_rejects(kw, status):
    assert _fwd(**kw) == status


@no_gpu
@pytest.mark.parametrize("kw,status", [
    (dict(mask=None), F.ERR_INVALID_ARG),
    (dict(idx=None), F.ERR_INVALID_ARG),
    (dict(cnt=None), F.ERR_INVALID_ARG),
    (dict(L=0), F.ERR_INVALID_ARG),
    (dict(M=0), F.ERR_INVALID_ARG),
    (dict(N=0), F.ERR_INVALID_ARG),
    (dict(H=-1), F.ERR_INVALID_ARG),
    (dict(idx=P + 4), F.ERR_INVALID_ARG),
    (dict(cap=48), F.ERR_CAPACITY),
    (dict(cap=66), F.ERR_CAPACITY),
])
def test_compact_rejects(kw, status):
    assert _cmp(**kw) == status


def _mfwd(**kw):
    a = dict(q=P, k=P, v=P, mask=P, B=1, H=1, L=64, d=128, M=64, N=16, scale=0.1, out=P, lse=P)
    a.update(kw)
    return F._lib.fgattn_masked_forward(a["q"], a["k"], a["v"], a["mask"], a["B"], a["H"], a["L"], a["d"], a["M"],
                                        a["N"], a["scale"], a["out"], a["lse"], None)


@no_gpu
@pytest.mark.parametrize("kw,status", [
    (dict(mask=None), F.ERR_INVALID_ARG),
    (dict(mask=P + 2), F.ERR_INVALID_ARG),
    (dict(q=None), F.ERR_INVALID_ARG),
    (dict(L=0), F.ERR_INVALID_ARG),
    (dict(N=0), F.ERR_INVALID_ARG),
    (dict(q=P + 8), F.ERR_INVALID_ARG),
    (dict(d=80), F.ERR_UNSUPPORTED),
    (dict(M=48), F.ERR_UNSUPPORTED),
    # rows of more than 256 mask words (here 32760 groups of one key: 1024 words)
    (dict(L=32760, N=1), F.ERR_UNSUPPORTED),
    (dict(L=8192 * 16 + 16, N=16), F.ERR_UNSUPPORTED),
])
def test_masked_forward_rejects(kw, status):
    assert _mfwd(**kw) == status


def _bwd(**kw):
    a = dict(q=P, k=P, v=P, out=P, dout=P, lse=P, idx=P, cnt=P, cap=64, B=1, H=1, L=64, d=128, M=64, N=16,
             scale=0.1, dq=P, dk=P, dv=P, delta=P)
    a.update(kw)
    return F._lib.fgattn_backward(a["q"], a["k"], a["v"], a["out"], a["dout"], a["lse"], a["idx"], a["cnt"],
                                  a["cap"], a["B"], a["H"], a["L"], a["d"], a["M"], a["N"], a["scale"], a["dq"],
                                  a["dk"], a["dv"], a["delta"], None)


def test_header_declares_backward():
    assert "fgattn_backward" in declared_functions()


@no_gpu
@pytest.mark.parametrize("kw,status", [
    (dict(q=None), F.ERR_INVALID_ARG),
    (dict(out=None), F.ERR_INVALID_ARG),
    (dict(dout=None), F.ERR_INVALID_ARG),
    (dict(lse=None), F.ERR_INVALID_ARG),
    (dict(dq=None), F.ERR_INVALID_ARG),
    (dict(dk=None), F.ERR_INVALID_ARG),
    (dict(dv=None), F.ERR_INVALID_ARG),
    (dict(delta=None), F.ERR_INVALID_ARG),
    (dict(cnt=None), F.ERR_INVALID_ARG),
    (dict(L=0), F.ERR_INVALID_ARG),
    (dict(N=0), F.ERR_INVALID_ARG),
    (dict(scale=float("inf")), F.ERR_INVALID_ARG),
    (dict(dout=P + 8), F.ERR_INVALID_ARG),
    (dict(dk=P + 4), F.ERR_INVALID_ARG),
    (dict(delta=P + 2), F.ERR_INVALID_ARG),
    (dict(cap=63), F.ERR_CAPACITY),
    (dict(d=80), F.ERR_UNSUPPORTED),
    (dict(d=256), F.ERR_UNSUPPORTED),
    (dict(M=256), F.ERR_UNSUPPORTED),
    (dict(M=48), F.ERR_UNSUPPORTED),
])
def test_backward_rejects(kw, status):
    assert _bwd(**kw) == status


@no_gpu
def test_backward_valid_call_without_gpu_reports_cuda_error():
    assert _bwd() == F.ERR_CUDA


@no_gpu
def test_valid_call_without_gpu_reports_cuda_error():
    # All arguments valid, so the launch is attempted; with no device it fails cleanly.
    assert _cmp() == F.ERR_CUDA


def _fwd_strided(qs=None, ks=None, vs=None, os_=None, **kw):
    a = dict(q=P, k=P, v=P, idx=P, cnt=P, cap=64, B=2, H=4, L=64, d=128, M=64, N=16, scale=0.1, out=P, lse=P)
    a.update(kw)
    blhd = (a["L"] * a["H"] * a["d"], a["d"], a["H"] * a["d"])  # [B][L][H][d]
    arr = lambda s: None if s == "null" else (ctypes.c_int64 * 3)(*(blhd if s is None else s))
    return F._lib.fgattn_forward_strided(a["q"], arr(qs), a["k"], arr(ks), a["v"], arr(vs), a["idx"], a["cnt"],
                                         a["cap"], a["B"], a["H"], a["L"], a["d"], a["M"], a["N"], a["scale"],
                                         a["out"], arr(os_), a["lse"], None)


def test_header_declares_strided_forward():
    assert "fgattn_forward_strided" in declared_functions()


@no_gpu
@pytest.mark.parametrize("kw,status", [
    (dict(qs="null"), F.ERR_INVALID_ARG),
    (dict(os_="null"), F.ERR_INVALID_ARG),
    (dict(qs=(64 * 4 * 128, 100, 4 * 128)), F.ERR_INVALID_ARG),    # head stride not a 16-byte multiple
    (dict(qs=(64 * 4 * 128, 64, 4 * 128)), F.ERR_INVALID_ARG),     # stride below one row
    (dict(ks=(64 * 4 * 128, 136, 4 * 136)), F.ERR_INVALID_ARG),    # k strides not whole rows
    (dict(vs=(64 * 4 * 128, 128, 4 * 128 + 8)), F.ERR_INVALID_ARG),  # v token stride not whole rows
    (dict(os_=(64 * 4 * 128, 128, -512)), F.ERR_INVALID_ARG),      # negative stride
    (dict(d=80), F.ERR_UNSUPPORTED),
    (dict(cap=63), F.ERR_CAPACITY),
])
def test_forward_strided_rejects(kw, status):
    assert _fwd_strided(**kw) == status


@no_gpu
def test_forward_strided_valid_call_without_gpu_reports_cuda_error():
    # [B][L][H][d] and a packed [B][L][3][H][d] projection are both accepted; the call fails
    # only at the launch (no device here).
    assert _fwd_strided() == F.ERR_CUDA
    packed = (64 * 3 * 4 * 128, 128, 3 * 4 * 128)
    assert _fwd_strided(qs=packed, ks=packed, vs=packed) == F.ERR_CUDA
    # the stride of an extent-1 dimension is ignored
    assert _fwd_strided(B=1, qs=(0, 128, 4 * 128)) == F.ERR_CUDA


def test_header_declares_host_pipeline():
    assert "fgattn_attention_from_host" in declared_functions()


def _from_host(**kw):
    a = dict(qh=P, kh=P, vh=P, mh=P, q=P, k=P, v=P, m=P, idx=P, cnt=P, cap=64, B=1, H=4, L=64, d=128, M=64, N=16,
             scale=0.1, out=P, lse=P, outh=P, lseh=P, hpg=2)
    a.update(kw)
    return F._lib.fgattn_attention_from_host(a["qh"], a["kh"], a["vh"], a["mh"], a["q"], a["k"], a["v"], a["m"],
                                             a["idx"], a["cnt"], a["cap"], a["B"], a["H"], a["L"], a["d"], a["M"],
                                             a["N"], a["scale"], a["out"], a["lse"], a["outh"], a["lseh"], a["hpg"],
                                             None)


@no_gpu
@pytest.mark.parametrize("kw,status", [
    (dict(qh=None), F.ERR_INVALID_ARG),
    (dict(outh=None), F.ERR_INVALID_ARG),
    (dict(lseh=None), F.ERR_INVALID_ARG),       # lse on the device but not on the host
    (dict(hpg=0), F.ERR_INVALID_ARG),
    (dict(idx=P + 4), F.ERR_INVALID_ARG),
    (dict(cap=60), F.ERR_CAPACITY),
    (dict(d=80), F.ERR_UNSUPPORTED),
    (dict(M=48), F.ERR_UNSUPPORTED),
])
def test_from_host_rejects(kw, status):
    assert _from_host(**kw) == status


def test_binding_refuses_host_tensors():
    """There is no CPU path: host tensors are refused before any library call."""
    q = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        F.forward(q, q, q, None, None, 16, 16)
    with pytest.raises(ValueError):
        F.forward(q.transpose(1, 2), q.transpose(1, 2), q.transpose(1, 2), None, None, 16, 16)
    with pytest.raises(ValueError):
        F.compact_mask(torch.zeros(1, 1, 1, 1, dtype=torch.int32), 1, 1, 16, 16, 16)
    with pytest.raises(ValueError):
        F.masked_forward_noalloc(q, q, q, torch.zeros(1, 1, 1, 1, dtype=torch.int32), 16, 16)


def test_binding_checks_extents():
    """The C ABI cannot see buffer extents; the binding refuses wrong ones before any call."""
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16)
    good_mask = torch.zeros(1, 1, 4, 1, dtype=torch.int32)  # L 64, M 16 -> QB 4; N 16 -> G 4 -> W 1
    with pytest.raises(ValueError, match="mask"):
        F.compact_mask(torch.zeros(1, 1, 4, 2, dtype=torch.int32), 1, 1, 64, 16, 16)
    with pytest.raises(ValueError, match="kept_idx"):
        F.compact_mask(good_mask, 1, 1, 64, 16, 16, kept_idx=torch.zeros(1, 1, 3, 64, dtype=torch.int32))
    with pytest.raises(ValueError, match="kept_cnt"):
        F.forward(q, q, q, torch.zeros(1, 1, 4, 64, dtype=torch.int32), torch.zeros(1, 1, 3, dtype=torch.int32),
                  16, 16)
    with pytest.raises(ValueError, match="cap >= L"):
        F.forward(q, q, q, torch.zeros(1, 1, 4, 32, dtype=torch.int32), torch.zeros(1, 1, 4, dtype=torch.int32),
                  16, 16)
    with pytest.raises(ValueError, match="lse"):
        F.forward(q, q, q, None, None, 16, 16, lse=torch.zeros(1, 1, 63))
    with pytest.raises(ValueError, match="mask"):
        F.masked_forward_noalloc(q, q, q, torch.zeros(1, 1, 5, 1, dtype=torch.int32), 16, 16)
    with pytest.raises(ValueError, match="mask"):
        F.attention_from_host(q, q, q, torch.zeros(1, 1, 4, 2, dtype=torch.int32), 16, 16)


def test_tensors_on_another_device_are_refused(monkeypatch):
    """The C ABI launches on the current device and cannot tell which GPU a pointer
    belongs to, so the binding refuses any device tensor (or stream) that is not on the
    current device, before a pointer reaches the library."""
    monkeypatch.setattr(F, "_current_device", lambda: 0)
    F._require_current_device([("q", 0), ("k", 0)])
    with pytest.raises(ValueError, match="cuda:1"):
        F._require_current_device([("q", 0), ("k", 1)])
    with pytest.raises(ValueError, match="stream"):
        F._require_current_device([("stream", 2)])
