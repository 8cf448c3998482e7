"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each check takes an oracle handle and raises AssertionError when the oracle
disagrees with a library routine (torch float64 softmax, scipy logsumexp), a brute
force evaluation on tiny inputs, an invariant or a closed form.  The same
checks run against deliberately broken builds of the oracle
(tests/test_oracle_mutants.py) to show that each planted mistake is caught.

What is pinned is the definition on the FG-Attn page ("FG-Attn: Leveraging
Fine-Grained Sparse Attention in Video Diffusion Models", Abstract): scores of
skipped M x N tiles are -inf; the rest is textbook softmax attention.
"""
from __future__ import annotations

import math

import numpy as np
import scipy.special
import torch

import workloads as W

TOL = 1e-10


def _f64(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.float64).numpy()


def _diag_tiles(L: int, M: int, N: int) -> set:
    """Brute force: the tile holding each row's own key index."""
    return {(i // M, i // N) for i in range(L)}


def _dense_kept(tiles: np.ndarray, L: int, M: int, N: int) -> np.ndarray:
    """Bool [L, L] score mask from bool tiles [QB, G] plus the diagonal tiles (loops)."""
    diag = _diag_tiles(L, M, N)
    keep = np.zeros((L, L), dtype=bool)
    for i in range(L):
        for j in range(L):
            keep[i, j] = bool(tiles[i // M, j // N]) or (i // M, j // N) in diag
    return keep


def _brute(q, k, v, keep, scale):
    """Textbook masked softmax attention in float64 (scipy-free logsumexp)."""
    s = scale * (q @ k.T)
    s = np.where(keep, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    lse = (m + np.log(np.exp(s - m).sum(axis=1, keepdims=True)))[:, 0]
    p = np.exp(s - lse[:, None])
    return p @ v, lse


def _run(oracle, q, k, v, tiles, M, N, scale):
    B, H, L, d = q.shape
    mask = W.pack_tiles(tiles)
    out, lse = oracle.attention(q, k, v, mask, M, N, scale, nthreads=2)
    QB = -(-L // M)
    out = out.reshape(B, H, QB * M, d)[:, :, :L]
    lse = lse.reshape(B, H, QB * M)[:, :, :L]
    return out, lse


# ---------------------------------------------------------------------------
def check_dense_matches_torch(oracle):
    """All tiles kept: the oracle is dense softmax attention (torch float64)."""
    for (L, d, M, N, seed) in [(100, 16, 16, 7, 1), (64, 64, 32, 64, 2), (48, 8, 16, 1, 3)]:
        q, k, v = W.random_qkv(1, 2, L, d, seed)
        QB, G = -(-L // M), -(-L // N)
        tiles = np.ones((1, 2, QB, G), dtype=bool)
        out, lse = _run(oracle, q, k, v, tiles, M, N, 1.0 / math.sqrt(d))
        qd, kd, vd = (x.to(torch.float64) for x in (q, k, v))
        s = torch.einsum("bhid,bhjd->bhij", qd, kd) / math.sqrt(d)
        ref = torch.softmax(s, dim=-1) @ vd
        # torch.logsumexp on CPU in float64 was seen off by ~3e-10 on some first calls in a
        # process; scipy's logsumexp of the same float64 scores is the library reference
        ref_lse = scipy.special.logsumexp(s.numpy(), axis=-1)
        assert np.abs(out - ref.numpy()).max() < TOL, "dense out differs from torch"
        assert np.abs(lse - ref_lse).max() < TOL, "dense lse differs from scipy's logsumexp"


def check_brute_force(oracle):
    """Random tiles (no diagonal in them): per-score -inf mask + diagonal, brute force."""
    cases = [(16, 8, 16, 1), (37, 8, 16, 3), (100, 8, 32, 8), (100, 64, 16, 16),
             (64, 8, 16, 2), (50, 8, 32, 50), (130, 8, 16, 7)]
    for ci, (L, d, M, N) in enumerate(cases):
        q, k, v = W.random_qkv(1, 2, L, d, 10 + ci)
        QB, G = -(-L // M), -(-L // N)
        tiles = W.random_tiles(1, 2, QB, G, 0.3, 20 + ci)
        scale = 0.37
        out, lse = _run(oracle, q, k, v, tiles, M, N, scale)
        for h in range(2):
            keep = _dense_kept(tiles[0, h], L, M, N)
            ro, rl = _brute(_f64(q[0, h]), _f64(k[0, h]), _f64(v[0, h]), keep, scale)
            assert np.abs(out[0, h] - ro).max() < TOL, f"brute force out differs (case {ci})"
            assert np.abs(lse[0, h] - rl).max() < TOL, f"brute force lse differs (case {ci})"


def check_empty_mask_keeps_diagonal(oracle):
    """All-zero mask: each row sees exactly the keys of its diagonal tiles."""
    L, d, M, N = 70, 8, 16, 5
    q, k, v = W.random_qkv(1, 1, L, d, 5)
    QB, G = -(-L // M), -(-L // N)
    tiles = np.zeros((1, 1, QB, G), dtype=bool)
    out, lse = _run(oracle, q, k, v, tiles, M, N, 0.5)
    keep = _dense_kept(tiles[0, 0], L, M, N)
    ro, rl = _brute(_f64(q[0, 0]), _f64(k[0, 0]), _f64(v[0, 0]), keep, 0.5)
    assert np.isfinite(out).all() and np.isfinite(lse).all()
    assert np.abs(out[0, 0] - ro).max() < TOL and np.abs(lse[0, 0] - rl).max() < TOL


def check_closed_forms(oracle):
    """Q = 0: out = mean of kept values, lse = ln(#kept keys).  V = c: out = c."""
    L, d, M, N = 90, 8, 16, 4
    _, k, v = W.random_qkv(1, 1, L, d, 6)
    q = torch.zeros_like(k)
    QB, G = -(-L // M), -(-L // N)
    tiles = W.random_tiles(1, 1, QB, G, 0.4, 7)
    out, lse = _run(oracle, q, k, v, tiles, M, N, 0.25)
    keep = _dense_kept(tiles[0, 0], L, M, N)
    vd = _f64(v[0, 0])
    for i in range(L):
        js = np.flatnonzero(keep[i])
        assert abs(lse[0, 0, i] - math.log(len(js))) < 1e-12, "Q=0: lse != ln(count)"
        assert np.abs(out[0, 0, i] - vd[js].mean(axis=0)).max() < 1e-12, "Q=0: out != mean(v)"
    qn, kn, _ = W.random_qkv(1, 1, L, d, 8)
    vc = torch.full_like(kn, 1.5)
    out, _ = _run(oracle, qn, kn, vc, tiles, M, N, 0.25)
    assert np.abs(out - 1.5).max() < 1e-12, "V=c: out != c"


def check_convex_hull(oracle):
    """Each output coordinate lies within [min, max] of the kept values."""
    L, d, M, N = 80, 8, 16, 6
    q, k, v = W.random_qkv(1, 1, L, d, 9, std=2.0)
    QB, G = -(-L // M), -(-L // N)
    tiles = W.random_tiles(1, 1, QB, G, 0.25, 11)
    out, _ = _run(oracle, q, k, v, tiles, M, N, 0.3)
    keep = _dense_kept(tiles[0, 0], L, M, N)
    vd = _f64(v[0, 0])
    for i in range(L):
        kv = vd[keep[i]]
        assert (out[0, 0, i] >= kv.min(axis=0) - 1e-12).all() and (out[0, 0, i] <= kv.max(axis=0) + 1e-12).all()


def check_single_group_is_dense(oracle):
    """N >= L: one key group, always the diagonal one, so any mask gives dense attention."""
    L, d, M = 50, 8, 16
    q, k, v = W.random_qkv(1, 1, L, d, 12)
    tiles = np.zeros((1, 1, -(-L // M), 1), dtype=bool)
    out, lse = _run(oracle, q, k, v, tiles, M, L, 0.4)
    ro, rl = _brute(_f64(q[0, 0]), _f64(k[0, 0]), _f64(v[0, 0]), np.ones((L, L), dtype=bool), 0.4)
    assert np.abs(out[0, 0] - ro).max() < TOL and np.abs(lse[0, 0] - rl).max() < TOL


def check_rows_past_end_are_nan(oracle):
    L, d, M, N = 40, 8, 16, 8
    q, k, v = W.random_qkv(1, 1, L, d, 13)
    mask = W.pack_tiles(np.ones((1, 1, 3, 5), dtype=bool))
    out, lse = oracle.attention(q, k, v, mask, M, N, 0.3, blocks=[2])
    assert np.isfinite(out[0, :8]).all() and np.isnan(out[0, 8:]).all() and np.isnan(lse[0, 8:]).all()


# ---------------------------------------------------------------------------
def _brute_lists(tiles: np.ndarray, L: int, M: int, N: int):
    """Kept key lists by brute force: key j kept for block qb iff its tile is."""
    QB = tiles.shape[-2]
    diag = _diag_tiles(L, M, N)
    lists = []
    for qb in range(QB):
        lists.append([j for j in range(L) if tiles[qb, j // N] or (qb, j // N) in diag])
    return lists


def check_compaction_brute(oracle):
    cases = [(37, 16, 3, 0.3), (100, 16, 1, 0.5), (64, 32, 64, 0.0), (257, 64, 16, 0.2),
             (33, 16, 8, 1.0), (200, 128, 7, 0.4), (1000, 64, 1, 0.1)]
    for ci, (L, M, N, dens) in enumerate(cases):
        QB, G = -(-L // M), -(-L // N)
        tiles = W.random_tiles(1, 2, QB, G, dens, 30 + ci)
        mask = W.pack_tiles(tiles)
        idx, cnt = oracle.compact(mask, 1, 2, L, M, N, cap=L + 5)
        for h in range(2):
            ref = _brute_lists(tiles[0, h], L, M, N)
            for qb in range(QB):
                n = int(cnt[0, h, qb])
                assert n == len(ref[qb]), f"count differs (case {ci})"
                assert list(idx[0, h, qb, :n]) == ref[qb], f"list differs (case {ci})"


def check_compaction_invariants(oracle):
    """Counts equal the sum of kept group sizes; lists are ascending, < L, and
    re-packing them into groups gives back the diagonal-forced tiles."""
    L, M, N = 300, 16, 7
    QB, G = -(-L // M), -(-L // N)
    tiles = W.random_tiles(1, 3, QB, G, 0.35, 40)
    mask = W.pack_tiles(tiles)
    idx, cnt = oracle.compact(mask, 1, 3, L, M, N)
    sizes = np.minimum(N, L - np.arange(G) * N)
    for h in range(3):
        for qb in range(QB):
            forced = tiles[0, h, qb].copy()
            lo, hi = qb * M // N, (min(qb * M + M, L) - 1) // N
            forced[lo:hi + 1] = True
            n = int(cnt[0, h, qb])
            lst = idx[0, h, qb, :n]
            assert n == int(sizes[forced].sum())
            assert (np.diff(lst) > 0).all() and lst.min() >= 0 and lst.max() < L
            rep = np.zeros(G, dtype=bool)
            rep[lst // N] = True
            assert (rep == forced).all()


# ---------------------------------------------------------------------------
# Backward pass: the gradients of the same definition with respect to q, k and v.
def _autograd(q, k, v, dout, keep, scale):
    """torch float64 autograd of masked softmax attention with loss = sum(out * dout)."""
    qd, kd, vd = (torch.from_numpy(_f64(x)).requires_grad_(True) for x in (q, k, v))
    s = scale * (qd @ kd.T)
    s = s.masked_fill(~torch.from_numpy(keep), float("-inf"))
    out = torch.softmax(s, dim=-1) @ vd
    (out * torch.from_numpy(_f64(dout))).sum().backward()
    return qd.grad.numpy(), kd.grad.numpy(), vd.grad.numpy()


def check_backward_matches_torch_autograd(oracle):
    """All tiles kept and random tiles (per-score -inf mask built with loops, plus the
    diagonal rule): the oracle's gradients equal torch float64 autograd."""
    cases = [(40, 8, 16, 40, 1.0), (37, 8, 16, 3, 0.3), (64, 16, 32, 8, 0.4), (50, 8, 16, 1, 0.2)]
    for ci, (L, d, M, N, dens) in enumerate(cases):
        q, k, v = W.random_qkv(1, 2, L, d, 50 + ci)
        dout, _, _ = W.random_qkv(1, 2, L, d, 60 + ci)
        QB, G = -(-L // M), -(-L // N)
        tiles = np.ones((1, 2, QB, G), dtype=bool) if dens >= 1.0 else W.random_tiles(1, 2, QB, G, dens, 70 + ci)
        scale = 0.31
        dq, dk, dv = oracle.backward(q, k, v, dout, W.pack_tiles(tiles), M, N, scale, nthreads=2)
        for h in range(2):
            keep = _dense_kept(tiles[0, h], L, M, N)
            rq, rk, rv = _autograd(q[0, h], k[0, h], v[0, h], dout[0, h], keep, scale)
            for name, a, b in (("dq", dq[0, h], rq), ("dk", dk[0, h], rk), ("dv", dv[0, h], rv)):
                assert np.abs(a - b).max() < TOL, f"{name} differs from autograd (case {ci})"


def check_backward_invariants(oracle):
    """sum_j dS_ij = 0 for every row, hence sum over keys of dk = 0; every row's
    probabilities sum to 1, hence sum over keys of dv = sum over queries of dout."""
    L, d, M, N = 90, 8, 16, 6
    q, k, v = W.random_qkv(1, 2, L, d, 80, std=1.5)
    dout, _, _ = W.random_qkv(1, 2, L, d, 81)
    QB, G = -(-L // M), -(-L // N)
    tiles = W.random_tiles(1, 2, QB, G, 0.3, 82)
    dq, dk, dv = oracle.backward(q, k, v, dout, W.pack_tiles(tiles), M, N, 0.4)
    assert np.abs(dk.sum(axis=2)).max() < 1e-10, "sum of dk over keys is not 0"
    assert np.abs(dv.sum(axis=2) - _f64(dout).sum(axis=2)).max() < 1e-10, "sum of dv != sum of dout"


def check_backward_closed_form(oracle):
    """V = c: every score's gradient vanishes (dP_ij = dout_i . c = D_i), so dq = dk = 0."""
    L, d, M, N = 60, 8, 16, 4
    q, k, _ = W.random_qkv(1, 1, L, d, 83)
    v = torch.full_like(q, -0.75)
    dout, _, _ = W.random_qkv(1, 1, L, d, 84)
    QB, G = -(-L // M), -(-L // N)
    tiles = W.random_tiles(1, 1, QB, G, 0.5, 85)
    dq, dk, dv = oracle.backward(q, k, v, dout, W.pack_tiles(tiles), M, N, 0.5)
    assert np.abs(dq).max() < 1e-12 and np.abs(dk).max() < 1e-12, "V=c: dq, dk not 0"
    assert np.abs(dv).max() > 0.1  # and dv is not trivially zero


ALL_CHECKS = [
    check_dense_matches_torch,
    check_brute_force,
    check_empty_mask_keeps_diagonal,
    check_closed_forms,
    check_convex_hull,
    check_single_group_is_dense,
    check_rows_past_end_are_nan,
    check_compaction_brute,
    check_compaction_invariants,
    check_backward_matches_torch_autograd,
    check_backward_invariants,
    check_backward_closed_form,
]
