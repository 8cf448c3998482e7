"""Gradients of the tile-sparse attention on the GPU against the CPU oracle.

The GPU path is the one a training step takes: compaction, forward (out, lse),
then the backward kernel on the forward's outputs.  The oracle computes the
gradients of the same definition in fp64 from q, k, v, dO and the mask alone.

Tolerance, from the arithmetic of the kernel: P and dS are rounded to bf16
(relative error at most 2^-9) for the five tensor-core products, Delta is
formed from the bf16 output of the forward (another 2^-9 relative on each term
of dO . O), and everything else accumulates in fp32.  Independent roundings
of 2^-9 over sums of many terms give a relative RMS error of about 1e-3, so
    ||g - ref||_2 / ||ref||_2 <= 1e-2   and   max |g - ref| <= 2e-2 * max |ref|
per gradient leave a factor of about five over the expected error, while a
wrong term (a dropped Delta, a missing scale, a transposed operand) moves the
result by tens of percent.
"""
import numpy as np
import pytest
import torch

import fine_grained_sparse_fgattn_b200 as F
import workloads as W

pytestmark = pytest.mark.gpu

GRAD_REL_RMS = 1e-2
GRAD_MAX_REL = 2e-2


def gpu_backward(q, k, v, dout, mask_np, M, N, scale, dense=False):
    B, H, L, d = q.shape
    dev = torch.device("cuda", 0)
    qd, kd, vd, gd = (t.to(dev) for t in (q, k, v, dout))
    if dense:
        idx = cnt = None
    else:
        idx, cnt = F.compact_mask(torch.from_numpy(mask_np.view(np.int32)).to(dev), B, H, L, M, N)
    out, lse = F.forward(qd, kd, vd, idx, cnt, M, N, scale)
    dq, dk, dv = F.backward(qd, kd, vd, out, gd, lse, idx, cnt, M, N, scale)
    bits = F.device_error()
    assert bits == 0, f"device error bits {bits:#x}"
    return dq.cpu().double().numpy(), dk.cpu().double().numpy(), dv.cpu().double().numpy()


def compare_grads(got, ref):
    stats = {}
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert np.isfinite(g).all(), f"{name}: non-finite values"
        rms = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30))
        mx = float(np.abs(g - r).max() / max(np.abs(r).max(), 1e-30))
        stats[name] = (rms, mx)
        assert rms <= GRAD_REL_RMS, (name, stats)
        assert mx <= GRAD_MAX_REL, (name, stats)
    return stats


def backward_case(oracle, L, d, M, N, density, H, seed, scale=None, dense=False, std=1.5):
    QB, G = -(-L // M), -(-L // N)
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    q, k, v = W.random_qkv(1, H, L, d, seed=seed, std=std)
    dout = W.random_grad(1, H, L, d, seed=seed)
    tiles = np.ones((1, H, QB, G), bool) if dense else W.random_tiles(1, H, QB, G, density, seed=seed + 1)
    mask = W.pack_tiles(tiles)
    got = gpu_backward(q, k, v, dout, mask, M, N, scale, dense=dense)
    ref = oracle.backward(q, k, v, dout, mask, M, N, scale)
    return compare_grads(got, ref)


CASES = [
    # L, d, M, N, density, H: one block, ragged ends, several chunks per list, N = 1 up to
    # N > L, empty masks (diagonal only) and full ones, every (d, M) pair
    (16, 64, 16, 1, 0.3, 1), (37, 128, 16, 3, 0.5, 2), (300, 64, 32, 4, 0.3, 2), (257, 128, 64, 1, 0.4, 1),
    (700, 128, 64, 16, 0.3, 1), (640, 128, 32, 64, 0.5, 1), (200, 64, 64, 2, 0.6, 1), (383, 128, 16, 1, 1.0, 1),
    (128, 128, 64, 128, 0.0, 1), (97, 64, 16, 100, 0.5, 1), (1000, 64, 64, 33, 0.1, 1), (513, 128, 32, 7, 0.25, 2),
    # 128-row blocks (two 64-row halves over one list): ragged last block, a last block
    # whose second half is past L, one block
    (700, 128, 128, 16, 0.3, 1), (450, 64, 128, 5, 0.4, 2), (100, 128, 128, 64, 0.5, 1),
    # d = 96 (tiles padded to 128 columns with zeros): every query-block height
    (300, 96, 64, 16, 0.3, 2), (257, 96, 16, 1, 0.4, 1), (200, 96, 128, 5, 0.35, 1), (130, 96, 32, 4, 0.3, 1),
]


@pytest.mark.parametrize("L,d,M,N,density,H", CASES)
def test_backward_matches_oracle(oracle, L, d, M, N, density, H):
    print(backward_case(oracle, L, d, M, N, density, H, seed=L * 5 + d + M + N))


@pytest.mark.parametrize("M,d", [(16, 64), (64, 128), (128, 128)])
def test_backward_dense_run(oracle, M, d):
    """No lists: every key kept, the same kernel reading keys 0 .. L-1."""
    print(backward_case(oracle, 301, d, M, 16, 1.0, 2, seed=11, dense=True))


def test_backward_large_scores(oracle):
    """Scores spanning tens of log units: P is exp(s - lse) for the forward's lse."""
    print(backward_case(oracle, 400, 128, 64, 8, 0.5, 1, seed=3, scale=0.3, std=3.0))


def test_backward_bad_index_is_flagged():
    """A corrupt list entry is replaced by key 0 and flagged; nothing faults."""
    L, d, M, N = 256, 128, 64, 16
    dev = torch.device("cuda", 0)
    q, k, v = (t.to(dev) for t in W.random_qkv(1, 1, L, d, seed=4))
    g = W.random_grad(1, 1, L, d, seed=4).to(dev)
    mask = torch.from_numpy(W.pack_tiles(np.ones((1, 1, L // M, L // N), bool)).view(np.int32)).to(dev)
    idx, cnt = F.compact_mask(mask, 1, 1, L, M, N)
    out, lse = F.forward(q, k, v, idx, cnt, M, N)
    F.device_error()
    idx[0, 0, 1, 5] = L + 7
    F.backward(q, k, v, out, g, lse, idx, cnt, M, N)
    assert F.device_error() & F.DEVERR_BAD_INDEX


def test_backward_full_wan_layer(oracle):
    """The Wan-480p-like layer at full size (B1 H40 L32760 d128, M64 N16, 70 %), in the
    launch configuration the benchmark times: every head against two properties that
    hold at any size (sum over keys of dk = 0, since every row's dS sums to zero; sum
    over keys of dv = sum over queries of dO, since every row's probabilities sum to
    one), and head 0 element by element against the oracle."""
    w = W.get("wan480p")
    dev = torch.device("cuda", 0)
    q, k, v = W.make_qkv(w, 0)
    g = W.random_grad(w.B, w.H, w.L, w.d, seed=17)
    mask = W.make_mask(w, 0)
    qd, kd, vd, gd = (t.to(dev) for t in (q, k, v, g))
    idx, cnt = F.compact_mask(torch.from_numpy(mask.view(np.int32)).to(dev), w.B, w.H, w.L, w.M, w.N)
    out, lse = F.forward(qd, kd, vd, idx, cnt, w.M, w.N, w.scale)
    dq, dk, dv = F.backward(qd, kd, vd, out, gd, lse, idx, cnt, w.M, w.N, w.scale)
    assert F.device_error() == 0
    # properties, every head: relative to the size of the summed terms
    sdk = dk.double().sum(dim=2)
    assert (sdk.abs().max() / dk.double().abs().sum(dim=2).max()).item() < 1e-3
    sdv = dv.double().sum(dim=2)
    sg = gd.double().sum(dim=2)
    assert ((sdv - sg).abs().max() / gd.double().abs().sum(dim=2).max()).item() < 1e-3
    # head 0 against the oracle
    h0 = range(1)
    q0, k0, v0 = W.make_qkv(w, 0, heads=h0)
    ref = oracle.backward(q0, k0, v0, g[:, :1], W.make_mask(w, 0, heads=h0), w.M, w.N, w.scale)
    got = tuple(t[:, :1].cpu().double().numpy() for t in (dq, dk, dv))
    print(compare_grads(got, ref))
