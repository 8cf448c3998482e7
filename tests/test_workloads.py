"""Seeded input generators (no GPU)."""
import numpy as np
import pytest
import torch

import workloads as W


def test_pack_bit_order():
    rng = np.random.default_rng(0)
    tiles = rng.random((2, 3, 70)) < 0.5
    m = W.pack_tiles(tiles)
    assert m.dtype == np.uint32 and m.shape == (2, 3, 3)
    for a in range(2):
        for r in range(3):
            for g in range(70):
                assert ((int(m[a, r, g // 32]) >> (g % 32)) & 1) == int(tiles[a, r, g])
            assert int(m[a, r, 2]) >> 6 == 0  # bits >= G are zero
    assert (W.unpack_tiles(m, 70) == tiles).all()


@pytest.mark.parametrize("name", ["perkey", "wan480p", "hunyuan720p"])
def test_fill_hits_target(name):
    w = W.get(name)
    tiles = W.make_tiles(w, 0, heads=range(2))
    sp = W.score_sparsity(tiles, w)
    assert abs(sp - w.sparsity) < 1e-3
    # every query block keeps the tile holding each row's own key
    i = np.arange(w.L)
    assert tiles[:, :, i // w.M, i // w.N].all()


def test_sweep_targets():
    w = W.get("hunyuan720p")
    for sp in (0.5, 0.9):
        t = W.make_tiles(w, 0, sparsity=sp, heads=range(1))
        assert abs(W.score_sparsity(t, w) - sp) < 1e-3
    assert W.make_tiles(w, 0, sparsity=0.0, heads=range(1)).all()


def test_tiny_is_window_plus_bernoulli():
    w = W.get("tiny")
    t = W.make_tiles(w, 0)
    st = W.structural_tiles(w)
    assert (t >= st).all()
    extra = (t & ~st).sum() / (~st).sum() / (w.B * w.H)
    assert 0.07 < extra < 0.13


def test_seeded_and_head_slices():
    w = W.get("perkey")
    a = W.make_tiles(w, 3, heads=range(1, 3))
    b = W.make_tiles(w, 3)
    assert (a == b[:, 1:3]).all()
    q1, k1, v1 = W.make_qkv(W.get("tiny"), 4)
    q2, k2, v2 = W.make_qkv(W.get("tiny"), 4, heads=range(1, 2))
    assert torch.equal(q1[:, 1:2], q2) and torch.equal(v1[:, 1:2], v2)
    q3, _, _ = W.make_qkv(W.get("tiny"), 5)
    assert not torch.equal(q1, q3)


def test_lowrank_component_peaks_scores():
    w = W.get("wan480p").with_(L=2048, grid=(1, 32, 64), H=1)
    q, k, _ = W.make_qkv(w, 0)
    s = (q[0, 0].float() @ k[0, 0].float().T) * w.scale
    assert s.diagonal().mean() > s.mean() + 5.0


@pytest.mark.parametrize("N", [1, 4, 16, 64])
def test_granularity_sweep_targets(N):
    """The sweep regenerates the same mask family per tile width at one score sparsity,
    with every row's own key kept."""
    w = W.get("gransweep").with_(N=N)
    tiles = W.make_tiles(w, 0, heads=range(1))
    assert abs(W.score_sparsity(tiles, w) - w.sparsity) < 1e-3
    i = np.arange(w.L)
    assert tiles[:, :, i // w.M, i // w.N].all()


def test_random_grad_is_seeded_and_independent_of_qkv():
    """The upstream gradient of the backward cases: same seed, same values; another
    seed, other values; and not a copy of the q/k/v streams of the same seed."""
    a = W.random_grad(1, 2, 40, 16, seed=5)
    b = W.random_grad(1, 2, 40, 16, seed=5)
    c = W.random_grad(1, 2, 40, 16, seed=6)
    q, k, v = W.random_qkv(1, 2, 40, 16, seed=5)
    assert a.dtype == torch.bfloat16 and a.shape == (1, 2, 40, 16)
    assert torch.equal(a, b) and not torch.equal(a, c)
    assert not any(torch.equal(a, t) for t in (q, k, v))
    assert abs(a.float().std().item() - 1.0) < 0.2
