"""Mask compaction on the GPU: bit-exact against the oracle's lists."""
import numpy as np
import pytest
import torch

import fine_grained_sparse_fgattn_b200 as F
import workloads as W

pytestmark = pytest.mark.gpu


def _compare(oracle, mask_np, B, H, L, M, N):
    dev = torch.device("cuda", 0)
    md = torch.from_numpy(np.ascontiguousarray(mask_np).view(np.int32)).to(dev)
    idx, cnt = F.compact_mask(md, B, H, L, M, N)
    torch.cuda.synchronize()
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    ridx, rcnt = oracle.compact(mask_np, B, H, L, M, N)
    assert (cnt == rcnt).all(), "kept counts differ"
    QB = -(-L // M)
    for row in range(B * H * QB):
        b, rem = divmod(row, H * QB)
        h, qb = divmod(rem, QB)
        n = int(rcnt[b, h, qb])
        assert np.array_equal(idx[b, h, qb, :n], ridx[b, h, qb, :n]), f"list differs at row {row}"
    return int(rcnt.sum())


@pytest.mark.parametrize("name,N,sp,heads", [
    ("tiny", None, None, None),
    ("perkey", None, None, 2),
    ("wan480p", None, None, 2),
    ("hunyuan720p", None, 0.7, 1),
    ("hunyuan720p", None, 0.9, 1),
    ("gransweep", 1, None, 1),
    ("gransweep", 4, None, 1),
    ("gransweep", 16, None, 1),
    ("gransweep", 64, None, 1),
])
def test_workload_masks(oracle, name, N, sp, heads):
    w = W.get(name)
    N = w.N if N is None else N
    hs = range(w.H if heads is None else heads)
    mask = W.make_mask(w, 0, N=N, sparsity=sp, heads=hs)
    _compare(oracle, mask, w.B, len(hs), w.L, w.M, N)


@pytest.mark.parametrize("L,M,N,density", [
    (1, 16, 1, 0.0), (1, 16, 8, 1.0), (17, 16, 1, 0.5), (100, 16, 3, 0.0), (100, 16, 3, 1.0),
    (257, 64, 7, 0.3), (1000, 128, 1, 0.2), (4097, 64, 33, 0.5), (64, 64, 100, 0.5), (33, 1, 1, 0.5),
    (2048, 32, 2, 0.05), (5000, 16, 1, 0.9),
])
def test_edge_masks(oracle, L, M, N, density):
    QB, G = -(-L // M), -(-L // N)
    tiles = W.random_tiles(2, 3, QB, G, density, seed=L + M + N)
    _compare(oracle, W.pack_tiles(tiles), 2, 3, L, M, N)


def test_untouched_tail_and_repeat():
    """Entries past kept_cnt keep their old contents; a second call gives identical lists."""
    L, M, N = 300, 16, 4
    QB, G = -(-L // M), -(-L // N)
    mask = W.pack_tiles(W.random_tiles(1, 1, QB, G, 0.2, seed=9))
    dev = torch.device("cuda", 0)
    md = torch.from_numpy(mask.view(np.int32)).to(dev)
    cap = F.kept_capacity(L)
    idx = torch.full((1, 1, QB, cap), -7, dtype=torch.int32, device=dev)
    cnt = torch.zeros((1, 1, QB), dtype=torch.int32, device=dev)
    F.compact_mask(md, 1, 1, L, M, N, kept_idx=idx, kept_cnt=cnt)
    i1 = idx.clone()
    F.compact_mask(md, 1, 1, L, M, N, kept_idx=idx, kept_cnt=cnt)
    assert torch.equal(i1, idx)
    c = cnt.cpu().numpy().reshape(-1)
    ii = idx.cpu().numpy().reshape(QB, cap)
    for r in range(QB):
        assert (ii[r, c[r]:] == -7).all()
