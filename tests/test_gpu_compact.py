"""Mask compaction on the GPU: bit-exact against the oracle's lists."""
import numpy as np
import pytest
import torch

import fine_grained_sparse_fgattn_b200 as F
import workloads as W

pytestmark = pytest.mark.gpu


def _compare_rows(idx, cnt, ridx, rcnt):
    """Bit-exact: counts everywhere, and every list entry below its row's count (entries
    past the count are untouched memory).  idx/cnt from the GPU, ridx/rcnt from the
    oracle (whose rows are L entries long; the GPU's are L rounded up to 16)."""
    assert (cnt == rcnt).all(), "kept counts differ"
    L = ridx.shape[-1]
    a = idx.reshape(-1, idx.shape[-1])[:, :L]
    b = ridx.reshape(-1, L)
    live = np.arange(L)[None, :] < rcnt.reshape(-1, 1)
    assert np.array_equal(a[live], b[live]), "kept lists differ"


def _compare(oracle, mask_np, B, H, L, M, N):
    dev = torch.device("cuda", 0)
    md = torch.from_numpy(np.ascontiguousarray(mask_np).view(np.int32)).to(dev)
    idx, cnt = F.compact_mask(md, B, H, L, M, N)
    torch.cuda.synchronize()
    ridx, rcnt = oracle.compact(mask_np, B, H, L, M, N)
    _compare_rows(idx.cpu().numpy(), cnt.cpu().numpy(), ridx, rcnt)
    return int(rcnt.sum())


@pytest.mark.parametrize("name,N,sp", [
    ("tiny", None, None),
    ("perkey", None, None),
    ("wan480p", None, None),
    ("hunyuan720p", None, 0.0),
    ("hunyuan720p", None, 0.5),
    ("hunyuan720p", None, 0.7),
    ("hunyuan720p", None, 0.9),
    ("gransweep", 1, None),
    ("gransweep", 4, None),
    ("gransweep", 16, None),
    ("gransweep", 64, None),
])
def test_workload_masks_full_arrays(oracle, name, N, sp):
    """Every head of the workload compacted in one launch (as the benchmark does), all
    rows compared with the oracle head by head (the oracle's lists of one head of the
    densest workload take 0.4 GB)."""
    w = W.get(name)
    N = w.N if N is None else N
    mask = W.make_mask(w, 0, N=N, sparsity=sp)
    dev = torch.device("cuda", 0)
    md = torch.from_numpy(np.ascontiguousarray(mask).view(np.int32)).to(dev)
    idx, cnt = F.compact_mask(md, w.B, w.H, w.L, w.M, N)
    torch.cuda.synchronize()
    assert F.device_error() == 0
    QB, Wd = w.QB, w.with_(N=N).W
    mflat = mask.reshape(w.B * w.H, QB, Wd)
    for bh in range(w.B * w.H):
        ridx, rcnt = oracle.compact(mflat[bh], 1, 1, w.L, w.M, N)
        b, h = divmod(bh, w.H)
        _compare_rows(idx[b, h].cpu().numpy(), cnt[b, h].cpu().numpy(), ridx, rcnt)


@pytest.mark.parametrize("L,M,N,density", [
    (1, 16, 1, 0.0), (1, 16, 8, 1.0), (17, 16, 1, 0.5), (100, 16, 3, 0.0), (100, 16, 3, 1.0),
    (257, 64, 7, 0.3), (1000, 128, 1, 0.2), (4097, 64, 33, 0.5), (64, 64, 100, 0.5), (33, 1, 1, 0.5),
    (2048, 32, 2, 0.05), (5000, 16, 1, 0.9),
    # rows of more than 64 words (eight warps per row): three batches over eight warps,
    # a ragged last group with int4 stores, all ones / all zeros, many batches per warp
    (2080, 64, 1, 0.3), (9002, 64, 4, 0.4), (5000, 16, 1, 1.0), (4200, 64, 2, 0.0), (40000, 128, 1, 0.3),
    (65 * 32 * 3 + 5, 16, 3, 0.5),
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
