"""The fused forward (fgattn_masked_forward: the mask read in place of kept
lists, each warp expanding its query block's row itself) against the two-call
path (fgattn_compact_mask + fgattn_forward) and the oracle.

Both paths run the same kernel code over the same keys in the same order, so
the results must be identical bit for bit; the oracle comparison states the
usual tolerances on top.
"""
import numpy as np
import pytest
import torch

import fine_grained_sparse_fgattn_b200 as F
import workloads as W
from gpu_common import block_rows, compare, sample_blocks

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _both(q, k, v, mask_np, M, N, scale):
    B, H, L, d = q.shape
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    md = torch.from_numpy(np.ascontiguousarray(mask_np).view(np.int32)).to(DEV)
    idx, cnt = F.compact_mask(md, B, H, L, M, N)
    o_ref, l_ref = F.forward(qd, kd, vd, idx, cnt, M, N, scale)
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, L), float("nan"), dtype=torch.float32, device=DEV)
    F.masked_forward(qd, kd, vd, md, M, N, scale, out=out, lse=lse)
    assert F.device_error() == 0
    return out, lse, o_ref, l_ref


FUZZ = [
    # L, d, M, N, density, H   (tile and gather layouts, both kernels, ragged ends, d 64/96/128)
    (16, 64, 16, 1, 0.3, 1), (37, 128, 16, 3, 0.5, 2), (300, 64, 32, 4, 0.3, 2), (257, 128, 64, 1, 0.4, 1),
    (700, 128, 64, 16, 0.3, 1), (129, 128, 128, 64, 0.5, 1), (600, 128, 128, 7, 0.25, 1), (200, 64, 64, 2, 0.6, 1),
    (640, 128, 32, 64, 0.5, 1), (1000, 128, 64, 33, 0.1, 1), (128, 128, 64, 128, 0.0, 1), (383, 128, 16, 1, 1.0, 1),
    (97, 64, 16, 100, 0.5, 1), (450, 128, 128, 1, 0.05, 2), (1, 128, 128, 1, 1.0, 1), (300, 96, 64, 16, 0.3, 2),
    (257, 96, 64, 1, 0.4, 1), (384, 96, 128, 32, 0.2, 1), (8192, 128, 64, 1, 0.3, 1), (5000, 128, 64, 16, 0.02, 1),
]


@pytest.mark.parametrize("L,d,M,N,density,H", FUZZ)
def test_fused_equals_two_calls_and_oracle(oracle, L, d, M, N, density, H):
    QB, G = -(-L // M), -(-L // N)
    q, k, v = W.random_qkv(1, H, L, d, seed=L * 3 + d + M + N, std=1.5)
    mask = W.pack_tiles(W.random_tiles(1, H, QB, G, density, seed=L + 5 * N))
    scale = 1.0 / np.sqrt(d)
    out, lse, o_ref, l_ref = _both(q, k, v, mask, M, N, scale)
    assert torch.equal(out, o_ref) and torch.equal(lse, l_ref)
    blocks = list(range(H * QB)) if H * QB <= 256 else sample_blocks(1, H, QB, 64, seed=L)
    o_orc, l_orc = oracle.attention(q, k, v, mask, M, N, scale, blocks=blocks)
    o_gpu, l_gpu = block_rows(out.float().cpu(), lse.cpu(), blocks, H, QB, M, L)
    compare(o_gpu, l_gpu, o_orc, l_orc)


@pytest.mark.parametrize("name,N,sp", [
    ("tiny", None, None), ("perkey", None, None), ("wan480p", None, None), ("hunyuan720p", None, 0.7),
    ("gransweep", 4, None), ("gransweep", 16, None), ("gransweep", 64, None),
])
def test_fused_full_workloads_bit_identical(oracle, name, N, sp):
    """Every workload whose mask rows fit the fused expansion (W <= 256 words), whole
    launch: identical to the two-call path on every row; 32 sampled blocks vs the oracle."""
    w = W.get(name)
    N = w.N if N is None else N
    q, k, v = W.make_qkv(w, 0)
    mask = W.make_mask(w, 0, N=N, sparsity=sp)
    out, lse, o_ref, l_ref = _both(q, k, v, mask, w.M, N, w.scale)
    assert torch.equal(out, o_ref) and torch.equal(lse, l_ref)
    blocks = sample_blocks(w.B, w.H, w.QB, 32, seed=17)
    o_orc, l_orc = oracle.attention(q, k, v, mask, w.M, N, w.scale, blocks=blocks)
    o_gpu, l_gpu = block_rows(out.float().cpu(), lse.cpu(), blocks, w.H, w.QB, w.M, w.L)
    compare(o_gpu, l_gpu, o_orc, l_orc)


def test_fused_refuses_rows_beyond_its_word_limit():
    """The granularity sweep's per-key point (N = 1, L = 32760: 1024 words per row) is
    refused before anything is enqueued; compact_mask + forward serves it."""
    B, H, L, d, M, N = 1, 1, 32760, 128, 64, 1
    QB, G = -(-L // M), -(-L // N)
    q = torch.zeros((B, H, L, d), dtype=torch.bfloat16, device=DEV)
    mask = torch.zeros((B, H, QB, -(-G // 32)), dtype=torch.int32, device=DEV)
    with pytest.raises(F.FgattnError) as e:
        F.masked_forward(q, q, q, mask, M, N)
    assert e.value.status == F.ERR_UNSUPPORTED
