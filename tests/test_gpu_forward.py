"""Tile-sparse attention forward on the GPU against the CPU oracle."""
import functools
import json
import os

import numpy as np
import pytest
import torch

import fine_grained_sparse_fgattn_b200 as F
import workloads as W
from gpu_common import block_rows, compare, parity_case, run_gpu, sample_blocks

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_golden_fixture():
    with open(os.path.join(HERE, "golden", "oracle_tiny.json")) as f:
        fx = json.load(f)
    B, H, L, d, M, N = fx["B"], fx["H"], fx["L"], fx["d"], fx["M"], fx["N"]
    as_bf16 = lambda key: torch.from_numpy(np.array(fx[key], dtype=np.uint16).astype(np.int16)).view(
        torch.bfloat16).reshape(B, H, L, d)
    q, k, v = as_bf16("q_bf16_bits"), as_bf16("k_bf16_bits"), as_bf16("v_bf16_bits")
    mask = np.array(fx["mask_u32"], dtype=np.uint32)
    out, lse, idx, cnt = run_gpu(q, k, v, mask, M, N, fx["scale"])
    assert cnt.reshape(-1).tolist() == fx["kept_cnt"]
    for r, lst in enumerate(fx["kept_idx"]):
        assert idx.reshape(-1, idx.shape[-1])[r, :len(lst)].tolist() == lst
    QB = -(-L // M)
    o_ref = np.full((QB, M, d), np.nan)
    l_ref = np.full((QB, M), np.nan)
    o_ref.reshape(-1, d)[:L] = np.array(fx["out"])
    l_ref.reshape(-1)[:L] = np.array(fx["lse"])
    o_gpu, l_gpu = block_rows(out, lse, list(range(QB)), H, QB, M, L)
    compare(o_gpu, l_gpu, o_ref, l_ref)


def test_tiny_workload_all_blocks(oracle):
    w = W.get("tiny")
    q, k, v = W.make_qkv(w, 0)
    stats, _ = parity_case(oracle, q, k, v, W.make_mask(w, 0), w.M, w.N, w.scale)
    print(stats)


FUZZ = [
    # L, d, M, N, density, H
    (16, 64, 16, 1, 0.3, 1), (37, 128, 16, 3, 0.5, 2), (130, 128, 16, 8, 0.2, 1), (300, 64, 32, 4, 0.3, 2),
    (257, 128, 64, 1, 0.4, 1), (700, 128, 64, 16, 0.3, 1), (129, 128, 128, 64, 0.5, 1), (600, 128, 128, 7, 0.25, 1),
    (200, 64, 64, 2, 0.6, 1), (513, 64, 128, 3, 0.3, 1), (640, 128, 32, 64, 0.5, 1), (1000, 128, 64, 33, 0.1, 1),
    (128, 128, 64, 128, 0.0, 1), (383, 128, 16, 1, 1.0, 1), (97, 64, 16, 100, 0.5, 1), (450, 128, 128, 1, 0.05, 2),
    # 128-row blocks (query-major kernel): one partial block, a single key, exact multiples,
    # keys of a chunk split unevenly between the two softmax halves
    (100, 128, 128, 16, 0.5, 1), (1, 128, 128, 1, 1.0, 1), (256, 64, 128, 128, 0.3, 2), (384, 128, 128, 32, 0.2, 1),
    (200, 128, 128, 5, 0.35, 1),
    # d = 96 (Q/K second panel of 32 columns, V and O padded to 128): every kernel and layout
    (300, 96, 64, 16, 0.3, 2), (257, 96, 64, 1, 0.4, 1), (200, 96, 16, 3, 0.5, 1), (640, 96, 32, 64, 0.5, 1),
    (130, 96, 32, 4, 0.3, 1), (513, 96, 128, 3, 0.3, 1), (384, 96, 128, 32, 0.2, 1), (97, 96, 128, 128, 1.0, 1),
    (700, 96, 64, 7, 0.1, 1),
]


@pytest.mark.parametrize("L,d,M,N,density,H", FUZZ)
def test_fuzz_all_blocks(oracle, L, d, M, N, density, H):
    QB, G = -(-L // M), -(-L // N)
    q, k, v = W.random_qkv(1, H, L, d, seed=L * 7 + d + M + N, std=1.5)
    tiles = W.random_tiles(1, H, QB, G, density, seed=L + 3 * N)
    parity_case(oracle, q, k, v, W.pack_tiles(tiles), M, N, 1.0 / np.sqrt(d))


def test_empty_mask_is_diagonal_only(oracle):
    L, d, M, N = 500, 128, 64, 5
    QB, G = -(-L // M), -(-L // N)
    q, k, v = W.random_qkv(1, 2, L, d, seed=5)
    parity_case(oracle, q, k, v, W.pack_tiles(np.zeros((1, 2, QB, G), bool)), M, N, 0.09)


def test_large_scores_rescale(oracle):
    """Scores spanning hundreds of log units force many reference updates and O rescales."""
    L, d, M, N = 900, 128, 64, 4
    QB, G = -(-L // M), -(-L // N)
    q, k, v = W.random_qkv(1, 1, L, d, seed=6, std=1.0)
    ramp = torch.linspace(0.1, 6.0, L).reshape(1, 1, L, 1)
    k = (k.float() * ramp).to(torch.bfloat16)  # later keys score higher -> the max keeps rising
    tiles = W.random_tiles(1, 1, QB, G, 0.5, seed=7)
    parity_case(oracle, q, k, v, W.pack_tiles(tiles), M, N, 0.3)


@pytest.mark.parametrize("M,d", [(64, 128), (128, 128), (64, 96), (128, 96)])
def test_dense_null_list_matches_all_ones(oracle, M, d):
    """A dense run (no lists) equals an all-ones mask.  Dense runs and M = 128 lists take
    the query-major kernel (identical values); M = 64 lists take the key-major one
    (same result within tolerance, both checked against the oracle)."""
    L, N = 777, 16
    QB, G = -(-L // M), -(-L // N)
    q, k, v = W.random_qkv(2, 2, L, d, seed=8)
    ones = W.pack_tiles(np.ones((2, 2, QB, G), bool))
    o1, l1, _, _ = run_gpu(q, k, v, ones, M, N, 0.1)
    o2, l2, _, _ = run_gpu(q, k, v, ones, M, N, 0.1, dense=True)
    if M == 128:
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
    blocks = list(range(2 * 2 * QB))
    o_ref, l_ref = oracle.attention(q, k, v, ones, M, N, 0.1, blocks=blocks)
    for o, l in ((o1, l1), (o2, l2)):
        o_gpu, l_gpu = block_rows(o, l, blocks, 2, QB, M, L)
        compare(o_gpu, l_gpu, o_ref, l_ref)


@functools.lru_cache(maxsize=2)
def _inputs(name, N, sp):
    w = W.get(name)
    q, k, v = W.make_qkv(w, 0)
    return w, q, k, v, W.make_mask(w, 0, N=N, sparsity=sp)


# Full-size workloads in the benchmark's launch configuration (every head in one
# call).  Each is checked against the oracle on the first block, the ragged last
# blocks, at least 256 further seeded blocks and one whole head; the per-key
# layer (1024 blocks) on every block.  The oracle's cost grows with the kept
# scores, so on the HunyuanVideo-like layer (929 blocks of 128 rows x 118800
# keys per head) the whole head is checked at 70 % and 90 %, and the densest
# point (0 %) takes its whole-launch check from the dense run of the same
# kernel instead (below).
@pytest.mark.parametrize("name,N,sp,whole_head", [
    ("perkey", None, None, None),
    ("wan480p", None, None, 0),
    ("hunyuan720p", None, 0.0, None),
    ("hunyuan720p", None, 0.5, None),
    ("hunyuan720p", None, 0.7, 0),
    ("hunyuan720p", None, 0.9, 0),
    ("gransweep", 1, None, 0),
    ("gransweep", 4, None, 0),
    ("gransweep", 16, None, 0),
    ("gransweep", 64, None, 0),
])
def test_workload_sampled_blocks(oracle, name, N, sp, whole_head):
    w, q, k, v, mask = _inputs(name, N, sp)
    N = w.N if N is None else N
    if name == "perkey":
        blocks = None  # every block of the launch
    else:
        blocks = sample_blocks(w.B, w.H, w.QB, 256, seed=11, whole_heads=(whole_head,) if whole_head is not None else ())
        assert len(blocks) >= 256 + (w.QB if whole_head is not None else 0)
    stats, (out, lse, idx, cnt) = parity_case(oracle, q, k, v, mask, w.M, N, w.scale, blocks=blocks)
    # every row of the whole launch is finite (all blocks, not only the sampled ones)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    if sp == 0.0:
        # all tiles kept: the list run equals the dense run of the same kernel on every row of the launch
        o2, l2, _, _ = run_gpu(q, k, v, mask, w.M, N, w.scale, dense=True)
        assert torch.equal(out, o2) and torch.equal(lse, l2)
    print(name, N, sp, stats)


def test_head_dim_96_wan_like_layer(oracle):
    """d = 96 at the Wan-480p-like shape and mask (4 heads): 256 seeded blocks, the ragged
    last blocks and one whole head against the oracle."""
    w = W.get("wan480p").with_(H=4, d=96)
    q, k, v = W.make_qkv(w, 0)
    mask = W.make_mask(w, 0)
    blocks = sample_blocks(w.B, w.H, w.QB, 256, seed=13, whole_heads=(1,))
    stats, (out, lse, _, _) = parity_case(oracle, q, k, v, mask, w.M, w.N, w.scale, blocks=blocks)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    print(stats)


@pytest.mark.parametrize("M", [64, 128])
def test_corrupt_inputs_report_device_errors(M):
    """Out-of-range indices and counts are caught by the kernel's own checks: error bits, no fault
    (M = 64: key-major kernel; M = 128: query-major kernel)."""
    L, d, N = 256, 128, 8
    QB = -(-L // M)
    dev = torch.device("cuda", 0)
    q, k, v = (x.to(dev) for x in W.random_qkv(1, 1, L, d, seed=3))
    cap = F.kept_capacity(L)
    idx = torch.arange(cap, dtype=torch.int32, device=dev).repeat(1, 1, QB, 1)
    cnt = torch.full((1, 1, QB), 100, dtype=torch.int32, device=dev)
    F.device_error(clear=True)
    idx[0, 0, 1, 5] = L + 3
    idx[0, 0, QB - 1, 7] = -1
    F.forward(q, k, v, idx, cnt, M, N)
    assert F.device_error(clear=True) & F.DEVERR_BAD_INDEX
    idx = torch.arange(cap, dtype=torch.int32, device=dev).repeat(1, 1, QB, 1)
    cnt[0, 0, 0] = 0
    cnt[0, 0, QB - 1] = cap + 50
    out, lse = F.forward(q, k, v, idx, cnt, M, N)
    assert F.device_error(clear=True) & F.DEVERR_BAD_COUNT
    assert F.device_error(clear=True) == 0
    # the block with a clamped count of 1 attends to key 0 only
    assert torch.equal(out[0, 0, :M], v[0, 0, 0].expand(M, d))


@pytest.mark.parametrize("M,N,d", [(64, 16, 128), (16, 3, 64), (32, 8, 128), (64, 1, 128), (128, 64, 128)])
def test_scores_rising_far_after_the_first_chunk(oracle, M, N, d):
    """Keys from position 400 on share a large component with every query, so their
    scores exceed the maxima of each block's first chunk by far more than 2^32:
    both kernels must raise their references (and rescale the partial sums and O)
    by large steps in the middle of an item."""
    L = 700
    QB, G = -(-L // M), -(-L // N)
    q, k, v = W.random_qkv(1, 2, L, d, seed=41)
    u = torch.zeros(d)
    u[0] = 1.0
    late = (torch.arange(L) >= 400).float().reshape(1, 1, L, 1)
    q = (q.float() + 4.0 * u).to(torch.bfloat16)
    k = (k.float() + late * 120.0 * u).to(torch.bfloat16)
    tiles = W.random_tiles(1, 2, QB, G, 0.5, seed=42)
    parity_case(oracle, q, k, v, W.pack_tiles(tiles), M, N, 1.0 / np.sqrt(d))
