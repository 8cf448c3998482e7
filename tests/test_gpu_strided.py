"""Forward on strided layouts ([B][L][H][d], a packed [B][L][3][H][d] projection,
mixed layouts) against the contiguous path (bit-identical: same kernel, same
lists, only the addressing differs) and against the oracle."""
import numpy as np
import pytest
import torch

import fine_grained_sparse_fgattn_b200 as F
import workloads as W
from gpu_common import block_rows, compare

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)

CASES = [
    # B, H, L, d, M, N, density, dense
    (2, 3, 700, 128, 64, 16, 0.3, False),   # tile layout, ragged last block and group
    (1, 4, 517, 128, 16, 3, 0.3, False),    # gather layout
    (2, 2, 300, 64, 32, 8, 0.4, False),     # d = 64
    (1, 2, 650, 128, 128, 64, 0.5, False),  # M = 128
    (2, 2, 400, 128, 64, 16, 1.0, True),    # dense run (no lists)
    (2, 2, 333, 96, 64, 16, 0.4, False),    # d = 96, tile layout
    (1, 3, 290, 96, 32, 5, 0.3, False),     # d = 96, gather layout
    (1, 2, 300, 96, 128, 16, 0.5, False),   # d = 96, M = 128
]


def _inputs(B, H, L, d, M, N, density, seed):
    QB, G = -(-L // M), -(-L // N)
    q, k, v = W.random_qkv(B, H, L, d, seed=seed, std=1.5)
    mask = W.pack_tiles(W.random_tiles(B, H, QB, G, density, seed=seed + 1))
    return q, k, v, mask


def _contiguous(q, k, v, idx, cnt, M, N, scale):
    out, lse = F.forward(q.to(DEV), k.to(DEV), v.to(DEV), idx, cnt, M, N, scale)
    return out, lse


def _lists(mask, B, H, L, M, N, dense):
    if dense:
        return None, None
    md = torch.from_numpy(mask.view(np.int32)).to(DEV)
    return F.compact_mask(md, B, H, L, M, N)


@pytest.mark.parametrize("B,H,L,d,M,N,density,dense", CASES)
@pytest.mark.parametrize("layout", ["blhd", "packed_qkv", "mixed"])
def test_strided_layouts(oracle, layout, B, H, L, d, M, N, density, dense):
    q, k, v, mask = _inputs(B, H, L, d, M, N, density, seed=L + d + M)
    scale = 1.0 / np.sqrt(d)
    idx, cnt = _lists(mask, B, H, L, M, N, dense)
    o_ref_gpu, l_ref_gpu = _contiguous(q, k, v, idx, cnt, M, N, scale)

    if layout == "blhd":  # every tensor [B][L][H][d]; out follows q's layout
        qs, ks, vs = (t.transpose(1, 2).contiguous().to(DEV).transpose(1, 2) for t in (q, k, v))
        out = None
    elif layout == "packed_qkv":  # one [B][L][3][H][d] projection; out [B][L][H][d]
        x = torch.stack([t.transpose(1, 2) for t in (q, k, v)], dim=2).contiguous().to(DEV)
        qs, ks, vs = (x[:, :, i].transpose(1, 2) for i in range(3))
        out = torch.full((B, L, H, d), float("nan"), dtype=torch.bfloat16, device=DEV).transpose(1, 2)
    else:  # q contiguous, k and v [B][L][H][d], out [B][L][H][d]
        qs = q.to(DEV)
        ks, vs = (t.transpose(1, 2).contiguous().to(DEV).transpose(1, 2) for t in (k, v))
        out = torch.full((B, L, H, d), float("nan"), dtype=torch.bfloat16, device=DEV).transpose(1, 2)
    o, l = F.forward(qs, ks, vs, idx, cnt, M, N, scale, out=out)
    assert not all(t.is_contiguous() for t in (qs, ks, vs, o))  # the strided entry point ran
    assert F.device_error() == 0
    # identical to the contiguous path, value for value
    assert torch.equal(o.float().cpu(), o_ref_gpu.float().cpu())
    assert torch.equal(l.cpu(), l_ref_gpu.cpu())
    # and within tolerance of the oracle on every block
    QB = -(-L // M)
    blocks = list(range(B * H * QB))
    omask = np.full_like(mask, 0xFFFFFFFF) if dense else mask
    o_orc, l_orc = oracle.attention(q, k, v, omask, M, N, scale, blocks=blocks)
    o_gpu, l_gpu = block_rows(o.float().cpu().contiguous(), l.cpu(), blocks, H, QB, M, L)
    compare(o_gpu, l_gpu, o_orc, l_orc)
