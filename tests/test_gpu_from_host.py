"""fgattn_attention_from_host (copy-in, compaction, forward, copy-out pipelined by
head groups) against the device path on the same data: identical values,
since every head group runs the same kernels on the same rows.  Ragged group
splits, both forward kernels (M = 64 key-major, M = 128 query-major) and two
calls in a row with different inputs."""
import numpy as np
import pytest
import torch

import fine_grained_sparse_fgattn_b200 as F
import workloads as W

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _case(B, H, L, d, M, N, density, seed):
    QB, G = -(-L // M), -(-L // N)
    q, k, v = W.random_qkv(B, H, L, d, seed=seed)
    mask = W.pack_tiles(W.random_tiles(B, H, QB, G, density, seed=seed + 1))
    return q, k, v, mask


def _device_path(q, k, v, mask, M, N, scale):
    B, H, L, d = q.shape
    md = torch.from_numpy(mask.view(np.int32)).to(DEV)
    idx, cnt = F.compact_mask(md, B, H, L, M, N)
    out, lse = F.forward(q.to(DEV), k.to(DEV), v.to(DEV), idx, cnt, M, N, scale)
    return out.cpu(), lse.cpu()


@pytest.mark.parametrize("B,H,L,d,M,N,hpg", [
    (2, 3, 300, 128, 64, 16, 2),    # 3 groups
    (1, 5, 700, 128, 128, 64, 2),   # ragged last group, query-major kernel
    (2, 2, 257, 64, 32, 3, 3),      # gather layout, ragged
    (1, 4, 129, 128, 16, 8, 8),     # one group
])
def test_pipeline_matches_device_path(B, H, L, d, M, N, hpg):
    scale = 1.0 / np.sqrt(d)
    for call, seed in enumerate((11, 29)):  # two calls in a row, different inputs
        q, k, v, mask = _case(B, H, L, d, M, N, 0.3, seed + L)
        ref_o, ref_l = _device_path(q, k, v, mask, M, N, scale)
        qh, kh, vh = (t.pin_memory() for t in (q, k, v))
        mh = torch.from_numpy(mask.view(np.int32)).pin_memory()
        out, lse = F.attention_from_host(qh, kh, vh, mh, M, N, scale, heads_per_group=hpg)
        torch.cuda.current_stream().synchronize()
        assert F.device_error() == 0
        assert torch.equal(out, ref_o), f"call {call}: out differs"
        assert torch.equal(lse, ref_l), f"call {call}: lse differs"
