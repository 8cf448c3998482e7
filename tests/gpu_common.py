"""Shared helpers for the GPU parity tests: run the CUDA path, run the oracle
on the same seeded inputs, compare.

Tolerances (fp32 accumulation, bf16 P for the P.V product, bf16 output):
  kept-index lists bit-exact;
  out: max |gpu - oracle| <= 2e-2 and ||gpu - oracle||_2 / ||oracle||_2 <= 5e-3;
  lse: max |gpu - oracle| <= 1e-3.
"""
from __future__ import annotations

import numpy as np
import torch

import workloads as W

OUT_MAX_ABS = 2e-2
OUT_REL_RMS = 5e-3
LSE_MAX_ABS = 1e-3


def run_gpu(q, k, v, mask_np, M, N, scale, dense=False):
    """CPU bf16 q/k/v + packed numpy mask -> (out fp32 [B,H,L,d], lse fp32 [B,H,L], idx, cnt) on host."""
    import fine_grained_sparse_fgattn_b200 as F
    B, H, L, d = q.shape
    dev = torch.device("cuda", 0)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    if dense:
        out, lse = F.forward(qd, kd, vd, None, None, M, N, scale)
        idx = cnt = None
    else:
        md = torch.from_numpy(mask_np.view(np.int32)).to(dev)
        idx, cnt = F.compact_mask(md, B, H, L, M, N)
        out, lse = F.forward(qd, kd, vd, idx, cnt, M, N, scale)
    bits = F.device_error()
    assert bits == 0, f"device error bits {bits:#x}"
    return (out.float().cpu(), lse.cpu(), None if idx is None else idx.cpu(), None if cnt is None else cnt.cpu())


def block_rows(out, lse, blocks, H, QB, M, L):
    """Gather rows of the listed flat blocks: [nb, M, d], [nb, M] (NaN past L)."""
    B = out.shape[0]
    d = out.shape[-1]
    o = np.full((len(blocks), M, d), np.nan)
    l = np.full((len(blocks), M), np.nan)
    of = out.reshape(B * H, L, d).numpy()
    lf = lse.reshape(B * H, L).numpy()
    for i, blk in enumerate(blocks):
        bh, qb = divmod(int(blk), QB)
        r0, r1 = qb * M, min(qb * M + M, L)
        o[i, : r1 - r0] = of[bh, r0:r1]
        l[i, : r1 - r0] = lf[bh, r0:r1]
    return o, l


def compare(o_gpu, l_gpu, o_ref, l_ref):
    ok = ~np.isnan(l_ref)
    assert (np.isnan(l_gpu) == ~ok).all(), "row coverage differs"
    dout = np.abs(o_gpu[ok] - o_ref[ok])
    stats = dict(
        out_max_abs=float(dout.max()),
        out_rel_rms=float(np.linalg.norm(o_gpu[ok] - o_ref[ok]) / max(np.linalg.norm(o_ref[ok]), 1e-30)),
        lse_max_abs=float(np.abs(l_gpu[ok] - l_ref[ok]).max()),
        rows=int(ok.sum()),
    )
    assert np.isfinite(o_gpu[ok]).all() and np.isfinite(l_gpu[ok]).all(), f"non-finite output {stats}"
    assert stats["out_max_abs"] <= OUT_MAX_ABS, stats
    assert stats["out_rel_rms"] <= OUT_REL_RMS, stats
    assert stats["lse_max_abs"] <= LSE_MAX_ABS, stats
    return stats


def sample_blocks(B, H, QB, n_random, seed, whole_heads=()):
    """First block, the ragged last block of the first and of the last head, at least
    n_random further distinct seeded blocks, and every block of the flat heads
    (b*H + h) listed in whole_heads."""
    rng = np.random.default_rng(seed)
    total = B * H * QB
    fixed = {0, QB - 1, total - 1, total - QB}
    for bh in whole_heads:
        fixed.update(range(bh * QB, (bh + 1) * QB))
    pool = np.setdiff1d(np.arange(total), np.fromiter(fixed, dtype=np.int64))
    extra = rng.choice(pool, size=min(n_random, pool.size), replace=False)
    return sorted(fixed | {int(x) for x in extra})


def parity_case(oracle, q, k, v, mask_np, M, N, scale, blocks=None, dense=False):
    B, H, L, d = q.shape
    QB = -(-L // M)
    out, lse, idx, cnt = run_gpu(q, k, v, mask_np, M, N, scale, dense=dense)
    if blocks is None:
        blocks = list(range(B * H * QB))
    o_ref, l_ref = oracle.attention(q, k, v, mask_np, M, N, scale, blocks=blocks)
    o_gpu, l_gpu = block_rows(out, lse, blocks, H, QB, M, L)
    return compare(o_gpu, l_gpu, o_ref, l_ref), (out, lse, idx, cnt)
