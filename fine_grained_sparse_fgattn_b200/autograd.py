"""torch.autograd binding of the tile-sparse attention ("FG-Attn: Leveraging
Fine-Grained Sparse Attention in Video Diffusion Models", Abstract: skipped
M x N tiles count as -inf scores).

The forward is fgattn_forward over the kept lists, the backward is
fgattn_backward over the same lists; this module only wires the two C-ABI
calls into autograd (saving q, k, v, out and lse between them).  The
gradients come back from the library in fp32 and autograd casts them to the
inputs' bf16.

    from fine_grained_sparse_fgattn_b200.autograd import tile_sparse_attention
    kept_idx, kept_cnt = F.compact_mask(mask, B, H, L, M, N)
    out = tile_sparse_attention(q, k, v, kept_idx, kept_cnt, M, N)   # q, k, v: contiguous bf16, requires_grad
    out.float().square().sum().backward()
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import backward as _backward
from . import forward as _forward


class TileSparseAttentionFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, kept_idx, kept_cnt, M: int, N: int, scale: float):
        out, lse = _forward(q, k, v, kept_idx, kept_cnt, M, N, scale)
        ctx.save_for_backward(q, k, v, out, lse, kept_idx, kept_cnt)
        ctx.cfg = (M, N, scale)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse, kept_idx, kept_cnt = ctx.saved_tensors
        M, N, scale = ctx.cfg
        dq, dk, dv = _backward(q, k, v, out, dout.contiguous(), lse, kept_idx, kept_cnt, M, N, scale)
        return dq, dk, dv, None, None, None, None, None


def tile_sparse_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, kept_idx: Optional[torch.Tensor],
                          kept_cnt: Optional[torch.Tensor], M: int, N: int,
                          scale: Optional[float] = None) -> torch.Tensor:
    """Differentiable tile-sparse attention: contiguous bf16 q, k, v [B, H, L, d] with
    d in {64, 96, 128}; kept lists from compact_mask (None = dense).  Returns out."""
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)
    return TileSparseAttentionFunction.apply(q, k, v, kept_idx, kept_cnt, int(M), int(N), scale)
