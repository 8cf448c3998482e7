"""Seeded synthetic inputs for tile-sparse video-DiT attention.

This module only draws random numbers and lays them out.  It holds none of the
attention arithmetic: no scores, no softmax, no mask compaction and no diagonal
forcing rule of the method (the generated masks *contain* the diagonal tiles,
as the workloads below specify, and the method forces them again on its own).
Both the CUDA path's tests and the CPU oracle take their inputs from here.

Workloads (shapes stand in for the video models named on the FG-Attn page,
"FG-Attn: Leveraging Fine-Grained Sparse Attention in Video Diffusion Models",
section "Recorded benchmark results": Wan 14B 480p 81 frames and HunyuanVideo
720p 129 frames; tile shape M x N with M >= 16, N >= 1 from its Abstract):

  tiny        B1 H2  L2048   grid 4x16x32   d64  M16  N8
  perkey      B1 H8  L8192   grid 8x32x32   d128 M64  N1
  wan480p     B1 H40 L32760  grid 21x30x52  d128 M64  N16   (rank-8 shared token component)
  hunyuan720p B1 H24 L118800 grid 33x45x80  d128 M128 N64   (sparsity 0 / 0.5 / 0.7 / 0.9)
  gransweep   B1 H24 L32760  grid 21x30x52  d128 M64  N in {1, 4, 16, 64}

Token index idx = t*(Hg*Wg) + y*Wg + x (raster order over the latent grid).
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Optional, Tuple

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    grid: Tuple[int, int, int]  # (T, Hg, Wg), T*Hg*Wg == L
    d: int
    M: int
    N: int
    mask: str            # "window_bernoulli" | "window_fill" | "window_stripe_fill" | "dense"
    sparsity: float      # target score-level sparsity for the *_fill masks
    qkv: str = "iid"     # "iid" | "lowrank8"
    window: Tuple[int, int, int] = (1, 4, 8)   # |dt|, |dy|, |dx| on centres
    p_extra: float = 0.1                      # Bernoulli extra tiles (window_bernoulli)
    stripe: Tuple[int, int] = (2, 2)          # |dy|, |dx| on centres, any frame

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def QB(self) -> int:
        return -(-self.L // self.M)

    @property
    def G(self) -> int:
        return -(-self.L // self.N)

    @property
    def W(self) -> int:
        return -(-self.G // 32)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 2048, (4, 16, 32), 64, 16, 8, "window_bernoulli", 0.5,
                     window=(1, 4, 8), p_extra=0.1),
    "perkey": Workload("perkey", 1, 8, 8192, (8, 32, 32), 128, 64, 1, "window_fill", 0.70,
                       window=(1, 4, 8)),
    "wan480p": Workload("wan480p", 1, 40, 32760, (21, 30, 52), 128, 64, 16,
                        "window_stripe_fill", 0.70, qkv="lowrank8", window=(0, 6, 10)),
    "hunyuan720p": Workload("hunyuan720p", 1, 24, 118800, (33, 45, 80), 128, 128, 64,
                            "window_stripe_fill", 0.70, window=(0, 6, 10)),
    "gransweep": Workload("gransweep", 1, 24, 32760, (21, 30, 52), 128, 64, 16,
                          "window_stripe_fill", 0.70, window=(0, 6, 10)),
}


def get(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return w.with_(**overrides) if overrides else w


# ---------------------------------------------------------------------------
# seeds: one independent stream per (purpose, seed, b, h)
# ---------------------------------------------------------------------------
def _stream_seed(seed: int, *parts) -> int:
    h = hashlib.sha256(repr((int(seed),) + tuple(parts)).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _torch_gen(seed: int, *parts) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(_stream_seed(seed, *parts))
    return g


# ---------------------------------------------------------------------------
# Q, K, V
# ---------------------------------------------------------------------------
def make_qkv(w: Workload, seed: int = 0, heads: Optional[range] = None):
    """Return bf16 CPU tensors q, k, v of shape [B, H, L, d] (contiguous).

    Every (b, h) slab comes from its own seeded stream, so a head range can be
    generated alone (a rank that owns heads [h0, h1) draws exactly those).
    Values are drawn in fp32 and rounded once to bf16 (round to nearest even).
    "lowrank8": Q = Zq + U Wh, K = Zk + U Wh, V = Zv with U in R^{L x 8} ~ N(0,1)
    shared by all heads and Wh in R^{8 x d} ~ N(0, 1/8) per head.
    """
    heads = range(w.H) if heads is None else heads
    nh = len(heads)
    q = torch.empty((w.B, nh, w.L, w.d), dtype=torch.bfloat16)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    U = None
    if w.qkv == "lowrank8":
        U = torch.randn((w.L, 8), generator=_torch_gen(seed, "U", w.name, w.L))
    for b in range(w.B):
        for j, h in enumerate(heads):
            for t, name in ((q, "q"), (k, "k"), (v, "v")):
                z = torch.randn((w.L, w.d), generator=_torch_gen(seed, name, w.name, b, h))
                if U is not None and name in ("q", "k"):
                    Wh = torch.randn((8, w.d), generator=_torch_gen(seed, "W", w.name, b, h)) / math.sqrt(8.0)
                    z = z + U @ Wh
                t[b, j].copy_(z.to(torch.bfloat16))
    return q, k, v


# ---------------------------------------------------------------------------
# tile masks
# ---------------------------------------------------------------------------
def _centres(L: int, size: int, grid) -> np.ndarray:
    """(t, y, x) of the centre token of each run of `size` consecutive tokens.

    The centre of a run [s, s+len) is token s + (len-1)//2 (len is ragged at
    the end of the sequence)."""
    T, Hg, Wg = grid
    n = -(-L // size)
    start = np.arange(n, dtype=np.int64) * size
    ln = np.minimum(size, L - start)
    c = start + (ln - 1) // 2
    t = c // (Hg * Wg)
    y = (c // Wg) % Hg
    x = c % Wg
    return np.stack([t, y, x], axis=1)


def _rows_keys(w: Workload, N: int):
    rows = np.minimum(w.M, w.L - np.arange(w.QB, dtype=np.int64) * w.M)
    G = -(-w.L // N)
    keys = np.minimum(N, w.L - np.arange(G, dtype=np.int64) * N)
    return rows, keys


def structural_tiles(w: Workload, N: Optional[int] = None) -> np.ndarray:
    """Bool [QB, G]: the window / stripe tiles plus the diagonal tiles (shared by all heads)."""
    N = w.N if N is None else N
    qc = _centres(w.L, w.M, w.grid).astype(np.int32)
    kc = _centres(w.L, N, w.grid).astype(np.int32)

    def _absdiff(a: int) -> np.ndarray:
        return np.abs(np.ascontiguousarray(qc[:, a])[:, None] - np.ascontiguousarray(kc[:, a])[None, :])

    dt, dy, dx = _absdiff(0), _absdiff(1), _absdiff(2)
    if w.mask == "dense":
        st = np.ones((qc.shape[0], kc.shape[0]), dtype=bool)
    else:
        wt, wy, wx = w.window
        st = (dt <= wt) & (dy <= wy) & (dx <= wx)
        if w.mask == "window_stripe_fill":
            sy, sx = w.stripe
            st |= (dy <= sy) & (dx <= sx)
    # diagonal tiles: the tile that holds each query row's own key index
    i = np.arange(w.L, dtype=np.int64)
    st[i // w.M, i // N] = True
    return st


def _fill_to_budget(st: np.ndarray, rows: np.ndarray, keys: np.ndarray, budget: int,
                    rng: np.random.Generator) -> np.ndarray:
    """Add uniformly chosen tiles until the kept score count reaches `budget`.

    Tiles are first drawn independently with the probability that meets the
    budget in expectation, then single tiles chosen uniformly at random are
    added (or removed, never a structural one) until the count lies in
    [budget, budget + largest tile)."""
    size = rows[:, None] * keys[None, :]
    kept = int(size[st].sum())
    if kept >= budget:
        return st.copy()
    cand = ~st
    cand_scores = int(size[cand].sum())
    p = min(1.0, (budget - kept) / max(cand_scores, 1))
    pick = cand & (rng.random(st.shape, dtype=np.float32) < p)
    out = st | pick
    total = kept + int(size[pick].sum())
    flat_out = out.reshape(-1)
    flat_pick = pick.reshape(-1)
    flat_size = size.reshape(-1)
    n = flat_out.size
    big = int(flat_size.max())
    while total < budget:
        for f in rng.integers(0, n, size=4096):
            if not flat_out[f]:
                flat_out[f] = True
                total += int(flat_size[f])
                if total >= budget:
                    break
    while total - budget >= big:
        for f in rng.integers(0, n, size=4096):
            if flat_pick[f] and flat_out[f]:
                flat_out[f] = False
                total -= int(flat_size[f])
                if total - budget < big:
                    break
    return out


def pack_tiles(tiles: np.ndarray) -> np.ndarray:
    """Bool [..., QB, G] -> uint32 [..., QB, W]; tile g is bit (g % 32) of word g // 32."""
    G = tiles.shape[-1]
    W = -(-G // 32)
    pad = W * 32 - G
    if pad:
        tiles = np.concatenate([tiles, np.zeros(tiles.shape[:-1] + (pad,), dtype=bool)], axis=-1)
    by = np.packbits(tiles, axis=-1, bitorder="little")  # [..., W*4] bytes, LSB first
    return np.ascontiguousarray(by).view("<u4").reshape(tiles.shape[:-1] + (W,))


def unpack_tiles(mask: np.ndarray, G: int) -> np.ndarray:
    """Inverse of pack_tiles (bits >= G dropped)."""
    by = np.ascontiguousarray(mask).view(np.uint8)
    bits = np.unpackbits(by, axis=-1, bitorder="little").astype(bool)
    return bits[..., :G]


def make_tiles(w: Workload, seed: int = 0, N: Optional[int] = None, sparsity: Optional[float] = None,
               heads: Optional[range] = None) -> np.ndarray:
    """Bool tile mask [B, H, QB, G] for workload w (N and sparsity may be overridden)."""
    N = w.N if N is None else N
    sp = w.sparsity if sparsity is None else sparsity
    heads = range(w.H) if heads is None else heads
    G = -(-w.L // N)
    if w.mask == "dense" or (w.mask.endswith("_fill") and sp <= 0.0):
        return np.ones((w.B, len(heads), w.QB, G), dtype=bool)
    st = structural_tiles(w, N)
    rows, keys = _rows_keys(w, N)
    out = np.empty((w.B, len(heads), w.QB, G), dtype=bool)
    budget = int(round((1.0 - sp) * w.L * w.L))
    for b in range(w.B):
        for j, h in enumerate(heads):
            rng = np.random.default_rng(_stream_seed(seed, "mask", w.name, N, sp, b, h))
            if w.mask == "window_bernoulli":
                out[b, j] = st | (rng.random(st.shape, dtype=np.float32) < w.p_extra)
            else:
                out[b, j] = _fill_to_budget(st, rows, keys, budget, rng)
    return out


def make_mask(w: Workload, seed: int = 0, N: Optional[int] = None, sparsity: Optional[float] = None,
              heads: Optional[range] = None) -> np.ndarray:
    """Packed uint32 mask [B, H, QB, W] (see pack_tiles for the bit order)."""
    return pack_tiles(make_tiles(w, seed, N, sparsity, heads))


def score_sparsity(tiles: np.ndarray, w: Workload, N: Optional[int] = None) -> float:
    """1 - kept scores / L^2, averaged over (b, h), counting ragged tiles by true size."""
    N = w.N if N is None else N
    rows, keys = _rows_keys(w, N)
    size = rows[:, None] * keys[None, :]
    kept = (tiles * size).sum(axis=(-1, -2))
    return float(1.0 - kept.mean() / (w.L * w.L))


def random_tiles(B: int, H: int, QB: int, G: int, density: float, seed: int) -> np.ndarray:
    """Plain Bernoulli(density) tiles (fuzz cases; no diagonal added)."""
    rng = np.random.default_rng(_stream_seed(seed, "fuzz", B, H, QB, G, density))
    return rng.random((B, H, QB, G)) < density


def random_qkv(B: int, H: int, L: int, d: int, seed: int, std: float = 1.0):
    """iid N(0, std^2) bf16 tensors [B, H, L, d] (fuzz cases)."""
    g = _torch_gen(seed, "fuzzqkv", B, H, L, d)
    q = (torch.randn((B, H, L, d), generator=g) * std).to(torch.bfloat16)
    k = (torch.randn((B, H, L, d), generator=g) * std).to(torch.bfloat16)
    v = torch.randn((B, H, L, d), generator=g).to(torch.bfloat16)
    return q, k, v


def random_grad(B: int, H: int, L: int, d: int, seed: int, std: float = 1.0) -> torch.Tensor:
    """iid N(0, std^2) bf16 upstream gradient dO [B, H, L, d] (backward cases)."""
    g = _torch_gen(seed, "fuzzgrad", B, H, L, d)
    return (torch.randn((B, H, L, d), generator=g) * std).to(torch.bfloat16)
