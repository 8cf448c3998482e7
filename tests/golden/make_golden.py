"""Write tests/golden/oracle_tiny.json from the CPU oracle alone.

Run from the repository root:  python tests/golden/make_golden.py
The fixture is a regression pin for the oracle (stored inputs as bf16 bit
patterns, stored outputs in float64) and a tiny GPU parity case (d=64, M=16,
N=3, L=40: three query blocks, a 14-group ragged key axis, a ragged last query
block).  Tile-skipping semantics: "FG-Attn: Leveraging Fine-Grained Sparse
Attention in Video Diffusion Models", Abstract.
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
import workloads as W  # noqa: E402

L, d, M, N, scale = 40, 64, 16, 3, 0.125


def main():
    q, k, v = W.random_qkv(1, 1, L, d, seed=2024)
    QB, G = -(-L // M), -(-L // N)
    tiles = W.random_tiles(1, 1, QB, G, 0.3, seed=2025)
    mask = W.pack_tiles(tiles)
    orc = O.Oracle()
    out, lse = orc.attention(q, k, v, mask, M, N, scale, nthreads=1)
    idx, cnt = orc.compact(mask, 1, 1, L, M, N)
    bits = lambda t: O._bits(t).reshape(-1).astype(int).tolist()
    fx = {
        "about": "oracle regression fixture; tile skipping per the FG-Attn page, Abstract",
        "B": 1, "H": 1, "L": L, "d": d, "M": M, "N": N, "scale": scale,
        "q_bf16_bits": bits(q), "k_bf16_bits": bits(k), "v_bf16_bits": bits(v),
        "mask_u32": mask.reshape(-1).astype(int).tolist(),
        "kept_cnt": cnt.reshape(-1).astype(int).tolist(),
        "kept_idx": [idx[0, 0, r, :cnt[0, 0, r]].astype(int).tolist() for r in range(QB)],
        "out": [[float(x) for x in row] for row in out.reshape(QB * M, d)[:L]],
        "lse": [float(x) for x in lse.reshape(-1)[:L]],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json")
    with open(path, "w") as f:
        json.dump(fx, f, separators=(",", ":"))
    print("wrote", path)


if __name__ == "__main__":
    main()
