"""Stored oracle outputs (written by tests/golden/make_golden.py) still reproduce."""
import json
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def load_fixture():
    with open(os.path.join(HERE, "golden", "oracle_tiny.json")) as f:
        fx = json.load(f)
    shape = (fx["B"], fx["H"], fx["L"], fx["d"])
    arr = lambda key: np.array(fx[key], dtype=np.uint16).reshape(shape)
    return fx, arr("q_bf16_bits"), arr("k_bf16_bits"), arr("v_bf16_bits"), np.array(fx["mask_u32"], dtype=np.uint32)


def test_golden_oracle(oracle):
    fx, q, k, v, mask = load_fixture()
    out, lse = oracle.attention(q, k, v, mask, fx["M"], fx["N"], fx["scale"])
    L, d, M = fx["L"], fx["d"], fx["M"]
    out = out.reshape(-1, d)[:L]
    lse = lse.reshape(-1)[:L]
    assert np.abs(out - np.array(fx["out"])).max() < 1e-12
    assert np.abs(lse - np.array(fx["lse"])).max() < 1e-12
    idx, cnt = oracle.compact(mask, 1, 1, L, M, fx["N"])
    assert cnt.reshape(-1).tolist() == fx["kept_cnt"]
    for r, lst in enumerate(fx["kept_idx"]):
        assert idx[0, 0, r, :len(lst)].tolist() == lst
