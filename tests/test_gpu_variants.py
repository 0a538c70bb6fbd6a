"""Variants of the method (GPU only): PCAAttn against the fp64 oracle.

PCAAttn (poster page, "More on tables", PCAAttn table caption) applies the
softmax to the reduced-dimensional scores of every token; the oracle's
pca_attn_row, pinned by the hand-worked fixture, is its definition. Every row
is checked with the parity tolerance of the cache type.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workloads
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def loki(cuda):
    import sparse_attention_decode_loki_b200 as m
    return m


PCA_CASES = [
    # name, base, overrides, d_lo, S_max
    ("tiny-f32", "tiny", {}, 32, 300),
    ("bf16-d32", "llama2-7b", dict(B=2, H_q=4, H_kv=4, S=3000, d=32), 32, 3000),
    ("bf16-d20-plane32", "llama2-7b", dict(B=1, H_q=2, H_kv=2, S=1500, d=20), 32, 1600),
    ("gqa4-d16", "llama2-7b", dict(B=2, H_q=8, H_kv=2, S=2049, d=16), 16, 2100),
    ("bf16-d64", "llama2-7b", dict(B=1, H_q=2, H_kv=2, S=777, d=64), 64, 800),
]


@pytest.mark.parametrize("name,base,over,d_lo,S_max", PCA_CASES, ids=[c[0] for c in PCA_CASES])
def test_pca_attention_matches_oracle(loki, cuda, name, base, over, d_lo, S_max):
    import torch
    wl = workloads.get(base)
    if over:
        wl = wl.with_(n_cal=512, name=f"pca-{name}", **over)
    inp = parity.host_inputs(wl)
    q = parity.to_device(inp.q, wl, cuda)
    V = parity.to_device(inp.V, wl, cuda, S_max=S_max)
    Klo = parity.to_device(inp.Kt[:, :, :, :d_lo], wl, cuda, S_max=S_max)
    P = torch.from_numpy(inp.P).to(cuda)
    out = loki.loki_pca_attention(q, Klo, V, P, wl.S, wl.d, wl.scale)
    out = out.float().cpu().numpy()
    err = 0.0
    for b in range(wl.B):
        for h in range(wl.H_q):
            hk = h // wl.G
            ref = oracle.pca_attn_row(inp.q[b, h].astype(np.float64), inp.Kt[b, hk].astype(np.float64),
                                      inp.V[b, hk].astype(np.float64),
                                      inp.P[hk].astype(np.float64), wl.d, wl.scale)
            err = max(err, float(np.abs(out[b, h] - ref).max()))
    assert err <= parity.OUT_TOL[wl.dtype], err
