"""Decodes whose attention reuses the scan's low-dimensional scores (GPU only).

When d covers at least half the head dimension, the attention kernel adds the
score the scan stored for each selected token (its products over the first d
columns) and reads only the key columns [d, D). These cases take the
multi-kernel path (top-k, then the gather) with d = D / 2 and above: the key
plane and the row layout, bf16 and fp32, a d that is not a multiple of a
16-byte chunk (no reuse), grouped query heads and a ragged split of the
selection over many warps. Every row is checked against the fp64 oracle.
"""
from __future__ import annotations

import pytest

import workloads
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def loki(cuda):
    import sparse_attention_decode_loki_b200 as m
    return m


CASES = [
    # name, overrides, plane d_lo (None: row layout), S_max
    ("plane-d64", dict(B=2, H_q=4, H_kv=4, S=3000, d=64, k=1200), 64, 3000),
    ("rows-d64", dict(B=2, H_q=4, H_kv=4, S=3000, d=64, k=1200), None, 3100),
    ("plane-d96-gqa2", dict(B=2, H_q=8, H_kv=4, S=2049, d=96, k=700), 128, 2100),
    ("plane-d68", dict(B=2, H_q=4, H_kv=4, S=1500, d=68, k=1100), 128, 1500),
    ("f32-rows-d64", dict(B=4, H_q=4, H_kv=2, S=700, d=64, k=600, dtype="f32"), None, 720),
    ("many-warps", dict(B=8, H_q=40, H_kv=40, S=2048, d=64, k=256), 64, 2048),
]


@pytest.mark.parametrize("name,over,d_lo,S_max", CASES, ids=[c[0] for c in CASES])
def test_decode_with_stored_scores_matches_oracle(loki, cuda, name, over, d_lo, S_max):
    import torch
    wl = workloads.get("llama2-7b").with_(n_cal=512, name=f"reuse-{name}", **over)
    inp = parity.host_inputs(wl)
    q = parity.to_device(inp.q, wl, cuda)
    Kt = parity.to_device(inp.Kt, wl, cuda, S_max=S_max)
    V = parity.to_device(inp.V, wl, cuda, S_max=S_max)
    P = torch.from_numpy(inp.P).to(cuda)
    if d_lo is None:
        out, idx = loki.loki_decode_attention(q, Kt, V, P, wl.S, wl.d, wl.k, wl.scale)
    else:
        Klo = Kt[..., :d_lo].contiguous()
        out, idx = loki.loki_decode_attention_plane(q, Kt, V, Klo, P, wl.S, wl.d, wl.k, wl.scale)
    torch.cuda.synchronize()
    assert loki.loki_device_error(reset=True) == 0
    out_h, idx_h = out.float().cpu().numpy(), idx.cpu().numpy()
    checks = [parity.check_row(inp, b, h, idx_h[b, h], out_h[b, h], wl.d, wl.k, wl.scale)
              for b in range(wl.B) for h in range(wl.H_q)]
    assert parity.summarize(checks)["rows"] == wl.B * wl.H_q
