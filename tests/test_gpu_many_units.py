"""Plane decodes with many (batch, KV head) units (GPU only).

At least one unit per SM, so the score scan's even split of rows over one
wave of CTAs cuts units between CTAs at arbitrary rows. These cases cover
grouped query heads, an odd row length (scalar score loads in top-k), fp32,
8-column planes with eight query heads per KV head and k = S, each row
checked against the fp64 oracle.
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
    # name, overrides, d_lo, S_max
    ("mha-160-units", dict(B=4, H_q=40, H_kv=40, S=1000, d=32, k=100), 32, 1024),
    ("gqa4-odd-S", dict(B=40, H_q=16, H_kv=4, S=2049, d=16, k=300), 16, 2100),
    ("f32", dict(B=75, H_q=2, H_kv=2, S=700, d=20, k=90, dtype="f32"), 32, 720),
    ("k-equals-S", dict(B=150, H_q=1, H_kv=1, S=64, d=8, k=64), 16, 64),
    ("max-S", dict(B=150, H_q=2, H_kv=1, S=4096, d=32, k=30), 32, 4096),
    ("g8-d8", dict(B=20, H_q=64, H_kv=8, S=513, d=8, k=50), 8, 520),
]


@pytest.mark.parametrize("name,over,d_lo,S_max", CASES, ids=[c[0] for c in CASES])
def test_many_unit_decode_matches_oracle(loki, cuda, name, over, d_lo, S_max):
    import torch
    wl = workloads.get("llama2-7b").with_(n_cal=512, name=f"units-{name}", **over)
    inp = parity.host_inputs(wl)
    q = parity.to_device(inp.q, wl, cuda)
    Kt = parity.to_device(inp.Kt, wl, cuda, S_max=S_max)
    V = parity.to_device(inp.V, wl, cuda, S_max=S_max)
    Klo = Kt[..., :d_lo].contiguous()
    P = torch.from_numpy(inp.P).to(cuda)
    out, idx = loki.loki_decode_attention_plane(q, Kt, V, Klo, P, wl.S, wl.d, wl.k, wl.scale)
    torch.cuda.synchronize()
    assert loki.loki_device_error(reset=True) == 0
    out_h, idx_h = out.float().cpu().numpy(), idx.cpu().numpy()
    checks = [parity.check_row(inp, b, h, idx_h[b, h], out_h[b, h], wl.d, wl.k, wl.scale)
              for b in range(wl.B) for h in range(wl.H_q)]
    assert parity.summarize(checks)["rows"] == wl.B * wl.H_q
