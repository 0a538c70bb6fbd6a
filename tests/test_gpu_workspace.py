"""Plane decodes on workspaces that hold leftovers (GPU only).

The decode writes every scratch word it reads (the query projection zeroes
the attention kernel's row counters each call), so whatever the workspace
held before must not matter: all bytes 0xFF, an int32 ramp (a counter and its
neighbour then look like consecutive values), or the state the previous call
left (two calls in a row must agree bit for bit). The shapes take the
multi-kernel path (at least two rows per SM): units scored by one CTA and
units split over several, grouped query heads and fp32. Every row is checked
against the fp64 oracle.
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
    ("mha-320-rows", dict(B=8, H_q=40, H_kv=40, S=2048, d=32, k=256), 32, 2048),
    ("g5-units-over-cta", dict(B=4, H_q=80, H_kv=16, S=8192, d=8, k=64), 8, 8192),
    ("gqa4-odd-S", dict(B=80, H_q=8, H_kv=2, S=1537, d=16, k=200), 16, 1600),
    ("f32", dict(B=150, H_q=2, H_kv=2, S=700, d=20, k=90, dtype="f32"), 32, 720),
]
FILLS = ["ff", "ramp", "twice"]


def _fill(ws, how):
    import torch
    if how == "ff":
        ws.fill_(0xFF)
    elif how == "ramp":
        n = ws.numel() // 4
        ws[: 4 * n].view(torch.int32).copy_(torch.arange(n, dtype=torch.int32, device=ws.device))


@pytest.mark.parametrize("fill", FILLS)
@pytest.mark.parametrize("name,over,d_lo,S_max", CASES, ids=[c[0] for c in CASES])
def test_decode_on_used_workspace_matches_oracle(loki, cuda, name, over, d_lo, S_max, fill):
    import torch
    wl = workloads.get("llama2-7b").with_(n_cal=512, name=f"ws-{name}", **over)
    inp = parity.host_inputs(wl)
    q = parity.to_device(inp.q, wl, cuda)
    Kt = parity.to_device(inp.Kt, wl, cuda, S_max=S_max)
    V = parity.to_device(inp.V, wl, cuda, S_max=S_max)
    Klo = Kt[..., :d_lo].contiguous()
    P = torch.from_numpy(inp.P).to(cuda)
    nbytes = loki.loki_decode_workspace_size(wl.B, wl.H_q, wl.H_kv, wl.S, 128, wl.d, wl.k)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=cuda)
    _fill(ws, fill)
    calls = 2 if fill == "twice" else 1
    outs = []
    for _ in range(calls):
        out, idx = loki.loki_decode_attention_plane(q, Kt, V, Klo, P, wl.S, wl.d, wl.k, wl.scale,
                                                    workspace=ws)
        torch.cuda.synchronize()
        assert loki.loki_device_error(reset=True) == 0
        outs.append((out.clone(), idx.clone()))
    if calls == 2:
        assert torch.equal(outs[0][1], outs[1][1])
        assert torch.equal(outs[0][0], outs[1][0])
    out_h, idx_h = outs[-1][0].float().cpu().numpy(), outs[-1][1].cpu().numpy()
    checks = [parity.check_row(inp, b, h, idx_h[b, h], out_h[b, h], wl.d, wl.k, wl.scale)
              for b in range(wl.B) for h in range(wl.H_q)]
    assert parity.summarize(checks)["rows"] == wl.B * wl.H_q
