"""The fused single-kernel decode (loki_decode_attention_fused) against the
fp64 oracle on the same seeded inputs, every row checked; plus its agreement
with the split pipeline and its shape limits (GPU only).

Tolerances are those of tests/parity.py: bit-exact selections outside the
tie band of the k-th low-dimensional score, outputs within 2e-2 (bf16) or
1e-4 (fp32) max-abs.
"""
from __future__ import annotations

import numpy as np
import pytest

import workloads
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def loki(cuda):
    import sparse_attention_decode_loki_b200 as m
    return m


def _upload(inp, dev, S, S_max, d_lo):
    import torch
    wl = inp.wl
    q = parity.to_device(inp.q, wl, dev)
    Kt = parity.to_device(inp.Kt[:, :, :S], wl, dev, S_max=S_max)
    V = parity.to_device(inp.V[:, :, :S], wl, dev, S_max=S_max)
    Kt_lo = parity.to_device(inp.Kt[:, :, :S, :d_lo], wl, dev, S_max=S_max)
    P = torch.from_numpy(inp.P).to(dev)
    return q, Kt, V, Kt_lo, P


def run_fused(loki, inp, dev, d_lo, S_max=None):
    import torch
    wl = inp.wl
    S_max = wl.S if S_max is None else S_max
    q, Kt, V, Kt_lo, P = _upload(inp, dev, wl.S, S_max, d_lo)
    out, idx = loki.loki_decode_attention_fused(q, Kt, V, Kt_lo, P, wl.S, wl.d, wl.k, wl.scale)
    torch.cuda.synchronize()
    assert loki.loki_device_error(reset=True) == 0, "a staged kernel's bounded wait gave up"
    return out.float().cpu().numpy(), idx.cpu().numpy()


def check_all(inp, out, idx):
    wl = inp.wl
    checks = [parity.check_row(inp, b, h, idx[b, h], out[b, h], wl.d, wl.k, wl.scale)
              for b in range(wl.B) for h in range(wl.H_q)]
    return parity.summarize(checks)


CASES = [
    # name, workload, overrides, d_lo, S_max
    ("tiny-f32", "tiny", {}, 32, 300),
    ("llama2-7b", "llama2-7b", {}, 32, None),
    ("llama2-13b", "llama2-13b", {}, 32, None),
    ("ragged-S-d20", "llama2-7b", dict(B=2, H_q=2, H_kv=2, S=1000, d=20, k=77), 32, 1024),
    ("k1", "llama2-7b", dict(B=1, H_q=2, H_kv=2, S=513, k=1), 32, 600),
    ("k-all", "llama2-7b", dict(B=1, H_q=2, H_kv=2, S=300, k=300), 32, 300),
    ("S1", "llama2-7b", dict(B=1, H_q=2, H_kv=2, S=1, k=1), 32, 8),
    ("d1-plane8", "llama2-7b", dict(B=1, H_q=2, H_kv=2, S=700, d=1, k=64), 8, 700),
    ("d64-plane64", "llama2-7b", dict(B=1, H_q=2, H_kv=2, S=640, d=64, k=100), 64, 700),
    ("d16-plane16", "llama2-7b", dict(B=2, H_q=2, H_kv=2, S=1200, d=16, k=150), 16, 1280),
    ("gqa2-B3", "llama2-7b", dict(B=3, H_q=4, H_kv=2, S=333, k=50), 32, 400),
    ("gqa4", "llama2-7b", dict(B=2, H_q=8, H_kv=2, S=2049, d=16, k=128), 16, 2100),
    ("gqa8", "llama2-7b", dict(B=1, H_q=16, H_kv=2, S=1500, d=24, k=200), 32, 1500),
    ("S-max-8192", "llama2-7b", dict(B=1, H_q=2, H_kv=2, S=8192, k=1024), 32, 8192),
    ("f32-d8-plane8", "tiny", dict(B=2, H_q=2, H_kv=2, S=777, d=8, k=99), 8, 800),
    ("f32-gqa4-plane16", "tiny", dict(B=1, H_q=8, H_kv=2, S=1030, d=13, k=40), 16, 1030),
    ("f32-plane4", "tiny", dict(S=256, d=3, k=10), 4, 256),
]


@pytest.mark.parametrize("name,base,over,d_lo,S_max", CASES, ids=[c[0] for c in CASES])
def test_fused_matches_oracle(loki, cuda, name, base, over, d_lo, S_max):
    wl = workloads.get(base)
    if over:
        wl = wl.with_(n_cal=min(wl.n_cal, 1024), name=f"fused-{name}", **over)
    inp = parity.host_inputs(wl)
    out, idx = run_fused(loki, inp, cuda, d_lo, S_max)
    s = check_all(inp, out, idx)
    assert s["rows"] == wl.B * wl.H_q


def test_fused_agrees_with_split_pipeline(loki, cuda):
    """Same inputs through the split four-kernel path (this shape has too few
    units for the automatic choice to fuse it): same selection outside the
    tie band, outputs within the tolerance."""
    wl = workloads.get("llama2-7b").with_(B=2, H_q=8, H_kv=4, S=3000, k=300, n_cal=1024,
                                          name="fused-vs-split")
    inp = parity.host_inputs(wl)
    q, Kt, V, Kt_lo, P = _upload(inp, cuda, wl.S, wl.S, 32)
    of, i_f = loki.loki_decode_attention_fused(q, Kt, V, Kt_lo, P, wl.S, wl.d, wl.k, wl.scale)
    os_, i_s = loki.loki_decode_attention_plane(q, Kt, V, Kt_lo, P, wl.S, wl.d, wl.k, wl.scale)
    of, os_ = of.float().cpu().numpy(), os_.float().cpu().numpy()
    i_f, i_s = i_f.cpu().numpy(), i_s.cpu().numpy()
    same = sum(np.array_equal(i_f[b, h], i_s[b, h]) for b in range(wl.B) for h in range(wl.H_q))
    assert same >= wl.B * wl.H_q - 2, same
    assert np.abs(of - os_).max() <= parity.OUT_TOL[wl.dtype]
    # and both against the oracle
    for b in range(wl.B):
        for h in range(wl.H_q):
            parity.check_row(inp, b, h, i_f[b, h], of[b, h], wl.d, wl.k, wl.scale)


def test_fused_repeated_calls_are_identical(loki, cuda):
    wl = workloads.get("llama2-7b").with_(B=2, H_q=4, H_kv=4, S=2000, k=256, n_cal=512,
                                          name="fused-repeat")
    inp = parity.host_inputs(wl)
    q, Kt, V, Kt_lo, P = _upload(inp, cuda, wl.S, wl.S, 32)
    a = loki.loki_decode_attention_fused(q, Kt, V, Kt_lo, P, wl.S, wl.d, wl.k, wl.scale)
    b = loki.loki_decode_attention_fused(q, Kt, V, Kt_lo, P, wl.S, wl.d, wl.k, wl.scale)
    assert (a[0] == b[0]).all() and (a[1] == b[1]).all()


@pytest.mark.parametrize("over,d_lo", [
    (dict(H_q=6, H_kv=2), 32),      # G = 3
    (dict(S=8193, k=10), 32),       # beyond the one-CTA top-k
    (dict(S=500, k=10), 128),       # 256-byte plane rows
])
def test_fused_rejects_unsupported_shapes(loki, cuda, over, d_lo):
    import torch
    a = dict(B=1, H_q=2, H_kv=2, S=500, k=10)
    a.update(over)
    dt = torch.bfloat16
    q = torch.zeros((a["B"], a["H_q"], 128), dtype=dt, device=cuda)
    Kt = torch.zeros((a["B"], a["H_kv"], a["S"], 128), dtype=dt, device=cuda)
    Kt_lo = torch.zeros((a["B"], a["H_kv"], a["S"], d_lo), dtype=dt, device=cuda)
    P = torch.zeros((a["H_kv"], 128, 128), dtype=torch.float32, device=cuda)
    with pytest.raises(loki.LokiError) as e:
        loki.loki_decode_attention_fused(q, Kt, Kt, Kt_lo, P, a["S"], 8, a["k"])
    assert e.value.status == 2
