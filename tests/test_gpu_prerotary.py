"""The pre-rotary variant (GPU only) against the fp64 oracle.

The basis is calibrated on the generated keys, which play the pre-rotary
keys; the rotary embedding of the input generator makes the post-rotary keys
(token positions 0 .. S-1) and query (position S-1) from them. The cache holds
the rotated pre-rotary keys' plane and the post-rotary keys; the selection is
checked outside the tie band of the pre-rotary scores and the output against
the attention of the post-rotary query over the oracle's selection.
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


def _post_rotary(inp, wl):
    """Post-rotary keys [B, H_kv, S, D] and queries [B, H_q, D], rounded to the cache type."""
    K_post = workloads.rope(inp.K, np.arange(wl.S), dtype=wl.dtype)
    q_post = workloads.rope(inp.q[:, :, None, :], [wl.S - 1], dtype=wl.dtype)[:, :, 0]
    return K_post, q_post


CASES = [
    # name, base, overrides, d_lo, S_max
    ("bf16-fused-scan", "llama2-7b", dict(B=2, H_q=8, H_kv=8, S=3000, d=32, k=400), 32, 3000),
    ("gqa4", "llama2-7b", dict(B=2, H_q=16, H_kv=4, S=2049, d=16, k=300), 16, 2100),
    ("d96-unfused", "llama2-7b", dict(B=2, H_q=8, H_kv=4, S=1500, d=32, k=200, D=96), 32, 1600),
    ("f32", "tiny", {}, 32, 300),
]


@pytest.mark.parametrize("name,base,over,d_lo,S_max", CASES, ids=[c[0] for c in CASES])
def test_prerotary_decode_matches_oracle(loki, cuda, name, base, over, d_lo, S_max):
    import torch
    wl = workloads.get(base)
    if over:
        wl = wl.with_(n_cal=512, name=f"prerot-{name}", **over)
    inp = parity.host_inputs(wl)
    K_post, q_post = _post_rotary(inp, wl)
    q = parity.to_device(inp.q, wl, cuda)
    qp = parity.to_device(q_post, wl, cuda)
    Kc = parity.to_device(K_post, wl, cuda, S_max=S_max)
    V = parity.to_device(inp.V, wl, cuda, S_max=S_max)
    Klo = parity.to_device(inp.Kt[..., :d_lo], wl, cuda, S_max=S_max)
    P = torch.from_numpy(inp.P).to(cuda)
    out, idx = loki.loki_decode_attention_prerotary(q, qp, Kc, V, Klo, P, wl.S, wl.d, wl.k,
                                                    wl.scale)
    torch.cuda.synchronize()
    assert loki.loki_device_error(reset=True) == 0
    out_h, idx_h = out.float().cpu().numpy(), idx.cpu().numpy()
    checks = [parity.check_row(inp, b, h, idx_h[b, h], out_h[b, h], wl.d, wl.k, wl.scale,
                               attend_with=(q_post[b, h], K_post[b, h // wl.G]))
              for b in range(wl.B) for h in range(wl.H_q)]
    assert parity.summarize(checks)["rows"] == wl.B * wl.H_q


def test_prerotary_append(loki, cuda):
    import torch
    wl = workloads.get("llama2-7b").with_(B=2, H_q=4, H_kv=4, S=300, n_cal=512, name="prerot-app")
    inp = parity.host_inputs(wl)
    T, pos, S_max, d_lo = 3, 100, 128, 32
    rng = np.random.default_rng(8)
    K_pre = workloads.to_cache_dtype(rng.standard_normal((2, 4, T, 128)), "bf16")
    K_post = workloads.rope(K_pre, np.arange(pos, pos + T), dtype="bf16")
    V_new = workloads.to_cache_dtype(rng.standard_normal((2, 4, T, 128)), "bf16")
    dt = torch.bfloat16
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(cuda).to(dt)  # noqa: E731
    Kc = torch.full((2, 4, S_max, 128), 7.0, dtype=dt, device=cuda)
    Vc = torch.full_like(Kc, 5.0)
    Klo = torch.full((2, 4, S_max, d_lo), 3.0, dtype=dt, device=cuda)
    P = torch.from_numpy(inp.P).to(cuda)
    loki.loki_append_keys_prerotary(t(K_pre), t(K_post), t(V_new), P, Kc, Vc, Klo, pos)
    torch.cuda.synchronize()
    assert loki.loki_device_error(reset=True) == 0
    rows = slice(pos, pos + T)
    np.testing.assert_array_equal(Kc[:, :, rows].float().cpu().numpy(), K_post)
    np.testing.assert_array_equal(Vc[:, :, rows].float().cpu().numpy(), V_new)
    got = Klo[:, :, rows].float().cpu().numpy().astype(np.float64)
    P64 = inp.P.astype(np.float64)
    exact = np.einsum("bhti,hic->bhtc", K_pre.astype(np.float64), P64)[..., :d_lo]
    want = oracle.round_to_dtype(exact, "bf16")
    sum_abs = np.einsum("bhti,hic->bhtc", np.abs(K_pre.astype(np.float64)), np.abs(P64))[..., :d_lo]
    assert np.all(np.abs(got - want) <= np.abs(want) * 2.0 ** -7 + 128 * 2.0 ** -24 * sum_abs
                  + 1e-30)
    # nothing else written
    mask = torch.ones(S_max, dtype=torch.bool)
    mask[rows] = False
    assert bool((Kc[:, :, mask] == 7.0).all()) and bool((Vc[:, :, mask] == 5.0).all())
    assert bool((Klo[:, :, mask] == 3.0).all())
