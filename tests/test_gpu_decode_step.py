"""loki_decode_step: the rotated append of the step's new tokens folded into
the decode (GPU only).

With a signed-permutation basis P (orthonormal, and exact in any precision)
the rotated keys are exactly representable, so the whole step -- append and
decode -- is checked against the fp64 oracle with the parity tolerances. With
a calibrated basis the appended rows are checked against the oracle's
rotation (within one unit in the last place plus the fp32 summation bound),
and the step is checked against the separate append and decode entry points,
which it must reproduce bit for bit (same kernels, same arithmetic).
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


def _signed_permutation(H, D, seed):
    rng = np.random.default_rng(seed)
    P = np.zeros((H, D, D))
    for h in range(H):
        perm = rng.permutation(D)
        sign = rng.choice([-1.0, 1.0], D)
        P[h, perm, np.arange(D)] = sign  # column c = +-e_perm[c]
    return P


CASES = [
    # name, overrides, T, S_max, plane d_lo
    ("small-rows", dict(B=2, H_q=8, H_kv=4, S=1500, k=200), 1, 1536, None),
    ("small-plane", dict(B=2, H_q=8, H_kv=4, S=1500, k=200), 1, 1536, 32),
    ("split-plane", dict(B=4, H_q=8, H_kv=8, S=3000, k=400), 1, 3000, 32),
    ("split-rows-T4", dict(B=4, H_q=8, H_kv=8, S=3000, k=400), 4, 3100, None),
    ("gqa4-plane-T3", dict(B=2, H_q=16, H_kv=4, S=2049, d=16, k=300), 3, 2100, 16),
    ("f32-plane", dict(B=2, H_q=4, H_kv=2, S=700, k=90, dtype="f32"), 2, 720, 32),
    # 32 units: the append, then the one-kernel cluster decode behind it
    ("cluster-plane-T4", dict(B=2, H_q=32, H_kv=16, S=2500, k=300), 4, 2600, 32),
]


@pytest.mark.parametrize("name,over,T,S_max,d_lo", CASES, ids=[c[0] for c in CASES])
def test_decode_step_exact_basis_matches_oracle(loki, cuda, name, over, T, S_max, d_lo):
    import torch
    wl = workloads.get("llama2-7b").with_(n_cal=256, name=f"step-{name}", **over)
    g = workloads.generate(wl, with_cal=False)
    P = _signed_permutation(wl.H_kv, wl.D, 7)
    K, V = g["K"], g["V"]
    Kt = np.stack([[oracle.rotate_keys(K[b, h], P[h], wl.dtype) for h in range(wl.H_kv)]
                   for b in range(wl.B)])
    pos = wl.S - T
    dt = parity.torch_dtype(wl)
    # the cache holds rows [0, pos); rows [pos, S_max) hold a NaN sentinel
    Kc = torch.full((wl.B, wl.H_kv, S_max, wl.D), float("nan"), dtype=dt, device=cuda)
    Vc = torch.full_like(Kc, float("nan"))
    Kc[:, :, :pos] = torch.from_numpy(Kt[:, :, :pos].astype(np.float32)).to(cuda).to(dt)
    Vc[:, :, :pos] = torch.from_numpy(V[:, :, :pos]).to(cuda).to(dt)
    Klo = None
    if d_lo is not None:
        Klo = torch.full((wl.B, wl.H_kv, S_max, d_lo), float("nan"), dtype=dt, device=cuda)
        Klo[:, :, :pos] = Kc[:, :, :pos, :d_lo]
    K_new = torch.from_numpy(np.ascontiguousarray(K[:, :, pos:])).to(cuda).to(dt)
    V_new = torch.from_numpy(np.ascontiguousarray(V[:, :, pos:])).to(cuda).to(dt)
    q = torch.from_numpy(g["q"]).to(cuda).to(dt)
    Pt = torch.from_numpy(P.astype(np.float32)).to(cuda)
    out, idx = loki.loki_decode_step(q, K_new, V_new, Pt, Kc, Vc, pos, wl.d, wl.k, wl.scale,
                                     Kt_lo=Klo)
    torch.cuda.synchronize()
    assert loki.loki_device_error(reset=True) == 0, "a staged kernel's bounded wait gave up"
    # the appended rows are the oracle's rotation, exactly; the plane copies them
    got = Kc[:, :, pos:wl.S].float().cpu().numpy()
    np.testing.assert_array_equal(got, Kt[:, :, pos:].astype(np.float32))
    np.testing.assert_array_equal(Vc[:, :, pos:wl.S].float().cpu().numpy(), V[:, :, pos:])
    if Klo is not None:
        assert torch.equal(Klo[:, :, pos:wl.S], Kc[:, :, pos:wl.S, :d_lo])
    assert bool(torch.isnan(Kc[:, :, wl.S:].float()).all())
    # and the decode over all S rows is the oracle's
    inp = parity.HostInputs(wl, g["q"], K, V, P.astype(np.float32), None, Kt, None)
    out_h = out.float().cpu().numpy()
    idx_h = idx.cpu().numpy()
    checks = [parity.check_row(inp, b, h, idx_h[b, h], out_h[b, h], wl.d, wl.k, wl.scale)
              for b in range(wl.B) for h in range(wl.H_q)]
    assert parity.summarize(checks)["rows"] == wl.B * wl.H_q


SEPARATE = [
    # base workload, overrides, plane: 160 units (the staged kernels) and the
    # Llama2-7B shape, 32 units (append, then the cluster decode)
    ("llama2-13b", dict(B=4, S=4096), False),
    ("llama2-13b", dict(B=4, S=4096), True),
    ("llama2-7b", dict(B=1, S=4096), True),
]


@pytest.mark.parametrize("base,over,plane", SEPARATE,
                         ids=["13b-rows", "13b-plane", "7b-plane-cluster"])
def test_decode_step_equals_append_then_decode(loki, cuda, base, over, plane):
    import torch
    wl = workloads.get(base).with_(name=f"step-vs-separate-{base}", **over)
    inp = parity.host_inputs(wl)
    T, S_max = 1, 4100
    pos = wl.S - T
    dt = parity.torch_dtype(wl)
    P = torch.from_numpy(inp.P).to(cuda)
    base_K = parity.to_device(inp.Kt[:, :, :pos], wl, cuda, S_max=S_max)
    base_V = parity.to_device(inp.V[:, :, :pos], wl, cuda, S_max=S_max)
    K_new = parity.to_device(np.ascontiguousarray(inp.K[:, :, pos:]), wl, cuda)
    V_new = parity.to_device(np.ascontiguousarray(inp.V[:, :, pos:]), wl, cuda)
    q = parity.to_device(inp.q, wl, cuda)

    def plane_of(Kc):
        return Kc[..., :wl.d].contiguous() if plane else None

    # the step
    K1, V1 = base_K.clone(), base_V.clone()
    L1 = plane_of(K1)
    out1, idx1 = loki.loki_decode_step(q, K_new, V_new, P, K1, V1, pos, wl.d, wl.k, wl.scale,
                                       Kt_lo=L1)
    # the separate entry points
    K2, V2 = base_K.clone(), base_V.clone()
    L2 = plane_of(K2)
    loki.loki_append_keys(K_new, V_new, P, K2, V2, pos, Kt_lo=L2)
    out2, idx2 = loki.loki_decode_attention(q, K2, V2, P, wl.S, wl.d, wl.k, wl.scale, Kt_lo=L2)
    torch.cuda.synchronize()
    assert loki.loki_device_error(reset=True) == 0
    assert torch.equal(K1[:, :, :wl.S], K2[:, :, :wl.S]) and torch.equal(V1[:, :, :wl.S],
                                                                      V2[:, :, :wl.S])
    if plane:
        assert torch.equal(L1[:, :, :wl.S], L2[:, :, :wl.S])
    assert torch.equal(idx1, idx2)
    assert torch.equal(out1, out2)
    # the appended keys against the oracle's rotation: one unit in the last
    # place of bf16 plus the fp32 summation bound
    got = K1[:, :, pos:wl.S].float().cpu().numpy().astype(np.float64)
    exact = np.einsum("bhti,hic->bhtc", inp.K[:, :, pos:].astype(np.float64),
                      inp.P.astype(np.float64))
    want = oracle.round_to_dtype(exact, "bf16")
    sum_abs = np.einsum("bhti,hic->bhtc", np.abs(inp.K[:, :, pos:].astype(np.float64)),
                        np.abs(inp.P.astype(np.float64)))
    tol = np.abs(want) * 2.0 ** -7 + 128 * 2.0 ** -24 * sum_abs + 1e-30
    assert np.all(np.abs(got - want) <= tol)


def test_decode_step_rejects_bad_arguments(loki, cuda):
    import torch
    dt = torch.bfloat16
    q = torch.zeros((1, 2, 128), dtype=dt, device=cuda)
    Kc = torch.zeros((1, 2, 64, 128), dtype=dt, device=cuda)
    P = torch.zeros((2, 128, 128), dtype=torch.float32, device=cuda)
    Kn = torch.zeros((1, 2, 1, 128), dtype=dt, device=cuda)
    with pytest.raises(ValueError):  # pos + T beyond S_max
        loki.loki_decode_step(q, Kn, Kn, P, Kc, Kc.clone(), 64, 8, 4)
    with pytest.raises(loki.LokiError) as e:  # k > S
        loki.loki_decode_step(q, Kn, Kn, P, Kc, Kc.clone(), 2, 8, 4)
    assert e.value.status == 1
