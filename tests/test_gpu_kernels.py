"""Unit tests of single steps through the C ABI (GPU only): top-k on
adversarial rows, sparse attention on hand-made selections, the rotated
append and the PCA calibration, each against the fp64 oracle.
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


def _t():
    import torch
    return torch


# ---------------------------------------------------------------------------
# top-k: exact integer decisions, compared bit for bit
# ---------------------------------------------------------------------------

def _adversarial_rows(S, seed):
    rng = np.random.default_rng(seed)
    rows = [
        np.zeros(S),                                   # all equal
        np.arange(S, dtype=np.float64),                # ascending
        -np.arange(S, dtype=np.float64),               # descending
        rng.integers(-3, 4, S).astype(np.float64),     # heavy ties
        rng.standard_normal(S),                        # generic
        np.where(rng.random(S) < 0.5, 0.0, -0.0),      # signed zeros only
        rng.standard_normal(S) * 1e-30,                # subnormal-range fp32 values
        np.concatenate([np.full(S // 2, 7.0), rng.standard_normal(S - S // 2)]),
    ]
    r = rng.standard_normal(S)
    r[rng.random(S) < 0.2] = np.nan                    # NaN ranks with -inf
    r[rng.random(S) < 0.1] = -np.inf
    r[rng.random(S) < 0.05] = np.inf
    rows.append(r)
    return np.stack(rows).astype(np.float32)


@pytest.mark.parametrize("S", [1, 7, 32, 100, 1000, 4096, 4099, 33000, 60001])
def test_topk_exact(loki, cuda, S):
    torch = _t()
    rows = _adversarial_rows(S, S)
    dev_scores = torch.from_numpy(rows).to(cuda)
    for k in sorted({min(S, 2), 1, max(1, S // 8), max(1, S // 2), max(1, S - 1), S}):
        got = loki.loki_topk(dev_scores, k).cpu().numpy()
        for i, r in enumerate(rows):
            want = oracle.select_topk(r.astype(np.float64), k)
            assert np.array_equal(got[i], want), (S, k, i)


# ---------------------------------------------------------------------------
# sparse attention on hand-made selections
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_sparse_single_token_returns_its_value(loki, cuda, dtype):
    torch = _t()
    wl = workloads.get("llama2-7b").with_(B=2, H_q=4, H_kv=2, S=500, dtype=dtype, n_cal=256,
                                          name=f"sparse-k1-{dtype}")
    inp = parity.host_inputs(wl)
    q_rot = torch.from_numpy(np.random.default_rng(1).standard_normal((2, 4, 128))
                             .astype(np.float32)).to(cuda)
    Kt = parity.to_device(inp.Kt, wl, cuda)
    V = parity.to_device(inp.V, wl, cuda)
    pick = np.array([[[3], [499], [0], [250]], [[17], [17], [100], [5]]], dtype=np.int32)
    out = loki.loki_sparse_attention(q_rot, Kt, V, torch.from_numpy(pick).to(cuda), wl.S)
    out = out.float().cpu().numpy()
    for b in range(2):
        for h in range(4):
            assert np.array_equal(out[b, h], inp.V[b, h // 2, pick[b, h, 0]])


def test_sparse_skips_out_of_range_indices(loki, cuda):
    torch = _t()
    wl = workloads.get("llama2-7b").with_(B=1, H_q=2, H_kv=2, S=300, n_cal=256, name="sparse-oob")
    inp = parity.host_inputs(wl)
    rng = np.random.default_rng(2)
    q_rot = rng.standard_normal((1, 2, 128)).astype(np.float32)
    idx = np.array([[[5, -1, 40, 299, 300, 77, 1 << 30, 12]] * 2], dtype=np.int32).reshape(1, 2, 8)
    idx[0, 1, :] = -7  # a row with no valid index yields zeros
    out = loki.loki_sparse_attention(torch.from_numpy(q_rot).to(cuda),
                                     parity.to_device(inp.Kt, wl, cuda),
                                     parity.to_device(inp.V, wl, cuda),
                                     torch.from_numpy(idx).to(cuda), wl.S, wl.scale)
    out = out.float().cpu().numpy()
    valid = np.array([5, 40, 299, 77, 12])
    ref = oracle.attend(q_rot[0, 0].astype(np.float64), inp.Kt[0, 0].astype(np.float64),
                        inp.V[0, 0].astype(np.float64), valid, wl.scale)
    assert np.abs(out[0, 0] - ref).max() < 2e-2
    assert np.all(out[0, 1] == 0)


@pytest.mark.parametrize("k", [1, 31, 64, 65, 700, 4096])
def test_sparse_split_sizes(loki, cuda, k):
    """Many split shapes: k below, at and above a CTA's share, rows spanning CTAs."""
    torch = _t()
    wl = workloads.get("llama2-7b").with_(B=3, H_q=6, H_kv=3, S=4096, n_cal=256,
                                          name="sparse-splits")
    inp = parity.host_inputs(wl)
    rng = np.random.default_rng(k)
    q_rot = rng.standard_normal((3, 6, 128)).astype(np.float32)
    idx = np.sort(np.stack([[rng.choice(wl.S, k, replace=False) for _ in range(6)]
                            for _ in range(3)]), axis=-1).astype(np.int32)
    out = loki.loki_sparse_attention(torch.from_numpy(q_rot).to(cuda),
                                     parity.to_device(inp.Kt, wl, cuda),
                                     parity.to_device(inp.V, wl, cuda),
                                     torch.from_numpy(idx).to(cuda), wl.S, wl.scale)
    out = out.float().cpu().numpy()
    for b in range(3):
        for h in range(6):
            ref = oracle.attend(q_rot[b, h].astype(np.float64), inp.Kt[b, h // 2].astype(np.float64),
                                inp.V[b, h // 2].astype(np.float64), idx[b, h], wl.scale)
            assert np.abs(out[b, h] - ref).max() < 2e-2, (b, h)


# ---------------------------------------------------------------------------
# append: K~ = round(K P) into the cache, V copied, other rows untouched
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("T,pos", [(1, 0), (1, 777), (13, 100), (64, 936)])
def test_append_matches_oracle_rotation(loki, cuda, dtype, T, pos):
    torch = _t()
    wl = workloads.get("llama2-7b").with_(B=2, H_q=3, H_kv=3, S=T, dtype=dtype, n_cal=512,
                                          name=f"append-{dtype}-{T}")
    inp = parity.host_inputs(wl)
    S_max = 1000
    dt = parity.torch_dtype(wl)
    Kc = torch.full((2, 3, S_max, 128), 3.0, dtype=dt, device=cuda)
    Vc = torch.full((2, 3, S_max, 128), -5.0, dtype=dt, device=cuda)
    P = torch.from_numpy(inp.P).to(cuda)
    loki.loki_append_keys(parity.to_device(inp.K, wl, cuda), parity.to_device(inp.V, wl, cuda), P,
                          Kc, Vc, pos)
    Kc = Kc.float().cpu().numpy()
    Vc = Vc.float().cpu().numpy()
    got = Kc[:, :, pos:pos + T]
    exact = np.einsum("bhti,hic->bhtc", inp.K.astype(np.float64), inp.P.astype(np.float64))
    want = oracle.round_to_dtype(exact, dtype)
    # one unit in the last place of the cache type, plus the fp32 summation bound
    ulp = np.abs(want) * (2.0 ** -7 if dtype == "bf16" else 2.0 ** -23)
    sum_abs = np.einsum("bhti,hic->bhtc", np.abs(inp.K.astype(np.float64)),
                        np.abs(inp.P.astype(np.float64)))
    tol = ulp + 128 * 2.0 ** -24 * sum_abs + 1e-30
    assert np.all(np.abs(got - want) <= tol)
    if dtype == "bf16":
        assert np.mean(got == want) > 0.98
    assert np.array_equal(Vc[:, :, pos:pos + T], inp.V)
    mask = np.ones(S_max, bool)
    mask[pos:pos + T] = False
    assert np.all(Kc[:, :, mask] == 3.0) and np.all(Vc[:, :, mask] == -5.0)
    # rotating back recovers the raw keys up to the cache rounding
    back = np.einsum("bhtc,hic->bhti", got.astype(np.float64), inp.P.astype(np.float64))
    assert np.abs(back - inp.K).max() < (0.05 if dtype == "bf16" else 1e-4)


@pytest.mark.parametrize("dtype,d_lo", [("bf16", 32), ("bf16", 16), ("f32", 36)])
def test_append_plane_copies_the_low_columns(loki, cuda, dtype, d_lo):
    torch = _t()
    wl = workloads.get("llama2-7b").with_(B=2, H_q=3, H_kv=3, S=9, dtype=dtype, n_cal=512,
                                          name=f"append-plane-{dtype}")
    inp = parity.host_inputs(wl)
    dt = parity.torch_dtype(wl)
    S_max, pos = 40, 17
    Kc = torch.zeros((2, 3, S_max, 128), dtype=dt, device=cuda)
    Vc = torch.zeros_like(Kc)
    Klo = torch.full((2, 3, S_max, d_lo), 9.0, dtype=dt, device=cuda)
    K2 = torch.zeros_like(Kc)
    V2 = torch.zeros_like(Kc)
    P = torch.from_numpy(inp.P).to(cuda)
    Kn, Vn = parity.to_device(inp.K, wl, cuda), parity.to_device(inp.V, wl, cuda)
    loki.loki_append_keys(Kn, Vn, P, Kc, Vc, pos, Kt_lo=Klo)
    loki.loki_append_keys(Kn, Vn, P, K2, V2, pos)
    # the rotated rows are the same with or without the plane, and the plane
    # holds exactly their first d_lo columns; other plane rows are untouched
    assert torch.equal(Kc, K2) and torch.equal(Vc, V2)
    assert torch.equal(Klo[:, :, pos:pos + wl.S], Kc[:, :, pos:pos + wl.S, :d_lo])
    mask = torch.ones(S_max, dtype=torch.bool)
    mask[pos:pos + wl.S] = False
    assert bool((Klo[:, :, mask] == 9.0).all())


# ---------------------------------------------------------------------------
# calibration: eigenvalues, vectors where the spectrum separates them,
# subspaces at every d used by the workloads
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "llama2-7b", "llama2-13b", "llama3-8b-gqa"])
def test_calibrate_matches_oracle(loki, cuda, name):
    torch = _t()
    wl = workloads.get(name)
    H = min(wl.H_kv, 8)
    cal = np.stack([workloads.calibration_keys(wl, h) for h in range(H)], axis=1)
    P, w = loki.loki_calibrate_pca(parity.to_device(cal, wl, cuda))
    P = P.cpu().numpy().astype(np.float64)
    w = w.cpu().numpy().astype(np.float64)
    for h in range(H):
        Po, wo = oracle.calibrate_pca(cal[:, h, :].astype(np.float64))
        np.testing.assert_allclose(w[h], wo, rtol=2e-6, atol=1e-7 * wo[0])
        np.testing.assert_allclose(P[h].T @ P[h], np.eye(128), atol=2e-6)
        # vector parity where each eigenvalue is separated from its neighbours
        gap = np.minimum(np.abs(np.diff(wo, prepend=np.inf)), np.abs(np.diff(wo, append=-np.inf)))
        sep = gap > 1e-6 * wo[0]
        err = np.abs(P[h] - Po).max(axis=0)
        # fp64 on both sides: the only visible difference is the fp32 output rounding
        assert np.all(err[sep] < 1e-5), (h, err[sep].max())
        for d in (16, 32, 64):
            Pi = P[h][:, :d] @ P[h][:, :d].T
            Po_ = Po[:, :d] @ Po[:, :d].T
            assert np.abs(Pi - Po_).max() < 1e-4
