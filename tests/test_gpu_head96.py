"""Heads of dimension 96 (GPU only) against the fp64 oracle.

The Loki pages report key ranks for models whose key dimension is 128 or 96
(poster page, "Loki: Low-Rank Keys for Efficient Sparse Attention", the
low-rank observation on the keys of several model families). Every entry
point that takes D accepts 96; the kernels keep the lane layout of 128
columns and leave the lanes past 96 idle. These cases run the row layout,
the key plane, the fused append, the paged cache, PCAAttn, the dense
baseline, the staged calls and the calibration at D = 96, each row checked
with the parity tolerances of the cache type.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workloads
from tests import parity
from tests.test_gpu_paged import _page_pool, _ragged_inputs

pytestmark = pytest.mark.gpu

D96 = dict(D=96, n_cal=512)


@pytest.fixture(scope="module")
def loki(cuda):
    import sparse_attention_decode_loki_b200 as m
    return m


def _wl(name, **over):
    return workloads.get("llama2-7b").with_(name=f"d96-{name}", **D96, **over)


DECODE_CASES = [
    # name, overrides, S_max, plane d_lo (None: row layout)
    ("rows", dict(B=2, H_q=8, H_kv=8, S=3000, d=32, k=400), 3100, None),
    ("plane", dict(B=2, H_q=8, H_kv=8, S=3000, d=32, k=400), 3000, 32),
    ("gqa4-plane", dict(B=2, H_q=16, H_kv=4, S=2049, d=16, k=300), 2100, 16),
    ("split-long", dict(B=1, H_q=4, H_kv=4, S=9000, d=24, k=2500), 9000, 32),
    ("f32-rows", dict(B=2, H_q=4, H_kv=2, S=700, d=20, k=90, dtype="f32"), 720, None),
    ("small-k", dict(B=3, H_q=2, H_kv=2, S=64, d=8, k=5), 64, 16),
    ("stored-scores-d48", dict(B=2, H_q=4, H_kv=4, S=3000, d=48, k=1200), 3000, 48),
]


@pytest.mark.parametrize("name,over,S_max,d_lo", DECODE_CASES, ids=[c[0] for c in DECODE_CASES])
def test_decode_d96_matches_oracle(loki, cuda, name, over, S_max, d_lo):
    import torch
    wl = _wl(name, **over)
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
    assert out.shape == (wl.B, wl.H_q, 96)
    out_h, idx_h = out.float().cpu().numpy(), idx.cpu().numpy()
    checks = [parity.check_row(inp, b, h, idx_h[b, h], out_h[b, h], wl.d, wl.k, wl.scale)
              for b in range(wl.B) for h in range(wl.H_q)]
    assert parity.summarize(checks)["rows"] == wl.B * wl.H_q


def test_staged_calls_d96(loki, cuda):
    """Projection, score scan (rows and plane), top-k and gather one by one."""
    import torch
    wl = _wl("staged", B=2, H_q=8, H_kv=4, S=1500, d=32, k=200)
    inp = parity.host_inputs(wl)
    q = parity.to_device(inp.q, wl, cuda)
    Kt = parity.to_device(inp.Kt, wl, cuda)
    V = parity.to_device(inp.V, wl, cuda)
    P = torch.from_numpy(inp.P).to(cuda)
    q_rot = loki.loki_project_query(q, P)
    assert q_rot.shape == (wl.B, wl.H_q, 96)
    s_rows = loki.loki_score_lowdim(q_rot, Kt, wl.S, wl.d)
    idx = loki.loki_topk(s_rows, wl.k)
    out = loki.loki_sparse_attention(q_rot, Kt, V, idx, wl.S, wl.scale)
    torch.cuda.synchronize()
    s_h, idx_h, out_h = s_rows.cpu().numpy(), idx.cpu().numpy(), out.float().cpu().numpy()
    checks = [parity.check_row(inp, b, h, idx_h[b, h], out_h[b, h], wl.d, wl.k, wl.scale,
                               gpu_scores=s_h[b, h])
              for b in range(wl.B) for h in range(wl.H_q)]
    parity.summarize(checks)
    # q~ against the oracle's projection, within the fp32 summation bound
    qr = q_rot.cpu().numpy().astype(np.float64)
    for b in range(wl.B):
        for h in range(wl.H_q):
            Ph = inp.P[h // wl.G].astype(np.float64)
            want = oracle.project_query(inp.q[b, h].astype(np.float64), Ph)
            bound = 98 * 2.0 ** -24 * (np.abs(inp.q[b, h]).astype(np.float64) @ np.abs(Ph))
            assert np.all(np.abs(qr[b, h] - want) <= bound + 1e-30)


def _signed_permutation(H, D, seed):
    rng = np.random.default_rng(seed)
    P = np.zeros((H, D, D))
    for h in range(H):
        P[h, rng.permutation(D), np.arange(D)] = rng.choice([-1.0, 1.0], D)
    return P


@pytest.mark.parametrize("d_lo", [None, 32])
def test_decode_step_d96_exact_basis(loki, cuda, d_lo):
    """The append folded into the step writes 96-wide rotated rows exactly
    (signed-permutation basis) and the decode over them is the oracle's."""
    import torch
    wl = _wl("step", B=2, H_q=8, H_kv=4, S=1500, d=32, k=200)
    g = workloads.generate(wl, with_cal=False)
    P = _signed_permutation(wl.H_kv, 96, 11)
    K, V = g["K"], g["V"]
    Kt = np.stack([[oracle.rotate_keys(K[b, h], P[h], wl.dtype) for h in range(wl.H_kv)]
                   for b in range(wl.B)])
    T, S_max = 2, 1536
    pos = wl.S - T
    dt = parity.torch_dtype(wl)
    Kc = torch.full((wl.B, wl.H_kv, S_max, 96), float("nan"), dtype=dt, device=cuda)
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
    out, idx = loki.loki_decode_step(q, K_new, V_new, torch.from_numpy(P.astype(np.float32)).to(cuda),
                                     Kc, Vc, pos, wl.d, wl.k, wl.scale, Kt_lo=Klo)
    torch.cuda.synchronize()
    assert loki.loki_device_error(reset=True) == 0
    np.testing.assert_array_equal(Kc[:, :, pos:wl.S].float().cpu().numpy(),
                                  Kt[:, :, pos:].astype(np.float32))
    np.testing.assert_array_equal(Vc[:, :, pos:wl.S].float().cpu().numpy(), V[:, :, pos:])
    if Klo is not None:
        assert torch.equal(Klo[:, :, pos:wl.S], Kc[:, :, pos:wl.S, :d_lo])
    assert bool(torch.isnan(Kc[:, :, wl.S:].float()).all())
    inp = parity.HostInputs(wl, g["q"], K, V, P.astype(np.float32), None, Kt, None)
    out_h, idx_h = out.float().cpu().numpy(), idx.cpu().numpy()
    checks = [parity.check_row(inp, b, h, idx_h[b, h], out_h[b, h], wl.d, wl.k, wl.scale)
              for b in range(wl.B) for h in range(wl.H_q)]
    parity.summarize(checks)


def test_paged_decode_d96(loki, cuda):
    import torch
    wl = _wl("paged", B=4, H_q=8, H_kv=4, d=32)
    lens, page_size, max_pages, k, d_lo = [1000, 17, 2500, 0], 64, 48, 300, 32
    P, seqs, q = _ragged_inputs(wl, lens, 1)
    Kp, Vp, Klo, bt, n_pages = _page_pool(wl, seqs, page_size, max_pages, d_lo, 2)
    dt = parity.torch_dtype(wl)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(cuda).to(dt)  # noqa: E731
    out, idx = loki.loki_decode_attention_paged(
        t(q), t(Kp), t(Vp), t(Klo), torch.from_numpy(P).to(cuda), torch.from_numpy(bt).to(cuda),
        torch.tensor(lens, dtype=torch.int32, device=cuda), wl.d, k, wl.scale)
    torch.cuda.synchronize()
    assert loki.loki_device_error(reset=True) == 0
    out, idx = out.float().cpu().numpy(), idx.cpu().numpy()
    checks = []
    for b, L in enumerate(lens):
        kb = min(k, L)
        for h in range(wl.H_q):
            assert np.all(idx[b, h, kb:] == -1)
            if kb == 0:
                assert np.all(out[b, h] == 0)
                continue
            _, V, Kt = seqs[b]
            hk = h // wl.G
            inp = parity.HostInputs(wl.with_(B=1, H_q=1, H_kv=1, S=L), q[b, h][None, None], None,
                                    V[hk][None, None], P[hk][None], None, Kt[hk][None, None], None)
            checks.append(parity.check_row(inp, 0, 0, idx[b, h, :kb], out[b, h], wl.d, kb,
                                           wl.scale))
    parity.summarize(checks)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_dense_and_pca_d96(loki, cuda, dtype):
    import torch
    wl = _wl(f"dense-{dtype}", B=2, H_q=8, H_kv=4, S=2100, d=32, dtype=dtype)
    inp = parity.host_inputs(wl)
    q = parity.to_device(inp.q, wl, cuda)
    K = parity.to_device(inp.K.astype(np.float32), wl, cuda, S_max=2200)
    V = parity.to_device(inp.V, wl, cuda, S_max=2200)
    out = loki.dense_decode_attention(q, K, V, wl.S, wl.scale).float().cpu().numpy()
    Klo = parity.to_device(inp.Kt[..., :32], wl, cuda, S_max=2200)
    pca = loki.loki_pca_attention(q, Klo, V, torch.from_numpy(inp.P).to(cuda), wl.S, wl.d,
                                  wl.scale).float().cpu().numpy()
    # dense runs on the raw keys as cached (rounded to the cache type)
    Kr = oracle.round_to_dtype(inp.K.astype(np.float64), wl.dtype)
    e_dense = e_pca = 0.0
    for b in range(wl.B):
        for h in range(wl.H_q):
            hk = h // wl.G
            ref = oracle.dense_decode_row(inp.q[b, h].astype(np.float64), Kr[b, hk],
                                          inp.V[b, hk].astype(np.float64), wl.scale)
            e_dense = max(e_dense, float(np.abs(out[b, h] - ref).max()))
            ref = oracle.pca_attn_row(inp.q[b, h].astype(np.float64), inp.Kt[b, hk].astype(np.float64),
                                      inp.V[b, hk].astype(np.float64), inp.P[hk].astype(np.float64),
                                      wl.d, wl.scale)
            e_pca = max(e_pca, float(np.abs(pca[b, h] - ref).max()))
    assert e_dense <= parity.OUT_TOL[wl.dtype], e_dense
    assert e_pca <= parity.OUT_TOL[wl.dtype], e_pca


def test_calibrate_d96(loki, cuda):
    wl = _wl("cal", H_kv=4)
    cal = np.stack([workloads.calibration_keys(wl, h) for h in range(wl.H_kv)], axis=1)
    assert cal.shape[2] == 96
    P, w = loki.loki_calibrate_pca(parity.to_device(cal, wl, cuda))
    P = P.cpu().numpy().astype(np.float64)
    w = w.cpu().numpy().astype(np.float64)
    for h in range(wl.H_kv):
        Po, wo = oracle.calibrate_pca(cal[:, h, :].astype(np.float64))
        np.testing.assert_allclose(w[h], wo, rtol=2e-6, atol=1e-7 * wo[0])
        np.testing.assert_allclose(P[h].T @ P[h], np.eye(96), atol=2e-6)
        for d in (16, 32, 64):
            assert np.abs(P[h][:, :d] @ P[h][:, :d].T - Po[:, :d] @ Po[:, :d].T).max() < 1e-4
