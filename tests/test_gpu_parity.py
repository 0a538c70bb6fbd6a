"""CUDA path against the fp64 oracle on the same seeded inputs (GPU only).

Full checks (every row) at the small workloads and edge cases; sampled rows
at the large workloads, which run in exactly the launch configuration the
benchmark times. See tests/parity.py for the tolerances.
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


def _torch():
    import torch
    return torch


def run_full(loki, inp, dev, S=None, S_max=None, d=None, k=None, with_steps=False, d_lo=None):
    torch = _torch()
    wl = inp.wl
    S = wl.S if S is None else S
    d = wl.d if d is None else d
    k = wl.k if k is None else k
    q = parity.to_device(inp.q, wl, dev)
    Kt = parity.to_device(inp.Kt[:, :, :S], wl, dev, S_max=S_max)
    V = parity.to_device(inp.V[:, :, :S], wl, dev, S_max=S_max)
    P = torch.from_numpy(inp.P).to(dev)
    Kt_lo = None
    if d_lo is not None:
        # the low-dim key plane holds a copy of the first d_lo rotated columns
        Kt_lo = parity.to_device(inp.Kt[:, :, :S, :d_lo], wl, dev, S_max=S_max)
    out, idx = loki.loki_decode_attention(q, Kt, V, P, S, d, k, wl.scale, Kt_lo=Kt_lo)
    res = {"out": out.float().cpu().numpy(), "idx": idx.cpu().numpy()}
    if with_steps:
        q_rot = loki.loki_project_query(q, P)
        res["q_rot"] = q_rot.cpu().numpy()
        res["scores"] = loki.loki_score_lowdim(q_rot, Kt if Kt_lo is None else Kt_lo, S,
                                               d).cpu().numpy()
    torch.cuda.synchronize()
    assert loki.loki_device_error(reset=True) == 0, "a staged kernel's bounded wait gave up"
    return res


def check_all_rows(inp, res, S=None, d=None, k=None, steps=False):
    wl = inp.wl
    d = wl.d if d is None else d
    k = wl.k if k is None else k
    checks = []
    for b in range(wl.B):
        for h in range(wl.H_q):
            checks.append(parity.check_row(
                inp, b, h, res["idx"][b, h], res["out"][b, h], d, k, wl.scale, S=S,
                gpu_scores=res["scores"][b, h] if steps else None))
    return parity.summarize(checks)


# ---------------------------------------------------------------------------
# workloads checked in full
# ---------------------------------------------------------------------------

def test_tiny_fp32_full(loki, cuda):
    inp = parity.host_inputs(workloads.get("tiny"))
    res = run_full(loki, inp, cuda, S_max=300, with_steps=True)
    s = check_all_rows(inp, res, steps=True)
    assert s["rows"] == 1
    # q~ matches the oracle's q P in fp32
    ref = np.einsum("bhi,hic->bhc", inp.q.astype(np.float64), inp.P.astype(np.float64))
    np.testing.assert_allclose(res["q_rot"], ref, rtol=1e-5, atol=1e-5 * np.abs(ref).max())


def test_llama2_7b_full(loki, cuda):
    inp = parity.host_inputs(workloads.get("llama2-7b"))
    res = run_full(loki, inp, cuda, with_steps=True)
    s = check_all_rows(inp, res, steps=True)
    assert s["rows"] == 32 and s["sets_identical"] >= 28, s


EDGE = [
    # name, overrides, S_max
    ("ragged-S-d20", dict(S=1000, d=20, k=77), 1024),
    ("k1", dict(S=513, k=1), 600),
    ("k-all", dict(S=300, k=300), 300),
    ("d1", dict(S=700, d=1, k=64), 700),
    ("d-full", dict(S=640, d=128, k=100), 700),
    ("S1", dict(S=1, k=1), 8),
    ("gqa2-B3", dict(B=3, H_q=4, H_kv=2, S=333, k=50), 400),
    ("gqa4", dict(B=2, H_q=8, H_kv=2, S=2049, d=16, k=128), 2100),
    ("gqa8", dict(B=1, H_q=16, H_kv=2, S=1500, d=24, k=200), 1500),
    ("gqa3", dict(B=2, H_q=6, H_kv=2, S=777, d=40, k=99), 800),
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("name,over,S_max", EDGE, ids=[e[0] for e in EDGE])
def test_edge_cases(loki, cuda, dtype, name, over, S_max):
    base = workloads.get("llama2-7b").with_(B=1, H_q=2, H_kv=2, n_cal=512, dtype=dtype,
                                            name=f"edge-{name}-{dtype}")
    wl = base.with_(**over)
    inp = parity.host_inputs(wl)
    res = run_full(loki, inp, cuda, S_max=S_max, with_steps=True)
    check_all_rows(inp, res, steps=True)


@pytest.mark.parametrize("name,d_lo", [("tiny", 32), ("tiny", 36), ("llama2-7b", 32),
                                       ("llama2-7b", 64)])
def test_plane_layout_full(loki, cuda, name, d_lo):
    inp = parity.host_inputs(workloads.get(name))
    res = run_full(loki, inp, cuda, S_max=inp.wl.S + 64, with_steps=True, d_lo=d_lo)
    check_all_rows(inp, res, steps=True)


PLANE_EDGE = [("ragged-S-d20", 24), ("d1", 8), ("d-full", 128), ("gqa4", 16), ("gqa3", 40),
              ("k1", 32)]


@pytest.mark.parametrize("name,d_lo", PLANE_EDGE, ids=[e[0] for e in PLANE_EDGE])
def test_plane_edge_cases(loki, cuda, name, d_lo):
    over, S_max = {e[0]: (e[1], e[2]) for e in EDGE}[name]
    wl = workloads.get("llama2-7b").with_(B=1, H_q=2, H_kv=2, n_cal=512,
                                          name=f"edge-{name}-bf16").with_(**over)
    inp = parity.host_inputs(wl)
    res = run_full(loki, inp, cuda, S_max=S_max, with_steps=True, d_lo=d_lo)
    check_all_rows(inp, res, steps=True)


def test_all_dims_all_tokens_is_dense(loki, cuda):
    torch = _torch()
    wl = workloads.get("llama2-7b").with_(H_q=4, H_kv=4, S=1024, name="dense-invariant")
    inp = parity.host_inputs(wl)
    res = run_full(loki, inp, cuda, d=128, k=wl.S)
    assert np.array_equal(res["idx"], np.broadcast_to(np.arange(wl.S), res["idx"].shape))
    # the same rotated inputs through the dense kernel (q~ rounded to the cache
    # dtype) and through the oracle's dense attention
    dev = cuda
    qr = np.einsum("bhi,hic->bhc", inp.q.astype(np.float64), inp.P.astype(np.float64))
    qr_t = torch.from_numpy(qr.astype(np.float32)).to(dev).to(torch.bfloat16)
    dense = loki.dense_decode_attention(qr_t, parity.to_device(inp.Kt, wl, dev),
                                        parity.to_device(inp.V, wl, dev), wl.S, wl.scale)
    dense = dense.float().cpu().numpy()
    for h in range(wl.H_q):
        ref = oracle.dense_decode_row(inp.q[0, h], inp.K[0, h], inp.V[0, h], wl.scale)
        # K~ is K P rounded to bf16, so compare against the unrotated textbook result
        assert np.abs(res["out"][0, h] - ref).max() < 3e-2
        assert np.abs(dense[0, h] - res["out"][0, h]).max() < 3e-2


# ---------------------------------------------------------------------------
# large workloads
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("plane", [False, True])
def test_llama2_13b_every_row(loki, cuda, plane):
    """The benchmark's workload and launch configuration, every (batch, head)
    row against the oracle."""
    inp = parity.host_inputs(workloads.get("llama2-13b"))
    res = run_full(loki, inp, cuda, d_lo=32 if plane else None)
    s = check_all_rows(inp, res)
    assert s["rows"] == 640


@pytest.mark.parametrize("plane", [False, True])
def test_llama3_8b_gqa_every_row(loki, cuda, plane):
    inp = parity.host_inputs(workloads.get("llama3-8b-gqa"))
    res = run_full(loki, inp, cuda, d_lo=16 if plane else None)
    s = check_all_rows(inp, res)
    assert s["rows"] == 128


def _check_block(wl, P, q, Kt, V, gidx, gout, row):
    inp = parity.HostInputs(wl, q[None, None, :], None, V[None, None], P[None], None,
                            Kt[None, None], None)
    inp.wl = wl.with_(B=1, H_q=1, H_kv=1)
    return parity.check_row(inp, 0, 0, gidx, gout, wl.d, wl.k, wl.scale)


def _sweep_group(B, S):
    return [p for p in workloads.sweep_points() if p.B == B and p.S == S]


SWEEP_GROUPS = sorted({(p.B, p.S) for p in workloads.sweep_points()})


@pytest.mark.parametrize("B,S", SWEEP_GROUPS, ids=[f"B{b}-S{s}" for b, s in SWEEP_GROUPS])
def test_sweep_every_point_sampled_rows(loki, cuda, B, S):
    """All six (d, k/S) points of one (B, S) of the sweep at full size, in the
    benchmark's layout (a key plane of d columns; the row layout where the
    plane does not fit the device). The points share their inputs (one seed),
    so the cache is filled once per (B, S): random filler everywhere and
    generator bytes in the blocks of 6 sampled rows, which are checked against
    the oracle."""
    torch = _torch()
    pts = _sweep_group(B, S)
    wl = pts[0]
    e = wl.elem_bytes
    kv_bytes = 2 * e * B * wl.H_kv * S * wl.D
    scores_bytes = 4 * B * wl.H_q * S
    margin = 3 << 30
    free, _ = torch.cuda.mem_get_info(cuda)
    if kv_bytes + scores_bytes + margin > free:
        pytest.skip(f"B={B}, S={S}: the cache ({kv_bytes / 1e9:.1f} GB) does not fit "
                    f"the free device memory ({free / 1e9:.1f} GB)")
    rows = workloads.sample_rows(wl, 6, 7)
    need_kv = sorted({h // wl.G for _, h in rows})
    Rs = {h: workloads.rotation(wl, h) for h in need_kv}
    P = np.tile(np.eye(wl.D, dtype=np.float32), (wl.H_kv, 1, 1))
    for h in need_kv:
        Pm, _ = oracle.calibrate_pca(workloads.calibration_keys(wl, h, Rs[h]))
        P[h] = Pm.astype(np.float32)
    dt = parity.torch_dtype(wl)
    g = torch.Generator(device=cuda)
    g.manual_seed(wl.seed + B + S)
    Kt = torch.randn((B, wl.H_kv, S, wl.D), generator=g, device=cuda, dtype=dt)
    V = torch.randn((B, wl.H_kv, S, wl.D), generator=g, device=cuda, dtype=dt)
    q = torch.randn((B, wl.H_q, wl.D), generator=g, device=cuda, dtype=dt)
    host = {}
    for b, h in rows:
        hk = h // wl.G
        if (b, hk) not in host:
            K = workloads.keys_block(wl, b, hk, Rs[hk])
            Vb = workloads.values_block(wl, b, hk)
            Ktb = oracle.rotate_keys(K, P[hk].astype(np.float64), wl.dtype).astype(np.float32)
            host[(b, hk)] = (Ktb, Vb)
            Kt[b, hk] = torch.from_numpy(Ktb).to(cuda).to(dt)
            V[b, hk] = torch.from_numpy(Vb).to(cuda).to(dt)
        q[b, h] = torch.from_numpy(workloads.query_vec(wl, b, h, Rs[hk])).to(cuda).to(dt)
    Pt = torch.from_numpy(P).to(cuda)
    qh = q.float().cpu().numpy()
    layouts = {}
    for pt in pts:
        free, _ = torch.cuda.mem_get_info(cuda)
        plane_bytes = e * B * wl.H_kv * S * pt.d
        Kt_lo = None
        if plane_bytes + scores_bytes + margin <= free:
            Kt_lo = Kt[..., : pt.d].contiguous()
        out, idx = loki.loki_decode_attention(q, Kt, V, Pt, S, pt.d, pt.k, pt.scale, Kt_lo=Kt_lo)
        out = out.float().cpu().numpy()
        idx = idx.cpu().numpy()
        assert loki.loki_device_error(reset=True) == 0, "a staged kernel's bounded wait gave up"
        layouts[pt.name] = "plane" if Kt_lo is not None else "rows"
        del Kt_lo
        checks = []
        for b, h in rows:
            hk = h // wl.G
            Ktb, Vb = host[(b, hk)]
            checks.append(_check_block(pt, P[hk], qh[b, h], Ktb, Vb, idx[b, h], out[b, h], (b, h)))
        assert parity.summarize(checks)["rows"] == 6
        torch.cuda.empty_cache()
    print(f"sweep B={B} S={S}: layouts {layouts}")
    del Kt, V
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# dense baseline
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "llama2-7b"])
def test_dense_full(loki, cuda, name):
    torch = _torch()
    wl = workloads.get(name)
    inp = parity.host_inputs(wl)
    out = loki.dense_decode_attention(parity.to_device(inp.q, wl, cuda),
                                      parity.to_device(inp.K, wl, cuda, S_max=wl.S + 40),
                                      parity.to_device(inp.V, wl, cuda, S_max=wl.S + 40),
                                      wl.S, wl.scale)
    out = out.float().cpu().numpy()
    ref = oracle.dense_decode(inp.q.astype(np.float64), inp.K.astype(np.float64),
                              inp.V.astype(np.float64), wl.S, wl.scale)
    assert np.abs(out - ref).max() <= parity.OUT_TOL[wl.dtype]
    torch.cuda.synchronize()


@pytest.mark.parametrize("G", [1, 2, 4, 8, 5])
def test_dense_groups(loki, cuda, G):
    wl = workloads.get("llama2-7b").with_(B=2, H_q=2 * G, H_kv=2, S=1111, n_cal=256,
                                          name=f"dense-g{G}")
    inp = parity.host_inputs(wl)
    out = loki.dense_decode_attention(parity.to_device(inp.q, wl, cuda),
                                      parity.to_device(inp.K, wl, cuda),
                                      parity.to_device(inp.V, wl, cuda), wl.S, wl.scale)
    out = out.float().cpu().numpy()
    ref = oracle.dense_decode(inp.q.astype(np.float64), inp.K.astype(np.float64),
                              inp.V.astype(np.float64), wl.S, wl.scale)
    assert np.abs(out - ref).max() <= parity.OUT_TOL[wl.dtype]
