"""Ragged batches over a paged KV-cache (GPU only): loki_decode_attention_paged
and loki_append_keys_paged against the fp64 oracle, every row on its own
sequence length.

Each sequence b has its own length S_b; its rotated keys, values and plane
rows are spread over a shuffled pool of pages named by a block table. The
oracle sees each sequence as the plain array of its S_b tokens and selects
min(k, S_b) of them; the GPU's selection must match outside the tie band,
padded with -1, and its output must be within the parity tolerance.
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


def _ragged_inputs(wl, lens, seed):
    """Per-sequence generator data with its own length; the oracle's basis and rotation."""
    Rs = [workloads.rotation(wl, h) for h in range(wl.H_kv)]
    P = np.ascontiguousarray(np.stack([oracle.calibrate_pca(workloads.calibration_keys(wl, h, Rs[h]))[0]
                                       for h in range(wl.H_kv)]), dtype=np.float32)
    seqs = []
    for b, L in enumerate(lens):
        K = np.stack([workloads.keys_block(wl, b, h, Rs[h], S=max(L, 1))[:L] for h in range(wl.H_kv)])
        V = np.stack([workloads.values_block(wl, b, h, S=max(L, 1))[:L] for h in range(wl.H_kv)])
        Kt = np.stack([oracle.rotate_keys(K[h], P[h].astype(np.float64), wl.dtype)
                       for h in range(wl.H_kv)]).astype(np.float32)
        seqs.append((K, V, Kt))
    q = np.stack([[workloads.query_vec(wl, b, h, Rs[h // wl.G]) for h in range(wl.H_q)]
                  for b in range(len(lens))])
    return P, seqs, q


def _page_pool(wl, seqs, page_size, max_pages, d_lo, seed, spare=3):
    """Scatter the sequences' rows over a shuffled pool; unused pages hold NaN."""
    rng = np.random.default_rng(seed)
    need = [-(-K.shape[1] // page_size) for K, _, _ in seqs]
    n_pages = sum(need) + spare
    order = rng.permutation(n_pages)
    bt = np.full((len(seqs), max_pages), -1, np.int32)
    Kp = np.full((n_pages, wl.H_kv, page_size, wl.D), np.nan, np.float32)
    Vp = np.full_like(Kp, np.nan)
    nxt = 0
    for b, (K, V, Kt) in enumerate(seqs):
        L = K.shape[1]
        for lp in range(need[b]):
            phys = int(order[nxt])
            nxt += 1
            bt[b, lp] = phys
            j0, j1 = lp * page_size, min(L, (lp + 1) * page_size)
            Kp[phys, :, : j1 - j0] = Kt[:, j0:j1]
            Vp[phys, :, : j1 - j0] = V[:, j0:j1]
    # block-table entries past a sequence's end point at a real page (never read)
    bt[bt < 0] = int(order[0])
    return Kp, Vp, Kp[..., :d_lo].copy(), bt, n_pages


CASES = [
    # name, workload overrides, lengths, page_size, max_pages, k, d_lo
    ("ragged-p16", dict(B=5, H_q=4, H_kv=4, d=32), [1000, 17, 1, 513, 64], 16, 64, 64, 32),
    ("ragged-p64-short", dict(B=4, H_q=4, H_kv=4, d=32), [40, 2000, 64, 0], 64, 32, 100, 32),
    ("full-and-partial-p256", dict(B=3, H_q=2, H_kv=2, d=32), [4096, 300, 2049], 256, 16, 512, 32),
    ("gqa4-p128", dict(B=3, H_q=16, H_kv=4, d=16), [1500, 4000, 129], 128, 32, 300, 16),
    ("f32-p32", dict(B=3, H_q=2, H_kv=2, d=20, dtype="f32"), [700, 5, 333], 32, 24, 90, 32),
    ("stored-scores-d64", dict(B=3, H_q=4, H_kv=4, d=64), [3000, 1200, 77], 32, 100, 600, 64),
]


@pytest.mark.parametrize("name,over,lens,page_size,max_pages,k,d_lo", CASES,
                         ids=[c[0] for c in CASES])
def test_paged_decode_matches_oracle(loki, cuda, name, over, lens, page_size, max_pages, k, d_lo):
    import torch
    wl = workloads.get("llama2-7b").with_(n_cal=512, name=f"paged-{name}", **over)
    P, seqs, q = _ragged_inputs(wl, lens, 1)
    Kp, Vp, Klo, bt, n_pages = _page_pool(wl, seqs, page_size, max_pages, d_lo, 2)
    dt = parity.torch_dtype(wl)
    dev = cuda
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(dt)  # noqa: E731
    out, idx = loki.loki_decode_attention_paged(
        t(q), t(Kp), t(Vp), t(Klo), torch.from_numpy(P).to(dev), torch.from_numpy(bt).to(dev),
        torch.tensor(lens, dtype=torch.int32, device=dev), wl.d, k, wl.scale)
    torch.cuda.synchronize()
    assert loki.loki_device_error(reset=True) == 0
    out = out.float().cpu().numpy()
    idx = idx.cpu().numpy()
    checks = []
    for b, L in enumerate(lens):
        kb = min(k, L)
        for h in range(wl.H_q):
            assert np.all(idx[b, h, kb:] == -1), (b, h)
            if kb == 0:
                assert np.all(out[b, h] == 0)
                continue
            K, V, Kt = seqs[b]
            hk = h // wl.G
            inp = parity.HostInputs(wl.with_(B=1, H_q=1, H_kv=1, S=L), q[b, h][None, None],
                                    None, V[hk][None, None], P[hk][None], None, Kt[hk][None, None],
                                    None)
            checks.append(parity.check_row(inp, 0, 0, idx[b, h, :kb], out[b, h], wl.d, kb,
                                           wl.scale))
    parity.summarize(checks)


def test_paged_append_writes_rotated_rows(loki, cuda):
    import torch
    wl = workloads.get("llama2-7b").with_(B=3, H_q=2, H_kv=2, n_cal=512, name="paged-append")
    lens = [100, 37, 1]
    P, seqs, q = _ragged_inputs(wl, lens, 3)
    page_size, max_pages, T = 16, 16, 5
    Kp, Vp, Klo, bt, n_pages = _page_pool(wl, seqs, page_size, max_pages, 32, 4, spare=6)
    # give every sequence room for T more tokens: extend its pages from the spares
    spare = [p for p in range(n_pages) if p not in set(bt[b, lp] for b in range(3)
                                                        for lp in range(-(-lens[b] // 16)))]
    for b, L in enumerate(lens):
        for lp in range(-(-L // 16), -(-(L + T) // 16)):
            bt[b, lp] = spare.pop()
    rng = np.random.default_rng(5)
    K_new = workloads.to_cache_dtype(rng.standard_normal((3, 2, T, 128)), "bf16")
    V_new = workloads.to_cache_dtype(rng.standard_normal((3, 2, T, 128)), "bf16")
    dev = cuda
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(torch.bfloat16)  # noqa: E731
    Kpd, Vpd, Klod = t(Kp), t(Vp), t(Klo)
    loki.loki_append_keys_paged(t(K_new), t(V_new), torch.from_numpy(P).to(dev), Kpd, Vpd,
                                torch.from_numpy(bt).to(dev),
                                torch.tensor(lens, dtype=torch.int32, device=dev), Kt_lo_pages=Klod)
    torch.cuda.synchronize()
    assert loki.loki_device_error(reset=True) == 0
    Kg, Vg, Lg = Kpd.float().cpu().numpy(), Vpd.float().cpu().numpy(), Klod.float().cpu().numpy()
    written = np.zeros(Kp.shape[:3], bool)
    for b, L in enumerate(lens):
        for tt in range(T):
            j = L + tt
            phys, slot = bt[b, j // page_size], j % page_size
            written[phys, :, slot] = True
            for h in range(2):
                exact = K_new[b, h, tt].astype(np.float64) @ P[h].astype(np.float64)
                want = oracle.round_to_dtype(exact, "bf16")
                tol = np.abs(want) * 2.0 ** -7 + 128 * 2.0 ** -24 * (
                    np.abs(K_new[b, h, tt]).astype(np.float64) @ np.abs(P[h]).astype(np.float64))
                assert np.all(np.abs(Kg[phys, h, slot] - want) <= tol + 1e-30)
                assert np.array_equal(Lg[phys, h, slot], Kg[phys, h, slot, :32])
                assert np.array_equal(Vg[phys, h, slot], V_new[b, h, tt])
    # nothing else changed
    np.testing.assert_array_equal(np.isnan(Kg[~written]), np.isnan(Kp[~written]))
    same = ~np.isnan(Kp[~written])
    assert np.array_equal(Kg[~written][same], Kp[~written][same].astype(np.float32))
