"""Shared pieces of the GPU parity tests.

Inputs come from the seeded generator (`workloads`); the PCA basis and the
rotated cache are computed by the fp64 oracle and rounded to the cache dtype,
so both paths consume identical bytes and nothing fed to the oracle comes
from the CUDA path. The GPU result is then compared with the oracle on the
same bytes.

Tolerances (the accuracy contract of this library):
  * selected index sets are bit-exact, except for tokens whose low-dimensional
    score lies within 1e-3 relative of the k-th score. The CUDA path computes
    q~ and the scores in fp32 (as the contract asks), and an fp32 sum cannot
    order two tokens whose exact scores differ by less than its rounding
    error; so a token also counts as tied when |s_j - s_k| is within the
    forward error bound of the two fp32 scores,
        (d + D + 2) * 2^-24 * (A_j + A_k),  A_j = sum_{i<d} |K~_ji| a_i,
        a_i = sum_c |q_c| |P_ci|
    (the fma-chain bound of q~ = q P over D terms, then of the d-term score).
    Tokens that pass only through this bound are counted apart
    (RowCheck.floor_only) and reported by the tests;
  * outputs within 2e-2 max-abs for bf16 and 1e-4 for fp32. Where the GPU set
    differs from the oracle's inside the band, the oracle attention is taken
    on the GPU's set (both sets are correct selections).
"""
from __future__ import annotations

import functools
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass
from typing import Dict, List, Optional, Tuple

import numpy as np

import oracle
import workloads

OUT_TOL = {"bf16": 2e-2, "f32": 1e-4}
BAND_REL = 1e-3
FP32_U = 2.0 ** -24


@dataclass
class HostInputs:
    wl: workloads.Workload
    q: np.ndarray        # [B, H_q, D] float32 (dtype-exact)
    K: np.ndarray        # [B, H_kv, S, D] raw keys
    V: np.ndarray        # [B, H_kv, S, D]
    P: np.ndarray        # [H_kv, D, D] float32 (oracle PCA, fp32-rounded)
    eig: np.ndarray      # [H_kv, D] fp64 (oracle)
    Kt: np.ndarray       # [B, H_kv, S, D] float32 (oracle rotation, dtype-rounded)
    K_cal: np.ndarray    # [n_cal, H_kv, D]


def _threads():
    return workloads._threads(None)


@functools.lru_cache(maxsize=3)
def host_inputs(wl: workloads.Workload) -> HostInputs:
    g = workloads.generate(wl)
    Ps, eigs = [], []
    for h in range(wl.H_kv):
        P, w = oracle.calibrate_pca(g["K_cal"][:, h, :])
        Ps.append(P)
        eigs.append(w)
    P32 = np.ascontiguousarray(np.stack(Ps), dtype=np.float32)
    Kt = np.empty_like(g["K"])

    def rot(bh):
        b, h = bh
        Kt[b, h] = oracle.rotate_keys(g["K"][b, h], P32[h].astype(np.float64), wl.dtype)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(rot, [(b, h) for b in range(wl.B) for h in range(wl.H_kv)]))
    return HostInputs(wl, g["q"], g["K"], g["V"], P32, np.stack(eigs), Kt, g["K_cal"])


def torch_dtype(wl):
    import torch
    return torch.float32 if wl.dtype == "f32" else torch.bfloat16


def to_device(x: np.ndarray, wl, dev, dtype=None, S_max: Optional[int] = None):
    """Upload float32 values (exact in the workload dtype) as the workload dtype.

    With S_max, a [B, H, S, D] array is placed in rows [0, S) of a
    [B, H, S_max, D] buffer whose other rows hold a NaN sentinel pattern, so a
    kernel that reads past S corrupts its result.
    """
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    t = t.to(dtype or torch_dtype(wl))
    if S_max is not None and S_max != x.shape[2]:
        buf = torch.full((x.shape[0], x.shape[1], S_max, x.shape[3]), float("nan"),
                         dtype=t.dtype, device=dev)
        buf[:, :, : x.shape[2]] = t
        t = buf
    return t


@dataclass
class RowCheck:
    row: Tuple[int, int]
    set_equal: bool
    band_diff: int
    max_err: float
    floor_only: int = 0


def fp32_score_bound(q: np.ndarray, P: np.ndarray, Kt: np.ndarray, d: int) -> np.ndarray:
    """Per-token bound on |fp32 score - exact score| for scores computed as
    q~ = q P (D-term fp32 fma chain) then s_j = q~[:d] . K~_j[:d] (d-term chain)."""
    D = P.shape[0]
    a = np.abs(np.asarray(q, np.float64)) @ np.abs(np.asarray(P, np.float64))
    A = np.abs(np.asarray(Kt, np.float64)[:, :d]) @ a[:d]
    return (d + D + 2) * FP32_U * A


def check_row(inp: HostInputs, b: int, h: int, gpu_idx: np.ndarray, gpu_out: np.ndarray,
              d: int, k: int, scale: float, S: Optional[int] = None,
              gpu_scores: Optional[np.ndarray] = None,
              attend_with: Optional[Tuple[np.ndarray, np.ndarray]] = None) -> RowCheck:
    """One row against the oracle: the selection outside the tie band, the
    scores (when given) within the fp32 bound, the output within OUT_TOL.

    attend_with = (query [D], keys [S, D]) replaces q~ and K~ in the exact
    attention over the selected tokens (the pre-rotary variant attends with
    its post-rotary query and keys)."""
    wl = inp.wl
    S = wl.S if S is None else S
    hk = h // wl.G
    Kt = inp.Kt[b, hk, :S].astype(np.float64)
    V = inp.V[b, hk, :S].astype(np.float64)
    P = inp.P[hk].astype(np.float64)
    q = inp.q[b, h].astype(np.float64)
    q_rot = oracle.project_query(q, P)
    s = oracle.lowdim_scores(q_rot, Kt, d)
    I = oracle.select_topk(s, k)
    gi = np.asarray(gpu_idx, dtype=np.int64)
    assert gi.shape == (k,), gi.shape
    assert np.all(np.diff(gi) > 0), "GPU indices must be strictly ascending"
    assert gi.min() >= 0 and gi.max() < S
    err_s = fp32_score_bound(q, P, Kt, d)
    if gpu_scores is not None:
        # the GPU scores obey the same forward error bound
        dev = np.abs(np.asarray(gpu_scores[:S], np.float64) - s)
        assert np.all(dev <= err_s + 1e-30), (
            f"row {(b, h)}: GPU score off by {dev.max():.3e} (bound {err_s[dev.argmax()]:.3e})")
    kpos = I[np.argmin(s[I])]
    kth = s[kpos]
    diff = np.setxor1d(I, gi)
    gap = np.abs(s[diff] - kth)
    rel = BAND_REL * abs(kth)
    floor = err_s[diff] + err_s[kpos]
    assert np.all(gap <= rel + floor), (
        f"row {(b, h)}: {len(diff)} tokens differ outside the tie band "
        f"(max |s-s_k| = {gap.max() if len(diff) else 0:.3e}, band {rel:.3e})")
    floor_only = int(np.sum(gap > rel))
    qa, Ka = (q_rot, Kt) if attend_with is None else (
        np.asarray(attend_with[0], np.float64), np.asarray(attend_with[1], np.float64)[:S])
    ref = oracle.attend(qa, Ka, V, gi if len(diff) else I, scale)
    err = float(np.abs(gpu_out.astype(np.float64) - ref).max())
    assert err <= OUT_TOL[wl.dtype], f"row {(b, h)}: max |out - oracle| = {err:.3e}"
    return RowCheck((b, h), len(diff) == 0, len(diff), err, floor_only)


def summarize(checks: List[RowCheck]) -> Dict[str, float]:
    s = {"rows": len(checks), "sets_identical": sum(c.set_equal for c in checks),
         "band_tokens": sum(c.band_diff for c in checks),
         "floor_only_tokens": sum(c.floor_only for c in checks),
         "max_err": max(c.max_err for c in checks)}
    print(f"parity: {s}")
    return s
