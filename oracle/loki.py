"""fp64 restatement of Loki, step by step, in the pages' order.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the
library path.

Notation: D head dimension, S cached tokens, d low-dimensional components, k
selected tokens, P the D x D PCA basis whose column c is principal component c
(eigenvalue-descending), K~ = K P the rotated keys held in the cache,
q~ = q P the rotated query.

Readings taken where the pages are silent (each also listed in the design
notes): PCA is covariance PCA (mean removed for the basis only; the rotation
is applied to raw keys so it stays orthogonal); the query is rotated by the
same basis as the keys; low-dimensional scores carry no softmax scale (only
their ranking is used); top-k ties go to the lower token index and the set is
returned in ascending token order; the softmax is renormalised over the
selected set only; the final scores use all D rotated dimensions, which equal
the unrotated scores because P is orthonormal.
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np


# ---------------------------------------------------------------------------
# Offline calibration
# ---------------------------------------------------------------------------

def covariance(X: np.ndarray) -> np.ndarray:
    """Sample covariance of calibration keys X [N, D]: centred, divided by N - 1.

    Loki pages: the study.space summary ("Loki uses principal component
    analysis (PCA) to reduce the dimensionality of key vectors") and the
    poster's Figure 1 caption (offline calibration with PCA). PCA is read as
    the eigen-decomposition of this covariance.
    """
    X = np.asarray(X, dtype=np.float64)
    n = X.shape[0]
    if n < 2:
        raise ValueError("need at least two calibration keys")
    Xc = X - X.mean(axis=0, keepdims=True)
    return (Xc.T @ Xc) / (n - 1)


def calibrate_pca(X: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Principal components of one head's calibration keys X [N, D].

    Returns (P [D, D], eigvals [D]): column c of P is the unit eigenvector of
    the covariance with the c-th largest eigenvalue (ties keep the library's
    order); each column's largest-magnitude entry (lowest index on a tie) is
    made positive. Poster page, "Visual Insights" Figure 1 caption: offline
    PCA gives the low-dimensional representation of the keys; the figure
    "rank at 90% explained variance" orders components by explained variance.
    The eigen-decomposition itself is the library's symmetric solver.
    """
    C = covariance(X)
    w, V = np.linalg.eigh(C)
    order = np.argsort(-w, kind="stable")
    w = w[order]
    V = V[:, order]
    piv = np.argmax(np.abs(V), axis=0)
    signs = np.where(V[piv, np.arange(V.shape[1])] < 0, -1.0, 1.0)
    return V * signs[None, :], w


def calibrate_pca_heads(keys: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """keys [N, H_kv, D] -> P [H_kv, D, D], eigvals [H_kv, D] (one basis per KV head)."""
    keys = np.asarray(keys, dtype=np.float64)
    Ps, ws = [], []
    for h in range(keys.shape[1]):
        P, w = calibrate_pca(keys[:, h, :])
        Ps.append(P)
        ws.append(w)
    return np.stack(Ps), np.stack(ws)


def explained_variance_rank(eigvals: np.ndarray, frac: float = 0.9) -> int:
    """Smallest r whose r largest eigenvalues explain at least `frac` of the variance.

    Poster page, rank figures under "More on figures" ("rank at 90% explained
    variance").
    """
    w = np.sort(np.asarray(eigvals, dtype=np.float64))[::-1]
    c = np.cumsum(w) / np.sum(w)
    return int(np.searchsorted(c, frac - 1e-15) + 1)


# ---------------------------------------------------------------------------
# KV-cache append: keys are stored rotated
# ---------------------------------------------------------------------------

def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp64 values to the cache element type, nearest-even, straight from fp64.

    'f32' rounds to IEEE binary32; 'bf16' keeps 8 significant bits (bfloat16
    has the binary32 exponent range, subnormal spacing 2^-133).
    """
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype != "bf16":
        raise ValueError(dtype)
    _, e = np.frexp(x)  # x = m 2^e, 0.5 <= |m| < 1
    quantum = np.ldexp(1.0, np.maximum(e - 8, -133))
    return np.rint(x / quantum) * quantum


def rotate_keys(K: np.ndarray, P: np.ndarray, dtype: Optional[str] = None) -> np.ndarray:
    """K~ = K P for keys K [..., D]; rounded to the cache dtype when given.

    Poster page, Figure 1 caption (keys are scored through their PCA
    projection) and "Loki's Computational Cost" (keys are appended to the
    KV-cache at each step). Reading: the cache keeps all D rotated columns,
    because the final scores need full-dimensional keys (poster TL;DR).
    """
    Kt = np.asarray(K, dtype=np.float64) @ np.asarray(P, dtype=np.float64)
    return Kt if dtype is None else round_to_dtype(Kt, dtype)


# ---------------------------------------------------------------------------
# Online decode step
# ---------------------------------------------------------------------------

def project_query(q: np.ndarray, P: np.ndarray) -> np.ndarray:
    """q~ = q P (all D components). Reading: the query uses the keys' basis."""
    return np.asarray(q, dtype=np.float64) @ np.asarray(P, dtype=np.float64)


def lowdim_scores(q_rot: np.ndarray, Kt: np.ndarray, d: int) -> np.ndarray:
    """Approximate scores s_j = sum_{i<d} q~_i K~_{j,i} for every cached token j.

    briefgpt.xyz abstract page and poster TL;DR: tokens are ranked by
    attention scores computed in the low-dimensional space of the first d
    principal components.
    """
    Kt = np.asarray(Kt, dtype=np.float64)
    return Kt[:, :d] @ np.asarray(q_rot, dtype=np.float64)[:d]


def select_topk(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores, ascending. Ties go to the lower index.

    Poster TL;DR and Figure 1 caption: the top-k tokens by approximate score
    are kept. Reading (pages silent): order by (-score, index), keep the first
    k, return them sorted by token index. NaN ranks lowest.
    """
    s = np.asarray(scores, dtype=np.float64)
    S = s.shape[0]
    if not 1 <= k <= S:
        raise ValueError("need 1 <= k <= S")
    key = np.where(np.isnan(s), -np.inf, s)
    order = np.lexsort((np.arange(S), -key))
    return np.sort(order[:k]).astype(np.int64)


def attend(q_rot: np.ndarray, Kt: np.ndarray, V: np.ndarray, idx: np.ndarray,
           scale: float) -> np.ndarray:
    """Exact softmax attention restricted to the selected tokens.

    a_j = scale * q~ . K~_j over all D dimensions, p = softmax(a) over the
    selected set only, out = sum_j p_j V_j. Poster TL;DR ("full-dimensional
    scores only for the selected tokens") and Figure 1 caption ("the
    full-dimensional keys are used to compute the final attention scores").
    """
    idx = np.asarray(idx)
    Ks = np.asarray(Kt, dtype=np.float64)[idx]
    Vs = np.asarray(V, dtype=np.float64)[idx]
    a = scale * (Ks @ np.asarray(q_rot, dtype=np.float64))
    p = np.exp(a - np.max(a))
    return (p @ Vs) / np.sum(p)


def loki_decode_row(q: np.ndarray, Kt: np.ndarray, V: np.ndarray, P: np.ndarray,
                    d: int, k: int, scale: float):
    """One (batch, query head): rotate q, score on d dims, pick top-k, attend.

    Returns (out [D], idx [k], lowdim scores [S], q~ [D]). Kt and V hold the S
    valid cache rows of the query head's KV head.
    """
    q_rot = project_query(q, P)
    s = lowdim_scores(q_rot, Kt, d)
    idx = select_topk(s, k)
    return attend(q_rot, Kt, V, idx, scale), idx, s, q_rot


def dense_decode_row(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """Full attention of one query over all S cached tokens (the baseline of every comparison)."""
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    a = scale * (K @ np.asarray(q, dtype=np.float64))
    p = np.exp(a - np.max(a))
    return (p @ V) / np.sum(p)


def pca_attn_row(q: np.ndarray, Kt: np.ndarray, V: np.ndarray, P: np.ndarray, d: int,
                 scale: float) -> np.ndarray:
    """PCAAttn variant: softmax directly on the d-dimensional scores over all tokens.

    Poster page, "More on tables", PCAAttn table caption: a variant that uses
    the reduced-dimensional attention scores directly (no top-k, no
    full-dimensional rescoring).
    """
    s = lowdim_scores(project_query(q, P), Kt, d)
    a = scale * s
    p = np.exp(a - np.max(a))
    return (p @ np.asarray(V, dtype=np.float64)) / np.sum(p)


def prerotary_decode_row(q_pre: np.ndarray, q_post: np.ndarray, Kt_pre: np.ndarray,
                         K_post: np.ndarray, V: np.ndarray, P: np.ndarray, d: int, k: int,
                         scale: float):
    """Pre-rotary variant: select on the pre-rotary keys, attend on the post-rotary ones.

    Poster page, "More on figures": the perplexity figure compares PCA
    transforms of pre- and post-rotary keys, and the rank figure shows both
    kinds of keys are low-rank. The pages give no mechanism; the reading: the
    basis P comes from pre-rotary keys, so the scores and the top-k take the
    pre-rotary query and keys in that basis (Kt_pre = K_pre P as cached), and
    the exact attention over the selected tokens takes the post-rotary query
    and keys, which the rotary embedding makes from them. Returns (out [D],
    idx [k]).
    """
    s = lowdim_scores(project_query(q_pre, P), Kt_pre, d)
    idx = select_topk(s, k)
    return attend(q_post, K_post, V, idx, scale), idx


# ---------------------------------------------------------------------------
# Batched wrappers (loops over rows; small sizes only)
# ---------------------------------------------------------------------------

def loki_decode(q: np.ndarray, Kt: np.ndarray, V: np.ndarray, P: np.ndarray, S: int,
                d: int, k: int, scale: Optional[float] = None):
    """q [B, H_q, D]; Kt, V [B, H_kv, >=S, D]; P [H_kv, D, D].

    Returns out [B, H_q, D] fp64, idx [B, H_q, k] int64, scores [B, H_q, S] fp64.
    Grouped-query attention: query head h uses KV head h // (H_q / H_kv) and
    makes its own selection (reading: per (batch, head) selection).
    """
    B, H_q, D = q.shape
    H_kv = Kt.shape[1]
    G = H_q // H_kv
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    out = np.zeros((B, H_q, D))
    idx = np.zeros((B, H_q, k), np.int64)
    sc = np.zeros((B, H_q, S))
    for b in range(B):
        for h in range(H_q):
            hk = h // G
            o, i, s, _ = loki_decode_row(q[b, h], Kt[b, hk, :S], V[b, hk, :S], P[hk], d, k, scale)
            out[b, h], idx[b, h], sc[b, h] = o, i, s
    return out, idx, sc


def dense_decode(q: np.ndarray, K: np.ndarray, V: np.ndarray, S: int,
                 scale: Optional[float] = None) -> np.ndarray:
    B, H_q, D = q.shape
    H_kv = K.shape[1]
    G = H_q // H_kv
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    out = np.zeros((B, H_q, D))
    for b in range(B):
        for h in range(H_q):
            out[b, h] = dense_decode_row(q[b, h], K[b, h // G, :S], V[b, h // G, :S], scale)
    return out
