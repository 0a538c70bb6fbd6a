"""Seeded synthetic decode workloads shaped like the Loki evaluation models.

This module only draws inputs. It holds none of Loki's arithmetic (no PCA, no
rotation, no scoring, no selection, no attention); both the fp64 CPU oracle and
the CUDA path take their inputs from here, and nothing else is shared between
them.

Why synthetic low-rank keys: the Loki pages (NeurIPS 2024 poster page,
"Visual Insights", Figure 1 caption; and the layer-wise rank figure under
"More on figures") report that about 80 of the 128 principal components of
real attention keys carry 90% of their variance. Real KV-caches of Llama2/3 on
WikiText/C4/BookCorpus need trained weights and datasets, so a generator with a
controlled spectrum stands in for them:

    K = (Z * sigma) @ R.T + noise,   Z ~ N(0, 1),  sigma_i = exp(-i / tau),
    noise ~ N(0, noise_std^2),       R = Haar-random orthogonal (QR of a Gaussian)

Queries are drawn the same way with the KV head's R; values are N(0, 1).
Everything is drawn in fp64 and rounded to the workload's cache dtype; the
rounded values are the bytes both paths consume.

Every (tensor kind, batch, head) block has its own counter-free PCG64 stream
seeded by ``SeedSequence([seed, kind, b, h])``, so any block can be regenerated
alone (sampled parity at full size) and blocks can be drawn in parallel.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Iterable, List, Optional, Tuple

import numpy as np

# stream kinds (part of the seed)
_KIND_R = 1
_KIND_KZ = 2
_KIND_KNOISE = 3
_KIND_V = 4
_KIND_QZ = 5
_KIND_QNOISE = 6
_KIND_CALZ = 7
_KIND_CALNOISE = 8


@dataclasses.dataclass(frozen=True)
class Workload:
    """One decode-attention problem: shapes, Loki hyper-parameters, generator recipe."""

    name: str
    B: int
    H_q: int
    H_kv: int
    D: int
    S: int
    d: int
    k: int
    dtype: str  # "f32" or "bf16": cache, query, value and output element type
    tau: float  # spectrum decay: sigma_i = exp(-i / tau)
    n_cal: int  # calibration keys per KV head
    seed: int
    noise_std: float = 0.01

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    # algorithmic bytes of one Loki layer-step: the low-dim key columns of every
    # cached token (once per KV head) plus full key and value rows of the k
    # selected tokens (per query head); q, P and out are under 1% and left out.
    def loki_bytes(self) -> int:
        e = self.elem_bytes
        return e * (self.B * self.H_kv * self.S * self.d + self.B * self.H_q * 2 * self.k * self.D)

    def moved_bytes(self) -> int:
        """loki_bytes less the key columns the attention does not re-read:
        with d >= D / 2 (d a whole number of 16-byte chunks, d < D) it adds
        the scan's stored score of each selected token and reads only key
        columns [d, D)."""
        e = self.elem_bytes
        chunk = 16 // e
        reuse = 2 * self.d >= self.D and self.d % chunk == 0 and self.d < self.D
        return self.loki_bytes() - (e * self.B * self.H_q * self.k * self.d if reuse else 0)

    def dense_bytes(self) -> int:
        e = self.elem_bytes
        return e * self.B * self.H_kv * 2 * self.S * self.D


def _wl(name, B, H_q, H_kv, S, d, k, dtype, tau, n_cal, seed, D=128):
    return Workload(name=name, B=B, H_q=H_q, H_kv=H_kv, D=D, S=S, d=d, k=k,
                    dtype=dtype, tau=tau, n_cal=n_cal, seed=seed)


# The five workloads. Seeds follow 1000 * (workload number).
WORKLOADS: Dict[str, Workload] = {
    # tiny single-head fp32 decode, tau = 16
    "tiny": _wl("tiny", 1, 1, 1, 256, 32, 64, "f32", 16.0, 1024, 1000),
    # Llama2-7B layer shape: MHA 32 heads, 4096 cached tokens, d = 32, k = 25%
    "llama2-7b": _wl("llama2-7b", 1, 32, 32, 4096, 32, 1024, "bf16", 20.0, 4096, 2000),
    # Llama2-13B batched decode: MHA 40 heads, B = 16, d = 32, k = 12.5%.
    # tau = 80 puts the 90%-variance rank at 80 of 128 (the rank the pages report).
    "llama2-13b": _wl("llama2-13b", 16, 40, 40, 4096, 32, 512, "bf16", 80.0, 4096, 3000),
    # Llama-3-8B GQA long context: 32 query heads over 8 KV heads, d = 16, k = 6.25%
    "llama3-8b-gqa": _wl("llama3-8b-gqa", 4, 32, 8, 32768, 16, 2048, "bf16", 12.0, 4096, 4000),
}


def sweep_points() -> List[Workload]:
    """Sweep at the Llama2-13B head shape (H = 40, D = 128, bf16, tau = 80)."""
    pts = []
    for B in (1, 8, 64):
        for S in (2048, 16384, 131072):
            for d in (16, 32, 64):
                for kf_num, kf_den in ((1, 8), (1, 4)):
                    k = S * kf_num // kf_den
                    name = f"sweep-B{B}-S{S}-d{d}-k{kf_num}of{kf_den}"
                    pts.append(_wl(name, B, 40, 40, S, d, k, "bf16", 80.0, 4096, 5000))
    return pts


def get(name: str) -> Workload:
    if name in WORKLOADS:
        return WORKLOADS[name]
    for p in sweep_points():
        if p.name == name:
            return p
    raise KeyError(name)


# ---------------------------------------------------------------------------
# dtype rounding of generated values (input encoding, not method arithmetic)
# ---------------------------------------------------------------------------

def to_cache_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp64 draws to the workload dtype; returns float32 holding exact values.

    bf16: round to fp32 first (nearest-even), then to bf16 (nearest-even on the
    upper 16 bits). This two-step rounding is the generator's definition of its
    bf16 draws; both paths consume the same rounded bytes.
    """
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    if dtype == "f32":
        return x32
    if dtype != "bf16":
        raise ValueError(dtype)
    u = x32.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(np.float32)


def bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are exactly bf16-representable."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    if np.any(u & np.uint32(0xFFFF)):
        raise ValueError("values are not bf16-representable")
    return (u >> np.uint32(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# streams
# ---------------------------------------------------------------------------

def _rng(wl: Workload, kind: int, a: int = 0, b: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([wl.seed, kind, a, b])))


def sigma(wl: Workload) -> np.ndarray:
    return np.exp(-np.arange(wl.D, dtype=np.float64) / wl.tau)


def rotation(wl: Workload, h_kv: int) -> np.ndarray:
    """Haar-random orthogonal D x D for one KV head (QR of a Gaussian, sign-fixed)."""
    g = _rng(wl, _KIND_R, h_kv).standard_normal((wl.D, wl.D))
    q, r = np.linalg.qr(g)
    return q * np.sign(np.diag(r))[None, :]


def _lowrank(wl: Workload, n: int, R: np.ndarray, rz: np.random.Generator,
             rn: np.random.Generator) -> np.ndarray:
    z = rz.standard_normal((n, wl.D))
    return (z * sigma(wl)[None, :]) @ R.T + wl.noise_std * rn.standard_normal((n, wl.D))


def keys_block(wl: Workload, b: int, h_kv: int, R: Optional[np.ndarray] = None,
               S: Optional[int] = None) -> np.ndarray:
    """Raw (unrotated) keys of one (batch, KV head): [S, D], dtype-rounded, float32."""
    R = rotation(wl, h_kv) if R is None else R
    S = wl.S if S is None else S
    x = _lowrank(wl, S, R, _rng(wl, _KIND_KZ, b, h_kv), _rng(wl, _KIND_KNOISE, b, h_kv))
    return to_cache_dtype(x, wl.dtype)


def values_block(wl: Workload, b: int, h_kv: int, S: Optional[int] = None) -> np.ndarray:
    S = wl.S if S is None else S
    return to_cache_dtype(_rng(wl, _KIND_V, b, h_kv).standard_normal((S, wl.D)), wl.dtype)


def query_vec(wl: Workload, b: int, h_q: int, R: Optional[np.ndarray] = None) -> np.ndarray:
    """One decode query [D] drawn like a key with its KV head's R."""
    h_kv = h_q // wl.G
    R = rotation(wl, h_kv) if R is None else R
    x = _lowrank(wl, 1, R, _rng(wl, _KIND_QZ, b, h_q), _rng(wl, _KIND_QNOISE, b, h_q))[0]
    return to_cache_dtype(x, wl.dtype)


def calibration_keys(wl: Workload, h_kv: int, R: Optional[np.ndarray] = None,
                     n: Optional[int] = None) -> np.ndarray:
    """Calibration keys of one KV head [n_cal, D] from streams separate from the cache."""
    R = rotation(wl, h_kv) if R is None else R
    n = wl.n_cal if n is None else n
    x = _lowrank(wl, n, R, _rng(wl, _KIND_CALZ, 0, h_kv), _rng(wl, _KIND_CALNOISE, 0, h_kv))
    return to_cache_dtype(x, wl.dtype)


def rope(x: np.ndarray, positions: np.ndarray, base: float = 10000.0,
         dtype: Optional[str] = None) -> np.ndarray:
    """Rotary position embedding of rows x [..., n, D] at token positions [n].

    The input-side transform that makes the post-rotary keys and queries of
    the pre-rotary variant from the generated (pre-rotary) ones: column pair
    (i, i + D/2) of the row at position t turns by the angle t * base^(-2i/D)
    (the half-split pairing). Computed in fp64; rounded to `dtype` when given.
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    half = D // 2
    inv = base ** (-2.0 * np.arange(half, dtype=np.float64) / D)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv[None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :half], x[..., half:]
    y = np.concatenate([a * c - b * s, a * s + b * c], axis=-1)
    return y if dtype is None else to_cache_dtype(y, dtype)


def _threads(threads: Optional[int]) -> int:
    if threads:
        return threads
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def generate(wl: Workload, threads: Optional[int] = None, with_keys: bool = True,
             with_cal: bool = True) -> Dict[str, np.ndarray]:
    """All inputs of a workload as float32 arrays of dtype-exact values.

    q [B, H_q, D]; K, V [B, H_kv, S, D] (K raw, unrotated); K_cal [n_cal, H_kv, D].
    """
    Rs = [rotation(wl, h) for h in range(wl.H_kv)]
    out: Dict[str, np.ndarray] = {}
    q = np.empty((wl.B, wl.H_q, wl.D), np.float32)
    for b in range(wl.B):
        for h in range(wl.H_q):
            q[b, h] = query_vec(wl, b, h, Rs[h // wl.G])
    out["q"] = q
    if with_keys:
        K = np.empty((wl.B, wl.H_kv, wl.S, wl.D), np.float32)
        V = np.empty((wl.B, wl.H_kv, wl.S, wl.D), np.float32)

        def job(bh: Tuple[int, int]):
            b, h = bh
            K[b, h] = keys_block(wl, b, h, Rs[h])
            V[b, h] = values_block(wl, b, h)

        units = [(b, h) for b in range(wl.B) for h in range(wl.H_kv)]
        with ThreadPoolExecutor(_threads(threads)) as ex:
            list(ex.map(job, units))
        out["K"] = K
        out["V"] = V
    if with_cal:
        cal = np.empty((wl.n_cal, wl.H_kv, wl.D), np.float32)
        for h in range(wl.H_kv):
            cal[:, h, :] = calibration_keys(wl, h, Rs[h])
        out["K_cal"] = cal
    return out


def sample_rows(wl: Workload, n: int, seed: int = 7) -> List[Tuple[int, int]]:
    """A seeded sample of (b, h_q) rows, always including the first and last row."""
    rows = wl.B * wl.H_q
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([wl.seed, 99, seed])))
    pick = {0, rows - 1}
    extra = min(n, rows) - len(pick)
    if extra > 0:
        pick.update(1 + int(x) for x in rng.choice(rows - 2, size=extra, replace=False))
    return sorted((r // wl.H_q, r % wl.H_q) for r in pick)


__all__ = [
    "Workload", "WORKLOADS", "sweep_points", "get", "to_cache_dtype", "bf16_bits",
    "sigma", "rotation", "keys_block", "values_block", "query_vec", "calibration_keys",
    "generate", "sample_rows",
]
