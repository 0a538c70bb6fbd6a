"""Loki decode-time sparse attention on B200 (sm_100a): Python binding.

Every function here only marshals torch tensors into the C ABI of libloki.so
(include/loki.h) and allocates outputs and workspaces the caller did not pass;
all arithmetic runs in the library's CUDA kernels on the tensors' device, on
the current torch stream. Names match the C entry points.

Loki ("Loki: Low-Rank Keys for Efficient Sparse Attention"; NeurIPS 2024
poster page, TL;DR and "Visual Insights" Figure 1 caption): keys are cached
rotated by a per-head PCA basis P; at each decode step the query is rotated,
tokens are ranked by their score on the first d principal components, the
top k are kept, and exact softmax attention runs over those k tokens only.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from ._lib import DTYPE_BF16, DTYPE_F32, LIB_PATH, LokiError, check, lib  # noqa: F401

__all__ = [
    "LokiError", "LIB_PATH",
    "loki_calibrate_pca", "loki_append_keys", "loki_decode_attention", "dense_decode_attention",
    "loki_append_keys_plane", "loki_decode_attention_plane", "loki_decode_attention_fused",
    "loki_decode_step", "loki_decode_attention_paged", "loki_append_keys_paged",
    "loki_paged_decode_workspace_size", "loki_pca_attention", "loki_pca_attention_workspace_size",
    "loki_decode_attention_noalloc", "loki_decode_attention_prerotary",
    "loki_append_keys_prerotary", "loki_decode_prerotary_workspace_size",
    "loki_project_query", "loki_score_lowdim", "loki_topk", "loki_sparse_attention",
    "loki_decode_workspace_size", "dense_decode_workspace_size",
    "loki_sparse_attention_workspace_size", "loki_calibrate_workspace_size",
    "loki_topk_workspace_size", "loki_device_error",
]


def loki_device_error(reset: bool = False) -> int:
    """Kernel error word of the current device (0 = no staged wait gave up)."""
    import ctypes
    code = ctypes.c_int(0)
    check(lib.loki_device_error(ctypes.byref(code), int(reset)), "loki_device_error")
    return code.value


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DTYPE_F32
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: use torch.float32 or torch.bfloat16")


def _cuda(*ts: torch.Tensor) -> torch.device:
    dev = ts[0].device
    for t in ts:
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")
        if t.device != dev:
            raise ValueError("all tensors must be on the same device")
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")
    return dev


def _expect(t: torch.Tensor, shape, dtype, name: str) -> None:
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} {list(shape)} (got {t.dtype} {list(t.shape)})")


def _stream(dev: torch.device) -> int:
    return torch.cuda.current_stream(dev).cuda_stream


def _ws(nbytes: int, dev: torch.device, ws: Optional[torch.Tensor]) -> torch.Tensor:
    if ws is None:
        ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    return ws


def _ws_bytes(ws: torch.Tensor) -> int:
    return ws.numel() * ws.element_size()


# ---------------------------------------------------------------------------
# workspace sizes
# ---------------------------------------------------------------------------

def loki_decode_workspace_size(B: int, H_q: int, H_kv: int, S: int, D: int, d: int, k: int) -> int:
    return int(lib.loki_decode_workspace_size(B, H_q, H_kv, S, D, d, k))


def dense_decode_workspace_size(B: int, H_q: int, H_kv: int, S: int, D: int) -> int:
    return int(lib.dense_decode_workspace_size(B, H_q, H_kv, S, D))


def loki_sparse_attention_workspace_size(B: int, H_q: int, k: int, D: int) -> int:
    return int(lib.loki_sparse_attention_workspace_size(B, H_q, k, D))


def loki_calibrate_workspace_size(N: int, H_kv: int, D: int) -> int:
    return int(lib.loki_calibrate_workspace_size(N, H_kv, D))


def loki_topk_workspace_size(rows: int, S: int, k: int) -> int:
    return int(lib.loki_topk_workspace_size(rows, S, k))


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------

def loki_calibrate_pca(keys: torch.Tensor, P: Optional[torch.Tensor] = None,
                       eigvals: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """keys [N, H_kv, D] -> (P [H_kv, D, D] fp32, eigvals [H_kv, D] fp32)."""
    dev = _cuda(keys)
    N, H_kv, D = keys.shape
    if P is None:
        P = torch.empty((H_kv, D, D), dtype=torch.float32, device=dev)
    if eigvals is None:
        eigvals = torch.empty((H_kv, D), dtype=torch.float32, device=dev)
    _cuda(keys, P, eigvals)
    _expect(P, (H_kv, D, D), torch.float32, "P")
    _expect(eigvals, (H_kv, D), torch.float32, "eigvals")
    ws = _ws(loki_calibrate_workspace_size(N, H_kv, D), dev, workspace)
    check(lib.loki_calibrate_pca(keys.data_ptr(), _dt(keys), N, H_kv, D, P.data_ptr(),
                                 eigvals.data_ptr(), ws.data_ptr(), _ws_bytes(ws), _stream(dev)),
          "loki_calibrate_pca")
    return P, eigvals


def loki_append_keys(K_new: torch.Tensor, V_new: torch.Tensor, P: torch.Tensor,
                     Kt_cache: torch.Tensor, V_cache: torch.Tensor, pos: int,
                     Kt_lo: Optional[torch.Tensor] = None) -> None:
    """Rotate K_new [B, H_kv, T, D] by P and write it, with V_new, into cache rows [pos, pos+T).

    With Kt_lo [B, H_kv, S_max, d_lo] the first d_lo rotated columns also go to
    that low-dimensional key plane (loki_append_keys_plane).
    """
    dev = _cuda(K_new, V_new, P, Kt_cache, V_cache)
    B, H_kv, T, D = K_new.shape
    S_max = Kt_cache.shape[2]
    if V_new.shape != K_new.shape or Kt_cache.shape != V_cache.shape:
        raise ValueError("shape mismatch")
    if Kt_cache.shape[:2] != (B, H_kv) or Kt_cache.shape[3] != D:
        raise ValueError("cache shape does not match K_new")
    for t in (V_new, Kt_cache, V_cache):
        if t.dtype != K_new.dtype:
            raise TypeError("K_new, V_new and the caches must share a dtype")
    if P.dtype != torch.float32 or tuple(P.shape) != (H_kv, D, D):
        raise ValueError("P must be float32 [H_kv, D, D]")
    if Kt_lo is None:
        check(lib.loki_append_keys(K_new.data_ptr(), V_new.data_ptr(), P.data_ptr(),
                                   Kt_cache.data_ptr(), V_cache.data_ptr(), B, H_kv, T, D, S_max,
                                   pos, _dt(K_new), _stream(dev)), "loki_append_keys")
        return
    _check_plane(Kt_lo, Kt_cache)
    check(lib.loki_append_keys_plane(K_new.data_ptr(), V_new.data_ptr(), P.data_ptr(),
                                     Kt_cache.data_ptr(), V_cache.data_ptr(), Kt_lo.data_ptr(),
                                     Kt_lo.shape[3], B, H_kv, T, D, S_max, pos, _dt(K_new),
                                     _stream(dev)), "loki_append_keys_plane")


def loki_append_keys_plane(K_new, V_new, P, Kt_cache, V_cache, Kt_lo, pos: int) -> None:
    """loki_append_keys that also fills the low-dimensional key plane Kt_lo."""
    loki_append_keys(K_new, V_new, P, Kt_cache, V_cache, pos, Kt_lo=Kt_lo)


def _check_plane(Kt_lo: torch.Tensor, Kt_cache: torch.Tensor) -> None:
    _cuda(Kt_lo, Kt_cache)
    # the C library takes d_lo from Kt_lo.shape[3] and strides the plane by it
    if Kt_lo.dim() != 4 or Kt_lo.shape[:3] != Kt_cache.shape[:3] or Kt_lo.dtype != Kt_cache.dtype:
        raise ValueError("Kt_lo must be [B, H_kv, S_max, d_lo] with the cache's dtype")


def _check_decode(q, Kt, V, P=None):
    dev = _cuda(q, Kt, V, *(() if P is None else (P,)))
    B, H_q, D = q.shape
    Bk, H_kv, S_max, Dk = Kt.shape
    if Bk != B or Dk != D or V.shape != Kt.shape:
        raise ValueError("q [B, H_q, D] and caches [B, H_kv, S_max, D] disagree")
    if Kt.dtype != q.dtype or V.dtype != q.dtype:
        raise TypeError("q and the caches must share a dtype")
    if P is not None and (P.dtype != torch.float32 or tuple(P.shape) != (H_kv, D, D)):
        raise ValueError("P must be float32 [H_kv, D, D]")
    return dev, B, H_q, H_kv, S_max, D


def loki_decode_attention(q: torch.Tensor, Kt_cache: torch.Tensor, V_cache: torch.Tensor,
                          P: torch.Tensor, S: int, d: int, k: int, scale: float = 0.0,
                          out: Optional[torch.Tensor] = None,
                          selected_idx: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None,
                          Kt_lo: Optional[torch.Tensor] = None
                          ) -> Tuple[torch.Tensor, torch.Tensor]:
    """One Loki decode step. Returns (out [B, H_q, D], selected_idx [B, H_q, k] int32).

    With Kt_lo (a low-dimensional key plane filled by loki_append_keys_plane)
    the score scan reads the plane (loki_decode_attention_plane).
    """
    dev, B, H_q, H_kv, S_max, D = _check_decode(q, Kt_cache, V_cache, P)
    if out is None:
        out = torch.empty_like(q)
    if selected_idx is None:
        selected_idx = torch.empty((B, H_q, k), dtype=torch.int32, device=dev)
    _cuda(q, out, selected_idx)
    _expect(out, q.shape, q.dtype, "out")
    _expect(selected_idx, (B, H_q, k), torch.int32, "selected_idx")
    if S > S_max:
        raise ValueError("S must be <= S_max")
    ws = _ws(loki_decode_workspace_size(B, H_q, H_kv, S, D, d, k), dev, workspace)
    if Kt_lo is None:
        check(lib.loki_decode_attention(q.data_ptr(), Kt_cache.data_ptr(), V_cache.data_ptr(),
                                        P.data_ptr(), B, H_q, H_kv, S, S_max, D, d, k,
                                        float(scale), _dt(q), out.data_ptr(),
                                        selected_idx.data_ptr(), ws.data_ptr(), _ws_bytes(ws),
                                        _stream(dev)), "loki_decode_attention")
    else:
        _check_plane(Kt_lo, Kt_cache)
        check(lib.loki_decode_attention_plane(q.data_ptr(), Kt_cache.data_ptr(),
                                              V_cache.data_ptr(), Kt_lo.data_ptr(),
                                              Kt_lo.shape[3], P.data_ptr(), B, H_q, H_kv, S, S_max,
                                              D, d, k, float(scale), _dt(q), out.data_ptr(),
                                              selected_idx.data_ptr(), ws.data_ptr(),
                                              _ws_bytes(ws), _stream(dev)),
              "loki_decode_attention_plane")
    return out, selected_idx


def loki_decode_attention_plane(q, Kt_cache, V_cache, Kt_lo, P, S: int, d: int, k: int,
                                scale: float = 0.0, out=None, selected_idx=None, workspace=None):
    """loki_decode_attention scoring from the low-dimensional key plane Kt_lo."""
    return loki_decode_attention(q, Kt_cache, V_cache, P, S, d, k, scale, out, selected_idx,
                                 workspace, Kt_lo=Kt_lo)


def loki_decode_step(q: torch.Tensor, K_new: torch.Tensor, V_new: torch.Tensor, P: torch.Tensor,
                     Kt_cache: torch.Tensor, V_cache: torch.Tensor, pos: int, d: int, k: int,
                     scale: float = 0.0, out: Optional[torch.Tensor] = None,
                     selected_idx: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None,
                     Kt_lo: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Append K_new, V_new [B, H_kv, T, D] at cache rows [pos, pos + T) (keys
    rotated by P; also into the key plane Kt_lo when given), then decode over
    the pos + T cached tokens. Returns (out, selected_idx) as loki_decode_attention."""
    dev, B, H_q, H_kv, S_max, D = _check_decode(q, Kt_cache, V_cache, P)
    _cuda(q, K_new, V_new)
    if K_new.dim() != 4 or K_new.shape[:2] != (B, H_kv) or K_new.shape[3] != D:
        raise ValueError("K_new must be [B, H_kv, T, D]")
    if V_new.shape != K_new.shape or K_new.dtype != q.dtype or V_new.dtype != q.dtype:
        raise ValueError("V_new must match K_new, with the caches' dtype")
    T = K_new.shape[2]
    S = pos + T
    if out is None:
        out = torch.empty_like(q)
    if selected_idx is None:
        selected_idx = torch.empty((B, H_q, k), dtype=torch.int32, device=dev)
    _cuda(q, out, selected_idx)
    _expect(out, q.shape, q.dtype, "out")
    _expect(selected_idx, (B, H_q, k), torch.int32, "selected_idx")
    if S > S_max:
        raise ValueError("pos + T must be <= S_max")
    d_lo = 0
    if Kt_lo is not None:
        _check_plane(Kt_lo, Kt_cache)
        d_lo = Kt_lo.shape[3]
    ws = _ws(loki_decode_workspace_size(B, H_q, H_kv, S, D, d, k), dev, workspace)
    check(lib.loki_decode_step(q.data_ptr(), K_new.data_ptr(), V_new.data_ptr(), P.data_ptr(),
                               Kt_cache.data_ptr(), V_cache.data_ptr(),
                               Kt_lo.data_ptr() if Kt_lo is not None else None, d_lo, B, H_q,
                               H_kv, T, pos, S_max, D, d, k, float(scale), _dt(q), out.data_ptr(),
                               selected_idx.data_ptr(), ws.data_ptr(), _ws_bytes(ws),
                               _stream(dev)), "loki_decode_step")
    return out, selected_idx


def loki_paged_decode_workspace_size(B: int, H_q: int, H_kv: int, page_size: int,
                                     max_pages: int, D: int, d: int, k: int) -> int:
    return int(lib.loki_paged_decode_workspace_size(B, H_q, H_kv, page_size, max_pages, D, d, k))


def _check_pages(Kt_pages, V_pages, Kt_lo_pages, block_table):
    if Kt_pages.dim() != 4 or V_pages.shape != Kt_pages.shape:
        raise ValueError("Kt_pages and V_pages must be [n_pages, H_kv, page_size, D]")
    if Kt_lo_pages is not None and (Kt_lo_pages.dim() != 4 or
                                    Kt_lo_pages.shape[:3] != Kt_pages.shape[:3] or
                                    Kt_lo_pages.dtype != Kt_pages.dtype):
        raise ValueError("Kt_lo_pages must be [n_pages, H_kv, page_size, d_lo] with the pages' dtype")
    if block_table.dtype != torch.int32 or block_table.dim() != 2:
        raise TypeError("block_table must be int32 [B, max_pages]")
    return Kt_pages.shape


def loki_decode_attention_paged(q: torch.Tensor, Kt_pages: torch.Tensor, V_pages: torch.Tensor,
                                Kt_lo_pages: torch.Tensor, P: torch.Tensor,
                                block_table: torch.Tensor, seq_lens: torch.Tensor, d: int, k: int,
                                scale: float = 0.0, out: Optional[torch.Tensor] = None,
                                selected_idx: Optional[torch.Tensor] = None,
                                workspace: Optional[torch.Tensor] = None
                                ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Decode a ragged batch over a paged cache (see include/loki.h).
    Returns (out [B, H_q, D], selected_idx [B, H_q, k] int32, -1 padded)."""
    dev = _cuda(q, Kt_pages, V_pages, Kt_lo_pages, P, block_table, seq_lens)
    n_pages, H_kv, page_size, D = _check_pages(Kt_pages, V_pages, Kt_lo_pages, block_table)
    B, H_q, Dq = q.shape
    if Dq != D or block_table.shape[0] != B or tuple(seq_lens.shape) != (B,):
        raise ValueError("q [B, H_q, D], block_table [B, max_pages], seq_lens [B] disagree")
    if seq_lens.dtype != torch.int32:
        raise TypeError("seq_lens must be int32")
    if Kt_pages.dtype != q.dtype or V_pages.dtype != q.dtype:
        raise TypeError("q and the pages must share a dtype")
    max_pages = block_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if selected_idx is None:
        selected_idx = torch.empty((B, H_q, k), dtype=torch.int32, device=dev)
    _cuda(q, out, selected_idx)
    _expect(out, q.shape, q.dtype, "out")
    _expect(selected_idx, (B, H_q, k), torch.int32, "selected_idx")
    ws = _ws(loki_paged_decode_workspace_size(B, H_q, H_kv, page_size, max_pages, D, d, k), dev,
             workspace)
    check(lib.loki_decode_attention_paged(q.data_ptr(), Kt_pages.data_ptr(), V_pages.data_ptr(),
                                          Kt_lo_pages.data_ptr(), Kt_lo_pages.shape[3],
                                          P.data_ptr(), block_table.data_ptr(),
                                          seq_lens.data_ptr(), B, H_q, H_kv, page_size, max_pages,
                                          n_pages, D, d, k, float(scale), _dt(q), out.data_ptr(),
                                          selected_idx.data_ptr(), ws.data_ptr(), _ws_bytes(ws),
                                          _stream(dev)), "loki_decode_attention_paged")
    return out, selected_idx


def loki_append_keys_paged(K_new: torch.Tensor, V_new: torch.Tensor, P: torch.Tensor,
                           Kt_pages: torch.Tensor, V_pages: torch.Tensor,
                           block_table: torch.Tensor, positions: torch.Tensor,
                           Kt_lo_pages: Optional[torch.Tensor] = None) -> None:
    """Rotate K_new [B, H_kv, T, D] by P into the page pool at tokens positions[b] + t."""
    dev = _cuda(K_new, V_new, P, Kt_pages, V_pages, block_table, positions,
                *(() if Kt_lo_pages is None else (Kt_lo_pages,)))
    n_pages, H_kv, page_size, D = _check_pages(Kt_pages, V_pages, Kt_lo_pages, block_table)
    B, Hk, T, Dk = K_new.shape
    if Hk != H_kv or Dk != D or V_new.shape != K_new.shape or tuple(positions.shape) != (B,):
        raise ValueError("K_new, V_new [B, H_kv, T, D] and positions [B] must match the pages")
    if positions.dtype != torch.int32:
        raise TypeError("positions must be int32")
    for t in (V_new, Kt_pages, V_pages):
        if t.dtype != K_new.dtype:
            raise TypeError("K_new, V_new and the pages must share a dtype")
    check(lib.loki_append_keys_paged(K_new.data_ptr(), V_new.data_ptr(), P.data_ptr(),
                                     Kt_pages.data_ptr(), V_pages.data_ptr(),
                                     Kt_lo_pages.data_ptr() if Kt_lo_pages is not None else None,
                                     Kt_lo_pages.shape[3] if Kt_lo_pages is not None else 0,
                                     block_table.data_ptr(), positions.data_ptr(), B, H_kv, T,
                                     page_size, block_table.shape[1], n_pages, D, _dt(K_new),
                                     _stream(dev)), "loki_append_keys_paged")


def loki_decode_attention_fused(q: torch.Tensor, Kt_cache: torch.Tensor, V_cache: torch.Tensor,
                                Kt_lo: torch.Tensor, P: torch.Tensor, S: int, d: int, k: int,
                                scale: float = 0.0, out: Optional[torch.Tensor] = None,
                                selected_idx: Optional[torch.Tensor] = None
                                ) -> Tuple[torch.Tensor, torch.Tensor]:
    """loki_decode_attention_plane as one kernel per (batch, KV head) unit
    (scores kept on chip; no workspace). Raises LokiError(LOKI_ERR_UNSUPPORTED)
    for shapes outside the kernel's limits (see include/loki.h)."""
    dev, B, H_q, H_kv, S_max, D = _check_decode(q, Kt_cache, V_cache, P)
    if out is None:
        out = torch.empty_like(q)
    if selected_idx is None:
        selected_idx = torch.empty((B, H_q, k), dtype=torch.int32, device=dev)
    _cuda(q, out, selected_idx)
    _expect(out, q.shape, q.dtype, "out")
    _expect(selected_idx, (B, H_q, k), torch.int32, "selected_idx")
    if S > S_max:
        raise ValueError("S must be <= S_max")
    _check_plane(Kt_lo, Kt_cache)
    check(lib.loki_decode_attention_fused(q.data_ptr(), Kt_cache.data_ptr(), V_cache.data_ptr(),
                                          Kt_lo.data_ptr(), Kt_lo.shape[3], P.data_ptr(), B, H_q,
                                          H_kv, S, S_max, D, d, k, float(scale), _dt(q),
                                          out.data_ptr(), selected_idx.data_ptr(), _stream(dev)),
          "loki_decode_attention_fused")
    return out, selected_idx


def loki_decode_attention_noalloc(q: torch.Tensor, Kt_cache: torch.Tensor, V_cache: torch.Tensor,
                                  P: torch.Tensor, S: int, d: int, k: int, scale: float = 0.0,
                                  out: Optional[torch.Tensor] = None,
                                  selected_idx: Optional[torch.Tensor] = None
                                  ) -> Tuple[torch.Tensor, torch.Tensor]:
    """loki_decode_attention with no workspace: the library's built-in scratch
    array is used (for callers that cannot allocate device memory; see
    include/loki.h for its limit and sharing rules)."""
    dev, B, H_q, H_kv, S_max, D = _check_decode(q, Kt_cache, V_cache, P)
    if out is None:
        out = torch.empty_like(q)
    if selected_idx is None:
        selected_idx = torch.empty((B, H_q, k), dtype=torch.int32, device=dev)
    _cuda(q, out, selected_idx)
    _expect(out, q.shape, q.dtype, "out")
    _expect(selected_idx, (B, H_q, k), torch.int32, "selected_idx")
    check(lib.loki_decode_attention_noalloc(q.data_ptr(), Kt_cache.data_ptr(), V_cache.data_ptr(),
                                            P.data_ptr(), B, H_q, H_kv, S, S_max, D, d, k,
                                            float(scale), _dt(q), out.data_ptr(),
                                            selected_idx.data_ptr(), _stream(dev)),
          "loki_decode_attention_noalloc")
    return out, selected_idx


def loki_project_query(q: torch.Tensor, P: torch.Tensor,
                       q_rot: Optional[torch.Tensor] = None) -> torch.Tensor:
    """q [B, H_q, D] -> q~ = q P, fp32 [B, H_q, D]."""
    dev = _cuda(q, P)
    B, H_q, D = q.shape
    H_kv = P.shape[0]
    _expect(P, (H_kv, D, D), torch.float32, "P")
    if q_rot is None:
        q_rot = torch.empty((B, H_q, D), dtype=torch.float32, device=dev)
    _cuda(q, q_rot)
    _expect(q_rot, (B, H_q, D), torch.float32, "q_rot")
    check(lib.loki_project_query(q.data_ptr(), P.data_ptr(), B, H_q, H_kv, D, _dt(q),
                                 q_rot.data_ptr(), _stream(dev)), "loki_project_query")
    return q_rot


def loki_score_lowdim(q_rot: torch.Tensor, Kt_cache: torch.Tensor, S: int, d: int,
                      scores: Optional[torch.Tensor] = None) -> torch.Tensor:
    """fp32 scores [B, H_q, S] on the first d rotated dimensions.

    Kt_cache is the rotated cache [B, H_kv, S_max, D] of heads of D = 128 or
    96 (q_rot is then [B, H_q, D]), or a low-dimensional key plane
    [B, H_kv, S_max, d_lo] of 128-wide heads (q_rot [B, H_q, 128]); its last
    dimension is the row width the scan strides by.
    """
    dev = _cuda(q_rot, Kt_cache)
    B, H_q, Dq = q_rot.shape
    Bk, H_kv, S_max, row = Kt_cache.shape
    want = row if row in (96, 128) else 128
    if q_rot.dtype != torch.float32 or Dq != want:
        raise TypeError(f"q_rot must be float32 [B, H_q, {want}]")
    if Bk != B or not 1 <= d <= row or S > S_max:
        raise ValueError("Kt_cache must be [B, H_kv, S_max >= S, row >= d]")
    if scores is None:
        scores = torch.empty((B, H_q, S), dtype=torch.float32, device=dev)
    if scores.shape != (B, H_q, S) or scores.dtype != torch.float32:
        raise ValueError("scores must be float32 [B, H_q, S]")
    _cuda(q_rot, scores)
    check(lib.loki_score_lowdim(q_rot.data_ptr(), Kt_cache.data_ptr(), B, H_q, H_kv, S, S_max, row,
                                d, _dt(Kt_cache), scores.data_ptr(), _stream(dev)),
          "loki_score_lowdim")
    return scores


def loki_topk(scores: torch.Tensor, k: int, selected_idx: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Per row of scores [..., S] fp32: k indices of the largest values (ties: lower index), ascending."""
    dev = _cuda(scores)
    if scores.dtype != torch.float32:
        raise TypeError("scores must be float32")
    S = scores.shape[-1]
    rows = scores.numel() // S
    if selected_idx is None:
        selected_idx = torch.empty((*scores.shape[:-1], k), dtype=torch.int32, device=dev)
    _cuda(scores, selected_idx)
    _expect(selected_idx, (*scores.shape[:-1], k), torch.int32, "selected_idx")
    ws = _ws(loki_topk_workspace_size(rows, S, k), dev, None)
    check(lib.loki_topk(scores.data_ptr(), rows, S, k, selected_idx.data_ptr(), ws.data_ptr(),
                        _ws_bytes(ws), _stream(dev)), "loki_topk")
    return selected_idx


def loki_sparse_attention(q_rot: torch.Tensor, Kt_cache: torch.Tensor, V_cache: torch.Tensor,
                          selected_idx: torch.Tensor, S: int, scale: float = 0.0,
                          out: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Exact attention of q~ over the selected tokens; out has the caches' dtype."""
    dev = _cuda(q_rot, Kt_cache, V_cache, selected_idx)
    B, H_q, D = q_rot.shape
    Bk, H_kv, S_max, Dk = Kt_cache.shape
    k = selected_idx.shape[-1]
    _expect(q_rot, (B, H_q, D), torch.float32, "q_rot")
    _expect(V_cache, Kt_cache.shape, Kt_cache.dtype, "V_cache")
    _expect(selected_idx, (B, H_q, k), torch.int32, "selected_idx")
    if Bk != B or Dk != D or S > S_max:
        raise ValueError("Kt_cache must be [B, H_kv, S_max >= S, D]")
    if out is None:
        out = torch.empty((B, H_q, D), dtype=Kt_cache.dtype, device=dev)
    _cuda(q_rot, out)
    _expect(out, (B, H_q, D), Kt_cache.dtype, "out")
    ws = _ws(loki_sparse_attention_workspace_size(B, H_q, k, D), dev, workspace)
    check(lib.loki_sparse_attention(q_rot.data_ptr(), Kt_cache.data_ptr(), V_cache.data_ptr(),
                                    selected_idx.data_ptr(), B, H_q, H_kv, S, S_max, D, k,
                                    float(scale), _dt(Kt_cache), out.data_ptr(), ws.data_ptr(),
                                    _ws_bytes(ws), _stream(dev)), "loki_sparse_attention")
    return out


def loki_pca_attention_workspace_size(B: int, H_q: int, H_kv: int, S: int, D: int) -> int:
    return int(lib.loki_pca_attention_workspace_size(B, H_q, H_kv, S, D))


def loki_pca_attention(q: torch.Tensor, Kt_lo: torch.Tensor, V_cache: torch.Tensor,
                       P: torch.Tensor, S: int, d: int, scale: float = 0.0,
                       out: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """PCAAttn: softmax over the d-dimensional scores of all S tokens (keys from
    the key plane Kt_lo [B, H_kv, S_max, d_lo]), times the values."""
    dev, B, H_q, H_kv, S_max, D = _check_decode(q, V_cache, V_cache, P)
    _check_plane(Kt_lo, V_cache)
    if out is None:
        out = torch.empty_like(q)
    _cuda(q, out)
    _expect(out, q.shape, q.dtype, "out")
    if S > S_max:
        raise ValueError("S must be <= S_max")
    ws = _ws(loki_pca_attention_workspace_size(B, H_q, H_kv, S, D), dev, workspace)
    check(lib.loki_pca_attention(q.data_ptr(), Kt_lo.data_ptr(), Kt_lo.shape[3],
                                 V_cache.data_ptr(), P.data_ptr(), B, H_q, H_kv, S, S_max, D, d,
                                 float(scale), _dt(q), out.data_ptr(), ws.data_ptr(),
                                 _ws_bytes(ws), _stream(dev)), "loki_pca_attention")
    return out


def loki_decode_prerotary_workspace_size(B: int, H_q: int, H_kv: int, S: int, D: int, d: int,
                                         k: int) -> int:
    return int(lib.loki_decode_prerotary_workspace_size(B, H_q, H_kv, S, D, d, k))


def loki_decode_attention_prerotary(q_pre: torch.Tensor, q_post: torch.Tensor,
                                    K_cache: torch.Tensor, V_cache: torch.Tensor,
                                    Kt_lo: torch.Tensor, P: torch.Tensor, S: int, d: int, k: int,
                                    scale: float = 0.0, out: Optional[torch.Tensor] = None,
                                    selected_idx: Optional[torch.Tensor] = None,
                                    workspace: Optional[torch.Tensor] = None
                                    ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Pre-rotary variant: select on q_pre P against the plane Kt_lo of the
    rotated pre-rotary keys, attend with q_post over the post-rotary keys
    K_cache. Returns (out [B, H_q, D], selected_idx [B, H_q, k] int32)."""
    dev, B, H_q, H_kv, S_max, D = _check_decode(q_pre, K_cache, V_cache, P)
    _expect(q_post, q_pre.shape, q_pre.dtype, "q_post")
    _cuda(q_pre, q_post)
    _check_plane(Kt_lo, K_cache)
    if out is None:
        out = torch.empty_like(q_pre)
    if selected_idx is None:
        selected_idx = torch.empty((B, H_q, k), dtype=torch.int32, device=dev)
    _cuda(q_pre, out, selected_idx)
    _expect(out, q_pre.shape, q_pre.dtype, "out")
    _expect(selected_idx, (B, H_q, k), torch.int32, "selected_idx")
    if S > S_max:
        raise ValueError("S must be <= S_max")
    ws = _ws(loki_decode_prerotary_workspace_size(B, H_q, H_kv, S, D, d, k), dev, workspace)
    check(lib.loki_decode_attention_prerotary(
        q_pre.data_ptr(), q_post.data_ptr(), K_cache.data_ptr(), V_cache.data_ptr(),
        Kt_lo.data_ptr(), Kt_lo.shape[3], P.data_ptr(), B, H_q, H_kv, S, S_max, D, d, k,
        float(scale), _dt(q_pre), out.data_ptr(), selected_idx.data_ptr(), ws.data_ptr(),
        _ws_bytes(ws), _stream(dev)), "loki_decode_attention_prerotary")
    return out, selected_idx


def loki_append_keys_prerotary(K_new_pre: torch.Tensor, K_new_post: torch.Tensor,
                               V_new: torch.Tensor, P: torch.Tensor, K_cache: torch.Tensor,
                               V_cache: torch.Tensor, Kt_lo: torch.Tensor, pos: int) -> None:
    """Append of the pre-rotary variant: (K_new_pre P)[:, :d_lo] to the plane,
    K_new_post and V_new unchanged to the caches, at rows [pos, pos + T)."""
    dev = _cuda(K_new_pre, K_new_post, V_new, P, K_cache, V_cache)
    B, H_kv, T, D = K_new_pre.shape
    S_max = K_cache.shape[2]
    for t in (K_new_post, V_new):
        _expect(t, K_new_pre.shape, K_new_pre.dtype, "K_new_post / V_new")
    _expect(V_cache, K_cache.shape, K_new_pre.dtype, "V_cache")
    if K_cache.dtype != K_new_pre.dtype or K_cache.shape[:2] != (B, H_kv) or K_cache.shape[3] != D:
        raise ValueError("K_cache must be [B, H_kv, S_max, D] of the new keys' dtype")
    if P.dtype != torch.float32 or tuple(P.shape) != (H_kv, D, D):
        raise ValueError("P must be float32 [H_kv, D, D]")
    _check_plane(Kt_lo, K_cache)
    check(lib.loki_append_keys_prerotary(
        K_new_pre.data_ptr(), K_new_post.data_ptr(), V_new.data_ptr(), P.data_ptr(),
        K_cache.data_ptr(), V_cache.data_ptr(), Kt_lo.data_ptr(), Kt_lo.shape[3], B, H_kv, T, D,
        S_max, pos, _dt(K_new_pre), _stream(dev)), "loki_append_keys_prerotary")


def dense_decode_attention(q: torch.Tensor, K_cache: torch.Tensor, V_cache: torch.Tensor, S: int,
                           scale: float = 0.0, out: Optional[torch.Tensor] = None,
                           workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Full decode attention over all S cached tokens."""
    dev, B, H_q, H_kv, S_max, D = _check_decode(q, K_cache, V_cache)
    if out is None:
        out = torch.empty_like(q)
    _cuda(q, out)
    _expect(out, q.shape, q.dtype, "out")
    if S > S_max:
        raise ValueError("S must be <= S_max")
    ws = _ws(dense_decode_workspace_size(B, H_q, H_kv, S, D), dev, workspace)
    check(lib.dense_decode_attention(q.data_ptr(), K_cache.data_ptr(), V_cache.data_ptr(), B, H_q,
                                     H_kv, S, S_max, D, float(scale), _dt(q), out.data_ptr(),
                                     ws.data_ptr(), _ws_bytes(ws), _stream(dev)),
          "dense_decode_attention")
    return out
