"""loki_decode_attention_noalloc: the decode step for callers that cannot
allocate device memory (a plugin inside a framework that owns every device
allocation, a thread that must not call cudaMalloc / cudaFree because they can
synchronise the device). Its scratch comes from a fixed 32 MiB array built into
the library instead of a caller workspace.

The GPU test calls it through the C ABI twice in a row and checks both results
against the workspace entry point on the same inputs, with the tolerances of
the parity tests. This file is named so that pytest collects it last.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest

import workloads
from tests import parity


def _lib():
    from sparse_attention_decode_loki_b200 import _lib as L
    return L


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point(cuda):
    import torch
    L = _lib()
    wl = workloads.get("llama2-7b").with_(B=2, H_q=8, H_kv=4, S=1500, d=32, k=200, n_cal=512,
                                          name="noalloc")
    inp = parity.host_inputs(wl)
    S_max = 1536
    q = parity.to_device(inp.q, wl, cuda)
    Kt = parity.to_device(inp.Kt, wl, cuda, S_max=S_max)
    V = parity.to_device(inp.V, wl, cuda, S_max=S_max)
    P = torch.from_numpy(inp.P).to(cuda)
    dt = L.DTYPE_BF16
    stream = torch.cuda.current_stream(cuda).cuda_stream
    args = (q.data_ptr(), Kt.data_ptr(), V.data_ptr(), P.data_ptr(), wl.B, wl.H_q, wl.H_kv, wl.S,
            S_max, wl.D, wl.d, wl.k, wl.scale)

    # the existing entry point with a caller-provided workspace
    ws_bytes = L.lib.loki_decode_workspace_size(wl.B, wl.H_q, wl.H_kv, wl.S, wl.D, wl.d, wl.k)
    assert 0 < ws_bytes <= (32 << 20)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=cuda)
    out_ref = torch.empty_like(q)
    idx_ref = torch.empty((wl.B, wl.H_q, wl.k), dtype=torch.int32, device=cuda)
    st = L.lib.loki_decode_attention(*args, dt, out_ref.data_ptr(), idx_ref.data_ptr(),
                                     ws.data_ptr(), ws_bytes, stream)
    assert st == 0, L.lib.loki_last_error()
    torch.cuda.synchronize()
    out_ref = out_ref.float().cpu().numpy()
    idx_ref = idx_ref.cpu().numpy()

    # two calls in a row through the built-in scratch; the second one starts
    # from whatever the first left in the shared array
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        idx = torch.full((wl.B, wl.H_q, wl.k), -1, dtype=torch.int32, device=cuda)
        st = L.lib.loki_decode_attention_noalloc(*args, dt, out.data_ptr(), idx.data_ptr(), stream)
        assert st == 0, (call, L.lib.loki_last_error())
        torch.cuda.synchronize()
        # no staged kernel's bounded wait gave up during the call
        code = ctypes.c_int(-1)
        assert L.lib.loki_device_error(ctypes.byref(code), 1) == 0
        assert code.value == 0, call
        idx_h = idx.cpu().numpy()
        out_h = out.float().cpu().numpy()
        assert np.array_equal(idx_h, idx_ref), call
        assert np.abs(out_h - out_ref).max() <= parity.OUT_TOL[wl.dtype], call


def test_noalloc_rejects_decodes_larger_than_its_scratch():
    # 64 x 40 rows of 131072 fp32 scores alone need 1.3 GB: rejected on the
    # host before any CUDA call (the pointers are never used)
    L = _lib()
    fake = 1 << 20
    st = L.lib.loki_decode_attention_noalloc(fake, fake, fake, fake, 64, 40, 40, 131072, 131072,
                                             128, 32, 16384, 0.0, L.DTYPE_BF16, fake, fake, None)
    assert st == 2
    assert "32 MiB" in L.lib.loki_last_error().decode()
