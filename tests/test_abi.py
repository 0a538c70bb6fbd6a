"""The C ABI without a GPU: the library loads, exports every declared entry
point, and rejects bad arguments on the host before touching CUDA.

Pointers passed here are fake (never dereferenced): every call below fails
argument validation, which runs before any CUDA call.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "loki.h")


def _declared():
    src = open(HEADER).read()
    return re.findall(r"LOKI_API\s+(?:const\s+char\s*\*|size_t|loki_status)\s+(\w+)\s*\(", src)


@pytest.fixture(scope="module")
def L():
    from sparse_attention_decode_loki_b200 import _lib
    return _lib


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L.lib, n), n
        assert n in L.PROTOTYPES, n
    assert sorted(L.PROTOTYPES) == sorted(names)


def test_status_strings(L):
    for code, name in L.STATUS.items():
        assert L.lib.loki_status_string(code).decode().startswith(name)


FAKE = 1 << 20  # 16- and 256-byte aligned, never dereferenced


def _decode(L, **kw):
    a = dict(q=FAKE, Kt=FAKE, V=FAKE, P=FAKE, B=2, H_q=4, H_kv=2, S=100, S_max=128, D=128, d=32,
             k=10, scale=0.0, dt=L.DTYPE_BF16, out=FAKE, idx=FAKE, ws=FAKE, ws_bytes=0,
             stream=None)
    a.update(kw)
    return L.lib.loki_decode_attention(a["q"], a["Kt"], a["V"], a["P"], a["B"], a["H_q"],
                                       a["H_kv"], a["S"], a["S_max"], a["D"], a["d"], a["k"],
                                       a["scale"], a["dt"], a["out"], a["idx"], a["ws"],
                                       a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(d=0), 1), (dict(d=129), 1), (dict(k=0), 1), (dict(k=101), 1),
    (dict(S=0), 1), (dict(S=200), 1), (dict(H_q=3), 1), (dict(H_q=32, H_kv=2), 2),
    (dict(D=64), 2), (dict(dt=7), 1), (dict(q=None), 1), (dict(Kt=None), 1),
    (dict(out=FAKE + 2), 1), (dict(idx=FAKE + 2), 1), (dict(ws=FAKE + 16), 1),
    (dict(B=0), 1), (dict(S=1 << 31, S_max=1 << 32, k=5), 2),
])
def test_decode_rejects_bad_arguments(L, kw, status):
    assert _decode(L, **kw) == status
    assert L.lib.loki_last_error().decode() != ""


def test_decode_rejects_short_workspace(L):
    need = L.lib.loki_decode_workspace_size(2, 4, 2, 100, 128, 32, 10)
    assert need > 0
    assert _decode(L, ws_bytes=need - 1) == 3
    assert "workspace" in L.lib.loki_last_error().decode()


def test_workspace_sizes_grow_with_problem(L):
    a = L.lib.loki_decode_workspace_size(1, 32, 32, 4096, 128, 32, 1024)
    b = L.lib.loki_decode_workspace_size(16, 40, 40, 4096, 128, 32, 512)
    assert 0 < a < b
    # scores dominate: B * H_q * S fp32 must fit
    assert b >= 16 * 40 * 4096 * 4
    assert L.lib.dense_decode_workspace_size(16, 40, 40, 4096, 128) > 0
    assert L.lib.loki_sparse_attention_workspace_size(16, 40, 512, 128) > 0
    assert L.lib.loki_calibrate_workspace_size(4096, 40, 128) >= 2 * 40 * 128 * 128 * 8
    assert L.lib.loki_decode_workspace_size(0, 1, 1, 1, 128, 1, 1) == 0


def test_other_entry_points_reject_bad_arguments(L):
    lib = L.lib
    # append: pos + T beyond S_max
    assert lib.loki_append_keys(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 4, 128, 10, 8,
                                L.DTYPE_BF16, None) == 1
    # calibrate: N < 2, D not a multiple of 16
    ws = lib.loki_calibrate_workspace_size(100, 2, 128)
    assert lib.loki_calibrate_pca(FAKE, L.DTYPE_F32, 1, 2, 128, FAKE, None, FAKE, ws, None) == 1
    assert lib.loki_calibrate_pca(FAKE, L.DTYPE_F32, 100, 2, 100, FAKE, None, FAKE, ws, None) == 2
    assert lib.loki_calibrate_pca(FAKE, L.DTYPE_F32, 100, 2, 128, FAKE, None, FAKE, ws - 1,
                                  None) == 3
    # topk: k > S, rows < 1
    assert lib.loki_topk(FAKE, 4, 10, 11, FAKE, None, 0, None) == 1
    assert lib.loki_topk(FAKE, 0, 10, 1, FAKE, None, 0, None) == 1
    # score: d out of range
    assert lib.loki_score_lowdim(FAKE, FAKE, 1, 1, 1, 10, 10, 128, 0, L.DTYPE_BF16, FAKE,
                                 None) == 1
    # sparse attention: workspace too small
    assert lib.loki_sparse_attention(FAKE, FAKE, FAKE, FAKE, 1, 1, 1, 10, 10, 128, 4, 0.0,
                                     L.DTYPE_BF16, FAKE, FAKE, 0, None) == 3
    # dense: H_q not a multiple of H_kv
    assert lib.dense_decode_attention(FAKE, FAKE, FAKE, 1, 3, 2, 10, 10, 128, 0.0,
                                      L.DTYPE_BF16, FAKE, FAKE, 1 << 20, None) == 1
    # project: misaligned output
    assert lib.loki_project_query(FAKE, FAKE, 1, 1, 1, 128, L.DTYPE_F32, FAKE + 4, None) == 1


def test_plane_entry_points_reject_bad_arguments(L):
    lib = L.lib
    ws = lib.loki_decode_workspace_size(1, 2, 2, 100, 128, 32, 10)

    def args(**kw):
        return dict(dict(Kt_lo=FAKE, d_lo=32, d=32), **kw)

    def dec(Kt_lo, d_lo, d):
        return lib.loki_decode_attention_plane(FAKE, FAKE, FAKE, Kt_lo, d_lo, FAKE, 1, 2, 2, 100,
                                               100, 128, d, 10, 0.0, L.DTYPE_BF16, FAKE, FAKE,
                                               FAKE, ws, None)
    assert dec(**args(d=33)) == 1            # d > d_lo
    assert dec(**args(d_lo=20, d=16)) == 1   # d_lo * 2 bytes not a multiple of 16
    assert dec(**args(Kt_lo=None)) == 1
    assert dec(**args(Kt_lo=FAKE + 8)) == 1  # misaligned plane
    assert lib.loki_append_keys_plane(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 129, 1, 2, 1, 128, 10,
                                      0, L.DTYPE_BF16, None) == 1
    # the score scan takes a plane's row width: rows must be a multiple of 16 bytes
    # (20 bf16 = 40 bytes is not) and hold at least d columns
    assert lib.loki_score_lowdim(FAKE, FAKE, 1, 1, 1, 10, 10, 20, 8, L.DTYPE_BF16, FAKE,
                                 None) == 1
    assert lib.loki_score_lowdim(FAKE, FAKE, 1, 1, 1, 10, 10, 24, 25, L.DTYPE_BF16, FAKE,
                                 None) == 1


def test_python_binding_requires_cuda_tensors():
    torch = pytest.importorskip("torch")
    import sparse_attention_decode_loki_b200 as loki
    q = torch.zeros(1, 1, 128)
    with pytest.raises(ValueError):
        loki.dense_decode_attention(q, torch.zeros(1, 1, 4, 128), torch.zeros(1, 1, 4, 128), 4)


def test_fused_entry_point_rejects_bad_arguments(L):
    lib = L.lib

    def dec(**kw):
        a = dict(Kt_lo=FAKE, d_lo=32, H_q=2, H_kv=2, S=100, d=32, k=10, out=FAKE)
        a.update(kw)
        return lib.loki_decode_attention_fused(FAKE, FAKE, FAKE, a["Kt_lo"], a["d_lo"], FAKE, 1,
                                               a["H_q"], a["H_kv"], a["S"], 100, 128, a["d"],
                                               a["k"], 0.0, L.DTYPE_BF16, a["out"], FAKE, None)
    assert dec(d=33) == 1              # d > d_lo
    assert dec(d_lo=20, d=16) == 1     # plane row not a multiple of 16 bytes
    assert dec(Kt_lo=None) == 1
    assert dec(k=0) == 1
    assert dec(k=101) == 1             # k > S
    assert dec(H_q=3) == 1             # H_q not a multiple of H_kv
    assert dec(out=FAKE + 2) == 1      # misaligned output
    assert L.lib.loki_last_error().decode() != ""


def test_paged_entry_points_reject_bad_arguments(L):
    f = 1 << 20  # fake, 1 MiB-aligned device pointers (never dereferenced)
    ws = L.lib.loki_paged_decode_workspace_size(2, 4, 4, 16, 8, 128, 32, 64)
    assert ws > 0

    def dec(page_size=16, max_pages=8, n_pages=20, d_lo=32, d=32, k=64, q=f, H_q=4, H_kv=4):
        return L.lib.loki_decode_attention_paged(q, f, f, f, d_lo, f, f, f, 2, H_q, H_kv, page_size,
                                                 max_pages, n_pages, 128, d, k, 0.0, L.DTYPE_BF16,
                                                 f, f, f, ws, None)

    assert dec(page_size=0) == 1
    assert dec(n_pages=0) == 1
    assert dec(d=40) == 1                     # d > d_lo
    assert dec(k=16 * 8 + 1) == 1             # k beyond page_size * max_pages
    assert dec(d_lo=128, d=32) == 2           # plane rows the paged scan does not take
    assert dec(H_q=16, H_kv=2, d_lo=32) == 2  # G * d_lo > 64
    assert dec(page_size=4096, max_pages=128, k=64) == 2  # more than 262144 tokens
    assert dec(q=f + 2) == 1                  # misaligned
    assert L.lib.loki_decode_attention_paged(f, f, f, f, 32, f, f, f, 2, 4, 4, 16, 8, 20, 128,
                                             32, 64, 0.0, L.DTYPE_BF16, f, f, f, ws - 1, None) == 3
    # the append
    assert L.lib.loki_append_keys_paged(f, f, f, f, f, None, 0, f, f, 2, 4, 0, 16, 8, 20, 128,
                                        L.DTYPE_BF16, None) == 1  # T = 0
    assert L.lib.loki_append_keys_paged(f, f, f, f, f, f, 12, f, f, 2, 4, 1, 16, 8, 20, 128,
                                        L.DTYPE_BF16, None) == 1  # plane row of 24 bytes
    assert L.lib.loki_append_keys_paged(f, f, f, f, f, None, 0, f, f + 1, 2, 4, 1, 16, 8, 20, 128,
                                        L.DTYPE_BF16, None) == 1  # misaligned positions


def test_decode_step_rejects_bad_arguments_on_the_host(L):
    f = 1 << 20
    ws = L.lib.loki_decode_workspace_size(1, 2, 2, 64, 128, 32, 8)
    # T = 0, a NULL new key, k > pos + T
    assert L.lib.loki_decode_step(f, f, f, f, f, f, None, 0, 1, 2, 2, 0, 10, 64, 128, 32, 8, 0.0,
                                  L.DTYPE_BF16, f, f, f, ws, None) == 1
    assert L.lib.loki_decode_step(f, None, f, f, f, f, None, 0, 1, 2, 2, 1, 10, 64, 128, 32, 8,
                                  0.0, L.DTYPE_BF16, f, f, f, ws, None) == 1
    assert L.lib.loki_decode_step(f, f, f, f, f, f, None, 0, 1, 2, 2, 1, 2, 64, 128, 32, 8, 0.0,
                                  L.DTYPE_BF16, f, f, f, ws, None) == 1
