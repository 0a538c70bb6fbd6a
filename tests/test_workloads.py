"""The seeded input generator: determinism, block independence, dtype exactness."""
import math

import numpy as np

import workloads


def test_blocks_are_deterministic_and_independent():
    wl = workloads.get("tiny").with_(B=2, H_q=2, H_kv=2, S=64)
    a = workloads.keys_block(wl, 1, 1)
    b = workloads.keys_block(wl, 1, 1)
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, workloads.keys_block(wl, 0, 1))
    full = workloads.generate(wl, threads=2)
    np.testing.assert_array_equal(full["K"][1, 1], a)
    np.testing.assert_array_equal(full["V"][0, 1], workloads.values_block(wl, 0, 1))
    np.testing.assert_array_equal(full["q"][1, 0], workloads.query_vec(wl, 1, 0))
    assert full["K_cal"].shape == (wl.n_cal, 2, wl.D)


def test_bf16_values_are_exact():
    wl = workloads.get("llama2-7b").with_(S=128, H_q=2, H_kv=2)
    K = workloads.keys_block(wl, 0, 0)
    bits = workloads.bf16_bits(K)
    back = (bits.astype(np.uint32) << 16).view(np.float32)
    np.testing.assert_array_equal(back, K)


def test_rotation_is_orthogonal():
    wl = workloads.get("llama3-8b-gqa")
    R = workloads.rotation(wl, 3)
    np.testing.assert_allclose(R.T @ R, np.eye(wl.D), atol=1e-12)


def test_gqa_queries_use_their_kv_head_basis():
    wl = workloads.get("llama3-8b-gqa")
    # the query of head 5 lives in KV head 1's subspace: its energy sits in the
    # leading columns of that head's R, not of another head's
    q = workloads.query_vec(wl, 0, 5).astype(np.float64)
    e_own = np.sum((q @ workloads.rotation(wl, 1))[:8] ** 2)
    e_other = np.sum((q @ workloads.rotation(wl, 2))[:8] ** 2)
    assert e_own > 4 * e_other


def test_sweep_has_54_points_and_sample_rows():
    pts = workloads.sweep_points()
    assert len(pts) == 54
    assert all(p.k * 8 == p.S or p.k * 4 == p.S for p in pts)
    wl = workloads.get("llama2-13b")
    rows = workloads.sample_rows(wl, 16)
    assert len(rows) == 16 and rows[0] == (0, 0) and rows[-1] == (wl.B - 1, wl.H_q - 1)
    assert len(set(rows)) == 16


def test_rope_is_a_position_dependent_rotation():
    """Rotary embedding: identity at position 0, norm-preserving per column
    pair, and q(m) . k(n) depends only on m - n."""
    rng = np.random.default_rng(0)
    D = 16
    x = rng.standard_normal((5, D))
    np.testing.assert_allclose(workloads.rope(x, np.zeros(5)), x, atol=0)
    y = workloads.rope(x, np.arange(5) * 7.0)
    h = D // 2
    np.testing.assert_allclose(x[:, :h] ** 2 + x[:, h:] ** 2, y[:, :h] ** 2 + y[:, h:] ** 2,
                               rtol=1e-12)
    q, k = rng.standard_normal(D), rng.standard_normal(D)
    a = workloads.rope(q[None], [9.0])[0] @ workloads.rope(k[None], [4.0])[0]
    b = workloads.rope(q[None], [105.0])[0] @ workloads.rope(k[None], [100.0])[0]
    assert abs(a - b) < 1e-12
    # one hand value: D = 2, position 1, angle 1 rad
    np.testing.assert_allclose(workloads.rope(np.array([[1.0, 0.0]]), [1.0])[0],
                               [math.cos(1.0), math.sin(1.0)], rtol=1e-15)


def test_moved_bytes_drop_only_the_reused_key_columns():
    """With d >= D / 2 (whole 16-byte chunks) the gather skips key columns
    [0, d); otherwise a step moves the ideal bytes."""
    wl = workloads.get("llama2-13b")
    assert wl.moved_bytes() == wl.loki_bytes()  # d = 32 < D / 2
    pt = [p for p in workloads.sweep_points() if p.d == 64][0]
    assert pt.moved_bytes() == pt.loki_bytes() - 2 * pt.B * pt.H_q * pt.k * 64
    odd = pt.with_(d=68)  # 68 bf16 columns are not whole 16-byte chunks
    assert odd.moved_bytes() == odd.loki_bytes()
    f32 = pt.with_(dtype="f32", d=64)
    assert f32.moved_bytes() == f32.loki_bytes() - 4 * f32.B * f32.H_q * f32.k * 64
