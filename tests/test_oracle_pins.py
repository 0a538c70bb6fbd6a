"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign, a transposed operand, an off-by-one) fails it: hand-worked
fixtures, closed forms of the synthetic spectrum, brute force on tiny inputs,
and invariants that follow from the definitions.
"""
import itertools
import math

import numpy as np
import pytest

import oracle
import workloads
from tests import golden_io


# ---------------------------------------------------------------------------
# hand-worked fixtures
# ---------------------------------------------------------------------------

def test_worked_decode_example():
    g = golden_io.load("loki_worked_d2.txt")
    d, k = int(g["d"]), int(g["k"])
    Kt = oracle.rotate_keys(g["K"], g["P"])
    np.testing.assert_array_equal(Kt, g["expect_Kt"])
    q_rot = oracle.project_query(g["q"], g["P"])
    np.testing.assert_array_equal(q_rot, g["expect_q_rot"])
    s = oracle.lowdim_scores(q_rot, Kt, d)
    np.testing.assert_array_equal(s, g["expect_scores"])
    idx = oracle.select_topk(s, k)
    np.testing.assert_array_equal(idx, g["expect_idx"])
    out = oracle.attend(q_rot, Kt, g["V"], idx, g["scale"])
    np.testing.assert_allclose(out, g["expect_out"], rtol=0, atol=1e-12)
    out2, idx2, _, _ = oracle.loki_decode_row(g["q"], Kt, g["V"], g["P"], d, k, g["scale"])
    np.testing.assert_allclose(out2, g["expect_out"], rtol=0, atol=1e-12)
    np.testing.assert_array_equal(idx2, g["expect_idx"])
    dense = oracle.dense_decode_row(g["q"], g["K"], g["V"], g["scale"])
    np.testing.assert_allclose(dense, g["expect_dense"], rtol=1e-13, atol=0)
    pa = oracle.pca_attn_row(g["q"], Kt, g["V"], g["P"], d, g["scale"])
    np.testing.assert_allclose(pa, g["expect_pca_attn"], rtol=1e-13, atol=0)


def test_worked_pca_example():
    g = golden_io.load("pca_worked_2d.txt")
    np.testing.assert_allclose(oracle.covariance(g["X"]), g["expect_cov"], rtol=1e-13, atol=1e-13)
    P, w = oracle.calibrate_pca(g["X"])
    np.testing.assert_allclose(w, g["expect_eigvals"], rtol=1e-13)
    np.testing.assert_allclose(P, g["expect_P"], atol=1e-13)
    assert oracle.explained_variance_rank(w, 0.9) == int(g["expect_rank90"])


# ---------------------------------------------------------------------------
# calibration: closed forms and definitions
# ---------------------------------------------------------------------------

def _rand_sym_data(seed, n=300, D=12):
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((D, D))
    return rng.standard_normal((n, D)) @ A + rng.standard_normal(D) * 5.0


def test_calibrate_is_an_eigendecomposition():
    X = _rand_sym_data(1)
    C = oracle.covariance(X)
    P, w = oracle.calibrate_pca(X)
    D = C.shape[0]
    # eigen-pairs by definition: C v_c = lambda_c v_c, column by column
    np.testing.assert_allclose(C @ P, P * w[None, :], atol=1e-10 * np.abs(C).max())
    np.testing.assert_allclose(P.T @ P, np.eye(D), atol=1e-12)
    assert np.all(np.diff(w) <= 0), "eigenvalues must be descending"
    # sign rule: each column's largest-magnitude entry is positive
    piv = np.argmax(np.abs(P), axis=0)
    assert np.all(P[piv, np.arange(D)] > 0)
    # covariance is centred and divides by N - 1: compare with the definition
    # written as a double sum over pairs of samples (no mean needed):
    # C = 1/(2N(N-1)) sum_{a,b} (x_a - x_b)(x_a - x_b)^T
    n = X.shape[0]
    diff = X[:, None, :] - X[None, :, :]
    C_pairs = np.einsum("abi,abj->ij", diff, diff) / (2.0 * n * (n - 1))
    np.testing.assert_allclose(C, C_pairs, rtol=1e-10, atol=1e-10)


def test_calibrate_ignores_mean_offset():
    X = _rand_sym_data(2)
    P1, w1 = oracle.calibrate_pca(X)
    P2, w2 = oracle.calibrate_pca(X + np.linspace(-100, 100, X.shape[1])[None, :])
    np.testing.assert_allclose(w1, w2, rtol=1e-9)
    np.testing.assert_allclose(P1, P2, atol=1e-8)


def test_calibrate_recovers_generator_spectrum():
    # closed form: cov = R diag(sigma^2) R^T + noise^2 I, so the eigenvalues are
    # sigma_i^2 + noise^2 and the top eigenvectors are +-columns of R.
    wl = workloads.get("tiny")
    n = 20000
    R = workloads.rotation(wl, 0)
    X = workloads.calibration_keys(wl, 0, R, n=n)
    P, w = oracle.calibrate_pca(X)
    expect = workloads.sigma(wl) ** 2 + wl.noise_std ** 2
    top = 24
    # sampling error of a Gaussian variance estimate is lambda * sqrt(2/n)
    np.testing.assert_allclose(w[:top], expect[:top], rtol=6 * math.sqrt(2.0 / n))
    align = np.abs(np.sum(P[:, :6] * R[:, :6], axis=0))
    assert np.all(align > 0.97), align


def test_rank90_closed_form_for_tau80():
    # sigma_i^2 = rho^i with rho = exp(-2/80): the top-r share is
    # (1 - rho^r) / (1 - rho^D); the 90% rank solves rho^r <= 1 - 0.9 (1 - rho^D).
    D, tau = 128, 80.0
    rho = math.exp(-2.0 / tau)
    r_closed = math.ceil(math.log(1.0 - 0.9 * (1.0 - rho ** D)) / math.log(rho))
    assert r_closed == 80
    lam = np.exp(-2.0 * np.arange(D) / tau)
    assert oracle.explained_variance_rank(lam, 0.9) == r_closed
    # and on calibrated synthetic keys of the Llama2-13B-shaped workload
    wl = workloads.get("llama2-13b")
    _, w = oracle.calibrate_pca(workloads.calibration_keys(wl, 3))
    assert abs(oracle.explained_variance_rank(w, 0.9) - 80) <= 3


# ---------------------------------------------------------------------------
# rotation and dtype rounding
# ---------------------------------------------------------------------------

def test_rotation_is_orthogonal_change_of_basis():
    X = _rand_sym_data(3, D=16)
    P, _ = oracle.calibrate_pca(X)
    K = np.random.default_rng(4).standard_normal((50, 16))
    Kt = oracle.rotate_keys(K, P)
    np.testing.assert_allclose(Kt @ P.T, K, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(Kt, axis=1), np.linalg.norm(K, axis=1), rtol=1e-12)


def test_bf16_rounding_hand_values():
    r = oracle.round_to_dtype
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties to the even mantissa (1)
    assert r(np.array([1 + 2.0 ** -8]), "bf16")[0] == 1.0
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even)
    assert r(np.array([1 + 3 * 2.0 ** -8]), "bf16")[0] == 1 + 2.0 ** -6
    assert r(np.array([-(1 + 3 * 2.0 ** -8)]), "bf16")[0] == -(1 + 2.0 ** -6)
    # just above the midpoint rounds up
    assert r(np.array([1 + 2.0 ** -8 + 2.0 ** -30]), "bf16")[0] == 1 + 2.0 ** -7
    assert r(np.array([255.0, 257.0, 0.0]), "bf16").tolist() == [255.0, 256.0, 0.0]
    assert r(np.array([1.0 + 2.0 ** -30]), "f32")[0] == 1.0


def test_bf16_rounding_matches_generator_encoding():
    # two independent encoders (exponent/rint here, integer bit trick in the
    # generator) must agree on fp32-exact inputs, where no double rounding occurs
    x = np.random.default_rng(5).standard_normal(100000).astype(np.float32).astype(np.float64)
    a = oracle.round_to_dtype(x, "bf16")
    b = workloads.to_cache_dtype(x, "bf16").astype(np.float64)
    np.testing.assert_array_equal(a, b)


# ---------------------------------------------------------------------------
# scores, selection, attention
# ---------------------------------------------------------------------------

def test_full_dim_rotated_scores_equal_unrotated():
    wl = workloads.get("tiny")
    R = workloads.rotation(wl, 0)
    P, _ = oracle.calibrate_pca(workloads.calibration_keys(wl, 0, R))
    K = workloads.keys_block(wl, 0, 0, R).astype(np.float64)
    q = workloads.query_vec(wl, 0, 0, R).astype(np.float64)
    s = oracle.lowdim_scores(oracle.project_query(q, P), oracle.rotate_keys(K, P), wl.D)
    np.testing.assert_allclose(s, K @ q, rtol=1e-11, atol=1e-12)
    # positive scaling of q does not change the selection
    s2 = oracle.lowdim_scores(oracle.project_query(3.7 * q, P), oracle.rotate_keys(K, P), 16)
    s1 = oracle.lowdim_scores(oracle.project_query(q, P), oracle.rotate_keys(K, P), 16)
    np.testing.assert_array_equal(oracle.select_topk(s1, 40), oracle.select_topk(s2, 40))


def _brute_topk(s, k):
    """Max-sum k-subset; among equal sums the lexicographically smallest index tuple."""
    best, best_set = None, None
    for c in itertools.combinations(range(len(s)), k):
        tot = sum(s[i] for i in c)
        if best is None or tot > best:
            best, best_set = tot, c
    return np.array(best_set)


@pytest.mark.parametrize("seed", range(12))
def test_topk_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    S = int(rng.integers(1, 11))
    # integer-valued scores force ties; some rows get negatives, zeros and -0.0
    s = rng.integers(-3, 4, size=S).astype(np.float64)
    if seed % 3 == 0:
        s[s == 0] = -0.0
    for k in range(1, S + 1):
        got = oracle.select_topk(s, k)
        want = _brute_topk(s, k)
        np.testing.assert_array_equal(got, want)
        sel = np.zeros(S, bool)
        sel[got] = True
        if k < S:
            assert s[sel].min() >= s[~sel].max()


def test_topk_k1_is_argmax_and_permutation_equivariant():
    rng = np.random.default_rng(9)
    s = rng.standard_normal(200)
    assert oracle.select_topk(s, 1)[0] == int(np.argmax(s))
    perm = rng.permutation(200)
    got = oracle.select_topk(s[perm], 30)
    np.testing.assert_array_equal(np.sort(perm[got]), oracle.select_topk(s, 30))


def test_topk_nan_ranks_lowest():
    s = np.array([np.nan, -5.0, np.nan, -7.0])
    np.testing.assert_array_equal(oracle.select_topk(s, 2), [1, 3])
    np.testing.assert_array_equal(oracle.select_topk(s, 3), [0, 1, 3])


def test_attend_special_cases():
    rng = np.random.default_rng(11)
    S, D = 64, 8
    Kt = rng.standard_normal((S, D))
    V = rng.standard_normal((S, D))
    q = rng.standard_normal(D)
    # a single selected token returns its value row exactly
    j = 17
    np.testing.assert_allclose(oracle.attend(q, Kt, V, np.array([j]), 0.5), V[j], atol=1e-15)
    # q = 0 makes all scores equal: the output is the mean of the selected values
    idx = np.array([1, 5, 9, 40])
    np.testing.assert_allclose(oracle.attend(np.zeros(D), Kt, V, idx, 1.0), V[idx].mean(0), atol=1e-14)
    # order of the selected set does not matter
    np.testing.assert_allclose(oracle.attend(q, Kt, V, idx[::-1], 0.3),
                               oracle.attend(q, Kt, V, idx, 0.3), atol=1e-14)
    # huge scores do not overflow (max-subtraction)
    out = oracle.attend(1e4 * q, Kt, V, idx, 1.0)
    assert np.all(np.isfinite(out))


def test_loki_with_all_dims_and_all_tokens_is_dense():
    wl = workloads.get("tiny")
    R = workloads.rotation(wl, 0)
    P, _ = oracle.calibrate_pca(workloads.calibration_keys(wl, 0, R))
    K = workloads.keys_block(wl, 0, 0, R).astype(np.float64)
    V = workloads.values_block(wl, 0, 0).astype(np.float64)
    q = workloads.query_vec(wl, 0, 0, R).astype(np.float64)
    Kt = oracle.rotate_keys(K, P)
    out, idx, _, _ = oracle.loki_decode_row(q, Kt, V, P, wl.D, wl.S, wl.scale)
    np.testing.assert_array_equal(idx, np.arange(wl.S))
    np.testing.assert_allclose(out, oracle.dense_decode_row(q, K, V, wl.scale), atol=1e-12)


def test_gqa_head_mapping():
    # query heads 0,1 read KV head 0 and heads 2,3 read KV head 1 (consecutive
    # query heads share a KV head): make each KV head's values constant
    B, H_q, H_kv, S, D = 1, 4, 2, 32, 8
    rng = np.random.default_rng(12)
    q = rng.standard_normal((B, H_q, D))
    Kt = rng.standard_normal((B, H_kv, S, D))
    V = np.zeros((B, H_kv, S, D))
    V[0, 0] = 1.0
    V[0, 1] = -2.0
    P = np.stack([np.eye(D)] * H_kv)
    out, _, _ = oracle.loki_decode(q, Kt, V, P, S, 4, 8)
    np.testing.assert_allclose(out[0, :2], 1.0, atol=1e-14)
    np.testing.assert_allclose(out[0, 2:], -2.0, atol=1e-14)
    dense = oracle.dense_decode(q, Kt, V, S)
    np.testing.assert_allclose(dense[0, :2], 1.0, atol=1e-14)
    np.testing.assert_allclose(dense[0, 2:], -2.0, atol=1e-14)


def test_selection_prefers_high_lowdim_score_tokens_on_lowrank_keys():
    # quality sanity, not parity: with d = 32 of a tau = 16 spectrum nearly all
    # of the key energy is kept, so Loki's set overlaps the exact top-k heavily
    wl = workloads.get("tiny")
    R = workloads.rotation(wl, 0)
    P, _ = oracle.calibrate_pca(workloads.calibration_keys(wl, 0, R))
    K = workloads.keys_block(wl, 0, 0, R).astype(np.float64)
    q = workloads.query_vec(wl, 0, 0, R).astype(np.float64)
    Kt = oracle.rotate_keys(K, P)
    idx = oracle.select_topk(oracle.lowdim_scores(oracle.project_query(q, P), Kt, wl.d), wl.k)
    exact = oracle.select_topk(K @ q, wl.k)
    assert len(np.intersect1d(idx, exact)) >= 0.9 * wl.k


def test_calibrate_heads_closed_form_per_head():
    # Each head gets 8 keys +-a_i e_i, so its centred covariance is exactly
    # diag(2 a_i^2) / (N - 1): the eigenvalues are known in closed form and
    # the principal components are the axes sorted by variance. Head 2 is
    # head 0 turned by 30 degrees in the (0, 1) plane, so its components are
    # the turned axes. The per-head orders are 3-cycles, so a transposed basis
    # or a head mix-up gives a different P.
    a = {0: [1.0, 3.0, 2.0, 0.5], 1: [2.0, 0.5, 1.0, 3.0]}
    D, N = 4, 8
    th = math.radians(30.0)
    R = np.eye(D)
    R[0, 0], R[0, 1], R[1, 0], R[1, 1] = math.cos(th), -math.sin(th), math.sin(th), math.cos(th)
    keys = np.zeros((N, 3, D))
    for h in (0, 1):
        for i in range(D):
            keys[2 * i, h, i] = a[h][i]
            keys[2 * i + 1, h, i] = -a[h][i]
    keys[:, 2, :] = keys[:, 0, :] @ R.T
    P, w = oracle.calibrate_pca_heads(keys)
    assert P.shape == (3, D, D) and w.shape == (3, D)
    var = {h: 2.0 * np.square(a[h]) / (N - 1) for h in (0, 1)}
    E = np.eye(D)
    expect_P = {
        0: E[:, [1, 2, 0, 3]],
        1: E[:, [3, 0, 2, 1]],
        2: np.stack([R @ E[:, 1], E[:, 2], R @ E[:, 0], E[:, 3]], axis=1),
    }
    expect_w = {0: np.sort(var[0])[::-1], 1: np.sort(var[1])[::-1], 2: np.sort(var[0])[::-1]}
    for h in range(3):
        np.testing.assert_allclose(w[h], expect_w[h], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(P[h], expect_P[h], atol=1e-12)


# ---------------------------------------------------------------------------
# the pre-rotary variant
# ---------------------------------------------------------------------------

def test_prerotary_hand_worked():
    """Selection on the rotated pre-rotary keys (first d columns), attention
    with the post-rotary query and keys. Worked by hand: P swaps the two
    axes, so q~ = (2, 1) and K~pre = [[1, 0], [0.5, 0], [0, 3]]; on d = 1 the
    scores are (2, 1, 0). Selecting on d = 2 (scores (2, 1, 3)), on the
    unrotated keys ((0, 0, 3)) or on the post-rotary ones ((0, 2, 10)) would
    pick token 2 instead of token 0."""
    P = np.array([[0.0, 1.0], [1.0, 0.0]])
    q_pre, q_post = np.array([1.0, 2.0]), np.array([1.0, 0.0])
    K_pre = np.array([[0.0, 1.0], [0.0, 0.5], [3.0, 0.0]])
    K_post = np.array([[0.0, 1.0], [2.0, 0.0], [5.0, 5.0]])
    V = np.array([[10.0, 0.0], [0.0, 20.0], [7.0, 7.0]])
    Kt_pre = oracle.rotate_keys(K_pre, P)
    out, idx = oracle.prerotary_decode_row(q_pre, q_post, Kt_pre, K_post, V, P, 1, 1, 1.0)
    np.testing.assert_array_equal(idx, [0])
    np.testing.assert_array_equal(out, [10.0, 0.0])
    # k = 2: tokens {0, 1}; post-rotary logits (0, 2)
    out, idx = oracle.prerotary_decode_row(q_pre, q_post, Kt_pre, K_post, V, P, 1, 2, 1.0)
    np.testing.assert_array_equal(idx, [0, 1])
    e2 = math.exp(2.0)
    np.testing.assert_allclose(out, [10.0 / (1 + e2), 20.0 * e2 / (1 + e2)], rtol=1e-14)


def test_prerotary_without_rotary_is_loki():
    """With no rotary embedding (post = pre) the variant is Loki itself: the
    exact scores q . K_j equal q~ . K~_j because P is orthonormal."""
    rng = np.random.default_rng(3)
    S, D, d, k = 40, 8, 3, 7
    K = rng.standard_normal((S, D))
    V = rng.standard_normal((S, D))
    q = rng.standard_normal(D)
    P, _ = oracle.calibrate_pca(rng.standard_normal((200, D)) * np.linspace(3, 0.1, D))
    Kt = oracle.rotate_keys(K, P)
    out, idx = oracle.prerotary_decode_row(q, q, Kt, K, V, P, d, k, 0.4)
    want, widx, _, _ = oracle.loki_decode_row(q, Kt, V, P, d, k, 0.4)
    np.testing.assert_array_equal(idx, widx)
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)
