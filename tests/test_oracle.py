"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these compares the oracle with itself: each check uses a value printed
on the pages (tests/golden/, each file names its source), a textbook routine
(numpy.linalg.norm), a closed form that holds for a special input, or finite
differences of the plain ``DoRALinear`` forward.  Each is chosen so that a
plausible slip (a dropped term, a wrong sign or factor, a transposed operand,
a norm over the wrong axis) fails at least one of them.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _rand_module(rng, d_out, d_in, r, scale_b=0.3):
    W0 = rng.standard_normal((d_out, d_in))
    A = rng.standard_normal((r, d_in)) / np.sqrt(d_in)
    B = scale_b * rng.standard_normal((d_out, r))
    return W0, A, B


# ---------------------------------------------------------------- counts

def test_param_counts_match_printed_values():
    g = _gold("param_counts.json")
    for c in g["cases"]:
        assert c["d"] * c["k"] == c["n_full"]
        assert oracle.lora_param_count(c["d"], c["k"], c["r"]) == c["n_lora"]
        if "n_dora" in c:
            assert oracle.dora_param_count(c["d"], c["k"], c["r"]) == c["n_dora"]
        if "ratio_full_over_lora" in c:
            assert c["n_full"] // c["n_lora"] == c["ratio_full_over_lora"]


def test_lora_scale_is_alpha_over_r():
    # s = alpha / r; the workloads use alpha = 2r throughout, so s = 2.
    assert oracle.lora_scale(16, 8) == 2.0
    assert oracle.lora_scale(768, 384) == 2.0
    assert oracle.lora_scale(32, 8) == 4.0


def test_factored_memory_reduction_15x():
    g = _gold("factored_memory.json")
    ratio = g["d_out"] * g["d_in"] / oracle.factored_intermediate_elems(g["d_out"], g["r"])
    assert round(ratio) == g["reduction_x"]


# ---------------------------------------------------------------- worked examples

def test_arrow_and_rotation_examples():
    g = _gold("arrow_example.json")
    for c in g["cases"]:
        W0 = np.array([c["w0"]])
        # rank-1 update s*B*A equal to the printed update vector: A = update, B = 1, s = 1
        A = np.array([c["update"]])
        B = np.array([[1.0]])
        n = oracle.dense_row_norm(W0, A, B, 1.0)
        assert n[0] == pytest.approx(c["norm"], rel=1e-15)
        nf = oracle.factored_row_norm(W0, A, B, 1.0)
        assert nf[0] == pytest.approx(c["norm"], rel=1e-15)
        Wm = oracle.merged_weight(W0, A, B, np.array([c["m"]]), 1.0)
        np.testing.assert_allclose(Wm[0], c["merged_row"], rtol=0, atol=1e-15)
        # the merged row has length m and points along w0 + update
        assert np.linalg.norm(Wm[0]) == pytest.approx(c["m"], rel=1e-15)


def test_arrow_example_through_compose():
    # y = W' x for the arrow layer, once through the merged weight and once
    # through the composition contract with base = W0 x, lora = (x A^T) B^T.
    g = _gold("arrow_example.json")["cases"][0]
    W0 = np.array([g["w0"]])
    A = np.array([g["update"]])
    B = np.array([[1.0]])
    m = np.array([g["m"]])
    x = np.eye(2)
    base = x @ W0.T
    lora = (x @ A.T) @ B.T
    n = np.array([g["norm"]])
    y = oracle.compose_fwd(base, lora, m, n, 1.0, 1e-12)
    np.testing.assert_allclose(y[:, 0], g["merged_row"], rtol=1e-15, atol=1e-15)


# ---------------------------------------------------------------- norm identities

@pytest.mark.parametrize("shape", [(7, 5, 3), (16, 12, 4), (33, 17, 20), (1, 9, 1), (5, 3, 8)])
@pytest.mark.parametrize("s", [0.5, 2.0, -1.5])
def test_factored_equals_dense_norm(shape, s):
    rng = np.random.default_rng(hash((shape, s)) % 2**32)
    W0, A, B = _rand_module(rng, *shape)
    nd = oracle.dense_row_norm(W0, A, B, s)
    nf = oracle.factored_row_norm(W0, A, B, s)
    np.testing.assert_allclose(nf, nd, rtol=1e-12)


def test_dense_norm_identity_A_is_textbook_rownorm():
    # r = d_in and A = I: W0 + sBA = W0 + sB, whose row norms numpy computes.
    rng = np.random.default_rng(1)
    d_out, d = 11, 6
    W0 = rng.standard_normal((d_out, d))
    B = rng.standard_normal((d_out, d))
    s = 1.75
    want = np.linalg.norm(W0 + s * B, axis=1)
    np.testing.assert_allclose(oracle.dense_row_norm(W0, np.eye(d), B, s), want, rtol=1e-14)
    np.testing.assert_allclose(oracle.factored_row_norm(W0, np.eye(d), B, s), want, rtol=1e-13)


def test_norm_orthonormal_A_and_orthogonal_base():
    # A with orthonormal rows: ||B_i A|| = ||B_i||.  With W0 orthogonal to A's
    # row space the cross term vanishes: n^2 = ||W0_i||^2 + s^2 ||B_i||^2
    # (Pythagoras).  With W0 inside A's row space, W0_i = w_i A and
    # n = ||w_i + s B_i||.  A slip in the cross term's factor 2s, or in the
    # Gram term's s^2, fails one of the two.
    rng = np.random.default_rng(2)
    d_out, d_in, r = 9, 10, 4
    Q, _ = np.linalg.qr(rng.standard_normal((d_in, d_in)))
    A = Q[:, :r].T                      # orthonormal rows
    perp = Q[:, r:].T                   # basis of the orthogonal complement
    B = rng.standard_normal((d_out, r))
    s = 1.3
    W0_perp = rng.standard_normal((d_out, d_in - r)) @ perp
    want = np.sqrt(np.linalg.norm(W0_perp, axis=1) ** 2 + s * s * np.linalg.norm(B, axis=1) ** 2)
    for fn in (oracle.dense_row_norm, oracle.factored_row_norm):
        np.testing.assert_allclose(fn(W0_perp, A, B, s), want, rtol=1e-12)
    w = rng.standard_normal((d_out, r))
    W0_in = w @ A
    want_in = np.linalg.norm(w + s * B, axis=1)
    for fn in (oracle.dense_row_norm, oracle.factored_row_norm):
        np.testing.assert_allclose(fn(W0_in, A, B, s), want_in, rtol=1e-12)


def test_norm_is_per_output_row():
    # Permuting output rows (rows of W0 and B together) permutes n; permuting
    # input columns (columns of W0 and A together) leaves n unchanged.
    rng = np.random.default_rng(3)
    W0, A, B = _rand_module(rng, 13, 8, 3)
    s = 2.0
    n = oracle.dense_row_norm(W0, A, B, s)
    p = rng.permutation(13)
    np.testing.assert_allclose(oracle.dense_row_norm(W0[p], A, B[p], s), n[p], rtol=1e-14)
    np.testing.assert_allclose(oracle.factored_row_norm(W0[p], A, B[p], s), n[p], rtol=1e-12)
    q = rng.permutation(8)
    np.testing.assert_allclose(oracle.dense_row_norm(W0[:, q], A[:, q], B, s), n, rtol=1e-14)
    np.testing.assert_allclose(oracle.factored_row_norm(W0[:, q], A[:, q], B, s), n, rtol=1e-12)


def test_norm_homogeneity_and_scale_invariance():
    rng = np.random.default_rng(4)
    W0, A, B = _rand_module(rng, 10, 7, 3)
    s, c = 2.0, -3.0
    m = rng.uniform(0.5, 2.0, 10)
    n = oracle.factored_row_norm(W0, A, B, s)
    n_c = oracle.factored_row_norm(c * W0, A, c * B, s)
    np.testing.assert_allclose(n_c, abs(c) * n, rtol=1e-13)
    g, _, _ = oracle.magnitude_scale(m, n, 1e-12)
    g_c, _, _ = oracle.magnitude_scale(abs(c) * m, n_c, 1e-12)
    np.testing.assert_allclose(g_c, g, rtol=1e-13)


def test_zero_row_clamps_to_eps():
    W0 = np.zeros((3, 4)); W0[1] = [3.0, 4.0, 0.0, 0.0]
    A = np.ones((2, 4)); B = np.zeros((3, 2))
    n = oracle.factored_row_norm(W0, A, B, 2.0)
    np.testing.assert_array_equal(n, [0.0, 5.0, 0.0])
    m = np.array([1.0, 5.0, 2.0])
    eps = 2.0 ** -7
    g, gm1, nc = oracle.magnitude_scale(m, n, eps)
    np.testing.assert_array_equal(nc, [eps, 5.0, eps])
    np.testing.assert_array_equal(g, [1.0 / eps, 1.0, 2.0 / eps])
    np.testing.assert_allclose(gm1, g - 1.0, rtol=1e-15)


# ---------------------------------------------------------------- compose

def test_init_invariant_output_equals_base_exactly():
    # m0 = ||W0_i|| and B0 = 0 give W' = W0, so y = base bit for bit.
    rng = np.random.default_rng(5)
    W0, A, _ = _rand_module(rng, 6, 5, 2)
    B = np.zeros((6, 2))
    n = oracle.dense_row_norm(W0, A, B, 2.0)
    m = n.copy()
    x = rng.standard_normal((4, 5))
    base = x @ W0.T
    lora = (x @ A.T) @ B.T
    y = oracle.compose_fwd(base, lora, m, n, 2.0, 1e-12)
    np.testing.assert_array_equal(y, base)


def test_compose_equals_dora_linear_forward():
    # The composition contract (base + (g-1) base + g s lora) reproduces the
    # plain DoRALinear forward x W'^T with the merged weight.
    rng = np.random.default_rng(6)
    d_out, d_in, r, T = 12, 9, 4, 7
    W0, A, B = _rand_module(rng, d_out, d_in, r)
    m = rng.uniform(0.5, 2.0, d_out)
    s = 2.0
    x = rng.standard_normal((T, d_in))
    n = oracle.dense_row_norm(W0, A, B, s)
    y = oracle.compose_fwd(x @ W0.T, (x @ A.T) @ B.T, m, n, s, 1e-12)
    np.testing.assert_allclose(y, oracle.dora_linear_forward(x, W0, A, B, m, s), rtol=1e-12, atol=1e-13)


def test_compose_delta_completes_the_dense_dora_forward():
    # Y_base + dY must be the plain DoRALinear forward with the merged weight
    # (the caller's side of the composition contract).
    rng = np.random.default_rng(61)
    d_out, d_in, r, T = 10, 7, 3, 6
    W0, A, B = _rand_module(rng, d_out, d_in, r)
    m = rng.uniform(0.5, 2.0, d_out)
    s = 1.5
    x = rng.standard_normal((T, d_in))
    n = oracle.dense_row_norm(W0, A, B, s)
    d = oracle.compose_delta(x @ W0.T, (x @ A.T) @ B.T, m, n, s, 1e-12)
    np.testing.assert_allclose(x @ W0.T + d, oracle.dora_linear_forward(x, W0, A, B, m, s),
                               rtol=1e-12, atol=1e-13)


def test_compose_delta_special_cases():
    rng = np.random.default_rng(62)
    base = rng.standard_normal((4, 5)); lora = rng.standard_normal((4, 5))
    n = rng.uniform(0.5, 2.0, 5)
    # g = 1: the delta is the LoRA branch alone
    np.testing.assert_allclose(oracle.compose_delta(base, lora, n, n, 2.0, 1e-12), 2.0 * lora,
                               rtol=1e-15, atol=0)
    # m = 2 n, lora = 0: the delta is base itself (g - 1 = 1)
    np.testing.assert_allclose(oracle.compose_delta(base, np.zeros_like(lora), 2 * n, n, 2.0, 1e-12),
                               base, rtol=1e-15, atol=0)


def test_compose_g_equal_one_is_lora_forward():
    rng = np.random.default_rng(7)
    base = rng.standard_normal((5, 6)); lora = rng.standard_normal((5, 6))
    n = rng.uniform(0.5, 2.0, 6)
    y = oracle.compose_fwd(base, lora, n, n, 1.5, 1e-12)
    np.testing.assert_allclose(y, base + 1.5 * lora, rtol=1e-15, atol=0)


# ---------------------------------------------------------------- backward

def _fd(f, x, h=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        xp = x.copy(); xp[i] += h
        xm = x.copy(); xm[i] -= h
        g[i] = (f(xp) - f(xm)) / (2 * h)
    return g


def test_backward_matches_finite_differences_of_compose():
    rng = np.random.default_rng(8)
    T, d_out, s, eps = 4, 5, 2.0, 1e-12
    base = rng.standard_normal((T, d_out)); lora = rng.standard_normal((T, d_out))
    dy = rng.standard_normal((T, d_out))
    n = rng.uniform(0.5, 2.0, d_out); m = n * rng.uniform(0.9, 1.1, d_out)
    d_base, d_lora, dm = oracle.compose_bwd(dy, base, lora, m, n, s, eps)
    L = lambda b, l, mm: float(np.sum(dy * oracle.compose_fwd(b, l, mm, n, s, eps)))
    np.testing.assert_allclose(d_base, _fd(lambda b: L(b, lora, m), base), rtol=1e-7, atol=1e-9)
    np.testing.assert_allclose(d_lora, _fd(lambda l: L(base, l, m), lora), rtol=1e-7, atol=1e-9)
    np.testing.assert_allclose(dm, _fd(lambda mm: L(base, lora, mm), m), rtol=1e-7, atol=1e-9)


def test_backward_matches_dora_linear_with_detached_norm():
    # dm: the norm does not depend on m, so the gradient of the plain module
    # forward with respect to m is the compose's dm.  dB: with the norm held
    # fixed (detached), the chain rule through lora = (x A^T) B^T gives
    # dL/dB = d_lora^T (x A^T).
    rng = np.random.default_rng(9)
    d_out, d_in, r, T, s = 6, 5, 3, 4, 2.0
    W0, A, B = _rand_module(rng, d_out, d_in, r)
    m = rng.uniform(0.5, 2.0, d_out)
    x = rng.standard_normal((T, d_in))
    dy = rng.standard_normal((T, d_out))
    n = oracle.dense_row_norm(W0, A, B, s)
    base, xa = x @ W0.T, x @ A.T
    lora = xa @ B.T
    _, d_lora, dm = oracle.compose_bwd(dy, base, lora, m, n, s, 1e-12)
    f_m = lambda mm: float(np.sum(dy * oracle.dora_linear_forward(x, W0, A, B, mm, s)))
    np.testing.assert_allclose(dm, _fd(f_m, m), rtol=1e-7, atol=1e-9)

    def f_B_detached(Bv):
        V = W0 + s * (Bv @ A)
        W = (m / n)[:, None] * V          # n frozen
        return float(np.sum(dy * (x @ W.T)))
    np.testing.assert_allclose(d_lora.T @ xa, _fd(f_B_detached, B), rtol=1e-7, atol=1e-9)


def test_dm_is_linear_in_dy():
    rng = np.random.default_rng(10)
    T, d_out = 6, 4
    base = rng.standard_normal((T, d_out)); lora = rng.standard_normal((T, d_out))
    n = rng.uniform(0.5, 2, d_out); m = rng.uniform(0.5, 2, d_out)
    dy1 = rng.standard_normal((T, d_out)); dy2 = rng.standard_normal((T, d_out))
    _, _, a = oracle.compose_bwd(dy1, base, lora, m, n, 2.0, 1e-12)
    _, _, b = oracle.compose_bwd(dy2, base, lora, m, n, 2.0, 1e-12)
    _, _, c = oracle.compose_bwd(2 * dy1 - 3 * dy2, base, lora, m, n, 2.0, 1e-12)
    np.testing.assert_allclose(c, 2 * a - 3 * b, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- training variants

def test_inner_worked_example_and_forward_relation():
    # inner = base + s lora by hand; and y = g * inner (the forward is the
    # magnitude scale applied to inner, whatever the split of y into base and
    # correction).
    inner = oracle.compose_inner(np.array([[1.0, 2.0]]), np.array([[3.0, 4.0]]), 0.5)
    np.testing.assert_array_equal(inner, [[2.5, 4.0]])
    rng = np.random.default_rng(12)
    T, d_out, s, eps = 5, 4, 1.5, 1e-12
    base = rng.standard_normal((T, d_out)); lora = rng.standard_normal((T, d_out))
    n = rng.uniform(0.5, 2.0, d_out); m = rng.uniform(0.5, 2.0, d_out)
    y = oracle.compose_fwd(base, lora, m, n, s, eps)
    np.testing.assert_allclose(y, (m / n) * oracle.compose_inner(base, lora, s), rtol=1e-14)


def test_backward_from_inner_matches_finite_differences():
    # L(inner, m) = sum dy * g(m) * inner; dm by finite differences in m, and
    # d_base / d_lora by finite differences of the full forward in base / lora.
    rng = np.random.default_rng(13)
    T, d_out, s, eps = 4, 5, 2.0, 1e-12
    base = rng.standard_normal((T, d_out)); lora = rng.standard_normal((T, d_out))
    dy = rng.standard_normal((T, d_out))
    n = rng.uniform(0.5, 2.0, d_out); m = n * rng.uniform(0.9, 1.1, d_out)
    inner = base + s * lora
    d_base, d_lora, dm = oracle.compose_bwd_from_inner(dy, inner, m, n, s, eps)
    L = lambda b, l, mm: float(np.sum(dy * oracle.compose_fwd(b, l, mm, n, s, eps)))
    np.testing.assert_allclose(d_base, _fd(lambda b: L(b, lora, m), base), rtol=1e-7, atol=1e-9)
    np.testing.assert_allclose(d_lora, _fd(lambda l: L(base, l, m), lora), rtol=1e-7, atol=1e-9)
    np.testing.assert_allclose(dm, _fd(lambda mm: L(base, lora, mm), m), rtol=1e-7, atol=1e-9)


def test_frozen_backward_matches_finite_differences():
    rng = np.random.default_rng(14)
    T, d_out, s, eps = 3, 4, 0.75, 1e-12
    base = rng.standard_normal((T, d_out)); lora = rng.standard_normal((T, d_out))
    dy = rng.standard_normal((T, d_out))
    n = rng.uniform(0.5, 2.0, d_out); m = rng.uniform(0.5, 2.0, d_out)
    d_base, d_lora = oracle.compose_bwd_frozen(dy, m, n, s, eps)
    L = lambda b, l: float(np.sum(dy * oracle.compose_fwd(b, l, m, n, s, eps)))
    np.testing.assert_allclose(d_base, _fd(lambda b: L(b, lora), base), rtol=1e-7, atol=1e-9)
    np.testing.assert_allclose(d_lora, _fd(lambda l: L(base, l), lora), rtol=1e-7, atol=1e-9)


# ---------------------------------------------------------------- merged weight

def test_merged_rows_have_the_magnitude_as_norm():
    # With n the true row norm of W0 + sBA, every row of W' has norm m
    # (numpy.linalg.norm), whatever the direction.
    rng = np.random.default_rng(15)
    W0, A, B = _rand_module(rng, 9, 7, 3)
    m = rng.uniform(0.5, 2.0, 9)
    n = np.linalg.norm(W0 + 2.0 * (B @ A), axis=1)
    Wm = oracle.merge_weight_given_norm(W0, A, B, m, n, 2.0, 1e-12)
    np.testing.assert_allclose(np.linalg.norm(Wm, axis=1), m, rtol=1e-13)
    # ... and points along W0 + sBA (cosine 1 per row)
    V = W0 + 2.0 * (B @ A)
    cos = np.sum(Wm * V, axis=1) / (np.linalg.norm(Wm, axis=1) * np.linalg.norm(V, axis=1))
    np.testing.assert_allclose(cos, 1.0, rtol=1e-13)


def test_merged_init_is_w0_exactly():
    # B = 0 and m = ||W0_i||: the merged weight is W0 (DoRA's initial weight).
    rng = np.random.default_rng(16)
    W0 = rng.standard_normal((6, 5)); A = rng.standard_normal((2, 5)); B = np.zeros((6, 2))
    m = np.linalg.norm(W0, axis=1)
    np.testing.assert_allclose(oracle.merge_weight_given_norm(W0, A, B, m, m, 3.0, 1e-12), W0,
                               rtol=1e-15, atol=0)


def test_merged_forward_equals_compose():
    # x W'^T = compose(base = x W0^T, lora = x A^T B^T): merging is exact.
    rng = np.random.default_rng(17)
    d_out, d_in, r, T, s, eps = 7, 6, 3, 5, 1.5, 1e-12
    W0, A, B = _rand_module(rng, d_out, d_in, r)
    n = rng.uniform(0.5, 2.0, d_out); m = rng.uniform(0.5, 2.0, d_out)
    x = rng.standard_normal((T, d_in))
    y = x @ oracle.merge_weight_given_norm(W0, A, B, m, n, s, eps).T
    ref = oracle.compose_fwd(x @ W0.T, (x @ A.T) @ B.T, m, n, s, eps)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- d_in shards

def test_shard_partials_add_up_to_the_dense_squared_norm():
    # Any column split: the shards' squared partials sum to ||(W0 + sBA)_i||^2
    # computed densely (brute force on the materialised V).
    rng = np.random.default_rng(18)
    W0, A, B = _rand_module(rng, 7, 13, 4)
    s = 1.7
    V = W0 + s * (B @ A)
    dense_sq = np.sum(V * V, axis=1)
    for cuts in ([0, 13], [0, 5, 13], [0, 1, 2, 9, 13], [0, 0, 13]):
        total = sum(oracle.factored_row_norm_sq(W0[:, a:b], A[:, a:b], B, s)
                    for a, b in zip(cuts[:-1], cuts[1:]))
        np.testing.assert_allclose(total, dense_sq, rtol=1e-12)
    # one shard's partial is not the whole (the split matters)
    part = oracle.factored_row_norm_sq(W0[:, :5], A[:, :5], B, s)
    assert not np.allclose(part, dense_sq, rtol=1e-3)


# ---------------------------------------------------------------- planted mistakes

def test_pins_catch_planted_mistakes():
    """Each planted slip in the factored norm breaks the factored == dense pin."""
    rng = np.random.default_rng(11)
    W0, A, B = _rand_module(rng, 8, 6, 3)
    s = 2.0
    nd = oracle.dense_row_norm(W0, A, B, s)

    def slip(kind):
        G = A @ A.T
        U = W0 @ A.T
        base = np.sum(W0 * W0, axis=1)
        cross = np.sum(B * U, axis=1)
        gram = np.sum((B @ G) * B, axis=1)
        if kind == "no_cross":
            cross = 0 * cross
        if kind == "cross_factor_s":
            return np.sqrt(base + s * cross + s * s * gram)
        if kind == "gram_factor_s":
            return np.sqrt(base + 2 * s * cross + s * gram)
        if kind == "sign":
            return np.sqrt(np.maximum(base - 2 * s * cross + s * s * gram, 0))
        if kind == "transposed_gram":
            gram = np.sum((B @ (A.T @ A)[:3, :3]) * B, axis=1)
        return np.sqrt(base + 2 * s * cross + s * s * gram)

    for kind in ("no_cross", "cross_factor_s", "gram_factor_s", "sign", "transposed_gram"):
        assert not np.allclose(slip(kind), nd, rtol=1e-6), kind
