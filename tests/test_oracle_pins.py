"""Pins of the float64 oracle against what the pages and the mathematics fix.

None of these retype the oracle's own formula: each compares it with a worked
example the pages print, a closed form, an invariant, a library routine that
computes the same thing another way, or brute force on tiny inputs.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as O
from matrix_roots_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _spd(rng, n, cond=100.0):
    q = W.haar_orthogonal(rng, n)[0]
    lam = np.geomspace(1.0 / cond, 1.0, n)
    return (q * lam) @ q.T, q, lam


# ---------------------------------------------------------------- O1 ----------

def test_partition_worked_example_dash_section4():
    g = json.load(open(os.path.join(GOLDEN, "dash_stacking_example.json")))
    plan = O.plan_blocks([tuple(g["layer_shape"])], g["block_size"])
    gb = {(int(r), int(c)): int(n) for r, c, n in plan["g_buckets"]}
    fb = {int(n): int(c) for n, c in plan["f_buckets"]}
    full, rest = g["gradient_stacks"]["G_full"], g["gradient_stacks"]["G_rest"]
    assert gb == {(full[1], full[2]): full[0], (rest[1], rest[2]): rest[0]}
    sf, sr = g["factor_stacks"]["S_full"], g["factor_stacks"]["S_rest"]
    assert fb == {sf[1]: sf[0], sr[1]: sr[0]}
    # S_full holds L_full, R_full and R_rest; S_rest holds only L_rest
    B = plan["blocks"]
    rest_rows = B[:, 5] == 256
    assert np.all(B[rest_rows, 9] == 1) and np.all(B[~rest_rows, 9] == 0)
    assert np.all(B[:, 11] == 0)


def test_partition_tiles_every_layer_once():
    rng = np.random.default_rng(3)
    shapes = [(int(rng.integers(1, 300)), int(rng.integers(1, 300))) for _ in range(12)]
    for bs in (0, 7, 64, 128, 1000):
        plan = O.plan_blocks(shapes, bs)
        cover = [np.zeros(s, dtype=np.int64) for s in shapes]
        for b in plan["blocks"]:
            li, br, bc, r0, c0, r, c = (int(x) for x in b[:7])
            cover[li][r0:r0 + r, c0:c0 + c] += 1
            if bs > 0:
                assert r <= bs and c <= bs
        assert all(np.all(cv == 1) for cv in cover)
        # bucket indices are dense 0..count-1 in every bucket
        B = plan["blocks"]
        for k, row in enumerate(plan["g_buckets"]):
            idx = sorted(int(i) for i in B[B[:, 7] == k, 8])
            assert idx == list(range(int(row[-1])))
        for k, row in enumerate(plan["f_buckets"]):
            idx = sorted([int(i) for i in B[B[:, 9] == k, 10]] + [int(i) for i in B[B[:, 11] == k, 12]])
            assert idx == list(range(int(row[-1])))


def test_partition_right_factors_dense_and_ordered():
    plan = O.plan_blocks([(256, 256)], 64)
    B = plan["blocks"]
    assert B.shape[0] == 16
    assert list(B[:, 10]) == list(range(16))          # all L first ...
    assert list(B[:, 12]) == list(range(16, 32))      # ... then all R, row-major


def test_partition_transformer_counts():
    plan = O.plan_blocks(W.transformer_shapes(), 1024)
    assert plan["g_buckets"].tolist() == [[1024, 1024, 96]]
    assert plan["f_buckets"].tolist() == [[1024, 192]]


@pytest.mark.parametrize("d,B,expect", [(5, 0, [5]), (5, 5, [5]), (5, 6, [5]), (10, 5, [5, 5]),
                                        (11, 5, [5, 5, 1]), (32000, 1024, [1024] * 31 + [256])])
def test_split_dim(d, B, expect):
    assert O.split_dim(d, B) == expect


def test_stack_unstack_roundtrip():
    shapes = [(70, 33), (5, 200)]
    rng = np.random.default_rng(0)
    grads = [rng.standard_normal(s) for s in shapes]
    plan = O.plan_blocks(shapes, 32)
    st = O.stack_gradients(plan, grads)
    back = O.unstack_directions(plan, st, shapes)
    for a, b in zip(grads, back):
        assert np.array_equal(a, b)


# ---------------------------------------------------------------- O2 ----------

def test_stats_brute_force_loops():
    rng = np.random.default_rng(1)
    G = rng.standard_normal((3, 5))
    L0 = rng.standard_normal((3, 3))
    R0 = rng.standard_normal((5, 5))
    L, R = O.update_stats(G, L0, R0, beta2=0.7, alpha=0.3)
    for i in range(3):
        for j in range(3):
            acc = sum(G[i, k] * G[j, k] for k in range(5))
            assert math.isclose(L[i, j], 0.7 * L0[i, j] + 0.3 * acc, rel_tol=1e-13, abs_tol=1e-13)
    for i in range(5):
        for j in range(5):
            acc = sum(G[k, i] * G[k, j] for k in range(3))
            assert math.isclose(R[i, j], 0.7 * R0[i, j] + 0.3 * acc, rel_tol=1e-13, abs_tol=1e-13)


def test_stats_repeated_gradient_closed_form():
    rng = np.random.default_rng(2)
    G = rng.standard_normal((6, 4))
    U, sig, Vt = np.linalg.svd(G, full_matrices=False)
    beta2, k = 0.9, 7
    L, R = np.zeros((6, 6)), np.zeros((4, 4))
    for _ in range(k):
        L, R = O.update_stats(G, L, R, beta2)
    c = sum(beta2 ** j for j in range(k))
    assert np.allclose(L, c * (U * sig ** 2) @ U.T, atol=1e-12)
    assert np.allclose(R, c * (Vt.T * sig ** 2) @ Vt, atol=1e-12)
    assert math.isclose(np.trace(L), np.trace(R), rel_tol=1e-13)


# ---------------------------------------------------------------- O3 ----------

def test_exact_root_fourth_power_identity():
    rng = np.random.default_rng(4)
    A, _, _ = _spd(rng, 12, cond=1e4)
    eps = 1e-6
    X = O.inv_root_exact(A, eps)
    X4 = np.linalg.matrix_power(X, 4)
    res = np.linalg.norm(X4 @ (A + eps * np.eye(12)) - np.eye(12)) / math.sqrt(12)
    assert res < 1e-10


def test_exact_root_diagonal_closed_form():
    d = np.array([1e-4, 0.5, 3.0, 17.0])
    X = O.inv_root_exact(np.diag(d), 1e-3)
    assert np.allclose(X, np.diag((d + 1e-3) ** -0.25), rtol=1e-14, atol=0)


def test_exact_root_commuting_pairs():
    rng = np.random.default_rng(5)
    q = W.haar_orthogonal(rng, 9)[0]
    l1, l2 = rng.uniform(0.1, 2, 9), rng.uniform(0.1, 2, 9)
    A, B = (q * l1) @ q.T, (q * l2) @ q.T
    lhs = O.inv_root_exact(A @ B, 0.0)
    rhs = O.inv_root_exact(A, 0.0) @ O.inv_root_exact(B, 0.0)
    assert np.allclose(lhs, rhs, atol=1e-12)


def test_exact_root_spd_construction():
    _, q, lam = W.spd_stack(count=2, n=32)
    for b in range(2):
        A = (q[b] * lam[b]) @ q[b].T
        X = O.inv_root_exact(A, 1e-8)
        ref = (q[b] * (lam[b] + 1e-8) ** -0.25) @ q[b].T
        assert O.rel_fro(X, ref) < 1e-8


def test_exact_root_clamps_rank_deficient():
    rng = np.random.default_rng(6)
    G = rng.standard_normal((6, 2))
    L = G @ G.T                    # rank 2, four zero eigenvalues (+ roundoff)
    X = O.inv_root_exact(L, 1e-4)
    w = np.linalg.eigvalsh(X)
    assert np.sum(np.isclose(w, 1e-4 ** -0.25, rtol=1e-6)) == 4


def test_exact_root_scalar():
    assert math.isclose(O.inv_root_exact(np.array([[16.0]]), 0.0)[0, 0], 0.5, rel_tol=1e-15)


# Kronecker bound and the one-sided bounds of the Shampoo notes, brute force.

@pytest.mark.parametrize("m,n", [(2, 2), (2, 3), (3, 2), (3, 4), (4, 4)])
def test_kronecker_bound_brute_force(m, n):
    rng = np.random.default_rng(10 * m + n)
    eps = 1e-3
    r = min(m, n)
    X = eps * np.eye(m * n)
    Lt = eps * np.eye(m)
    Rt = eps * np.eye(n)
    for t in range(6):
        G = rng.standard_normal((m, n))
        g = G.reshape(-1)                         # row-major vec
        X = X + np.outer(g, g) / r
        Lt, Rt = O.update_stats(G, Lt, Rt, beta2=1.0)
        # one-sided: (1/r) g g^T <= G G^T (x) I  and  <= I (x) G^T G
        one = np.outer(g, g) / r
        assert np.linalg.eigvalsh(np.kron(G @ G.T, np.eye(n)) - one).min() >= -1e-10
        assert np.linalg.eigvalsh(np.kron(np.eye(m), G.T @ G) - one).min() >= -1e-10
        # Kronecker: X <= L^{1/2} (x) R^{1/2}
        K = np.kron(O.spd_power(Lt, 0.5), O.spd_power(Rt, 0.5))
        assert np.linalg.eigvalsh(K - X).min() >= -1e-10


def test_trace_bound_unit_spectral_norm():
    rng = np.random.default_rng(11)
    m, n, T = 5, 4, 9
    L = np.zeros((m, m))
    for _ in range(T):
        G = rng.standard_normal((m, n))
        G /= np.linalg.norm(G, 2)
        L, _ = O.update_stats(G, L, np.zeros((n, n)), beta2=1.0)
    assert np.trace(O.spd_power(L, 0.25)) <= m * T ** 0.25 + 1e-12


# ---------------------------------------------------------------- O4 scale -----

def test_frobenius_scale_loops():
    rng = np.random.default_rng(12)
    A = rng.standard_normal((5, 5))
    eps = 0.25
    tot = 0.0
    for i in range(5):
        for j in range(5):
            a = A[i, j] + (eps if i == j else 0.0)
            tot += a * a
    assert math.isclose(O.frobenius_scale(A, eps), math.sqrt(tot), rel_tol=1e-14)


def test_power_iteration_bounds_and_limits():
    rng = np.random.default_rng(13)
    A, q, lam = _spd(rng, 40, cond=1e3)
    starts = rng.standard_normal((16, 40))
    lmax = lam[-1]
    for iters in (0, 1, 3, 10):
        s = O.power_iteration_scale(A, 0.0, starts, iters)
        assert s <= lmax * (1 + 1e-12)
        assert s >= lam[0] - 1e-12
    # a spectral gap gives convergence to lambda_max
    lam2 = lam.copy()
    lam2[-1] = 3.0
    A2 = (q * lam2) @ q.T
    assert math.isclose(O.power_iteration_scale(A2, 0.0, starts, 60), 3.0, rel_tol=1e-10)
    # a start vector equal to the top eigenvector is exact at once
    assert math.isclose(O.power_iteration_scale(A, 0.5, q[:, -1:].T, 0), lmax + 0.5, rel_tol=1e-12)


# ---------------------------------------------------------------- O4 NDB -------

def test_ndb_matmul_count_matches_dash():
    g = json.load(open(os.path.join(GOLDEN, "dash_matmul_counts.json")))["newton_db"]
    per, saved = g["matmuls_per_iteration"], g["first_iteration_saves"]
    A = np.eye(4) * 0.5
    for k in (1, 2, 5):
        _, _, mm = O.ndb_matrix(A, k)
        assert mm == per * k - saved
        _, total = O.ndb_inv_root(A, 0.0, 1.0, k)
        assert total == g["calls_for_inverse_fourth_root"] * (per * k - saved)


def test_ndb_first_iteration_closed_form_equals_general_step():
    rng = np.random.default_rng(14)
    A, _, _ = _spd(rng, 6)
    I = np.eye(6)
    # the general iteration started from Z_0 = I, written out by hand
    T = 0.5 * (3 * I - I @ A)
    Y1, Z1 = A @ T, T @ I
    Y, Z, _ = O.ndb_matrix(A, 1)
    assert np.allclose(Y, Y1, atol=1e-15) and np.allclose(Z, Z1, atol=1e-15)


def test_ndb_replay_equals_matrix_iteration():
    rng = np.random.default_rng(15)
    L, _, _ = _spd(rng, 10, cond=1e3)
    for k in (1, 2, 4, 9):
        for s in (1.0, 2.5):
            X1, _ = O.ndb_inv_root(L, 1e-4, s, k)
            X2 = O.ndb_inv_root_replay(L, 1e-4, s, k)
            assert O.rel_fro(X2, X1) < 1e-11


def test_ndb_converges_to_exact_root():
    rng = np.random.default_rng(16)
    L, _, lam = _spd(rng, 16, cond=50.0)
    s = lam[-1] * 1.1
    X, _ = O.ndb_inv_root(L, 1e-6, s, 30)
    assert O.rel_fro(X, O.inv_root_exact(L, 1e-6)) < 1e-12


def test_ndb_scalar_fixed_point_and_limits():
    y, z = O.ndb_scalar(np.array([1.0]), 7)
    assert y[0] == 1.0 and z[0] == 1.0
    a = np.array([0.01, 0.3, 1.7, 2.9])
    y, z = O.ndb_scalar(a, 60)
    assert np.allclose(y, np.sqrt(a), rtol=1e-13) and np.allclose(z, 1 / np.sqrt(a), rtol=1e-13)
    y1, z1 = O.ndb_scalar(a, 1)
    assert np.allclose(y1, a * (3 - a) / 2) and np.allclose(z1, (3 - a) / 2)


# ---------------------------------------------------------------- O4 CN --------

def test_cn_invariant_and_replay():
    rng = np.random.default_rng(17)
    L, _, lam = _spd(rng, 8, cond=200.0)
    s = O.frobenius_scale(L, 1e-5)
    A = (L + 1e-5 * np.eye(8)) / s
    I = np.eye(8)
    X, M = I.copy(), A.copy()
    for k in range(1, 6):
        Xk, mm = O.cn_matrix(A, k)
        assert mm == 4 * k
        # invariant of the coupled iteration: M_k = X_k^4 A
        T = (5 * I - M) / 4
        X, M = X @ T, np.linalg.matrix_power(T, 4) @ M
        assert np.allclose(M, np.linalg.matrix_power(Xk, 4) @ A, atol=1e-11)
        assert O.rel_fro(O.cn_inv_root_replay(L, 1e-5, s, k), O.cn_inv_root(L, 1e-5, s, k)[0]) < 1e-11


def test_cn_converges_to_exact_root():
    rng = np.random.default_rng(18)
    L, _, _ = _spd(rng, 12, cond=30.0)
    s = O.frobenius_scale(L, 1e-6)
    X, _ = O.cn_inv_root(L, 1e-6, s, 40)
    assert O.rel_fro(X, O.inv_root_exact(L, 1e-6)) < 1e-12


# ---------------------------------------------------------------- O4 CHEB ------

def test_cheb_coefficients_match_numpy_interpolation():
    from numpy.polynomial import chebyshev as C
    for d, eps in ((5, 0.1), (32, 1e-3), (60, 1e-6)):
        c = O.cheb_coefficients(d, eps)
        ref = C.chebinterpolate(lambda t: (eps + (t + 1) / 2) ** -0.25, d)
        assert np.allclose(c, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_cheb_interpolates_at_nodes():
    d, eps = 9, 0.05
    c = O.cheb_coefficients(d, eps)
    from numpy.polynomial import chebyshev as C
    nodes = C.chebpts1(d + 1)
    assert np.allclose(C.chebval(nodes, c), (eps + (nodes + 1) / 2) ** -0.25, rtol=1e-12)


def test_clenshaw_scalar_matches_chebval():
    from numpy.polynomial import chebyshev as C
    rng = np.random.default_rng(19)
    c = rng.standard_normal(12)
    t = np.linspace(-1, 1, 33)
    assert np.allclose(O.clenshaw_scalar(c, t), C.chebval(t, c), atol=1e-12)


def test_cheb_matrix_count_and_replay():
    g = json.load(open(os.path.join(GOLDEN, "dash_matmul_counts.json")))["chebyshev_clenshaw"]
    assert g["optimised_matmuls"] == "d - 1"
    rng = np.random.default_rng(20)
    L, _, _ = _spd(rng, 9, cond=100.0)
    s = O.frobenius_scale(L)
    for d in (0, 1, 2, 3, 8, 32):
        X, mm = O.cheb_inv_root(L, 1e-3, s, d)
        assert mm == max(d - 1, 0)
        assert O.rel_fro(O.cheb_inv_root_replay(L, 1e-3, s, d), X) < 1e-11


def test_cheb_high_degree_reaches_damped_root():
    # with eps inside the scaled interval the polynomial approximates
    # (L/s + eps I)^{-1/4}, i.e. s^{1/4} (L + s eps I)^{-1/4}
    rng = np.random.default_rng(21)
    L, _, _ = _spd(rng, 10, cond=10.0)
    s = O.frobenius_scale(L)
    X, _ = O.cheb_inv_root(L, 0.05, s, 80)
    assert O.rel_fro(X, O.inv_root_exact(L, 0.05 * s)) < 1e-10


# ---------------------------------------------------------------- models -------

def test_round_mantissa_matches_ieee_half():
    # fp16 keeps 10 explicit mantissa bits: inside its normal range, rounding
    # a float32 to 10 bits (ties to even) is exactly numpy's half conversion
    rng = np.random.default_rng(30)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-8, 8, 20000))).astype(np.float32)
    x = x[(np.abs(x) > 6.2e-5) & (np.abs(x) < 6.0e4)]
    assert np.array_equal(O.round_mantissa(x, 10), x.astype(np.float16).astype(np.float32))


def test_truncate_mantissa_values():
    one = np.float32(1.0)
    u = np.float32(2.0 ** -10)
    x = np.array([1 + 2 ** -11 + 2 ** -12, 1 + u + 2 ** -11, -(1 + u - 2 ** -12), 3.0], dtype=np.float32)
    assert list(O.truncate_mantissa(x, 10)) == [one, one + u, -one, np.float32(3.0)]
    y = np.random.default_rng(31).standard_normal(1000).astype(np.float32)
    t = O.truncate_mantissa(y, 10)
    assert np.all(np.abs(t) <= np.abs(y)) and np.all(np.abs(y - t) < np.abs(y) * 2.0 ** -10)


def test_precision_models_bracket_exact_result():
    rng = np.random.default_rng(32)
    L, _, _ = _spd(rng, 24, cond=50.0)
    s = O.frobenius_scale(L, 1e-3)
    e32 = O.precision_floor(L, 1e-3, s, "ndb", 10, "fp32")
    e16 = O.precision_floor(L, 1e-3, s, "ndb", 10, "fp16")
    ebf = O.precision_floor(L, 1e-3, s, "ndb", 10, "bf16")
    assert e32 < 1e-5 < e16 < ebf < 1e-1


# ---------------------------------------------------------------- O5 -----------

def test_direction_frobenius_bounds():
    rng = np.random.default_rng(22)
    AL, _, lL = _spd(rng, 7, cond=50.0)
    AR, _, lR = _spd(rng, 5, cond=80.0)
    G = rng.standard_normal((7, 5))
    D = O.precondition(O.inv_root_exact(AL, 0.0), G, O.inv_root_exact(AR, 0.0))
    g = np.linalg.norm(G)
    lo = (lL[-1] * lR[-1]) ** -0.25 * g
    hi = (lL[0] * lR[0]) ** -0.25 * g
    assert lo * (1 - 1e-12) <= np.linalg.norm(D) <= hi * (1 + 1e-12)


def test_direction_fixed_gradient_closed_form():
    rng = np.random.default_rng(23)
    n, k, beta2, eps = 8, 5, 0.999, 1e-6
    U = W.haar_orthogonal(rng, n)[0]
    V = W.haar_orthogonal(rng, n)[0]
    sig = 1.0 / np.arange(1, n + 1)
    G = (U * sig) @ V.T
    L, R = np.zeros((n, n)), np.zeros((n, n))
    for _ in range(k):
        L, R = O.update_stats(G, L, R, beta2)
    c = sum(beta2 ** j for j in range(k))
    D = O.precondition(O.inv_root_exact(L, eps), G, O.inv_root_exact(R, eps))
    ref = (U * (sig * (c * sig ** 2 + eps) ** -0.5)) @ V.T
    assert O.rel_fro(D, ref) < 1e-10


# ---------------------------------------------------------------- O6 -----------

@pytest.mark.parametrize("kind", ["sgd", "adagrad", "adam"])
def test_graft_step_length_invariant(kind):
    rng = np.random.default_rng(24)
    W0 = rng.standard_normal((6, 9))
    G = rng.standard_normal((6, 9))
    D = rng.standard_normal((6, 9)) * 7.0
    m = rng.standard_normal((6, 9)) * 0.1
    v = rng.uniform(0.1, 1.0, (6, 9))
    W1, m1, v1, rhos = O.graft_update(W0, G, D, m, v, kind, lr=0.3, beta1=0.9, beta2=0.99,
                                      eps=1e-8, wd=0.0, step=3)
    if kind == "sgd":
        graft = G
    elif kind == "adagrad":
        graft = G / (np.sqrt(v + G * G) + 1e-8)
    else:
        mm = 0.9 * m + 0.1 * G
        vv = 0.99 * v + 0.01 * G * G
        graft = (mm / (1 - 0.9 ** 3)) / (np.sqrt(vv / (1 - 0.99 ** 3)) + 1e-8)
    assert math.isclose(np.linalg.norm(W1 - W0), 0.3 * np.linalg.norm(graft), rel_tol=1e-12)
    # direction is D's, length is the graft's
    cos = np.sum((W0 - W1) * D) / (np.linalg.norm(W0 - W1) * np.linalg.norm(D))
    assert math.isclose(cos, 1.0, rel_tol=1e-12)


def test_graft_adam_first_step_is_sign_like():
    G = np.array([[2.0, -0.5], [1e-3, -4.0]])
    W1, m, v, _ = O.graft_update(np.zeros((2, 2)), G, np.ones((2, 2)), np.zeros((2, 2)),
                                 np.zeros((2, 2)), "adam", 1.0, 0.9, 0.999, 0.0, 0.0, 1)
    # bias correction makes m_hat = G and v_hat = G^2 at step 1: |graft| = 1 per entry
    assert math.isclose(np.linalg.norm(W1), 2.0, rel_tol=1e-12)


def test_graft_weight_decay_and_zero_direction():
    W0 = np.full((3, 3), 2.0)
    W1, _, _, rhos = O.graft_update(W0, np.ones((3, 3)), np.zeros((3, 3)), None, None, "sgd",
                                    lr=0.1, beta1=0, beta2=0, eps=0, wd=0.5, step=1)
    assert rhos == [0.0]
    assert np.allclose(W1, 2.0 * (1 - 0.05))


def test_graft_blockwise_groups():
    rng = np.random.default_rng(25)
    G = rng.standard_normal((4, 4))
    D = rng.standard_normal((4, 4))
    groups = [(slice(0, 2), slice(None)), (slice(2, 4), slice(None))]
    W1, _, _, rhos = O.graft_update(np.zeros((4, 4)), G, D, None, None, "sgd", 1.0, 0, 0, 0, 0, 1,
                                    groups=groups)
    for (sl, rho) in zip(groups, rhos):
        assert math.isclose(np.linalg.norm(W1[sl]), np.linalg.norm(G[sl]), rel_tol=1e-12)


def test_full_step_sgd_graft_length():
    shapes = [(12, 10)]
    st = O.ShampooState(shapes, 4, "sgd")
    rng = np.random.default_rng(26)
    W0 = [np.zeros(shapes[0])]
    G = [rng.standard_normal(shapes[0])]
    W1 = O.shampoo_step(st, W0, G, beta2=1.0, alpha=1.0, eps=1e-6, method="evd", iters=0,
                        scaling="frobenius", graft="sgd", lr=0.1)
    assert math.isclose(np.linalg.norm(W1[0]), 0.1 * np.linalg.norm(G[0]), rel_tol=1e-12)
    # NDB (converged) and EVD agree on a well-conditioned step
    st2 = O.ShampooState(shapes, 4, "sgd")
    st2.factors = [f.copy() for f in st.factors]
    st3 = O.ShampooState(shapes, 4, "sgd")
    st3.factors = [f.copy() for f in st.factors]
    G2 = [rng.standard_normal(shapes[0])]
    a = O.shampoo_step(st2, W1, G2, beta2=1.0, alpha=1.0, eps=1e-6, method="evd", iters=0,
                       scaling="frobenius", graft="sgd", lr=0.1)
    b = O.shampoo_step(st3, W1, G2, beta2=1.0, alpha=1.0, eps=1e-6, method="ndb", iters=40,
                       scaling="frobenius", graft="sgd", lr=0.1)
    assert O.rel_fro(b[0], a[0]) < 1e-9


def test_stale_roots_between_preconditioner_updates():
    """Roots every f steps ("3D-Shampoo optimizer" README, Hyperparameters:
    preconditioning_compute_steps).  One full-rank 8x8 block, the same G every
    step, beta2 = 1, eps = 0, exact roots, no grafting, lr = 1: after k steps
    L = k G G^T, so a fresh root gives D_k = k^(-1/2) D_1 exactly, while a
    stale root (computed at step 1) gives D_k = D_1."""
    rng = np.random.default_rng(3)
    G = rng.standard_normal((8, 8))
    kw = dict(beta2=1.0, alpha=1.0, eps=0.0, method="evd", iters=0, scaling="frobenius", graft="none", lr=1.0)

    def deltas(f, steps):
        st = O.ShampooState([(8, 8)], 8, "none")
        W = [np.zeros((8, 8))]
        out = []
        for _ in range(steps):
            W2 = O.shampoo_step(st, W, [G], precond_every=f, **kw)
            out.append(W2[0] - W[0])
            W = W2
        return out

    d1 = deltas(1, 3)
    d2 = deltas(2, 3)
    assert np.allclose(d1[1], d1[0] / math.sqrt(2.0), rtol=1e-9, atol=0)
    assert np.allclose(d1[2], d1[0] / math.sqrt(3.0), rtol=1e-9, atol=0)
    assert np.array_equal(d2[0], d1[0])
    assert np.allclose(d2[1], d2[0], rtol=1e-12, atol=0)          # stale: roots of step 1
    assert np.allclose(d2[2], d1[0] / math.sqrt(3.0), rtol=1e-9, atol=0)  # recomputed at step 3


@pytest.mark.parametrize("p", [2, 8])
def test_ndb_root_power_chain(p):
    """Root power p (reading R12): Newton-DB chains log2(p) calls.  On a
    well-conditioned SPD matrix (kappa 10) 25 iterations per call converge,
    so the result is the plain definition (L + eps I)^(-1/p) from the
    eigendecomposition; the matrix form and the eigenvalue replay agree."""
    rng = np.random.default_rng(30 + p)
    Q = np.linalg.qr(rng.standard_normal((12, 12)))[0]
    lam = np.linspace(0.1, 1.0, 12)
    L = (Q * lam) @ Q.T
    s = O.frobenius_scale(L, 1e-6)
    X, mm = O.ndb_inv_root(L, 1e-6, s, 25, p=p)
    assert mm == O.ndb_calls(p) * (1 + 3 * 24)
    assert O.rel_fro(X, (Q * (lam + 1e-6) ** (-1.0 / p)) @ Q.T) < 1e-10
    assert O.rel_fro(O.ndb_inv_root_replay(L, 1e-6, s, 25, p), X) < 1e-10
    # X^p (L + eps I) = I
    assert np.linalg.norm(np.linalg.matrix_power(X, p) @ (L + 1e-6 * np.eye(12)) - np.eye(12)) < 1e-9


def test_plan_layerwise_is_per_layer_global_stacking():
    """Layerwise stacking ([DASH] §4: DASH-LAYERWISE stacks per layer): a
    single layer plans exactly as with stacking across layers, and for
    several layers every bucket holds one layer's blocks, in the order and
    with the counts that layer's own plan gives."""
    one = [(4096, 1024)]
    a, b = O.plan_blocks(one, 1024), O.plan_blocks(one, 1024, layerwise=True)
    for k in ("blocks", "g_buckets", "f_buckets"):
        assert np.array_equal(a[k], b[k])
    shapes = [(300, 200), (200, 300), (128, 128), (300, 200)]
    lw = O.plan_blocks(shapes, 128, layerwise=True)
    gb_off = fb_off = 0
    for li, shp in enumerate(shapes):
        own = O.plan_blocks([shp], 128)
        mine = lw["blocks"][lw["blocks"][:, 0] == li]
        assert np.array_equal(mine[:, 1:7], own["blocks"][:, 1:7])
        assert np.array_equal(mine[:, [7, 9, 11]] - [gb_off, fb_off, fb_off], own["blocks"][:, [7, 9, 11]])
        assert np.array_equal(mine[:, [8, 10, 12]], own["blocks"][:, [8, 10, 12]])
        assert np.array_equal(lw["g_buckets"][gb_off:gb_off + len(own["g_buckets"])], own["g_buckets"])
        assert np.array_equal(lw["f_buckets"][fb_off:fb_off + len(own["f_buckets"])], own["f_buckets"])
        gb_off += len(own["g_buckets"])
        fb_off += len(own["f_buckets"])
    assert gb_off == len(lw["g_buckets"]) and fb_off == len(lw["f_buckets"])


# ---- warm-started coupled Newton (reading R14) ------------------------------

def _haar(n, rng):
    q, r = np.linalg.qr(rng.standard_normal((n, n)))
    return q * np.sign(np.diag(r))


@pytest.mark.parametrize("p", [2, 4, 8])
def test_cn_warm_from_exact_root_is_a_fixed_point(p):
    """Started at the exact root, M_0 = I, so T = I and every iterate stays
    at the start: the exact (L + eps I)^{-1/p} is a fixed point."""
    rng = np.random.default_rng(5)
    Q = _haar(24, rng)
    lam = 10.0 ** rng.uniform(-3, 1, 24)
    L = (Q * lam) @ Q.T
    X0 = (Q * (lam + 1e-4) ** (-1.0 / p)) @ Q.T
    X = O.cn_inv_root_warm(L, X0, 1e-4, 6, p)
    assert O.rel_fro(X, X0) < 1e-12


@pytest.mark.parametrize("p", [2, 4, 8])
def test_cn_warm_commuting_start_is_the_scalar_recurrence(p):
    """A start that shares L's eigenvectors keeps the iteration diagonal in
    that basis: eigenvalue by eigenvalue x = x0 * (cold scalar recurrence on
    m0 = x0^p a).  Checks the matrix products (order, powers, the M_0
    product) against the scalar update."""
    rng = np.random.default_rng(6)
    Q = _haar(20, rng)
    lam = 10.0 ** rng.uniform(-2, 0, 20)
    L = (Q * lam) @ Q.T
    x0 = (lam * rng.uniform(0.7, 1.4, 20)) ** (-1.0 / p)
    X0 = (Q * x0) @ Q.T
    a = lam + 1e-3
    x = x0 * O.cn_scalar(x0 ** p * a, 5, p)
    assert O.rel_fro(O.cn_inv_root_warm(L, X0, 1e-3, 5, p), (Q * x) @ Q.T) < 1e-12


def test_cn_warm_from_scaled_identity_is_cold_cn():
    """X0 = s^{-1/p} I commutes with everything: M_0 = A/s and X_k =
    s^{-1/p} times the cold iterate, i.e. the cold coupled Newton with
    scale s."""
    rng = np.random.default_rng(7)
    B = rng.standard_normal((32, 48))
    L = B @ B.T
    s = O.frobenius_scale(L, 1e-6)
    X0 = s ** (-0.25) * np.eye(32)
    cold, _ = O.cn_inv_root(L, 1e-6, s, 9)
    assert O.rel_fro(O.cn_inv_root_warm(L, X0, 1e-6, 9), cold) < 1e-12


def test_cn_warm_start_improves_a_stale_root():
    """One statistics update later (beta2 = 0.999, one new gradient), the
    previous exact root does not commute with the new factor, so the warm
    iteration settles at its own fixed point instead of the exact root: it
    gets there within three iterations and is better than the stale root
    it started from."""
    rng = np.random.default_rng(8)
    G = [rng.standard_normal((64, 256)) for _ in range(2)]
    L0 = G[0] @ G[0].T
    L1 = 0.999 * L0 + G[1] @ G[1].T * 1e-3
    eps = 1e-3
    exact = O.inv_root_exact(L1, eps)
    X0 = O.inv_root_exact(L0, eps)
    e_start = O.rel_fro(X0, exact)
    e3 = O.rel_fro(O.cn_inv_root_warm(L1, X0, eps, 3), exact)
    e10 = O.rel_fro(O.cn_inv_root_warm(L1, X0, eps, 10), exact)
    assert e3 < 0.5 * e_start
    assert abs(e3 - e10) < 1e-3 * e10


# ---- EVD roots with the dampening heuristics (reading R15) -------------------

def _known_spectrum(lam, seed):
    rng = np.random.default_rng(seed)
    q, r = np.linalg.qr(rng.standard_normal((len(lam), len(lam))))
    Q = q * np.sign(np.diag(r))
    return Q, (Q * np.asarray(lam, np.float64)) @ Q.T


# L's eigenvalues, eps = 1e-2, and the diagonal each heuristic gives in
# L's eigenbasis, written out by hand from [DASH] B.1-B.2:
#   corrected     (max(l, 0) + eps)^(-1/4)
#   shifted_relu  (l - eps)^(-1/4) where l > eps, else 0
#   abs_add       (|l| + eps)^(-1/4)
#   shmp          mu = l + eps has min 0.006 > 0, so l + 2 eps
_LAM = [3.0, 0.5, 2e-2, 5e-3, 0.0, -4e-3]
_EXPECT = {
    "corrected": [3.01, 0.51, 0.03, 0.015, 0.01, 0.01],
    "shifted_relu": [2.99, 0.49, 0.01, None, None, None],
    "abs_add": [3.01, 0.51, 0.03, 0.015, 0.01, 0.014],
    "shmp": [3.02, 0.52, 0.04, 0.025, 0.02, 0.016],
}


@pytest.mark.parametrize("heuristic", ["corrected", "shifted_relu", "abs_add", "shmp"])
def test_evd_heuristics_on_a_known_spectrum(heuristic):
    Q, L = _known_spectrum(_LAM, 21)
    f = np.array([0.0 if d is None else d ** -0.25 for d in _EXPECT[heuristic]])
    assert O.rel_fro(O.evd_inv_root(L, 1e-2, heuristic), (Q * f) @ Q.T) < 1e-10


def test_evd_shmp_with_a_negative_damped_eigenvalue():
    """mu_min = -0.05 + 0.01 < 0: SHMP shifts every mu by -mu_min + eps, so
    the smallest lands on eps and the others on l + eps - mu_min + eps."""
    lam = [2.0, 0.1, -0.05]
    Q, L = _known_spectrum(lam, 22)
    d = np.array([2.0 + 0.01 + 0.04 + 0.01, 0.1 + 0.01 + 0.04 + 0.01, 0.01])
    assert O.rel_fro(O.evd_inv_root(L, 1e-2, "shmp", p=2), (Q * d ** -0.5) @ Q.T) < 1e-10


def test_evd_corrected_is_the_exact_root_and_shifted_relu_kills_the_null_space():
    rng = np.random.default_rng(23)
    G = rng.standard_normal((16, 5))
    L = G @ G.T  # rank 5 of 16
    assert O.rel_fro(O.evd_inv_root(L, 1e-3), O.inv_root_exact(L, 1e-3)) < 1e-9
    X = O.evd_inv_root(L, 1e-3, "shifted_relu")
    null = np.linalg.svd(G.T)[2][5:]  # orthonormal rows spanning L's null space
    assert np.abs(X @ null.T).max() < 1e-9 * np.abs(X).max()
    # on the range it is (lambda - eps)^(-1/4)
    w, U = np.linalg.eigh(L)
    U5, w5 = U[:, -5:], w[-5:]
    assert O.rel_fro(U5.T @ X @ U5, np.diag((w5 - 1e-3) ** -0.25)) < 1e-9


# ---- one-sided layers and shape interpretation (readings R16, R17) ----------

def test_plan_one_sided_layers():
    """A one-sided layer keeps left factors only, in stacks of its own."""
    shapes = [(128, 96), (128, 96), (64, 64)]
    pl = O.plan_blocks(shapes, 64, left_only=[False, True, False])
    blk = pl["blocks"]
    one = blk[blk[:, 0] == 1]
    assert (one[:, 11] == -1).all() and (one[:, 12] == -1).all()
    assert (blk[blk[:, 0] != 1][:, 11] >= 0).all()
    # no stack mixes sides
    assert set(one[:, 7]).isdisjoint(set(blk[blk[:, 0] != 1][:, 7]))
    assert set(one[:, 9]).isdisjoint(set(blk[blk[:, 0] != 1][:, 9]))
    assert all(pl["f_sides"][f] == 1 for f in one[:, 9])
    # with no one-sided layer the tables are the two-sided plan's
    a, b = O.plan_blocks(shapes, 64), O.plan_blocks(shapes, 64, left_only=[False] * 3)
    for k in ("blocks", "g_buckets", "f_buckets", "f_sides"):
        assert np.array_equal(a[k], b[k])
    assert (a["f_sides"] == 0).all()


def test_one_sided_step_is_the_svd_closed_form():
    """One step, beta2 = 1, one block: L = G G^T, X_L = (L + eps I)^{-1/2},
    so D = U diag(s / sqrt(s^2 + eps)) V^T from the SVD G = U diag(s) V^T,
    and with no graft W = -lr D."""
    rng = np.random.default_rng(31)
    G = rng.standard_normal((24, 40))
    st = O.ShampooState([(24, 40)], 0, "none", left_only=[True])
    W = O.shampoo_step(st, [np.zeros((24, 40))], [G], beta2=1.0, alpha=1.0, eps=1e-2, method="evd",
                       iters=0, scaling="frobenius", graft="none", lr=0.5)
    U, sv, Vt = np.linalg.svd(G, full_matrices=False)
    D = (U * (sv / np.sqrt(sv ** 2 + 1e-2))) @ Vt
    assert O.rel_fro(W[0], -0.5 * D) < 1e-10
    assert len(st.factors) == 1 and st.factors[0].shape == (1, 24, 24)


def test_matrix_shape_merges_trailing_dimensions():
    assert O.matrix_shape((384, 3, 16, 16)) == (384, 768)
    assert O.matrix_shape((512, 5, 5, 64)) == (512, 1600)
    assert O.matrix_shape((7, 9)) == (7, 9)
    assert O.matrix_shape((10,)) is None and O.matrix_shape(()) is None


def test_statistics_frequency_updates_on_schedule():
    """statistics_compute_steps = 2: the statistics after steps 1..4 hold
    the gradients of steps 1 and 3 only (beta2 = 1: a plain sum)."""
    rng = np.random.default_rng(41)
    G = [rng.standard_normal((8, 6)) for _ in range(4)]
    st = O.ShampooState([(8, 6)], 0, "sgd")
    W = [np.zeros((8, 6))]
    for t in range(4):
        W = O.shampoo_step(st, W, [G[t]], beta2=1.0, alpha=1.0, eps=1e-3, method="evd", iters=0,
                           scaling="frobenius", graft="sgd", lr=0.1, stats_every=2)
    lb, li, rb, ri = (int(x) for x in st.plan["blocks"][0][9:13])
    assert np.allclose(st.factors[lb][li], G[0] @ G[0].T + G[2] @ G[2].T, rtol=1e-12)
    assert np.allclose(st.factors[rb][ri], G[0].T @ G[0] + G[2].T @ G[2], rtol=1e-12)
