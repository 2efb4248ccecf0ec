"""GPU parity of every hot-path call against the float64 oracle.

Each test feeds identical seeded float32 inputs to the CUDA path (through the
C ABI) and to the oracle, and compares element by element (relative
Frobenius error) at sizes that span several 128-wide tiles plus a ragged
tail.  Integer work (block tables, stacking) must be bit-exact.
"""
import math

import numpy as np
import pytest

import oracle as O
from matrix_roots_b200 import binding as B
from matrix_roots_b200 import workloads as W

from gpu_util import rel, spd_stack, to_dev

pytestmark = pytest.mark.gpu

RAGGED = [(200, 136), (64, 300), (4, 8)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from matrix_roots_b200 import build
    build.build()
    B.lib()
    yield
    assert B.device_error() == 0


def _grads(shapes, seed):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal(s).astype(np.float32) for s in shapes]


# ------------------------------------------------------------------ a1 ------

@pytest.mark.parametrize("shapes,bs", [(RAGGED, 128), ([(32000 // 8, 2048 // 4)], 128), (RAGGED, 0)])
def test_stack_blocks_bit_exact(shapes, bs):
    import torch
    plan = B.Plan(shapes, bs).bind()
    t = plan.tables()
    grads = _grads(shapes, 1)
    g_dev = [to_dev(g) for g in grads]
    stacks = [torch.full((int(c), int(r), int(k)), float("nan"), device="cuda") for r, k, c in t["g_buckets"]]
    B.stack_blocks(plan, g_dev, stacks)
    ref = O.stack_gradients(O.plan_blocks(shapes, bs), grads)
    for s, r in zip(stacks, ref):
        assert np.array_equal(s.cpu().numpy(), r.astype(np.float32))


# ------------------------------------------------------------------ a2 ------

@pytest.mark.parametrize("bs", [128, 0])
@pytest.mark.parametrize("dtype,tol", [("fp32", 2e-5), ("tf32", 3e-3), ("fp16", 3e-3), ("bf16", 2e-2)])
def test_update_stats(dtype, tol, bs):
    """Statistics against float64.  Block size 0 keeps the layers whole, so
    the factors (200, 136, 64, 300) span two or three 128-wide tiles with a
    ragged last one: the symmetric products are computed on their upper
    tiles and mirrored, reading the old statistics at the mirrored places."""
    import torch
    shapes = [(200, 136), (64, 300)]
    plan = B.Plan(shapes, bs).bind()
    t = plan.tables()
    grads = _grads(shapes, 2)
    ref_plan = O.plan_blocks(shapes, bs)
    g_st = O.stack_gradients(ref_plan, grads)
    rng = np.random.default_rng(3)
    f0 = []
    for n, c in t["f_buckets"]:
        f0.append(np.stack([spd_stack(1, int(n), 10.0, seed=int(rng.integers(1 << 30)))[0] for _ in range(int(c))]))
    g_dev = [to_dev(g.astype(np.float32)) for g in g_st]
    f_dev = [to_dev(f) for f in f0]
    B.update_stats(plan, g_dev, f_dev, beta2=0.9, alpha=0.3, dtype=dtype)
    torch.cuda.synchronize()
    ref = [f.astype(np.float64).copy() for f in f0]
    for b in ref_plan["blocks"]:
        gb, gi, lb, li, rb, ri = (int(x) for x in b[7:13])
        ref[lb][li], ref[rb][ri] = O.update_stats(g_st[gb][gi], f0[lb][li], f0[rb][ri], 0.9, 0.3)
    for got, r in zip(f_dev, ref):
        for i in range(r.shape[0]):
            assert rel(got[i].cpu().numpy(), r[i]) < tol


# ------------------------------------------------------------------ a3-a6 ---

def _replay(method, L, eps, s, iters):
    return O.inv_root(L, eps, method, iters, s, replay=True)


def _check_scale(method, scaling, L, eps, s_gpu):
    eps_s = 0.0 if method == "cheb" else eps
    if scaling == "frobenius":
        assert math.isclose(s_gpu, O.frobenius_scale(L, eps_s), rel_tol=1e-5)
    else:
        lmax = np.linalg.eigvalsh(L.astype(np.float64))[-1] + eps_s
        assert 0.5 * lmax <= s_gpu <= (1 + 1e-3) * lmax


@pytest.mark.parametrize("n", [64, 200])
@pytest.mark.parametrize("scaling", ["frobenius", "power"])
@pytest.mark.parametrize("dtype", ["fp32", "tf32"])
@pytest.mark.parametrize("method,iters", [("ndb", 12), ("cn", 12), ("cheb", 24)])
def test_inv_root_matches_replay(method, iters, dtype, scaling, n):
    A = spd_stack(5, n, cond=100.0, seed=n)
    eps = 1e-4
    starts = to_dev(W.power_iteration_starts(n, 16)) if scaling == "power" else None
    X, s, st = B.inv_root(to_dev(A), eps, method, iters, dtype, scaling, pi_vectors=16, pi_iters=10,
                          pi_starts=starts)
    X, s, st = X.cpu().numpy(), s.cpu().numpy(), st.cpu().numpy()
    assert np.all(st == 0)
    for b in range(A.shape[0]):
        L = A[b].astype(np.float64)
        _check_scale(method, scaling, L, eps, float(s[b]))
        ref = _replay(method, L, eps, float(s[b]), iters)
        tol = 1e-3
        if dtype == "tf32":  # 10-bit operands: bound from the arithmetic model
            tol = max(tol, 2 * O.precision_floor(L, eps, float(s[b]), method, iters, "tf32"))
        assert rel(X[b], ref) < tol, (b, rel(X[b], ref), tol)


@pytest.mark.parametrize("p", [2, 8])
@pytest.mark.parametrize("method,iters", [("ndb", 14), ("cn", 14), ("cheb", 24)])
def test_inv_root_root_powers(method, iters, p):
    """Root power p (reading R12): Newton-DB as log2(p) chained calls,
    coupled Newton with T^p by squarings, Chebyshev fitted to x^(-1/p);
    FP32 against the replay with the same p, at the stated 1e-3."""
    A = spd_stack(6, 128, cond=100.0, seed=40 + p)
    eps = 1e-4
    X, s, st = B.inv_root(to_dev(A), eps, method, iters, "fp32", "frobenius", p=p)
    X, s, st = X.cpu().numpy(), s.cpu().numpy(), st.cpu().numpy()
    assert np.all(st == 0)
    for b in range(A.shape[0]):
        L = A[b].astype(np.float64)
        ref = O.inv_root(L, eps, method, iters, float(s[b]), p)
        err = rel(X[b], ref)
        assert err < 1e-3, (b, err)


@pytest.mark.parametrize("dtype,tol", [("fp16", 2e-2), ("bf16", None)])
def test_cn_half_precision(dtype, tol):
    A = spd_stack(4, 128, cond=50.0, seed=11)
    X, s, st = B.inv_root(to_dev(A), 1e-4, "cn", 12, dtype, "frobenius")
    X, s, st = X.cpu().numpy(), s.cpu().numpy(), st.cpu().numpy()
    errs = [rel(X[b], _replay("cn", A[b].astype(np.float64), 1e-4, float(s[b]), 12)) for b in range(4)]
    print(f"CN {dtype} rel errors vs replay: {errs}")
    if tol is not None:
        assert max(errs) < tol
    else:  # report only; a non-finite result must be flagged
        for b in range(4):
            assert (st[b] != 0) == (not np.all(np.isfinite(X[b])))


def test_cheb_fp16_multiplication():
    A = spd_stack(4, 128, cond=50.0, seed=12)
    X, s, st = B.inv_root(to_dev(A), 1e-3, "cheb", 32, "fp16", "frobenius")
    X, s = X.cpu().numpy(), s.cpu().numpy()
    errs = [rel(X[b], _replay("cheb", A[b].astype(np.float64), 1e-3, float(s[b]), 32)) for b in range(4)]
    print(f"CHEB fp16 rel errors vs replay: {errs}")
    assert max(errs) < 2e-2


@pytest.mark.parametrize("method,iters", [("ndb", 1), ("ndb", 2), ("cn", 1), ("cn", 2), ("cheb", 0), ("cheb", 1),
                                          ("cheb", 2), ("cheb", 3)])
def test_inv_root_degenerate_iteration_counts(method, iters):
    A = spd_stack(3, 96, cond=20.0, seed=5)
    X, s, st = B.inv_root(to_dev(A), 1e-3, method, iters, "fp32", "frobenius")
    X, s = X.cpu().numpy(), s.cpu().numpy()
    for b in range(3):
        assert rel(X[b], _replay(method, A[b].astype(np.float64), 1e-3, float(s[b]), iters)) < 1e-4


@pytest.mark.parametrize("n", [4, 8, 36, 128, 132, 256, 384])
def test_inv_root_sizes_and_tails(n):
    A = spd_stack(2, n, cond=30.0, seed=n + 1)
    X, s, st = B.inv_root(to_dev(A), 1e-4, "ndb", 16, "fp32", "frobenius")
    X, s = X.cpu().numpy(), s.cpu().numpy()
    for b in range(2):
        assert rel(X[b], _replay("ndb", A[b].astype(np.float64), 1e-4, float(s[b]), 16)) < 1e-4


def test_inv_root_zero_matrix_closed_form():
    # L = 0: A = eps I, so X converges to eps^{-1/4} I
    A = np.zeros((2, 64, 64), dtype=np.float32)
    X, s, st = B.inv_root(to_dev(A), 1e-2, "ndb", 30, "fp32", "frobenius")
    assert np.allclose(X.cpu().numpy(), np.broadcast_to(np.eye(64) * 1e-2 ** -0.25, (2, 64, 64)), rtol=1e-5,
                       atol=1e-5)


def test_inv_root_nonfinite_status_is_per_matrix():
    A = spd_stack(4, 64, cond=10.0, seed=6)
    A[2, 3, 5] = np.nan
    X, s, st = B.inv_root(to_dev(A), 1e-4, "ndb", 10, "fp32", "frobenius")
    st = st.cpu().numpy()
    assert list(st) == [0, 0, 1, 0]
    X = X.cpu().numpy()
    for b in (0, 1, 3):
        assert rel(X[b], _replay("ndb", A[b].astype(np.float64), 1e-4, float(s[b]), 10)) < 1e-3


# ------------------------------------------------------------------ a7 ------

@pytest.mark.parametrize("dtype,tol", [("fp32", 1e-5), ("tf32", 3e-3)])
def test_precondition(dtype, tol):
    import torch
    shapes = [(200, 136), (64, 300)]
    plan = B.Plan(shapes, 128).bind()
    t = plan.tables()
    ref_plan = O.plan_blocks(shapes, 128)
    g_st = O.stack_gradients(ref_plan, _grads(shapes, 4))
    roots = [np.stack([spd_stack(1, int(n), 20.0, seed=10 * int(n) + i)[0] for i in range(int(c))])
             for n, c in t["f_buckets"]]
    g_dev = [to_dev(g.astype(np.float32)) for g in g_st]
    d_dev = [torch.empty_like(g) for g in g_dev]
    dn = torch.empty(plan.n_blocks, device="cuda")
    B.precondition(plan, [to_dev(r) for r in roots], g_dev, d_dev, dn, dtype)
    dn = dn.cpu().numpy()
    off = np.concatenate([[0], np.cumsum(t["g_buckets"][:, 2])])
    for b in ref_plan["blocks"]:
        gb, gi, lb, li, rb, ri = (int(x) for x in b[7:13])
        ref = O.precondition(roots[lb][li], g_st[gb][gi], roots[rb][ri])
        got = d_dev[gb][gi].cpu().numpy()
        assert rel(got, ref) < tol
        assert math.isclose(dn[off[gb] + gi], float(np.sum(ref * ref)), rel_tol=10 * tol)


# ------------------------------------------------------------------ a8 ------

@pytest.mark.parametrize("graft", ["none", "sgd", "adagrad", "adam"])
@pytest.mark.parametrize("per_block", [False, True])
def test_graft_step(graft, per_block):
    import torch
    shapes = [(200, 136), (64, 300)]
    plan = B.Plan(shapes, 128).bind()
    t = plan.tables()
    ref_plan = O.plan_blocks(shapes, 128)
    rng = np.random.default_rng(8)
    W0 = [rng.standard_normal(s).astype(np.float32) for s in shapes]
    G = [rng.standard_normal(s).astype(np.float32) for s in shapes]
    m0 = [(0.1 * rng.standard_normal(s)).astype(np.float32) for s in shapes]
    v0 = [rng.uniform(0.1, 1.0, s).astype(np.float32) for s in shapes]
    d_st = [(3 * rng.standard_normal((int(c), int(r), int(k)))).astype(np.float32) for r, k, c in t["g_buckets"]]
    dn = np.concatenate([np.sum(d.astype(np.float64) ** 2, axis=(1, 2)) for d in d_st]).astype(np.float32)
    Wd = [to_dev(w) for w in W0]
    md = [to_dev(m) for m in m0]
    vd = [to_dev(v) for v in v0]
    B.graft_step(plan, Wd, [to_dev(g) for g in G], [to_dev(d) for d in d_st], to_dev(dn), md, vd, graft, lr=0.05,
                 beta1=0.9, beta2=0.99, eps=1e-8, weight_decay=0.01, step=3, graft_per_block=per_block)
    torch.cuda.synchronize()
    D = O.unstack_directions(ref_plan, d_st, shapes)
    for li in range(len(shapes)):
        groups = None
        if per_block:
            groups = [(slice(int(b[3]), int(b[3] + b[5])), slice(int(b[4]), int(b[4] + b[6])))
                      for b in ref_plan["blocks"] if b[0] == li]
        w, m, v, _ = O.graft_update(W0[li], G[li], D[li], m0[li], v0[li], graft, 0.05, 0.9, 0.99, 1e-8, 0.01, 3,
                                    groups=groups)
        assert rel(Wd[li].cpu().numpy(), w) < 1e-6
        if graft == "adam":
            assert rel(md[li].cpu().numpy(), m) < 1e-6
        if graft in ("adam", "adagrad"):
            assert rel(vd[li].cpu().numpy(), v) < 1e-6
