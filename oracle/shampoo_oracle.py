"""Plain float64 CPU oracle for one blocked-Shampoo optimizer step.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
cpu_baseline / reference leg of ``bench.py`` may import or run this module.
It shares no code with the CUDA path (no kernels, headers, tables or
helpers) and imports nothing from it.  It is slow on purpose: every step is
written the way the pages state it, with NumPy float64 matmuls / ``eigh`` as
the only library primitives.

Sources (cited by short name below):

[DASH]        "DASH: Faster Shampoo via Batched Block Preconditioning and
              Efficient Inverse-Root Solvers" (Modoranu, Zmushko, Schultheis,
              Safaryan, Alistarh; arXiv 2602.02016v2), section summary.
[DistShampoo] "A Distributed Data-Parallel PyTorch Implementation of the
              Distributed Shampoo Optimizer for Training Neural Networks
              At-Scale" (Shi et al.), abstract.
[3D-Shampoo]  "3D-Shampoo optimizer" README ("Hyperparameters", "Tests").
[Notes]       "Shampoo" notes (speedrun/shampoo): "The guarantee", the
              one-sided bounds, "the Kronecker bound", "Roots on idle CPUs",
              "Spreading the preconditioners", "Grafting corrects ...".

Readings taken where the pages are silent or ambiguous (each one is also a
row of the readings table in the design notes):

R1  Block order inside a bucket: layers in input order; inside a layer all
    left factors (blocks row-major) before all right factors; buckets in order
    of first appearance.  Reproduces the listing order of [DASH] §4.
R2  Statistics: L <- beta2*L + alpha*G G^T with alpha = 1 by default (the
    "exponential moving average" of [DASH] §2 is alpha = 1 - beta2).
R3  Exact root: eigenvalues of L clamped at 0, then eps added once
    ([DASH] B.1 corrected spectrum).
R4  Newton-DB is the inverse-free coupled Newton-Schulz / Denman-Beavers
    form (3 matmuls per iteration, the first iteration closed-form).
    "iters" counts iterations per call; the second call starts from the
    first call's Y with Z = I and no re-scaling.
R5  Coupled Newton (Guo-Higham): M0 = A/s, X0 = I, T = ((p+1)I - M)/p,
    X <- X T, M <- T^p M.
R6  Chebyshev: x^{-1/p} fitted at the degree+1 first-kind Chebyshev nodes of
    [eps, 1+eps]; S = 2 L/s - I with L undamped; result s^{-1/p} p(S).
R7  Multi-power-iteration: V <- normalise(A V) `iters` times, then the
    largest Rayleigh quotient v^T A v; start vectors are an input.
R8  Grafting is layerwise by default; Adam bias-corrected with eps_g; decoupled
    weight decay W <- W - lr*rho*D - lr*wd*W; rho = 0 when ||D|| = 0.
R12 Root power p: p in {2, 4, 8} ([Notes] "Spreading the preconditioners":
    the square-root power is often effective for networks made mostly of
    linear layers); Newton-DB chains log2(p) calls, each on the previous
    call's Y; coupled Newton and Chebyshev take p directly.
R11 Preconditioner frequency f: statistics every step, roots on steps
    1, 1+f, 1+2f, ... and the last roots reused in between ([3D-Shampoo]
    Hyperparameters: preconditioning_compute_steps; [DASH] §1).  The
    statistics frequency s (statistics_compute_steps) likewise updates the
    statistics on steps 1, 1+s, ... only; every step is preconditioned.
R16 One-sided layers ([Notes] "Roots on idle CPUs": embedding and softmax
    layers, and layers too large for a right factor, are preconditioned on
    one side only, L^{-1/2} G, the alpha = 1 split of the Kronecker bound):
    such a layer keeps only left factors; its gradient and factor stacks are
    separate from the two-sided ones (bucket keys carry the side); its
    roots are inverse square roots, D = X_L G.  A layer whose large side is
    its rows is passed transposed by the caller.
R17 Shape interpretation ([DASH] D: a ViT embedding (E, 3, 16, 16) becomes
    (E, 768)): a parameter of rank > 2 is preconditioned as the matrix
    (first dimension, product of the others); rank 1 and 0 are not.
R15 EVD roots with the dampening heuristics of [DASH] B.1-B.2: the
    eigendecomposition is taken of L + eps I, mu = its eigenvalues, and
    lambda = mu - eps (the corrected spectrum).  corrected: (max(lambda, 0)
    + eps)^{-1/p} (= R3); shifted-ReLU: r = max(lambda - eps, 0), r^{-1/p}
    where r > 0 and 0 elsewhere (a rank-r_eps inverse); ABS-add:
    (|lambda| + eps)^{-1/p}; SHMP (the Distributed Shampoo adjustment B.1
    describes, eps added twice): mu - min(min(mu), 0) + eps.
R13 Layerwise stacking: the R1 partition and order with buckets keyed by
    (layer, shape), so no stack mixes layers ([DASH] §4, Stacking strategy).
R14 Warm-started coupled Newton ([Notes] "Roots on idle CPUs": the roots
    start from the previous root): X_0 = the previous root, M_0 = X_0^p A
    (the iteration's invariant M = X^p A), no scaling, then the R5 update.
    Exact when X_0 commutes with A; otherwise the result is the same
    iteration's, not A^{-1/p}.

Parity unpinned: the power-iteration iteration count (R7: no page fixes it),
the step-count example of [DASH] §3 (Frobenius scaling 5 -> 15 steps).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "BLOCK_FIELDS", "split_dim", "plan_blocks", "stack_gradients", "unstack_directions",
    "matrix_shape", "update_stats", "spd_power", "inv_root_exact", "EVD_HEURISTICS", "evd_root_factors", "evd_inv_root",
    "frobenius_scale", "power_iteration_scale",
    "ndb_matrix", "ndb_calls", "ndb_inv_root", "ndb_scalar", "ndb_inv_root_replay",
    "cn_matrix", "cn_inv_root", "cn_inv_root_warm", "cn_scalar", "cn_inv_root_replay",
    "cheb_coefficients", "clenshaw_scalar", "cheb_matrix", "cheb_inv_root", "cheb_inv_root_replay",
    "inv_root", "precondition", "graft_update", "ShampooState", "compute_roots", "shampoo_step",
    "rel_fro", "round_mantissa", "truncate_mantissa", "precision_floor",
]

# --------------------------------------------------------------------------
# O1  Block partitioning and stacking
#     [3D-Shampoo] Hyperparameters (block_size: split dimensions larger than
#     this; 0 = never split); [DASH] §1 (B x B blocking) and §4 Blocking
#     Strategy (same-shape blocks stacked into 3D tensors).
# --------------------------------------------------------------------------

BLOCK_FIELDS = ("layer", "block_row", "block_col", "row0", "col0", "rows", "cols",
                "g_bucket", "g_index", "l_bucket", "l_index", "r_bucket", "r_index")


def split_dim(d: int, block_size: int) -> list[int]:
    """Sizes of the blocks one dimension is cut into.

    A dimension larger than the block size becomes floor(d/B) blocks of B and
    one remainder block of d mod B (when nonzero); a dimension <= B, or
    B = 0, stays whole ([3D-Shampoo] Hyperparameters; [DASH] §4: V = 32000 at
    B = 1024 gives 31 full rows of blocks and one of 256).
    """
    if d <= 0:
        raise ValueError("dimension must be positive")
    if block_size <= 0 or d <= block_size:
        return [d]
    sizes = [block_size] * (d // block_size)
    if d % block_size:
        sizes.append(d % block_size)
    return sizes


def plan_blocks(shapes, block_size: int, layerwise: bool = False, left_only=None) -> dict:
    """Partition every layer into blocks and assign them to stacks.

    Returns int32 tables:
      blocks    (n_blocks, 13) with the columns of ``BLOCK_FIELDS``;
      g_buckets (n_g, 3)  rows, cols, count of each gradient-block stack;
      f_buckets (n_f, 2)  n, count of each preconditioner-factor stack;
      f_sides   (n_f,)    0: factors of two-sided blocks, 1: left factors of
                          one-sided blocks (reading R16).
    Gradient blocks are bucketed by (rows, cols), factors by n ([DASH] §4);
    the order inside buckets is reading R1.  ``layerwise`` keys the buckets
    by layer as well ([DASH] §4: DASH-LAYERWISE stacks per layer, DASH-GPU
    across all layers of a GPU).  ``left_only[i]`` true makes layer i
    one-sided: its blocks get no right factor (fields -1) and both its
    buckets are keyed by the side too.
    """
    blocks = []
    g_key_to_id: dict = {}
    g_counts: list = []
    f_key_to_id: dict = {}
    f_counts: list = []
    f_sides: list = []

    def f_slot(n, li, side):
        key = (li, n, side) if layerwise else (n, side)
        if key not in f_key_to_id:
            f_key_to_id[key] = len(f_counts)
            f_counts.append([n, 0])
            f_sides.append(side)
        b = f_key_to_id[key]
        idx = f_counts[b][1]
        f_counts[b][1] += 1
        return b, idx

    for li, (m, n) in enumerate(shapes):
        side = 1 if left_only is not None and left_only[li] else 0
        rs = split_dim(int(m), block_size)
        cs = split_dim(int(n), block_size)
        layer_blocks = []
        row0 = 0
        for br, r in enumerate(rs):
            col0 = 0
            for bc, c in enumerate(cs):
                key = (li, r, c, side) if layerwise else (r, c, side)
                if key not in g_key_to_id:
                    g_key_to_id[key] = len(g_counts)
                    g_counts.append([r, c, 0])
                gb = g_key_to_id[key]
                gi = g_counts[gb][2]
                g_counts[gb][2] += 1
                layer_blocks.append([li, br, bc, row0, col0, r, c, gb, gi, -1, -1, -1, -1])
                col0 += c
            row0 += r
        for blk in layer_blocks:          # all left factors of the layer, row-major
            blk[9], blk[10] = f_slot(blk[5], li, side)
        if not side:
            for blk in layer_blocks:      # then all right factors, row-major
                blk[11], blk[12] = f_slot(blk[6], li, side)
        blocks += layer_blocks
    return {
        "blocks": np.asarray(blocks, dtype=np.int32).reshape(-1, len(BLOCK_FIELDS)),
        "g_buckets": np.asarray(g_counts, dtype=np.int32).reshape(-1, 3),
        "f_buckets": np.asarray(f_counts, dtype=np.int32).reshape(-1, 2),
        "f_sides": np.asarray(f_sides, dtype=np.int32),
    }


def matrix_shape(shape):
    """The matrix a parameter is preconditioned as (reading R17): rank 2 as
    is, rank > 2 as (first dimension, product of the rest), else None."""
    shape = tuple(int(x) for x in shape)
    if len(shape) < 2:
        return None
    return (shape[0], int(np.prod(shape[1:])))


def stack_gradients(plan: dict, grads) -> list[np.ndarray]:
    """Copy every layer's gradient blocks into their (count, rows, cols) stacks."""
    stacks = [np.zeros((int(c), int(r), int(k)), dtype=np.float64) for (r, k, c) in plan["g_buckets"]]
    for b in plan["blocks"]:
        li, _, _, r0, c0, r, c, gb, gi = (int(x) for x in b[:9])
        stacks[gb][gi] = np.asarray(grads[li], dtype=np.float64)[r0:r0 + r, c0:c0 + c]
    return stacks


def unstack_directions(plan: dict, d_stacks, shapes) -> list[np.ndarray]:
    """Inverse of ``stack_gradients``: scatter blocks back into layer layout."""
    out = [np.zeros(s, dtype=np.float64) for s in shapes]
    for b in plan["blocks"]:
        li, _, _, r0, c0, r, c, gb, gi = (int(x) for x in b[:9])
        out[li][r0:r0 + r, c0:c0 + c] = d_stacks[gb][gi]
    return out


# --------------------------------------------------------------------------
# O2  Statistics update  ([DASH] §2 Preliminaries on Shampoo: moving averages
#     of G G^T and G^T G; beta2 = 1 gives AdaGrad sums)
# --------------------------------------------------------------------------

def update_stats(G, L, R, beta2: float, alpha: float = 1.0):
    """L <- beta2 L + alpha G G^T,  R <- beta2 R + alpha G^T G  (reading R2)."""
    G = np.asarray(G, dtype=np.float64)
    L_new = beta2 * np.asarray(L, dtype=np.float64) + alpha * (G @ G.T)
    R_new = beta2 * np.asarray(R, dtype=np.float64) + alpha * (G.T @ G)
    return L_new, R_new


# --------------------------------------------------------------------------
# O3  Exact inverse root by symmetric eigendecomposition
#     ([DASH] §3 EVD; B.1: eps added once, corrected spectrum)
# --------------------------------------------------------------------------

def spd_power(A, r: float, shift: float = 0.0):
    """Q diag((max(lam,0) + shift)^r) Q^T for symmetric A."""
    A = np.asarray(A, dtype=np.float64)
    A = 0.5 * (A + A.T)
    w, Q = np.linalg.eigh(A)
    w = np.clip(w, 0.0, None) + shift
    return (Q * w ** r) @ Q.T


def inv_root_exact(L, eps: float, p: int = 4):
    """(L + eps I)^{-1/p} with L's eigenvalues clamped at zero (reading R3)."""
    return spd_power(L, -1.0 / p, shift=eps)


EVD_HEURISTICS = ("corrected", "shifted_relu", "abs_add", "shmp")


def evd_root_factors(mu, eps: float, heuristic: str, p: int = 4):
    """f(mu) of reading R15 for the eigenvalues mu of L + eps I."""
    mu = np.asarray(mu, dtype=np.float64)
    lam = mu - eps
    if heuristic == "corrected":
        d = np.maximum(lam, 0.0) + eps
    elif heuristic == "abs_add":
        d = np.abs(lam) + eps
    elif heuristic == "shmp":
        d = mu - min(float(mu.min()), 0.0) + eps
    elif heuristic == "shifted_relu":
        r = np.maximum(lam - eps, 0.0)
        out = np.zeros_like(r)
        pos = r > 0
        out[pos] = r[pos] ** (-1.0 / p)
        return out
    else:
        raise ValueError(heuristic)
    return d ** (-1.0 / p)


def evd_inv_root(L, eps: float, heuristic: str = "corrected", p: int = 4):
    """Q diag(f(mu)) Q^T from eigh(L + eps I) ([DASH] B.1-B.2, reading R15)."""
    L = np.asarray(L, dtype=np.float64)
    A = 0.5 * (L + L.T) + eps * np.eye(L.shape[0])
    mu, Q = np.linalg.eigh(A)
    return (Q * evd_root_factors(mu, eps, heuristic, p)) @ Q.T


# --------------------------------------------------------------------------
# O4  Scaling  ([DASH] §3 Matrix scaling and Power-Iteration; §1)
# --------------------------------------------------------------------------

def frobenius_scale(L, eps: float = 0.0) -> float:
    """||L + eps I||_F, the Frobenius-norm scale of [DASH] §3."""
    A = np.asarray(L, dtype=np.float64) + eps * np.eye(L.shape[0])
    return float(np.sqrt(np.sum(A * A)))


def power_iteration_scale(L, eps: float, starts, iters: int) -> float:
    """Multi-power-iteration estimate of lambda_max(L + eps I) ([DASH] §3, §1).

    All start vectors (rows of ``starts``) are iterated in parallel:
    V <- normalise(A V), ``iters`` times; the estimate is the largest Rayleigh
    quotient v^T A v over the normalised vectors (reading R7).
    """
    A = np.asarray(L, dtype=np.float64) + eps * np.eye(L.shape[0])
    V = np.asarray(starts, dtype=np.float64).T.copy()
    V /= np.linalg.norm(V, axis=0, keepdims=True)
    for _ in range(iters):
        V = A @ V
        nrm = np.linalg.norm(V, axis=0, keepdims=True)
        nrm[nrm == 0] = 1.0
        V /= nrm
    rq = np.sum(V * (A @ V), axis=0)
    return float(np.max(rq))


# --------------------------------------------------------------------------
# Arithmetic models.  The matrix-form iterations below run in float64 by
# default (the oracle).  Given `prec`, the same steps run with float32
# storage and float32-accumulated products whose operands are first reduced
# to the named format: "fp32" (none), "tf32" (10 explicit mantissa bits,
# truncated), "bf16" (7 bits, rounded), "fp16" (IEEE half, rounded).  This models what an arithmetic can
# reach; tests use it only to derive error bounds ([DASH] A.3 and §5 report
# that reduced precision changes the result), never as an expected value.
# --------------------------------------------------------------------------

def round_mantissa(x, bits: int):
    """Round float32 values to `bits` explicit mantissa bits, ties to even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    drop = 23 - bits
    lsb = (u >> np.uint64(drop)) & np.uint64(1)
    u = (u + np.uint64((1 << (drop - 1)) - 1) + lsb) & ~np.uint64((1 << drop) - 1)
    return u.astype(np.uint32).view(np.float32).reshape(x.shape)


def _model(prec):
    """(matmul, store) of an arithmetic model; prec None = float64."""
    if prec is None:
        return (lambda a, b: a @ b), (lambda x: x)

    def f32(x):
        return np.asarray(x, dtype=np.float32)

    rnd = {"fp32": f32,
           "tf32": lambda x: truncate_mantissa(x, 10),
           "bf16": lambda x: round_mantissa(x, 7),
           "fp16": lambda x: f32(x).astype(np.float16).astype(np.float32)}[prec]
    return (lambda a, b: rnd(a) @ rnd(b)), f32


def truncate_mantissa(x, bits: int):
    """Keep `bits` explicit mantissa bits of float32 values (round toward 0).

    A TF32 tensor-core pass reads 32-bit operands and ignores their low 13
    mantissa bits, so the "tf32" model truncates rather than rounds."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    mask = np.uint32((0xFFFFFFFF << (23 - bits)) & 0xFFFFFFFF)
    return (x.view(np.uint32) & mask).view(np.float32).reshape(x.shape)


def precision_floor(L, eps: float, s: float, method: str, iters: int, prec: str, p: int = 4) -> float:
    """Relative Frobenius error the method reaches in arithmetic model `prec`.

    Runs the matrix-form iteration in the model and compares it with the
    float64 eigenvalue replay.  Used to derive test tolerances where the
    input's conditioning puts the stated ones beyond the arithmetic.
    """
    fn = {"ndb": ndb_inv_root, "cn": cn_inv_root, "cheb": cheb_inv_root}[method]
    if method == "ndb":
        X, _ = fn(L, eps, s, iters, prec, p)
    else:
        X, _ = fn(L, eps, s, iters, p, prec)
    return rel_fro(X, inv_root(L, eps, method, iters, s, p))


# --------------------------------------------------------------------------
# O4  Newton-DB  ([DASH] §3 Newton-DB: 3 matmuls per iteration, the first
#     iteration closed-form, inverse fourth root by chaining two calls)
# --------------------------------------------------------------------------

def ndb_matrix(Y0, iters: int, prec=None):
    """Coupled Newton iteration for (Y0^{1/2}, Y0^{-1/2}) in matrix form.

    Z_0 = I;  T_k = (3I - Z_k Y_k)/2;  Y_{k+1} = Y_k T_k;  Z_{k+1} = T_k Z_k.
    With Z_0 = I the first iteration needs only Y_0 T_0 (T_0 = (3I - Y_0)/2,
    Z_1 = T_0), so it costs 1 matmul instead of 3.
    Returns (Y, Z, number_of_matmuls).  `prec`: arithmetic model (above).
    """
    if iters < 1:
        raise ValueError("iters >= 1")
    mul, st = _model(prec)
    Y0 = st(np.asarray(Y0, dtype=np.float64))
    I = st(np.eye(Y0.shape[0]))
    T = st(0.5 * (3.0 * I - Y0))
    Y = st(mul(Y0, T))
    Z = T
    mm = 1
    for _ in range(iters - 1):
        T = st(0.5 * (3.0 * I - st(mul(Z, Y))))
        Y, Z = st(mul(Y, T)), st(mul(T, Z))
        mm += 3
    return Y, Z, mm


def ndb_calls(p: int) -> int:
    """Chained Newton-DB calls for the root power p = 2^c (reading R12)."""
    if p not in (2, 4, 8):
        raise ValueError("Newton-DB roots: p in (2, 4, 8)")
    return {2: 1, 4: 2, 8: 3}[p]


def ndb_inv_root(L, eps: float, s: float, iters: int, prec=None, p: int = 4):
    """X ~ (L + eps I)^{-1/p} by chained Newton-DB calls (reading R4).

    Call 1 on A/s gives Y ~ (A/s)^{1/2}, Z ~ (A/s)^{-1/2}; each further call
    runs on the previous Y and halves the power again: two calls give
    Z ~ (A/s)^{-1/4} (the pages' chain), three (A/s)^{-1/8}.  X = s^{-1/p} Z.
    Returns (X, matmuls).
    """
    _, st = _model(prec)
    A = np.asarray(L, dtype=np.float64) + eps * np.eye(L.shape[0])
    Y, mm = st(A / s), 0
    for _ in range(ndb_calls(p)):
        Y, Z, m = ndb_matrix(Y, iters, prec)
        mm += m
    return s ** (-1.0 / p) * np.asarray(Z, np.float64), mm


def ndb_scalar(a, iters: int):
    """The Newton-DB recurrence on scalars (the eigenvalues of Y0)."""
    a = np.asarray(a, dtype=np.float64)
    t = 0.5 * (3.0 - a)
    y, z = a * t, t
    for _ in range(iters - 1):
        t = 0.5 * (3.0 - z * y)
        y, z = y * t, t * z
    return y, z


def ndb_inv_root_replay(L, eps: float, s: float, iters: int, p: int = 4):
    """Same result as ``ndb_inv_root`` via its eigenvalues.

    Every Newton-DB iterate is a polynomial in A, so it shares A's
    eigenvectors; running the scalar recurrence on each eigenvalue gives the
    iteration's exact-arithmetic result at O(n^3) instead of O(iters n^3).
    """
    L = np.asarray(L, dtype=np.float64)
    w, Q = np.linalg.eigh(0.5 * (L + L.T))
    y = (w + eps) / s
    for _ in range(ndb_calls(p)):
        y, z = ndb_scalar(y, iters)
    return (Q * (s ** (-1.0 / p) * z)) @ Q.T


# --------------------------------------------------------------------------
# O4  Coupled Newton  ([Notes] "Roots on idle CPUs": coupled Newton, Guo and
#     Higham / Iannazzo; [DASH] §1, §5)
# --------------------------------------------------------------------------

def cn_matrix(M0, iters: int, p: int = 4, prec=None, X0=None):
    """Coupled Newton for M0^{-1/p}: X0 = I (or the given start), T =
    ((p+1)I - M)/p, X <- X T, M <- T^p M.  Returns (X, matmuls); T^p by
    binary powering (2 products for p = 4, so 4 matmuls per iteration)."""
    mul, st = _model(prec)
    M = st(np.asarray(M0, dtype=np.float64))
    I = st(np.eye(M.shape[0]))
    X = I.copy() if X0 is None else st(np.asarray(X0, dtype=np.float64))
    mm = 0
    for _ in range(iters):
        T = st(((p + 1) * I - M) / p)
        X = st(mul(X, T))
        mm += 1
        Tp, base, e = None, T, p
        while e:
            if e & 1:
                if Tp is None:
                    Tp = base
                else:
                    Tp = st(mul(Tp, base))
                    mm += 1
            e >>= 1
            if e:
                base = st(mul(base, base))
                mm += 1
        M = st(mul(Tp, M))
        mm += 1
    return X, mm


def cn_inv_root(L, eps: float, s: float, iters: int, p: int = 4, prec=None):
    """X ~ (L + eps I)^{-1/p} by coupled Newton on A/s; X = s^{-1/p} X_k."""
    _, st = _model(prec)
    A = np.asarray(L, dtype=np.float64) + eps * np.eye(L.shape[0])
    X, mm = cn_matrix(st(A / s), iters, p, prec)
    return s ** (-1.0 / p) * np.asarray(X, np.float64), mm


def cn_inv_root_warm(L, X0, eps: float, iters: int, p: int = 4):
    """(L + eps I)^{-1/p} by coupled Newton warm-started from a previous root
    X0 (reading R14): M_0 = X0^p (L + eps I), X_0 = X0, then the update of
    ``cn_matrix``; no scaling and no final multiplier.  Float64."""
    A = np.asarray(L, dtype=np.float64) + eps * np.eye(L.shape[0])
    X0 = np.asarray(X0, dtype=np.float64)
    M0 = np.linalg.matrix_power(X0, p) @ A
    X, _ = cn_matrix(M0, iters, p, X0=X0)
    return np.asarray(X, np.float64)


def cn_scalar(a, iters: int, p: int = 4):
    a = np.asarray(a, dtype=np.float64)
    m, x = a.copy(), np.ones_like(a)
    for _ in range(iters):
        t = ((p + 1) - m) / p
        x = x * t
        m = t ** p * m
    return x


def cn_inv_root_replay(L, eps: float, s: float, iters: int, p: int = 4):
    L = np.asarray(L, dtype=np.float64)
    w, Q = np.linalg.eigh(0.5 * (L + L.T))
    x = cn_scalar((w + eps) / s, iters, p)
    return (Q * (s ** (-1.0 / p) * x)) @ Q.T


# --------------------------------------------------------------------------
# O4  Chebyshev approximation  ([DASH] A.1 real case, A.2 matrix case and the
#     optimised Clenshaw recurrence with d-1 matmuls)
# --------------------------------------------------------------------------

def cheb_coefficients(degree: int, eps: float, p: int = 4):
    """Coefficients c_0..c_d of x^{-1/p} on [eps, 1+eps] in T_k(t), t in [-1, 1].

    Interpolation at the degree+1 first-kind Chebyshev nodes
    t_j = cos(pi (j + 1/2)/(d+1)), x_j = eps + (t_j + 1)/2 (reading R6):
    c_k = 2/(d+1) sum_j f(x_j) T_k(t_j), with c_0 halved so the series is
    sum_k c_k T_k(t).
    """
    N = degree + 1
    j = np.arange(N, dtype=np.float64)
    theta = math.pi * (j + 0.5) / N
    x = eps + (np.cos(theta) + 1.0) / 2.0
    f = x ** (-1.0 / p)
    c = np.empty(N)
    for k in range(N):
        c[k] = 2.0 / N * np.sum(f * np.cos(k * theta))
    c[0] *= 0.5
    return c


def clenshaw_scalar(c, t):
    """sum_k c_k T_k(t) by Clenshaw's backward recurrence ([DASH] A.1)."""
    t = np.asarray(t, dtype=np.float64)
    b1 = np.zeros_like(t)
    b2 = np.zeros_like(t)
    for k in range(len(c) - 1, 0, -1):
        b1, b2 = c[k] + 2.0 * t * b1 - b2, b1
    return c[0] + t * b1 - b2


def cheb_matrix(S, c, prec=None):
    """sum_k c_k T_k(S) by the optimised matrix Clenshaw recurrence ([DASH] A.2).

    B_d = c_d I, B_{d-1} = c_{d-1} I + 2 c_d S, B_k = c_k I + 2 S B_{k+1} - B_{k+2}
    for k = d-2 .. 1, result c_0 I + S B_1 - B_2: d-1 matmuls in all.
    Returns (P, matmuls).
    """
    mul, st = _model(prec)
    S = st(np.asarray(S, dtype=np.float64))
    I = st(np.eye(S.shape[0]))
    d = len(c) - 1
    if d == 0:
        return c[0] * I, 0
    if d == 1:
        return st(c[0] * I + c[1] * S), 0
    b2 = st(c[d] * I)                       # B_{k+2}
    b1 = st(c[d - 1] * I + 2.0 * c[d] * S)  # B_{k+1}
    mm = 0
    for k in range(d - 2, 0, -1):
        b1, b2 = st(c[k] * I + 2.0 * st(mul(S, b1)) - b2), b1
        mm += 1
    P = st(c[0] * I + st(mul(S, b1)) - b2)
    return P, mm + 1


def cheb_inv_root(L, eps: float, s: float, degree: int, p: int = 4, prec=None):
    """X = s^{-1/p} sum_k c_k T_k(2 L/s - I)  ~  (L + s eps I)^{-1/p}."""
    _, st = _model(prec)
    L = np.asarray(L, dtype=np.float64)
    S = st(2.0 * L / s - np.eye(L.shape[0]))
    P, mm = cheb_matrix(S, cheb_coefficients(degree, eps, p), prec)
    return s ** (-1.0 / p) * np.asarray(P, np.float64), mm


def cheb_inv_root_replay(L, eps: float, s: float, degree: int, p: int = 4):
    L = np.asarray(L, dtype=np.float64)
    w, Q = np.linalg.eigh(0.5 * (L + L.T))
    x = clenshaw_scalar(cheb_coefficients(degree, eps, p), 2.0 * w / s - 1.0)
    return (Q * (s ** (-1.0 / p) * x)) @ Q.T


def inv_root(L, eps: float, method: str, iters: int, scale: float, p: int = 4, replay: bool = True, prec=None):
    """Dispatch to the method (eigenvalue replay when ``replay``; the matrix
    form in arithmetic model ``prec`` when one is given)."""
    if prec is not None and method != "evd":
        fn = {"ndb": ndb_inv_root, "cn": cn_inv_root, "cheb": cheb_inv_root}[method]
        return fn(L, eps, scale, iters, prec=prec, p=p)[0] if method == "ndb" else fn(L, eps, scale, iters, p, prec)[0]
    if method == "ndb":
        return ndb_inv_root_replay(L, eps, scale, iters, p) if replay else ndb_inv_root(L, eps, scale, iters, p=p)[0]
    if method == "cn":
        return cn_inv_root_replay(L, eps, scale, iters, p) if replay else cn_inv_root(L, eps, scale, iters, p)[0]
    if method == "cheb":
        return cheb_inv_root_replay(L, eps, scale, iters, p) if replay else cheb_inv_root(L, eps, scale, iters, p)[0]
    if method == "evd":
        return inv_root_exact(L, eps, p)
    raise ValueError(method)


# --------------------------------------------------------------------------
# O5  Search direction  ([DASH] §2: two-sided preconditioning)
# --------------------------------------------------------------------------

def precondition(XL, G, XR):
    """D = L^{-1/4} G R^{-1/4} for one block."""
    return np.asarray(XL, np.float64) @ np.asarray(G, np.float64) @ np.asarray(XR, np.float64)


# --------------------------------------------------------------------------
# O6  Grafting and parameter update  ([DASH] §2 Adam grafting;
#     [3D-Shampoo] Hyperparameters graft_type / weight_decay; [Notes]
#     "Roots on idle CPUs" and "Spreading the preconditioners": grafting
#     sets each layer's step length)
# --------------------------------------------------------------------------

def graft_update(W, G, D, m, v, kind: str, lr: float, beta1: float, beta2: float,
                 eps: float, wd: float, step: int, groups=None):
    """One grafted update of one layer (reading R8).

    kind: "none" | "sgd" | "adagrad" | "adam".  The graft direction is
    SGD: G;  AdaGrad: G / (sqrt(v) + eps) with v <- v + G^2;
    Adam: m_hat / (sqrt(v_hat) + eps) with bias-corrected moments.
    rho = ||graft||_F / ||D||_F over the layer (or over each entry of
    ``groups``, a list of index tuples for blockwise grafting), and
    W <- W - lr rho D - lr wd W.  Returns (W, m, v, rho_list).
    """
    W = np.asarray(W, np.float64).copy()
    G = np.asarray(G, np.float64)
    D = np.asarray(D, np.float64)
    m = None if m is None else np.asarray(m, np.float64).copy()
    v = None if v is None else np.asarray(v, np.float64).copy()
    if kind == "none":
        graft = None
    elif kind == "sgd":
        graft = G
    elif kind == "adagrad":
        v = v + G * G
        graft = G / (np.sqrt(v) + eps)
    elif kind == "adam":
        m = beta1 * m + (1.0 - beta1) * G
        v = beta2 * v + (1.0 - beta2) * G * G
        mhat = m / (1.0 - beta1 ** step)
        vhat = v / (1.0 - beta2 ** step)
        graft = mhat / (np.sqrt(vhat) + eps)
    else:
        raise ValueError(kind)
    if groups is None:
        groups = [(slice(None), slice(None))]
    rhos = []
    upd = np.zeros_like(W)
    for sl in groups:
        if graft is None:
            rho = 1.0
        else:
            dn = math.sqrt(float(np.sum(D[sl] ** 2)))
            gn = math.sqrt(float(np.sum(graft[sl] ** 2)))
            rho = gn / dn if dn > 0 else 0.0
        upd[sl] = rho * D[sl]
        rhos.append(rho)
    W = W - lr * upd - lr * wd * W
    return W, m, v, rhos


# --------------------------------------------------------------------------
# Whole step (composition of O1..O6)
# --------------------------------------------------------------------------

class ShampooState:
    """Optimizer state of the oracle: factor stacks and graft moments."""

    def __init__(self, shapes, block_size: int, graft: str, left_only=None):
        self.shapes = [tuple(int(x) for x in s) for s in shapes]
        self.plan = plan_blocks(self.shapes, block_size, left_only=left_only)
        self.factors = [np.zeros((int(c), int(n), int(n))) for (n, c) in self.plan["f_buckets"]]
        need = graft in ("adam", "adagrad")
        self.m = [np.zeros(s) for s in self.shapes] if graft == "adam" else [None] * len(self.shapes)
        self.v = [np.zeros(s) for s in self.shapes] if need else [None] * len(self.shapes)
        self.step = 0
        self.roots = None  # the last computed inverse roots, per factor bucket


def compute_roots(state, eps, method, iters, scaling, pi_starts, pi_iters, scales_out, replay, prec,
                  evd_heuristic="corrected"):
    """Inverse fourth roots of every factor of the state (a3-a6; EVD with
    the heuristic of reading R15); inverse square roots for the factors of
    one-sided layers (reading R16)."""
    roots = [np.empty_like(f) for f in state.factors]
    for fb, stack in enumerate(state.factors):
        p = 2 if state.plan["f_sides"][fb] else 4
        for i in range(stack.shape[0]):
            Lf = stack[i]
            if method == "evd":
                s = 1.0
            elif scaling == "frobenius":
                s = frobenius_scale(Lf, 0.0 if method == "cheb" else eps)
            else:
                s = power_iteration_scale(Lf, 0.0 if method == "cheb" else eps, pi_starts, pi_iters)
            if scales_out is not None:
                scales_out[(fb, i)] = s
            if method == "evd" and evd_heuristic != "corrected":
                roots[fb][i] = evd_inv_root(Lf, eps, evd_heuristic, p)
            else:
                roots[fb][i] = inv_root(Lf, eps, method, iters, s, p=p, replay=replay, prec=prec)
    return roots


def shampoo_step(state: ShampooState, W, grads, *, beta2: float, alpha: float, eps: float,
                 method: str, iters: int, scaling: str, graft: str, lr: float,
                 beta1: float = 0.9, graft_beta2: float = 0.999, graft_eps: float = 1e-8,
                 wd: float = 0.0, pi_starts=None, pi_iters: int = 10, scales_out=None,
                 replay: bool = True, prec=None, precond_every: int = 1, evd_heuristic: str = "corrected",
                 stats_every: int = 1):
    """One optimizer step over all layers; returns the new weights.

    ``scales_out`` (optional dict) receives the per-factor scale used, keyed by
    (bucket, index), so a caller can replay with another scale.

    ``precond_every`` = f: the statistics are updated every step, the inverse
    roots only on steps 1, 1 + f, 1 + 2f, ...; the steps between reuse the
    last roots ("3D-Shampoo optimizer" README, Hyperparameters:
    preconditioning_compute_steps; DASH §1: roots every 10-100 steps).
    """
    plan = state.plan
    state.step += 1
    g_st = stack_gradients(plan, grads)
    stats_step = (state.step - 1) % max(int(stats_every), 1) == 0
    for b in (plan["blocks"] if stats_step else []):
        gb, gi, lb, lix, rb, rix = (int(x) for x in b[7:13])
        if rb < 0:  # one-sided layer: left statistics only (reading R16)
            g = np.asarray(g_st[gb][gi], dtype=np.float64)
            state.factors[lb][lix] = beta2 * state.factors[lb][lix] + alpha * (g @ g.T)
            continue
        state.factors[lb][lix], state.factors[rb][rix] = update_stats(
            g_st[gb][gi], state.factors[lb][lix], state.factors[rb][rix], beta2, alpha)
    if prec is not None:  # the arithmetic model also stores the statistics in float32
        state.factors = [f.astype(np.float32).astype(np.float64) for f in state.factors]
    if state.roots is not None and (state.step - 1) % max(int(precond_every), 1) != 0:
        roots = state.roots
    else:
        roots = compute_roots(state, eps, method, iters, scaling, pi_starts, pi_iters, scales_out, replay, prec,
                              evd_heuristic)
        state.roots = roots
    d_st = [np.empty_like(g) for g in g_st]
    for b in plan["blocks"]:
        gb, gi, lb, lix, rb, rix = (int(x) for x in b[7:13])
        if rb < 0:
            d_st[gb][gi] = np.asarray(roots[lb][lix], np.float64) @ np.asarray(g_st[gb][gi], np.float64)
            continue
        d_st[gb][gi] = precondition(roots[lb][lix], g_st[gb][gi], roots[rb][rix])
    D = unstack_directions(plan, d_st, state.shapes)
    newW = []
    for li in range(len(state.shapes)):
        w, m, v, _ = graft_update(W[li], grads[li], D[li], state.m[li], state.v[li], graft, lr,
                                  beta1, graft_beta2, graft_eps, wd, state.step)
        state.m[li], state.v[li] = m, v
        newW.append(w)
    return newW


def rel_fro(x, ref) -> float:
    """||x - ref||_F / ||ref||_F."""
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = float(np.linalg.norm(ref))
    return float(np.linalg.norm(x - ref)) / (den if den > 0 else 1.0)
