"""Helpers shared by the GPU parity tests (inputs, tolerances, comparisons)."""
import numpy as np

import oracle as O
from matrix_roots_b200 import workloads as W

# Relative-Frobenius tolerances.  FP32 (three fp16 passes on a scaled hi/lo
# split) and TF32 roots and the direction: 1e-3 (stated target).  FP16
# coupled Newton: 2e-2 (stated).  Where the input's conditioning makes 1e-3
# unreachable for IEEE float32 arithmetic itself, the bound is three times
# the error the same iteration reaches in float32 numpy
# (oracle.precision_floor), never below 1e-3.
TOL = {"fp32": 1e-3, "tf32": 1e-3, "fp16": 2e-2, "bf16": None}


def spd_stack(count, n, cond, seed=0):
    rng = np.random.default_rng(seed)
    q = W.haar_orthogonal(rng, n, count)
    lam = np.geomspace(1.0, 1.0 / cond, n)[None, :] * rng.uniform(0.5, 2.0, (count, 1))
    a = np.einsum("bik,bk,bjk->bij", q, lam, q)
    return (0.5 * (a + np.swapaxes(a, 1, 2))).astype(np.float32)


def to_dev(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def rel(x, ref):
    return O.rel_fro(x, ref)
