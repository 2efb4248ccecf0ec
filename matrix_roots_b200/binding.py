"""ctypes binding of libshampoo (include/shampoo.h), argument marshalling only.

Every function here forwards to the C entry point of the same name; torch
tensors only supply device memory (``data_ptr``) and the CUDA stream.  There
is no fallback: if the library is missing or the GPU is absent, calls raise.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libshampoo.so")

SHP_OK, SHP_ERR_INVALID_ARG, SHP_ERR_SHAPE, SHP_ERR_WORKSPACE, SHP_ERR_CUDA, SHP_ERR_UNSUPPORTED = range(6)
METHODS = {"ndb": 0, "cn": 1, "cheb": 2}
DTYPES = {"fp32": 0, "tf32": 1, "fp16": 2, "bf16": 3}
SCALINGS = {"frobenius": 0, "power": 1}
GRAFTS = {"none": 0, "sgd": 1, "adagrad": 2, "adam": 3}
BLOCK_FIELDS = 13

EXPORTS = [
    "shampoo_last_error", "shampoo_version", "shampoo_launch_count", "shampoo_device_error",
    "shampoo_plan_create", "shampoo_plan_create_ex", "shampoo_plan_destroy", "shampoo_plan_sizes",
    "shampoo_plan_tables", "shampoo_plan_factor_sides",
    "shampoo_plan_bind", "shampoo_stack_blocks",
    "shampoo_update_stats_workspace_bytes", "shampoo_update_stats",
    "shampoo_inv_root_workspace_bytes", "shampoo_inv_root", "shampoo_inv_root_static",
    "shampoo_inv_root_warm_workspace_bytes", "shampoo_inv_root_warm", "shampoo_inv_root_evd",
    "shampoo_precondition_workspace_bytes", "shampoo_precondition",
    "shampoo_graft_step_workspace_bytes", "shampoo_graft_step",
]


class ShampooError(RuntimeError):
    def __init__(self, code: int, where: str, msg: str):
        super().__init__(f"{where} failed with status {code}: {msg}")
        self.code = code


_lib = None
c_int32, c_size_t, c_float, c_void_p = ctypes.c_int32, ctypes.c_size_t, ctypes.c_float, ctypes.c_void_p
P = ctypes.POINTER


def lib() -> ctypes.CDLL:
    """Loads libshampoo.so once (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m matrix_roots_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "shampoo_last_error": (ctypes.c_char_p, []),
        "shampoo_version": (c_int32, []),
        "shampoo_launch_count": (ctypes.c_uint64, []),
        "shampoo_device_error": (c_int32, [P(c_int32)]),
        "shampoo_plan_create": (c_int32, [P(c_int32), P(c_int32), c_int32, c_int32, P(c_void_p)]),
        "shampoo_plan_create_ex": (c_int32, [P(c_int32), P(c_int32), P(c_int32), c_int32, c_int32, c_int32,
                                             P(c_void_p)]),
        "shampoo_plan_factor_sides": (c_int32, [c_void_p, P(c_int32)]),
        "shampoo_plan_destroy": (None, [c_void_p]),
        "shampoo_plan_sizes": (c_int32, [c_void_p, P(c_int32), P(c_int32), P(c_int32), P(c_size_t)]),
        "shampoo_plan_tables": (c_int32, [c_void_p, P(c_int32), P(c_int32), P(c_int32)]),
        "shampoo_plan_bind": (c_int32, [c_void_p, c_void_p, c_size_t, c_void_p]),
        "shampoo_stack_blocks": (c_int32, [c_void_p, P(c_void_p), P(c_void_p), c_void_p]),
        "shampoo_update_stats_workspace_bytes": (c_size_t, [c_void_p, c_int32]),
        "shampoo_update_stats": (c_int32, [c_void_p, P(c_void_p), P(c_void_p), c_float, c_float, c_int32,
                                           c_void_p, c_size_t, c_void_p]),
        "shampoo_inv_root_workspace_bytes": (c_size_t, [c_int32] * 6),
        "shampoo_inv_root": (c_int32, [c_void_p, c_int32, c_int32, c_float, c_int32, c_int32, c_int32, c_int32,
                                       c_int32, c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_size_t, c_void_p]),
        "shampoo_inv_root_static": (c_int32, [c_void_p, c_int32, c_int32, c_float, c_int32, c_int32, c_int32,
                                              c_int32, c_int32, c_int32, c_int32, c_void_p, c_void_p, c_void_p,
                                              c_void_p, c_void_p]),
        "shampoo_inv_root_warm_workspace_bytes": (c_size_t, [c_int32] * 3),
        "shampoo_inv_root_warm": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, c_float, c_int32, c_int32,
                                            c_int32, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
        "shampoo_inv_root_evd": (c_int32, [c_void_p, c_int32, c_int32, c_float, c_int32, c_int32, c_void_p,
                                           c_void_p, c_void_p, c_void_p]),
        "shampoo_precondition_workspace_bytes": (c_size_t, [c_void_p, c_int32]),
        "shampoo_precondition": (c_int32, [c_void_p, P(c_void_p), P(c_void_p), P(c_void_p), c_void_p, c_int32,
                                           c_void_p, c_size_t, c_void_p]),
        "shampoo_graft_step_workspace_bytes": (c_size_t, [c_void_p]),
        "shampoo_graft_step": (c_int32, [c_void_p, P(c_void_p), P(c_void_p), P(c_void_p), c_void_p, P(c_void_p),
                                         P(c_void_p), c_int32, c_float, c_float, c_float, c_float, c_float,
                                         c_int32, c_int32, c_void_p, c_size_t, c_void_p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(code: int, where: str) -> None:
    if code != SHP_OK:
        raise ShampooError(code, where, lib().shampoo_last_error().decode())


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _ptrs(ts) -> ctypes.Array:
    arr = (c_void_p * max(1, len(ts)))()
    for i, t in enumerate(ts):
        arr[i] = _ptr(t)
    return arr


def _stream(stream) -> int:
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _enum(table: dict, v) -> int:
    return table[v] if isinstance(v, str) else int(v)


def _workspace(nbytes: int, device):
    import torch
    # 256-byte alignment: torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------------------

def version() -> int:
    return int(lib().shampoo_version())


def launch_count() -> int:
    return int(lib().shampoo_launch_count())


def device_error() -> int:
    out = c_int32(0)
    _check(lib().shampoo_device_error(ctypes.byref(out)), "shampoo_device_error")
    return int(out.value)


class Plan:
    """Host block plan (shampoo_plan_create_ex) plus its bound device tables;
    ``layerwise`` stacks per layer (SHP_PLAN_LAYERWISE); ``left_only`` (one
    flag per layer, or None) makes layers one-sided."""

    def __init__(self, shapes, block_size: int, layerwise: bool = False, left_only=None):
        self.shapes = [(int(m), int(n)) for (m, n) in shapes]
        rows = (c_int32 * len(self.shapes))(*[m for m, _ in self.shapes])
        cols = (c_int32 * len(self.shapes))(*[n for _, n in self.shapes])
        lo = None
        if left_only is not None:
            if len(left_only) != len(self.shapes):
                raise ValueError("left_only needs one flag per layer")
            lo = (c_int32 * len(self.shapes))(*[1 if x else 0 for x in left_only])
        h = c_void_p()
        _check(lib().shampoo_plan_create_ex(rows, cols, lo, len(self.shapes), int(block_size), 1 if layerwise else 0,
                                            ctypes.byref(h)), "shampoo_plan_create_ex")
        self.handle = h
        nb, ng, nf, db = c_int32(), c_int32(), c_int32(), c_size_t()
        _check(lib().shampoo_plan_sizes(h, ctypes.byref(nb), ctypes.byref(ng), ctypes.byref(nf), ctypes.byref(db)),
               "shampoo_plan_sizes")
        self.n_blocks, self.n_gbuckets, self.n_fbuckets = nb.value, ng.value, nf.value
        self.device_bytes = db.value
        self.device_tables = None

    def tables(self) -> dict:
        b = np.zeros((self.n_blocks, BLOCK_FIELDS), dtype=np.int32)
        g = np.zeros((self.n_gbuckets, 3), dtype=np.int32)
        f = np.zeros((self.n_fbuckets, 2), dtype=np.int32)
        _check(lib().shampoo_plan_tables(self.handle, b.ctypes.data_as(P(c_int32)), g.ctypes.data_as(P(c_int32)),
                                         f.ctypes.data_as(P(c_int32))), "shampoo_plan_tables")
        sides = np.zeros(self.n_fbuckets, dtype=np.int32)
        _check(lib().shampoo_plan_factor_sides(self.handle, sides.ctypes.data_as(P(c_int32))),
               "shampoo_plan_factor_sides")
        return {"blocks": b, "g_buckets": g, "f_buckets": f, "f_sides": sides}

    def bind(self, device="cuda", stream=None):
        import torch
        self.device_tables = torch.empty(self.device_bytes, dtype=torch.uint8, device=device)
        _check(lib().shampoo_plan_bind(self.handle, _ptr(self.device_tables), self.device_bytes, _stream(stream)),
               "shampoo_plan_bind")
        return self

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and _lib is not None:
            _lib.shampoo_plan_destroy(h)
            self.handle = None


def stack_blocks(plan: Plan, grads, g_stacks, stream=None) -> None:
    _check(lib().shampoo_stack_blocks(plan.handle, _ptrs(grads), _ptrs(g_stacks), _stream(stream)),
           "shampoo_stack_blocks")


def update_stats_workspace_bytes(plan: Plan, dtype="fp32") -> int:
    return int(lib().shampoo_update_stats_workspace_bytes(plan.handle, _enum(DTYPES, dtype)))


def update_stats(plan: Plan, g_stacks, f_stacks, beta2: float, alpha: float = 1.0, dtype="fp32",
                 workspace=None, stream=None) -> None:
    need = update_stats_workspace_bytes(plan, dtype)
    if workspace is None:
        workspace = _workspace(need, g_stacks[0].device)
    _check(lib().shampoo_update_stats(plan.handle, _ptrs(g_stacks), _ptrs(f_stacks), float(beta2), float(alpha),
                                      _enum(DTYPES, dtype), _ptr(workspace), workspace.numel(), _stream(stream)),
           "shampoo_update_stats")


def inv_root_workspace_bytes(count: int, n: int, method="ndb", dtype="fp32", scaling="frobenius",
                             pi_vectors: int = 16) -> int:
    return int(lib().shampoo_inv_root_workspace_bytes(int(count), int(n), _enum(METHODS, method),
                                                      _enum(DTYPES, dtype), _enum(SCALINGS, scaling),
                                                      int(pi_vectors)))


def inv_root(A, eps: float, method="ndb", iters: int = 20, dtype="fp32", scaling="frobenius", p: int = 4,
             pi_vectors: int = 16, pi_iters: int = 10, pi_starts=None, out=None, scale_out=None, status_out=None,
             workspace=None, stream=None):
    """Inverse p-th roots of a (count, n, n) float32 CUDA stack; returns (X, scale, status)."""
    import torch
    count, n = int(A.shape[0]), int(A.shape[1])
    dev = A.device
    X = out if out is not None else torch.empty_like(A)
    s = scale_out if scale_out is not None else torch.empty(count, dtype=torch.float32, device=dev)
    st = status_out if status_out is not None else torch.empty(count, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = _workspace(inv_root_workspace_bytes(count, n, method, dtype, scaling, pi_vectors), dev)
    _check(lib().shampoo_inv_root(_ptr(A), count, n, float(eps), int(p), _enum(METHODS, method), int(iters),
                                  _enum(DTYPES, dtype), _enum(SCALINGS, scaling), int(pi_vectors), int(pi_iters),
                                  _ptr(pi_starts), _ptr(X), _ptr(s), _ptr(st), _ptr(workspace), workspace.numel(),
                                  _stream(stream)), "shampoo_inv_root")
    return X, s, st


def inv_root_warm_workspace_bytes(count: int, n: int, dtype="fp32") -> int:
    return int(lib().shampoo_inv_root_warm_workspace_bytes(count, n, _enum(DTYPES, dtype)))


def inv_root_warm(A, X0, eps: float, iters: int = 3, dtype="fp32", p: int = 4, out=None, status_out=None,
                  workspace=None, stream=None):
    """Coupled Newton warm-started from the previous roots X0 (same shape as
    A); returns (X, status).  ``out`` may be X0."""
    import torch
    count, n = int(A.shape[0]), int(A.shape[1])
    X = out if out is not None else torch.empty_like(A)
    st = status_out if status_out is not None else torch.empty(count, dtype=torch.int32, device=A.device)
    if workspace is None:
        workspace = _workspace(inv_root_warm_workspace_bytes(count, n, dtype), A.device)
    _check(lib().shampoo_inv_root_warm(_ptr(A), _ptr(X0), count, n, float(eps), int(p), int(iters),
                                       _enum(DTYPES, dtype), _ptr(X), _ptr(st), _ptr(workspace), workspace.numel(),
                                       _stream(stream)), "shampoo_inv_root_warm")
    return X, st


EVD_HEURISTICS = {"corrected": 0, "shifted_relu": 1, "abs_add": 2, "shmp": 3}
EVD_MAX_N = 128


def inv_root_evd(A, eps: float, heuristic="corrected", p: int = 4, out=None, eig_out=None, status_out=None,
                 want_eig: bool = False, stream=None):
    """Inverse p-th roots of a (count, n, n) float32 CUDA stack by Jacobi
    eigendecomposition with a dampening heuristic; returns (X, eigenvalues
    of L ascending or None, status).  ``out`` may be A."""
    import torch
    count, n = int(A.shape[0]), int(A.shape[1])
    X = out if out is not None else torch.empty_like(A)
    ev = eig_out if eig_out is not None else (
        torch.empty((count, n), dtype=torch.float32, device=A.device) if want_eig else None)
    st = status_out if status_out is not None else torch.empty(count, dtype=torch.int32, device=A.device)
    _check(lib().shampoo_inv_root_evd(_ptr(A), count, n, float(eps), int(p), _enum(EVD_HEURISTICS, heuristic),
                                      _ptr(X), _ptr(ev), _ptr(st), _stream(stream)), "shampoo_inv_root_evd")
    return X, ev, st


STATIC_SCRATCH_BYTES = 32 << 20


def inv_root_static(A, eps: float, method="ndb", iters: int = 20, dtype="fp32", scaling="frobenius", p: int = 4,
                    pi_vectors: int = 16, pi_iters: int = 10, pi_starts=None, out=None, scale_out=None,
                    status_out=None, stream=None):
    """shampoo_inv_root_static: same as inv_root, scratch from the library's
    fixed device array (for callers that cannot allocate); returns (X, scale, status)."""
    import torch
    count, n = int(A.shape[0]), int(A.shape[1])
    X = out if out is not None else torch.empty_like(A)
    s = scale_out if scale_out is not None else torch.empty(count, dtype=torch.float32, device=A.device)
    st = status_out if status_out is not None else torch.empty(count, dtype=torch.int32, device=A.device)
    _check(lib().shampoo_inv_root_static(_ptr(A), count, n, float(eps), int(p), _enum(METHODS, method), int(iters),
                                         _enum(DTYPES, dtype), _enum(SCALINGS, scaling), int(pi_vectors),
                                         int(pi_iters), _ptr(pi_starts), _ptr(X), _ptr(s), _ptr(st),
                                         _stream(stream)), "shampoo_inv_root_static")
    return X, s, st


def precondition_workspace_bytes(plan: Plan, dtype="fp32") -> int:
    return int(lib().shampoo_precondition_workspace_bytes(plan.handle, _enum(DTYPES, dtype)))


def precondition(plan: Plan, roots, g_stacks, d_stacks, block_dnorm2, dtype="fp32", workspace=None,
                 stream=None) -> None:
    if workspace is None:
        workspace = _workspace(precondition_workspace_bytes(plan, dtype), g_stacks[0].device)
    _check(lib().shampoo_precondition(plan.handle, _ptrs(roots), _ptrs(g_stacks), _ptrs(d_stacks),
                                      _ptr(block_dnorm2), _enum(DTYPES, dtype), _ptr(workspace), workspace.numel(),
                                      _stream(stream)), "shampoo_precondition")


def graft_step_workspace_bytes(plan: Plan) -> int:
    return int(lib().shampoo_graft_step_workspace_bytes(plan.handle))


def graft_step(plan: Plan, W, G, d_stacks, block_dnorm2, m, v, graft="adam", lr=1e-3, beta1=0.9, beta2=0.999,
               eps=1e-8, weight_decay=0.0, step=1, graft_per_block=False, workspace=None, stream=None) -> None:
    if workspace is None:
        workspace = _workspace(graft_step_workspace_bytes(plan), W[0].device)
    mm = _ptrs(m) if m is not None else None
    vv = _ptrs(v) if v is not None else None
    _check(lib().shampoo_graft_step(plan.handle, _ptrs(W), _ptrs(G) if G is not None else None, _ptrs(d_stacks),
                                    _ptr(block_dnorm2), mm, vv, _enum(GRAFTS, graft), float(lr), float(beta1),
                                    float(beta2), float(eps), float(weight_decay), int(step),
                                    int(bool(graft_per_block)), _ptr(workspace), workspace.numel(),
                                    _stream(stream)), "shampoo_graft_step")
