"""Host-side checks of the C ABI that need no GPU.

The library must load on a machine without a GPU (the CUDA runtime is linked
statically and only touches the driver on the first device call), export
every entry point include/shampoo.h declares, plan blocks exactly as the
oracle does, and reject bad arguments before enqueueing anything.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
from matrix_roots_b200 import binding as B
from matrix_roots_b200 import build as build_mod
from matrix_roots_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    build_mod.build()
    return B.lib()


def _declared():
    txt = open(os.path.join(ROOT, "include", "shampoo.h")).read()
    return sorted(set(re.findall(r"SHP_API[^;(]*?\b(shampoo_\w+)\s*\(", txt)))


def test_header_declarations_match_binding_list():
    assert _declared() == sorted(B.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(B.LIB_PATH)
    for name in _declared():
        assert hasattr(L, name), name


def test_version():
    assert B.version() >= 100


SHAPE_CASES = [
    ([(32000, 2048)], 1024),
    ([(256, 256)], 64),
    (W.transformer_shapes(), 1024),
    ([(200, 136), (64, 300), (7, 5), (1024, 1)], 128),
    ([(17, 33), (33, 17)], 0),
    ([(4096, 1024), (1024, 4096), (1000, 1000)], 512),
]


@pytest.mark.parametrize("layerwise", [False, True])
@pytest.mark.parametrize("shapes,bs", SHAPE_CASES)
def test_plan_tables_bit_exact_with_oracle(shapes, bs, layerwise):
    plan = B.Plan(shapes, bs, layerwise)
    got = plan.tables()
    ref = O.plan_blocks(shapes, bs, layerwise)
    for k in ("blocks", "g_buckets", "f_buckets", "f_sides"):
        assert got[k].dtype == np.int32
        assert np.array_equal(got[k], ref[k]), k


def test_plan_random_shapes_bit_exact():
    rng = np.random.default_rng(7)
    for _ in range(20):
        shapes = [(int(rng.integers(1, 3000)), int(rng.integers(1, 3000))) for _ in range(int(rng.integers(1, 9)))]
        bs = int(rng.choice([0, 64, 128, 500, 1024]))
        if bs == 0:
            shapes = [(min(m, 4096), min(n, 4096)) for m, n in shapes]
        lw = bool(rng.integers(0, 2))
        lo = [bool(x) for x in rng.integers(0, 2, len(shapes))] if rng.integers(0, 2) else None
        got = B.Plan(shapes, bs, lw, lo).tables()
        ref = O.plan_blocks(shapes, bs, lw, lo)
        for k in ("blocks", "g_buckets", "f_buckets", "f_sides"):
            assert np.array_equal(got[k], ref[k]), (shapes, bs, lw, lo, k)


@pytest.mark.parametrize("layerwise", [False, True])
def test_plan_one_sided_bit_exact_with_oracle(layerwise):
    shapes = W.transformer_shapes()[:6] + [(200, 136), (64, 300)]
    lo = [i % 3 == 1 for i in range(len(shapes))]
    got = B.Plan(shapes, 512, layerwise, lo).tables()
    ref = O.plan_blocks(shapes, 512, layerwise, lo)
    for k in ("blocks", "g_buckets", "f_buckets", "f_sides"):
        assert np.array_equal(got[k], ref[k]), k
    assert got["f_sides"].sum() > 0


def test_plan_unknown_flags_refused():
    L = B.lib()
    rows = (ctypes.c_int32 * 1)(64)
    cols = (ctypes.c_int32 * 1)(64)
    h = ctypes.c_void_p()
    assert L.shampoo_plan_create_ex(rows, cols, None, 1, 64, 2, ctypes.byref(h)) == B.SHP_ERR_INVALID_ARG


def test_plan_rejects_bad_input():
    with pytest.raises(B.ShampooError) as e:
        B.Plan([], 128)
    assert e.value.code == B.SHP_ERR_INVALID_ARG
    with pytest.raises(B.ShampooError) as e:
        B.Plan([(0, 5)], 128)
    assert e.value.code == B.SHP_ERR_SHAPE
    with pytest.raises(B.ShampooError) as e:
        B.Plan([(5, 5)], -1)
    assert e.value.code == B.SHP_ERR_INVALID_ARG
    with pytest.raises(B.ShampooError) as e:
        B.Plan([(10000, 16)], 0)       # whole dimension above SHP_MAX_N
    assert e.value.code == B.SHP_ERR_SHAPE


def test_workspace_queries():
    # invalid requests give 0, valid ones grow with the stack
    assert B.inv_root_workspace_bytes(4, 6, "ndb") == 0          # n % 4 != 0
    assert B.inv_root_workspace_bytes(0, 64, "ndb") == 0
    a = B.inv_root_workspace_bytes(4, 64, "ndb", "fp32")
    b = B.inv_root_workspace_bytes(8, 64, "ndb", "fp32")
    c = B.inv_root_workspace_bytes(8, 64, "ndb", "tf32")
    assert 0 < a < b and c < b
    assert B.inv_root_workspace_bytes(8, 64, "ndb", "fp32", "power", 16) > b
    plan = B.Plan([(256, 256)], 64)
    assert B.update_stats_workspace_bytes(plan, "fp32") >= 16 * 64 * 64 * 4  # fp16 hi + lo planes
    assert B.graft_step_workspace_bytes(plan) == 16 * 8


def _call_inv_root(**over):
    L = B.lib()
    args = dict(A=0x1000, count=4, n=64, eps=1e-6, p=4, method=0, iters=20, dtype=0, scaling=0, pi_vectors=16,
                pi_iters=10, pi_starts=0, X=0x2000, scale=0x3000, status=0x4000, ws=0x10000, ws_bytes=1 << 30,
                stream=0)
    args.update(over)
    return L.shampoo_inv_root(args["A"], args["count"], args["n"], args["eps"], args["p"], args["method"],
                              args["iters"], args["dtype"], args["scaling"], args["pi_vectors"], args["pi_iters"],
                              args["pi_starts"], args["X"], args["scale"], args["status"], args["ws"],
                              args["ws_bytes"], args["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(A=0), B.SHP_ERR_INVALID_ARG),
    (dict(X=0), B.SHP_ERR_INVALID_ARG),
    (dict(method=7), B.SHP_ERR_INVALID_ARG),
    (dict(dtype=9), B.SHP_ERR_INVALID_ARG),
    (dict(scaling=3), B.SHP_ERR_INVALID_ARG),
    (dict(n=6), B.SHP_ERR_SHAPE),
    (dict(n=0), B.SHP_ERR_SHAPE),
    (dict(n=16384), B.SHP_ERR_SHAPE),
    (dict(count=0), B.SHP_ERR_SHAPE),
    (dict(p=3), B.SHP_ERR_UNSUPPORTED),
    (dict(p=16), B.SHP_ERR_UNSUPPORTED),
    (dict(iters=0), B.SHP_ERR_INVALID_ARG),
    (dict(eps=float("nan")), B.SHP_ERR_INVALID_ARG),
    (dict(eps=-1.0), B.SHP_ERR_INVALID_ARG),
    (dict(scaling=1, pi_starts=0), B.SHP_ERR_INVALID_ARG),
    (dict(scaling=1, pi_starts=0x5000, pi_vectors=12), B.SHP_ERR_INVALID_ARG),
    (dict(ws=0x10001), B.SHP_ERR_INVALID_ARG),
    (dict(ws_bytes=1024), B.SHP_ERR_WORKSPACE),
])
def test_inv_root_rejects_before_enqueue(over, code):
    # pointers are never dereferenced: every case fails in the argument checks
    assert _call_inv_root(**over) == code
    assert B.lib().shampoo_last_error().decode() != ""


def test_calls_need_a_bound_plan():
    plan = B.Plan([(64, 64)], 0)
    L = B.lib()
    arr = (ctypes.c_void_p * 1)(0x1000)
    assert L.shampoo_stack_blocks(plan.handle, arr, arr, None) == B.SHP_ERR_INVALID_ARG
    assert L.shampoo_update_stats(plan.handle, arr, arr, 1.0, 1.0, 0, None, 0, None) == B.SHP_ERR_INVALID_ARG
    assert L.shampoo_precondition(plan.handle, arr, arr, arr, 0x1000, 0, None, 0, None) == B.SHP_ERR_INVALID_ARG
    assert L.shampoo_graft_step(plan.handle, arr, arr, arr, 0x1000, None, None, 1, 0.1, 0.9, 0.999, 1e-8, 0.0, 1,
                                0, None, 0, None) == B.SHP_ERR_INVALID_ARG


def _call_warm(**over):
    L = B.lib()
    args = dict(A=0x1000, X0=0x2000, count=4, n=64, eps=1e-6, p=4, iters=3, dtype=0, X=0x3000, status=0x4000,
                ws=0x10000, ws_bytes=1 << 30, stream=0)
    args.update(over)
    return L.shampoo_inv_root_warm(args["A"], args["X0"], args["count"], args["n"], args["eps"], args["p"],
                                   args["iters"], args["dtype"], args["X"], args["status"], args["ws"],
                                   args["ws_bytes"], args["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(A=0), B.SHP_ERR_INVALID_ARG),
    (dict(X0=0), B.SHP_ERR_INVALID_ARG),
    (dict(X0=0x2004), B.SHP_ERR_INVALID_ARG),
    (dict(dtype=9), B.SHP_ERR_INVALID_ARG),
    (dict(n=6), B.SHP_ERR_SHAPE),
    (dict(count=0), B.SHP_ERR_SHAPE),
    (dict(p=3), B.SHP_ERR_UNSUPPORTED),
    (dict(iters=0), B.SHP_ERR_INVALID_ARG),
    (dict(eps=-1.0), B.SHP_ERR_INVALID_ARG),
    (dict(ws_bytes=1024), B.SHP_ERR_WORKSPACE),
])
def test_inv_root_warm_rejects_before_enqueue(over, code):
    assert _call_warm(**over) == code


def test_inv_root_warm_workspace_is_the_cn_workspace():
    assert B.inv_root_warm_workspace_bytes(8, 64) == B.inv_root_workspace_bytes(8, 64, "cn", "fp32")
    assert B.inv_root_warm_workspace_bytes(8, 6) == 0


def _call_evd(**over):
    L = B.lib()
    args = dict(A=0x1000, count=4, n=64, eps=1e-6, p=4, heuristic=0, X=0x2000, eig=0, status=0x4000, stream=0)
    args.update(over)
    return L.shampoo_inv_root_evd(args["A"], args["count"], args["n"], args["eps"], args["p"], args["heuristic"],
                                  args["X"], args["eig"], args["status"], args["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(A=0), B.SHP_ERR_INVALID_ARG),
    (dict(X=0), B.SHP_ERR_INVALID_ARG),
    (dict(status=0), B.SHP_ERR_INVALID_ARG),
    (dict(heuristic=4), B.SHP_ERR_INVALID_ARG),
    (dict(heuristic=-1), B.SHP_ERR_INVALID_ARG),
    (dict(eps=float("inf")), B.SHP_ERR_INVALID_ARG),
    (dict(n=0), B.SHP_ERR_SHAPE),
    (dict(n=129), B.SHP_ERR_SHAPE),
    (dict(count=0), B.SHP_ERR_SHAPE),
    (dict(p=3), B.SHP_ERR_UNSUPPORTED),
])
def test_inv_root_evd_rejects_before_enqueue(over, code):
    assert _call_evd(**over) == code


def test_header_is_plain_c(tmp_path):
    """The boundary is a C ABI: the header compiles as C99 with every
    warning on, and a C program links against the library's symbols."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text('#include "shampoo.h"\n'
                   'int main(void) {\n'
                   '  shp_plan* p = 0;\n'
                   '  int32_t r = 64, c = 32;\n'
                   '  if (shampoo_plan_create(&r, &c, 1, 0, &p) != SHP_OK) return 1;\n'
                   '  shampoo_plan_destroy(p);\n'
                   '  return shampoo_version() > 0 ? 0 : 2;\n'
                   '}\n')
    exe = tmp_path / "use"
    lib_dir = os.path.dirname(B.LIB_PATH)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", lib_dir, "-l:" + os.path.basename(B.LIB_PATH),
                    "-Wl,-rpath," + lib_dir], check=True)
    assert subprocess.run([str(exe)]).returncode == 0
