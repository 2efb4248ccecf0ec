"""Host-side helpers that need no GPU: the matrix view of N-d parameters
(DASH D: a (E, 3, 16, 16) patch embedding is preconditioned as (E, 768)),
the optimizer's one-sided layer selection and the EVD work count that
bench.py reports against the FP64 peak."""
import numpy as np
import pytest

import oracle as O
from matrix_roots_b200 import optimizer as OPT


@pytest.mark.parametrize("shape", [(384, 3, 16, 16), (512, 5, 5, 64), (7, 9), (10,), (), (4, 1, 1)])
def test_matrix_shape_matches_the_oracle_reading(shape):
    assert OPT.matrix_shape(shape) == O.matrix_shape(shape)


def test_matrix_view_is_a_view():
    import torch
    t = torch.arange(2 * 3 * 4 * 5, dtype=torch.float32).reshape(2, 3, 4, 5)
    v = OPT.matrix_view(t)
    assert v.shape == (2, 60) and v.data_ptr() == t.data_ptr()
    v[1, 7] = -1.0
    assert t.reshape(-1)[67] == -1.0
    assert OPT.matrix_view(torch.zeros(5)) is None


def test_evd_work_count():
    import bench
    # one sweep of a 4 x 4 matrix: 6 rotations, 16 * 4 flops each
    assert bench.evd_fp64_flops(4, np.array([1])) == 6 * 16 * 4
    assert bench.evd_fp64_flops(128, np.array([10, 20])) == 30 * (128 * 127 / 2) * 16 * 128


def test_root_flop_counts():
    import bench
    n = 1024
    # Newton-DB-20: two calls of 1 + 3 * 19 products; dense products
    assert bench.root_flops(n, 1, "ndb", 20, "frobenius", 16, 10) == 2 * 57 * 2.0 * n ** 3
    # Chebyshev products are symmetric: n^2 (n + 1) each, d - 1 of them
    assert bench.root_flops(n, 2, "cheb", 32, "frobenius", 16, 10) == 2 * 31 * n * n * (n + 1.0)
    assert bench.root_flops(n, 1, "cheb", 32, "frobenius", 16, 10, dense=True) == 31 * 2.0 * n ** 3


@pytest.mark.parametrize("bad", [
    dict(method="svd"), dict(dtype="fp64"), dict(scaling="spectral"), dict(graft="lion"),
    dict(evd_heuristic="relu"), dict(root_p=3), dict(block_size=-1), dict(precond_every=0),
    dict(stats_every=0), dict(iters=0), dict(eps=-1e-6), dict(eps=float("nan")),
    dict(scaling="power", pi_vectors=12), dict(method="evd", block_size=256), dict(one_sided=(5,)),
])
def test_config_check_refuses_bad_options(bad):
    cfg = OPT.ShampooConfig(**bad)
    with pytest.raises(ValueError):
        cfg.check(n_layers=3)


def test_config_check_accepts_the_workload_settings():
    OPT.ShampooConfig().check(3)
    OPT.ShampooConfig(method="cheb", iters=0).check()
    OPT.ShampooConfig(method="evd", block_size=128, evd_heuristic="shmp", one_sided=(0, 2)).check(3)
    OPT.ShampooConfig(scaling="power", pi_vectors=16, dtype="tf32", graft="adam", root_p=8).check()


def test_bench_reference_arm_json_contract():
    """bench.py --impl reference prints one JSON line with the keys the
    driver reads (on the host cores, no GPU)."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--config",
                          "tiny_dense", "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                         timeout=300, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 3 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1


@pytest.mark.parametrize("config", ["spd_stack", "evd_stack"])
def test_bench_reference_arm_for_root_only_workloads(config):
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--config", config],
                         capture_output=True, text=True, timeout=120, cwd=root)
    assert out.returncode == 0
    d = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][-1])
    assert d["impl"] == "reference" and "unavailable" in d
