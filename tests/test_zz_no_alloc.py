"""shampoo_inv_root_static: the inverse root for callers that cannot allocate.

Callers inside a CUDA graph capture, allocator callbacks, or programs with a
fixed memory budget cannot call cudaMalloc when they need a root; this entry
point takes its scratch from a fixed device array the library owns.  The
test calls it through the C ABI twice in a row (the array keeps the previous
call's contents) and compares each result with the workspace-taking
shampoo_inv_root on the same inputs, within the parity tolerance the other
root tests use (1e-3 relative Frobenius); oversize requests must be refused.
This file is collected last so that a stop-at-first-failure run has already
run every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle as O
from matrix_roots_b200 import binding as B

from gpu_util import spd_stack, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    assert torch.cuda.is_available()
    from matrix_roots_b200 import build
    build.build()
    B.lib()


@pytest.mark.parametrize("method,iters,n,count", [("ndb", 12, 128, 6), ("cn", 10, 64, 9), ("cheb", 20, 96, 5)])
def test_static_scratch_matches_workspace_call(method, iters, n, count):
    import torch
    assert B.inv_root_workspace_bytes(count, n, method, "fp32") <= B.STATIC_SCRATCH_BYTES
    ref_X, ref_s, ref_st = B.inv_root(to_dev(spd_stack(count, n, 100.0, seed=n)), 1e-4, method, iters, "fp32")
    ref_X = ref_X.cpu().numpy()
    for call in range(2):  # second call reuses the array the first one left behind
        A = to_dev(spd_stack(count, n, 100.0, seed=n))
        X = torch.full_like(A, float("nan"))
        s = torch.zeros(count, device="cuda")
        st = torch.full((count,), -1, dtype=torch.int32, device="cuda")
        L = B.lib()
        code = L.shampoo_inv_root_static(A.data_ptr(), count, n, 1e-4, 4, B.METHODS[method], iters,
                                         B.DTYPES["fp32"], B.SCALINGS["frobenius"], 16, 10, None, X.data_ptr(),
                                         s.data_ptr(), st.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert code == B.SHP_OK, L.shampoo_last_error().decode()
        torch.cuda.synchronize()
        Xh = X.cpu().numpy()
        assert np.all(st.cpu().numpy() == 0)
        assert np.allclose(s.cpu().numpy(), ref_s.cpu().numpy(), rtol=1e-6)
        for b in range(count):
            assert O.rel_fro(Xh[b], ref_X[b]) < 1e-3, (call, b)


def test_static_scratch_refuses_oversize_requests():
    L = B.lib()
    count, n = 4, 1024
    need = B.inv_root_workspace_bytes(count, n, "ndb", "fp32")
    assert need > B.STATIC_SCRATCH_BYTES
    code = L.shampoo_inv_root_static(ctypes.c_void_p(0x1000), count, n, 1e-6, 4, 0, 20, 0, 0, 16, 10, None,
                                     ctypes.c_void_p(0x2000), ctypes.c_void_p(0x3000), ctypes.c_void_p(0x4000), None)
    assert code == B.SHP_ERR_WORKSPACE
    assert "SHP_STATIC_SCRATCH_BYTES" in L.shampoo_last_error().decode()
