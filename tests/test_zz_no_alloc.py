"""The allocation-free split-K entry point (et_run_splitk_noalloc), for
callers that cannot allocate device memory, against the graph-based
et_run_splitk on the same inputs, on two calls in a row (the second call
reuses the shared device array the first one left behind).

Tolerance, as in the split-K parity tests: per element
|got - ref| <= 1e-5 * sum_k |A[i,k]| against the fp64 oracle, and the two
entry points within that bound of each other."""
import ctypes

import numpy as np
import pytest

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)
import event_driven_persistent_b200 as et  # noqa: E402


def test_noalloc_matches_graph_entry_point_twice():
    lib = ctypes.CDLL(et.LIB_PATH)
    fn = lib.et_run_splitk_noalloc
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    stream = torch.cuda.current_stream().cuda_stream
    g = et.et_build_graph(et.ET_GRAPH_SPLITK, "static", 4096)
    try:
        for rows, seed in ((2048, 1), (1000, 7)):
            A = np.random.default_rng(seed).uniform(-1, 1, (rows, 128)).astype(np.float32)
            Ad = torch.from_numpy(A).cuda()
            B_ref = torch.zeros((rows, 4), device="cuda")
            C_ref = torch.zeros((rows,), device="cuda")
            et.et_run_splitk(g, Ad, rows, B_ref, C_ref)
            assert et.et_sync_status(g) == 0
            B_na = torch.full((rows, 4), float("nan"), device="cuda")
            C_na = torch.full((rows,), float("nan"), device="cuda")
            assert fn(Ad.data_ptr(), rows, B_na.data_ptr(), C_na.data_ptr(), stream) == 0
            scale_c = np.abs(A.astype(np.float64)).sum(1)
            _, C_o = oracle.splitk(A, 32)
            c_ref, c_na = C_ref.cpu().numpy(), C_na.cpu().numpy()
            assert np.all(np.abs(c_na - C_o) <= 1e-5 * scale_c)
            assert np.all(np.abs(c_na - c_ref) <= 1e-5 * scale_c)
            b_ref, b_na = B_ref.cpu().numpy(), B_na.cpu().numpy()
            scale_b = np.stack([np.abs(A[:, 32 * j:32 * j + 32]).astype(np.float64).sum(1) for j in range(4)], 1)
            assert np.all(np.abs(b_na - b_ref) <= 1e-5 * scale_b)
    finally:
        et.et_destroy_graph(g)
