"""Split-K megakernel vs the oracle ("Event Tensor：用“事件张量”编译动态
Megakernel", §Split-K reduction 示例), through the C ABI, on the GPU.

Tolerance (fp32 sums of 32 and 128 uniform[-1,1] terms vs the fp64
oracle): |got - ref| <= 1e-5 * sum_k |A[i,k]| per row, for B and C."""
import numpy as np
import pytest

import oracle
import workloads as W
from oracle import dag

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)
import event_driven_persistent_b200 as et  # noqa: E402
from gpu_util import dev, host  # noqa: E402


def run(g, A):
    rows = A.shape[0]
    Ad = dev(A)
    nch = (A.shape[1] + 31) // 32
    Bd = torch.full((rows, nch), float("nan"), device="cuda")
    Cd = torch.full((rows,), float("nan"), device="cuda")
    et.et_run_splitk(g, Ad, rows, Bd, Cd)
    st = et.et_sync_status(g)
    return st, host(Bd), host(Cd)


def check(A, B, C):
    Bref, Cref = oracle.splitk(A, 32)
    absA = np.abs(A.astype(np.float64))
    scaleB = np.stack([absA[:, 32 * j:32 * j + 32].sum(1) for j in range(Bref.shape[1])], 1)
    assert np.all(np.abs(B - Bref) <= 1e-5 * scaleB + 1e-30)
    assert np.all(np.abs(C - Cref) <= 1e-5 * absA.sum(1) + 1e-30)
    assert np.max(np.abs(C - Cref)) / np.max(np.abs(Cref)) <= 1e-5


@pytest.mark.parametrize("sched", ["static", "dynamic", "hybrid", "unfused"])
def test_splitk_config_parity(sched):
    g = et.et_build_graph(et.ET_GRAPH_SPLITK, sched, 2048)
    try:
        A = W.splitk_inputs(2048)
        for _ in range(3):  # repeated runs on one graph (counter sets alternate)
            st, B, C = run(g, A)
            assert st == 0
            check(A, B, C)
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("fetch_batch", [1, 2, 4])
def test_splitk_batched_pops(fetch_batch):
    """The dynamic schedule with F queue slots reserved per atomic pop
    (several tasks per CTA in flight from one reservation): results, and
    dependency order with random delays."""
    g = et.et_build_graph(et.ET_GRAPH_SPLITK, "dynamic", 512, fetch_batch=fetch_batch,
                          debug_flags=et.ET_DEBUG_TRACE | et.ET_DEBUG_DELAY)
    try:
        A = W.splitk_inputs(512)
        for _ in range(2):
            st, B, C = run(g, A)
            assert st == 0
            check(A, B, C)
        graph = dag.splitk_graph(512, 128, 32, 32, "dynamic")
        errs = dag.check_trace(graph, et.et_get_trace(g))
        assert errs == [], errs[:5]
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "dynamic", "hybrid"])
@pytest.mark.parametrize("rows", [1, 31, 33, 1000, 4096])
def test_splitk_ragged_and_symbolic_rows(sched, rows):
    g = et.et_build_graph(et.ET_GRAPH_SPLITK, sched, 4096)
    try:
        A = np.random.default_rng(rows).uniform(-1, 1, (rows, 128)).astype(np.float32)
        st, B, C = run(g, A)
        assert st == 0
        check(A, B, C)
    finally:
        et.et_destroy_graph(g)


def test_splitk_ragged_columns():
    g = et.et_build_graph(et.ET_GRAPH_SPLITK, "dynamic", 256, splitk_cols=100)
    try:
        A = np.random.default_rng(5).uniform(-1, 1, (200, 100)).astype(np.float32)
        Ad = dev(A)
        Bd = torch.zeros((200, 4), device="cuda")
        Cd = torch.zeros((200,), device="cuda")
        et.et_run_splitk(g, Ad, 200, Bd, Cd)
        assert et.et_sync_status(g) == 0
        Bref, Cref = oracle.splitk(A, 32)
        assert np.allclose(host(Bd), Bref, atol=1e-4) and np.allclose(host(Cd), Cref, atol=1e-4)
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "dynamic", "hybrid", "unfused"])
@pytest.mark.parametrize("delay", [False, True])
def test_splitk_dependency_order(sched, delay):
    flags = et.ET_DEBUG_TRACE | (et.ET_DEBUG_DELAY if delay else 0)
    g = et.et_build_graph(et.ET_GRAPH_SPLITK, sched, 512, debug_flags=flags)
    try:
        A = W.splitk_inputs(512)
        st, B, C = run(g, A)
        assert st == 0
        check(A, B, C)
        graph = dag.splitk_graph(512, 128, 32, 32, sched)
        trace = et.et_get_trace(g)
        errs = dag.check_trace(graph, trace)
        assert errs == [], errs[:5]
        errs = dag.check_dataflow(dag.splitk_dataflow(512, 128, 32, 32), trace)
        assert errs == [], errs[:5]
        errs = dag.check_event_counts(graph, et.et_get_event_counts(g))
        assert errs == [], errs[:5]
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "dynamic"])
def test_splitk_wait_timeout_reports_and_recovers(sched):
    bad = et.et_build_graph(et.ET_GRAPH_SPLITK, sched, 256, debug_flags=et.ET_DEBUG_BAD_COUNT, timeout_ms=50.0)
    try:
        A = W.splitk_inputs(256)
        st, _, _ = run(bad, A)
        assert st == et.ET_ERR_TIMEOUT
        assert et.et_get_diag(bad)[0] != 0
    finally:
        et.et_destroy_graph(bad)
    good = et.et_build_graph(et.ET_GRAPH_SPLITK, sched, 256)
    try:
        st, B, C = run(good, A)
        assert st == 0
        check(A, B, C)
    finally:
        et.et_destroy_graph(good)


@pytest.mark.parametrize("sched", ["static", "dynamic"])
def test_splitk_pending_error_refuses_next_run(sched):
    """After a device error the next run is refused with ET_ERR_PENDING (the
    failing kernel mirrors its status into mapped host memory) until
    et_sync_status collects the error; then runs launch again."""
    g = et.et_build_graph(et.ET_GRAPH_SPLITK, sched, 256, debug_flags=et.ET_DEBUG_BAD_COUNT, timeout_ms=50.0)
    try:
        A = dev(W.splitk_inputs(256))
        B = torch.zeros((256, 4), device="cuda")
        C = torch.zeros((256,), device="cuda")
        et.et_run_splitk(g, A, 256, B, C)
        torch.cuda.synchronize()      # the run has ended in its timeout; the error is not collected
        with pytest.raises(et.EtError) as e:
            et.et_run_splitk(g, A, 256, B, C)
        assert e.value.status == et.ET_ERR_PENDING
        assert et.et_sync_status(g) == et.ET_ERR_TIMEOUT
        et.et_run_splitk(g, A, 256, B, C)   # launches again (and times out again: the count is still wrong)
        assert et.et_sync_status(g) == et.ET_ERR_TIMEOUT
    finally:
        et.et_destroy_graph(g)


def test_splitk_two_launch_control():
    """The kernel-per-operator control computes the same reduction."""
    for rows, cols in ((2048, 128), (77, 100)):
        A = np.random.default_rng(rows).uniform(-1, 1, (rows, cols)).astype(np.float32)
        nch = -(-cols // 32)
        Bd = torch.zeros((rows, nch), device="cuda")
        Cd = torch.zeros((rows,), device="cuda")
        et.et_run_splitk_two_launch(dev(A), rows, cols, 32, Bd, Cd)
        torch.cuda.synchronize()
        Bref, Cref = oracle.splitk(A, 32)
        scale = np.abs(A.astype(np.float64)).sum(1)
        assert np.all(np.abs(host(Cd) - Cref) <= 1e-5 * scale)
        scale_b = np.stack([np.abs(A[:, 32 * j:32 * j + 32]).astype(np.float64).sum(1) for j in range(nch)], 1)
        assert np.all(np.abs(host(Bd) - Bref) <= 1e-5 * scale_b)
