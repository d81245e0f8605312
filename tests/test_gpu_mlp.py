"""Fused decode MLP megakernel (RMSNorm -> gate/up -> SiLU*mul -> down) vs
the oracle, through the C ABI, on the GPU.

Tolerance (bf16 GEMMs with fp32 accumulation vs the fp64 oracle): max
|y - y_ref| / max |y_ref| <= 1e-2 over the output."""
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
from gpu_util import dev, empty_bf16, host, maxnorm_err  # noqa: E402

TOL = 1e-2


def run_mlp(g, d, B):
    X, gam, Wgu, Wd = dev(d["X"]), dev(d["gamma"]), dev(d["Wgu"]), dev(d["Wd"])
    Y = empty_bf16(B, d["X"].shape[1])
    et.et_run_mlp(g, B, X, gam, Wgu, Wd, Y)
    st = et.et_sync_status(g)
    return st, host(Y, np.uint16)


@pytest.mark.parametrize("sched", ["static", "dynamic", "hybrid", "unfused"])
@pytest.mark.parametrize("B", [1, 5, 16, 33])
def test_mlp_small_dims(sched, B):
    hidden, inter = 256, 512
    g = et.et_build_graph(et.ET_GRAPH_MLP, sched, 64, hidden=hidden, inter=inter)
    try:
        d = W.mlp_inputs(B, hidden=hidden, inter=inter)
        st, Y = run_mlp(g, d, B)
        assert st == 0
        ref = oracle.mlp(d["X"], d["gamma"], d["Wgu"], d["Wd"])
        assert maxnorm_err(Y, ref) <= TOL
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "dynamic"])
def test_mlp_multi_chunk_and_repeat(sched):
    hidden, inter = 512, 2048  # K chunks of 1024 for the down GEMM
    g = et.et_build_graph(et.ET_GRAPH_MLP, sched, 128, hidden=hidden, inter=inter)
    try:
        for B in (7, 128, 2):
            d = W.mlp_inputs(B, hidden=hidden, inter=inter)
            st, Y = run_mlp(g, d, B)
            assert st == 0
            assert maxnorm_err(Y, oracle.mlp(d["X"], d["gamma"], d["Wgu"], d["Wd"])) <= TOL
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "dynamic", "hybrid", "unfused"])
def test_mlp_dependency_order(sched):
    hidden, inter, B = 256, 2048, 3
    flags = et.ET_DEBUG_TRACE | et.ET_DEBUG_DELAY
    g = et.et_build_graph(et.ET_GRAPH_MLP, sched, 16, hidden=hidden, inter=inter, debug_flags=flags)
    try:
        d = W.mlp_inputs(B, hidden=hidden, inter=inter)
        st, Y = run_mlp(g, d, B)
        assert st == 0
        info = et.et_get_info(g)
        graph = dag.mlp_graph(B, hidden, inter, info["mlp_gu_tile"], info["mlp_down_tile"], info["mlp_kchunk"],
                              sched)
        trace = et.et_get_trace(g)
        errs = dag.check_trace(graph, trace)
        assert errs == [], errs[:5]
        rw = dag.mlp_dataflow(B, hidden, inter, info["mlp_gu_tile"], info["mlp_down_tile"], info["mlp_kchunk"])
        errs = dag.check_dataflow(rw, trace)
        assert errs == [], errs[:5]
        errs = dag.check_event_counts(graph, et.et_get_event_counts(g))
        assert errs == [], errs[:5]
        assert maxnorm_err(Y, oracle.mlp(d["X"], d["gamma"], d["Wgu"], d["Wd"])) <= TOL
    finally:
        et.et_destroy_graph(g)


@pytest.fixture(scope="module")
def full_mlp():
    d = W.mlp_inputs(16)
    return d, {k: dev(v) for k, v in d.items()}


@pytest.mark.parametrize("sched", ["static", "dynamic"])
@pytest.mark.parametrize("B", [1, 4, 16, 64])
def test_mlp_full_size_every_row(full_mlp, sched, B):
    """Llama-3-8B-shaped MLP (4096 -> 2x14336 -> 4096) at B in {1,4,16,64};
    the oracle evaluates every row."""
    d, t = full_mlp
    g = et.et_build_graph(et.ET_GRAPH_MLP, sched, 64)
    try:
        X = W.mlp_inputs(B, weights=False)["X"]
        Y = empty_bf16(B, 4096)
        et.et_run_mlp(g, B, dev(X), t["gamma"], t["Wgu"], t["Wd"], Y)
        assert et.et_sync_status(g) == 0
        rows = list(range(B))
        ref = oracle.mlp_rows(X, d["gamma"], d["Wgu"], d["Wd"], rows)
        assert maxnorm_err(host(Y, np.uint16)[rows], ref) <= TOL
    finally:
        et.et_destroy_graph(g)
