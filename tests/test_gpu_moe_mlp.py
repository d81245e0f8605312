"""MoE layer -> dense MLP megakernel vs the oracle, through the C ABI.

"Event Tensor：用“事件张量”编译动态 Megakernel", §端到端低 batch serving: the MoE
GroupGEMM and the dense MLP GEMM pipelined across stages in one megakernel.

Checks (the graph exports no routing; the MoE-only graph's tests check it
bit for bit): Y1 (the MoE output) against the oracle's per-token evaluation
on every token whose k-th and (k+1)-th logits are more than 1e-3 apart (the
device's selection is then the oracle's), and Y2 against the oracle's MLP of
the device's Y1 on every token, both within max |got - ref| / max |ref| <=
1e-2; event counts equal to the expansion's wait counts; dependency order by
ticket (event level and data level).
"""
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
SMALL = dict(hidden=256, inter=128, n_experts=16, top_k=4, mlp_inter=512)


def run(g, d, m, T, t=None):
    t = t or {n: dev(v) for n, v in list(d.items()) + list(m.items()) if n != "X"}
    H = d["X"].shape[1]
    Y1, Y2 = empty_bf16(T, H), empty_bf16(T, H)
    et.et_run_moe_mlp(g, T, dev(d["X"][:T]), t["Wr"], t["bias"], t["W1"], t["W2"], t["gamma"], t["Wgu"], t["Wd"],
                      Y1, Y2)
    st = et.et_sync_status(g)
    return st, host(Y1, np.uint16), host(Y2, np.uint16)


def check(d, m, T, k, y1, y2):
    X = d["X"][:T]
    tk, w = oracle.topk_softmax(oracle.router_logits(X, d["Wr"], d["bias"]), k)
    rows = list(range(T))
    ref1 = oracle.moe_rows_given_routing(X, d["W1"], d["W2"], rows, tk, w)
    # the device may pick another expert at a near-tie of the logits: compare
    # Y1 where the oracle's selection is unambiguous, Y2 on the device's Y1
    lg = oracle.router_logits(X, d["Wr"], d["bias"])
    srt = np.sort(lg, 1)[:, ::-1]
    clear = [t for t in rows if srt[t, k - 1] - srt[t, k] > 1e-3]
    assert maxnorm_err(y1[clear], ref1[clear]) <= TOL
    ref2 = oracle.mlp_rows(y1, m["gamma"], m["Wgu"], m["Wd"], rows)
    assert maxnorm_err(y2, ref2) <= TOL


@pytest.fixture(scope="module")
def small():
    return (W.moe_inputs(128, hidden=256, inter=128, E=16, zipf_s=0.8),
            W.dense_mlp_weights(hidden=256, inter=512))


@pytest.mark.parametrize("sched", ["static", "dynamic", "hybrid", "unfused"])
@pytest.mark.parametrize("T", [1, 37, 128])
def test_moe_mlp_small_dims(small, sched, T):
    d, m = small
    g = et.et_build_graph(et.ET_GRAPH_MOE_MLP, sched, 128, **SMALL)
    try:
        st, y1, y2 = run(g, d, m, T)
        assert st == 0
        check(d, m, T, 4, y1, y2)
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "dynamic", "hybrid", "unfused"])
def test_moe_mlp_dependency_order(small, sched):
    d, m = small
    T = 21
    g = et.et_build_graph(et.ET_GRAPH_MOE_MLP, sched, 64, debug_flags=et.ET_DEBUG_TRACE | et.ET_DEBUG_DELAY, **SMALL)
    try:
        st, y1, y2 = run(g, d, m, T)
        assert st == 0
        info = et.et_get_info(g)
        trace = et.et_get_trace(g)
        n_kc = max(r[2] for r in trace if r[0] == dag.OP_MOE_ROUTER) + 1
        counts = et.et_get_event_counts(g)
        n_cb = sum(1 for kind, _, _ in counts if kind == 26)
        cb = 1 if n_cb == T else -(-T // n_cb)
        # the expansion needs the run's routing: this graph does not export it, so
        # take the oracle's, on an input where every token's k-th and (k+1)-th
        # logits are well apart (the device's selection is then the same)
        lg = oracle.router_logits(d["X"][:T], d["Wr"], d["bias"])
        tk, _ = oracle.topk_softmax(lg, 4)
        srt = np.sort(lg, 1)[:, ::-1]
        assert np.all(srt[:, 3] - srt[:, 4] > 1e-3), "a near-tie in the routing of this seeded input"
        kw = dict(tt=info["moe_tt"], n_kc=n_kc, tkt=info["moe_tkt"], bm=info["moe_bm"],
                  n_n1=128 // info["moe_n1_tile"], n_n2=256 // info["moe_n2_tile"], cb=cb)
        mk = dict(hidden=256, inter=512, gu_tile=info["mlp_gu_tile"], down_tile=info["mlp_down_tile"],
                  kchunk=info["mlp_kchunk"])
        graph, _ = dag.moe_mlp_graph(tk, 16, gt=info["moe_gt"], sched=sched, **kw, **mk)
        errs = dag.check_trace(graph, trace)
        assert errs == [], errs[:5]
        errs = dag.check_dataflow(dag.moe_mlp_dataflow(tk, E=16, **kw, **mk), trace)
        assert errs == [], errs[:5]
        errs = dag.check_event_counts(graph, counts)
        assert errs == [], errs[:5]
        check(d, m, T, 4, y1, y2)
    finally:
        et.et_destroy_graph(g)


@pytest.fixture(scope="module")
def full():
    d = W.moe_inputs(1, zipf_s=1.2)
    m = W.dense_mlp_weights()
    t = {n: dev(v) for n, v in list(d.items()) + list(m.items()) if n != "X"}
    g = {s: et.et_build_graph(et.ET_GRAPH_MOE_MLP, s, 128) for s in ("static", "dynamic", "hybrid")}
    yield d, m, t, g
    for h in g.values():
        et.et_destroy_graph(h)


@pytest.mark.parametrize("sched", ["static", "dynamic", "hybrid"])
@pytest.mark.parametrize("T", [1, 16, 128])
def test_moe_mlp_full_size(full, sched, T):
    """Qwen3-30B-A3B-shaped MoE layer then its dense MLP shape (2048 -> 6144
    -> 2048), every token."""
    d, m, t, g = full
    dT = dict(d)
    dT["X"] = W.moe_inputs(T, weights=False)["X"]
    st, y1, y2 = run(g[sched], dT, m, T, t)
    assert st == 0
    check(dT, m, T, 8, y1, y2)
