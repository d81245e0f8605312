"""MoE layer megakernel vs the oracle, through the C ABI, on the GPU.

"Event Tensor：用“事件张量”编译动态 Megakernel", §Data-dependent event
update, §Data-dependent task triggering, §完整 MoE layer.

Checks (the tolerances are the ones the method's acceptance fixes):
  * router logits: |l - l_ref| <= 1e-5 * (sum_k |x_k Wr_ek| + |bias_e|), the
    error scale of an fp32-accumulated dot product (the device accumulates
    bf16 products in fp32 on the tensor cores, the oracle in fp64);
  * top-k indices, pair CSR (indptr) and permutation: bit-exact against the
    oracle evaluated on the device's own logits (the floating-point
    decision is then taken on identical fp32 values);
  * routing weights: relative 1e-5 against the oracle's softmax of the same
    logits;
  * the oracle's own end-to-end top-k agrees except on tokens whose k-th
    and (k+1)-th logits are closer than twice the logit error bound;
  * Y: max |y - y_ref| / max |y_ref| <= 1e-2 (bf16 GEMMs, fp32 accumulate).
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

TOL_Y = 1e-2


def run_moe(g, d, T, k, E, t=None):
    t = t or {n: dev(d[n]) for n in ("Wr", "bias", "W1", "W2")}
    X = dev(d["X"][:T])
    H = d["X"].shape[1]
    Y = empty_bf16(T, H)
    tk = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    tw = torch.zeros((T, k), dtype=torch.float32, device="cuda")
    ip = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
    pm = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
    lg = torch.zeros((T, E), dtype=torch.float32, device="cuda")
    et.et_run_moe(g, T, X, t["Wr"], t["bias"], t["W1"], t["W2"], Y, tk, tw, ip, pm, lg)
    st = et.et_sync_status(g)
    return st, dict(y=host(Y, np.uint16), topk=host(tk), w=host(tw), indptr=host(ip), perm=host(pm),
                    logits=host(lg))


def check_routing(d, out, k, E, T):
    X = d["X"][:T]
    xf = W.bf16_bits_to_f32(X).astype(np.float64)
    wf = W.bf16_bits_to_f32(d["Wr"]).astype(np.float64)
    scale = np.abs(xf) @ np.abs(wf).T + np.abs(d["bias"]).astype(np.float64)
    ref_l = oracle.router_logits(X, d["Wr"], d["bias"])
    bound = 1e-5 * scale
    assert np.all(np.abs(out["logits"] - ref_l) <= bound)
    # bit-exact integer decisions on the device's own logits
    tk_o, w_o = oracle.topk_softmax(out["logits"], k)
    assert np.array_equal(out["topk"], tk_o)
    assert np.all(np.abs(out["w"] - w_o) <= 1e-5 * np.abs(w_o))
    grp = oracle.group(out["topk"], E, 128)
    assert np.array_equal(out["indptr"], grp["indptr"])
    assert np.array_equal(out["perm"], grp["perm"])
    # end to end: the oracle's own selection differs only at near-ties
    tk_ref, _ = oracle.topk_softmax(ref_l, k)
    for t in np.nonzero(np.any(np.sort(tk_ref, 1) != np.sort(out["topk"], 1), axis=1))[0]:
        srt = np.sort(ref_l[t])[::-1]
        assert srt[k - 1] - srt[k] <= 2 * bound[t].max(), "token %d: routing differs beyond a near-tie" % t
    return w_o, grp


SMALL = dict(hidden=256, inter=128, n_experts=16, top_k=4)


@pytest.fixture(scope="module")
def small_inputs():
    return W.moe_inputs(300, hidden=256, inter=128, E=16, zipf_s=0.8)


@pytest.mark.parametrize("sched", ["static", "dynamic", "hybrid", "unfused"])
@pytest.mark.parametrize("T", [1, 5, 37, 300])
def test_moe_small_dims(small_inputs, sched, T):
    d = small_inputs
    g = et.et_build_graph(et.ET_GRAPH_MOE, sched, 512, **SMALL)
    try:
        st, out = run_moe(g, d, T, 4, 16)
        assert st == 0
        w_o, grp = check_routing(d, out, 4, 16, T)
        y_ref = oracle.moe_grouped(d["X"][:T], d["W1"], d["W2"], out["topk"], w_o, grp["indptr"], grp["perm"])
        assert maxnorm_err(out["y"], y_ref) <= TOL_Y
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "dynamic", "hybrid"])
@pytest.mark.parametrize("T", [1, 21, 150])
def test_moe_e24_top8(sched, T):
    """E = 24 (the last 16-expert group of a router thread holds 8 experts),
    every one of the 8 slots taken, a ragged last router task."""
    E, k = 24, 8
    d = W.moe_inputs(T, hidden=256, inter=128, E=E, zipf_s=1.5)
    g = et.et_build_graph(et.ET_GRAPH_MOE, sched, 256, hidden=256, inter=128, n_experts=E, top_k=k)
    try:
        st, out = run_moe(g, d, T, k, E)
        assert st == 0
        w_o, grp = check_routing(d, out, k, E, T)
        y_ref = oracle.moe_grouped(d["X"][:T], d["W1"], d["W2"], out["topk"], w_o, grp["indptr"], grp["perm"])
        assert maxnorm_err(out["y"], y_ref) <= TOL_Y
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "dynamic", "hybrid"])
def test_moe_symbolic_T_repeated_runs(small_inputs, sched):
    """One graph, one binary, T changing from run to run (no rebuild)."""
    d = small_inputs
    g = et.et_build_graph(et.ET_GRAPH_MOE, sched, 512, **SMALL)
    try:
        for T in (300, 1, 64, 129, 2, 300):
            st, out = run_moe(g, d, T, 4, 16)
            assert st == 0
            w_o, grp = check_routing(d, out, 4, 16, T)
            y_ref = oracle.moe_grouped(d["X"][:T], d["W1"], d["W2"], out["topk"], w_o, grp["indptr"], grp["perm"])
            assert maxnorm_err(out["y"], y_ref) <= TOL_Y
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "dynamic", "hybrid", "unfused"])
@pytest.mark.parametrize("T", [3, 200])
def test_moe_dependency_order(small_inputs, sched, T):
    d = small_inputs
    g = et.et_build_graph(et.ET_GRAPH_MOE, sched, 256, debug_flags=et.ET_DEBUG_TRACE | et.ET_DEBUG_DELAY,
                          **SMALL)
    try:
        st, out = run_moe(g, d, T, 4, 16)
        assert st == 0
        info = et.et_get_info(g)
        # the router split of a run is fixed by its size bucket; read it from the trace
        trace = et.et_get_trace(g)
        rt = [r for r in trace if r[0] == dag.OP_MOE_ROUTER]
        n_kc = max(r[2] for r in rt) + 1
        n_n1, n_n2 = 128 // info["moe_n1_tile"], 256 // info["moe_n2_tile"]
        graph, _ = dag.moe_graph(out["topk"], 16, info["moe_tt"], n_kc, info["moe_tkt"], info["moe_gt"], info["moe_bm"],
                                 n_n1, n_n2, info["moe_cb"], sched)
        errs = dag.check_trace(graph, trace)
        assert errs == [], errs[:5]
        rw = dag.moe_dataflow(out["topk"], n_kc, info["moe_tkt"], info["moe_tt"], info["moe_bm"], n_n1, n_n2,
                              info["moe_cb"], 16)
        errs = dag.check_dataflow(rw, trace)
        assert errs == [], errs[:5]
        errs = dag.check_event_counts(graph, et.et_get_event_counts(g))
        assert errs == [], errs[:5]
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "dynamic", "hybrid"])
@pytest.mark.parametrize("T", [150, 300])
def test_moe_staged_rows(small_inputs, sched, T):
    """Stage-1 token rows staged once in grouped order by the grouping tasks
    (moe_xp_min_T lowered so that small dims take that path): Y against the
    grouped oracle, and dependency order and event counts as above."""
    d = small_inputs
    g = et.et_build_graph(et.ET_GRAPH_MOE, sched, 512, debug_flags=et.ET_DEBUG_TRACE | et.ET_DEBUG_DELAY,
                          moe_xp_min_T=129, **SMALL)
    try:
        st, out = run_moe(g, d, T, 4, 16)
        assert st == 0
        w_o, grp = check_routing(d, out, 4, 16, T)
        y_ref = oracle.moe_grouped(d["X"][:T], d["W1"], d["W2"], out["topk"], w_o, grp["indptr"], grp["perm"])
        assert maxnorm_err(out["y"], y_ref) <= TOL_Y
        info = et.et_get_info(g)
        trace = et.et_get_trace(g)
        n_kc = max(r[2] for r in trace if r[0] == dag.OP_MOE_ROUTER) + 1
        n_n1, n_n2 = 128 // info["moe_n1_tile"], 256 // info["moe_n2_tile"]
        counts = et.et_get_event_counts(g)
        n_cb = sum(1 for kind, _, _ in counts if kind == 26)  # the run's combine blocks (size bucket)
        cb = 1 if n_cb == T else -(-T // n_cb)
        graph, _ = dag.moe_graph(out["topk"], 16, info["moe_tt"], n_kc, info["moe_tkt"], info["moe_gt"], info["moe_bm"],
                                 n_n1, n_n2, cb, sched)
        errs = dag.check_trace(graph, trace)
        assert errs == [], errs[:5]
        rw = dag.moe_dataflow(out["topk"], n_kc, info["moe_tkt"], info["moe_tt"], info["moe_bm"], n_n1, n_n2,
                              cb, 16)
        errs = dag.check_dataflow(rw, trace)
        assert errs == [], errs[:5]
        errs = dag.check_event_counts(graph, counts)
        assert errs == [], errs[:5]
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "dynamic"])
def test_moe_timeout_reports(small_inputs, sched):
    d = small_inputs
    g = et.et_build_graph(et.ET_GRAPH_MOE, sched, 64, debug_flags=et.ET_DEBUG_BAD_COUNT, timeout_ms=50.0, **SMALL)
    try:
        st, _ = run_moe(g, d, 10, 4, 16)
        assert st == et.ET_ERR_TIMEOUT
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "dynamic"])
def test_moe_pending_error_refuses_next_run(small_inputs, sched):
    """A device error (a wait count one too high, 50 ms limit) makes the next
    et_run_moe return ET_ERR_PENDING without launching, until et_sync_status
    collects the error."""
    d = small_inputs
    g = et.et_build_graph(et.ET_GRAPH_MOE, sched, 64, debug_flags=et.ET_DEBUG_BAD_COUNT, timeout_ms=50.0, **SMALL)
    try:
        t = {n: dev(d[n]) for n in ("Wr", "bias", "W1", "W2")}
        X = dev(d["X"][:10])
        Y = empty_bf16(10, 256)
        et.et_run_moe(g, 10, X, t["Wr"], t["bias"], t["W1"], t["W2"], Y)
        torch.cuda.synchronize()
        with pytest.raises(et.EtError) as e:
            et.et_run_moe(g, 10, X, t["Wr"], t["bias"], t["W1"], t["W2"], Y)
        assert e.value.status == et.ET_ERR_PENDING
        assert et.et_sync_status(g) == et.ET_ERR_TIMEOUT
    finally:
        et.et_destroy_graph(g)


# ------------------------------------------------------------- full size --
# Qwen3-30B-A3B-shaped layer (hidden 2048 -> 128 experts x SwiGLU 768, top-8,
# Zipf(s) expert bias), every size the benchmark times, both schedules.

FULL_T = [1, 16, 128, 256, 1024, 4096]
FULL_S = [0.0, 1.2, 1.5]


@pytest.fixture(scope="module")
def full_moe():
    d = W.moe_inputs(1, zipf_s=1.2)
    t = {n: dev(d[n]) for n in ("Wr", "W1", "W2")}
    g = {s: et.et_build_graph(et.ET_GRAPH_MOE, s, 4096) for s in ("static", "dynamic", "hybrid")}
    cache = {}
    yield d, t, g, cache
    for h in g.values():
        et.et_destroy_graph(h)


def _sample_tokens(T, topk, k, E, seed):
    """Every token up to 256; beyond, one routed pair of every m-tile
    (128 grouped rows of one expert) plus the first and last token."""
    if T <= 256:
        return list(range(T))
    grp = oracle.group(topk, E, 128)
    rng = np.random.default_rng(seed)
    toks = {0, T - 1}
    for e in range(E):
        for r0 in range(grp["indptr"][e], grp["indptr"][e + 1], 128):
            r1 = min(r0 + 128, grp["indptr"][e + 1])
            toks.add(int(grp["perm"][rng.integers(r0, r1)]) // k)
    return sorted(toks)


FULL_CASES = [(T, z, s) for T in FULL_T for z in FULL_S for s in ("static", "dynamic")] + \
    [(T, 1.2, "hybrid") for T in (1, 128, 4096)]


@pytest.mark.parametrize("T,zipf,sched", FULL_CASES)
def test_moe_full_size(full_moe, sched, zipf, T):
    """Routing bit-exact for every token (on the device's logits), event
    counts equal to the expansion's wait counts, and Y against the oracle's
    per-token evaluation with the device's routing: every token up to
    T = 256, a token of every m-tile beyond."""
    d, t, graphs, cache = full_moe
    E, k = 128, 8
    dT = dict(d)
    dT["X"] = W.moe_inputs(T, weights=False)["X"]
    dT["bias"] = W.expert_bias(E, zipf)
    tt = dict(t)
    tt["bias"] = dev(dT["bias"])
    g = graphs[sched]
    st, out = run_moe(g, dT, T, k, E, tt)
    assert st == 0
    w_o, grp = check_routing(dT, out, k, E, T)
    # every event received its wait count (data-dependent ones from this routing)
    counts = et.et_get_event_counts(g)
    n_kc = max([c for kind, _, c in counts if kind == 20] + [1])
    n_cb = sum(1 for kind, _, _ in counts if kind == 26)
    cb = 1 if n_cb == T else -(-T // n_cb)
    info = et.et_get_info(g)
    graph, _ = dag.moe_graph(out["topk"], E, info["moe_tt"], n_kc, info["moe_tkt"], info["moe_gt"], info["moe_bm"],
                             768 // info["moe_n1_tile"], 2048 // info["moe_n2_tile"], cb, sched)
    errs = dag.check_event_counts(graph, counts)
    assert errs == [], errs[:5]
    toks = _sample_tokens(T, out["topk"], k, E, seed=T)
    need = [i for i in toks if (zipf, T, i, out["topk"][i].tobytes(), w_o[i].tobytes()) not in cache]
    if need:
        ref = oracle.moe_rows_given_routing(dT["X"], d["W1"], d["W2"], need, out["topk"][need], w_o[need])
        for i, row in zip(need, ref):
            cache[(zipf, T, i, out["topk"][i].tobytes(), w_o[i].tobytes())] = row
    y_ref = np.stack([cache[(zipf, T, i, out["topk"][i].tobytes(), w_o[i].tobytes())] for i in toks])
    assert maxnorm_err(out["y"][toks], y_ref) <= TOL_Y


@pytest.mark.parametrize("flags", ["trace", "trace+cta"])
def test_cta_timing_records(small_inputs, flags):
    """ET_DEBUG_CTA_TIMES adds one record per CTA (op ET_OP_CTA, a = CTA
    index) with entry <= set-up done <= exit, and only together with
    ET_DEBUG_TRACE; the task records are unchanged."""
    d = small_inputs
    dbg = et.ET_DEBUG_TRACE | (et.ET_DEBUG_CTA_TIMES if flags == "trace+cta" else 0)
    g = et.et_build_graph(et.ET_GRAPH_MOE, "dynamic", 64, debug_flags=dbg, **SMALL)
    try:
        st, _ = run_moe(g, d, 21, 4, 16)
        assert st == 0
        tr = et.et_get_trace(g)
        cta = [r for r in tr if r[0] == 60]
        tasks = [r for r in tr if r[0] != 60]
        assert tasks, "no task records"
        if flags == "trace":
            assert cta == []
            return
        n = et.et_get_info(g)["n_ctas"]
        assert sorted(r[1] for r in cta) == list(range(n))
        for r in cta:  # (op, a, b, sm, start, end, t_fetch, t_ready, t_acc, t_end)
            assert r[6] <= r[7] <= r[9]
        assert min(r[6] for r in cta) <= min(r[6] for r in tasks)
        assert max(r[9] for r in cta) >= max(r[9] for r in tasks)
    finally:
        et.et_destroy_graph(g)
