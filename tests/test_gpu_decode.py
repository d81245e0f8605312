"""Decode-layer megakernel vs the oracle, through the C ABI, on the GPU.

"Event Tensor：用“事件张量”编译动态 Megakernel", §端到端低 batch serving (the
decoding pipeline: Attention, RoPE, KV-cache, Norm, MLP in one megakernel;
the Q branch and the K branch in parallel), §Data-dependent task triggering
(the attention of a request runs as a run-time number of split tasks).

Checks: Y and the attention block's output h1 within max |got - ref| /
max |ref| <= 1e-2 (bf16 outputs of bf16 GEMMs with fp32 accumulation and an
fp32 softmax against the fp64 oracle); the appended cache entries within the
same bound, every other cache entry unchanged bit for bit.
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
WKEYS = ("g1", "Wqkv", "gq", "gk", "Wo", "g2", "Wgu", "Wd")
SMALL = dict(hidden=1024, inter=512, n_heads=4, n_kv_heads=2, head_dim=128)
SMALL_IN = dict(hidden=1024, inter=512, n_q=4, n_kv=2, hd=128)


def run_decode(g, d, B, wt=None, pos=None):
    wt = wt or {k: dev(d[k]) for k in WKEYS}
    pos = d["pos"][:B] if pos is None else np.asarray(pos, np.int32)
    H = d["X"].shape[1]
    Kc, Vt = dev(d["Kc"][:B]), dev(W.v_cache_device(d["Vc"][:B]))
    Y, h1 = empty_bf16(B, H), empty_bf16(B, H)
    et.et_run_decode(g, B, dev(d["X"][:B]), dev(pos), wt, Kc, Vt, Y, h1)
    st = et.et_sync_status(g)
    return st, dict(y=host(Y, np.uint16), h1=host(h1, np.uint16), Kc=host(Kc, np.uint16),
                    Vc=W.v_cache_device(host(Vt, np.uint16)))


def check(d, out, B, n_q, n_kv, pos=None, rows=None):
    pos = d["pos"][:B] if pos is None else np.asarray(pos, np.int32)
    rows = list(range(B)) if rows is None else rows
    w = {k: d[k] for k in WKEYS}
    ref = oracle.decode_layer(d["X"][rows], pos[rows], w, d["Kc"][rows], d["Vc"][rows], n_q, n_kv)
    assert maxnorm_err(out["y"][rows], ref["y"]) <= TOL
    assert maxnorm_err(out["h1"][rows], ref["h1"]) <= TOL
    for i, b in enumerate(rows):
        p = int(pos[b])
        for name in ("Kc", "Vc"):
            got, want, before = out[name][b], ref[name][i], d[name][b]
            assert maxnorm_err(got[:, p], want[:, p]) <= TOL
            keep = np.ones(got.shape[1], bool)
            keep[p] = False
            assert np.array_equal(got[:, keep], before[:, keep])


@pytest.fixture(scope="module")
def small_inputs():
    return W.decode_inputs(40, ctx_lo=1, ctx_hi=590, max_ctx=600, **SMALL_IN)


@pytest.mark.parametrize("sched", ["static", "dynamic", "hybrid", "unfused"])
@pytest.mark.parametrize("B", [1, 5, 33])
def test_decode_small_dims(small_inputs, sched, B):
    d = small_inputs
    g = et.et_build_graph(et.ET_GRAPH_DECODE, sched, 40, max_ctx=600, **SMALL)
    try:
        st, out = run_decode(g, d, B)
        assert st == 0
        check(d, out, B, 4, 2)
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "hybrid"])
def test_decode_edge_positions(small_inputs, sched):
    """One key (position 0); the last key of a 128-key stage and the first of
    the next (127, 128); the last key of a split and a split holding only the
    new key (split - 1, split); the last cache position (599)."""
    d = small_inputs
    g = et.et_build_graph(et.ET_GRAPH_DECODE, sched, 8, max_ctx=600, **SMALL)
    try:
        sp = et.et_get_info(g)["dec_split"]
        pos = np.array([0, 127, 128, sp - 1, sp, 599], np.int32)
        assert pos.max() < 600
        st, out = run_decode(g, d, 6, pos=pos)
        assert st == 0
        check(d, out, 6, 4, 2, pos=pos)
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "hybrid"])
def test_decode_symbolic_B_repeated_runs(small_inputs, sched):
    """One graph and binary, B changing from run to run (no rebuild)."""
    d = small_inputs
    g = et.et_build_graph(et.ET_GRAPH_DECODE, sched, 40, max_ctx=600, **SMALL)
    try:
        for B in (7, 1, 40, 2):
            st, out = run_decode(g, d, B)
            assert st == 0
            check(d, out, B, 4, 2)
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched,B", [("static", 5), ("dynamic", 5), ("hybrid", 5), ("unfused", 5),
                                     ("dynamic", 12), ("hybrid", 40), ("static", 40)])
def test_decode_dependency_order(small_inputs, sched, B):
    """Trace order, data flow and event counts against the oracle's task
    graph; B = 12 and 40 run the longer queued splits (1024 and 2048 keys)."""
    d = small_inputs
    g = et.et_build_graph(et.ET_GRAPH_DECODE, sched, max(B, 8), max_ctx=600,
                          debug_flags=et.ET_DEBUG_TRACE | et.ET_DEBUG_DELAY, **SMALL)
    try:
        st, out = run_decode(g, d, B)
        assert st == 0
        info = et.et_get_info(g)
        assert info["dec_split"] == (512 if sched in ("static", "unfused") or B < 8 else (1024 if B < 32 else 2048))
        kw = dict(nq=4, nkv=2, n_kc=info["dec_qkv_kc"], split=info["dec_split"], n_m=1024 // 128,
                  n_gu=512 // info["mlp_gu_tile"], gu_tile=info["mlp_gu_tile"], kchunk=info["mlp_kchunk"],
                  n_c=512 // info["mlp_kchunk"])
        pos = d["pos"][:B]
        graph = dag.decode_graph(pos, sched=sched, **kw)
        trace = et.et_get_trace(g)
        errs = dag.check_trace(graph, trace)
        assert errs == [], errs[:5]
        errs = dag.check_dataflow(dag.decode_dataflow(pos, **kw), trace)
        assert errs == [], errs[:5]
        errs = dag.check_event_counts(graph, et.et_get_event_counts(g))
        assert errs == [], errs[:5]
        check(d, out, B, 4, 2)
    finally:
        et.et_destroy_graph(g)


def test_decode_bad_position_reports_invalid(small_inputs):
    d = small_inputs
    g = et.et_build_graph(et.ET_GRAPH_DECODE, "static", 8, max_ctx=600, timeout_ms=200.0, **SMALL)
    try:
        st, _ = run_decode(g, d, 3, pos=[5, 600, 7])
        assert st == et.ET_ERR_INVALID
        st, out = run_decode(g, d, 3)   # the graph recovers after et_sync_status
        assert st == 0
        check(d, out, 3, 4, 2)
    finally:
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "hybrid"])
def test_decode_timeout_reports(small_inputs, sched):
    d = small_inputs
    g = et.et_build_graph(et.ET_GRAPH_DECODE, sched, 8, max_ctx=600, debug_flags=et.ET_DEBUG_BAD_COUNT,
                          timeout_ms=50.0, **SMALL)
    try:
        st, _ = run_decode(g, d, 3)
        assert st == et.ET_ERR_TIMEOUT
    finally:
        et.et_destroy_graph(g)


# ------------------------------------------------------------- full size --
# Llama-3-8B-shaped layer: hidden 4096, 32 query / 8 KV heads of 128, SwiGLU
# 14336, per-request context uniform in 512..4096.

@pytest.fixture(scope="module")
def full_decode():
    d = W.decode_inputs(64)
    wt = {k: dev(d[k]) for k in WKEYS}
    graphs = {s: et.et_build_graph(et.ET_GRAPH_DECODE, s, 64) for s in ("static", "hybrid", "dynamic")}
    yield d, wt, graphs
    for g in graphs.values():
        et.et_destroy_graph(g)


@pytest.mark.parametrize("sched", ["static", "hybrid", "dynamic"])
@pytest.mark.parametrize("B", [1, 16, 37, 64])
def test_decode_full_size(full_decode, sched, B):
    d, wt, graphs = full_decode
    st, out = run_decode(graphs[sched], d, B, wt)
    assert st == 0
    check(d, out, B, 32, 8)
