"""Pins of the brute-force DAG expansion (event tensor = parametric task DAG)
against hand-enumerated graphs, and of the trace checker against planted
mistakes.

"Event Tensor：用“事件张量”编译动态 Megakernel": §Graph Function (maps
"ij->i" / "i->i"), §Event Tensor 的本质：参数化的 Task DAG,
§Data-dependent event update, §Data-dependent task triggering.
"""
import numpy as np

from oracle import dag


def test_splitk_two_tiles_by_hand():
    g = dag.splitk_graph(rows=64, cols=128, chunk=32, tile_rows=32, sched="static")
    P, F = dag.OP_SK_PARTIAL, dag.OP_SK_FINAL
    want_edges = {((P, i, j), (F, i, 0)) for i in range(2) for j in range(4)}
    assert g.edges == want_edges
    assert len(g.tasks) == 10
    # every event gets exactly its wait count of producers (E = ETensor((n,), wait_count=4))
    for i in range(2):
        assert len(g.event_producers[("E", i)]) == g.wait_count[("E", i)] == 4


def test_splitk_unfused_is_a_barrier():
    g = dag.splitk_graph(rows=64, cols=128, chunk=32, tile_rows=32, sched="unfused")
    assert len(g.edges) == 8 * 2  # every partial -> every final


def test_moe_tiny_by_hand():
    # T=2 tokens, k=2, E=3 experts, one token tile, one router task per token, one group, bm=1
    topk = np.array([[2, 0], [0, 1]])
    g, mtiles = dag.moe_graph(topk, E=3, tt=2, n_kc=1, tkt=1, gt=2, bm=1, n_n1=1, n_n2=1, cb=1, sched="dynamic")
    # grouping: expert 0 <- (0,1),(1,0); expert 1 <- (1,1); expert 2 <- (0,0); bm=1 -> 4 m-tiles
    assert [(e, m, rows) for (e, m, rows) in mtiles] == [
        (0, 0, [(0, 1)]), (0, 1, [(1, 0)]), (1, 0, [(1, 1)]), (2, 0, [(0, 0)])]
    R, SC, GR, S1, S2, CB = (dag.OP_MOE_ROUTER, dag.OP_MOE_SCAN, dag.OP_MOE_GROUP,
                             dag.OP_MOE_S1, dag.OP_MOE_S2, dag.OP_MOE_COMBINE)
    # one grouping tile: two router tasks (one token each), the scan groups
    want = {((R, j, 0), (SC, 0, 0)) for j in range(2)}
    want |= {((SC, 0, 0), (S1, f, 0)) for f in range(4)}
    want |= {((S1, f, 0), (S2, f, 0)) for f in range(4)}
    # combine block b = token b (cb = 1): rows of m-tile f belong to tokens 0,1,1,0
    want |= {((S2, 0, 0), (CB, 0, 0)), ((S2, 1, 0), (CB, 1, 0)), ((S2, 2, 0), (CB, 1, 0)),
             ((S2, 3, 0), (CB, 0, 0))}
    assert g.edges == want
    assert (GR, 0, 0) not in g.tasks
    # expert event counts = number of pairs routed to the expert
    assert len(g.event_producers[("E_exp", 0)]) == 2
    assert len(g.event_producers[("E_exp", 1)]) == 1
    assert len(g.event_producers[("E_exp", 2)]) == 1


def _trace_from_order(graph):
    """A valid trace: tasks in a topological order, one after another."""
    indeg = {t: 0 for t in graph.tasks}
    succ = {t: [] for t in graph.tasks}
    for p, c in graph.edges:
        indeg[c] += 1
        succ[p].append(c)
    ready = [t for t in graph.tasks if indeg[t] == 0]
    recs, tick = [], 0
    while ready:
        t = ready.pop()
        recs.append((t[0], t[1], t[2], 0, tick, tick + 1))
        tick += 2
        for c in succ[t]:
            indeg[c] -= 1
            if indeg[c] == 0:
                ready.append(c)
    return recs


def test_checker_accepts_valid_and_catches_planted_mistakes():
    g = dag.mlp_graph(B=2, hidden=256, inter=256, gu_tile=64, down_tile=128, kchunk=128, sched="static")
    recs = _trace_from_order(g)
    assert dag.check_trace(g, recs) == []
    # a consumer that starts before its producer ended
    bad = [list(r) for r in recs]
    i_red = next(i for i, r in enumerate(bad) if r[0] == dag.OP_MLP_REDUCE)
    bad[i_red][4] = -5
    assert any("edge violated" in e for e in dag.check_trace(g, bad))
    # a missing task and a duplicated task
    assert any("never ran" in e for e in dag.check_trace(g, recs[1:]))
    assert any("twice" in e for e in dag.check_trace(g, recs + recs[:1]))


def test_moe_two_tiles_by_hand():
    # T=3 tokens in tiles of 2: router -> scan -> group per tile; top-1 of 2 experts
    topk = np.array([[1], [0], [1]])
    g, mtiles = dag.moe_graph(topk, E=2, tt=2, n_kc=2, tkt=2, gt=2, bm=2, n_n1=1, n_n2=1, cb=2, sched="dynamic")
    R, SC, GR, S1, S2, CB = (dag.OP_MOE_ROUTER, dag.OP_MOE_SCAN, dag.OP_MOE_GROUP,
                             dag.OP_MOE_S1, dag.OP_MOE_S2, dag.OP_MOE_COMBINE)
    # expert 0 <- token 1 (m-tile 0); expert 1 <- tokens 0, 2 (m-tile 1)
    assert [(e, rows) for (e, m, rows) in mtiles] == [(0, [(1, 0)]), (1, [(0, 0), (2, 0)])]
    # two K chunks per router block: every chunk task precedes the scan
    want = {((R, j, c), (SC, 0, 0)) for j in range(2) for c in range(2)}
    want |= {((SC, 0, 0), (GR, q, 0)) for q in range(2)}
    # group 0 (tokens 0,1) touches experts 1 and 0; group 1 (token 2) touches expert 1
    want |= {((GR, 0, 0), (S1, 0, 0)), ((GR, 0, 0), (S1, 1, 0)), ((GR, 1, 0), (S1, 1, 0))}
    want |= {((S1, f, 0), (S2, f, 0)) for f in range(2)}
    want |= {((S2, 0, 0), (CB, 0, 0)), ((S2, 1, 0), (CB, 0, 0)), ((S2, 1, 0), (CB, 1, 0))}
    assert g.edges == want


# ------------------------------------------- wait counts and data-level order --
# §Event Tensor 的本质 (an event's wait count = the producer notifications it
# needs), §Data-dependent event update (E_exp[e] starts at the number of
# pairs routed to e).

import heapq


def _trace_priority(graph, first, last=frozenset()):
    """A valid trace of `graph` (tasks one after another, in a topological
    order) that runs the tasks in `first` as early and those in `last` as
    late as the graph allows."""
    indeg = {t: 0 for t in graph.tasks}
    succ = {t: [] for t in graph.tasks}
    for p, c in graph.edges:
        indeg[c] += 1
        succ[p].append(c)
    prio = lambda t: 0 if t in first else (2 if t in last else 1)  # noqa: E731
    heap = [(prio(t), i, t) for i, t in enumerate(graph.tasks) if indeg[t] == 0]
    heapq.heapify(heap)
    order_ix = {t: i for i, t in enumerate(graph.tasks)}
    recs, tick = [], 0
    while heap:
        _, _, t = heapq.heappop(heap)
        recs.append((t[0], t[1], t[2], 0, tick, tick + 1))
        tick += 2
        for c in succ[t]:
            indeg[c] -= 1
            if indeg[c] == 0:
                heapq.heappush(heap, (prio(c), order_ix[c], c))
    return recs


def _moe_case(T, sched, n_kc=2, tt=4, cb=2, seed=0):
    rng = np.random.default_rng(seed)
    E, k = 5, 2
    topk = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    kw = dict(E=E, tt=tt, n_kc=n_kc, tkt=2, gt=tt, bm=3, n_n1=2, n_n2=2, cb=cb)
    g, mt = dag.moe_graph(topk, sched=sched, **kw)
    rw = dag.moe_dataflow(topk, n_kc=n_kc, tkt=2, tt=tt, bm=3, n_n1=2, n_n2=2, cb=cb, E=E)
    return topk, g, mt, rw


def test_wait_counts_of_every_graph():
    for sched in ("static", "dynamic", "unfused"):
        assert dag.check_wait_counts(dag.splitk_graph(100, 128, 32, 32, sched)) == []
        assert dag.check_wait_counts(dag.mlp_graph(3, 256, 512, 64, 128, 256, sched)) == []
        for T in (3, 9):
            for n_kc in (1, 2):
                _, g, _, _ = _moe_case(T, sched, n_kc=n_kc)
                assert dag.check_wait_counts(g) == [], (T, sched, n_kc)


def test_expert_event_count_is_pairs_routed():
    topk, g, _, _ = _moe_case(9, "dynamic")
    for e in range(5):
        n = int(np.sum(topk == e))
        if n:
            assert g.wait_count[("E_exp", e)] == n


def test_event_counts_check_against_device_records():
    _, g, _, _ = _moe_case(9, "dynamic")
    names = {v: k for k, v in dag.EVENT_KIND.items()}
    recs = [(names[ev[0]], ev[1] if len(ev) > 1 else 0, n) for ev, n in g.wait_count.items()]
    recs.append((names["E_grp"], 0, 0))   # an event this schedule does not use: no notification
    assert dag.check_event_counts(g, recs) == []
    short = [r if i else (r[0], r[1], r[2] - 1) for i, r in enumerate(recs)]
    assert any("received" in e for e in dag.check_event_counts(g, short))
    stray = recs[:-1] + [(names["E_grp"], 0, 1)]   # a notification of an event the graph does not use
    assert any("E_grp" in e for e in dag.check_event_counts(g, stray))


def test_dataflow_accepts_every_event_order():
    for sched in ("static", "dynamic", "unfused"):
        for T, n_kc in ((3, 1), (9, 2)):
            _, g, _, rw = _moe_case(T, sched, n_kc=n_kc)
            for first in (set(), {t for t in g.tasks if t[0] == dag.OP_MOE_COMBINE}):
                assert dag.check_dataflow(rw, _trace_priority(g, first)) == []
    g = dag.mlp_graph(3, 256, 512, 64, 128, 256, "dynamic")
    assert dag.check_dataflow(dag.mlp_dataflow(3, 256, 512, 64, 128, 256), _trace_priority(g, set())) == []
    g = dag.splitk_graph(100, 128, 32, 32, "dynamic")
    assert dag.check_dataflow(dag.splitk_dataflow(100, 128, 32, 32), _trace_priority(g, set())) == []


def _drop(g, pred):
    g.edges = {(p, c) for (p, c) in g.edges if not pred(p, c)}
    return g


def test_dataflow_catches_a_dependency_missing_from_the_event_design():
    """Plant a missing true dependency in the event graph (as a kernel with a
    wrong event map would have it); a trace that follows the mutilated graph
    passes the event-level check but not the data-level one."""
    S1, S2, CB, R, SC = dag.OP_MOE_S1, dag.OP_MOE_S2, dag.OP_MOE_COMBINE, dag.OP_MOE_ROUTER, dag.OP_MOE_SCAN
    plants = [
        # stage 2 of m-tile 0 no longer waits for stage-1 column tile 1
        (lambda p, c: p == (S1, 0, 1) and c[0] == S2 and c[1] == 0, {(S2, 0, 0), (S2, 0, 1)}, {(S1, 0, 1)}),
        # combine block 0 no longer waits for the stage-2 tasks of m-tile 0
        (lambda p, c: p[0] == S2 and p[1] == 0 and c == (CB, 0, 0), {(CB, 0, 0)}, {(S2, 0, 0), (S2, 0, 1)}),
        # the scan no longer waits for router K chunk 1 of block 0
        (lambda p, c: p == (R, 0, 1) and c == (SC, 0, 0), {(SC, 0, 0)}, {(R, 0, 1)}),
    ]
    for pred, first, last in plants:
        topk, g, mt, rw = _moe_case(9, "dynamic", n_kc=2, tt=16, cb=4)
        # make sure the planted consumer really reads what the dropped producer writes
        g = _drop(g, pred)
        recs = _trace_priority(g, first, last)
        assert dag.check_trace(g, recs) == []
        errs = dag.check_dataflow(rw, recs)
        assert any("read before write" in e for e in errs), errs[:3]


# ----------------------------------------------------------- decode layer --
# §端到端低 batch serving (Q and K branches in parallel), §Data-dependent task
# triggering (the split count of a request follows its context length).

def _decode_case(sched, pos=(3, 9, 0)):
    kw = dict(nq=4, nkv=2, n_kc=2, split=4, n_m=2, n_gu=4, gu_tile=64, kchunk=128, n_c=2)
    g = dag.decode_graph(list(pos), sched=sched, **kw)
    rw = dag.decode_dataflow(list(pos), **kw)
    return g, rw


def test_decode_splits_follow_positions():
    g, _ = _decode_case("static", pos=(3, 9, 0))
    A = dag.OP_DEC_ATTN
    splits = sorted((t[1], t[2]) for t in g.tasks if t[0] == A)
    # request 0 (4 keys): 1 split, request 1 (10 keys): 3 splits, request 2 (1 key): 1 split; 2 KV heads
    assert splits == sorted([(0, 0), (1, 0)] + [(2, s) for s in range(3)] + [(3, s) for s in range(3)] +
                            [(4, 0), (5, 0)])
    assert g.wait_count[("D_att", 2)] == 3 and g.wait_count[("D_att", 0)] == 1
    # the Q branch of head 1 (group 0) precedes every split of group 0 only
    assert ((dag.OP_DEC_QBR, 1, 0), (A, 2, 1)) in g.edges
    assert ((dag.OP_DEC_QBR, 1, 0), (A, 3, 1)) not in g.edges


def test_decode_wait_counts_and_dataflow():
    for sched in ("static", "dynamic", "hybrid", "unfused"):
        g, rw = _decode_case(sched)
        assert dag.check_wait_counts(g) == []
        assert dag.check_dataflow(rw, _trace_priority(g, set())) == []


def test_decode_dataflow_catches_a_split_before_its_cache_append():
    """A split holding the new position read before the K branch appended
    the new key is a real violation; the event-level check misses it once
    the edge is dropped from the event graph."""
    g, rw = _decode_case("static", pos=(3, 9, 0))
    A, KBR = dag.OP_DEC_ATTN, dag.OP_DEC_KBR
    # request 1, group 0 is bg = 2; position 9 lies in split 2 (keys 8..11); K head tile of group 0 is n = 4
    g2 = _drop(g, lambda p, c: p == (KBR, 4, 0) and c == (A, 2, 2))
    recs = _trace_priority(g2, {(A, 2, 2)}, {(KBR, 4, 0)})
    assert dag.check_trace(g2, recs) == []
    assert any("read before write" in e for e in dag.check_dataflow(rw, recs))


# ------------------------------------------------------- MoE -> dense MLP --

def test_moe_mlp_graph_counts_and_dataflow():
    """The combine of block b notifies the MLP's E_norm once per token (count
    T); the MLP's gate/up tasks follow every combine."""
    for sched in ("static", "dynamic", "unfused"):
        topk = np.array([[1, 0], [0, 2], [2, 1]])
        kw = dict(E=3, tt=4, n_kc=1, tkt=2, gt=4, bm=2, n_n1=1, n_n2=1, cb=2)
        mk = dict(hidden=256, inter=256, gu_tile=64, down_tile=128, kchunk=128)
        g, _ = dag.moe_mlp_graph(topk, sched=sched, **kw, **mk)
        assert dag.check_wait_counts(g) == []
        assert g.wait_count[("E_norm",)] == 3
        for b in range(2):
            assert ((dag.OP_MOE_COMBINE, b, 0), (dag.OP_MLP_GATEUP, 0, 0)) in g.edges
        rw = dag.moe_mlp_dataflow(topk, n_kc=1, tkt=2, tt=4, bm=2, n_n1=1, n_n2=1, cb=2, E=3, **mk)
        assert dag.check_dataflow(rw, _trace_priority(g, set())) == []
        # the MLP reading a token's input before its combine wrote it is caught
        g2 = _drop(g, lambda p, c: p == (dag.OP_MOE_COMBINE, 1, 0) and c[0] == dag.OP_MLP_GATEUP)
        recs = _trace_priority(g2, {t for t in g2.tasks if t[0] == dag.OP_MLP_GATEUP}, {(dag.OP_MOE_COMBINE, 1, 0)})
        assert dag.check_trace(g2, recs) == []
        assert any("read before write" in e for e in dag.check_dataflow(rw, recs))
