"""Brute-force expansion of event-tensor task graphs, and an order checker.

TEST INFRASTRUCTURE ONLY.  An event tensor is a compact, parametric form of
a task DAG: ``producer task -> event -> consumer task`` given by an event
shape, a wait count and einsum-like coordinate maps ("Event Tensor：用
“事件张量”编译动态 Megakernel", §Event Tensor 的本质：参数化的 Task DAG).
Here the DAG is written out in full, task by task and edge by edge, from
those maps and from the runtime tensors (topk) that data-dependent maps
read (§Data-dependent event update, §Data-dependent task triggering), so
that a device execution trace can be checked against it:

* every task of the graph ran exactly once, and nothing else ran;
* for every edge p -> c, p finished before c started (tickets from one
  global counter, taken by c after its wait and by p before its notify);
* every event received exactly its wait count of notifications.

Tasks are tuples ``(op, a, b)``; the op names and coordinates follow the
trace record format of the device library (see ``include/et.h``).
"""
from collections import defaultdict

import numpy as np

# op codes of trace records (an interface: the same numbers are declared in
# include/et.h, where the record format is defined)
OP_SK_PARTIAL, OP_SK_FINAL = 1, 2
OP_MLP_NORM, OP_MLP_GATEUP, OP_MLP_DOWN, OP_MLP_REDUCE = 10, 11, 12, 13
OP_MOE_ROUTER, OP_MOE_SCAN, OP_MOE_GROUP, OP_MOE_S1, OP_MOE_S2, OP_MOE_COMBINE = (
    20, 22, 23, 24, 25, 26)


def _cdiv(a, b):
    return (a + b - 1) // b


class Graph:
    """Explicit DAG: tasks, edges, and per-event producer lists."""

    def __init__(self):
        self.tasks = []
        self.edges = set()
        self.event_producers = defaultdict(list)   # event -> producer tasks
        self.event_consumers = defaultdict(list)   # event -> consumer tasks
        self.wait_count = {}                        # event -> declared wait count

    def add_task(self, t):
        self.tasks.append(t)

    def produce(self, task, event):
        self.event_producers[event].append(task)

    def consume(self, task, event):
        self.event_consumers[event].append(task)

    def finish(self):
        """Edges = every producer of an event -> every consumer of it."""
        for ev, cons in self.event_consumers.items():
            for p in self.event_producers.get(ev, []):
                for c in cons:
                    self.edges.add((p, c))
        return self


def splitk_graph(rows, cols, chunk, tile_rows, sched):
    """Split-K: producer (i, j) --"ij->i"--> E[i] --"i->i"--> consumer i.
    The unfused control replaces E by one event that every partial notifies
    and every final waits on."""
    g = Graph()
    n = _cdiv(rows, tile_rows)
    J = _cdiv(cols, chunk)
    for i in range(n):
        for j in range(J):
            t = (OP_SK_PARTIAL, i, j)
            g.add_task(t)
            g.produce(t, ("E", i) if sched != "unfused" else ("Eall",))
    for i in range(n):
        t = (OP_SK_FINAL, i, 0)
        g.add_task(t)
        g.consume(t, ("E", i) if sched != "unfused" else ("Eall",))
    for i in range(n):
        g.wait_count[("E", i)] = J
    g.wait_count[("Eall",)] = n * J
    return g.finish()


def mlp_graph(B, hidden, inter, gu_tile, down_tile, kchunk, sched):
    """Decode MLP: norm rows -> gate/up tiles -> down (tile, K-chunk) -> reduce.
      norm b        --"b->"-->   E_norm            (count B)
      E_norm        --"->n"-->   gate/up n
      gate/up n     --"n->c"-->  E_h[c], c = n*gu_tile // kchunk
      E_h[c]        --"mc->c"--> down (m, c)
      down (m, c)   --"mc->m"--> E_y[m]            (count = #chunks)
      E_y[m]        --"m->m"-->  reduce m
    Unfused: each operator boundary is one event."""
    g = Graph()
    n_gu = _cdiv(inter, gu_tile)
    n_m = _cdiv(hidden, down_tile)
    n_c = _cdiv(inter, kchunk)
    unf = sched == "unfused"
    for b in range(B):
        t = (OP_MLP_NORM, b, 0)
        g.add_task(t)
        g.produce(t, ("E_norm",))
    for n in range(n_gu):
        t = (OP_MLP_GATEUP, n, 0)
        g.add_task(t)
        g.consume(t, ("E_norm",))
        g.produce(t, ("E_h_all",) if unf else ("E_h", (n * gu_tile) // kchunk))
    for m in range(n_m):
        for c in range(n_c):
            t = (OP_MLP_DOWN, m, c)
            g.add_task(t)
            g.consume(t, ("E_h_all",) if unf else ("E_h", c))
            g.produce(t, ("E_y_all",) if unf else ("E_y", m))
    for m in range(n_m):
        t = (OP_MLP_REDUCE, m, 0)
        g.add_task(t)
        g.consume(t, ("E_y_all",) if unf else ("E_y", m))
    g.wait_count[("E_norm",)] = B
    return g.finish()


def moe_graph(topk, E, tt, n_kc, tkt, gt, bm, n_n1, n_n2, cb, sched):
    """MoE layer, expanded with the runtime routing `topk` [T, k]:
      router (j, c)   --"jc->j"-->           E_rt[j]         (count = #K chunks n_kc; tkt
                                                             tokens per block j)
      the chunk task completing E_rt[j] routes block j (logits, top-k,
      softmax), so every router (j, c) precedes:
      router (j, *)   --"j->"-->             E_tk            (count = #token blocks)
      E_tk            -->                    scan
      one grouping tile (T <= tt): the scan is the grouping task:
      scan            --> E_exp[topk[i,:]] for every token i
      several grouping tiles:
      scan            -->                    E_sc            (count 1)
      E_sc            --"->g"-->             group g         (gt tokens)
      group g         --> E_exp[topk[i,:]] for every token i of group g
                                               (count of E_exp[e] = #pairs routed to e)
      E_exp[e]        --> stage1 tasks[task_indptr[e] : task_indptr[e+1]] x n1 tiles
      stage1 (f, n)   --"fn->f"-->           E_s1[f]         (count = #n1 tiles)
      E_s1[f]         --"f->fn"-->           stage2 (f, n)
      stage2 (f, n)   --> E_cb[i // cb] for every row (token i) of m-tile f
      E_cb[b]         -->                    combine b
    Static scheduling replaces grouping -> E_exp -> stage1 by one coarse event
    (every grouping task -> every stage1 task).  Unfused replaces every
    operator boundary by one event."""
    topk = np.asarray(topk)
    T, k = topk.shape
    g = Graph()
    n_tt = _cdiv(T, tt)
    n_tk = _cdiv(T, tkt)
    n_g = _cdiv(T, gt)
    n_cb = _cdiv(T, cb)
    unf = sched == "unfused"
    static = sched == "static"
    # grouping by brute force: pairs per expert in token order
    rows_of = [[] for _ in range(E)]
    for t in range(T):
        for s in range(k):
            rows_of[int(topk[t, s])].append((t, s))
    mtiles = []   # flat m-tile list: (expert, tile index, [(t, s) rows])
    for e in range(E):
        r = rows_of[e]
        for m in range(_cdiv(len(r), bm)):
            mtiles.append((e, m, r[m * bm:(m + 1) * bm]))
    for j in range(n_tk):
        for c in range(n_kc):
            task = (OP_MOE_ROUTER, j, c)
            g.add_task(task)
            g.produce(task, ("E_tk",))
    scan = (OP_MOE_SCAN, 0, 0)
    g.add_task(scan)
    g.consume(scan, ("E_tk",))
    if n_tt == 1:
        if unf or static:
            g.produce(scan, ("E_grp",))
        else:
            for i in range(T):
                for s in range(k):
                    g.produce(scan, ("E_exp", int(topk[i, s])))
    else:
        g.produce(scan, ("E_sc",))
        for q in range(n_g):
            task = (OP_MOE_GROUP, q, 0)
            g.add_task(task)
            g.consume(task, ("E_sc",))
            if unf or static:
                g.produce(task, ("E_grp",))
            else:
                for i in range(q * gt, min(T, (q + 1) * gt)):
                    for s in range(k):
                        g.produce(task, ("E_exp", int(topk[i, s])))
    for f, (e, m, rows) in enumerate(mtiles):
        for n in range(n_n1):
            task = (OP_MOE_S1, f, n)
            g.add_task(task)
            g.consume(task, ("E_grp",) if (unf or static) else ("E_exp", e))
            g.produce(task, ("E_s1_all",) if unf else ("E_s1", f))
    for f, (e, m, rows) in enumerate(mtiles):
        for n in range(n_n2):
            task = (OP_MOE_S2, f, n)
            g.add_task(task)
            g.consume(task, ("E_s1_all",) if unf else ("E_s1", f))
            if unf:
                g.produce(task, ("E_s2_all",))
            else:
                for (t, s) in rows:
                    g.produce(task, ("E_cb", t // cb))
    for b in range(n_cb):
        task = (OP_MOE_COMBINE, b, 0)
        g.add_task(task)
        g.consume(task, ("E_s2_all",) if unf else ("E_cb", b))
    return g.finish(), mtiles


def check_trace(graph, records):
    """records: iterable of (op, a, b, sm, start_ticket, end_ticket).
    Returns a list of violation strings (empty = the trace is valid)."""
    errs = []
    seen = {}
    for r in records:
        key = (int(r[0]), int(r[1]), int(r[2]))
        if key in seen:
            errs.append("task ran twice: %r" % (key,))
        seen[key] = (int(r[4]), int(r[5]))
        if int(r[4]) > int(r[5]):
            errs.append("task ended before it started: %r" % (key,))
    want = set(graph.tasks)
    got = set(seen)
    for t in sorted(want - got):
        errs.append("task never ran: %r" % (t,))
    for t in sorted(got - want):
        errs.append("unexpected task ran: %r" % (t,))
    for (p, c) in graph.edges:
        if p in seen and c in seen and not seen[p][1] < seen[c][0]:
            errs.append("edge violated: %r (end %d) -> %r (start %d)" % (p, seen[p][1], c, seen[c][0]))
    return errs
