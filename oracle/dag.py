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
* every event received exactly its wait count of notifications
  (``check_wait_counts`` on the expansion itself, ``check_event_counts``
  against the counts the device reports after a run).

The event graph restates which events the device library uses.  A second,
independent check does not look at events at all: ``*_dataflow`` derives
from what each operator computes the data every task reads and writes
(router logits of a token, the grouped row of a routed pair, a column tile
of the stage-1 output, the combine accumulator of a token, ...), and
``check_dataflow`` requires every writer of an item to finish before any
task that reads it starts.  A dependency missing from the device's event
design (and so from the event graph) is still caught there.

Tasks are tuples ``(op, a, b)``; the op names and coordinates follow the
trace record format of the device library (see ``include/et.h``).  An
"inline" task is work the device runs inside another task (the top-k of a
router block, run by the router task that completes the block); it has no
trace record, and edges through it are contracted.
"""
from collections import defaultdict

import numpy as np

# op codes of trace records (an interface: the same numbers are declared in
# include/et.h, where the record format is defined)
OP_SK_PARTIAL, OP_SK_FINAL = 1, 2
OP_MLP_NORM, OP_MLP_GATEUP, OP_MLP_DOWN, OP_MLP_REDUCE = 10, 11, 12, 13
OP_MOE_ROUTER, OP_MOE_SCAN, OP_MOE_GROUP, OP_MOE_S1, OP_MOE_S2, OP_MOE_COMBINE = (
    20, 22, 23, 24, 25, 26)
(OP_DEC_NORM1, OP_DEC_QKV, OP_DEC_QBR, OP_DEC_KBR, OP_DEC_VBR, OP_DEC_ATTN, OP_DEC_MERGE, OP_DEC_OPROJ,
 OP_DEC_NORM2, OP_DEC_GATEUP, OP_DEC_DOWN, OP_DEC_RED) = range(30, 42)


def _cdiv(a, b):
    return (a + b - 1) // b


# event kinds of the device's event-count records (an interface: the same
# numbers are declared in include/et.h) -> event names used below
EVENT_KIND = {1: "E", 2: "Eall", 10: "E_norm", 11: "E_h", 12: "E_y", 13: "E_h_all", 14: "E_y_all",
              20: "E_rt", 21: "E_tk", 22: "E_sc", 23: "E_grp", 24: "E_exp", 25: "E_s1", 26: "E_cb",
              27: "E_s1_all", 28: "E_s2_all",
              40: "D_n1", 41: "D_qkv", 42: "D_g", 43: "D_att", 44: "D_ag", 45: "D_o", 46: "D_n2", 47: "D_h",
              48: "D_y", 49: "D_branch_all", 50: "D_merge_all", 51: "D_gu_all", 52: "D_down_all"}
_SCALAR_EVENTS = {"Eall", "E_norm", "E_h_all", "E_y_all", "E_tk", "E_sc", "E_grp", "E_s1_all", "E_s2_all",
                  "D_n1", "D_o", "D_n2", "D_branch_all", "D_merge_all", "D_gu_all", "D_down_all"}


def event_key(kind, index):
    name = EVENT_KIND[kind]
    return (name,) if name in _SCALAR_EVENTS else (name, index)


class Graph:
    """Explicit DAG: tasks, edges, per-event producer lists (one entry per
    notification, so a task that notifies an event n times is listed n
    times) and the declared wait count of every event a counter realises."""

    def __init__(self):
        self.tasks = []
        self.inline = set()
        self.edges = set()
        self.event_producers = defaultdict(list)   # event -> producer tasks (with multiplicity)
        self.event_consumers = defaultdict(list)   # event -> consumer tasks
        self.wait_count = {}                        # counted event -> declared wait count

    def add_task(self, t, inline=False):
        self.tasks.append(t)
        if inline:
            self.inline.add(t)

    def produce(self, task, event, n=1):
        self.event_producers[event].extend([task] * n)

    def consume(self, task, event):
        self.event_consumers[event].append(task)

    def counted(self, event, wait_count):
        """`event` is a device counter that fires at `wait_count` notifications."""
        self.wait_count[event] = int(wait_count)

    def finish(self):
        """Edges = every producer of an event -> every consumer of it, with
        inline tasks contracted (pred -> inline -> succ becomes pred -> succ)."""
        raw = set()
        for ev, cons in self.event_consumers.items():
            for p in set(self.event_producers.get(ev, [])):
                for c in cons:
                    raw.add((p, c))
        if self.inline:
            pred, succ = defaultdict(set), defaultdict(set)
            for p, c in raw:
                pred[c].add(p)
                succ[p].add(c)
            for t in self.inline:
                for p in pred[t]:
                    for c in succ[t]:
                        raw.add((p, c))
                        pred[c].add(p)
                        succ[p].add(c)
            raw = {(p, c) for (p, c) in raw if p not in self.inline and c not in self.inline}
        self.edges = raw
        self.tasks = [t for t in self.tasks if t not in self.inline]
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
    # E = ETensor((n,), wait_count=#chunks): each row tile's final waits for its partials
    if sched != "unfused":
        for i in range(n):
            g.counted(("E", i), J)
    else:
        g.counted(("Eall",), n * J)
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
    # wait counts: every row normalised (a symbolic count B); a K chunk of h
    # holds kchunk / gu_tile gate/up tiles; an output tile sums every chunk
    g.counted(("E_norm",), B)
    if unf:
        g.counted(("E_h_all",), n_gu)
        g.counted(("E_y_all",), n_m * n_c)
    else:
        for c in range(n_c):
            g.counted(("E_h", c), sum(1 for n in range(n_gu) if (n * gu_tile) // kchunk == c))
        for m in range(n_m):
            g.counted(("E_y", m), n_c)
    return g.finish()


def moe_graph(topk, E, tt, n_kc, tkt, gt, bm, n_n1, n_n2, cb, sched):
    """MoE layer, expanded with the runtime routing `topk` [T, k]:
      router (j, c)   --"jc->j"-->           E_rt[j]         (count = #K chunks n_kc; tkt
                                                             tokens per block j; only with n_kc > 1)
      E_rt[j]         -->                    route j         (inline: top-k + softmax of block j,
                                                             run by the chunk task completing E_rt[j])
      route j         --"j->"-->             E_tk            (count = #token blocks)
      E_tk            -->                    scan
      one grouping tile (T <= tt): the scan is the grouping task and
      triggers the stage-1 tasks itself (E_exp has no counter then):
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
    counts = [len(r) for r in rows_of]
    for j in range(n_tk):
        route = ("route", j)
        g.add_task(route, inline=True)
        for c in range(n_kc):
            task = (OP_MOE_ROUTER, j, c)
            g.add_task(task)
            if n_kc > 1:
                g.produce(task, ("E_rt", j))
            else:
                g.produce(task, ("E_rt1", j))   # one chunk: the router task routes its own block
        if n_kc > 1:
            g.consume(route, ("E_rt", j))
            g.counted(("E_rt", j), n_kc)
        else:
            g.consume(route, ("E_rt1", j))
        g.produce(route, ("E_tk",))
    g.counted(("E_tk",), n_tk)
    scan = (OP_MOE_SCAN, 0, 0)
    g.add_task(scan)
    g.consume(scan, ("E_tk",))
    if n_tt == 1:
        if unf or static:
            g.produce(scan, ("E_grp",))
            g.counted(("E_grp",), 1)
        else:
            for i in range(T):
                for s in range(k):
                    g.produce(scan, ("E_exp", int(topk[i, s])))
    else:
        g.produce(scan, ("E_sc",))
        g.counted(("E_sc",), 1)
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
        if unf or static:
            g.counted(("E_grp",), n_g)
        else:
            # data-dependent initial count: the number of pairs routed to e
            for e in range(E):
                if counts[e]:
                    g.counted(("E_exp", e), counts[e])
    for f, (e, m, rows) in enumerate(mtiles):
        for n in range(n_n1):
            task = (OP_MOE_S1, f, n)
            g.add_task(task)
            g.consume(task, ("E_grp",) if (unf or static) else ("E_exp", e))
            g.produce(task, ("E_s1_all",) if unf else ("E_s1", f))
        if not unf:
            g.counted(("E_s1", f), n_n1)
    if unf:
        g.counted(("E_s1_all",), len(mtiles) * n_n1)
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
        if unf:
            g.consume(task, ("E_grp",))
            g.consume(task, ("E_s2_all",))
        else:
            g.consume(task, ("E_cb", b))
            # every stage-2 column tile of every routed pair of the block's tokens
            ntok = min(cb, T - b * cb)
            g.counted(("E_cb", b), k * n_n2 * ntok)
    if unf:
        g.counted(("E_s2_all",), len(mtiles) * n_n2)
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


# ------------------------------------------------------------ wait counts --

def check_wait_counts(graph):
    """Every counted event has exactly its wait count of producer
    notifications in the expansion.  Returns violation strings."""
    errs = []
    for ev, want in sorted(graph.wait_count.items(), key=repr):
        got = len(graph.event_producers.get(ev, []))
        if got != want:
            errs.append("event %r: %d producer notifications, wait count %d" % (ev, got, want))
    return errs


def check_event_counts(graph, device_counts):
    """device_counts: (kind, index, count) records of the device's events
    after a run.  Every event the expansion counts received exactly its wait
    count of notifications; every other event of the device received none.
    Returns violation strings."""
    errs = []
    seen = set()
    for kind, index, count in device_counts:
        key = event_key(int(kind), int(index))
        seen.add(key)
        want = graph.wait_count.get(key, 0)
        if int(count) != want:
            errs.append("event %r received %d notifications, wait count %d" % (key, int(count), want))
    for key in graph.wait_count:
        if key not in seen:
            errs.append("event %r has no device counter" % (key,))
    return errs


# --------------------------------------------------------------- dataflow --
# Read and write sets of each task, from what its operator computes.  Items:
#   ("logit", t, c)   K chunk c of token t's router logits
#   ("route", t)      top-k experts and weights of token t (a function of all
#                     of t's logit chunks; the router tasks of t's block write it)
#   ("csr",)          expert counts, pair CSR, m-tile CSR (needs every token's route)
#   ("row", r)        the routed pair placed at grouped row r
#   ("h", r, n)       stage-1 output of grouped row r, column tile n
#   ("acc", t, n)     token t's combine accumulator, column tile n (summed by stage 2)
#   ("y", t)          token t's output

def moe_dataflow(topk, n_kc, tkt, tt, bm, n_n1, n_n2, cb, E):
    """{task: (reads, writes)} of every task of the MoE layer given the
    runtime routing; the task split (tkt, n_kc, tt, bm, n-tiles, cb) is the
    device's tiling, the items each task touches follow from the operators."""
    topk = np.asarray(topk)
    T, k = topk.shape
    rw = {}
    # stable grouping by brute force: expert-major, ascending token
    order = [(t, s) for e in range(E) for t in range(T) for s in range(k) if int(topk[t, s]) == e]
    row_of = {pair: r for r, pair in enumerate(order)}
    # ("row", r): grouped row r placed (its pair index, and, where the device
    # stages stage-1 rows in grouped order, its copy of the token's X row)
    all_route = {("route", t) for t in range(T)}
    for j in range(_cdiv(T, tkt)):
        toks = range(j * tkt, min(T, (j + 1) * tkt))
        for c in range(n_kc):
            w = {("logit", t, c) for t in toks} | {("route", t) for t in toks}
            rw[(OP_MOE_ROUTER, j, c)] = (set(), w)
    n_tt = _cdiv(T, tt)
    sc_w = {("csr",)}
    if n_tt == 1:
        sc_w |= {("row", r) for r in range(len(order))}
    rw[(OP_MOE_SCAN, 0, 0)] = (set(all_route), sc_w)
    if n_tt > 1:
        for g in range(n_tt):
            toks = range(g * tt, min(T, (g + 1) * tt))
            rows = {("row", row_of[(t, s)]) for t in toks for s in range(k)}
            rw[(OP_MOE_GROUP, g, 0)] = ({("csr",)} | all_route, rows)
    f = 0
    for e in range(E):
        rows_e = [r for r, (t, s) in enumerate(order) if int(topk[t, s]) == e]
        for m in range(_cdiv(len(rows_e), bm)):
            rows = rows_e[m * bm:(m + 1) * bm]
            toks = {order[r][0] for r in rows}
            base = {("csr",)} | {("row", r) for r in rows}
            for n in range(n_n1):
                rw[(OP_MOE_S1, f, n)] = (set(base), {("h", r, n) for r in rows})
            h_all = {("h", r, n) for r in rows for n in range(n_n1)}
            for n in range(n_n2):
                rw[(OP_MOE_S2, f, n)] = (base | h_all | {("route", t) for t in toks},
                                         {("acc", t, n) for t in toks})
            f += 1
    for b in range(_cdiv(T, cb)):
        toks = range(b * cb, min(T, (b + 1) * cb))
        rw[(OP_MOE_COMBINE, b, 0)] = ({("acc", t, n) for t in toks for n in range(n_n2)},
                                      {("y", t) for t in toks})
    return rw


def mlp_dataflow(B, hidden, inter, gu_tile, down_tile, kchunk):
    """Decode MLP: norm b writes xn row b; gate/up tile n reads every xn row
    and writes h columns of tile n; down (m, c) reads the h columns of K
    chunk c and writes partial (m, c); reduce m reads every partial of m."""
    rw = {}
    n_gu, n_m, n_c = _cdiv(inter, gu_tile), _cdiv(hidden, down_tile), _cdiv(inter, kchunk)
    for b in range(B):
        rw[(OP_MLP_NORM, b, 0)] = (set(), {("xn", b)})
    for n in range(n_gu):
        rw[(OP_MLP_GATEUP, n, 0)] = ({("xn", b) for b in range(B)}, {("h", n)})
    for m in range(n_m):
        for c in range(n_c):
            cols = {("h", n) for n in range(n_gu) if c * kchunk <= n * gu_tile < (c + 1) * kchunk}
            rw[(OP_MLP_DOWN, m, c)] = (cols, {("part", m, c)})
        rw[(OP_MLP_REDUCE, m, 0)] = ({("part", m, c) for c in range(n_c)}, {("y", m)})
    return rw


def splitk_dataflow(rows, cols, chunk, tile_rows):
    """Split-K: partial (i, j) writes B[rows of tile i, j]; final i reads
    B[rows of tile i, every j]."""
    rw = {}
    n, J = _cdiv(rows, tile_rows), _cdiv(cols, chunk)
    for i in range(n):
        for j in range(J):
            rw[(OP_SK_PARTIAL, i, j)] = (set(), {("B", i, j)})
        rw[(OP_SK_FINAL, i, 0)] = ({("B", i, j) for j in range(J)}, {("C", i)})
    return rw


def check_dataflow(rw, records):
    """Every task that reads an item starts after every task that writes it
    has finished (read-after-write by ticket).  records as in check_trace.
    Returns violation strings."""
    start, end = {}, {}
    for r in records:
        key = (int(r[0]), int(r[1]), int(r[2]))
        start[key], end[key] = int(r[4]), int(r[5])
    writers = defaultdict(list)
    for task, (_, writes) in rw.items():
        for it in writes:
            writers[it].append(task)
    errs = []
    for task, (reads, _) in rw.items():
        if task not in start:
            errs.append("task never ran: %r" % (task,))
            continue
        for it in reads:
            for w in writers.get(it, []):
                if w == task:
                    continue
                if w not in end:
                    errs.append("writer of %r never ran: %r" % (it, w))
                elif not end[w] < start[task]:
                    errs.append("read before write: %r reads %r, written by %r (end %d, start %d)"
                                % (task, it, w, end[w], start[task]))
    return errs


# ------------------------------------------------------------ decode layer --

def decode_graph(pos, nq, nkv, n_kc, split, n_m, n_gu, gu_tile, kchunk, n_c, sched):
    """One decode step for len(pos) requests (pos[b] = the new token's
    position), expanded with the run-time positions:
      N1 b          --"b->"-->      D_n1              (count B)
      D_n1          --"->nc"-->     QKV (n, c)
      QKV (n, c)    --"nc->n"-->    D_qkv[n]          (count = #K chunks)
      D_qkv[n]      -->             branch n          (Q: norm + RoPE; K: norm + RoPE +
                                                       cache append; V: cache append)
      branch n      --"n->g"-->     D_g[g]            (count = query heads per group + 2)
      D_g[g]        --"g->bgs"-->   ATTN (b, g, s)    s < ceil((pos[b] + 1) / split):
                                                      tasks[split_indptr[b] : split_indptr[b+1]]
      ATTN (b,g,s)  --"bgs->bg"-->  D_att[b, g]       (count = the request's split count)
      D_att[b, g]   -->             merge (b, g)
      merge (b, g)  --"bg->g"-->    D_ag[g]           (count B)
      D_ag[g]       --"g->mg"-->    o-proj (m, g)
      o-proj (m, c) -->             D_o               (count = #tiles x #groups)
      D_o           -->             N2 b  --> D_n2 (count B) --> gate/up n --> D_h[c] --> down (m, c)
                                    --> D_y[m] (count = #K chunks) --> reduce m
    Unfused: branch -> D_branch_all -> every split; merge -> D_merge_all ->
    every o-proj; gate/up -> D_gu_all -> every down; down -> D_down_all ->
    every reduce (the other edges are already operator-wide)."""
    pos = [int(v) for v in pos]
    B = len(pos)
    grp = nq // nkv
    n_heads = nq + 2 * nkv
    unf = sched == "unfused"
    g = Graph()
    for b in range(B):
        t = (OP_DEC_NORM1, b, 0)
        g.add_task(t)
        g.produce(t, ("D_n1",))
    g.counted(("D_n1",), B)
    for n in range(n_heads):
        kind = OP_DEC_QBR if n < nq else (OP_DEC_KBR if n < nq + nkv else OP_DEC_VBR)
        grp_of = n // grp if n < nq else (n - nq if n < nq + nkv else n - nq - nkv)
        br = (kind, n, 0)
        g.add_task(br)
        for c in range(n_kc):
            t = (OP_DEC_QKV, n, c)
            g.add_task(t)
            g.consume(t, ("D_n1",))
            g.produce(t, ("D_qkv", n))
        g.counted(("D_qkv", n), n_kc)
        g.consume(br, ("D_qkv", n))
        g.produce(br, ("D_branch_all",) if unf else ("D_g", grp_of))
    if unf:
        g.counted(("D_branch_all",), n_heads)
    else:
        for gg in range(nkv):
            g.counted(("D_g", gg), grp + 2)
    for b in range(B):
        ns = (pos[b] + 1 + split - 1) // split
        for gg in range(nkv):
            bg = b * nkv + gg
            mg = (OP_DEC_MERGE, bg, 0)
            g.add_task(mg)
            for s_ in range(ns):
                t = (OP_DEC_ATTN, bg, s_)
                g.add_task(t)
                g.consume(t, ("D_branch_all",) if unf else ("D_g", gg))
                g.produce(t, ("D_att", bg))
            g.counted(("D_att", bg), ns)
            g.consume(mg, ("D_att", bg))
            g.produce(mg, ("D_merge_all",) if unf else ("D_ag", gg))
    if unf:
        g.counted(("D_merge_all",), B * nkv)
    else:
        for gg in range(nkv):
            g.counted(("D_ag", gg), B)
    for c in range(nkv):
        for m in range(n_m):
            t = (OP_DEC_OPROJ, m, c)
            g.add_task(t)
            g.consume(t, ("D_merge_all",) if unf else ("D_ag", c))
            g.produce(t, ("D_o",))
    g.counted(("D_o",), n_m * nkv)
    for b in range(B):
        t = (OP_DEC_NORM2, b, 0)
        g.add_task(t)
        g.consume(t, ("D_o",))
        g.produce(t, ("D_n2",))
    g.counted(("D_n2",), B)
    for n in range(n_gu):
        t = (OP_DEC_GATEUP, n, 0)
        g.add_task(t)
        g.consume(t, ("D_n2",))
        g.produce(t, ("D_gu_all",) if unf else ("D_h", (n * gu_tile) // kchunk))
    if unf:
        g.counted(("D_gu_all",), n_gu)
    else:
        for c in range(n_c):
            g.counted(("D_h", c), sum(1 for n in range(n_gu) if (n * gu_tile) // kchunk == c))
    for m in range(n_m):
        for c in range(n_c):
            t = (OP_DEC_DOWN, m, c)
            g.add_task(t)
            g.consume(t, ("D_gu_all",) if unf else ("D_h", c))
            g.produce(t, ("D_down_all",) if unf else ("D_y", m))
        if not unf:
            g.counted(("D_y", m), n_c)
    if unf:
        g.counted(("D_down_all",), n_m * n_c)
    for m in range(n_m):
        t = (OP_DEC_RED, m, 0)
        g.add_task(t)
        g.consume(t, ("D_down_all",) if unf else ("D_y", m))
    return g.finish()


def decode_dataflow(pos, nq, nkv, n_kc, split, n_m, n_gu, gu_tile, kchunk, n_c):
    """{task: (reads, writes)} of one decode step, from what each operator
    computes.  Items: ("xn", b), ("qkv", n) (head tile n's sums over every K
    chunk), ("q", h), ("knew", g) / ("vnew", g) (the cache entries of this
    step: position pos[b] of every request b), ("part", b, g, s),
    ("attn", b, g), ("o", m) (o-proj sums), ("h1", b), ("xn2", b), ("hm", n),
    ("down", m), ("y", m).  A split reads the new cache entries only if its
    keys include pos[b]; the older entries are not written in this step."""
    pos = [int(v) for v in pos]
    B = len(pos)
    grp = nq // nkv
    n_heads = nq + 2 * nkv
    rw = {}
    for b in range(B):
        rw[(OP_DEC_NORM1, b, 0)] = (set(), {("xn", b)})
    xn_all = {("xn", b) for b in range(B)}
    for n in range(n_heads):
        for c in range(n_kc):
            rw[(OP_DEC_QKV, n, c)] = (set(xn_all), {("qkv", n)})
        if n < nq:
            rw[(OP_DEC_QBR, n, 0)] = ({("qkv", n)}, {("q", n)})
        elif n < nq + nkv:
            rw[(OP_DEC_KBR, n, 0)] = ({("qkv", n)}, {("knew", n - nq)})
        else:
            rw[(OP_DEC_VBR, n, 0)] = ({("qkv", n)}, {("vnew", n - nq - nkv)})
    for b in range(B):
        ns = (pos[b] + 1 + split - 1) // split
        for gg in range(nkv):
            bg = b * nkv + gg
            qs = {("q", gg * grp + h) for h in range(grp)}
            for s_ in range(ns):
                reads = set(qs)
                if s_ * split <= pos[b] < (s_ + 1) * split:
                    reads |= {("knew", gg), ("vnew", gg)}
                rw[(OP_DEC_ATTN, bg, s_)] = (reads, {("part", b, gg, s_)})
            rw[(OP_DEC_MERGE, bg, 0)] = ({("part", b, gg, s_) for s_ in range(ns)}, {("attn", b, gg)})
    for c in range(nkv):
        for m in range(n_m):
            rw[(OP_DEC_OPROJ, m, c)] = ({("attn", b, c) for b in range(B)}, {("o", m)})
    for b in range(B):
        rw[(OP_DEC_NORM2, b, 0)] = ({("o", m) for m in range(n_m)}, {("h1", b), ("xn2", b)})
    for n in range(n_gu):
        rw[(OP_DEC_GATEUP, n, 0)] = ({("xn2", b) for b in range(B)}, {("hm", n)})
    for m in range(n_m):
        for c in range(n_c):
            cols = {("hm", n) for n in range(n_gu) if c * kchunk <= n * gu_tile < (c + 1) * kchunk}
            rw[(OP_DEC_DOWN, m, c)] = (cols, {("down", m)})
        rw[(OP_DEC_RED, m, 0)] = ({("down", m)} | {("h1", b) for b in range(B)}, {("y", m)})
    return rw


# ---------------------------------------------------------- MoE -> dense MLP --

def moe_mlp_graph(topk, E, tt, n_kc, tkt, gt, bm, n_n1, n_n2, cb, sched, hidden, inter, gu_tile, down_tile,
                  kchunk):
    """The MoE layer (moe_graph) followed by a dense MLP on its output: each
    combine task CB(b) also normalises its tokens for the MLP and notifies
    E_norm once per token (count T); the MLP's gate/up, down and reduce
    tasks follow as in mlp_graph (no norm tasks of their own)."""
    g, mt = moe_graph(topk, E, tt, n_kc, tkt, gt, bm, n_n1, n_n2, cb, sched)
    T = len(topk)
    unf = sched == "unfused"
    m = mlp_graph(T, hidden, inter, gu_tile, down_tile, kchunk, sched)
    for b in range(_cdiv(T, cb)):
        g.produce((OP_MOE_COMBINE, b, 0), ("E_norm",), n=min(cb, T - b * cb))
    for t in m.tasks:
        if t[0] != OP_MLP_NORM:
            g.add_task(t)
    for ev, cons in m.event_consumers.items():
        for c in cons:
            g.consume(c, ev)
    for ev, prods in m.event_producers.items():
        if ev != ("E_norm",):
            for p_ in prods:
                g.produce(p_, ev)
    for ev, wc in m.wait_count.items():
        g.counted(ev, wc)
    # mlp_graph's finish() already ran on m; rebuild this graph's edges
    g.edges = set()
    g.tasks = list(dict.fromkeys(g.tasks))
    return g.finish(), mt


def moe_mlp_dataflow(topk, n_kc, tkt, tt, bm, n_n1, n_n2, cb, E, hidden, inter, gu_tile, down_tile, kchunk):
    """moe_dataflow plus the MLP: CB(b) also writes ("xn", t) of its tokens,
    the MLP tasks read and write as in mlp_dataflow."""
    rw = moe_dataflow(topk, n_kc, tkt, tt, bm, n_n1, n_n2, cb, E)
    T = len(topk)
    for b in range(_cdiv(T, cb)):
        r, w = rw[(OP_MOE_COMBINE, b, 0)]
        rw[(OP_MOE_COMBINE, b, 0)] = (r, w | {("xn", t) for t in range(b * cb, min(T, (b + 1) * cb))})
    for task, v in mlp_dataflow(T, hidden, inter, gu_tile, down_tile, kchunk).items():
        if task[0] != OP_MLP_NORM:
            rw[task] = v
    return rw
