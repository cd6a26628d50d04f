"""Checks of a built task graph that hold for any correct builder.

A graph is any object with numpy arrays task_type/op/layer/idx/dep/trig,
event_count/first/last and raw edges edge_src/edge_dst (final task ids).
"""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
EMPTY = 10


def check_invariants(g):
    nt, ne = g.task_type.size, g.event_count.size
    dep, trig = g.task_dep, g.task_trig
    assert ((dep >= -1) & (dep < ne)).all() and ((trig >= -1) & (trig < ne)).all()
    # each event's dependents are exactly its [first, last] range
    by_dep = np.full(ne, 0)
    np.add.at(by_dep, dep[dep >= 0], 1)
    assert (by_dep == g.event_last - g.event_first + 1).all()
    for e in range(ne):
        f, l = g.event_first[e], g.event_last[e]
        assert 0 <= f <= l < nt
        assert (dep[f:l + 1] == e).all()
    # the trigger count is the number of triggering tasks
    by_trig = np.zeros(ne, dtype=np.int64)
    np.add.at(by_trig, trig[trig >= 0], 1)
    assert (by_trig == g.event_count).all()
    assert (g.event_count >= 1).all()
    # linear order is topological: every trigger of a task's event precedes it
    last_trigger = np.full(ne, -1)
    np.maximum.at(last_trigger, trig[trig >= 0], np.nonzero(trig >= 0)[0])
    has = dep >= 0
    assert (last_trigger[dep[has]] < np.nonzero(has)[0]).all()
    # events are numbered in the order their last trigger is placed
    order = np.argsort(last_trigger, kind="stable")
    assert (order == np.arange(ne)).all()


def simulate_random(g, seed, check_edges=True):
    """Run the graph with a random choice among ready tasks; check every raw edge."""
    rng = np.random.default_rng(seed)
    nt, ne = g.task_type.size, g.event_count.size
    got = np.zeros(ne, dtype=np.int64)
    ready = list(np.nonzero(g.task_dep < 0)[0])
    finish = np.full(nt, -1)
    start = np.full(nt, -1)
    clock = 0
    while ready:
        i = int(rng.integers(len(ready)))
        ready[i], ready[-1] = ready[-1], ready[i]
        t = ready.pop()
        start[t] = clock
        clock += 1
        finish[t] = clock
        clock += 1
        e = g.task_trig[t]
        if e >= 0:
            got[e] += 1
            if got[e] == g.event_count[e]:
                ready.extend(range(g.event_first[e], g.event_last[e] + 1))
    assert (finish >= 0).all(), "some tasks never became ready"
    if check_edges and g.edge_src.size:
        assert (finish[g.edge_src] <= start[g.edge_dst]).all()


def simulate_static_queues(g, workers):
    """Worker w runs tasks w, w+W, ... in order; must finish without deadlock."""
    nt, ne = g.task_type.size, g.event_count.size
    got = np.zeros(ne, dtype=np.int64)
    head = list(range(min(workers, nt)))
    done = 0
    while done < nt:
        progressed = False
        for w in range(len(head)):
            t = head[w]
            while t < nt:
                e = g.task_dep[t]
                if e >= 0 and got[e] < g.event_count[e]:
                    break
                te = g.task_trig[t]
                if te >= 0:
                    got[te] += 1
                t += workers
                done += 1
                progressed = True
            head[w] = t
        assert progressed, "static per-worker queues deadlocked"


def load_golden(name):
    cfg, nodes, edges, tasks, events = {}, [], [], [], []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            parts = line.split()
            if parts[0] == "config":
                for kv in parts[1:]:
                    k, v = kv.split("=")
                    cfg[k] = int(v)
            elif parts[0] == "node":
                nodes.append((parts[1], int(parts[2]), int(parts[3])))
            elif parts[0] == "edge":
                edges.append((parts[1], parts[2]))
            elif parts[0] == "task":
                tasks.append([int(x) for x in parts[2:]])
            elif parts[0] == "event":
                events.append([int(x) for x in parts[2:]])
    return cfg, nodes, edges, np.array(tasks, dtype=np.int32), np.array(events, dtype=np.int32)


def assert_tables_equal(g, tasks, events):
    got_t = np.stack([g.task_type, g.task_op, g.task_layer, g.task_idx, g.task_dep,
                      g.task_trig], axis=1)
    got_e = np.stack([g.event_count, g.event_first, g.event_last], axis=1)
    np.testing.assert_array_equal(got_t, tasks)
    np.testing.assert_array_equal(got_e, events)


def assert_graphs_equal(a, b):
    for name in ("task_type", "task_op", "task_layer", "task_idx", "task_dep", "task_trig",
                 "event_count", "event_first", "event_last"):
        np.testing.assert_array_equal(getattr(a, name), getattr(b, name), err_msg=name)


def random_dag(seed, n_ops=(3, 8), per_op=(1, 6), p_edge=0.35):
    """Random op-ordered task DAG: (task_op, task_idx, edges)."""
    rng = np.random.default_rng(seed)
    ops = int(rng.integers(*n_ops))
    task_op, task_idx = [], []
    for o in range(ops):
        for i in range(int(rng.integers(*per_op))):
            task_op.append(o)
            task_idx.append(i)
    n = len(task_op)
    edges = []
    for c in range(n):
        for a in range(n):
            if task_op[a] < task_op[c] and rng.random() < p_edge / max(1, task_op[c] - task_op[a]):
                edges.append((a, c))
    perm = rng.permutation(n)  # builders must not depend on input order
    inv = np.argsort(perm)
    task_op = [task_op[p] for p in perm]
    task_idx = [task_idx[p] for p in perm]
    edges = [(int(inv[a]), int(inv[c])) for a, c in edges]
    return task_op, task_idx, edges


def closed_form_counts(w, kv_capacity, W, col_align=16, apw=4, min_chunk=64):
    """Task and event counts of the decode graph (no empty tasks are needed)."""
    cdiv = lambda a, b: -(-a // b)
    aup = lambda a, b: cdiv(a, b) * b
    rep = w.n_q_heads // w.n_kv_heads
    G = (rep + 2) * w.head_dim
    Nqkv = w.n_kv_heads * G
    m = next((m for m in range(col_align, G + 1, col_align) if G % m == 0 and cdiv(Nqkv, m) <= W), G)
    t_qkv = cdiv(Nqkv, m)
    tiles = lambda N: cdiv(N, aup(cdiv(N, W), col_align))
    sp = max(1, apw * W // (w.batch * w.n_kv_heads))
    chunk = max(min_chunk, aup(cdiv(kv_capacity, sp), 64))
    S = cdiv(kv_capacity, chunk)
    n_attn = w.batch * w.n_kv_heads * S
    per_layer = t_qkv + n_attn + tiles(w.hidden) + tiles(w.ffn) + tiles(w.hidden)
    tasks = 1 + w.n_layers * per_layer + tiles(w.vocab) + 1
    # events per layer: x (QKV input), one per kv group (QKV -> ATTN), attention
    # output (ATTN -> O), O output, GATE_UP output; plus the final hidden state
    # (-> LM_HEAD) and the LM partials (-> ARGMAX).
    ev_layer = 1 + w.n_kv_heads + 3
    events = w.n_layers * ev_layer + 2
    return tasks, events
