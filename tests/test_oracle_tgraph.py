"""Pins of the oracle's task-graph builder: hand-derived tables, invariants,
closed-form counts and execution semantics on decode and random graphs."""
import numpy as np
import pytest

import graph_checks as gc
import oracle
import synth

pytestmark = pytest.mark.usefixtures("built_libs")


def _golden_decode(name):
    cfg, _, _, tasks, events = gc.load_golden(name)
    w = synth.Workload("golden", cfg["layers"], cfg["hidden"], cfg["q_heads"], cfg["kv_heads"],
                       cfg["head_dim"], cfg["ffn"], cfg["vocab"], 0, cfg["batch"], 1)
    g = oracle.tgraph_decode(w, cfg["kv_capacity"], cfg["workers"], cfg["col_align"],
                             cfg["apw"], cfg["min_chunk"], attn_jit=cfg.get("jit", 0))
    return g, tasks, events


@pytest.mark.parametrize("name", ["tgraph_tiny1_w2_s1.txt", "tgraph_tiny1_w2_s4.txt",
                                  "tgraph_tiny1_w2_b2_jit.txt"])
def test_decode_graph_matches_hand_derived_tables(name):
    g, tasks, events = _golden_decode(name)
    gc.assert_tables_equal(g, tasks, events)


@pytest.mark.parametrize("name", ["tgraph_norm_dep.txt", "tgraph_norm_trig.txt"])
def test_normalisation_matches_hand_derived_tables(name):
    _, nodes, edges, tasks, events = gc.load_golden(name)
    index = {n[0]: i for i, n in enumerate(nodes)}
    g = oracle.tgraph_from_edges([n[1] for n in nodes], [n[2] for n in nodes],
                                 [(index[a], index[b]) for a, b in edges])
    gc.assert_tables_equal(g, tasks, events)


CONFIGS = [(synth.TINY, 148), (synth.TINY, 1), (synth.TINY, 2), (synth.TINY, 7),
           (synth.Q06B, 148), (synth.Q06B, 7), (synth.Q8B, 148), (synth.Q8B, 2),
           (synth.Q8B_B8, 148), (synth.Q8B_B16, 148)]


@pytest.mark.parametrize("w,W", CONFIGS, ids=[f"{w.name}-W{W}" for w, W in CONFIGS])
def test_decode_graph_invariants_counts_and_semantics(w, W):
    cap = w.kv_capacity(0)
    g = oracle.tgraph_decode(w, cap, W)
    gc.check_invariants(g)
    assert (g.task_type != gc.EMPTY).all()  # group-aligned QKV tiles need no empty tasks
    assert (g.task_type >= 1).all() and (g.task_type <= 9).all()
    tasks, events = gc.closed_form_counts(w, cap, W)
    assert (g.n_tasks, g.n_events) == (tasks, events)
    gc.simulate_random(g, seed=W)
    gc.simulate_static_queues(g, W)


def test_qwen3_8b_bs1_graph_size():
    # 36 layers x (QKV 128 + ATTN 136 + O 128 + GATE_UP 128 + DOWN 128)
    # + EMBED + LM_HEAD 147 + ARGMAX on 148 workers; 36 x 12 + 2 events.
    g = oracle.tgraph_decode(synth.Q8B, synth.Q8B.kv_capacity(0), 148)
    assert g.n_tasks == 23477 and g.n_events == 434
    assert (g.qkv_rows, g.o_rows, g.gu_rows, g.down_rows, g.lm_rows) == (48, 32, 96, 32, 1040)
    assert (g.splits, g.chunk) == (17, 64)


@pytest.mark.parametrize("seed", range(40))
def test_random_dags(seed):
    op, idx, edges = gc.random_dag(seed)
    g = oracle.tgraph_from_edges(op, idx, edges)
    gc.check_invariants(g)
    gc.simulate_random(g, seed)
    gc.simulate_static_queues(g, 1 + seed % 5)
    assert g.edge_src.size == len(set(edges))


def test_random_dags_exercise_normalisation():
    empties = 0
    for seed in range(40):
        op, idx, edges = gc.random_dag(seed)
        empties += int((oracle.tgraph_from_edges(op, idx, edges).task_type == gc.EMPTY).sum())
    assert empties > 0


def test_build_is_deterministic_and_input_order_free():
    op, idx, edges = gc.random_dag(123)
    a = oracle.tgraph_from_edges(op, idx, edges)
    perm = np.random.default_rng(0).permutation(len(op))
    inv = np.argsort(perm)
    b = oracle.tgraph_from_edges([op[p] for p in perm], [idx[p] for p in perm],
                                 [(int(inv[x]), int(inv[y])) for x, y in edges])
    gc.assert_graphs_equal(a, b)
    w = synth.Q06B
    gc.assert_graphs_equal(oracle.tgraph_decode(w, 576, 148), oracle.tgraph_decode(w, 576, 148))


def test_rejects_backward_edges():
    with pytest.raises(ValueError):
        oracle.tgraph_from_edges([0, 1], [0, 0], [(1, 0)])
