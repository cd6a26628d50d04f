"""The library's host graph builder against the oracle's independent builder:
bit-exact tables on every workload, hand-derived goldens and random graphs."""
import numpy as np
import pytest

import graph_checks as gc
import oracle
import persistent_runtime_b200 as prb
import synth

pytestmark = pytest.mark.usefixtures("built_libs")

CONFIGS = [(synth.TINY, 148), (synth.TINY, 1), (synth.TINY, 2), (synth.TINY, 7),
           (synth.Q06B, 148), (synth.Q06B, 132), (synth.Q8B, 148), (synth.Q8B, 3),
           (synth.Q8B_B8, 148), (synth.Q8B_B16, 148)]


def default_col_align(w):
    # the library's default tile alignment: 4 rows at batch 1 (every SM gets a
    # tile of the row operators), 16 for the tensor-core path of batch >= 2;
    # its default attention tasks per worker is 1
    return 4 if w.batch == 1 else 16


def default_jit(w):
    # JIT attention is opt-in: the library's default fixes the splits at build time
    return 0


@pytest.mark.parametrize("w,W", CONFIGS, ids=[f"{w.name}-W{W}" for w, W in CONFIGS])
@pytest.mark.parametrize("align", [16, None, "aot"], ids=["align16", "default", "jit"])
def test_decode_graph_bit_exact_with_oracle(w, W, align):
    cap = w.kv_capacity(0)
    if align is None:  # the library's defaults against the oracle with the same values
        mine = prb.plan_graph(w, cap, W)
        ref = oracle.tgraph_decode(w, cap, W, default_col_align(w), 1, 64, default_jit(w))
    elif align == "aot":  # JIT attention where the batch allows it (batch >= 2)
        jit = int(w.batch > 1)
        mine = prb.plan_graph(w, cap, W, attn_jit=1 if jit else 0)
        ref = oracle.tgraph_decode(w, cap, W, default_col_align(w), 1, 64, jit)
    else:
        mine = prb.plan_graph(w, cap, W, col_align=align, attn_tasks_per_worker=4)
        ref = oracle.tgraph_decode(w, cap, W, align, 4, 64, default_jit(w))
    gc.assert_graphs_equal(mine, ref)
    np.testing.assert_array_equal(mine.edge_src, ref.edge_src)
    np.testing.assert_array_equal(mine.edge_dst, ref.edge_dst)
    assert mine.tiling == (ref.qkv_rows, ref.o_rows, ref.gu_rows, ref.down_rows, ref.lm_rows,
                           ref.splits, ref.chunk)
    gc.check_invariants(mine)


@pytest.mark.parametrize("col_align,apw,min_chunk", [(8, 4, 64), (4, 2, 128), (32, 8, 64)])
def test_tuning_variants_bit_exact(col_align, apw, min_chunk):
    w = synth.Q8B_B8
    cap = w.kv_capacity(3)
    for jit in (-1, 1):
        mine = prb.plan_graph(w, cap, 148, col_align=col_align, attn_tasks_per_worker=apw,
                              attn_min_chunk=min_chunk, attn_jit=jit)
        ref = oracle.tgraph_decode(w, cap, 148, col_align, apw, min_chunk, int(jit > 0))
        gc.assert_graphs_equal(mine, ref)


@pytest.mark.parametrize("name", ["tgraph_tiny1_w2_s1.txt", "tgraph_tiny1_w2_s4.txt",
                                  "tgraph_tiny1_w2_b2_jit.txt"])
def test_decode_goldens(name):
    cfg, _, _, tasks, events = gc.load_golden(name)
    w = synth.Workload("golden", cfg["layers"], cfg["hidden"], cfg["q_heads"], cfg["kv_heads"],
                       cfg["head_dim"], cfg["ffn"], cfg["vocab"], 0, cfg["batch"], 1)
    g = prb.plan_graph(w, cfg["kv_capacity"], cfg["workers"], col_align=cfg["col_align"],
                       attn_tasks_per_worker=cfg["apw"], attn_min_chunk=cfg["min_chunk"],
                       attn_jit=cfg.get("jit", 0))
    gc.assert_tables_equal(g, tasks, events)
    if cfg.get("jit", 0):
        assert g.tiling[5] == 3 and g.tiling[6] == 0  # S slots per pair, chunk set per step


@pytest.mark.parametrize("name", ["tgraph_norm_dep.txt", "tgraph_norm_trig.txt"])
def test_normalisation_goldens(name):
    _, nodes, edges, tasks, events = gc.load_golden(name)
    index = {n[0]: i for i, n in enumerate(nodes)}
    g = prb.graph_from_edges([n[1] for n in nodes], [n[2] for n in nodes],
                             [(index[a], index[b]) for a, b in edges])
    gc.assert_tables_equal(g, tasks, events)


@pytest.mark.parametrize("seed", range(60))
def test_random_dags_bit_exact(seed):
    op, idx, edges = gc.random_dag(seed, n_ops=(3, 10), per_op=(1, 7))
    mine = prb.graph_from_edges(op, idx, edges)
    ref = oracle.tgraph_from_edges(op, idx, edges)
    gc.assert_graphs_equal(mine, ref)
    gc.check_invariants(mine)
    gc.simulate_random(mine, seed)
