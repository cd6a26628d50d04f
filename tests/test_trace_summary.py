"""The per-task trace summary (persistent_runtime_b200/trace.py) on a trace
written by hand for a host-only graph: every figure it reports follows from
the planted timestamps (no device)."""
import json

import numpy as np
import pytest

import persistent_runtime_b200 as prb
import persistent_runtime_b200.trace as mktrace
import synth

# planted schedule of one layer (ns from the layer's start): (ready, end) per task type
PHASES = {2: (0, 10_000), 3: (11_000, 18_000), 5: (20_000, 26_000), 6: (26_500, 50_000),
          7: (50_200, 64_000)}
LAYER_NS = 65_000
WAIT_NS = 500


@pytest.fixture(scope="module")
def planted():
    w = synth.TINY
    g = prb.plan_graph(w, 64, 4)
    types, layers = np.asarray(g.task_type), np.asarray(g.task_layer)
    n = len(types)
    words = np.zeros((n, mktrace.WORDS), dtype=np.uint64)
    t0 = 1_000_000
    for i in range(n):
        ty, ly = int(types[i]), int(layers[i])
        if ty in PHASES:
            r, e = PHASES[ty]
            ready, end = t0 + ly * LAYER_NS + r, t0 + ly * LAYER_NS + e
        elif ty == 1:  # EMBED before layer 0
            ready, end = t0 - 5_000, t0 - 1_000
        else:  # LM head and argmax after the last layer
            ready, end = t0 + w.n_layers * LAYER_NS, t0 + w.n_layers * LAYER_NS + 4_000
        words[i] = [ready - WAIT_NS, ready, end, (7 << 32) | (i % 4), ready + 100, end - 100,
                    0, ready + 150]
    return w, g, words


def test_layer_phases_follow_the_planted_schedule(planted):
    w, g, words = planted
    ph = mktrace.layer_phases(words.reshape(-1), g)
    assert ph["layers"] == w.n_layers
    assert ph["qkv_us"] == pytest.approx(10.0)
    assert ph["attn_window_us"] == pytest.approx(10.0)  # last QKV end -> first O ready
    assert ph["attn_tasks_us"] == pytest.approx(7.0)
    assert ph["o_us"] == pytest.approx(6.0)
    assert ph["gateup_us"] == pytest.approx(23.5)
    assert ph["down_us"] == pytest.approx(13.8)
    assert ph["layer_us"] == pytest.approx(65.0)  # only layers with a successor count


def test_summary_wait_and_busy_fractions(planted, tmp_path):
    _, g, words = planted
    s = mktrace.summarize(words.reshape(-1), g)
    ran = words[:, 2] > 0
    span = (int(words[ran, 2].max()) - int(words[ran, 0].min())) / 1e3
    assert s["span_us"] == pytest.approx(span)
    assert s["workers"] == 4
    n = int(ran.sum())
    assert s["event_wait_frac"] == pytest.approx(n * WAIT_NS / 1e3 / (4 * span))
    body = ((words[:, 2].astype(np.int64) - words[:, 1].astype(np.int64)) / 1e3).sum()
    assert s["busy_frac"] == pytest.approx(body / (4 * span))
    assert s["per_type"]["QKV"]["prologue_us_mean"] == pytest.approx(0.1)
    assert s["per_type"]["QKV"]["epilogue_us_mean"] == pytest.approx(0.1)
    assert s["per_type"]["QKV"]["first_stage_after_prologue_us_mean"] == pytest.approx(0.05)
    out = tmp_path / "t.json"
    mktrace.to_chrome(words.reshape(-1), g, str(out))
    ev = json.load(open(out))["traceEvents"]
    assert sum(1 for e in ev if e["name"] == "wait") == n
