"""Per-task trace of the persistent kernel (see mk_set_trace in include/mk.h).

Each task writes eight words: {wait begin, ready, end, (smid << 32) | worker,
prologue done, streaming done, L2 prefetch bytes so far, first ring stage
available} in %globaltimer nanoseconds (the phase marks are 0 for tasks
without those phases).  `summarize` reports where
worker time goes (waiting on events vs. prologue / streaming / epilogue of the
task bodies) per task type; `to_chrome` writes the Chrome trace-event JSON
format (one row per worker) for chrome://tracing or Perfetto.
"""
from __future__ import annotations

import json

import numpy as np

from . import TASK_NAMES

WORDS = 8


def _fields(trace: np.ndarray):
    t = np.asarray(trace, dtype=np.uint64).reshape(-1, WORDS).astype(np.int64)
    wait0, ready, end = t[:, 0], t[:, 1], t[:, 2]
    worker = t[:, 3] & 0xFFFFFFFF
    smid = t[:, 3] >> 32
    pro, loop = t[:, 4], t[:, 5]
    return wait0, ready, end, worker, smid, pro, loop, t[:, 7]


def summarize(trace: np.ndarray, graph) -> dict:
    """Wait / busy split of one traced step (all times in microseconds)."""
    wait0, ready, end, worker, _, pro, loop, first = _fields(trace)
    ran = end > 0
    origin = int(wait0[ran].min())
    span = (int(end[ran].max()) - origin) / 1e3
    n_workers = int(worker[ran].max()) + 1
    wait = (ready - wait0)[ran] / 1e3
    body = (end - ready)[ran] / 1e3
    has = ran & (pro > 0) & (loop > 0)
    per_type = {}
    types = np.asarray(graph.task_type)
    for ty in np.unique(types[ran]):
        sel = ran & (types == ty)
        selh = has & (types == ty)
        ent = {"tasks": int(sel.sum()), "body_us_mean": float(((end - ready)[sel] / 1e3).mean()),
               "body_us_max": float(((end - ready)[sel] / 1e3).max()),
               "wait_us_mean": float(((ready - wait0)[sel] / 1e3).mean()),
               "wait_us_total": float(((ready - wait0)[sel] / 1e3).sum()),
               "body_us_total": float(((end - ready)[sel] / 1e3).sum())}
        if selh.any():
            ent["prologue_us_mean"] = float(((pro - ready)[selh] / 1e3).mean())
            ent["stream_us_mean"] = float(((loop - pro)[selh] / 1e3).mean())
            ent["epilogue_us_mean"] = float(((end - loop)[selh] / 1e3).mean())
        self_ = sel & (first > 0) & (pro > 0)
        if self_.any():
            # > 0: the first ring stage arrived after the prologue (HBM wait)
            ent["first_stage_after_prologue_us_mean"] = float(
                (np.maximum(first - pro, 0)[self_] / 1e3).mean())
        per_type[TASK_NAMES.get(int(ty), str(ty))] = ent
    ops = np.asarray(graph.task_op)[ran]
    r, e = ready[ran], end[ran]
    op_spans = []
    for o in np.unique(ops):
        sel = ops == o
        op_spans.append((int(o), (int(r[sel].min()) - origin) / 1e3,
                         (int(e[sel].max()) - origin) / 1e3))
    pf = np.asarray(trace, dtype=np.uint64).reshape(-1, WORDS)[:, 6].astype(np.int64)
    pf_total = 0
    for w in np.unique(worker[ran]):
        pf_total += int(pf[ran & (worker == w)].max())
    return {"span_us": span, "workers": n_workers, "l2_prefetch_bytes_total": pf_total,
            "event_wait_frac": float(wait.sum() / (n_workers * span)),
            "busy_frac": float(body.sum() / (n_workers * span)),
            "per_type": per_type, "op_spans": op_spans,
            "layer_phases": layer_phases(trace, graph)}


def layer_phases(trace: np.ndarray, graph) -> dict | None:
    """Mean over decoder layers of where a layer's time goes on the critical
    path (microseconds): each projection from its first task becoming ready to
    its last task ending, and the attention window from the last QKV task's
    end to the first O task's start, in which only K/V rows, attention
    partials and L2 prefetches move.  `layer_us` runs from one layer's first
    QKV start to the next one's."""
    wait0, ready, end, *_ = _fields(trace)
    ran = end > 0
    types, layers = np.asarray(graph.task_type), np.asarray(graph.task_layer)
    spans = {}
    for ty in (2, 3, 5, 6, 7):
        for ly in np.unique(layers[ran & (types == ty)]):
            sel = ran & (types == ty) & (layers == ly)
            spans[(ty, int(ly))] = (int(ready[sel].min()), int(end[sel].max()))
    lys = sorted(ly for ty, ly in spans if ty == 2)
    rows = []
    for ly in lys:
        if not all((ty, ly) in spans for ty in (2, 3, 5, 6, 7)):
            return None
        q, a, o, g, d = (spans[(ty, ly)] for ty in (2, 3, 5, 6, 7))
        nxt = spans.get((2, ly + 1))
        rows.append([q[1] - q[0], o[0] - q[1], a[1] - a[0], o[1] - o[0], g[1] - g[0], d[1] - d[0],
                     (nxt[0] - q[0]) if nxt else np.nan])
    if not rows:
        return None
    m = np.nanmean(np.asarray(rows, dtype=np.float64), axis=0) / 1e3
    keys = ("qkv_us", "attn_window_us", "attn_tasks_us", "o_us", "gateup_us", "down_us", "layer_us")
    return {"layers": len(rows), **{k: float(v) for k, v in zip(keys, m)}}


def to_chrome(trace: np.ndarray, graph, path: str) -> None:
    wait0, ready, end, worker, smid, pro, loop, first = _fields(trace)
    ran = end > 0
    origin = int(wait0[ran].min())
    ev = []
    for i in np.nonzero(ran)[0]:
        name = TASK_NAMES.get(int(graph.task_type[i]), "?")
        tid = int(worker[i])
        if ready[i] > wait0[i]:
            ev.append({"name": "wait", "ph": "X", "ts": (wait0[i] - origin) / 1e3,
                       "dur": (ready[i] - wait0[i]) / 1e3, "pid": 0, "tid": tid,
                       "args": {"task": int(i), "event": int(graph.task_dep[i])}})
        ev.append({"name": name, "ph": "X", "ts": (ready[i] - origin) / 1e3,
                   "dur": (end[i] - ready[i]) / 1e3, "pid": 0, "tid": tid,
                   "args": {"task": int(i), "layer": int(graph.task_layer[i]),
                            "idx": int(graph.task_idx[i]), "sm": int(smid[i]),
                            "prologue_us": float((pro[i] - ready[i]) / 1e3) if pro[i] else None,
                            "stream_us": float((loop[i] - pro[i]) / 1e3) if loop[i] else None,
                            "first_stage_us": float((first[i] - ready[i]) / 1e3) if first[i] else None}})
    with open(path, "w") as f:
        json.dump({"traceEvents": ev, "displayTimeUnit": "ns"}, f)
