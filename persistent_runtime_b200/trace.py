"""Per-task trace of the persistent kernel (see mk_set_trace in include/mk.h).

Each task writes {wait begin, ready, end, (smid << 32) | worker} in %globaltimer
nanoseconds.  `summarize` reports where worker time goes (waiting on events vs.
running task bodies) per task type; `to_chrome` writes the Chrome trace-event
JSON format (one row per worker) for chrome://tracing or Perfetto.
"""
from __future__ import annotations

import json

import numpy as np

from . import TASK_NAMES


def _fields(trace: np.ndarray):
    t = np.asarray(trace, dtype=np.uint64).reshape(-1, 4)
    wait0 = t[:, 0].astype(np.int64)
    ready = t[:, 1].astype(np.int64)
    end = t[:, 2].astype(np.int64)
    worker = (t[:, 3] & np.uint64(0xFFFFFFFF)).astype(np.int64)
    smid = (t[:, 3] >> np.uint64(32)).astype(np.int64)
    return wait0, ready, end, worker, smid


def summarize(trace: np.ndarray, graph) -> dict:
    """Wait / busy split of one traced step (all times in microseconds)."""
    wait0, ready, end, worker, _ = _fields(trace)
    ran = end > 0
    origin = int(wait0[ran].min())
    span = (int(end[ran].max()) - origin) / 1e3
    n_workers = int(worker[ran].max()) + 1
    wait = (ready - wait0)[ran] / 1e3
    body = (end - ready)[ran] / 1e3
    # gaps between a task's end and the next task's wait begin on the same worker
    per_type = {}
    types = np.asarray(graph.task_type)[ran]
    for ty in np.unique(types):
        sel = types == ty
        per_type[TASK_NAMES.get(int(ty), str(ty))] = {
            "tasks": int(sel.sum()), "body_us_mean": float(body[sel].mean()),
            "body_us_max": float(body[sel].max()), "wait_us_mean": float(wait[sel].mean()),
            "wait_us_total": float(wait[sel].sum()), "body_us_total": float(body[sel].sum())}
    # per-operator critical path: first ready to last end
    ops = np.asarray(graph.task_op)[ran]
    r, e = ready[ran], end[ran]
    op_spans = []
    for o in np.unique(ops):
        sel = ops == o
        op_spans.append((int(o), (int(r[sel].min()) - origin) / 1e3, (int(e[sel].max()) - origin) / 1e3))
    return {"span_us": span, "workers": n_workers,
            "event_wait_frac": float(wait.sum() / (n_workers * span)),
            "busy_frac": float(body.sum() / (n_workers * span)),
            "per_type": per_type, "op_spans": op_spans}


def to_chrome(trace: np.ndarray, graph, path: str) -> None:
    wait0, ready, end, worker, smid = _fields(trace)
    ran = end > 0
    origin = int(wait0[ran].min())
    ev = []
    for i in np.nonzero(ran)[0]:
        name = TASK_NAMES.get(int(graph.task_type[i]), "?")
        if ready[i] > wait0[i]:
            ev.append({"name": "wait", "ph": "X", "ts": (wait0[i] - origin) / 1e3,
                       "dur": (ready[i] - wait0[i]) / 1e3, "pid": 0, "tid": int(worker[i]),
                       "args": {"task": int(i), "event": int(graph.task_dep[i])}})
        ev.append({"name": name, "ph": "X", "ts": (ready[i] - origin) / 1e3,
                   "dur": (end[i] - ready[i]) / 1e3, "pid": 0, "tid": int(worker[i]),
                   "args": {"task": int(i), "layer": int(graph.task_layer[i]),
                            "idx": int(graph.task_idx[i]), "sm": int(smid[i])}})
    with open(path, "w") as f:
        json.dump({"traceEvents": ev, "displayTimeUnit": "ns"}, f)
