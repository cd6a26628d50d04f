"""CPU oracle for the decode step and its task graph.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` leg of ``bench.py`` may import this package.  The GPU library
(``persistent_runtime_b200``) never imports it, and it never imports the GPU
library: the two share no code.  Both are fed the same host buffers from the
seeded generator in ``synth``.

``oracle_step.cpp`` is the plain single-threaded fp32 decode step;
``oracle_tgraph.cpp`` is an independent, plain implementation of the task-graph
construction (tiling, raw events, fusion, reduction, normalisation, BFS).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmk_oracle.so")
_SOURCES = ["oracle_step.cpp", "oracle_tgraph.cpp"]
_lib = None


def build(verbose: bool = False) -> str:
    """Compile the oracle with g++ (-O2, no fp contraction so sums stay in order)."""
    srcs = [os.path.join(_HERE, s) for s in _SOURCES]
    cmd = ["g++", "-std=c++17", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", *srcs, "-o", _LIB_PATH]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    return _LIB_PATH


class OracleCfg(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("ffn", ctypes.c_int32),
                ("vocab", ctypes.c_int32), ("tied", ctypes.c_int32),
                ("eps", ctypes.c_float), ("pad0", ctypes.c_int32),
                ("theta", ctypes.c_double), ("batch", ctypes.c_int32),
                ("kv_capacity", ctypes.c_int32)]


_P16 = ctypes.POINTER(ctypes.c_uint16)


class OracleLayer(ctypes.Structure):
    _fields_ = [(n, _P16) for n in ("attn_norm", "wq", "wk", "wv", "q_norm", "k_norm", "wo",
                                    "mlp_norm", "w_gate", "w_up", "w_down")]


class OracleWeights(ctypes.Structure):
    _fields_ = [("embed", _P16), ("lm_head", _P16), ("final_norm", _P16),
                ("layers", ctypes.POINTER(OracleLayer))]


def _load():
    global _lib
    if _lib is not None:
        return _lib
    srcs = [os.path.join(_HERE, s) for s in _SOURCES]
    if not os.path.exists(_LIB_PATH) or any(
            os.path.getmtime(s) > os.path.getmtime(_LIB_PATH) for s in srcs):
        build()
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    lib.oracle_rmsnorm.argtypes = [vp, vp, ctypes.c_int, f32, vp]
    lib.oracle_gemv.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, vp]
    lib.oracle_rope.argtypes = [vp, ctypes.c_int, ctypes.c_int, ctypes.c_double]
    lib.oracle_silu.argtypes = [f32]
    lib.oracle_silu.restype = f32
    lib.oracle_attention.argtypes = [vp, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp]
    lib.oracle_argmax.argtypes = [vp, ctypes.c_int]
    lib.oracle_argmax.restype = i32
    lib.oracle_round_bf16.argtypes = [f32]
    lib.oracle_round_bf16.restype = ctypes.c_uint16
    lib.oracle_decode_step_ex.argtypes = [ctypes.POINTER(OracleCfg), ctypes.POINTER(OracleWeights),
                                          vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int,
                                          ctypes.c_int]
    lib.oracle_decode_step_ex.restype = ctypes.c_int
    lib.oracle_tgraph_decode.argtypes = [ctypes.POINTER(OracleCfg), ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.POINTER(vp)]
    lib.oracle_tgraph_decode.restype = ctypes.c_int
    lib.oracle_tgraph_from_edges.argtypes = [ctypes.c_int, vp, vp, ctypes.c_int, vp, vp,
                                             ctypes.POINTER(vp)]
    lib.oracle_tgraph_from_edges.restype = ctypes.c_int
    lib.oracle_tgraph_sizes.argtypes = [vp, vp, vp, vp]
    lib.oracle_tgraph_tiling.argtypes = [vp, vp]
    lib.oracle_tgraph_tasks.argtypes = [vp] * 7
    lib.oracle_tgraph_events.argtypes = [vp] * 4
    lib.oracle_tgraph_edges.argtypes = [vp] * 3
    lib.oracle_tgraph_free.argtypes = [vp]
    _lib = lib
    return lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


# --------------------------------------------------------------------------
# Building blocks (exposed so tests can pin each one separately)
# --------------------------------------------------------------------------
def rmsnorm(x, gain_bf16, eps: float) -> np.ndarray:
    x = _f32(x)
    g = np.ascontiguousarray(gain_bf16, dtype=np.uint16)
    out = np.empty_like(x)
    _load().oracle_rmsnorm(_ptr(x), _ptr(g), x.size, eps, _ptr(out))
    return out


def gemv(w_bf16, x) -> np.ndarray:
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    x = _f32(x)
    y = np.empty(w.shape[0], dtype=np.float32)
    _load().oracle_gemv(_ptr(w), w.shape[0], w.shape[1], _ptr(x), _ptr(y))
    return y


def rope(v, pos: int, theta: float) -> np.ndarray:
    out = _f32(v).copy()
    _load().oracle_rope(_ptr(out), out.size, pos, theta)
    return out


def silu(x: float) -> float:
    return float(_load().oracle_silu(x))


def attention(q, k_bf16, v_bf16, want_probs: bool = False):
    """q: [nh][D] fp32; k, v: [n_pos][D] bf16 bits.  Returns out [nh][D] (and probs)."""
    q = _f32(q)
    k = np.ascontiguousarray(k_bf16, dtype=np.uint16)
    v = np.ascontiguousarray(v_bf16, dtype=np.uint16)
    nh, d = q.shape
    n_pos = k.shape[0]
    out = np.empty((nh, d), dtype=np.float32)
    probs = np.empty((nh, n_pos), dtype=np.float32) if want_probs else None
    _load().oracle_attention(_ptr(q), _ptr(k), _ptr(v), n_pos, nh, d, _ptr(out), _ptr(probs))
    return (out, probs) if want_probs else out


def argmax(v) -> int:
    v = _f32(v)
    return int(_load().oracle_argmax(_ptr(v), v.size))


def round_bf16(x: float) -> int:
    return int(_load().oracle_round_bf16(x))


# --------------------------------------------------------------------------
# Whole decode step
# --------------------------------------------------------------------------
def make_cfg(w, kv_capacity: int) -> OracleCfg:
    return OracleCfg(w.n_layers, w.hidden, w.n_q_heads, w.n_kv_heads, w.head_dim, w.ffn,
                     w.vocab, int(w.tied_embeddings), w.rms_eps, 0, w.rope_theta, w.batch,
                     kv_capacity)


class Model:
    """Holds ctypes views of host weight arrays (arrays must outlive the model)."""

    def __init__(self, workload, weights: dict, kv_capacity: int):
        self.w = workload
        self.cfg = make_cfg(workload, kv_capacity)
        self._keep = []
        layers = (OracleLayer * workload.n_layers)()
        for l, lw in enumerate(weights["layers"]):
            for name, _ in OracleLayer._fields_:
                arr = np.ascontiguousarray(lw[name], dtype=np.uint16)
                self._keep.append(arr)
                setattr(layers[l], name, arr.ctypes.data_as(_P16))
        self._layers = layers

        def p(a):
            if a is None:
                return _P16()
            a = np.ascontiguousarray(a, dtype=np.uint16)
            self._keep.append(a)
            return a.ctypes.data_as(_P16)

        self.weights = OracleWeights(p(weights["embed"]), p(weights["lm_head"]),
                                     p(weights["final_norm"]), layers)

    def step(self, tokens_in, kv_len, k_cache, v_cache, want_logits=True, want_hidden=True,
             seq_mask=None, layers_run: int = -1, vocab_run: int = -1):
        """Runs one decode step in place on kv_len / caches.  Returns dict of outputs."""
        w = self.w
        tokens_in = np.ascontiguousarray(tokens_in, dtype=np.int32)
        tokens_out = np.zeros(w.batch, dtype=np.int32)
        assert kv_len.dtype == np.int32 and kv_len.flags.c_contiguous
        assert k_cache.dtype == np.uint16 and k_cache.flags.c_contiguous
        assert v_cache.dtype == np.uint16 and v_cache.flags.c_contiguous
        logits = np.zeros((w.batch, w.vocab), dtype=np.float32) if want_logits else None
        hidden = np.zeros((w.batch, w.hidden), dtype=np.float32) if want_hidden else None
        mask = None if seq_mask is None else np.ascontiguousarray(seq_mask, dtype=np.uint8)
        rc = _load().oracle_decode_step_ex(ctypes.byref(self.cfg), ctypes.byref(self.weights),
                                           _ptr(tokens_in), _ptr(tokens_out), _ptr(kv_len),
                                           _ptr(k_cache), _ptr(v_cache), _ptr(logits),
                                           _ptr(hidden), _ptr(mask), layers_run, vocab_run)
        if rc != 0:
            raise ValueError("oracle_decode_step rejected the inputs (kv_len or token range)")
        return {"tokens": tokens_out, "logits": logits, "hidden": hidden}


# --------------------------------------------------------------------------
# Task graph
# --------------------------------------------------------------------------
class TGraph:
    """Host tables of a built graph: tasks in linear order, events by id."""

    def __init__(self, handle):
        lib = _load()
        nt, ne, ned = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        lib.oracle_tgraph_sizes(handle, ctypes.byref(nt), ctypes.byref(ne), ctypes.byref(ned))
        nt, ne, ned = nt.value, ne.value, ned.value
        cols = [np.empty(nt, dtype=np.int32) for _ in range(6)]
        lib.oracle_tgraph_tasks(handle, *[_ptr(c) for c in cols])
        self.task_type, self.task_op, self.task_layer, self.task_idx, self.task_dep, \
            self.task_trig = cols
        ev = [np.empty(ne, dtype=np.int32) for _ in range(3)]
        lib.oracle_tgraph_events(handle, *[_ptr(c) for c in ev])
        self.event_count, self.event_first, self.event_last = ev
        ed = [np.empty(ned, dtype=np.int32) for _ in range(2)]
        lib.oracle_tgraph_edges(handle, *[_ptr(c) for c in ed])
        self.edge_src, self.edge_dst = ed
        til = np.empty(7, dtype=np.int32)
        lib.oracle_tgraph_tiling(handle, _ptr(til))
        (self.qkv_rows, self.o_rows, self.gu_rows, self.down_rows, self.lm_rows, self.splits,
         self.chunk) = [int(x) for x in til]
        lib.oracle_tgraph_free(handle)

    @property
    def n_tasks(self) -> int:
        return int(self.task_type.size)

    @property
    def n_events(self) -> int:
        return int(self.event_count.size)


def tgraph_decode(workload, kv_capacity: int, num_workers: int, col_align: int = 16,
                  attn_tasks_per_worker: int = 4, attn_min_chunk: int = 64,
                  attn_jit: int = 0) -> TGraph:
    cfg = make_cfg(workload, kv_capacity)
    h = ctypes.c_void_p()
    rc = _load().oracle_tgraph_decode(ctypes.byref(cfg), num_workers, col_align,
                                      attn_tasks_per_worker, attn_min_chunk, int(attn_jit),
                                      ctypes.byref(h))
    if rc != 0:
        raise ValueError(f"oracle_tgraph_decode failed ({rc})")
    return TGraph(h)


def tgraph_from_edges(task_op, task_idx, edges) -> TGraph:
    op = np.ascontiguousarray(task_op, dtype=np.int32)
    idx = np.ascontiguousarray(task_idx, dtype=np.int32)
    e = np.asarray(edges, dtype=np.int32).reshape(-1, 2)
    src = np.ascontiguousarray(e[:, 0])
    dst = np.ascontiguousarray(e[:, 1])
    h = ctypes.c_void_p()
    rc = _load().oracle_tgraph_from_edges(op.size, _ptr(op), _ptr(idx), src.size, _ptr(src),
                                          _ptr(dst), ctypes.byref(h))
    if rc != 0:
        raise ValueError(f"oracle_tgraph_from_edges failed ({rc})")
    return TGraph(h)
