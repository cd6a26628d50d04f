"""Python binding of libmk.so, the decode-step megakernel (C ABI in include/mk.h).

Argument marshalling only: every step of the decode path runs in the library's
CUDA kernels.  torch is used for device memory and streams.  If libmk.so is
missing the import of the binding fails loudly: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmk.so")

MK_OK, MK_ERR_ARG, MK_ERR_CUDA, MK_ERR_OOM, MK_ERR_GRAPH = 0, -1, -2, -3, -4
MK_ERR_NOT_LOADED, MK_ERR_TIMEOUT, MK_ERR_DEVICE = -5, -6, -7
TASK_NAMES = {0: "GENERIC", 1: "EMBED", 2: "QKV", 3: "ATTN", 4: "MERGE", 5: "OPROJ",
              6: "GATEUP", 7: "DOWN", 8: "LMHEAD", 9: "ARGMAX", 10: "EMPTY"}

# Every symbol declared in include/mk.h.
EXPORTS = ("mk_plan_graph", "mk_graph_from_edges", "mk_build_graph", "mk_load_weights",
           "mk_decode_step", "mk_decode_steps", "mk_decode_steps_paged", "mk_decode_step_perop",
           "mk_decode_step_noalloc",
           "mk_sync_status", "mk_reset",
           "mk_graph_export", "mk_get_info", "mk_final_hidden", "mk_debug_set_event_count",
           "mk_set_trace", "mk_set_timeout_us", "mk_last_error", "mk_destroy")


class MkError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"mk status {status}: {msg}")
        self.status = status


class ModelConfig(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("hidden", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("ffn", ctypes.c_int),
                ("vocab", ctypes.c_int), ("tied_embeddings", ctypes.c_int),
                ("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_double),
                ("batch", ctypes.c_int), ("kv_capacity", ctypes.c_int)]


class Tuning(ctypes.Structure):
    _fields_ = [("num_workers", ctypes.c_int), ("col_align", ctypes.c_int),
                ("attn_tasks_per_worker", ctypes.c_int), ("attn_min_chunk", ctypes.c_int),
                ("ring_stages", ctypes.c_int),
                ("ring_stage_bytes", ctypes.c_int), ("l2_prefetch_bytes", ctypes.c_int),
                ("wait_timeout_us", ctypes.c_uint), ("kv_page_size", ctypes.c_int),
                ("l2_stream_policy", ctypes.c_int), ("attn_jit", ctypes.c_int),
                ("dispatch", ctypes.c_int)]


_PP = ctypes.POINTER(ctypes.c_void_p)


class Weights(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("final_norm", ctypes.c_void_p),
                ("lm_head", ctypes.c_void_p)] + [
        (n, _PP) for n in ("attn_norm", "wq", "wk", "wv", "q_norm", "k_norm", "wo", "mlp_norm",
                           "w_gate", "w_up", "w_down")]


_I32P = ctypes.POINTER(ctypes.c_int32)


class GraphView(ctypes.Structure):
    _fields_ = [("n_tasks", ctypes.c_int32), ("n_events", ctypes.c_int32),
                ("n_edges", ctypes.c_int32), ("num_workers", ctypes.c_int32)] + [
        (n, _I32P) for n in ("task_type", "task_op", "task_layer", "task_idx", "task_dep",
                             "task_trig", "event_count", "event_first", "event_last",
                             "edge_src", "edge_dst")] + [
        (n, ctypes.c_int32) for n in ("qkv_rows", "o_rows", "gu_rows", "down_rows", "lm_rows",
                                      "attn_splits", "attn_chunk")] + [
        ("mma_mb", ctypes.c_int32 * 5), ("mma_kcb", ctypes.c_int32 * 5)]


class Info(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("device", "num_workers", "n_tasks", "n_events",
                                               "n_ops", "smem_bytes", "ring_stages",
                                               "ring_stage_bytes")] + [
        ("weight_bytes", ctypes.c_int64), ("act_bytes", ctypes.c_int64)]


_lib = None


def lib():
    """The loaded libmk.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: run `python -m persistent_runtime_b200.build`"
                          " (there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_int
    H = ctypes.POINTER(vp)
    sig = {
        "mk_plan_graph": ([ctypes.POINTER(ModelConfig), ctypes.POINTER(Tuning), i32, H], st),
        "mk_graph_from_edges": ([i32, vp, vp, i32, vp, vp, H], st),
        "mk_build_graph": ([ctypes.POINTER(ModelConfig), ctypes.POINTER(Tuning), i32, H], st),
        "mk_load_weights": ([vp, ctypes.POINTER(Weights), vp], st),
        "mk_decode_step": ([vp, vp, vp, vp, vp, vp, vp, vp], st),
        "mk_decode_step_perop": ([vp, vp, vp, vp, vp, vp, vp, vp], st),
        "mk_decode_steps": ([vp, i32, vp, vp, vp, vp, vp, vp, vp], st),
        "mk_decode_steps_paged": ([vp, i32, vp, vp, vp, vp, vp, i32, vp, vp, vp], st),
        "mk_decode_step_noalloc": ([vp, vp, vp, vp, vp, vp, vp, vp], st),
        "mk_sync_status": ([vp, vp, vp], st),
        "mk_reset": ([vp, vp], st),
        "mk_graph_export": ([vp, ctypes.POINTER(GraphView)], st),
        "mk_get_info": ([vp, ctypes.POINTER(Info)], st),
        "mk_final_hidden": ([vp, ctypes.POINTER(vp)], st),
        "mk_debug_set_event_count": ([vp, i32, i32, vp], st),
        "mk_set_trace": ([vp, vp, ctypes.c_int64], st),
        "mk_set_timeout_us": ([vp, ctypes.c_uint], st),
        "mk_last_error": ([vp], ctypes.c_char_p),
        "mk_destroy": ([vp], None),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def _check(rc: int, h=None):
    if rc != MK_OK:
        msg = lib().mk_last_error(h)
        raise MkError(rc, msg.decode() if msg else "")


def make_config(w, kv_capacity: int) -> ModelConfig:
    """ModelConfig from any object with the workload attributes (see synth.Workload)."""
    return ModelConfig(w.n_layers, w.hidden, w.n_q_heads, w.n_kv_heads, w.head_dim, w.ffn,
                       w.vocab, int(w.tied_embeddings), w.rms_eps, w.rope_theta, w.batch,
                       kv_capacity)


def make_tuning(**kw) -> Tuning:
    t = Tuning()
    for k, v in kw.items():
        setattr(t, k, v)
    return t


@dataclass
class Graph:
    """Host copy of a graph's tables (same field names as the oracle's)."""
    task_type: np.ndarray
    task_op: np.ndarray
    task_layer: np.ndarray
    task_idx: np.ndarray
    task_dep: np.ndarray
    task_trig: np.ndarray
    event_count: np.ndarray
    event_first: np.ndarray
    event_last: np.ndarray
    edge_src: np.ndarray
    edge_dst: np.ndarray
    num_workers: int
    tiling: tuple
    mma_tiling: tuple = ()  # ((mb, kcb) of QKV, O, GATE_UP, DOWN, LM_HEAD) at batch >= 2

    @property
    def n_tasks(self):
        return int(self.task_type.size)

    @property
    def n_events(self):
        return int(self.event_count.size)


def _export(h) -> Graph:
    v = GraphView()
    _check(lib().mk_graph_export(h, ctypes.byref(v)), h)

    def arr(p, n):
        return np.ctypeslib.as_array(p, shape=(n,)).copy() if n else np.zeros(0, np.int32)

    return Graph(*(arr(getattr(v, f), v.n_tasks) for f in
                   ("task_type", "task_op", "task_layer", "task_idx", "task_dep", "task_trig")),
                 *(arr(getattr(v, f), v.n_events) for f in
                   ("event_count", "event_first", "event_last")),
                 arr(v.edge_src, v.n_edges), arr(v.edge_dst, v.n_edges), v.num_workers,
                 (v.qkv_rows, v.o_rows, v.gu_rows, v.down_rows, v.lm_rows, v.attn_splits,
                  v.attn_chunk),
                 tuple((int(v.mma_mb[i]), int(v.mma_kcb[i])) for i in range(5)))


def plan_graph(w, kv_capacity: int, num_workers: int, **tuning) -> Graph:
    """Host-only graph construction (mk_plan_graph)."""
    h = ctypes.c_void_p()
    cfg = make_config(w, kv_capacity)
    t = make_tuning(**tuning)
    _check(lib().mk_plan_graph(ctypes.byref(cfg), ctypes.byref(t), num_workers, ctypes.byref(h)))
    try:
        return _export(h)
    finally:
        lib().mk_destroy(h)


def graph_from_edges(task_op, task_idx, edges) -> Graph:
    op = np.ascontiguousarray(task_op, dtype=np.int32)
    idx = np.ascontiguousarray(task_idx, dtype=np.int32)
    e = np.asarray(edges, dtype=np.int32).reshape(-1, 2)
    src, dst = np.ascontiguousarray(e[:, 0]), np.ascontiguousarray(e[:, 1])
    h = ctypes.c_void_p()
    _check(lib().mk_graph_from_edges(op.size, op.ctypes.data, idx.ctypes.data, src.size,
                                     src.ctypes.data, dst.ctypes.data, ctypes.byref(h)))
    try:
        return _export(h)
    finally:
        lib().mk_destroy(h)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return t.data_ptr()


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


class Megakernel:
    """One handle: graph + device state for one model shape and batch."""

    def __init__(self, w, kv_capacity: int, device: int = 0, **tuning):
        self.w = w
        self.kv_capacity = kv_capacity
        self.device = device
        self._h = ctypes.c_void_p()
        cfg = make_config(w, kv_capacity)
        t = make_tuning(**tuning)
        _check(lib().mk_build_graph(ctypes.byref(cfg), ctypes.byref(t), device,
                                    ctypes.byref(self._h)))
        self._keep = []

    def close(self):
        if self._h:
            lib().mk_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self):
        return self._h

    def load_weights(self, weights: dict, stream=None):
        """weights: torch tensors (bf16 or int16/uint16 bit patterns), same keys as synth."""
        Ly = self.w.n_layers
        arrays = {}
        for name in ("attn_norm", "wq", "wk", "wv", "q_norm", "k_norm", "wo", "mlp_norm",
                     "w_gate", "w_up", "w_down"):
            arr = (ctypes.c_void_p * Ly)(*[weights["layers"][l][name].data_ptr() for l in range(Ly)])
            arrays[name] = arr
        W = Weights(weights["embed"].data_ptr(), weights["final_norm"].data_ptr(),
                    None if weights.get("lm_head") is None else weights["lm_head"].data_ptr(),
                    *[ctypes.cast(arrays[n], _PP) for n in
                      ("attn_norm", "wq", "wk", "wv", "q_norm", "k_norm", "wo", "mlp_norm",
                       "w_gate", "w_up", "w_down")])
        _check(lib().mk_load_weights(self._h, ctypes.byref(W), _stream_ptr(stream)), self._h)

    def decode_step(self, tokens_in, tokens_out, kv_len, k_cache, v_cache, logits=None,
                    stream=None):
        _check(lib().mk_decode_step(self._h, _ptr(tokens_in), _ptr(tokens_out), _ptr(kv_len),
                                    _ptr(k_cache), _ptr(v_cache), _ptr(logits),
                                    _stream_ptr(stream)), self._h)

    def decode_steps(self, n_steps, tokens_in, tokens_out, kv_len, k_cache, v_cache, logits=None,
                     stream=None):
        """n_steps steps in one launch; tokens_out holds n_steps x batch tokens."""
        _check(lib().mk_decode_steps(self._h, n_steps, _ptr(tokens_in), _ptr(tokens_out),
                                     _ptr(kv_len), _ptr(k_cache), _ptr(v_cache), _ptr(logits),
                                     _stream_ptr(stream)), self._h)

    def decode_steps_paged(self, n_steps, tokens_in, tokens_out, kv_len, k_pool, v_pool,
                           n_pages, page_table, logits=None, stream=None):
        """n_steps steps on paged K/V pools [n_pages][Ly][Hkv][P][D] with a page table
        [batch][ceil(kv_capacity / P)] (handle built with kv_page_size = P)."""
        _check(lib().mk_decode_steps_paged(self._h, n_steps, _ptr(tokens_in), _ptr(tokens_out),
                                           _ptr(kv_len), _ptr(k_pool), _ptr(v_pool), n_pages,
                                           _ptr(page_table), _ptr(logits), _stream_ptr(stream)),
               self._h)

    def decode_step_perop(self, tokens_in, tokens_out, kv_len, k_cache, v_cache, logits=None,
                          stream=None):
        _check(lib().mk_decode_step_perop(self._h, _ptr(tokens_in), _ptr(tokens_out),
                                          _ptr(kv_len), _ptr(k_cache), _ptr(v_cache),
                                          _ptr(logits), _stream_ptr(stream)), self._h)

    def decode_step_noalloc(self, tokens_in, tokens_out, kv_len, k_cache, v_cache, logits=None,
                            stream=None):
        """mk_decode_step with its working buffers in the library's static region."""
        _check(lib().mk_decode_step_noalloc(self._h, _ptr(tokens_in), _ptr(tokens_out),
                                            _ptr(kv_len), _ptr(k_cache), _ptr(v_cache),
                                            _ptr(logits), _stream_ptr(stream)), self._h)

    def sync_status(self, stream=None):
        """Returns (status, detail[4]); status 0 = ok."""
        d = (ctypes.c_int32 * 4)()
        rc = lib().mk_sync_status(self._h, _stream_ptr(stream), d)
        return rc, list(d)

    def reset(self, stream=None):
        _check(lib().mk_reset(self._h, _stream_ptr(stream)), self._h)

    def graph(self) -> Graph:
        return _export(self._h)

    def info(self) -> Info:
        i = Info()
        _check(lib().mk_get_info(self._h, ctypes.byref(i)), self._h)
        return i

    def final_hidden_ptr(self) -> int:
        p = ctypes.c_void_p()
        _check(lib().mk_final_hidden(self._h, ctypes.byref(p)), self._h)
        return p.value

    def set_event_count(self, event: int, count: int, stream=None):
        _check(lib().mk_debug_set_event_count(self._h, event, count, _stream_ptr(stream)),
               self._h)

    def set_trace(self, buf=None):
        """buf: int64/uint64 torch tensor with >= 8 * n_tasks elements, or None."""
        if buf is None:
            _check(lib().mk_set_trace(self._h, None, 0), self._h)
        else:
            _check(lib().mk_set_trace(self._h, buf.data_ptr(), buf.numel() * buf.element_size()),
                   self._h)

    def set_timeout_us(self, us: int):
        _check(lib().mk_set_timeout_us(self._h, us), self._h)
