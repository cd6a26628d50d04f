"""Seeded synthetic workloads for the decode step.

This module holds no arithmetic of the decode step.  It defines the named
workload shapes and fills host buffers with seeded bf16 normals and integers
(the generator is documented in ``synth.c``).  The CPU oracle and the GPU
library both receive the buffers made here; neither imports the other.

Weights are ~N(0, 0.02) in bf16, norm gains are 1 + N(0, 0.1) in bf16, cached
K/V rows 0..L_b-1 are N(0, 1) in bf16 and rows >= L_b are zero, token ids are
uniform in [0, vocab), and per-sequence KV lengths of the mixed-length batch are
uniform integers in [256, 4096].
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, replace
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmk_synth.so")
_lib = None


def build(verbose: bool = False) -> str:
    """Compile the generator into ``synth/libmk_synth.so`` (gcc, -O2)."""
    import subprocess

    src = os.path.join(_HERE, "synth.c")
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-pthread",
           "-ffp-contract=off", src, "-o", _LIB_PATH, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        build()
    lib = ctypes.CDLL(_LIB_PATH)
    lib.synth_normal_bf16.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint64,
                                      ctypes.c_uint64, ctypes.c_uint64, ctypes.c_double,
                                      ctypes.c_double, ctypes.c_int]
    lib.synth_normal_bf16.restype = ctypes.c_int
    lib.synth_uniform_int.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint64,
                                      ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64,
                                      ctypes.c_int64]
    lib.synth_uniform_int.restype = ctypes.c_int
    lib.synth_u64_at.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64]
    lib.synth_u64_at.restype = ctypes.c_uint64
    _lib = lib
    return lib


def default_threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


# ----------------------------------------------------------------------------
# Workload shapes
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    """Shape of a Qwen3-style decoder plus the batch/KV state of one run."""

    name: str
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    tied_embeddings: int
    batch: int
    kv_len: Optional[int]          # fixed length for every sequence, or None = drawn
    kv_len_range: tuple = (0, 0)   # inclusive range when drawn
    steps: int = 1
    rms_eps: float = 1e-6
    rope_theta: float = 1e6

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def kv_lens(self, seed: int = 0) -> np.ndarray:
        if self.kv_len is not None:
            return np.full(self.batch, self.kv_len, dtype=np.int32)
        lo, hi = self.kv_len_range
        return uniform_int(self.batch, seed, TID_KV_LENS, lo, hi)

    def kv_capacity(self, seed: int = 0) -> int:
        """Cache rows per (layer, sequence, kv head): longest start length + steps."""
        return int(self.kv_lens(seed).max()) + self.steps

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY = Workload("tiny", 2, 256, 4, 2, 64, 768, 4096, 0, 1, 32, steps=1)
Q06B = Workload("qwen3-0.6b", 28, 1024, 16, 8, 128, 3072, 151936, 1, 1, 512, steps=64)
Q8B = Workload("qwen3-8b", 36, 4096, 32, 8, 128, 12288, 151936, 0, 1, 1024, steps=64)
Q8B_B8 = Workload("qwen3-8b-b8", 36, 4096, 32, 8, 128, 12288, 151936, 0, 8, None,
                  kv_len_range=(256, 4096), steps=64)
Q8B_B16 = Workload("qwen3-8b-b16", 36, 4096, 32, 8, 128, 12288, 151936, 0, 16, 8192, steps=32)

# Profiling case: the 8B layer shapes with 4 layers (2.7 GB of weights), small
# enough for multi-pass counter captures.
Q8B_4L = Q8B.with_(name="qwen3-8b-4layer", n_layers=4)
# Profiling case of the batched kernel: 4 of the 8B layers at batch 16, 1024
# cached rows per sequence (about 4.5 GB on the device).
Q8B_B16_4L = Q8B_B16.with_(name="qwen3-8b-b16-4layer", n_layers=4, kv_len=1024)

# The same at batch 8 (the one-column-tile instantiation of the batched kernel).
Q8B_B8_4L = Q8B_B8.with_(name="qwen3-8b-b8-4layer", n_layers=4, kv_len=1024)

WORKLOADS = {w.name: w for w in (TINY, Q06B, Q8B, Q8B_B8, Q8B_B16, Q8B_4L, Q8B_B16_4L, Q8B_B8_4L)}

# ----------------------------------------------------------------------------
# Stream ids (one counter stream per tensor)
# ----------------------------------------------------------------------------
TID_EMBED, TID_LM_HEAD, TID_FINAL_NORM, TID_TOKENS, TID_KV_LENS = 1, 2, 3, 5, 6
LAYER_KINDS = ("attn_norm", "wq", "wk", "wv", "q_norm", "k_norm", "wo",
               "mlp_norm", "w_gate", "w_up", "w_down")
GAIN_KINDS = ("attn_norm", "q_norm", "k_norm", "mlp_norm")


def layer_tid(layer: int, kind: str) -> int:
    return 1000 + layer * 32 + LAYER_KINDS.index(kind)


def kv_tid(which: int, layer: int, b: int, g: int) -> int:
    """Stream of cached rows for (K=0 / V=1, layer, sequence, kv head)."""
    return (0x4B56 << 48) | (which << 44) | (layer << 28) | (b << 14) | g


# ----------------------------------------------------------------------------
# Fillers
# ----------------------------------------------------------------------------
def fill_normal_bf16(ptr: int, n: int, seed: int, tid: int, mean: float, std: float,
                     offset: int = 0, threads: Optional[int] = None) -> None:
    """Write n bf16 values of stream (seed, tid) starting at element `offset` to ptr."""
    lib = _load()
    rc = lib.synth_normal_bf16(ctypes.c_void_p(ptr), n, seed, tid, offset, mean, std,
                               threads or default_threads())
    if rc != 0:
        raise RuntimeError("synth_normal_bf16 failed")


def normal_bf16(shape, seed: int, tid: int, mean: float = 0.0, std: float = 1.0,
                offset: int = 0, threads: Optional[int] = None) -> np.ndarray:
    """bf16 bit patterns (uint16) of shape `shape` from stream (seed, tid)."""
    out = np.empty(shape, dtype=np.uint16)
    fill_normal_bf16(out.ctypes.data, out.size, seed, tid, mean, std, offset, threads)
    return out


def uniform_int(n: int, seed: int, tid: int, lo: int, hi: int, offset: int = 0) -> np.ndarray:
    lib = _load()
    out = np.empty(n, dtype=np.int32)
    rc = lib.synth_uniform_int(ctypes.c_void_p(out.ctypes.data), n, seed, tid, offset, lo, hi)
    if rc != 0:
        raise RuntimeError("synth_uniform_int failed")
    return out


def u64_at(seed: int, tid: int, i: int) -> int:
    return int(_load().synth_u64_at(seed, tid, i))


# ----------------------------------------------------------------------------
# bf16 helpers (bit-pattern level; no method arithmetic)
# ----------------------------------------------------------------------------
def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 bit patterns, nearest-even."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        r[nan] = 0x7FC0
    return r


# ----------------------------------------------------------------------------
# Whole-workload inputs
# ----------------------------------------------------------------------------
def weight_shapes(w: Workload) -> dict:
    H, F = w.hidden, w.ffn
    return {
        "attn_norm": (H,), "wq": (w.q_dim, H), "wk": (w.kv_dim, H), "wv": (w.kv_dim, H),
        "q_norm": (w.head_dim,), "k_norm": (w.head_dim,), "wo": (H, w.q_dim),
        "mlp_norm": (H,), "w_gate": (F, H), "w_up": (F, H), "w_down": (H, F),
    }


def make_weights(w: Workload, seed: int = 0, threads: Optional[int] = None) -> dict:
    """All weights as bf16 bit patterns (numpy uint16), nn.Linear layout [out][in].

    Returns {"embed", "lm_head" (None when tied), "final_norm", "layers": [dict]}.
    """
    shapes = weight_shapes(w)
    out = {
        "embed": normal_bf16((w.vocab, w.hidden), seed, TID_EMBED, 0.0, 0.02, threads=threads),
        "lm_head": None if w.tied_embeddings else
        normal_bf16((w.vocab, w.hidden), seed, TID_LM_HEAD, 0.0, 0.02, threads=threads),
        "final_norm": normal_bf16((w.hidden,), seed, TID_FINAL_NORM, 1.0, 0.1, threads=threads),
        "layers": [],
    }
    for l in range(w.n_layers):
        layer = {}
        for kind in LAYER_KINDS:
            mean, std = (1.0, 0.1) if kind in GAIN_KINDS else (0.0, 0.02)
            layer[kind] = normal_bf16(shapes[kind], seed, layer_tid(l, kind), mean, std,
                                      threads=threads)
        out["layers"].append(layer)
    return out


def make_tokens(w: Workload, seed: int = 0) -> np.ndarray:
    return uniform_int(w.batch, seed, TID_TOKENS, 0, w.vocab - 1)


def fill_kv_rows(dst: np.ndarray, which: int, layer: int, b: int, g: int, rows: int,
                 seed: int, threads: Optional[int] = None) -> None:
    """Fill rows [0, rows) of one [Lcap][D] cache slab with N(0,1) bf16, rest zero."""
    D = dst.shape[-1]
    dst[...] = 0
    if rows > 0:
        flat = dst.reshape(-1)
        fill_normal_bf16(flat.ctypes.data, rows * D, seed, kv_tid(which, layer, b, g), 0.0, 1.0,
                         threads=threads)


def make_kv(w: Workload, kv_lens: np.ndarray, kv_capacity: int, seed: int = 0,
            threads: Optional[int] = None):
    """K and V caches [Ly][B][Hkv][Lcap][D] (bf16 bits)."""
    shape = (w.n_layers, w.batch, w.n_kv_heads, kv_capacity, w.head_dim)
    k = np.zeros(shape, dtype=np.uint16)
    v = np.zeros(shape, dtype=np.uint16)
    for l in range(w.n_layers):
        for b in range(w.batch):
            for g in range(w.n_kv_heads):
                fill_kv_rows(k[l, b, g], 0, l, b, g, int(kv_lens[b]), seed, threads)
                fill_kv_rows(v[l, b, g], 1, l, b, g, int(kv_lens[b]), seed, threads)
    return k, v
