"""Host-side tiling of the batched projections (batch >= 2), from the graph
export of host-only handles (no device).

Each projection task streams row blocks of `mb` 16-row m-tiles in ring stages
of `kcb` 16-column k-blocks; the 8 compute warps split a stage's k-blocks, and
a warp holds the B fragments of its k-blocks of one stage in registers
(6 per warp with one 8-column operand tile, 3 with two), so:
- kcb is a multiple of 8 and at most 8 x that limit,
- a stage (mb x kcb x 512 bytes) fits the ring stage,
- mb is at most 6 (the accumulator arrays).
The default Qwen3-8B configurations must also keep their bytes on the
guard-free stage bodies (compile-time m-tile and k-block counts) that the
batched kernel has for the common shapes.
"""
import pytest

import persistent_runtime_b200 as prb
import synth

# (m-tiles, k-blocks per warp) of the guard-free stage bodies
FIXED = {1: {(2, 6), (3, 4), (2, 3), (3, 3), (6, 2), (2, 2), (3, 2)},
         2: {(2, 3), (3, 3), (6, 2), (2, 2), (3, 2)}}


def max_kpw(nn):
    return 6 if nn == 1 else 3


def plan(w, cap=1100, **tuning):
    return prb.plan_graph(w, cap, 148, **tuning)


def op_dims(w, g):
    """(rows of the operator, rows per task, K) of each projection."""
    rep = w.n_q_heads // w.n_kv_heads
    n_qkv = w.n_kv_heads * (rep + 2) * w.head_dim
    t = g.tiling
    return [(n_qkv, t[0], w.hidden), (w.hidden, t[1], w.n_q_heads * w.head_dim),
            (2 * w.ffn, 2 * t[2], w.hidden), (w.hidden, t[3], w.ffn), (w.vocab, t[4], w.hidden)]


def stage_shapes(w, g):
    """Bytes one step streams per (m-tiles, k-blocks per warp) stage shape: every
    layer's four projections and the LM head once."""
    nn = (w.batch + 7) // 8
    out = {}
    for i, ((rows, per_task, K), (mb, kcb)) in enumerate(zip(op_dims(w, g), g.mma_tiling)):
        times = 1 if i == 4 else w.n_layers
        KB = K // 16
        chunks = [min(kcb, KB - k0) for k0 in range(0, KB, kcb)]
        for r0 in range(0, rows, per_task):
            mt = (min(rows, r0 + per_task) - r0 + 15) // 16
            for m0 in range(0, mt, mb):
                nm = min(mb, mt - m0)
                for nkb in chunks:
                    key = (nm, nkb // 8)
                    out[key] = out.get(key, 0) + times * nm * nkb * 512
    assert all(k[1] <= max_kpw(nn) for k in out)
    return out


def test_batch1_handles_export_no_tensor_core_tiling():
    g = plan(synth.Q8B)
    assert g.mma_tiling == ((0, 0),) * 5


@pytest.mark.parametrize("B,expect", [
    (8, ((3, 32), (2, 48), (6, 16), (2, 48), (6, 16))),
    (16, ((3, 24), (2, 24), (6, 16), (2, 24), (6, 16))),
])
def test_qwen3_8b_default_tiling(B, expect):
    # 48-row QKV, 32-row O/DOWN, 96-pair GATE_UP and 1040-row LM-head tasks;
    # 48 KB stages (96 tiles of 512 bytes)
    g = plan(synth.Q8B.with_(name=f"q8b-b{B}", batch=B))
    assert g.mma_tiling == expect


@pytest.mark.parametrize("wl", ["tiny", "qwen3-0.6b", "qwen3-8b"])
@pytest.mark.parametrize("B", [2, 5, 8, 9, 16])
@pytest.mark.parametrize("stage_kb", [10, 24, 36, 48, 64, 96])
@pytest.mark.parametrize("col_align", [16, 48])
def test_tiling_bounds(wl, B, stage_kb, col_align):
    w = synth.WORKLOADS[wl].with_(name=f"{wl}-b{B}", batch=B, kv_len=64, kv_len_range=None)
    g = plan(w, cap=200, ring_stage_bytes=stage_kb * 1024, col_align=col_align)
    nn = (B + 7) // 8
    if min(kcb for _, kcb in g.mma_tiling) < 8:
        return  # such a ring stage is rejected when the handle is built
    for (rows, per_task, K), (mb, kcb) in zip(op_dims(w, g), g.mma_tiling):
        assert 1 <= mb <= 6
        assert mb <= max(1, per_task // 16)
        assert kcb % 8 == 0 and 8 <= kcb <= 8 * max_kpw(nn)
        assert mb * kcb * 512 <= stage_kb * 1024
        assert (K // 16) % 8 == 0  # every k chunk, the last one too, is whole warp shares
    stage_shapes(w, g)


@pytest.mark.parametrize("B", [8, 16])
def test_qwen3_8b_bytes_run_on_guard_free_stages(B):
    w = synth.Q8B.with_(name=f"q8b-b{B}", batch=B)
    g = plan(w)
    shapes = stage_shapes(w, g)
    total = sum(shapes.values())
    fixed = sum(v for k, v in shapes.items() if k in FIXED[(B + 7) // 8])
    assert fixed / total > 0.99, shapes
