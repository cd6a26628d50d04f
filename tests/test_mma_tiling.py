"""Host-side tiling of the batched projections (batch >= 2), from the graph
export of host-only handles (no device).

The batched projections run on tcgen05 tensor cores: a task's rows (padded to
16) run in passes of at most 256 rows (one accumulator of 128 TMEM lanes x N
columns), and a pass streams ring stages of `kcb` 16-column k-blocks.  A
stage's slot holds the weights (N x 32 bytes per k-block), the operand chunk
(512 x nn bytes per k-block, nn 8-sequence tiles) and 4 KB that the operand
descriptors read past the chunk, so:
- mb (16-row m-tiles of a full pass) is at most 16 and covers the task,
- kcb >= 1 and the three parts of a full stage fit the ring stage,
- kcb is at most the operator's K / 16 k-blocks.
Stages then cover each pass's k-blocks exactly once, in order.
"""
import pytest

import persistent_runtime_b200 as prb
import synth

SLACK = 4096
MAX_N = 256


def plan(w, cap=1100, **tuning):
    return prb.plan_graph(w, cap, 148, **tuning)


def op_dims(w, g):
    """(rows of the operator, rows per task, K) of each projection."""
    rep = w.n_q_heads // w.n_kv_heads
    n_qkv = w.n_kv_heads * (rep + 2) * w.head_dim
    t = g.tiling
    return [(n_qkv, t[0], w.hidden), (w.hidden, t[1], w.n_q_heads * w.head_dim),
            (2 * w.ffn, 2 * t[2], w.hidden), (w.hidden, t[3], w.ffn), (w.vocab, t[4], w.hidden)]


def kblocks_per_stage(stage_bytes, N, nn, KB):
    return min(KB, max(1, (stage_bytes - SLACK) // (N * 32 + 512 * nn)))


def test_batch1_handles_export_no_tensor_core_tiling():
    g = plan(synth.Q8B)
    assert g.mma_tiling == ((0, 0),) * 5


@pytest.mark.parametrize("B,expect", [
    (8, ((3, 22), (2, 29), (12, 6), (2, 29), (16, 5))),
    (16, ((3, 17), (2, 22), (12, 6), (2, 22), (16, 4))),
])
def test_qwen3_8b_default_tiling(B, expect):
    # 48-row QKV, 32-row O/DOWN, 96-pair GATE_UP and 1040-row LM-head tasks
    # (passes of 256 rows); 48 KB stages
    g = plan(synth.Q8B.with_(name=f"q8b-b{B}", batch=B))
    assert g.mma_tiling == expect


@pytest.mark.parametrize("wl", ["tiny", "qwen3-0.6b", "qwen3-8b"])
@pytest.mark.parametrize("B", [2, 5, 8, 9, 16])
@pytest.mark.parametrize("stage_kb", [10, 16, 24, 36, 48, 64, 96])
@pytest.mark.parametrize("col_align", [16, 48])
def test_tiling_bounds_and_stage_coverage(wl, B, stage_kb, col_align):
    w = synth.WORKLOADS[wl].with_(name=f"{wl}-b{B}", batch=B, kv_len=64, kv_len_range=None)
    sb = stage_kb * 1024
    g = plan(w, cap=200, ring_stage_bytes=sb, col_align=col_align)
    nn = (B + 7) // 8
    if min(kcb for _, kcb in g.mma_tiling) < 1:
        return  # such a ring stage is rejected when the handle is built
    for (rows, per_task, K), (mb, kcb) in zip(op_dims(w, g), g.mma_tiling):
        KB = K // 16
        assert 1 <= mb <= MAX_N // 16
        assert mb * 16 == min(MAX_N, -(-per_task // 16) * 16)
        assert 1 <= kcb <= KB
        assert kcb * (mb * 16 * 32 + 512 * nn) + SLACK <= sb
        # every task: passes of <= 256 rows, stages cover each pass's k-blocks once
        rows_p = -(-rows // 16) * 16
        for r0 in range(0, rows, per_task):
            trows = min(per_task, rows_p - r0)
            assert trows % 16 == 0
            covered = 0
            for q0 in range(0, trows, MAX_N):
                N = min(MAX_N, trows - q0)
                nkb = kblocks_per_stage(sb, N, nn, KB)
                assert nkb * (N * 32 + 512 * nn) + SLACK <= sb
                kb = 0
                while kb < KB:
                    here = min(nkb, KB - kb)
                    covered += here * N * 32
                    kb += here
                assert kb == KB
            assert covered == trows * K * 2


def test_too_small_ring_stage_is_rejected_by_the_tiling():
    # 8 KB stages cannot hold one 256-row k-block (8 KB) plus the operand and slack
    g = plan(synth.Q8B.with_(name="q8b-b16", batch=16), ring_stage_bytes=8 * 1024)
    assert g.mma_tiling[4][1] == 0
