"""Batched decode steps (2..16 sequences; projections on tensor cores) against
the CPU oracle, through the C ABI (libmk.so).

With batch >= 2 every projection runs as mma.sync on fragment-ordered weights
with hi/lo bf16 activations, and attention on mma.sync over TMA K/V tiles,
its splits fixed at build time or (attn_jit) cut from the live KV lengths at
run time.  The tolerances are those of the batch-1 tests.
"""
import numpy as np
import pytest

import synth
from gpu_helpers import Case, compare_step, kv_rows_close, torch

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("built_libs")]


def tiny_batch(B, lo=0, hi=96, **kw):
    """The tiny decoder at batch B, per-sequence cache lengths drawn in [lo, hi]."""
    return synth.TINY.with_(name=f"tiny-b{B}", batch=B, kv_len=None, kv_len_range=(lo, hi), **kw)


@pytest.mark.parametrize("B,tied", [(2, 0), (3, 1), (8, 0), (9, 1), (16, 0)])
def test_tiny_batch_step_matches_oracle(B, tied):
    # 2..8 sequences use one 8-column tile, 9..16 two; B = 3 and 9 leave zero
    # padded columns; lengths start at 0 (only the new row)
    w = tiny_batch(B, tied_embeddings=tied)
    c = Case(w, seed=10 + B, extra_cap=2)
    k, v, lens = c.k.copy(), c.v.copy(), c.lens.copy()
    got = c.gpu_step()
    ref = c.oracle_step(k=k, v=v, lens=lens)
    compare_step(ref, got, w, f"tiny-b{B}")
    np.testing.assert_array_equal(got["kv_len"], c.lens + 1)
    kv_rows_close(c, k, v, c.lens, bf16_inputs=True)


def test_tiny_batch16_split_attention_mixed_lengths():
    # capacity ~760 over 16 sequences x 2 kv heads: several splits per head,
    # so the last-arriving split merges and writes the O projection's operand
    w = tiny_batch(16, lo=0, hi=700)
    c = Case(w, seed=31, extra_cap=60)
    assert c.mk.graph().tiling[5] > 1
    k, v, lens = c.k.copy(), c.v.copy(), c.lens.copy()
    got = c.gpu_step()
    ref = c.oracle_step(k=k, v=v, lens=lens)
    compare_step(ref, got, w, "tiny-b16-split")
    kv_rows_close(c, k, v, c.lens, bf16_inputs=True)


def test_batch_multi_step_lockstep_determinism_and_per_operator_path():
    w = tiny_batch(8, lo=10, hi=300, steps=4)
    c = Case(w, seed=32)
    k, v, lens = c.k.copy(), c.v.copy(), c.lens.copy()
    tok = c.tokens.copy()
    for step in range(4):
        got = c.gpu_step(tokens=tok)
        ref = c.oracle_step(tokens=tok, k=k, v=v, lens=lens)
        compare_step(ref, got, w, f"b8 step{step}")
        tok = ref["tokens"].copy()  # both sides continue from the oracle's token
    # the same state twice, then through the per-operator launches: bitwise equal
    c.reset_device_state()
    a = c.gpu_step()
    c.reset_device_state()
    b = c.gpu_step()
    c.reset_device_state()
    d = c.gpu_step(perop=True)
    for key in ("tokens", "logits", "hidden", "kv_len"):
        np.testing.assert_array_equal(a[key], b[key])
        np.testing.assert_array_equal(a[key], d[key])


def test_qwen3_06b_batch8_step_matches_oracle():
    # tied 151936-row LM head: its fragment-ordered copy is built in row slabs
    w = synth.Q06B.with_(name="qwen3-0.6b-b8", batch=8, kv_len=None, kv_len_range=(1, 600))
    c = Case(w, seed=33, extra_cap=2)
    k, v, lens = c.k.copy(), c.v.copy(), c.lens.copy()
    got = c.gpu_step()
    ref = c.oracle_step(k=k, v=v, lens=lens)
    compare_step(ref, got, w, "0.6b-b8")
    kv_rows_close(c, k, v, c.lens, bf16_inputs=True)


_WEIGHTS_8B = {}


def _weights_8b(seed):
    # the 8B-shaped weights are the same streams at every batch size
    if seed not in _WEIGHTS_8B:
        _WEIGHTS_8B.clear()
        _WEIGHTS_8B[seed] = synth.make_weights(synth.Q8B, seed)
    return _WEIGHTS_8B[seed]


@pytest.mark.parametrize("w,seqs", [(synth.Q8B_B8, (0, 5)), (synth.Q8B_B16, (0, 15))],
                         ids=["qwen3-8b-b8", "qwen3-8b-b16"])
def test_qwen3_8b_batched_full_size_sampled_sequences(w, seqs):
    # The batched 8B workloads at full size, with the capacity (longest cache
    # + the workload's steps) and one-CTA-per-SM launch the bench uses.  The
    # oracle computes the sampled sequences only (seq_mask); every sequence's
    # token and kv_len update is still checked for validity.
    t = torch()
    c = Case(w, seed=0, weights=_weights_8b(0))
    assert c.mk.info().num_workers == t.cuda.get_device_properties(0).multi_processor_count
    got = c.gpu_step()
    mask = np.zeros(w.batch, dtype=np.uint8)
    mask[list(seqs)] = 1
    lens = c.lens.copy()
    ref = c.model.step(c.tokens, lens, c.k, c.v, seq_mask=mask)  # appends rows in c.k / c.v
    compare_step(ref, got, w, w.name, seqs=seqs)
    np.testing.assert_array_equal(got["kv_len"], c.lens + 1)
    assert ((got["tokens"] >= 0) & (got["tokens"] < w.vocab)).all()
    for b in seqs:
        L = int(c.lens[b])
        for dev, host in ((c.d_k, c.k), (c.d_v, c.v)):
            g = synth.bf16_to_f32(dev[:, b, :, L].cpu().numpy().view(np.uint16)).astype(np.float64)
            r = synth.bf16_to_f32(host[:, b, :, L]).astype(np.float64)
            assert np.all(np.abs(g - r) <= 1e-2 * np.max(np.abs(r), axis=-1, keepdims=True))


def test_tiny_batch_eight_position_attention_blocks():
    # 10 KB ring stages: K/V stages of 40 positions (not a whole number of
    # 16-position blocks), so the tensor-core attention takes its 8-position
    # blocks; the projections run 1- and 2-m-tile stages of 8 and 16 k-blocks
    w = tiny_batch(8, lo=0, hi=200)
    c = Case(w, seed=34, extra_cap=2, ring_stage_bytes=10240, ring_stages=8)
    chunk = c.mk.graph().tiling[6]
    pps = min(256, chunk, 10240 // (4 * w.head_dim) // 8 * 8)
    assert pps % 16 != 0
    k, v, lens = c.k.copy(), c.v.copy(), c.lens.copy()
    got = c.gpu_step()
    ref = c.oracle_step(k=k, v=v, lens=lens)
    compare_step(ref, got, w, "tiny-b8-np8")
    kv_rows_close(c, k, v, c.lens, bf16_inputs=True)


def _with_lengths(c, lens):
    """Re-seed the case's caches for explicit per-sequence lengths."""
    c.lens = np.asarray(lens, dtype=np.int32)
    c.k, c.v = synth.make_kv(c.w, c.lens, c.cap, c.seed)
    c.reset_device_state()
    return c


@pytest.mark.parametrize("jit", [1, 0], ids=["jit", "fixed-splits"])
def test_tiny_batch_attention_jit_and_fixed_splits_match_oracle(jit):
    # mixed lengths from 0 (only the new row) to 700: JIT pieces that cover
    # the end of one (sequence, kv head) and the start of the next, pairs
    # merged from several pieces, and pairs done by one piece
    w = tiny_batch(12, lo=0, hi=700)
    c = Case(w, seed=35, extra_cap=4, attn_jit=jit)
    assert (c.mk.graph().tiling[6] == 0) == (jit == 1)
    k, v, lens = c.k.copy(), c.v.copy(), c.lens.copy()
    got = c.gpu_step()
    ref = c.oracle_step(k=k, v=v, lens=lens)
    compare_step(ref, got, w, f"tiny-b12-jit{jit}")
    kv_rows_close(c, k, v, c.lens, bf16_inputs=True)


def test_tiny_batch_jit_pieces_over_many_short_pairs():
    # 15 empty caches and one of 900 rows on 148 workers: the short pairs
    # (one position each) share tasks, the long one is cut across many
    w = tiny_batch(16, lo=0, hi=0)
    c = Case(w, seed=36, extra_cap=904, attn_jit=1)
    lens = np.zeros(16, dtype=np.int32)
    lens[11] = 900
    _with_lengths(c, lens)
    k, v, L = c.k.copy(), c.v.copy(), c.lens.copy()
    got = c.gpu_step()
    ref = c.oracle_step(k=k, v=v, lens=L)
    compare_step(ref, got, w, "tiny-b16-short-pairs")
    kv_rows_close(c, k, v, c.lens, bf16_inputs=True)
