"""GPU decode step against the CPU oracle, through the C ABI (libmk.so)."""
import numpy as np
import pytest

import synth
from gpu_helpers import Case, compare_step, kv_rows_close, torch

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("built_libs")]


@pytest.mark.parametrize("tied", [0, 1])
def test_tiny_step_matches_oracle(tied):
    w = synth.TINY.with_(tied_embeddings=tied)
    c = Case(w, seed=1)
    got = c.gpu_step()
    k, v, lens = c.k.copy(), c.v.copy(), c.lens.copy()
    ref = c.oracle_step(k=k, v=v, lens=lens)
    compare_step(ref, got, w, "tiny")
    np.testing.assert_array_equal(got["kv_len"], c.lens + 1)
    kv_rows_close(c, k, v, c.lens)


def test_tiny_long_cache_uses_split_attention_and_merge():
    # kv capacity 1000 with 148 workers -> several splits per (sequence, kv head)
    w = synth.TINY.with_(kv_len=700)
    c = Case(w, seed=2, extra_cap=300)
    g = c.mk.graph()
    assert g.tiling[5] > 1  # attention splits
    got = c.gpu_step()
    ref = c.oracle_step(k=c.k.copy(), v=c.v.copy(), lens=c.lens.copy())
    compare_step(ref, got, w, "tiny-split")


@pytest.mark.parametrize("L", [0, 1, 63, 64, 65, 511])
def test_tiny_edge_lengths(L):
    # empty cache (only the new row), one cached row, and chunk boundaries
    w = synth.TINY.with_(kv_len=L)
    c = Case(w, seed=3, extra_cap=600 - L, attn_min_chunk=64)
    got = c.gpu_step()
    ref = c.oracle_step(k=c.k.copy(), v=c.v.copy(), lens=c.lens.copy())
    compare_step(ref, got, w, f"tiny-L{L}")


def test_persistent_and_per_operator_paths_are_bitwise_identical():
    w = synth.TINY.with_(kv_len=300)
    c = Case(w, seed=4, extra_cap=10)
    a = c.gpu_step()
    c.reset_device_state()
    b = c.gpu_step(perop=True)
    for key in ("tokens", "logits", "hidden", "kv_len"):
        np.testing.assert_array_equal(a[key], b[key])


def test_run_to_run_determinism_and_multi_step_lockstep():
    w = synth.TINY.with_(kv_len=40, steps=4)
    c = Case(w, seed=5)
    k, v, lens = c.k.copy(), c.v.copy(), c.lens.copy()
    tok = c.tokens.copy()
    for step in range(4):
        got = c.gpu_step(tokens=tok)
        ref = c.oracle_step(tokens=tok, k=k, v=v, lens=lens)
        compare_step(ref, got, w, f"step{step}")
        tok = ref["tokens"].copy()  # both sides continue from the oracle's token
    # determinism: replay from the same state twice
    c.reset_device_state()
    a = c.gpu_step()
    c.reset_device_state()
    b = c.gpu_step()
    np.testing.assert_array_equal(a["logits"], b["logits"])
    np.testing.assert_array_equal(a["hidden"], b["hidden"])


def test_qwen3_06b_step_matches_oracle():
    w = synth.Q06B
    c = Case(w, seed=0, extra_cap=8)
    k, v, lens = c.k.copy(), c.v.copy(), c.lens.copy()
    tok = c.tokens.copy()
    for step in range(2):
        got = c.gpu_step(tokens=tok)
        ref = c.oracle_step(tokens=tok, k=k, v=v, lens=lens)
        compare_step(ref, got, w, f"0.6b step{step}")
        tok = ref["tokens"].copy()
    kv_rows_close(c, k, v, c.lens + 1, untouched=c.lens)


def test_bad_inputs_are_rejected_and_write_nothing():
    import persistent_runtime_b200 as prb
    t = torch()
    w = synth.TINY
    c = Case(w, seed=6, extra_cap=1)
    c.d_len.fill_(c.cap)  # kv_len + 1 > capacity
    k0 = c.d_k.clone()
    c.mk.decode_step(c.d_tok, c.d_out, c.d_len, c.d_k, c.d_v, c.d_logits)
    rc, detail = c.mk.sync_status()
    assert rc == prb.MK_ERR_DEVICE
    assert int(c.d_len[0]) == c.cap and t.equal(c.d_k, k0)
    # later steps are no-ops until reset
    c.d_len.fill_(3)
    c.mk.decode_step(c.d_tok, c.d_out, c.d_len, c.d_k, c.d_v, c.d_logits)
    assert c.mk.sync_status()[0] == prb.MK_ERR_DEVICE and int(c.d_len[0]) == 3
    c.mk.reset()
    c.reset_device_state()
    c.d_tok.fill_(w.vocab)  # token out of range
    c.mk.decode_step(c.d_tok, c.d_out, c.d_len, c.d_k, c.d_v, c.d_logits)
    assert c.mk.sync_status()[0] == prb.MK_ERR_DEVICE
    c.mk.reset()
    c.reset_device_state()
    c.gpu_step()


def test_event_wait_times_out_cleanly_and_recovers():
    # Raising one event's trigger count by one makes its waiters time out:
    # the kernel must return an error status (no trap, no hang) and the
    # context must stay usable.
    import persistent_runtime_b200 as prb
    w = synth.TINY
    c = Case(w, seed=7)
    g = c.mk.graph()
    e = int(g.n_events // 2)
    c.mk.set_timeout_us(20000)
    c.mk.set_event_count(e, int(g.event_count[e]) + 1)
    c.mk.decode_step(c.d_tok, c.d_out, c.d_len, c.d_k, c.d_v, c.d_logits)
    rc, detail = c.mk.sync_status()
    assert rc == prb.MK_ERR_TIMEOUT, (rc, detail)
    assert detail[0] == prb.MK_ERR_TIMEOUT
    c.mk.set_event_count(e, int(g.event_count[e]))
    c.mk.set_timeout_us(2000000)
    c.mk.reset()
    c.reset_device_state()
    got = c.gpu_step()
    ref = c.oracle_step(k=c.k.copy(), v=c.v.copy(), lens=c.lens.copy())
    compare_step(ref, got, w, "after-timeout")


def test_qwen3_8b_bs1_full_size_step_matches_oracle():
    # The bench's workload and launch configuration: 36 layers, hidden 4096,
    # 151936 vocab, 1024 cached rows, capacity 1024 + 64, one CTA per SM.
    w = synth.Q8B
    c = Case(w, seed=0, extra_cap=64)
    assert c.mk.info().num_workers == torch().cuda.get_device_properties(0).multi_processor_count
    k, v, lens = c.k.copy(), c.v.copy(), c.lens.copy()
    got = c.gpu_step()
    ref = c.oracle_step(k=k, v=v, lens=lens)
    compare_step(ref, got, w, "8b")
    kv_rows_close(c, k, v, c.lens)


def test_misaligned_caches_are_rejected_on_the_host():
    # The host checks the cache pointers before any launch (bulk and tensor
    # copies need 16-byte alignment), so nothing runs on the GPU.
    import persistent_runtime_b200 as prb
    w = synth.TINY
    c = Case(w, seed=8)
    k_off = c.d_k.view(-1)[1:]  # 2 bytes past an aligned start
    with pytest.raises(prb.MkError) as ei:
        c.mk.decode_step(c.d_tok, c.d_out, c.d_len, k_off, c.d_v, c.d_logits)
    assert ei.value.status == prb.MK_ERR_ARG and "aligned" in str(ei.value)
    got = c.gpu_step()  # the handle is still usable
    assert (got["kv_len"] == c.lens + 1).all()
