"""Dispatch mode: a scheduler CTA in the same launch hands ready tasks to the
workers (the pages' scheduler design, kept as an ablation of the static
queues).  Task bodies do not depend on the SM that runs them, so a dispatch
handle (SMs - 1 workers) gives bitwise what a static handle built for the
same worker count gives, and both match the oracle."""
import numpy as np
import pytest

import synth
from gpu_helpers import Case, compare_step, kv_rows_close, torch

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("built_libs")]


def _sms():
    return torch().cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("w,bf16_inputs", [
    (synth.TINY.with_(kv_len=700), False),
    (synth.TINY.with_(name="tiny-b8", batch=8, kv_len=None, kv_len_range=(0, 300)), True),
    (synth.Q06B, False)], ids=["tiny-split", "tiny-batch8", "qwen3-0.6b"])
def test_dispatch_mode_matches_static_queues_and_oracle(w, bf16_inputs):
    W = _sms() - 1
    c = Case(w, seed=51, extra_cap=4, dispatch=1)
    assert c.mk.info().num_workers == W
    k, v, lens = c.k.copy(), c.v.copy(), c.lens.copy()
    got = c.gpu_step()
    ref = c.oracle_step(k=k, v=v, lens=lens)
    compare_step(ref, got, w, f"{w.name}-dispatch")
    kv_rows_close(c, k, v, c.lens, bf16_inputs=bf16_inputs)
    s = Case(w, seed=51, extra_cap=4, num_workers=W, weights=c.weights)
    other = s.gpu_step()
    for key in ("tokens", "logits", "hidden", "kv_len"):
        np.testing.assert_array_equal(got[key], other[key])


def test_dispatch_mode_runs_one_step_per_launch():
    import persistent_runtime_b200 as prb
    t = torch()
    w = synth.TINY.with_(kv_len=40, steps=2)
    c = Case(w, seed=52, extra_cap=4, dispatch=1)
    out = t.zeros((2, w.batch), dtype=t.int32, device="cuda")
    with pytest.raises(prb.MkError):
        c.mk.decode_steps(2, c.d_tok, out, c.d_len, c.d_k, c.d_v, c.d_logits)
    with pytest.raises(prb.MkError):
        c.mk.decode_step_noalloc(c.d_tok, c.d_out, c.d_len, c.d_k, c.d_v, c.d_logits)
    # consecutive single steps keep working (the queues are reset per launch)
    for _ in range(3):
        c.mk.decode_step(c.d_tok, c.d_tok, c.d_len, c.d_k, c.d_v, c.d_logits)
    assert c.mk.sync_status()[0] == 0
    assert int(c.d_len[0]) == 43
