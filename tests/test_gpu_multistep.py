"""mk_decode_steps: n decode steps in one persistent launch with the token fed
back on the device, against n calls of mk_decode_step (bitwise) and the CPU
oracle (each step fed the token the GPU chose)."""
import numpy as np
import pytest

import synth
from gpu_helpers import Case, lockstep_oracle, torch

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("built_libs")]


def _run_steps(c, n):
    t = torch()
    c.reset_device_state()
    out = t.zeros((n, c.w.batch), dtype=t.int32, device="cuda")
    c.mk.decode_steps(n, c.d_tok, out, c.d_len, c.d_k, c.d_v, c.d_logits)
    rc, detail = c.mk.sync_status()
    assert rc == 0, (rc, detail)
    return (out.cpu().numpy(), c.d_logits.cpu().numpy(), c.d_len.cpu().numpy(),
            c.d_k.cpu().numpy(), c.d_v.cpu().numpy())


def _run_single(c, n):
    t = torch()
    c.reset_device_state()
    toks = []
    for _ in range(n):
        c.mk.decode_step(c.d_tok, c.d_tok, c.d_len, c.d_k, c.d_v, c.d_logits)
        toks.append(c.d_tok.cpu().numpy().copy())
    rc, detail = c.mk.sync_status()
    assert rc == 0, (rc, detail)
    return (np.stack(toks), c.d_logits.cpu().numpy(), c.d_len.cpu().numpy(),
            c.d_k.cpu().numpy(), c.d_v.cpu().numpy())


@pytest.mark.parametrize("w,tuning", [(synth.TINY.with_(kv_len=40, steps=6), {}),
                                      (synth.TINY.with_(name="tiny-b5", batch=5, kv_len=None,
                                                        kv_len_range=(0, 300), steps=6), {}),
                                      (synth.Q06B.with_(steps=4), {}),
                                      # the attention-window L2 prefetch, off by default
                                      # for layers this small: its cursor restarts
                                      # with every step of the launch
                                      (synth.Q06B.with_(steps=4), {"l2_prefetch_bytes": 1 << 20})],
                         ids=["tiny", "tiny-batch5-split", "qwen3-0.6b", "qwen3-0.6b-prefetch"])
def test_multistep_equals_single_steps_bitwise(w, tuning):
    n = w.steps
    c = Case(w, seed=41, **tuning)
    a = _run_steps(c, n)
    b = _run_single(c, n)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    np.testing.assert_array_equal(a[2], c.lens + n)


@pytest.mark.parametrize("w,bf16_inputs,tuning", [
    (synth.TINY.with_(kv_len=20, steps=4), False, {}),
    (synth.TINY.with_(name="tiny-b5", batch=5, kv_len=None, kv_len_range=(0, 300), steps=4), True, {}),
    (synth.TINY.with_(name="tiny-b5", batch=5, kv_len=None, kv_len_range=(0, 300), steps=4), True,
     {"attn_jit": 1})],
    ids=["tiny", "tiny-batch5-split", "tiny-batch5-jit"])
def test_multistep_matches_oracle_stepwise(w, bf16_inputs, tuning):
    # the oracle replays the launch's steps fed with the tokens the GPU chose:
    # every step's token and appended K/V rows, and the last step's logits and
    # hidden state, agree within the step tolerances (with JIT attention the
    # pieces are recut from the lengths every step)
    n = w.steps
    c = Case(w, seed=42, **tuning)
    toks, logits, lens, gk, gv = _run_steps(c, n)
    last = {"tokens": toks[-1], "logits": logits, "hidden": c.gpu_hidden(), "kv_len": lens}
    lockstep_oracle(c, toks, last, gk.view(np.uint16), gv.view(np.uint16), bf16_inputs, "multistep")
    np.testing.assert_array_equal(lens, c.lens + n)


def test_multistep_rejects_steps_past_the_capacity():
    import persistent_runtime_b200 as prb
    t = torch()
    w = synth.TINY.with_(kv_len=40, steps=2)
    c = Case(w, seed=43, extra_cap=2)
    out = t.zeros((3, w.batch), dtype=t.int32, device="cuda")
    k0 = c.d_k.clone()
    c.mk.decode_steps(3, c.d_tok, out, c.d_len, c.d_k, c.d_v, c.d_logits)  # 40 + 3 > 42
    rc, _ = c.mk.sync_status()
    assert rc == prb.MK_ERR_DEVICE
    assert t.equal(c.d_k, k0) and int(c.d_len[0]) == 40
    c.mk.reset()
