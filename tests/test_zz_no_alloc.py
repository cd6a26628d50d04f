"""mk_decode_step_noalloc against mk_decode_step, through the C ABI.

The allocation-free step keeps its working buffers in the library's static
device region (for callers that cannot call cudaMalloc when they need another
stepping context).  Two calls in a row must give what two calls of the
ordinary step give, within the tolerances of the other parity tests.  This file
is collected last so that a stop at the first failure has run every other test
already; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest

import synth
from gpu_helpers import LOGIT_TOL, Case, torch

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("built_libs")]


def _two_steps(case, fn):
    t = torch()
    case.reset_device_state()
    out = []
    for _ in range(2):
        fn(case.d_tok, case.d_tok, case.d_len, case.d_k, case.d_v, case.d_logits)
        rc, detail = case.mk.sync_status()
        assert rc == 0, (rc, detail)
        out.append({"tokens": case.d_tok.cpu().numpy().copy(),
                    "logits": case.d_logits.cpu().numpy().copy(),
                    "kv_len": case.d_len.cpu().numpy().copy()})
    t.cuda.synchronize()
    return out, case.d_k.cpu().numpy().copy(), case.d_v.cpu().numpy().copy()


@pytest.mark.parametrize("w", [synth.TINY.with_(kv_len=300), synth.Q06B,
                               synth.TINY.with_(batch=5, kv_len=None, kv_len_range=(0, 300))],
                         ids=["tiny-split", "qwen3-0.6b", "tiny-batch5"])
def test_noalloc_step_matches_decode_step_twice(w):
    c = Case(w, seed=21, extra_cap=4)
    ref, ref_k, ref_v = _two_steps(c, c.mk.decode_step)
    got, got_k, got_v = _two_steps(c, c.mk.decode_step_noalloc)
    for a, b in zip(ref, got):
        np.testing.assert_array_equal(a["tokens"], b["tokens"])
        np.testing.assert_array_equal(a["kv_len"], b["kv_len"])
        scale = np.max(np.abs(a["logits"]))
        assert np.max(np.abs(a["logits"] - b["logits"])) <= LOGIT_TOL * scale
    kg = synth.bf16_to_f32(got_k.view(np.uint16)).astype(np.float64)
    kr = synth.bf16_to_f32(ref_k.view(np.uint16)).astype(np.float64)
    vg = synth.bf16_to_f32(got_v.view(np.uint16)).astype(np.float64)
    vr = synth.bf16_to_f32(ref_v.view(np.uint16)).astype(np.float64)
    assert np.max(np.abs(kg - kr)) <= 1e-2 * np.max(np.abs(kr))
    assert np.max(np.abs(vg - vr)) <= 1e-2 * np.max(np.abs(vr))


def test_noalloc_rejects_steps_beyond_the_static_region():
    import persistent_runtime_b200 as prb
    # 36 8B-shaped layers with a 60000-row cache and 4 attention tasks per
    # worker (73 splits per head): the split partials alone need about 43 MiB,
    # more than the 16 MiB region; the size is checked before anything else,
    # so no weights are needed
    w = synth.Q8B.with_(kv_len=60000)
    t = torch()
    mk = prb.Megakernel(w, 60004, 0, attn_tasks_per_worker=4)
    buf = t.zeros(8, dtype=t.int32, device="cuda")
    with pytest.raises(prb.MkError) as ei:
        mk.decode_step_noalloc(buf, buf, buf, buf, buf)
    assert ei.value.status == prb.MK_ERR_ARG
    assert "static region" in str(ei.value)
    mk.close()
