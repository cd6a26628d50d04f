"""mk_decode_step_noalloc against mk_decode_step and the oracle, through the C ABI.

The allocation-free step is for callers that cannot call cudaMalloc when they
need another stepping context (a host program that hands out device memory
through its own allocator, or code that must not synchronise the device).  It
keeps its working buffers in the library's static device region and runs the
same kernel, with the same tiling and fixed-order reductions, as the ordinary
step on the same inputs, so two calls in a row must give bitwise what two calls
of the ordinary step give: tokens, logits, kv_len and both caches.  The first
step is also checked against the CPU oracle.  A batch-12 case runs after a call
of another shape, so the region's padding columns hold stale data.  This file
is collected last so that a stop at the first failure has run every other test
already; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest

import synth
from gpu_helpers import Case, check_tokens, compare_logits, rows_close, torch

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
    return (out, case.d_k.cpu().numpy().view(np.uint16).copy(),
            case.d_v.cpu().numpy().view(np.uint16).copy())


def _check(case):
    ref, ref_k, ref_v = _two_steps(case, case.mk.decode_step)
    got, got_k, got_v = _two_steps(case, case.mk.decode_step_noalloc)
    for a, b in zip(ref, got):
        for key in ("tokens", "logits", "kv_len"):
            np.testing.assert_array_equal(a[key], b[key])
    np.testing.assert_array_equal(got_k, ref_k)
    np.testing.assert_array_equal(got_v, ref_v)
    # the first step against the oracle (logits, token and appended rows)
    k, v, kl = case.k.copy(), case.v.copy(), case.lens.copy()
    oracle_ref = case.oracle_step(k=k, v=v, lens=kl)
    first, first_k, first_v = _first_step(case)
    compare_logits(oracle_ref, first["logits"], case.w, "noalloc")
    check_tokens(oracle_ref, first["tokens"], case.w, "noalloc")
    rows_close(first_k, first_v, k, v, case.lens, bf16_inputs=case.w.batch > 1, ctx="noalloc")


def _first_step(case):
    case.reset_device_state()
    case.mk.decode_step_noalloc(case.d_tok, case.d_out, case.d_len, case.d_k, case.d_v,
                                case.d_logits)
    rc, detail = case.mk.sync_status()
    assert rc == 0, (rc, detail)
    return ({"tokens": case.d_out.cpu().numpy(), "logits": case.d_logits.cpu().numpy()},
            case.d_k.cpu().numpy().view(np.uint16), case.d_v.cpu().numpy().view(np.uint16))


@pytest.mark.parametrize("w", [synth.TINY.with_(kv_len=300), synth.Q06B,
                               synth.TINY.with_(batch=5, kv_len=None, kv_len_range=(0, 300))],
                         ids=["tiny-split", "qwen3-0.6b", "tiny-batch5"])
def test_noalloc_step_matches_decode_step_twice(w):
    _check(Case(w, seed=21, extra_cap=4))


def test_noalloc_batch12_after_another_shape():
    # a batch-5 call first fills the region with another layout; the batch-12
    # handle (two 8-sequence operand tiles, four padding columns) must still
    # match the ordinary step bitwise
    other = Case(synth.TINY.with_(batch=5, kv_len=None, kv_len_range=(0, 300)), seed=22,
                 extra_cap=4)
    _first_step(other)
    other.mk.close()
    _check(Case(synth.TINY.with_(batch=12, kv_len=None, kv_len_range=(0, 200)), seed=23,
                extra_cap=4))


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
