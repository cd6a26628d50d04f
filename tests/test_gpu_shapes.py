"""Decoder shapes beyond the named workloads, at batch 1 (CUDA-core kernel)
and batch 3 (tensor-core kernel): q:kv head ratios 8, 1 and 3 (the kernels
pad the ratio to a power of two), a vocabulary that is not a multiple of 16
(the batched LM head pads its last 16-row tile), and hidden / FFN widths
that are multiples of 256 but not powers of two."""
import numpy as np
import pytest

import synth
from gpu_helpers import Case, compare_step, kv_rows_close

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("built_libs")]

SHAPES = {
    # name: (hidden, q heads, kv heads, head_dim, ffn, vocab)
    "rep8": (512, 8, 1, 64, 1024, 4096),
    "mha": (256, 4, 4, 64, 768, 4096),
    "rep3": (384 * 2, 6, 2, 128, 1280, 4001),
}


@pytest.mark.parametrize("batch", [1, 3])
@pytest.mark.parametrize("name", sorted(SHAPES))
def test_shape_step_matches_oracle(name, batch):
    H, hq, hkv, D, F, V = SHAPES[name]
    w = synth.Workload(f"shape-{name}-b{batch}", 2, H, hq, hkv, D, F, V, batch % 2, batch,
                       None, kv_len_range=(0, 150), steps=2)
    c = Case(w, seed=50 + batch)
    k, v, lens = c.k.copy(), c.v.copy(), c.lens.copy()
    got = c.gpu_step()
    ref = c.oracle_step(k=k, v=v, lens=lens)
    compare_step(ref, got, w, w.name)
    np.testing.assert_array_equal(got["kv_len"], c.lens + 1)
    kv_rows_close(c, k, v, c.lens, bf16_inputs=batch > 1)
    assert ((got["tokens"] >= 0) & (got["tokens"] < V)).all()
