"""Paged K/V pools (mk_decode_steps_paged) against the contiguous layout.

The same seeded inputs run through a handle built for contiguous caches and
one built with kv_page_size = P.  The pools hold the cache rows in pages
scattered by a random permutation (with spare pages); results must be
bitwise those of the contiguous run (the stage partition is the same in
these cases, so is the arithmetic), the appended rows must land in the right
pages, and the oracle, replaying the steps with the GPU's tokens, must agree
with every step's token, every appended row and the last step's logits and
hidden state."""
import numpy as np
import pytest

import synth
from gpu_helpers import Case, dev_u16, lockstep_oracle, torch

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("built_libs")]

P = 64


def to_pool(cache, P, seed, spare=3):
    """[Ly][B][Hkv][cap][D] -> pool [n_pages][Ly][Hkv][P][D] and table [B][max_pages]."""
    Ly, B, Hkv, cap, D = cache.shape
    mp = -(-cap // P)
    n_pages = B * mp + spare
    perm = np.random.default_rng(seed).permutation(n_pages).astype(np.int32)
    table = perm[:B * mp].reshape(B, mp).copy()
    pool = np.zeros((n_pages, Ly, Hkv, P, D), dtype=np.uint16)
    for b in range(B):
        for j in range(mp):
            rows = cache[:, b, :, j * P:(j + 1) * P, :]
            pool[table[b, j], :, :, :rows.shape[2], :] = rows
    return pool, table, n_pages


def from_pool(pool, table, cap):
    n_pages, Ly, Hkv, P, D = pool.shape
    B, mp = table.shape
    out = np.zeros((Ly, B, Hkv, mp * P, D), dtype=np.uint16)
    for b in range(B):
        for j in range(mp):
            out[:, b, :, j * P:(j + 1) * P, :] = pool[table[b, j]]
    return out[:, :, :, :cap, :]


def run_pair(w, seed, n_steps, against_oracle=False):
    t = torch()
    ref = Case(w, seed=seed)
    out_r = t.zeros((n_steps, w.batch), dtype=t.int32, device="cuda")
    ref.mk.decode_steps(n_steps, ref.d_tok, out_r, ref.d_len, ref.d_k, ref.d_v, ref.d_logits)
    assert ref.mk.sync_status()[0] == 0
    pg = Case(w, seed=seed, kv_page_size=P)
    kp, table, n_pages = to_pool(pg.k, P, seed)
    vp, _, _ = to_pool(pg.v, P, seed)
    d_kp, d_vp = dev_u16(kp), dev_u16(vp)
    d_table = t.from_numpy(table).cuda()
    out_p = t.zeros((n_steps, w.batch), dtype=t.int32, device="cuda")
    pg.mk.decode_steps_paged(n_steps, pg.d_tok, out_p, pg.d_len, d_kp, d_vp, n_pages, d_table,
                             pg.d_logits)
    rc, detail = pg.mk.sync_status()
    assert rc == 0, (rc, detail)
    np.testing.assert_array_equal(out_p.cpu().numpy(), out_r.cpu().numpy())
    np.testing.assert_array_equal(pg.d_logits.cpu().numpy(), ref.d_logits.cpu().numpy())
    np.testing.assert_array_equal(pg.d_len.cpu().numpy(), ref.d_len.cpu().numpy())
    np.testing.assert_array_equal(pg.gpu_hidden(), ref.gpu_hidden())
    cap = ref.cap
    kk = from_pool(d_kp.cpu().numpy().view(np.uint16), table, cap)
    vv = from_pool(d_vp.cpu().numpy().view(np.uint16), table, cap)
    np.testing.assert_array_equal(kk, ref.d_k.cpu().numpy().view(np.uint16))
    np.testing.assert_array_equal(vv, ref.d_v.cpu().numpy().view(np.uint16))
    if against_oracle:
        last = {"tokens": out_p.cpu().numpy()[-1], "logits": pg.d_logits.cpu().numpy(),
                "hidden": pg.gpu_hidden(), "kv_len": pg.d_len.cpu().numpy()}
        lockstep_oracle(pg, out_p.cpu().numpy(), last, kk, vv, w.batch > 1, "paged")
    return pg, d_kp, d_vp, d_table, n_pages


@pytest.mark.parametrize("w,n", [(synth.TINY.with_(kv_len=150, steps=3), 1),
                                 (synth.TINY.with_(name="tiny-b3", batch=3, kv_len=None,
                                                   kv_len_range=(0, 300), steps=3), 3),
                                 (synth.Q06B.with_(steps=3), 3)],
                         ids=["tiny", "tiny-batch3-split", "qwen3-0.6b"])
def test_paged_equals_contiguous_bitwise_and_matches_oracle(w, n):
    run_pair(w, 61, n, against_oracle=True)


def test_paged_rejects_bad_tables_and_wrong_entry_points():
    import persistent_runtime_b200 as prb
    t = torch()
    w = synth.TINY.with_(kv_len=100, steps=2)
    pg, d_kp, d_vp, d_table, n_pages = run_pair(w, 62, 1)
    pg.reset_device_state()
    k0 = d_kp.clone()
    bad = d_table.clone()
    bad[0, 1] = n_pages  # a page the pools do not have, under a used position
    out = t.zeros((1, w.batch), dtype=t.int32, device="cuda")
    pg.mk.decode_steps_paged(1, pg.d_tok, out, pg.d_len, d_kp, d_vp, n_pages, bad, pg.d_logits)
    assert pg.mk.sync_status()[0] == prb.MK_ERR_DEVICE
    assert t.equal(d_kp, k0) and int(pg.d_len[0]) == 100
    pg.mk.reset()
    with pytest.raises(prb.MkError):  # a paged handle has no contiguous step
        pg.mk.decode_step(pg.d_tok, pg.d_out, pg.d_len, pg.d_k, pg.d_v, pg.d_logits)
    with pytest.raises(prb.MkError):
        pg.mk.decode_step_noalloc(pg.d_tok, pg.d_out, pg.d_len, pg.d_k, pg.d_v, pg.d_logits)
