"""The run-time (JIT) partition of attention work, restated from its rule and
checked for the properties the kernel relies on (host only, no device).

Rule: the pairs (b, g), b < B, g < Hkv, each with n_b = L_b + 1 positions (the
cached rows and the new one), lie end to end on one line of T positions in
order b * Hkv + g; A tasks each take C consecutive positions, C = the larger of
ceil(T / A) and ceil(max n_b / (S - 1)), rounded up to 16, where S =
ceil(A / (B * Hkv)) + 2 is the number of partial slots per pair.  A task's
pieces are the pairs its positions fall in; the piece of pair p in task a is
partial slot a - floor(P_p / C) of the floor((P_p + n_p - 1) / C) -
floor(P_p / C) + 1 tasks that touch p (P_p: the line position of p's row 0).
"""
import math

import numpy as np
import pytest

import persistent_runtime_b200 as prb
import synth


def partition(lens, Hkv, A):
    B = len(lens)
    S = math.ceil(A / (B * Hkv)) + 2
    n = [int(L) + 1 for L in lens]
    T = sum(x * Hkv for x in n)
    C = max(math.ceil(T / A), math.ceil(max(n) / (S - 1)))
    C = (C + 15) // 16 * 16
    pieces = []  # (task, b, g, r0, r1, slot, expect)
    P = 0
    for b in range(B):
        for g in range(Hkv):
            first, last = P // C, (P + n[b] - 1) // C
            for a in range(first, last + 1):
                r0 = max(0, a * C - P)
                r1 = min(n[b], (a + 1) * C - P)
                pieces.append((a, b, g, r0, r1, a - first, last - first + 1))
            P += n[b]
    return pieces, S, C, T


@pytest.mark.parametrize("seed", range(200))
def test_jit_pieces_cover_every_position_once_within_the_slot_bound(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(2, 17))
    Hkv = int(rng.choice([1, 2, 8]))
    A = int(rng.choice([1, 7, 64, 148, 296]))
    kind = seed % 4
    if kind == 0:
        lens = rng.integers(0, 9000, B)
    elif kind == 1:
        lens = np.full(B, int(rng.integers(0, 9000)))
    elif kind == 2:  # one long sequence among empty ones
        lens = np.zeros(B, dtype=int)
        lens[int(rng.integers(0, B))] = int(rng.integers(1000, 9000))
    else:
        lens = rng.integers(0, 40, B)
    pieces, S, C, T = partition(lens, Hkv, A)
    assert C % 16 == 0 and C * A >= T
    covered = {}
    for a, b, g, r0, r1, slot, expect in pieces:
        assert 0 <= a < A
        assert 0 <= r0 < r1 <= lens[b] + 1
        assert 0 <= slot < expect <= S
        covered.setdefault((b, g), []).append((r0, r1, slot, expect))
    for b in range(B):
        for g in range(Hkv):
            segs = sorted(covered[(b, g)])
            assert segs[0][0] == 0 and segs[-1][1] == lens[b] + 1
            for (x0, x1, _, _), (y0, _, _, _) in zip(segs, segs[1:]):
                assert x1 == y0  # contiguous, no overlap
            assert [s[2] for s in segs] == list(range(len(segs)))  # slots 0 .. expect-1
            assert all(s[3] == len(segs) for s in segs)  # every piece knows the count
            # exactly one piece holds the new row (position L_b)
            assert sum(1 for s in segs if s[1] == lens[b] + 1) == 1
    # every task's work is at most C positions
    work = np.zeros(A, dtype=int)
    for a, b, g, r0, r1, _, _ in pieces:
        work[a] += r1 - r0
    assert work.max() <= C


def test_jit_spreads_equal_long_pairs_over_all_workers():
    # 16 sequences x 8 kv heads at 8192 cached rows on 148 workers: every task
    # gets the same share (to 16 positions), where fixed splits give 128 tasks
    pieces, S, C, T = partition(np.full(16, 8192), 8, 148)
    work = np.zeros(148, dtype=int)
    for a, b, g, r0, r1, _, _ in pieces:
        work[a] += r1 - r0
    assert work.max() - work[work > 0].min() <= 16 * 128
    assert (work > 0).sum() >= 147


def test_library_exports_the_jit_tiling():
    # JIT attention (opt-in, batch >= 2): apw * W tasks per layer,
    # S = ceil(apw W / (B Hkv)) + 2 partial slots, chunk 0
    w = synth.Q8B_B16
    g = prb.plan_graph(w, 8224, 148, attn_jit=1)
    assert g.tiling[5] == math.ceil(148 / 128) + 2 and g.tiling[6] == 0
    types, layers = np.asarray(g.task_type), np.asarray(g.task_layer)
    assert int(np.sum((types == 3) & (layers == 0))) == 148
    assert prb.plan_graph(w, 8224, 148).tiling[6] > 0  # default: splits fixed at build time
