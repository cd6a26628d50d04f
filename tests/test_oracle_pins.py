"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks a closed form, an invariant, a special case that reduces to a
textbook result, or brute force in float64 on tiny inputs.  Together they are
chosen so that a dropped term, a wrong sign or index, or a transposed operand
in the oracle fails at least one of them.
"""
import math

import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.usefixtures("built_libs")

rng = np.random.default_rng(1234)


def bf16_exact(x):
    """Round float64 data to bf16 bit patterns (via float32, as the generator does)."""
    return synth.f32_to_bf16(np.asarray(x, dtype=np.float32))


# --------------------------------------------------------------------------- RMSNorm
def test_rmsnorm_constant_vector_closed_form():
    # x = c (constant): mean(x^2) = c^2, so y_i = g_i * c / sqrt(c^2 + eps).
    n, eps = 512, 1e-6
    g = bf16_exact(1 + 0.1 * rng.standard_normal(n))
    for c in (3.0, -0.25, 1e-4):
        y = oracle.rmsnorm(np.full(n, c), g, eps)
        expect = synth.bf16_to_f32(g).astype(np.float64) * c / math.sqrt(c * c + eps)
        np.testing.assert_allclose(y, expect, rtol=2e-6, atol=0)


def test_rmsnorm_scale_invariance_and_unit_rms():
    n, eps = 1024, 1e-6
    x = rng.standard_normal(n).astype(np.float32)
    ones = bf16_exact(np.ones(n))
    y1 = oracle.rmsnorm(x, ones, eps)
    y2 = oracle.rmsnorm(8.0 * x, ones, eps)  # power of two: x scales exactly
    np.testing.assert_allclose(y1, y2, rtol=1e-5, atol=1e-7)
    # with unit gain the output has root-mean-square 1 (up to eps)
    assert abs(math.sqrt(float(np.mean(y1.astype(np.float64) ** 2))) - 1.0) < 1e-5


# --------------------------------------------------------------------------- RoPE
def test_rope_position_zero_is_identity():
    v = rng.standard_normal(128).astype(np.float32)
    np.testing.assert_array_equal(oracle.rope(v, 0, 1e6), v)


def test_rope_preserves_pair_norms_and_inverts():
    D, theta = 128, 1e6
    v = rng.standard_normal(D).astype(np.float32)
    for pos in (1, 17, 1023, 8191):
        r = oracle.rope(v, pos, theta).astype(np.float64)
        half = D // 2
        n0 = np.hypot(v[:half].astype(np.float64), v[half:].astype(np.float64))
        n1 = np.hypot(r[:half], r[half:])
        np.testing.assert_allclose(n1, n0, rtol=1e-6)
        back = oracle.rope(r.astype(np.float32), -pos, theta)
        np.testing.assert_allclose(back, v, rtol=1e-5, atol=1e-5)


def test_rope_rotation_angle_per_pair():
    # Pair i = (i, i + D/2) rotates counter-clockwise by pos * theta^(-2i/D).
    D, theta, pos = 64, 1e6, 5
    half = D // 2
    v = np.zeros(D, dtype=np.float32)
    v[:half] = 1.0  # each pair starts at angle 0
    r = oracle.rope(v, pos, theta).astype(np.float64)
    measured = np.arctan2(r[half:], r[:half])
    for i in range(half):
        want = math.remainder(pos * theta ** (-2.0 * i / D), 2 * math.pi)
        assert abs(math.remainder(measured[i] - want, 2 * math.pi)) < 1e-6, i


def test_rope_scores_depend_only_on_relative_position():
    D, theta = 128, 1e6
    q = rng.standard_normal(D).astype(np.float32)
    k = rng.standard_normal(D).astype(np.float32)
    a = float(np.dot(oracle.rope(q, 100, theta).astype(np.float64),
                     oracle.rope(k, 90, theta).astype(np.float64)))
    b = float(np.dot(oracle.rope(q, 1010, theta).astype(np.float64),
                     oracle.rope(k, 1000, theta).astype(np.float64)))
    assert abs(a - b) < 1e-4 * (abs(a) + 1)


# --------------------------------------------------------------------------- attention
def test_attention_single_row_returns_v_exactly():
    D = 128
    q = rng.standard_normal((4, D)).astype(np.float32)
    k = bf16_exact(rng.standard_normal((1, D)))
    v = bf16_exact(rng.standard_normal((1, D)))
    out = oracle.attention(q, k, v)
    for h in range(4):
        np.testing.assert_array_equal(out[h], synth.bf16_to_f32(v[0]))


def test_attention_equal_keys_give_mean_of_v():
    D, n = 64, 37
    q = rng.standard_normal((2, D)).astype(np.float32)
    krow = bf16_exact(rng.standard_normal(D))
    k = np.tile(krow, (n, 1))
    v = bf16_exact(rng.standard_normal((n, D)))
    out, probs = oracle.attention(q, k, v, want_probs=True)
    np.testing.assert_allclose(probs, 1.0 / n, rtol=1e-6)
    mean = synth.bf16_to_f32(v).astype(np.float64).mean(axis=0)
    for h in range(2):
        np.testing.assert_allclose(out[h], mean, rtol=1e-5, atol=1e-6)


def test_attention_probabilities_two_rows_closed_form():
    # Scores s = (q . k_j) / sqrt(D): with q = sqrt(D) e_0 and k_j = (c_j, 0, ...),
    # s_j = c_j, so p = (1, e^{c1 - c0}) / (1 + e^{c1 - c0}).
    D = 64
    q = np.zeros((1, D), dtype=np.float32)
    q[0, 0] = math.sqrt(D)
    k = np.zeros((2, D), dtype=np.uint16)
    c0, c1 = 0.5, 2.0  # both exact in bf16
    k[0, 0], k[1, 0] = bf16_exact([c0])[0], bf16_exact([c1])[0]
    v = np.zeros((2, D), dtype=np.uint16)
    v[0, 1], v[1, 1] = bf16_exact([1.0])[0], bf16_exact([-3.0])[0]
    out, probs = oracle.attention(q, k, v, want_probs=True)
    p1 = math.exp(c1 - c0) / (1 + math.exp(c1 - c0))
    np.testing.assert_allclose(probs[0], [1 - p1, p1], rtol=1e-6)
    np.testing.assert_allclose(out[0, 1], (1 - p1) * 1.0 + p1 * -3.0, rtol=1e-6)
    assert out[0, 0] == 0.0


def test_attention_matches_float64_brute_force():
    for n_pos, nh, D in ((1, 1, 16), (5, 2, 64), (64, 4, 128)):
        q = rng.standard_normal((nh, D)).astype(np.float32)
        k = bf16_exact(rng.standard_normal((n_pos, D)))
        v = bf16_exact(rng.standard_normal((n_pos, D)))
        out, probs = oracle.attention(q, k, v, want_probs=True)
        kf = synth.bf16_to_f32(k).astype(np.float64)
        vf = synth.bf16_to_f32(v).astype(np.float64)
        for h in range(nh):
            s = kf @ q[h].astype(np.float64) / math.sqrt(D)
            p = np.exp(s - s.max())
            p /= p.sum()
            np.testing.assert_allclose(probs[h], p, rtol=1e-5, atol=1e-7)
            np.testing.assert_allclose(out[h], p @ vf, rtol=1e-5, atol=1e-6)
            assert abs(float(probs[h].astype(np.float64).sum()) - 1.0) < 1e-6


# --------------------------------------------------------------------------- GEMV, SiLU, argmax
def test_gemv_one_hot_returns_weight_column():
    N, K = 48, 4096
    w = bf16_exact(0.02 * rng.standard_normal((N, K)))
    for j in (0, 1, 2047, K - 1):
        x = np.zeros(K, dtype=np.float32)
        x[j] = 1.0
        np.testing.assert_array_equal(oracle.gemv(w, x), synth.bf16_to_f32(w[:, j]))


def test_gemv_matches_float64_dot_and_orientation():
    N, K = 40, 12288
    w = bf16_exact(0.02 * rng.standard_normal((N, K)))
    x = rng.standard_normal(K).astype(np.float32)
    y = oracle.gemv(w, x)
    ref = synth.bf16_to_f32(w).astype(np.float64) @ x.astype(np.float64)
    np.testing.assert_allclose(y, ref, rtol=1e-4, atol=2e-5)


def test_silu_special_values_and_odd_identity():
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(40.0) - 40.0) < 1e-5
    assert abs(oracle.silu(-40.0)) < 1e-12
    # silu(x) - silu(-x) = x * (sigmoid(x) + sigmoid(-x)) = x
    for x in (0.3, 1.7, -2.5, 6.0):
        assert abs((oracle.silu(x) - oracle.silu(-x)) - x) < 1e-6 * max(1, abs(x))
    assert abs(oracle.silu(1.0) - 1.0 / (1.0 + math.exp(-1.0))) < 1e-7


def test_argmax_planted_and_ties():
    v = rng.standard_normal(151936).astype(np.float32)
    v[123457] = 100.0
    assert oracle.argmax(v) == 123457
    v[99] = 100.0
    assert oracle.argmax(v) == 99  # tie resolves to the lowest index
    assert oracle.argmax(np.full(7, -1.0)) == 0


def test_bf16_rounding_is_nearest_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even mantissa.
    assert oracle.round_bf16(1.0 + 2 ** -8) == 0x3F80
    assert oracle.round_bf16(1.0 + 3 * 2 ** -8) == 0x3F82
    assert oracle.round_bf16(1.0 + 2 ** -8 + 2 ** -20) == 0x3F81
    assert oracle.round_bf16(-2.0) == 0xC000


# --------------------------------------------------------------------------- whole step
def _zero_mixing(weights):
    for lw in weights["layers"]:
        for name in ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down"):
            lw[name] = np.zeros_like(lw[name])
    return weights


def _run_step(w, weights, seed=0, kv_lens=None):
    lens = w.kv_lens(seed) if kv_lens is None else kv_lens
    cap = int(lens.max()) + w.steps
    k, v = synth.make_kv(w, lens, cap, seed)
    tok = synth.make_tokens(w, seed)
    m = oracle.Model(w, weights, cap)
    kl = lens.copy()
    out = m.step(tok, kl, k, v)
    return tok, lens, kl, k, v, out


def test_step_with_zero_mixing_keeps_embedding_and_appends_zero_rows():
    w = synth.TINY.with_(batch=2)
    weights = _zero_mixing(synth.make_weights(w, 3))
    tok, lens, kl, k, v, out = _run_step(w, weights, seed=3)
    np.testing.assert_array_equal(kl, lens + 1)
    for b in range(w.batch):
        # residual stream = float(E[token]) exactly: every projection adds 0
        np.testing.assert_array_equal(out["hidden"][b], synth.bf16_to_f32(weights["embed"][tok[b]]))
        for l in range(w.n_layers):  # +0 or -0: the zero vector, rotated
            assert not synth.bf16_to_f32(k[l, b, :, lens[b]]).any()
            assert not synth.bf16_to_f32(v[l, b, :, lens[b]]).any()
        x = out["hidden"][b].astype(np.float64)
        xn = synth.bf16_to_f32(weights["final_norm"]) * x / math.sqrt(np.mean(x * x) + w.rms_eps)
        logits = synth.bf16_to_f32(weights["lm_head"]).astype(np.float64) @ xn
        np.testing.assert_allclose(out["logits"][b], logits, rtol=1e-4, atol=1e-6)
        assert out["tokens"][b] == int(np.argmax(out["logits"][b]))


def test_step_tied_head_with_equal_norm_rows_returns_input_token():
    # E rows are distinct +-1 vectors (equal norms), unit final gain, no mixing:
    # logits_j = E_j . E_t / rms is maximal only at j = t (Cauchy-Schwarz).
    w = synth.TINY.with_(tied_embeddings=1, batch=3)
    weights = _zero_mixing(synth.make_weights(w, 5))
    signs = np.where(rng.standard_normal((w.vocab, w.hidden)) > 0, 1.0, -1.0)
    weights["embed"] = bf16_exact(signs)
    weights["lm_head"] = None
    weights["final_norm"] = bf16_exact(np.ones(w.hidden))
    tok, _, _, _, _, out = _run_step(w, weights, seed=5)
    np.testing.assert_array_equal(out["tokens"], tok)


def test_step_gqa_uniform_attention_through_permuted_o_projection():
    # Zero K/V projections and zero cached keys make every score 0, so each q
    # head averages the L cached V rows of its kv head and the new (zero) row:
    # o_h = c_{g(h)} * L / (L + 1) where every cached V row of kv head g holds c_g.
    # W_o is a permutation (y_n = o_{pi(n)}), the MLP is zero, so the hidden
    # state is E[t] + sum over layers of the permuted o.
    w = synth.TINY
    L = int(w.kv_len)
    cap = L + 1
    weights = _zero_mixing(synth.make_weights(w, 7))
    H, qd, D, rep = w.hidden, w.q_dim, w.head_dim, w.n_q_heads // w.n_kv_heads
    perm = rng.permutation(qd)
    for lw in weights["layers"]:
        wo = np.zeros((H, qd), dtype=np.float32)
        wo[np.arange(H), perm] = 1.0
        lw["wo"] = bf16_exact(wo)
    consts = {}
    k = np.zeros((w.n_layers, 1, w.n_kv_heads, cap, D), dtype=np.uint16)
    v = np.zeros_like(k)
    for l in range(w.n_layers):
        for g in range(w.n_kv_heads):
            c = [0.5, -1.25, 2.0, 0.75][(l * w.n_kv_heads + g) % 4]
            consts[(l, g)] = c
            v[l, 0, g, :L, :] = bf16_exact([c])[0]
    tok = synth.make_tokens(w, 7)
    kl = np.array([L], dtype=np.int32)
    out = oracle.Model(w, weights, cap).step(tok, kl, k, v)
    expect = synth.bf16_to_f32(weights["embed"][tok[0]]).astype(np.float64)
    for l in range(w.n_layers):
        o = np.zeros(qd)
        for h in range(w.n_q_heads):
            o[h * D:(h + 1) * D] = consts[(l, h // rep)] * L / (L + 1)
        expect = expect + o[perm]
    np.testing.assert_allclose(out["hidden"][0], expect, rtol=1e-6, atol=1e-6)


def test_step_new_key_is_rotated_to_position_kv_len():
    # E[t] = 1 (constant), unit attention gain, W_k = [I | 0]: k = x_hat is a
    # constant vector, the k-norm with unit gain keeps it constant, so every
    # rotate-half pair (c, c) of the stored key starts at angle pi/4 and must
    # end at angle pi/4 + pos * theta^(-2i/D) with pos = kv_len.
    w = synth.TINY
    weights = _zero_mixing(synth.make_weights(w, 9))
    D, H = w.head_dim, w.hidden
    tok = synth.make_tokens(w, 9)
    weights["embed"] = weights["embed"].copy()
    weights["embed"][tok[0]] = bf16_exact(np.ones(H))
    for lw in weights["layers"]:
        lw["attn_norm"] = bf16_exact(np.ones(H))
        lw["k_norm"] = bf16_exact(np.ones(D))
        wk = np.zeros((w.kv_dim, H), dtype=np.float32)
        wk[np.arange(w.kv_dim), np.arange(w.kv_dim)] = 1.0
        lw["wk"] = bf16_exact(wk)
    L = 21
    cap = L + 1
    k = np.zeros((w.n_layers, 1, w.n_kv_heads, cap, D), dtype=np.uint16)
    v = np.zeros_like(k)
    kl = np.array([L], dtype=np.int32)
    oracle.Model(w, weights, cap).step(tok, kl, k, v)
    half = D // 2
    for l in range(w.n_layers):
        for g in range(w.n_kv_heads):
            row = synth.bf16_to_f32(k[l, 0, g, L]).astype(np.float64)
            ang = np.arctan2(row[half:], row[:half])
            for i in range(half):
                want = math.pi / 4 + L * w.rope_theta ** (-2.0 * i / D)
                assert abs(math.remainder(ang[i] - want, 2 * math.pi)) < 2e-2, (l, g, i)
            np.testing.assert_allclose(np.hypot(row[:half], row[half:]), math.sqrt(2), rtol=1e-2)


def _numpy_step_f64(w, weights, tok, lens, k, v):
    """Independent float64 restatement of the decode step, vectorised per layer."""
    f = lambda a: synth.bf16_to_f32(a).astype(np.float64)
    B, D, Hq, Hkv = w.batch, w.head_dim, w.n_q_heads, w.n_kv_heads
    rep = Hq // Hkv
    eps = w.rms_eps

    def norm(x, g):
        return f(g) * x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)

    def rot(x, pos):  # x [..., D]
        i = np.arange(D // 2)
        ang = pos * w.rope_theta ** (-2.0 * i / D)
        c, s = np.cos(ang).astype(np.float32).astype(np.float64), np.sin(ang).astype(np.float32).astype(np.float64)
        a, b = x[..., :D // 2], x[..., D // 2:]
        return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)

    hidden, logits = [], []
    for b in range(B):
        pos = int(lens[b])
        x = f(weights["embed"][tok[b]])
        for l, lw in enumerate(weights["layers"]):
            xn = norm(x, lw["attn_norm"])
            q = (f(lw["wq"]) @ xn).reshape(Hq, D)
            kk = (f(lw["wk"]) @ xn).reshape(Hkv, D)
            vv = (f(lw["wv"]) @ xn).reshape(Hkv, D)
            q = rot(norm(q, lw["q_norm"]), pos)
            kk = rot(norm(kk, lw["k_norm"]), pos)
            kc = f(k[l, b, :, :pos + 1]).copy()
            vc = f(v[l, b, :, :pos + 1]).copy()
            kc[:, pos] = f(bf16_exact(kk))
            vc[:, pos] = f(bf16_exact(vv))
            o = np.zeros((Hq, D))
            for h in range(Hq):
                s = kc[h // rep] @ q[h] / math.sqrt(D)
                p = np.exp(s - s.max())
                o[h] = (p / p.sum()) @ vc[h // rep]
            x = x + f(lw["wo"]) @ o.reshape(-1)
            xn = norm(x, lw["mlp_norm"])
            g = f(lw["w_gate"]) @ xn
            u = f(lw["w_up"]) @ xn
            x = x + f(lw["w_down"]) @ (g / (1 + np.exp(-g)) * u)
        hidden.append(x)
        lm = weights["lm_head"] if weights["lm_head"] is not None else weights["embed"]
        logits.append(f(lm) @ norm(x, weights["final_norm"]))
    return np.array(hidden), np.array(logits)


@pytest.mark.parametrize("batch,tied", [(1, 0), (3, 1)])
def test_step_matches_float64_restatement_on_tiny(batch, tied):
    w = synth.TINY.with_(batch=batch, tied_embeddings=tied, kv_len=None, kv_len_range=(0, 40))
    weights = synth.make_weights(w, 11)
    lens = w.kv_lens(11)
    cap = int(lens.max()) + 1
    k, v = synth.make_kv(w, lens, cap, 11)
    tok = synth.make_tokens(w, 11)
    hid64, log64 = _numpy_step_f64(w, weights, tok, lens, k, v)
    kl = lens.copy()
    out = oracle.Model(w, weights, cap).step(tok, kl, k, v)
    rel = np.linalg.norm(out["hidden"] - hid64) / np.linalg.norm(hid64)
    assert rel < 1e-5, rel
    assert np.max(np.abs(out["logits"] - log64)) < 1e-4 * np.max(np.abs(log64))
    np.testing.assert_array_equal(kl, lens + 1)


def test_step_rejects_full_cache_and_bad_tokens():
    w = synth.TINY
    weights = synth.make_weights(w, 0)
    cap = 33
    k = np.zeros((w.n_layers, 1, w.n_kv_heads, cap, w.head_dim), dtype=np.uint16)
    v = np.zeros_like(k)
    m = oracle.Model(w, weights, cap)
    kl = np.array([33], dtype=np.int32)
    with pytest.raises(ValueError):
        m.step(np.array([1], dtype=np.int32), kl, k, v)
    assert kl[0] == 33 and not k.any()
    kl = np.array([3], dtype=np.int32)
    with pytest.raises(ValueError):
        m.step(np.array([w.vocab], dtype=np.int32), kl, k, v)
    assert kl[0] == 3


# ------------------------------------------------------------ per-head q/k RMSNorm
def _constant_heads(n_heads, D, H, consts):
    """Projection rows of head h all equal to consts[h] / H: with x_hat constant
    (= 1 / sqrt(1 + eps)), head h's output is the constant consts[h] * x_hat."""
    w = np.zeros((n_heads * D, H), dtype=np.float64)
    for h, c in enumerate(consts):
        w[h * D:(h + 1) * D, :] = c / H
    return bf16_exact(w)


def _unit_input(w, weights, tok):
    weights["embed"] = weights["embed"].copy()
    weights["embed"][tok[0]] = bf16_exact(np.ones(w.hidden))
    for lw in weights["layers"]:
        lw["attn_norm"] = bf16_exact(np.ones(w.hidden))
    return weights


def test_step_k_norm_is_per_head_with_the_k_gain():
    # Both kv heads project to constants of very different magnitude (0.5 and
    # -3), the k gain is non-unit and differs from the q gain.  A per-head
    # norm maps head g to g_k * sign(c_g) * |c_g| / sqrt(c_g^2 + eps); at
    # kv_len 0 RoPE is the identity, so that is the appended key row (bf16).
    # A norm over the concatenated heads, a dropped gain, or the q gain in
    # its place gives other rows.
    w = synth.TINY.with_(n_layers=1, kv_len=0)
    D, H = w.head_dim, w.hidden
    weights = _zero_mixing(synth.make_weights(w, 13))
    tok = synth.make_tokens(w, 13)
    weights = _unit_input(w, weights, tok)
    xh = 1.0 / math.sqrt(1.0 + w.rms_eps)
    consts = [0.5, -3.0]
    lw = weights["layers"][0]
    lw["wk"] = _constant_heads(w.n_kv_heads, D, H, consts)
    lw["k_norm"] = bf16_exact(0.5 + np.arange(D) / D)
    lw["q_norm"] = bf16_exact(2.0 - np.arange(D) / D)
    k = np.zeros((1, 1, w.n_kv_heads, 1, D), dtype=np.uint16)
    v = np.zeros_like(k)
    kl = np.array([0], dtype=np.int32)
    oracle.Model(w, weights, 1).step(tok, kl, k, v)
    gk = synth.bf16_to_f32(lw["k_norm"]).astype(np.float64)
    for g, c in enumerate(consts):
        kc = np.float32(np.float32(c) * np.float32(xh))  # the constant head value
        expect = gk * float(kc) / math.sqrt(float(kc) ** 2 + w.rms_eps)
        got = synth.bf16_to_f32(k[0, 0, g, 0]).astype(np.float64)
        np.testing.assert_allclose(got, synth.bf16_to_f32(bf16_exact(expect)), rtol=0, atol=0)
        # the two heads differ only by the sign: per-head normalisation
        assert np.allclose(np.abs(got), gk, rtol=8e-3)


def test_step_q_norm_is_per_head_with_the_q_gain():
    # q head h projects to the constant c_h (magnitudes 0.25 ... 3), the q
    # gain g_q is non-unit; W_k = W_v = 0, so the new key and value are 0.
    # With one cached row (K_0, V_0 = 1) the new token at position 1 attends
    # with probability p_h = sigmoid(s_h) to row 0 and 1 - p_h to the new row,
    # s_h = rope_1(g_q * sign(c_h) * |c_h| / sqrt(c_h^2 + eps)) . K_0 / sqrt(D).
    # W_o = I then puts o_h = p_h * 1 into the hidden state: hidden = 1 + p_h.
    w = synth.TINY.with_(n_layers=1, kv_len=1)
    D, H, Hq = w.head_dim, w.hidden, w.n_q_heads
    rep = Hq // w.n_kv_heads
    weights = _zero_mixing(synth.make_weights(w, 17))
    tok = synth.make_tokens(w, 17)
    weights = _unit_input(w, weights, tok)
    xh = 1.0 / math.sqrt(1.0 + w.rms_eps)
    consts = [0.25, -3.0, 1.5, -0.5]
    lw = weights["layers"][0]
    lw["wq"] = _constant_heads(Hq, D, H, consts)
    lw["q_norm"] = bf16_exact(0.5 + np.arange(D) / D)
    lw["k_norm"] = bf16_exact(2.0 - np.arange(D) / D)
    lw["wo"] = bf16_exact(np.eye(H, w.q_dim))
    k0 = bf16_exact(np.random.default_rng(3).standard_normal((w.n_kv_heads, D)))
    k = np.zeros((1, 1, w.n_kv_heads, 2, D), dtype=np.uint16)
    v = np.zeros_like(k)
    k[0, 0, :, 0, :] = k0
    v[0, 0, :, 0, :] = bf16_exact(np.ones(D))
    kl = np.array([1], dtype=np.int32)
    out = oracle.Model(w, weights, 2).step(tok, kl, k, v)
    gq = synth.bf16_to_f32(lw["q_norm"]).astype(np.float64)
    half = D // 2
    i = np.arange(half)
    ang = 1.0 * w.rope_theta ** (-2.0 * i / D)
    cs, sn = np.cos(ang), np.sin(ang)
    expect = np.ones(H)
    for h, c in enumerate(consts):
        qc = float(np.float32(np.float32(c) * np.float32(xh)))
        q = gq * qc / math.sqrt(qc * qc + w.rms_eps)
        qr = np.concatenate([q[:half] * cs - q[half:] * sn, q[half:] * cs + q[:half] * sn])
        s = qr @ synth.bf16_to_f32(k0[h // rep]).astype(np.float64) / math.sqrt(D)
        expect[h * D:(h + 1) * D] += 1.0 / (1.0 + math.exp(-s))
    np.testing.assert_allclose(out["hidden"][0], expect, rtol=2e-6, atol=2e-6)
    # the appended row is zero (W_k = W_v = 0)
    assert not synth.bf16_to_f32(k[0, 0, :, 1]).any() and not synth.bf16_to_f32(v[0, 0, :, 1]).any()
