"""Shared set-up for the GPU parity tests: seeded inputs, oracle run, comparison."""
import numpy as np

import oracle
import synth

# Tolerances of the bf16 decode step against the fp32 oracle.
LOGIT_TOL = 2e-2      # max |d logit| <= LOGIT_TOL * max |logit|
HIDDEN_TOL = 1e-2     # ||d hidden|| / ||hidden|| <= HIDDEN_TOL
SEPARATION = 4e-2     # argmax must match exactly when top1 - top2 > SEPARATION * max|logit|


def torch():
    import torch as t
    return t


def dev_u16(a: np.ndarray):
    """bf16 bit patterns on the GPU (int16 storage; only the bits matter)."""
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def dev_weights(weights: dict) -> dict:
    out = {"embed": dev_u16(weights["embed"]), "final_norm": dev_u16(weights["final_norm"]),
           "lm_head": None if weights["lm_head"] is None else dev_u16(weights["lm_head"]),
           "layers": [{k: dev_u16(v) for k, v in lw.items()} for lw in weights["layers"]]}
    return out


class Case:
    """One seeded workload instance: host inputs, oracle model, GPU handle."""

    def __init__(self, w, seed=0, extra_cap=None, weights=None, **tuning):
        import persistent_runtime_b200 as prb
        t = torch()
        self.w = w
        self.seed = seed
        self.weights = synth.make_weights(w, seed) if weights is None else weights
        self.lens = w.kv_lens(seed)
        self.cap = int(self.lens.max()) + (w.steps if extra_cap is None else extra_cap)
        self.k, self.v = synth.make_kv(w, self.lens, self.cap, seed)
        self.tokens = synth.make_tokens(w, seed)
        self.model = oracle.Model(w, self.weights, self.cap)
        self.mk = prb.Megakernel(w, self.cap, 0, **tuning)
        dw = dev_weights(self.weights)
        self.mk.load_weights(dw)
        t.cuda.synchronize()
        del dw
        self.reset_device_state()

    def reset_device_state(self):
        t = torch()
        self.d_k = dev_u16(self.k)
        self.d_v = dev_u16(self.v)
        self.d_len = t.from_numpy(self.lens.copy()).cuda()
        self.d_tok = t.from_numpy(self.tokens.copy()).cuda()
        self.d_out = t.zeros(self.w.batch, dtype=t.int32, device="cuda")
        self.d_logits = t.zeros((self.w.batch, self.w.vocab), dtype=t.float32, device="cuda")

    def gpu_step(self, perop=False, tokens=None):
        t = torch()
        if tokens is not None:
            self.d_tok.copy_(t.from_numpy(np.asarray(tokens, dtype=np.int32)))
        fn = self.mk.decode_step_perop if perop else self.mk.decode_step
        fn(self.d_tok, self.d_out, self.d_len, self.d_k, self.d_v, self.d_logits)
        rc, detail = self.mk.sync_status()
        assert rc == 0, (rc, detail)
        return {"tokens": self.d_out.cpu().numpy(), "logits": self.d_logits.cpu().numpy(),
                "hidden": self.gpu_hidden(), "kv_len": self.d_len.cpu().numpy()}

    def gpu_hidden(self):
        """fp32 [batch][hidden] residual stream after the last layer of the latest step."""
        n = self.w.batch * self.w.hidden
        hidden = _wrap_device_f32(self.mk.final_hidden_ptr(), n).view(self.w.batch, -1).clone()
        return hidden.cpu().numpy()

    def oracle_step(self, tokens=None, k=None, v=None, lens=None):
        k = self.k if k is None else k
        v = self.v if v is None else v
        lens = self.lens if lens is None else lens
        tok = self.tokens if tokens is None else tokens
        return self.model.step(tok, lens, k, v)


def _wrap_device_f32(ptr: int, n: int):
    """A torch tensor viewing n fp32 values at a device address owned by the library."""
    t = torch()

    class _Holder:
        __cuda_array_interface__ = {"shape": (n,), "typestr": "<f4", "data": (ptr, False),
                                    "version": 3, "strides": None}

    return t.as_tensor(_Holder(), device="cuda")


def check_tokens(ref, tokens, w, ctx="", seqs=None):
    """The GPU's token of each sequence: the oracle's argmax when its top two
    logits are well separated, else a token whose oracle logit is within the
    logit tolerance of the maximum."""
    for b in (range(w.batch) if seqs is None else seqs):
        lo = ref["logits"][b].astype(np.float64)
        scale = np.max(np.abs(lo))
        top = np.sort(lo)[-2:]
        tok = int(tokens[b])
        if top[1] - top[0] > SEPARATION * scale:
            assert tok == int(ref["tokens"][b]), f"{ctx} b={b}: token {tok} != {ref['tokens'][b]}"
        else:
            assert lo[tok] >= top[1] - LOGIT_TOL * scale, f"{ctx} b={b}: token {tok} not near max"


def compare_logits(ref, logits, w, ctx="", seqs=None):
    """max |d logit| <= LOGIT_TOL * max |logit| per sequence; returns the ratios."""
    out = {}
    for b in (range(w.batch) if seqs is None else seqs):
        lo, lg = ref["logits"][b].astype(np.float64), logits[b].astype(np.float64)
        scale = np.max(np.abs(lo))
        err = np.max(np.abs(lo - lg))
        assert err <= LOGIT_TOL * scale, f"{ctx} b={b}: max|dlogit| {err} > {LOGIT_TOL}*{scale}"
        out[b] = float(err / scale)
    return out


def compare_step(ref, got, w, ctx="", seqs=None):
    """Asserts the tolerances (for the sequences seqs, default all); returns a
    dict of the measured errors."""
    errs = compare_logits(ref, got["logits"], w, ctx, seqs)
    out = {}
    for b in (range(w.batch) if seqs is None else seqs):
        h0, h1 = ref["hidden"][b].astype(np.float64), got["hidden"][b].astype(np.float64)
        rel = np.linalg.norm(h0 - h1) / np.linalg.norm(h0)
        assert rel <= HIDDEN_TOL, f"{ctx} b={b}: hidden rel L2 {rel}"
        out[b] = (errs[b], float(rel))
    check_tokens(ref, got["tokens"], w, ctx, seqs)
    return out


def rows_close(gk, gv, ref_k, ref_v, lens, seqs=None, bf16_inputs=False, ctx=""):
    """Rows appended at position lens[b] of the caches gk / gv (bf16 bit
    patterns, [Ly][B][Hkv][cap][D]) against the oracle's ref_k / ref_v.  At
    batch 1 the GPU's and the oracle's fp32 values differ only in summation
    order, so after rounding to bf16 almost every element is bit-identical
    (> 90 %).  With batch >= 2 (bf16_inputs) the projection input is itself
    rounded to bf16, a relative change of up to 2^-9 per element; with the
    rounding of both outputs the expected difference is about 2^-9 of the
    row's RMS, so the bound is 2^-7 of it (4x margin).  Element-wise, every
    value is within 1e-2 of the row's largest magnitude."""
    for b in (range(gk.shape[1]) if seqs is None else seqs):
        L = int(lens[b])
        for arr_g, arr_r in ((gk, ref_k), (gv, ref_v)):
            a = synth.bf16_to_f32(arr_g[:, b, :, L]).astype(np.float64)
            r = synth.bf16_to_f32(arr_r[:, b, :, L]).astype(np.float64)
            scale = np.max(np.abs(r), axis=-1, keepdims=True)
            assert np.all(np.abs(a - r) <= 1e-2 * scale), f"{ctx} b={b}: appended K/V row differs"
            if bf16_inputs:
                rel = float(np.sqrt(np.mean((a - r) ** 2) / np.mean(r ** 2)))
                assert rel <= 2.0 ** -7, f"{ctx} b={b}: appended rows differ by {rel:.2e} (RMS)"
            else:
                same = float(np.mean(arr_g[:, b, :, L] == arr_r[:, b, :, L]))
                assert same > 0.9, f"{ctx} b={b}: {same:.3f} of the appended row bit-identical"


def kv_rows_close(case, ref_k, ref_v, lens, untouched=None, seqs=None, bf16_inputs=False):
    """rows_close on the case's device caches; rows the step never wrote
    (below lens[b], or below untouched[b]) must be untouched."""
    gk = case.d_k.cpu().numpy().view(np.uint16)
    gv = case.d_v.cpu().numpy().view(np.uint16)
    rows_close(gk, gv, ref_k, ref_v, lens, seqs, bf16_inputs)
    for b in (range(case.w.batch) if seqs is None else seqs):
        U = int(lens[b]) if untouched is None else int(untouched[b])
        np.testing.assert_array_equal(gk[:, b, :, :U], case.k[:, b, :, :U])


def lockstep_oracle(case, toks, last, gk, gv, bf16_inputs=False, ctx=""):
    """The GPU ran len(toks) steps from the case's initial state: step s wrote
    the tokens toks[s], the last step's logits and hidden state are `last`,
    and gk / gv are the caches afterwards (contiguous layout, bf16 bits).
    The oracle replays the same steps fed with the GPU's tokens; every step's
    token, every appended row and the last step's logits and hidden state must
    agree within the step tolerances, and rows below the initial lengths must
    be untouched."""
    k, v, kl = case.k.copy(), case.v.copy(), case.lens.copy()
    tok = case.tokens.copy()
    n = len(toks)
    ref = None
    for s in range(n):
        ref = case.oracle_step(tokens=tok, k=k, v=v, lens=kl)
        check_tokens(ref, toks[s], case.w, f"{ctx} step {s}")
        tok = np.asarray(toks[s], dtype=np.int32).copy()
    compare_step(ref, last, case.w, f"{ctx} last step")
    for s in range(n):
        rows_close(gk, gv, k, v, case.lens + s, bf16_inputs=bf16_inputs, ctx=f"{ctx} step {s}")
    for b in range(case.w.batch):
        L = int(case.lens[b])
        np.testing.assert_array_equal(gk[:, b, :, :L], case.k[:, b, :, :L])
        np.testing.assert_array_equal(gv[:, b, :, :L], case.v[:, b, :, :L])
    np.testing.assert_array_equal(kl, case.lens + n)
