"""Decode-step benchmark: one persistent launch per step vs one launch per operator.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl mk|reference]

Prints ONE JSON line (rank 0).  The workload defaults to the Qwen3-8B-shaped
decoder at batch 1 with 1024 cached positions per sequence; all inputs are
seeded synthetic data (bf16 weights ~N(0, 0.02), gains 1 + N(0, 0.1), cached
K/V ~N(0, 1)).  `value` is microseconds per decode step (device time, CUDA
events, max over ranks); per step the whole weight set (15.3 GB) streams from
HBM, far more than the 126 MB L2, so no explicit L2 flush is needed.

Multi-GPU: the decode step does not shard without a per-layer exchange, so N
GPUs run N independent replicas (no data-path collective); a barrier brackets
the timed region and the reported time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "us per decode step & achieved HBM GB/s vs 8 TB/s (Qwen3-8B-shaped, bs=1)"
UNIT = "us/step"
HBM_NOMINAL_GBS = 8000.0


# ----------------------------------------------------------------------------
# Algorithmic bytes
# ----------------------------------------------------------------------------
def step_bytes(w, lens) -> int:
    """Bytes one decode step must move: every weight matrix and gain once, the B
    embedding rows, L_b cached K and V rows per (layer, sequence, kv head) and
    the appended K/V rows."""
    H, F, D, Ly = w.hidden, w.ffn, w.head_dim, w.n_layers
    rep = w.n_q_heads // w.n_kv_heads
    n_qkv = w.n_kv_heads * (rep + 2) * D
    per_layer = n_qkv * H + H * w.q_dim + 2 * F * H + H * F + 2 * H + 2 * D
    weights = 2 * (Ly * per_layer + w.vocab * H + H)
    emb = 2 * w.batch * H
    kv_row = 2 * D * w.n_kv_heads * Ly * 2  # K and V, every layer and kv head
    kv_read = kv_row * int(np.sum(lens))
    kv_write = kv_row * w.batch
    return int(weights + emb + kv_read + kv_write)


def steps_bytes(w, lens0, k) -> int:
    return sum(step_bytes(w, np.asarray(lens0) + i) for i in range(k))


# ----------------------------------------------------------------------------
# Clocks during the timed region (NVML reads only)
# ----------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device: int, period_s: float = 0.005):
        self.samples, self.reasons = [], set()
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: clocks stay unreported
            self.err = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# Helpers
# ----------------------------------------------------------------------------
def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in ("mk_worker.cu", "runtime.cuh"):
        with open(os.path.join(ROOT, "persistent_runtime_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def traffic_record(workload: str):
    """DRAM bytes per launch from a committed ncu summary of the same kernel source."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    ent = rec.get(workload)
    if not ent or ent.get("kernel_hash") != kernel_hash():
        return None
    return ent


def gen_inputs(w, seed, cap):
    lens = w.kv_lens(seed)
    tokens = synth.make_tokens(w, seed)
    weights = synth.make_weights(w, seed)
    k, v = synth.make_kv(w, lens, cap, seed)
    return weights, lens, tokens, k, v


def paged_pools(cache, P, seed):
    """[Ly][B][Hkv][cap][D] rows -> pool [n_pages][Ly][Hkv][P][D] with the pages of
    every sequence scattered by a seeded permutation, and the page table
    [B][ceil(cap / P)]."""
    Ly, B, Hkv, cap, D = cache.shape
    mp = -(-cap // P)
    n_pages = B * mp
    table = np.random.default_rng(seed).permutation(n_pages).astype(np.int32).reshape(B, mp)
    pool = np.zeros((n_pages, Ly, Hkv, P, D), dtype=np.uint16)
    for b in range(B):
        for j in range(mp):
            rows = cache[:, b, :, j * P:(j + 1) * P, :]
            pool[table[b, j], :, :, :rows.shape[2], :] = rows
    return pool, table, n_pages


def upload(torch, a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


# ----------------------------------------------------------------------------
# CPU oracle timing
# ----------------------------------------------------------------------------
def oracle_time_step(w, weights, lens, tokens, k, v, cap, layers_run=-1, vocab_run=-1,
                     seq_mask=None):
    import oracle
    oracle.build() if not os.path.exists(os.path.join(ROOT, "oracle", "libmk_oracle.so")) else None
    m = oracle.Model(w, weights, cap)
    kl = lens.copy()
    t0 = time.perf_counter()
    m.step(tokens, kl, k, v, want_logits=False, want_hidden=False, layers_run=layers_run,
           vocab_run=vocab_run, seq_mask=seq_mask)
    return time.perf_counter() - t0


def sample_fraction(w, layers_run, vocab_run, lens):
    """Share of a full step's bytes that a (layers_run, vocab_run) sample touches."""
    full = step_bytes(w, lens)
    D, H = w.head_dim, w.hidden
    rep = w.n_q_heads // w.n_kv_heads
    n_qkv = w.n_kv_heads * (rep + 2) * D
    per_layer = 2 * (n_qkv * H + H * w.q_dim + 3 * w.ffn * H + 2 * H + 2 * D)
    kv = 2 * D * w.n_kv_heads * 2 * int(np.sum(lens) + w.batch)
    part = layers_run * (per_layer + kv) + 2 * vocab_run * H
    return part / full


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = synth.WORKLOADS[args.workload]
    cap = w.kv_capacity(args.seed) + max(args.steps, args.warmup)
    weights, lens, tokens, k, v = gen_inputs(w, args.seed, cap)
    layers_run = max(1, w.n_layers // 18)
    vocab_run = max(1, w.vocab // 18)
    frac = sample_fraction(w, layers_run, vocab_run, lens)
    for _ in range(args.warmup):
        oracle_time_step(w, weights, lens, tokens, k, v, cap, layers_run, vocab_run)
    times = [oracle_time_step(w, weights, lens, tokens, k, v, cap, layers_run, vocab_run)
             for _ in range(args.steps)]
    us = 1e6 * float(np.mean(times)) / frac
    sample = (f"each step: {layers_run} of {w.n_layers} layers + {vocab_run} of {w.vocab} LM-head "
              f"rows ({100 * frac:.1f}% of the step's bytes), time scaled by bytes")
    out = {"impl": "reference", "metric": METRIC, "value": us, "unit": UNIT, "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": us / 1000,
           "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
           "data": "synthetic", "config": workload_config(w, lens, args.gpus),
           "cpu_baseline": dict({"value": us, "unit": UNIT, "cores": 1, "kind": "oracle",
                                 "sample": sample}, **host_cpu()),
           "e2e": {"value": us, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))
    return 0


def reduce_max(x: float, world: int, dist=None, device: str = "cuda") -> float:
    """The largest x over the ranks (every rank calls it; world 1 needs no
    process group)."""
    if world == 1:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def workload_config(w, lens, n):
    return {"workload": f"{w.name} bs{w.batch} kv{int(np.max(lens))}",
            "model": f"{w.name}-shaped decoder, {w.n_layers} layers, hidden {w.hidden}, "
                     f"{w.n_q_heads}/{w.n_kv_heads} heads x {w.head_dim}, ffn {w.ffn}, "
                     f"vocab {w.vocab}, {'tied' if w.tied_embeddings else 'untied'} LM head",
            "global_batch": w.batch * n, "seq_len": int(np.max(lens)),
            "parallelism": "replicas" if n > 1 else "single GPU",
            "l2": "inputs larger than L2: every step streams all weights (>100x L2)"}


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------
# The other configurations of the same model family, measured by default after
# the headline workload: (workload, timed steps).  Steps follow the workload's
# own decode length (64 steps at 0.6B and 8B batch 8, 32 at 8B batch 16).
OTHER_WORKLOADS = (("qwen3-0.6b", 64), ("qwen3-8b-b8", 64), ("qwen3-8b-b16", 32))


def host_cpu():
    """Cores and model name of the host (for the CPU baseline's context)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model}


class Gpu:
    """Process-wide GPU context: torch, the process group, the library."""

    def __init__(self):
        import torch
        import torch.distributed as dist

        import persistent_runtime_b200 as prb

        self.torch, self.dist, self.prb = torch, dist, prb
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        local = int(os.environ.get("LOCAL_RANK", "0"))
        if self.world > 1:
            from datetime import timedelta
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timedelta(seconds=600),
                                    device_id=torch.device("cuda", local))
        else:
            torch.cuda.set_device(0)
        self.dev = torch.cuda.current_device()

    def barrier(self):
        self.torch.cuda.synchronize()
        if self.world > 1:
            self.dist.barrier()
        self.torch.cuda.synchronize()

    def max_over_ranks(self, x: float) -> float:
        return reduce_max(x, self.world, self.dist, "cuda")

    def close(self):
        if self.world > 1:
            self.dist.destroy_process_group()


def device_weights(g, w, seed):
    """Seeded weights of workload w uploaded once (host copy returned too)."""
    weights = synth.make_weights(w, seed)
    torch = g.torch
    dw = {"embed": upload(torch, weights["embed"]), "final_norm": upload(torch, weights["final_norm"]),
          "lm_head": None if weights["lm_head"] is None else upload(torch, weights["lm_head"]),
          "layers": [{n: upload(torch, a) for n, a in lw.items()} for lw in weights["layers"]]}
    return weights, dw


def measure(g, w, args, steps, warmup, dw, tuning, *, baselines=True, trace_path="",
            event_trace=False, keep_host=False):
    """One workload: µs per step of K single-step launches (the value), the
    end-to-end loop with host buffers, the per-operator arms, one multi-step
    launch and, optionally, a traced step (outside every timed region).
    Returns (result dict, host inputs for the CPU baseline or None)."""
    torch, prb = g.torch, g.prb
    lens = w.kv_lens(args.seed)
    cap = int(lens.max()) + max(steps, warmup)
    tokens = synth.make_tokens(w, args.seed)
    mk = prb.Megakernel(w, cap, g.dev, **tuning)
    mk.load_weights(dw)
    torch.cuda.synchronize()
    k_host, v_host = synth.make_kv(w, lens, cap, args.seed)
    paged = tuning.get("kv_page_size", 0)
    if paged:
        # the same rows in pages scattered over the pools by a seeded permutation
        kp, table, n_pages = paged_pools(k_host, paged, args.seed)
        vp, _, _ = paged_pools(v_host, paged, args.seed)
        d_k, d_v = upload(torch, kp), upload(torch, vp)
        d_table = torch.from_numpy(table).cuda()
        del kp, vp
    else:
        d_k, d_v = upload(torch, k_host), upload(torch, v_host)
    if not keep_host:
        k_host = v_host = None
    d_len = torch.from_numpy(lens.copy()).cuda()
    d_tok = torch.from_numpy(tokens.copy()).cuda()
    d_logits = None
    stream = torch.cuda.current_stream()

    def reset():
        d_len.copy_(torch.from_numpy(lens))
        d_tok.copy_(torch.from_numpy(tokens))

    def check():
        rc, detail = mk.sync_status()
        if rc != 0:
            raise RuntimeError(f"device status {rc} {detail}")

    def timed(fn, k):
        reset()
        g.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(k):
            fn()
        e1.record(stream)
        g.barrier()
        check()
        return g.max_over_ranks(e0.elapsed_time(e1))

    def run_steps(n, out):
        if paged:
            mk.decode_steps_paged(n, d_tok, out, d_len, d_k, d_v, n_pages, d_table, d_logits)
        else:
            mk.decode_steps(n, d_tok, out, d_len, d_k, d_v, d_logits)

    step = lambda: run_steps(1, d_tok)  # noqa: E731

    # warm-up
    reset()
    for _ in range(warmup):
        step()
    check()

    # timed region: persistent megakernel, one launch per step
    with ClockSampler(g.dev) as clocks:
        ms = timed(step, steps)
    us_step = 1000.0 * ms / steps
    bytes_k = steps_bytes(w, lens, steps)
    gbs = bytes_k / (ms * 1e-3) / 1e9
    tok_s = g.world * w.batch * steps / (ms * 1e-3)

    # end to end through the public API with host buffers
    h_tok = torch.from_numpy(tokens.copy()).pin_memory()
    h_out = torch.empty_like(h_tok).pin_memory()

    def e2e_step():
        d_tok.copy_(h_tok, non_blocking=True)
        run_steps(1, d_tok)
        h_out.copy_(d_tok, non_blocking=True)
        stream.synchronize()
        h_tok.copy_(h_out)

    h_tok.copy_(torch.from_numpy(tokens))
    e2e_us = 1000.0 * timed(e2e_step, steps) / steps

    base = {}
    if baselines and not paged:  # the per-operator arms take no page table
        perop = lambda: mk.decode_step_perop(d_tok, d_tok, d_len, d_k, d_v, d_logits)  # noqa
        reset()
        for _ in range(warmup):
            perop()
        check()
        base["perop_eager_us"] = 1000.0 * timed(perop, steps) / steps
        try:
            cg = torch.cuda.CUDAGraph()
            reset()
            side = torch.cuda.Stream()
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                perop()  # warm the side stream
            torch.cuda.synchronize()
            reset()
            with torch.cuda.graph(cg):
                perop()
            torch.cuda.synchronize()
            for _ in range(warmup):
                cg.replay()
            check()
            base["perop_graph_us"] = 1000.0 * timed(cg.replay, steps) / steps
            del cg
        except Exception as e:  # capture refused: report why
            base["perop_graph_error"] = str(e)[:200]
        base["perop_launches_per_step"] = mk.info().n_ops

    # the same K steps as ONE launch (mk_decode_steps: tokens fed back on the
    # device); reported beside the one-launch-per-step loop above
    multi_out = torch.zeros((steps, w.batch), dtype=torch.int32, device="cuda")
    reset()
    run_steps(warmup, multi_out)
    check()
    multi_us = 1000.0 * timed(lambda: run_steps(steps, multi_out), 1) / steps

    trace_summary = None
    if trace_path or event_trace:
        from persistent_runtime_b200 import trace as mktrace
        gr = mk.graph()
        buf = torch.zeros(8 * gr.n_tasks, dtype=torch.int64, device="cuda")
        mk.set_trace(buf)
        reset()
        step()
        check()
        mk.set_trace(None)
        tr = buf.cpu().numpy().view(np.uint64)
        trace_summary = mktrace.summarize(tr, gr)
        if trace_path:
            mktrace.to_chrome(tr, gr, trace_path)
        trace_summary.pop("op_spans")

    peak, peak_kind = measured_peaks()
    traffic = traffic_record(w.name)
    res = {
        "value": us_step, "unit": UNIT, "steps": steps, "warmup": warmup,
        "ms_per_step": us_step / 1000.0,
        "config": dict(workload_config(w, lens, g.world), **({"kv_page_size": paged} if paged else {})),
        "tokens_per_s": tok_s, "hbm_gbs": gbs, "frac_of_8tbs": gbs / HBM_NOMINAL_GBS,
        "bytes_per_step": bytes_k / steps,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                     "frac": gbs / peak, "peak_kind": f"{peak_kind} copy bandwidth",
                     "kernel": "mk_worker_kernel (persistent, one launch per step)",
                     "traffic": None if traffic is None else traffic["dram_bytes_per_launch"]},
        "e2e": {"value": e2e_us, "unit": UNIT, "h2d_bytes_per_step": 4 * w.batch,
                "d2h_bytes_per_step": 4 * w.batch},
        "multistep": {"value": multi_us, "unit": UNIT, "steps_per_launch": steps,
                      "note": "the same steps in one mk_decode_steps launch"},
        "gpu_launches": steps,
        "clocks": clocks.summary(),
        "baselines": base,
    }
    if trace_summary is not None:
        res["event_wait_frac"] = trace_summary["event_wait_frac"]
        res["trace"] = trace_summary
    mk.close()
    host = (lens, tokens, k_host, v_host, cap) if keep_host else None
    return res, host


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--workload", default="qwen3-8b", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="mk", choices=["mk", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-baselines", action="store_true", help="skip the per-operator arms")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="measure only --workload (by default the line also carries the other "
                         "configurations of the model family)")
    ap.add_argument("--tuning", default="", help="k=v,... passed to mk_tuning")
    ap.add_argument("--kv-page-size", type=int, default=0,
                    help="run on paged K/V pools with this many positions per page")
    ap.add_argument("--trace", default="", help="write a Chrome trace of one step to this path")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        return run_reference(args)

    g = Gpu()
    w = synth.WORKLOADS[args.workload]
    tuning = {}
    for kv in filter(None, args.tuning.split(",")):
        key, val = kv.split("=")
        tuning[key] = int(val)
    if args.kv_page_size:
        tuning["kv_page_size"] = args.kv_page_size
    keep_host = g.rank == 0 and g.world == 1 and not args.no_cpu_baseline
    weights, dw = device_weights(g, w, args.seed)
    if not keep_host:
        weights = None
    res, host = measure(g, w, args, args.steps, args.warmup, dw, tuning,
                        baselines=not args.no_baselines, trace_path=args.trace, event_trace=True,
                        keep_host=keep_host)
    result = {"metric": METRIC, "value": res.pop("value"), "unit": UNIT, "n_gpus": g.world,
              "steps": args.steps, "warmup": args.warmup, "ms_per_step": res.pop("ms_per_step"),
              "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
              "data": "synthetic", "config": res.pop("config")}
    res.pop("steps"), res.pop("warmup"), res.pop("unit")
    result.update(res)
    if keep_host:
        lens, tokens, k_host, v_host, cap = host
        if w.batch == 1:
            t = oracle_time_step(w, weights, lens, tokens, k_host, v_host, cap)
            sample = "one full decode step of the same workload, single-threaded fp32 oracle"
        else:
            # the oracle advances each sequence on its own: time sequence 0's
            # full step and scale by the batch (the step's bytes per sequence
            # are the same weights plus that sequence's cache)
            mask = np.zeros(w.batch, dtype=np.uint8)
            mask[0] = 1
            t = w.batch * oracle_time_step(w, weights, lens, tokens, k_host, v_host, cap,
                                           seq_mask=mask)
            sample = (f"sequence 0's full decode step (kv {int(lens[0])}), single-threaded fp32 "
                      f"oracle, times {w.batch} sequences")
        result["cpu_baseline"] = dict({"value": 1e6 * t, "unit": UNIT, "cores": 1, "kind": "oracle",
                                       "sample": sample}, **host_cpu())
        host = k_host = v_host = None
    weights = None

    if not args.no_other_workloads and not args.kv_page_size:
        # the other configurations: same model family; the 8B configurations
        # share the headline's weights (same seed and shapes)
        others = {}
        def same_shape(a, b):
            return (a.n_layers, a.hidden, a.n_q_heads, a.n_kv_heads, a.ffn, a.vocab,
                    a.tied_embeddings) == (b.n_layers, b.hidden, b.n_q_heads, b.n_kv_heads,
                                           b.ffn, b.vocab, b.tied_embeddings)
        # workloads that share the loaded weights first
        order = sorted(OTHER_WORKLOADS, key=lambda e: not same_shape(synth.WORKLOADS[e[0]], w))
        cur = w
        for name, steps in order:
            ow = synth.WORKLOADS[name]
            if ow.name == w.name:
                continue
            if not same_shape(ow, cur):
                dw = None
                g.torch.cuda.empty_cache()
                _, dw = device_weights(g, ow, args.seed)
                cur = ow
            r, _ = measure(g, ow, args, steps, args.warmup, dw, {}, baselines=not args.no_baselines,
                           event_trace=True)
            others[r["config"]["workload"]] = {
                k: r[k] for k in ("value", "unit", "steps", "tokens_per_s", "hbm_gbs",
                                  "bytes_per_step", "e2e", "multistep", "baselines", "clocks",
                                  "event_wait_frac")}
            others[r["config"]["workload"]]["roofline_frac"] = r["roofline"]["frac"]
        result["other_workloads"] = others
    dw = None
    g.close()
    if g.rank == 0:
        print(json.dumps(result))
    return 0


if __name__ == "__main__":
    sys.exit(main())
