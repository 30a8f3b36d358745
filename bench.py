"""Throughput of the two-point ZO probe step on B200 (one JSON line on rank 0).

One step = zo_probe_plan + zo_score (both candidates of every prompt, one
packed batch) + zo_step (c and the banked update), on the OPT-13B-shaped
decoder with batch 64 by default (synthetic ragged prompts, random-init bf16
weights drawn on the device).  The metric is scored tokens/s (prefill tokens
of the physical batch) with ZO steps/s beside it; the GEMM kernel's live
roofline, the whole-step roofline fraction, the end-to-end number through
the public API with host buffers, the oracle on the host cores, the SM
clocks and the kernel launch count are reported on the same line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload opt-13b-b64]
    python bench.py --impl reference ...   (the CPU oracle as the reference arm)
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from zeroth_order_fine_b200 import workload as wl  # noqa: E402

METRIC = "ZO steps/s & scored tokens/s (OPT-13B shape, batch 64); % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def gemm_traffic():
    """Per-launch DRAM bytes of the tensor-core GEMM from the committed ncu summary,
    or None when the kernel source changed after the counters were taken."""
    import hashlib
    prof = os.path.join(ROOT, "profiles", "gemm_traffic_opt13b_b64.md")
    src = os.path.join(ROOT, "zeroth_order_fine_b200", "csrc", "k_gemm_tc.cu")
    if not (os.path.exists(prof) and os.path.exists(src)):
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    fields = {}
    for line in open(prof):
        if ":" in line and line.strip().startswith(("source_sha256", "traffic_bytes_per_launch")):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    if fields.get("source_sha256") != sha:
        return None
    try:
        return float(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ---- algorithmic work of one step ----------------------------------------------------

def step_work(w: wl.Workload, batches, n_slots: int):
    """Algorithmic FLOPs and HBM bytes of one step over the given per-rank batches."""
    sh = w.shape
    es = 2 if sh.dtype == wl.DTYPE_BF16 else 4
    flops = 0.0
    bytes_ = 0.0
    T_all = 0
    S_all = 0
    for b in batches:
        rows = list(b.prompts) * 2 + list(b.fg_prompts)
        tls = list(b.target_lens) * 2 + list(b.fg_target_lens)
        T = sum(len(r) for r in rows)
        S = int(sum(tls))
        T_all += T
        S_all += S
        flops += 2.0 * sh.body_params() * T                      # every decoder linear, all rows
        flops += 2.0 * sh.vocab * sh.d_model * S                 # lm_head at scored positions only
        ctx = sum(L * (L + 1) / 2 for L in (len(r) for r in rows))
        flops += 4.0 * ctx * sh.q_dim * sh.n_layers              # QK^T and PV, causal
        for m in w.matrices:                                     # shrink + expand of the bank
            di, do = sh.matrix_dims(m)
            flops += 2.0 * T * (di + do) * w.rank * (1 + n_slots) * sh.n_layers
        # bytes: weights once; activations ~ 10 passes of T x d per layer (fp32 residual
        # read+write twice, bf16 normalised inputs, q/k/v, attention out, FFN act in/out)
        act = T * (8 * sh.d_model * 4 + (2 * sh.d_model + sh.q_dim + 2 * sh.kv_dim) * es
                   + 2 * sh.d_ffn * es) * sh.n_layers
        bytes_ += act + sh.vocab * sh.d_model * es
    bytes_ += (sh.body_params() + sh.vocab * sh.d_model) * es    # per rank weights, once
    return flops, bytes_, T_all, S_all


def generate_work(w: wl.Workload, batch, G: int):
    """(prefill FLOPs, decode bytes) of one generation step of G new tokens per row: the
    prompts of both candidates as one packed prefill (the scoring step's FLOPs), then G - 1
    decode steps that each read every weight and the lm_head once and each row's k|v cache
    (its prompt plus the tokens generated so far) once."""
    sh = w.shape
    es = 2 if sh.dtype == wl.DTYPE_BF16 else 4
    flops, _, _, _ = step_work(w, [batch], 1)
    w_bytes = (sh.body_params() + sh.vocab * sh.d_model) * es
    kv_row = 2 * sh.kv_dim * sh.n_layers * es
    lens = np.concatenate([batch.seq_lens, batch.seq_lens]).astype(np.float64)
    kv_bytes = sum(float(np.sum(lens + g + 1)) * kv_row for g in range(G - 1))
    return flops, (G - 1) * w_bytes + kv_bytes


def fp8_flops(w: wl.Workload, batches) -> float:
    """The part of step_work's FLOPs that the fp8 option runs in E4M3: the base products of
    q|k|v and the FFN input projections (the norm-fed matrices)."""
    sh = w.shape
    n_in = 2 * sh.d_ffn if sh.arch == wl.ARCH_QWEN3 else sh.d_ffn
    per_tok = 2.0 * sh.d_model * (sh.q_dim + 2 * sh.kv_dim + n_in) * sh.n_layers
    return per_tok * sum(b.n_tokens_physical for b in batches)


# ---- clocks during the timed region -----------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (FileNotFoundError, OSError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---- the oracle on the host cores -------------------------------------------------------

_SAMPLE_WEIGHTS = {}
# Workloads whose whole step (every layer, every prompt) the oracle runs in the CPU baseline;
# the larger ones are timed on one layer and scaled by the layer count ("extrapolated").
FULL_ORACLE = ("tiny", "opt-1.3b-b16")


def _sample_weights(sh: wl.ModelShape, n_layers: int):
    """Weights of the oracle's timing sample, drawn with numpy's generator (their values do
    not change the oracle's work; the oracle's own counter-stream init of full-width layers
    would take longer than the scoring itself)."""
    import torch

    from oracle import model as om
    key = (sh.name, n_layers)
    if key in _SAMPLE_WEIGHTS:
        return _SAMPLE_WEIGHTS[key]
    rng = np.random.default_rng(0)

    def t(*shape, mean=0.0):
        return torch.from_numpy(rng.standard_normal(shape, dtype=np.float32) * 0.02 + mean).double()

    d = sh.d_model
    layers = []
    for _ in range(n_layers):
        layer = {}
        for m in sh.matrices():
            di, do = sh.matrix_dims(m)
            layer[f"W{m}"] = t(do, di)
            if sh.arch == wl.ARCH_OPT:
                layer[f"b{m}"] = t(do)
        layer["ln1_w"], layer["ln2_w"] = t(d, mean=1.0), t(d, mean=1.0)
        if sh.arch == wl.ARCH_OPT:
            layer["ln1_b"], layer["ln2_b"] = t(d), t(d)
        else:
            layer["q_norm"], layer["k_norm"] = t(sh.head_dim, mean=1.0), t(sh.head_dim, mean=1.0)
        layers.append(layer)
    tok = t(sh.vocab, d)
    one = wl.shrink_shape(sh, n_layers=n_layers)
    weights = om.Weights(one, tok, t(sh.max_pos, d) if sh.arch == wl.ARCH_OPT else None,
                         t(d, mean=1.0), t(d) if sh.arch == wl.ARCH_OPT else None,
                         tok if sh.tie_lm_head else t(sh.vocab, d), layers)
    _SAMPLE_WEIGHTS[key] = weights
    return weights


def oracle_sample(w: wl.Workload, n_prompts: int = 2, seed: int = 0):
    """Time the CPU oracle on a bounded sample of the workload.

    For the small workloads (FULL_ORACLE) the sample is the whole step: every prompt of the
    seeded batch (both candidate rows) through every layer, plan + score + update.  For
    the others it is n_prompts prompts through ONE decoder layer plus the final norm and
    the lm_head at their scored positions, and the layer time is scaled by n_layers; the
    result says so ("extrapolated": true, with the measured seconds and the scale).
    """
    import torch

    from oracle import zo as ozo
    sh = w.shape
    full = w.name in FULL_ORACLE
    n_lay = sh.n_layers if full else 1
    weights = _sample_weights(sh, n_lay)
    run = ozo.OracleRun(weights, w.run_seed, w.nu, w.rank, range(n_lay), w.matrices, w.scale_mode)
    if full:
        batch = wl.make_batch(w, seed=w.data_seed + 7919 * seed)
    else:
        batch = wl.make_batch(w, batch=n_prompts, fg_rows=min(w.fg_rows, n_prompts),
                              seed=w.data_seed + 7919 * seed)
    t0 = time.perf_counter()
    run.plan(0, w.eps)
    run.score(batch.prompts, batch.target_lens, batch.fg_prompts, batch.fg_target_lens)
    run.step(w.lr)
    secs_sample = time.perf_counter() - t0
    T = batch.n_tokens_physical
    P = len(batch.prompts)
    if full:
        secs_step = secs_sample
        sample = (f"the whole step: {P} prompts ({2 * P} candidate rows, {T} tokens) through "
                  f"all {sh.n_layers} layers + lm_head, plan + score + update; oracle float64 "
                  f"on the host cores")
        scale = 1
    else:
        # the lm_head part is already inside secs_sample once; scale only the layer part
        hs = torch.zeros(int(2 * batch.target_lens.sum() + batch.fg_target_lens.sum()),
                         sh.d_model, dtype=torch.float64)
        t1 = time.perf_counter()
        logits = hs @ weights.lm_head.T
        torch.logsumexp(logits, dim=-1)
        secs_head = time.perf_counter() - t1
        secs_step = (secs_sample - secs_head) * sh.n_layers + secs_head
        scale = sh.n_layers
        sample = (f"{P} prompts ({2 * P} candidate rows, {T} tokens) through 1 of "
                  f"{sh.n_layers} layers + lm_head at the scored positions, layer time scaled "
                  f"x{sh.n_layers} (extrapolated); oracle float64 on the host cores")
    return {"secs_per_sample_step": secs_step, "tokens": T, "tokens_per_s": T / secs_step,
            "sample": sample, "extrapolated": not full, "sample_seconds": secs_sample,
            "layer_scale": scale, "cores": torch.get_num_threads()}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch
    per_step = []
    for i in range(args.warmup + args.steps):
        r = oracle_sample(w, n_prompts=args.ref_prompts, seed=i)
        if i >= args.warmup:
            per_step.append(r)
    tok = sum(r["tokens"] for r in per_step)
    secs = sum(r["secs_per_sample_step"] for r in per_step)
    value = tok / secs
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "scored tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * secs / len(per_step), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "extrapolated": per_step[0]["extrapolated"],
            "config": {"workload": w.name, "model": w.shape.name, "global_batch": w.batch},
            "cpu_baseline": {"value": value, "unit": "scored tokens/s", "kind": "oracle",
                             "cores": per_step[0]["cores"], "sample": per_step[0]["sample"],
                             "extrapolated": per_step[0]["extrapolated"],
                             "layer_scale": per_step[0]["layer_scale"],
                             "sample_seconds_per_step": [round(r["sample_seconds"], 3)
                                                         for r in per_step]},
            "e2e": {"value": value, "unit": "scored tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---- one op alone ----------------------------------------------------------------------

def run_kernel(args):
    """Time one op over --launches launches after 3 warm-up launches (CUDA events)."""
    import torch

    from zeroth_order_fine_b200 import zo
    g = torch.Generator(device="cuda").manual_seed(0)
    M, N, K = args.m, args.n, args.k
    if args.kernel == "gemm" and args.fp8:
        x = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
        W = (torch.randn(N, K, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
        xq, sx = zo.zo_op_quantize_rows_e4m3(x)
        wq, sw = zo.zo_op_quantize_rows_e4m3(W)
        fn = lambda: zo.zo_op_linear_fp8(xq, sx, wq, sw)  # noqa: E731
        work, unit = 2.0 * M * N * K, "TFLOP/s"
        bytes_ = M * K + N * K + M * N * 2
    elif args.kernel == "gemm":
        x = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
        W = (torch.randn(N, K, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
        y = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
        fn = lambda: zo.zo_op_linear(x, W, out=y, impl=zo.IMPL_TENSOR_CORES)  # noqa: E731
        work, unit = 2.0 * M * N * K, "TFLOP/s"
        bytes_ = (M * K + N * K + M * N) * 2
    elif args.kernel == "lm_head":
        h = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
        E = (torch.randn(N, K, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
        tg = torch.randint(0, N, (M,), device="cuda", generator=g, dtype=torch.int32)
        fn = lambda: zo.zo_op_lm_head_logprob(h, E, tg, impl=zo.IMPL_TENSOR_CORES)  # noqa: E731
        work, unit = 2.0 * M * N * K, "TFLOP/s"
        bytes_ = (M * K + N * K) * 2
    else:
        w = wl.WORKLOADS["opt-13b-b64"]
        b = wl.make_batch(w)
        lens = np.concatenate([b.seq_lens, b.seq_lens])
        T = int(lens.sum())
        H = w.shape.n_heads
        qkv = torch.randn(T, 3 * H * 128, device="cuda", generator=g).to(torch.bfloat16)
        fn = lambda: zo.zo_op_attention(qkv, lens, H, H, 128, impl=zo.IMPL_TENSOR_CORES)  # noqa
        work = 4.0 * sum(L * (L + 1) / 2 for L in lens) * H * 128
        unit = "TFLOP/s"
        bytes_ = T * 4 * H * 128 * 2
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.launches):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.launches
    assert zo.zo_op_error_word() == 0
    print(json.dumps({"kernel": args.kernel + ("-e4m3" if args.fp8 else ""), "m": M, "n": N,
                      "k": K, "ms_per_launch": ms,
                      "achieved": work / (ms / 1e3) / 1e12, "unit": unit,
                      "gb_per_s": bytes_ / (ms / 1e3) / 1e9}), flush=True)
    return 0


# ---- the CUDA path ------------------------------------------------------------------

def run_generate(args, w: wl.Workload):
    """Generation-query steps (zo_probe_plan + zo_generate + zo_step) on one GPU: greedy
    decoding of --generate tokens per candidate row with the KV cache."""
    import torch

    from zeroth_order_fine_b200 import zo
    G = args.generate
    if args.layers:
        # fewer decoder layers of the same shapes: small device footprint for profiler captures
        w = dataclasses.replace(w, shape=dataclasses.replace(w.shape, n_layers=args.layers))
    sh = w.shape
    batch = wl.make_batch(w, fg_rows=0)
    model = zo.DeviceModel(sh, w.weight_seed)
    tg = zo.make_targets(sh.n_layers, w.matrices, w.scale_mode)
    T = batch.n_tokens_physical
    B = len(batch.prompts)
    h = zo.Handle(model, w.run_seed, w.nu, w.rank, tg, max_tokens=T, max_rows=2 * B,
                  max_scored=2 * B, max_slots=8, fp8=1 if args.fp8 else 0, max_new=G)
    toks = torch.from_numpy(batch.packed()).cuda()
    t = [0]

    def step():
        h.zo_probe_plan(t[0], w.eps)
        h.zo_generate(toks, batch.seq_lens, G)
        h.zo_step(w.lr, want_c=False)
        t[0] += 1

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    peaks, peak_kind = load_peaks()
    flops, decode_bytes = generate_work(w, batch, G)
    t_prefill = flops / (peaks["bf16_tflops_sustained"] * 1e12)
    t_decode = decode_bytes / (peaks["hbm_gbs"] * 1e9)
    roof_ms = (t_prefill + t_decode) * 1000.0
    s = h.zo_stats()
    print(json.dumps({
        "mode": "generate", "workload": w.name, "layers": sh.n_layers, "new_tokens_per_row": G,
        "rows": 2 * B,
        "prompt_tokens": T, "ms_per_step": ms, "steps": args.steps, "warmup": args.warmup,
        "generated_tokens_per_s": 2 * B * G / (ms / 1000.0),
        "dtype": "e4m3 (q|k|v, FFN-in) + bf16" if args.fp8 else "bf16",
        "roofline": {"prefill_ms": t_prefill * 1000.0, "decode_ms": t_decode * 1000.0,
                     "roofline_ms": roof_ms, "frac": roof_ms / ms,
                     "peak": f"{peak_kind} bf16 {peaks['bf16_tflops_sustained']} TFLOP/s sustained "
                             f"(prefill), HBM {peaks['hbm_gbs']} GB/s (decode: weights + cache "
                             f"once per token)"},
        "last_error_code": s["last_error_code"]}), flush=True)
    h.close()
    return 0


def cobatch_leg(steps: int, warmup: int = 2):
    """Co-serving analogue on the co-batching workload (Qwen3-8B shape, 16 prompts as 32
    probe rows plus 32 unperturbed foreground rows, lengths 64..512, MeZO-style r = 64 on all
    seven matrices): the mixed physical batch against the probe rows alone and the foreground
    rows alone, timed on one handle with CUDA events on the launching stream."""
    import torch

    from zeroth_order_fine_b200 import zo
    w = wl.WORKLOADS["qwen3-8b-cobatch"]
    sh = w.shape
    batch = wl.make_batch(w)
    model = zo.DeviceModel(sh, w.weight_seed)
    T = batch.n_tokens_physical
    S = int(2 * batch.target_lens.sum() + batch.fg_target_lens.sum())
    R = 2 * w.batch + len(batch.fg_prompts)
    h = zo.Handle(model, w.run_seed, w.nu, w.rank,
                  zo.make_targets(sh.n_layers, w.matrices, w.scale_mode),
                  max_tokens=T, max_rows=R, max_scored=S, max_slots=4)
    stream = torch.cuda.current_stream()
    toks = torch.from_numpy(batch.packed()).cuda()
    ftoks = torch.from_numpy(batch.fg_packed()).cuda()
    args_fg = (ftoks, batch.fg_seq_lens, batch.fg_target_lens)
    t = 0
    for _ in range(warmup):
        h.zo_probe_plan(t, w.eps)
        h.zo_score_cobatch(toks, batch.seq_lens, batch.target_lens, *args_fg)
        h.zo_step(w.lr, want_c=False)
        t += 1
    h.zo_probe_plan(t, w.eps)

    def timed(fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    mixed = timed(lambda: h.zo_score_cobatch(toks, batch.seq_lens, batch.target_lens, *args_fg))
    probe = timed(lambda: h.zo_score(toks, batch.seq_lens, batch.target_lens))
    fg = timed(lambda: h.zo_score_foreground(*args_fg))
    h.zo_step(w.lr, want_c=False)
    err = h.zo_stats()["last_error_code"]
    h.close()
    del model
    torch.cuda.empty_cache()
    fg_T = int(batch.fg_seq_lens.sum())
    return {"workload": w.name, "probe_rows": 2 * w.batch, "foreground_rows": len(batch.fg_prompts),
            "tokens": T, "foreground_tokens": fg_T, "mixed_batch_ms": mixed,
            "probe_rows_alone_ms": probe, "foreground_rows_alone_ms": fg,
            "mixed_vs_separate": mixed / (probe + fg),
            "mixed_tokens_per_s": T / (mixed / 1000.0),
            "separate_tokens_per_s": T / ((probe + fg) / 1000.0),
            "steps": steps, "last_error_code": err}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="opt-13b-b64", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    # prompts in the oracle's timing sample of the larger workloads: the reference arm's
    # per-step sample (about 4 s of CPU work for OPT-13B b64), and the one cpu_baseline
    # sample of the default line (about 10 s)
    ap.add_argument("--ref-prompts", type=int, default=16)
    ap.add_argument("--baseline-prompts", type=int, default=40)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the whole-step CUDA graph leg")
    ap.add_argument("--no-cobatch", action="store_true",
                    help="skip the co-batching leg (Qwen3-8B probe + foreground rows)")
    ap.add_argument("--layers", type=int, default=0,
                    help="run only this many decoder layers of the workload's shapes (small "
                         "device footprint for profiler captures; not a bench line)")
    ap.add_argument("--generate", type=int, default=0,
                    help="generation-query steps: greedy tokens per candidate row (zo_generate)")
    ap.add_argument("--fp8", action="store_true",
                    help="E4M3 base products for q|k|v and the FFN input (zo_options.fp8)")
    ap.add_argument("--cuda-cores", action="store_true", help="GEMMs on CUDA cores only")
    ap.add_argument("--kernel", choices=["gemm", "attention", "lm_head"],
                    help="time one op alone (kernel microbenchmark, used for ncu captures)")
    ap.add_argument("--m", type=int, default=4096)
    ap.add_argument("--n", type=int, default=5120)
    ap.add_argument("--k", type=int, default=5120)
    ap.add_argument("--launches", type=int, default=10)
    ap.add_argument("--byte-run", type=int, default=0,
                    help="run this many consecutive steps of the banked run and report the "
                         "state-transition bytes (1000 on opt-13b-b16 for the pages' comparison)")
    args = ap.parse_args()
    if args.kernel:
        return run_kernel(args)
    w = wl.WORKLOADS[args.workload]
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args, w)
    if args.generate:
        return run_generate(args, w)

    import torch
    import torch.distributed as dist

    from zeroth_order_fine_b200 import dp, zo

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    stream = torch.cuda.current_stream()

    if args.layers:
        # fewer decoder layers of the same shapes (per-launch GEMM shapes unchanged): for
        # profiler captures only, and the line says so
        w = dataclasses.replace(w, shape=dataclasses.replace(w.shape, n_layers=args.layers))
    sh = w.shape
    batch = wl.make_batch(w, seed=w.data_seed + 1000 * rank)
    model = zo.DeviceModel(sh, w.weight_seed)
    tg = zo.make_targets(sh.n_layers, w.matrices, w.scale_mode)
    T = batch.n_tokens_physical
    S = int(2 * batch.target_lens.sum() + batch.fg_target_lens.sum())
    R = 2 * w.batch + len(batch.fg_prompts)
    slots = max(8, args.byte_run // w.nu + 2)
    h = zo.Handle(model, w.run_seed, w.nu, w.rank, tg, max_tokens=T, max_rows=R, max_scored=S,
                  max_slots=slots, impl=1 if args.cuda_cores else 0, profile=0 if args.byte_run else 1,
                  fp8=1 if args.fp8 else 0)
    toks = torch.from_numpy(batch.packed()).cuda()
    ftoks = torch.from_numpy(batch.fg_packed()).cuda() if batch.fg_prompts else None
    sums = torch.zeros(2, dtype=torch.float64, device="cuda")
    step_no = [0]

    def one_step(tokens, want_c=False):
        t = step_no[0]
        h.zo_probe_plan(t, w.eps)
        if ftoks is not None:
            h.zo_score_cobatch(tokens, batch.seq_lens, batch.target_lens, ftoks, batch.fg_seq_lens,
                               batch.fg_target_lens)
        else:
            h.zo_score(tokens, batch.seq_lens, batch.target_lens)
        if world > 1:
            c = dp.dp_step(h, w.lr, sums, want_c=want_c)   # one 16-byte all-reduce per step
        else:
            c = h.zo_step(w.lr, want_c=want_c)
        step_no[0] += 1
        return c

    if args.byte_run:
        t0 = time.perf_counter()
        window_ms = []
        tw = t0
        for i in range(args.byte_run):
            one_step(toks)
            if (i + 1) % w.nu == 0:
                torch.cuda.synchronize()
                now = time.perf_counter()
                window_ms.append(round(1000 * (now - tw) / w.nu, 2))
                tw = now
        torch.cuda.synchronize()
        secs = time.perf_counter() - t0
        st = h.zo_stats()
        if rank == 0:
            print(json.dumps({"byte_run": args.byte_run, "workload": w.name, "nu": w.nu,
                              "bank_slots": st["bank_slots"],
                              "state_transition_bytes": st["state_transition_bytes"],
                              "dense_ref_bytes": st["dense_ref_bytes"],
                              "dense_ref_bytes_targets": st["dense_ref_bytes_targets"],
                              "frac_of_dense": st["state_transition_bytes"] / st["dense_ref_bytes"],
                              "frac_of_dense_targets": st["state_transition_bytes"] /
                              st["dense_ref_bytes_targets"],
                              "seconds": secs, "ms_per_step": 1000 * secs / args.byte_run,
                              "ms_per_step_by_window": window_ms,
                              "last_error_code": st["last_error_code"]}), flush=True)
        h.close()
        return 0
    for _ in range(args.warmup):
        one_step(toks)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    s0 = h.zo_stats()
    gpu_uuid = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    clk = ClockSampler(gpu_uuid)
    clk.start()
    time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ev0.record(stream)
    for _ in range(args.steps):
        one_step(toks)
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = clk.stop()
    ms = ev0.elapsed_time(ev1) / args.steps
    s1 = h.zo_stats()
    if s1["last_error_code"] not in (0,):
        raise RuntimeError(f"library reported error {s1['last_error_code']} during the run")
    if world > 1:
        t_ = torch.tensor([ms], dtype=torch.float64, device="cuda")
        dist.all_reduce(t_, op=dist.ReduceOp.MAX)
        ms = float(t_.item())

    # matched-query control: the same physical queries (zo_score only, no plan or
    # update), to set the complete step against the queries it requires
    torch.cuda.synchronize()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h.zo_probe_plan(step_no[0], w.eps)
    c0.record(stream)
    for _ in range(args.steps):
        if ftoks is not None:
            h.zo_score_cobatch(toks, batch.seq_lens, batch.target_lens, ftoks, batch.fg_seq_lens,
                               batch.fg_target_lens)
        else:
            h.zo_score(toks, batch.seq_lens, batch.target_lens)
    c1.record(stream)
    torch.cuda.synchronize()
    control_ms = c0.elapsed_time(c1) / args.steps
    h.zo_step(w.lr, want_c=False)
    step_no[0] += 1
    cobatch = None
    if ftoks is not None:
        # co-serving analogue: probe rows alone and foreground rows alone vs the mixed batch
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h.zo_probe_plan(step_no[0], w.eps)
        p0.record(stream)
        for _ in range(args.steps):
            h.zo_score(toks, batch.seq_lens, batch.target_lens)
        p1.record(stream)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            h.zo_score_foreground(ftoks, batch.fg_seq_lens, batch.fg_target_lens)
        f1.record(stream)
        torch.cuda.synchronize()
        probe_ms = p0.elapsed_time(p1) / args.steps
        fg_ms = f0.elapsed_time(f1) / args.steps
        cobatch = {"mixed_batch_ms": control_ms, "probe_rows_alone_ms": probe_ms,
                   "foreground_rows_alone_ms": fg_ms,
                   "mixed_vs_separate": control_ms / (probe_ms + fg_ms)}
        h.zo_step(w.lr, want_c=False)
        step_no[0] += 1

    # whole-step CUDA graph: the same probe steps, each one graph launch (zo_step_graph)
    graph = None
    if world == 1 and ftoks is None and not args.no_graph:
        for _ in range(2):                              # capture (and a window, if one opens)
            h.zo_step_graph(toks, batch.seq_lens, batch.target_lens, w.eps, w.lr)
            step_no[0] += 1
        torch.cuda.synchronize()
        g_s = h.zo_stats()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(args.steps):
            h.zo_step_graph(toks, batch.seq_lens, batch.target_lens, w.eps, w.lr)
        g1.record(stream)
        torch.cuda.synchronize()
        step_no[0] += args.steps
        g_e = h.zo_stats()
        g_ms = g0.elapsed_time(g1) / args.steps
        graph = {"ms_per_step": g_ms, "scored_tokens_per_s": T / (g_ms / 1000.0),
                 "eager_over_graph": ms / g_ms,
                 "captures_in_timed_region": int(g_e["graph_captures"] - g_s["graph_captures"]),
                 "replays_in_timed_region": int(g_e["graph_replays"] - g_s["graph_replays"])}

    # e2e: the same steps through the public API with host buffers (pinned), the
    # H2D copy of the step's tokens and the D2H read of c inside the timed region
    e2e = None
    if not args.no_e2e:
        host_toks = torch.from_numpy(batch.packed()).pin_memory()
        dev_buf = torch.empty_like(toks)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            dev_buf.copy_(host_toks, non_blocking=True)
            one_step(dev_buf, want_c=True)           # zo_step copies c (8 bytes) to the host
        torch.cuda.synchronize()
        e2e_s = (time.perf_counter() - t0) / args.steps
        if world > 1:
            t_ = torch.tensor([e2e_s], dtype=torch.float64, device="cuda")
            dist.all_reduce(t_, op=dist.ReduceOp.MAX)
            e2e_s = float(t_.item())
        e2e = {"value": world * T / e2e_s, "unit": "scored tokens/s",
               "h2d_bytes_per_step": int(host_toks.numel() * 4), "d2h_bytes_per_step": 8}

    peaks, peak_kind = load_peaks()
    n_slots = s1["bank_slots"]
    flops, bytes_, T1, S1 = step_work(w, [batch], n_slots)
    flops_all = flops * world
    tok_s = world * T / (ms / 1000.0)
    steps_s = 1000.0 / ms
    d_ms = s1["tc_gemm_ms"] - s0["tc_gemm_ms"]
    d_fl = s1["tc_gemm_flops"] - s0["tc_gemm_flops"]
    d_n = s1["tc_gemm_launches"] - s0["tc_gemm_launches"]
    gemm_tflops = d_fl / (d_ms / 1000.0) / 1e12 if d_ms > 0 else None
    peak_t = peaks["bf16_tflops_sustained"]
    if args.fp8:
        # E4M3 share at twice the measured bf16 rate (the nominal dense ratio), the rest at it
        f8 = fp8_flops(w, [batch])
        t_fl = (flops - f8) / (peak_t * 1e12) + f8 / (2 * peak_t * 1e12)
    else:
        t_fl = flops / (peak_t * 1e12)
    roof_t = max(t_fl, bytes_ / (peaks["hbm_gbs"] * 1e9))
    peak_g = peak_t
    if args.fp8 and d_fl > 0:
        f8g = fp8_flops(w, [batch]) * args.steps          # E4M3 FLOPs among the timed GEMMs
        peak_g = d_fl / ((d_fl - f8g) / peak_t + f8g / (2 * peak_t))
    line = {
        "metric": METRIC, "value": tok_s, "unit": "scored tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 (q|k|v, FFN-in) + bf16" if args.fp8 else "bf16",
        "data": "synthetic (random-init weights drawn on the device, Zipf(1.1) ragged prompts)",
        "config": {"workload": w.name, "model": sh.name, "global_batch": w.batch * world,
                   "prompts_per_gpu": w.batch, "physical_rows_per_gpu": R,
                   "tokens_per_gpu": T, "scored_positions_per_gpu": S, "rank": w.rank,
                   "targets": [wl.MATRIX_NAMES[m] for m in w.matrices],
                   "parallelism": f"dp{world}" if world > 1 else "single",
                   "l2": "inputs larger than L2 (weights %.1f GB read every step)" %
                         ((sh.body_params() + sh.vocab * sh.d_model) * 2 / 1e9),
                   "gemm_impl": "cuda-cores" if args.cuda_cores else "tcgen05",
                   "fp8": bool(args.fp8),
                   **({"layers_slice": args.layers, "note": "layer slice for profiling, not a "
                       "bench line"} if args.layers else {})},
        "steps_per_s": steps_s,
        "scored_tokens_per_s": tok_s,
        "target_tokens_per_s": world * S / (ms / 1000.0),
        "step_roofline": {"flops": flops_all, "bytes": bytes_ * world,
                          "roofline_ms": roof_t * 1000.0, "frac": roof_t * 1000.0 / ms,
                          "peak": f"{peak_kind} bf16 {peak_t} TFLOP/s sustained"
                                  + (" (E4M3 share at 2x)" if args.fp8 else "")
                                  + f", HBM {peaks['hbm_gbs']} GB/s"},
        "roofline": {"kernel": "tcgen05 GEMM (gemm_tc2_kernel SM pairs + gemm_tc_kernel; all epilogues)",
                     "bound": "tensor",
                     "achieved": gemm_tflops, "peak": peak_g, "unit": "TFLOP/s",
                     "frac": (gemm_tflops / peak_g) if gemm_tflops else None,
                     "traffic": gemm_traffic(), "launches_timed": d_n,
                     "algorithmic_flops_per_launch": d_fl / d_n if d_n else None,
                     "avg_launch_ms": d_ms / d_n if d_n else None,
                     "peak_kind": f"{peak_kind} (sustained: the kernel runs inside a long step)"
                                  + ("; E4M3 launches at 2x the bf16 figure" if args.fp8 else ""),
                     "share_of_step": (d_ms / args.steps) / ms if d_n else None},
        "state_transition": {"bytes_per_step": (s1["state_transition_bytes"] -
                                                s0["state_transition_bytes"]) / args.steps,
                             "dense_ref_bytes_per_step": (s1["dense_ref_bytes"] -
                                                          s0["dense_ref_bytes"]) / args.steps,
                             "dense_ref_targets_per_step": (s1["dense_ref_bytes_targets"] -
                                                            s0["dense_ref_bytes_targets"]) / args.steps},
        "phases_ms_per_step": {k: (s1[k] - s0[k]) / args.steps for k in ("ms_plan", "ms_score",
                                                                         "ms_step")},
        "matched_query_control": {"score_only_ms": control_ms, "step_over_control": ms / control_ms},
        "cobatch": cobatch,
        "step_graph": graph,
        "gpu_launches": int(s1["kernel_launches"] - s0["kernel_launches"]),
        "e2e": e2e,
        "clocks": clocks,
    }
    st = line["state_transition"]
    st["frac_of_dense"] = st["bytes_per_step"] / st["dense_ref_bytes_per_step"]
    st["frac_of_dense_targets"] = st["bytes_per_step"] / st["dense_ref_targets_per_step"]
    if cobatch is None and world == 1 and not args.no_cobatch:
        # the co-serving analogue on the co-batching workload, measured in the same run
        h.close()
        del model
        torch.cuda.empty_cache()
        line["cobatch"] = cobatch_leg(args.steps)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = oracle_sample(w, n_prompts=args.baseline_prompts)
        line["cpu_baseline"] = {"value": cb["tokens_per_s"], "unit": "scored tokens/s",
                                "cores": cb["cores"], "kind": "oracle", "sample": cb["sample"],
                                "extrapolated": cb["extrapolated"],
                                "sample_seconds": cb["sample_seconds"],
                                "layer_scale": cb["layer_scale"]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    h.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
