#!/usr/bin/env python
"""Throughput benchmark of the Psi-Spec decode iteration on one B200.

A step is one Psi-Spec iteration (draft pass, draft_sample, verify pass,
spec_verify + commit) over the whole batch.  The default workload is the
Qwen3-8B-shaped model (bf16, random init) with a rank-128 / alpha-256 LoRA,
B = 16, batch 1, on the 1K-input / 8K-output test: the prompt holds 1024
tokens and a request generates 8192, so its context runs from 1024 to 9216;
the timed window is centred on the mean context of that run (5120) by
prefilling a synthetic continuation first (the cost of an iteration depends
on the context length and on nothing else the synthetic tokens could change).

`value` is generated tokens/s over the timed steps (inputs resident, device
time by CUDA events, max over ranks); `e2e` is the same metric through the
public C ABI with the request ids copied from pinned host memory and the
emitted tokens copied back every step.  With --gpus N > 1 (torchrun) every
rank runs an independent replica on its own requests (the path has no
exchange step): replicas only, weak scaling.

--impl reference times the CPU oracle instead, on a bounded sample of the
same workload (see `oracle_step_sample`).
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# Clock sampling during the timed region.
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            # the timed region starts once the sampler is producing lines;
            # samples taken before it are dropped
            t0 = time.time()
            while not self.lines and time.time() - t0 < 3.0 and self.proc.poll() is None:
                time.sleep(0.01)
            self.lines.clear()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample).
# ---------------------------------------------------------------------------
def oracle_step_sample(cfg, context, tokens_per_step, budget_s=20.0):
    """Seconds per Psi-Spec iteration of the oracle, from a bounded sample.

    The sample runs the oracle's draft and verify forwards through ONE layer
    of the workload's shape (random float64 weights, a KV cache of `context`
    positions) plus the final norm, the LM head and the sampler over the
    block; the per-iteration time is layers x (one-layer time) + head time.
    """
    from oracle import model as om
    from oracle import psispec as ops

    one = dict(synth_shape(cfg), n_layers=1)
    rng = np.random.default_rng(0)
    params = {}
    for name, shp in om.param_names(one):
        params[name] = np.ones(shp) if name.endswith("norm") else rng.standard_normal(shp) * 0.02
    m = om.Model(one, params)
    Hkv, hd, B = one["n_kv_heads"], one["head_dim"], cfg["B"]
    cache = om.KVCache(one)
    cache.k[0] = rng.standard_normal((context, Hkv, hd))
    cache.v[0] = rng.standard_normal((context, Hkv, hd))
    st = ops.DecodeState(list(rng.integers(0, one["vocab"] - 1, context + 1)), cache, 0)
    head = params["lm_head"]
    t0 = time.perf_counter()
    reps = 0
    layer_t = head_t = 0.0
    while True:
        a = time.perf_counter()
        # one layer of the draft pass (B+1 rows) and of the verify pass (B rows)
        ops.draft_pass(m, st, B)
        cache2 = st.cache.copy()
        ops.verify_pass(m, cache2, st.c, [int(t) for t in rng.integers(0, one["vocab"], B)])
        b = time.perf_counter()
        # LM head over the 2B+1 rows, and the sampler over the block
        h = rng.standard_normal((2 * B + 1, one["d_model"]))
        logits = h @ head.T
        for i in range(B):
            ops.sample_token(logits[i], 0.5)
        ops.verify_block(list(logits[B:2 * B - 1]), list(logits[1:B]), [1] * (B - 1),
                         [0.5] * (B - 1), [0.5] * B, logits[2 * B])
        c = time.perf_counter()
        layer_t += b - a
        head_t += c - b
        reps += 1
        if c - t0 > budget_s or reps >= 3:
            break
    # the one-layer passes include the embedding/head of the 1-layer model;
    # subtract nothing (a small overestimate of the per-layer time)
    step_s = cfg["n_layers"] * layer_t / reps + head_t / reps
    desc = (f"oracle (numpy float64) draft+verify forwards of 1 of {cfg['n_layers']} layers at "
            f"context {context} plus LM head and sampler, x{reps}, scaled to {cfg['n_layers']} layers")
    return step_s, desc


# ---------------------------------------------------------------------------
# DRAM traffic of the dominant kernel, from the committed ncu summary.  The
# summary records a hash of the kernel's source files; the figure is used
# only while the sources still hash the same (else the traffic is unknown).
# ---------------------------------------------------------------------------
GEMM_SOURCES = ("lossless_diffusion_draft_b200/csrc/gemm_tc.cuh",
                "lossless_diffusion_draft_b200/csrc/tc_common.cuh")
GEMM_PROFILE = "profiles/gemm_tc_gate_up_qwen8b.md"


def source_hash(paths):
    import hashlib
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(top):
    import re
    path = os.path.join(ROOT, GEMM_PROFILE)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    h = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
    shape = re.search(r"shape:\s*M=(\d+) N=(\d+) K=(\d+)", text)
    b = re.search(r"dram_bytes_per_launch:\s*(\d+)", text)
    if not (h and shape and b) or h.group(1) != source_hash(GEMM_SOURCES):
        return None
    if tuple(int(x) for x in shape.groups()) != (top["m"], top["n"], top["k"]):
        return None
    return int(b.group(1))


def synth_shape(cfg):
    from lossless_diffusion_draft_b200 import synth
    return synth.model_shape(cfg)


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


# ---------------------------------------------------------------------------
# Workload set-up.
# ---------------------------------------------------------------------------
def kv_bytes_per_token(cfg):
    # bf16 models: K as an fp16 hi/lo pair and V in fp16 (three planes)
    esz, planes = (2, 3) if cfg["dtype"] == "bf16" else (4, 2)
    return cfg["n_layers"] * planes * cfg["n_kv_heads"] * cfg["head_dim"] * esz


def max_batch_that_fits(cfg, weight_bytes, max_ctx):
    free, _ = torch.cuda.mem_get_info()
    per_req = (-(-(max_ctx + cfg["B"] + 2) // 64) * 64) * kv_bytes_per_token(cfg)
    per_req += (2 * cfg["B"] + 1) * cfg["vocab"] * 4          # logits
    reserve = 6 << 30                                         # activations, workspaces
    return max(1, int((free - reserve) // per_req))


def run_uno(args, rank, world, device):
    from lossless_diffusion_draft_b200 import synth, uno

    cfg = dict(synth.CONFIGS[args.workload])
    if args.layers:
        cfg["n_layers"] = args.layers
    shape = synth.model_shape(cfg)
    shape["dtype"] = cfg["dtype"]
    B = cfg["B"]
    prompt_len, gen = cfg["prompt_len"], cfg["gen_tokens"]
    max_ctx = prompt_len + gen + B + 1
    params = synth.make_params(cfg, device)
    weight_bytes = sum(t.numel() * t.element_size() for t in params.values())
    batch = cfg["batch"] or max_batch_that_fits(cfg, weight_bytes, max_ctx)
    stream = torch.cuda.current_stream()
    ctx = uno.uno_init(shape, params, cfg["lora_rank"], cfg["lora_alpha"], B, batch, max_ctx,
                       cfg["seed"], stream)
    if args.no_pdl:
        uno.uno_set_pdl(ctx, False)
    if args.no_counter_sync:
        uno.uno_set_counter_sync(ctx, False)
    fused = uno.uno_set_fused(ctx, not args.no_fused) and not args.no_fused
    if args.no_graphs:
        uno.uno_set_graphs(ctx, False)

    # centre the timed window on the run's mean context
    mean_ctx = prompt_len + gen // 2
    est_tok = args.est_tokens_per_step
    start_ctx = max(prompt_len, int(mean_ctx - (args.warmup + args.steps) * est_tok / 2))
    P = start_ctx + 1
    prompts = synth.make_prompts(cfg, batch, P, seed=cfg["seed"] + 1000 * rank)
    streams = replica_streams(rank, batch)
    t0 = time.time()
    ids = uno.uno_prefill(ctx, torch.from_numpy(prompts).to(device), [P] * batch, streams=streams)
    torch.cuda.synchronize()
    prefill_s = time.time() - t0
    req = torch.tensor(ids, dtype=torch.int32, device=device)
    out = torch.zeros((batch, B + 1), dtype=torch.int32, device=device)
    K, W = args.steps, args.warmup
    n_new_all = torch.zeros((K, batch), dtype=torch.int32, device=device)
    for _ in range(W):
        uno.uno_spec_step(ctx, req, out, n_new_all[0])
    torch.cuda.synchronize()
    uno.uno_status(ctx)
    ctx_before = [uno.uno_request_state(ctx, i)[0] for i in ids[:1]][0]

    barrier(world)
    uno.uno_profile_begin(ctx, 0)          # launch counting only
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev_step = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        torch.cuda.synchronize()
        # a profiler started with --profile-from-start off sees the timed
        # steps only
        torch.cuda.profiler.start()
        ev0.record(stream)
        for k in range(K):
            uno.uno_spec_step(ctx, req, out, n_new_all[k])
            ev_step[k].record(stream)
        ev1.record(stream)
        torch.cuda.synchronize()
        torch.cuda.profiler.stop()
    prof = uno.uno_profile_end(ctx)
    barrier(world)
    ms = ev0.elapsed_time(ev1)
    step_ms = [ev0.elapsed_time(ev_step[0])] + [ev_step[k - 1].elapsed_time(ev_step[k])
                                                 for k in range(1, K)]
    tokens = int(n_new_all.sum().item())
    ctx_after = uno.uno_request_state(ctx, ids[0])[0]
    launches = sum(v[0] for v in prof.values())

    # per-kernel-class device time: the same number of steps again with event
    # pairs around every launch of the profiled classes
    uno.uno_profile_begin(ctx, (1 << uno.UNO_K_GEMM) | (1 << uno.UNO_K_ATTN) |
                          (1 << uno.UNO_K_SAMPLE) | (1 << uno.UNO_K_VERIFY) | (1 << uno.UNO_K_OTHER))
    for k in range(K):
        uno.uno_spec_step(ctx, req, out, n_new_all[k])
    kprof = uno.uno_profile_end(ctx)
    shapes = {}
    esz = 2 if cfg["dtype"] == "bf16" else 4
    for rec in uno.uno_profile_records(ctx):
        key = (rec["cls"], rec["m"], rec["n"], rec["k"], rec["r"])
        cnt, ms_sum = shapes.get(key, (0, 0.0))
        shapes[key] = (cnt + 1, ms_sum + rec["ms"])
    detail = []
    for (cls, m, n, k, r), (cnt, ms_sum) in sorted(shapes.items(), key=lambda kv: -kv[1][1]):
        row = {"cls": cls, "calls_per_step": cnt / K, "us_per_call": 1e3 * ms_sum / cnt,
               "ms_per_step": ms_sum / K}
        if cls == "gemm":
            row.update(m=m, n=n, k=k, r=r)
            wbytes = (n * k + n * r + m * k + m * r) * esz
            row["GBps"] = wbytes / (ms_sum / cnt / 1e3) / 1e9
        detail.append(row)

    # end to end through the C ABI with host buffers
    req_h = torch.tensor(ids, dtype=torch.int32).pin_memory()
    out_h = torch.zeros((batch, B + 1), dtype=torch.int32).pin_memory()
    nn_h = torch.zeros(batch, dtype=torch.int32).pin_memory()
    req_d = torch.empty_like(req)
    nn_d = torch.zeros(batch, dtype=torch.int32, device=device)
    e2e_tokens = 0
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(K):
        req_d.copy_(req_h, non_blocking=True)
        uno.uno_spec_step(ctx, req_d, out, nn_d)
        out_h.copy_(out, non_blocking=True)
        nn_h.copy_(nn_d, non_blocking=True)
        stream.synchronize()
        e2e_tokens += int(nn_h.sum())
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    uno.uno_status(ctx)

    # the AR-only decode of the same model from the same kernels (one token per
    # request per step, LoRA never read): the baseline Psi-Spec is measured
    # against
    ar_out = torch.zeros(batch, dtype=torch.int32, device=device)
    for _ in range(W):
        uno.uno_ar_step(ctx, req, ar_out)
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(K):
        uno.uno_ar_step(ctx, req, ar_out)
    a1.record(stream)
    torch.cuda.synchronize()
    ar_ms = a0.elapsed_time(a1) / K
    uno.uno_status(ctx)

    # aggregate over ranks: tokens summed, time = max
    ms_max = reduce_max(ms, world, device)
    e2e_ms_max = reduce_max(e2e_ms, world, device)
    tokens_all = reduce_sum(tokens, world, device)
    e2e_tokens_all = reduce_sum(e2e_tokens, world, device)

    info = dict(cfg=cfg, batch=batch, B=B, ms=ms_max, fused=fused, step_ms=step_ms, ar_ms=ar_ms, tokens=tokens_all, K=K, W=W,
                e2e_ms=e2e_ms_max, e2e_tokens=e2e_tokens_all, clocks=clk.summary(),
                launches=launches, kprof=kprof, prefill_s=prefill_s, detail=detail[:24],
                ctx_window=[ctx_before, ctx_after], weight_bytes=weight_bytes,
                h2d=req_h.numel() * 4, d2h=(out_h.numel() + nn_h.numel()) * 4)
    ctx.close()
    return info


def run_micro(args, device):
    """Kernel microbenchmarks (not the headline line): one kernel, K timed calls.

    gemm:        uno_gated_lora_linear at a decode shape (--shape M,N,K,r), bf16;
                 algorithmic bytes = weights + adapter + activations + fp32 output.
    spec_verify: the spec_verify workload, p/q fp32 [4096 = 256 x 16, 151936];
                 algorithmic bytes = both logit tensors read once.
    """
    from lossless_diffusion_draft_b200 import synth, uno
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pk = peaks()
    if args.workload == "gemm":
        M, N, K, r = (int(x) for x in args.shape.split(","))
        g = torch.Generator(device=device).manual_seed(0)
        X = torch.randn((M, K), generator=g, device=device).to(torch.bfloat16)
        W = (torch.randn((N, K), generator=g, device=device) * 0.02).to(torch.bfloat16)
        A = (torch.randn((r, K), generator=g, device=device) * 0.02).to(torch.bfloat16) if r else None
        Bl = (torch.randn((N, r), generator=g, device=device) * 0.002).to(torch.bfloat16) if r else None
        gate = torch.ones(M, device=device) if r else None
        Y = torch.empty((M, N), device=device)
        ws = torch.zeros(uno.uno_gated_lora_linear_workspace_bytes(M, N, K, r, uno.UNO_BF16),
                         dtype=torch.uint8, device=device)
        # the weights (>= tens of MB) are rotated through copies so that each
        # call streams from HBM, not from L2
        copies = max(1, int(512e6 // max(1, W.numel() * 2)))
        Ws = [W.clone() for _ in range(min(copies, 8))]
        call = lambda i: uno.uno_gated_lora_linear(X, Ws[i % len(Ws)], A, Bl, gate, 2.0, Y, ws)
        nbytes = (N * K + N * r + M * K + M * r + r * K) * 2 + M * N * 4
        unit, metric = "calls/s", f"gated_lora_linear M={M} N={N} K={K} r={r}"
    else:
        cfg = synth.SPEC_VERIFY_BENCH
        n_req, R, V = args.sv_requests or cfg["requests"], cfg["rows_per_request"], cfg["vocab"]
        p, q = synth.make_verify_logits(n_req * R, V, device, cfg["p_std"], cfg["q_noise_std"],
                                        cfg["logits_seed"])
        drafts = synth.make_drafts(q, seed=cfg["logits_seed"] + 1).view(n_req, R)
        p, q = p.view(n_req, R, V), q.view(n_req, R, V)
        streams = torch.arange(n_req, dtype=torch.int32, device=device)
        pos0 = torch.zeros(n_req, dtype=torch.int32, device=device)
        ws = torch.zeros(uno.uno_spec_verify_workspace_bytes(n_req, R, V), dtype=torch.uint8,
                         device=device)
        out = torch.empty((n_req, R + 1), dtype=torch.int32, device=device)
        n_out = torch.empty(n_req, dtype=torch.int32, device=device)
        call = lambda i: uno.uno_spec_verify(p, q, drafts, cfg["seed"], streams, pos0, out, n_out, ws)
        nbytes = 2 * n_req * R * V * 4
        unit, metric = "rows/s", "spec_verify [4096 x 151936] fp32 p and q"
    for i in range(args.warmup):
        call(i)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        ev0.record(stream)
        for i in range(args.steps):
            call(i)
        ev1.record(stream)
        torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1) / args.steps
    gbs = nbytes / (ms / 1e3) / 1e9
    value = (nbytes // (2 * V * 4) if args.workload == "spec_verify" else 1) / (ms / 1e3)
    line = {"metric": metric, "value": value, "unit": unit, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "dtype": "bf16" if args.workload == "gemm" else "f32", "data": "synthetic",
            "config": ({"workload": args.workload, "requests": nbytes // (2 * V * 4) // 16,
                        "rows": nbytes // (2 * V * 4), "vocab": V}
                       if args.workload == "spec_verify" else
                       {"workload": args.workload, "shape": args.shape}),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": None,
                         "algorithmic_bytes_per_call": nbytes, "peak_source": pk["source"]},
            "clocks": clk.summary()}
    print(json.dumps(line), flush=True)


def replica_streams(rank, batch):
    """Philox streams of a rank's requests: each replica draws from its own,
    disjoint from every other rank's."""
    return [rank * batch + i for i in range(batch)]


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def reduce_max(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([float(x)], device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return int(t.item())


def step_bytes(info):
    """Algorithmic HBM bytes of one iteration (per request KV at the window's
    mean context; weights once per pass for the whole batch)."""
    cfg = info["cfg"]
    esz = 2 if cfg["dtype"] == "bf16" else 4
    from lossless_diffusion_draft_b200 import synth
    base = lora = 0
    for name, shp, kind in synth.param_list(cfg):
        n = int(np.prod(shp)) * esz
        if kind in ("lora_a", "lora_b"):
            lora += n
        elif name != "embed":
            base += n
    ctx = sum(info["ctx_window"]) / 2
    kv = ctx * kv_bytes_per_token(cfg) * 2 * info["batch"]
    logits = (2 * cfg["B"] + 1) * cfg["vocab"] * 4 * 2 * info["batch"]
    return 2 * base + lora + kv + logits


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="uno", choices=["uno", "reference"])
    ap.add_argument("--workload", default="qwen8b",
                    choices=["qwen8b", "qwen8b_maxbatch", "small", "tiny", "gemm", "spec_verify"])
    ap.add_argument("--shape", default="17,4096,4096,128",
                    help="gemm microbenchmark shape M,N,K,r")
    ap.add_argument("--sv-requests", type=int, default=0,
                    help="spec_verify microbenchmark: requests (default: the workload's 256); "
                         "fewer only for small profiler captures")
    ap.add_argument("--no-pdl", action="store_true", help="plain stream-ordered launches")
    ap.add_argument("--no-fused", action="store_true",
                    help="unfused layer pipeline (separate LoRA-A GEMMs, norm, RoPE, SwiGLU)")
    ap.add_argument("--no-graphs", action="store_true", help="no CUDA-graph capture of steps")
    ap.add_argument("--no-counter-sync", action="store_true",
                    help="fused pipeline: GEMMs wait on grid dependencies, not completion counters")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the layer count (small cases for profiler captures; the "
                         "line's config records it)")
    ap.add_argument("--est-tokens-per-step", type=float, default=2.6)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    from lossless_diffusion_draft_b200 import synth
    if args.workload in ("gemm", "spec_verify"):
        from lossless_diffusion_draft_b200 import build
        build.build()
        run_micro(args, torch.device("cuda", local))
        return
    cfg = synth.CONFIGS[args.workload]
    metric = "generated tokens/s (Psi-Spec, 1K in / 8K out)"

    if args.impl == "reference":
        if rank != 0:
            return
        ctx_len = cfg["prompt_len"] + cfg["gen_tokens"] // 2
        tps = args.est_tokens_per_step
        times = []
        desc = ""
        for i in range(args.warmup + args.steps):
            s, desc = oracle_step_sample(cfg, ctx_len, tps, budget_s=0.0)
            if i >= args.warmup:
                times.append(s)
        step_s = sum(times) / len(times)
        value = tps * cfg["batch"] / step_s if cfg["batch"] else tps / step_s
        line = {"impl": "reference", "metric": metric, "value": value, "unit": "tokens/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": args.workload, "batch": cfg["batch"], "B": cfg["B"]},
                "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_cores(),
                                 "kind": "oracle", "sample": desc + f"; {tps} tokens per iteration assumed"},
                "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    from lossless_diffusion_draft_b200 import build
    build.build()

    info = run_uno(args, rank, world, device)
    pk = peaks()
    value = info["tokens"] / (info["ms"] / 1e3)
    e2e = info["e2e_tokens"] / (info["e2e_ms"] / 1e3)
    kp = info["kprof"]
    g_launch, g_ms, g_bytes = kp["gemm"]
    g_gbs = g_bytes / (g_ms / 1e3) / 1e9 if g_ms > 0 else None
    # the dominant kernel: the GEMM shape with the largest share of the step
    gemms = [d for d in info["detail"] if d["cls"] == "gemm"]
    top = max(gemms, key=lambda d: d["ms_per_step"]) if gemms else None
    if top:
        esz = 2 if cfg["dtype"] == "bf16" else 4
        top_bytes = (top["n"] * top["k"] + top["n"] * top["r"] + top["m"] * top["k"] +
                     top["m"] * top["r"]) * esz
        achieved = top_bytes / (top["us_per_call"] * 1e-6) / 1e9
        traffic = profiled_traffic(top)
        top_flops = 2.0 * top["m"] * top["n"] * (top["k"] + top["r"])
        # which roof binds: bytes at the measured copy rate against flops at
        # the measured bf16 rate (sustained: the kernel runs inside a long step)
        t_hbm = top_bytes / (pk["hbm_gbs"] * 1e9)
        tc_peak = pk["bf16_tflops_sustained"] or pk["bf16_tflops"]
        t_tc = top_flops / (tc_peak * 1e12)
        kernel_desc = (f"gated_lora_linear M={top['m']} N={top['n']} K={top['k']} "
                       "(gemm_tc_kernel, the step's largest GEMM)")
        common = {"kernel": kernel_desc, "algorithmic_bytes": top_bytes,
                  "algorithmic_flops": top_flops, "avg_launch_us": top["us_per_call"],
                  "launches_per_step": top["calls_per_step"], "peak_source": pk["source"],
                  "all_gemm_launches": {"achieved_GBps": g_gbs, "launches": g_launch,
                                        "avg_launch_us": g_ms * 1e3 / max(1, g_launch)}}
        if t_tc > t_hbm:
            tflops = top_flops / (top["us_per_call"] * 1e-6) / 1e12
            roofline = dict({"bound": "tensor", "achieved": tflops, "peak": tc_peak,
                             "unit": "TFLOP/s", "frac": tflops / tc_peak, "traffic": None,
                             "peak_kind": "bf16 sustained",
                             "note": "every activation row is fed as a bf16 hi/lo pair, so the "
                                     "tensor cores execute twice the algorithmic flops"}, **common)
        else:
            roofline = dict({"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"],
                             "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                             "traffic": traffic}, **common)
    else:
        roofline = {"bound": "hbm", "kernel": "gated_lora_linear (SIMT)", "achieved": g_gbs,
                    "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": (g_gbs / pk["hbm_gbs"]) if g_gbs else None, "traffic": None,
                    "peak_source": pk["source"]}
    per_step_ms = info["ms"] / info["K"]
    sb = step_bytes(info)
    step_roof = {"algorithmic_bytes_per_step": sb, "achieved_GBps": sb / (per_step_ms / 1e3) / 1e9,
                 "frac_of_hbm_peak": sb / (per_step_ms / 1e3) / 1e9 / pk["hbm_gbs"]}
    breakdown = {k: {"launches": v[0], "ms_per_step": v[1] / info["K"]} for k, v in kp.items()}

    line = {
        "metric": metric, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": info["K"], "warmup": info["W"], "ms_per_step": per_step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg["dtype"],
        "data": "synthetic (random-init weights, uniform-random prompt tokens)",
        "config": {"workload": args.workload, "n_layers": info["cfg"]["n_layers"],
                   "batch": info["batch"], "B": info["B"], "pdl": not args.no_pdl,
                   "fused": info["fused"],
                   "graphs": not args.no_graphs,
                   "prompt_len": cfg["prompt_len"], "gen_tokens": cfg["gen_tokens"],
                   "context_window": info["ctx_window"], "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (15+ GB of weights streamed per pass)"},
        "tokens_per_step": info["tokens"] / info["K"],
        "step_latency_ms": {"median": statistics.median(info["step_ms"]),
                            "min": min(info["step_ms"]), "max": max(info["step_ms"])},
        "mean_accepted_a": info["tokens"] / info["K"] / info["batch"] / max(1, world) - 1,
        "ar_only": {"value": info["batch"] / (info["ar_ms"] / 1e3), "unit": "tokens/s",
                    "ms_per_step": info["ar_ms"],
                    "note": "uno_ar_step on the same requests and kernels, one token per request"},
        "tpf": info["tokens"] / info["K"] / info["batch"] / 2 / max(1, world),
        "roofline": roofline, "step_roofline": step_roof, "kernel_breakdown": breakdown,
        "e2e": {"value": e2e, "unit": "tokens/s", "h2d_bytes_per_step": info["h2d"],
                "d2h_bytes_per_step": info["d2h"]},
        "gpu_launches": info["launches"], "clocks": info["clocks"],
        "kernel_detail": info["detail"],
        "prefill_s": info["prefill_s"],
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps = info["tokens"] / info["K"] / info["batch"]
        ctx_len = sum(info["ctx_window"]) // 2
        s, desc = oracle_step_sample(cfg, ctx_len, tps)
        line["cpu_baseline"] = {"value": tps * info["batch"] / s, "unit": "tokens/s",
                                "cores": cpu_cores(), "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
