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
same workload (see `OracleSample`).
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
    """SM clocks and clock-event reasons of one GPU while the timed region
    runs: NVML read every 10 ms from a thread (the timed regions are a few
    hundred ms long), else `nvidia-smi -lms 50`.  Read-only: no setting of
    the GPU is touched."""

    PERIOD_S = 0.01
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    NVML_BITS = {"hw_slowdown": "HwSlowdown", "hw_thermal_slowdown": "HwThermalSlowdown",
                 "sw_thermal_slowdown": "SwThermalSlowdown", "sw_power_cap": "SwPowerCap"}
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, enabled=True, nvml=None):
        self.gpu = gpu_index
        self.enabled = enabled
        self.samples = []          # (time, sm MHz, max sm MHz, set of reason names)
        self._t0 = float("inf")
        self.source = None
        self._nvml = nvml          # a pynvml-like module (tests pass a fake)
        self._proc = None
        self._thread = None
        self._stop = threading.Event()

    def _uuid(self):
        import re
        try:
            u = str(torch.cuda.get_device_properties(self.gpu).uuid)
        except Exception:
            return None
        m = re.search(r"[0-9a-fA-F]{8}(-[0-9a-fA-F]{4}){3}-[0-9a-fA-F]{12}", u)
        return "GPU-" + m.group(0) if m else None

    def _nvml_start(self):
        nv = self._nvml
        if nv is None:
            import pynvml as nv
        nv.nvmlInit()
        uuid, h = self._uuid(), None
        if uuid:
            try:
                h = nv.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                h = None
        if h is None:
            h = nv.nvmlDeviceGetHandleByIndex(self.gpu)
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        bits = {}
        for name, suffix in self.NVML_BITS.items():
            b = getattr(nv, "nvmlClocksEventReason" + suffix, None)
            bits[name] = b if b is not None else getattr(nv, "nvmlClocksThrottleReason" + suffix)

        def read():
            mask = get_reasons(h)
            return (float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                    float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)),
                    {n for n, b in bits.items() if mask & b})

        read()   # fails here, before the timed region, if NVML cannot read

        def loop():
            while not self._stop.is_set():
                t = time.time()
                try:
                    self.samples.append((t,) + read())
                except Exception:
                    break
                self._stop.wait(self.PERIOD_S)
            try:
                nv.nvmlShutdown()
            except Exception:
                pass
        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        self.source = "nvml"

    def _smi_start(self):
        self._proc = subprocess.Popen(
            ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
             "--format=csv,noheader,nounits", "-lms", "50"],
            stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        lines = []

        def reader():
            for line in self._proc.stdout:
                lines.append(line.strip())
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    sm, mx = float(f[1]), float(f[2])
                except ValueError:
                    continue
                self.samples.append((time.time(), sm, mx, {n for n, v in zip(self.REASONS, f[5:9])
                                                           if v.lower() == "active"}))
        self._thread = threading.Thread(target=reader, daemon=True)
        self._thread.start()
        # the timed region starts once the sampler is producing lines
        t0 = time.time()
        while not lines and time.time() - t0 < 3.0 and self._proc.poll() is None:
            time.sleep(0.01)
        self.source = "nvidia-smi"

    def __enter__(self):
        if not self.enabled:
            return self
        try:
            self._nvml_start()
        except Exception:
            try:
                self._smi_start()
            except OSError:
                self._proc = None
        self._t0 = time.time()   # samples taken before the timed region are dropped
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._proc:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
        if self._thread:
            self._thread.join(timeout=5)

    def summary(self):
        smp = [x for x in self.samples if x[0] >= self._t0]
        if not smp:
            return None
        return {"sm_mhz": statistics.median(x[1] for x in smp), "sm_max_mhz": smp[-1][2],
                "reasons": sorted(set().union(*(x[3] for x in smp))),
                "samples": len(smp), "source": self.source}


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample).
# ---------------------------------------------------------------------------
class OracleSample:
    """The CPU oracle on a bounded sample of a workload's Psi-Spec iteration.

    The oracle's own iteration (draft forward, draft_sample, verify forward,
    spec_verify with its residual or bonus draw, commit) runs on a ONE-layer
    model of the workload's shape - full vocabulary, random float64 weights
    (base N(0, 0.02), LoRA B N(0, b_std)), a KV cache of `context` random
    positions - which gives the cost of the LM head and the sampler and the
    tokens the iteration emits.  The draft and verify forwards of one layer
    alone (a 16-token vocabulary, so no head cost) are timed beside it.  The
    iteration time of the L-layer model is then
        T(iteration, 1 layer) + (L - 1) * T(one layer's two forwards),
    and the tokens per iteration are those the sampled iterations emitted.
    """

    def __init__(self, cfg, context, seed=0):
        from oracle import model as om
        from oracle import psispec as ops
        self.om, self.ops, self.cfg = om, ops, cfg
        self.L = cfg["n_layers"]
        rng = np.random.default_rng(seed)
        self.full = self._model(dict(synth_shape(cfg), n_layers=1), rng)
        small = dict(synth_shape(cfg), n_layers=1, vocab=16, mask_id=15)
        self.layer = self._model(small, rng)
        Hkv, hd = cfg["n_kv_heads"], cfg["head_dim"]
        cache = om.KVCache(self.full.shape)
        cache.k[0] = rng.standard_normal((context, Hkv, hd))
        cache.v[0] = rng.standard_normal((context, Hkv, hd))
        toks = [int(t) for t in rng.integers(0, cfg["vocab"] - 1, context + 1)]
        self.state = ops.DecodeState(toks, cache, 0)
        self.context = context

    def _model(self, shape, rng):
        params = {}
        for name, shp in self.om.param_names(shape):
            if name.endswith("norm"):
                params[name] = np.ones(shp)
            else:
                std = self.cfg["lora_b_std"] if name.endswith(".B") else 0.02
                params[name] = rng.standard_normal(shp, dtype=np.float32).astype(np.float64) * std
        return self.om.Model(shape, params)

    def step(self, it):
        """One sampled iteration: (seconds for the L-layer model, tokens emitted)."""
        ops, B = self.ops, self.cfg["B"]
        st = self.state
        t0 = time.perf_counter()
        _, res = ops.spec_step(self.full, st, B, self.cfg["seed"] + it)
        t1 = time.perf_counter()
        small = ops.DecodeState([1] * (st.c + 1), st.cache, 0)
        ops.draft_pass(self.layer, small, B)
        cache2 = st.cache.copy()
        ops.verify_pass(self.layer, cache2, st.c, [1] * B)
        t2 = time.perf_counter()
        return (t1 - t0) + (self.L - 1) * (t2 - t1), len(res.emitted)

    def describe(self, n):
        return (f"oracle (numpy float64) Psi-Spec iterations on a 1-layer model of the workload's "
                f"shape (full vocabulary) at context {self.context}, plus {self.L - 1} x the draft and "
                f"verify forwards of one layer; {n} sampled iterations; tokens per iteration "
                f"measured from those iterations")


def oracle_baseline(cfg, context, budget_s=20.0, max_iters=3):
    """(tokens/s, seconds per iteration, tokens per iteration, description)."""
    s = OracleSample(cfg, context)
    t0 = time.perf_counter()
    times, toks = [], []
    while True:
        t, n = s.step(len(times))
        times.append(t)
        toks.append(n)
        if time.perf_counter() - t0 > budget_s or len(times) >= max_iters:
            break
    step_s = sum(times) / len(times)
    tpi = sum(toks) / len(toks)
    return tpi / step_s, step_s, tpi, s.describe(len(times))


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
    """KV-cache bytes a token holds in the library's layout (capacity): bf16
    models keep K as an fp16 hi/lo pair and V in fp16 (three planes)."""
    esz, planes = (2, 3) if cfg["dtype"] == "bf16" else (4, 2)
    return cfg["n_layers"] * planes * cfg["n_kv_heads"] * cfg["head_dim"] * esz


def kv_bytes_algorithmic(cfg):
    """KV bytes of a token in the model's own precision (K and V, each
    n_layers x n_kv_heads x head_dim elements): the roofline's figure
    (147,456 bytes for the Qwen3-8B shape in bf16)."""
    esz = 2 if cfg["dtype"] == "bf16" else 4
    return cfg["n_layers"] * 2 * cfg["n_kv_heads"] * cfg["head_dim"] * esz


def max_batch_that_fits(cfg, weight_bytes, max_ctx):
    free, _ = torch.cuda.mem_get_info()
    per_req = (-(-(max_ctx + cfg["B"] + 2) // 64) * 64) * kv_bytes_per_token(cfg)
    per_req += (2 * cfg["B"] + 1) * cfg["vocab"] * 4          # logits
    reserve = 6 << 30                                         # activations, workspaces
    return max(1, int((free - reserve) // per_req))


def step_profile(ctx, req, out, n_new, K, cfg):
    """Per-launch event times of K more steps, grouped by kernel class and GEMM
    shape: (per-class {launches, ms}, detail rows sorted by time per step)."""
    from lossless_diffusion_draft_b200 import uno
    uno.uno_profile_begin(ctx, (1 << uno.UNO_K_GEMM) | (1 << uno.UNO_K_ATTN) |
                          (1 << uno.UNO_K_SAMPLE) | (1 << uno.UNO_K_VERIFY) | (1 << uno.UNO_K_OTHER))
    for _ in range(K):
        uno.uno_spec_step(ctx, req, out, n_new)
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
    return kprof, detail


class Workload:
    """A context with `batch` requests prefilled to `context` tokens each."""

    def __init__(self, cfg, params, batch, context, rank, device, args):
        from lossless_diffusion_draft_b200 import synth, uno
        self.uno, self.cfg, self.batch, self.device = uno, cfg, batch, device
        shape = synth.model_shape(cfg)
        shape["dtype"] = cfg["dtype"]
        B = cfg["B"]
        self.B = B
        self.max_ctx = cfg["prompt_len"] + cfg["gen_tokens"] + B + 1
        self.ctx = uno.uno_init(shape, params, cfg["lora_rank"], cfg["lora_alpha"], B, batch,
                                self.max_ctx, cfg["seed"], torch.cuda.current_stream())
        if args.no_pdl:
            uno.uno_set_pdl(self.ctx, False)
        if args.no_counter_sync:
            uno.uno_set_counter_sync(self.ctx, False)
        self.fused = uno.uno_set_fused(self.ctx, not args.no_fused) and not args.no_fused
        if args.no_graphs:
            uno.uno_set_graphs(self.ctx, False)
        self.rank = rank
        self.ids = None
        self.out = torch.zeros((batch, B + 1), dtype=torch.int32, device=device)
        self.prefill(context)

    def prefill(self, context):
        """(Re-)admit every request with a synthetic prompt of `context` + 1
        tokens (cached: `context`, pending: the last)."""
        from lossless_diffusion_draft_b200 import synth
        uno = self.uno
        if self.ids is not None:
            for i in self.ids:
                uno.uno_release(self.ctx, i)
        P = context + 1
        prompts = synth.make_prompts(self.cfg, self.batch, P, seed=self.cfg["seed"] + 1000 * self.rank)
        t0 = time.time()
        self.ids = uno.uno_prefill(self.ctx, torch.from_numpy(prompts).to(self.device),
                                   [P] * self.batch, streams=replica_streams(self.rank, self.batch))
        torch.cuda.synchronize()
        self.prefill_s = time.time() - t0
        self.req = torch.tensor(self.ids, dtype=torch.int32, device=self.device)

    def cached(self):
        return self.uno.uno_request_state(self.ctx, self.ids[0])[0]

    def time_steps(self, K, W, world, ar=False, clocks=True, profile_range=False):
        """K timed steps after W untimed ones (device time by CUDA events,
        barrier and synchronize on both sides): dict(ms, tokens, step_ms,
        clocks, ctx_window, launches)."""
        uno, stream = self.uno, torch.cuda.current_stream()
        B = self.B
        # one output buffer for every step, so that each step replays the same
        # captured graph; each step's counts are copied into n_hist after it
        n_new = torch.zeros(self.batch, dtype=torch.int32, device=self.device)
        n_hist = torch.zeros((max(K, 1), self.batch), dtype=torch.int32, device=self.device)
        ar_out = torch.zeros(self.batch, dtype=torch.int32, device=self.device)

        def step(k):
            if ar:
                uno.uno_ar_step(self.ctx, self.req, ar_out)
            else:
                uno.uno_spec_step(self.ctx, self.req, self.out, n_new)
                n_hist[k].copy_(n_new, non_blocking=True)
        for _ in range(W):
            step(0)
        torch.cuda.synchronize()
        uno.uno_status(self.ctx)
        c0 = self.cached()
        barrier(world)
        uno.uno_profile_begin(self.ctx, 0)          # launch counting only
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        with ClockSampler(torch.cuda.current_device(), enabled=clocks) as clk:
            torch.cuda.synchronize()
            if profile_range:
                torch.cuda.profiler.start()
            ev0.record(stream)
            for k in range(K):
                step(k)
                ev[k].record(stream)
            ev1.record(stream)
            torch.cuda.synchronize()
            if profile_range:
                torch.cuda.profiler.stop()
        prof = uno.uno_profile_end(self.ctx)
        barrier(world)
        uno.uno_status(self.ctx)
        step_ms = [ev0.elapsed_time(ev[0])] + [ev[k - 1].elapsed_time(ev[k]) for k in range(1, K)]
        tokens = K * self.batch if ar else int(n_hist.sum().item())
        return dict(ms=ev0.elapsed_time(ev1), tokens=tokens, step_ms=step_ms,
                    clocks=clk.summary() if clocks else None, ctx_window=[c0, self.cached()],
                    launches=sum(v[0] for v in prof.values()), K=K)

    def e2e(self, K, W, world):
        """The same steps end to end through the C ABI: request ids copied from
        pinned host memory, emitted tokens and counts copied back, every step.
        W untimed steps first, with the same buffers: the library captures a
        step's graph on the second call with new buffer addresses, which is
        set-up, not a step."""
        uno, stream = self.uno, torch.cuda.current_stream()
        req_h = torch.tensor(self.ids, dtype=torch.int32).pin_memory()
        out_h = torch.zeros((self.batch, self.B + 1), dtype=torch.int32).pin_memory()
        nn_h = torch.zeros(self.batch, dtype=torch.int32).pin_memory()
        req_d = torch.empty_like(self.req)
        nn_d = torch.zeros(self.batch, dtype=torch.int32, device=self.device)
        def step():
            req_d.copy_(req_h, non_blocking=True)
            uno.uno_spec_step(self.ctx, req_d, self.out, nn_d)
            out_h.copy_(self.out, non_blocking=True)
            nn_h.copy_(nn_d, non_blocking=True)
            stream.synchronize()
            return int(nn_h.sum())
        for _ in range(W):
            step()
        tokens = 0
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            tokens += step()
        e1.record(stream)
        torch.cuda.synchronize()
        uno.uno_status(self.ctx)
        return dict(ms=e0.elapsed_time(e1), tokens=tokens, h2d=req_h.numel() * 4,
                    d2h=(out_h.numel() + nn_h.numel()) * 4)

    def close(self):
        self.ctx.close()


def gemm_roofline(detail, cfg, pk, steps_in_long_run=True):
    """Roofline of the step's dominant GEMM (largest share of the step):
    HBM-bound (algorithmic bytes over the measured copy rate) or tensor-bound
    (algorithmic flops over the measured bf16 rate, sustained: the kernel
    runs inside a long step), whichever binds."""
    gemms = [d for d in detail if d["cls"] == "gemm"]
    if not gemms:
        return None
    top = max(gemms, key=lambda d: d["ms_per_step"])
    esz = 2 if cfg["dtype"] == "bf16" else 4
    top_bytes = (top["n"] * top["k"] + top["n"] * top["r"] + top["m"] * top["k"] +
                 top["m"] * top["r"]) * esz
    top_flops = 2.0 * top["m"] * top["n"] * (top["k"] + top["r"])
    sec = top["us_per_call"] * 1e-6
    t_hbm = top_bytes / (pk["hbm_gbs"] * 1e9)
    tc_peak = (pk["bf16_tflops_sustained"] or pk["bf16_tflops"]) if steps_in_long_run else pk["bf16_tflops"]
    t_tc = top_flops / (tc_peak * 1e12)
    common = {"kernel": f"gated_lora_linear M={top['m']} N={top['n']} K={top['k']} r={top['r']} "
                        "(gemm_tc_kernel, the step's largest GEMM)",
              "algorithmic_bytes": top_bytes, "algorithmic_flops": top_flops,
              "avg_launch_us": top["us_per_call"], "launches_per_step": top["calls_per_step"],
              "peak_source": pk["source"]}
    if t_tc > t_hbm:
        tflops = top_flops / sec / 1e12
        # bf16 models feed every activation row as a hi/lo pair of bf16 rows:
        # the tensor cores execute twice the algorithmic flops
        executed = 2 * tflops if cfg["dtype"] == "bf16" else tflops
        return dict({"bound": "tensor", "achieved": tflops, "peak": tc_peak, "unit": "TFLOP/s",
                     "frac": tflops / tc_peak, "traffic": None, "peak_kind": "bf16 sustained",
                     "executed_TFLOPs": executed, "executed_frac": executed / tc_peak}, **common)
    achieved = top_bytes / sec / 1e9
    return dict({"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                 "frac": achieved / pk["hbm_gbs"], "traffic": profiled_traffic(top)}, **common)


def run_uno(args, rank, world, device):
    """The headline workload (and, on one GPU, the other measurements the
    line carries); returns the JSON line's fields."""
    from lossless_diffusion_draft_b200 import synth, uno

    cfg = dict(synth.CONFIGS[args.workload])
    if args.layers:
        cfg["n_layers"] = args.layers
    if args.batch:
        cfg["batch"] = args.batch
    B, prompt_len, gen = cfg["B"], cfg["prompt_len"], cfg["gen_tokens"]
    pk = peaks()
    params = synth.make_params(cfg, device)
    weight_bytes = sum(t.numel() * t.element_size() for t in params.values())
    max_ctx = prompt_len + gen + B + 1
    batch = cfg["batch"] or max_batch_that_fits(cfg, weight_bytes, max_ctx)
    K, W = args.steps, args.warmup
    # the timed window is centred on the run's mean context
    mean_ctx = prompt_len + gen // 2
    start = max(prompt_len, int(mean_ctx - (W + K) * args.est_tokens_per_step / 2))
    wl = Workload(cfg, params, batch, start, rank, device, args)
    head = wl.time_steps(K, W, world, profile_range=args.profile_range)
    kprof, detail = step_profile(wl.ctx, wl.req, wl.out, torch.zeros(batch, dtype=torch.int32,
                                                                     device=device), K, cfg)
    e2e = wl.e2e(K, W, world)
    ar = wl.time_steps(K, W, world, ar=True, clocks=False)
    res = dict(cfg=cfg, batch=batch, head=head, kprof=kprof, detail=detail, e2e=e2e, ar=ar,
               fused=wl.fused, prefill_s=wl.prefill_s, weight_bytes=weight_bytes, pk=pk)

    extras = world == 1 and not args.headline_only and args.workload == "qwen8b"
    if extras:
        # contexts across the 1K -> 9K run (the step's cost grows with the
        # context: KV bytes); a whole-run estimate from them by Simpson's rule
        pts = {}
        # the last point ends inside the request's pages even if every step
        # emitted B + 1 tokens
        for c0 in (prompt_len, prompt_len + gen - (W + K) * (B + 1)):
            wl.prefill(c0)
            pts[c0] = wl.time_steps(K, W, world, clocks=False)
        pts[head["ctx_window"][0]] = head
        res["contexts"] = pts
        # the benchmark tap: a trained drafter's acceptance (a = 4: five
        # tokens per iteration, TPF 2.5) at the mean context
        wl.prefill(start)
        uno.uno_debug_set_fixed_accept(wl.ctx, 4)
        res["fixed_accept"] = dict(wl.time_steps(K, W, world, clocks=False), a=4)
        uno.uno_debug_set_fixed_accept(wl.ctx, 0)
    wl.close()
    if extras:
        del wl
        torch.cuda.empty_cache()
        res["cohorts"] = run_cohorts(args, cfg, params, rank, world, device)
        res["tree"] = run_tree(args, cfg, params, rank, world, device)
        res["max_batch"] = run_max_batch(args, cfg, params, rank, world, device, pk)
        res["spec_verify_micro"] = spec_verify_micro(args, device, pk)
    return res


def run_cohorts(args, cfg, params, rank, world, device, batch=16):
    """Cohort-interleaved steps against plain steps on the same requests: 16
    requests at the 1K-token context, as two cohorts of 8 (each call one
    forward over 8 drafting and 8 verifying requests) and as plain steps of
    16 (two forwards).  Device time by CUDA events over the same number of
    forwards; tokens counted from the emitted counts."""
    from lossless_diffusion_draft_b200 import uno
    cfg = dict(cfg, batch=batch)
    B, K = cfg["B"], max(4, args.steps // 2)
    wl = Workload(cfg, params, batch, cfg["prompt_len"], rank, device, args)
    plain = wl.time_steps(K, 3, world, clocks=False)
    wl.prefill(cfg["prompt_len"])
    half = batch // 2
    a, b = wl.req[:half].clone(), wl.req[half:].clone()
    out = torch.zeros((half, B + 1), dtype=torch.int32, device=device)
    n_new = torch.zeros(half, dtype=torch.int32, device=device)
    n_hist = torch.zeros((2 * K, half), dtype=torch.int32, device=device)
    uno.uno_spec_step_cohorts(wl.ctx, a, None, out, n_new)
    for k in range(4):                                   # warm-up (and graph capture)
        d, v = (b, a) if k % 2 == 0 else (a, b)
        uno.uno_spec_step_cohorts(wl.ctx, d, v, out, n_new)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for k in range(2 * K):                               # 2K forwards, as K plain steps
        d, v = (b, a) if k % 2 == 0 else (a, b)
        uno.uno_spec_step_cohorts(wl.ctx, d, v, out, n_new)
        n_hist[k].copy_(n_new, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    uno.uno_status(wl.ctx)
    ms = e0.elapsed_time(e1)
    tokens = int(n_hist.sum().item())
    wl.close()
    return {"batch": batch, "context": cfg["prompt_len"], "forwards": 2 * K,
            "plain": {"tokens_per_s": rate(plain), "ms_per_forward": plain["ms"] / plain["K"] / 2},
            "cohorts": {"tokens_per_s": tokens / (ms / 1e3), "ms_per_forward": ms / (2 * K)},
            "note": "two cohorts of 8 out of phase (one forward per call) against plain steps of 16 "
                    "(two forwards per step); per request both do one draft and one verify "
                    "forward per iteration"}


def run_tree(args, cfg, params, rank, world, device):
    """The tree sampler at batch 1 and the mean context: one request, k = 1
    (the linear sampler), 2 and 4 drafted chains, each timed over the same
    number of steps from the same state.  The context is made with two
    request slots so that the second slot's pages hold the chains' scratch
    pages."""
    from lossless_diffusion_draft_b200 import synth, uno
    B = cfg["B"]
    K = max(4, args.steps // 2)
    shape = synth.model_shape(cfg)
    shape["dtype"] = cfg["dtype"]
    max_ctx = cfg["prompt_len"] + cfg["gen_tokens"] + B + 1
    ctx = uno.uno_init(shape, params, cfg["lora_rank"], cfg["lora_alpha"], B, 2, max_ctx,
                       cfg["seed"], torch.cuda.current_stream())
    P = cfg["prompt_len"] + cfg["gen_tokens"] // 2 + 1
    prompt = torch.from_numpy(synth.make_prompts(cfg, 1, P, seed=cfg["seed"] + 1000 * rank)).to(device)
    out = torch.zeros((1, B + 1), dtype=torch.int32, device=device)
    n_new = torch.zeros(1, dtype=torch.int32, device=device)
    n_hist = torch.zeros((K, 1), dtype=torch.int32, device=device)
    res = {}
    for k in (1, 2, 4):
        uno.uno_set_tree(ctx, k)
        ids = uno.uno_prefill(ctx, prompt, [P], streams=replica_streams(rank, 1))
        req = torch.tensor(ids, dtype=torch.int32, device=device)
        for _ in range(3):
            uno.uno_spec_step(ctx, req, out, n_new)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(K):
            uno.uno_spec_step(ctx, req, out, n_new)
            n_hist[i].copy_(n_new, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        uno.uno_status(ctx)
        ms = e0.elapsed_time(e1)
        tok = int(n_hist.sum().item())
        res[str(k)] = {"tokens_per_s": tok / (ms / 1e3), "ms_per_step": ms / K,
                       "tokens_per_step": tok / K}
        uno.uno_release(ctx, ids[0])
    ctx.close()
    return {"batch": 1, "context": P - 1, "steps": K, "chains": res,
            "note": "tree sampler with k drafted chains (k = 1: the linear sampler); random-init "
                    "weights, so the drafter's acceptance is low"}


def run_max_batch(args, cfg, params, rank, world, device, pk):
    """The same model at the largest batch whose KV cache (1024 + 8192 tokens
    per request) fits beside the weights, at the run's mean context."""
    cfg = dict(cfg, batch=0)
    B, prompt_len, gen = cfg["B"], cfg["prompt_len"], cfg["gen_tokens"]
    weight_bytes = sum(t.numel() * t.element_size() for t in params.values())
    max_ctx = prompt_len + gen + B + 1
    batch = max_batch_that_fits(cfg, weight_bytes, max_ctx)
    K, W = max(3, args.steps // 2), 3
    start = max(prompt_len, int(prompt_len + gen // 2 - (W + K) * args.est_tokens_per_step / 2))
    wl = Workload(cfg, params, batch, start, rank, device, args)
    head = wl.time_steps(K, W, world)
    _, detail = step_profile(wl.ctx, wl.req, wl.out, torch.zeros(batch, dtype=torch.int32,
                                                                 device=device), 2, cfg)
    e2e = wl.e2e(K, W, world)
    ar = wl.time_steps(K, W, world, ar=True, clocks=False)
    wl.close()
    ms = head["ms"] / head["K"]
    value = head["tokens"] / (head["ms"] / 1e3)
    ar_value = ar["tokens"] / (ar["ms"] / 1e3)
    return {"value": value, "unit": "tokens/s", "batch": batch, "steps": K, "warmup": W,
            "ms_per_step": ms, "tokens_per_step": head["tokens"] / K,
            "tpf": head["tokens"] / K / batch / 2, "context_window": head["ctx_window"],
            "prefill_s": wl.prefill_s,
            "e2e": {"value": e2e["tokens"] / (e2e["ms"] / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                    "ms_per_step": e2e["ms"] / K, "tokens_per_step": e2e["tokens"] / K},
            "ar_only": {"value": ar_value, "unit": "tokens/s", "ms_per_step": ar["ms"] / ar["K"]},
            "psi_spec_over_ar": value / ar_value,
            "roofline": gemm_roofline(detail, cfg, pk), "clocks": head["clocks"],
            "kernel_detail": detail[:8]}


def spec_verify_micro(args, device, pk, n_req=None):
    """spec_verify on the microbenchmark workload: fp32 p, q [4096 = 256 x 16,
    151936] (p ~ N(0, 3), q = p + N(0, 0.5)), drafts drawn from q, Philox
    seed 7.  Algorithmic bytes: both logit tensors read once."""
    from lossless_diffusion_draft_b200 import synth, uno
    cfg = synth.SPEC_VERIFY_BENCH
    n_req, R, V = n_req or cfg["requests"], cfg["rows_per_request"], cfg["vocab"]
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
    stream = torch.cuda.current_stream()
    call = lambda: uno.uno_spec_verify(p, q, drafts, cfg["seed"], streams, pos0, out, n_out, ws)
    # about half a second of calls, so the clock sampler sees several samples
    K = max(args.steps, 500)
    for _ in range(max(args.warmup, 3)):
        call()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        ev0.record(stream)
        for _ in range(K):
            call()
        ev1.record(stream)
        torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1) / K
    nbytes = 2 * n_req * R * V * 4
    gbs = nbytes / (ms / 1e3) / 1e9
    a = n_out.float().mean().item()
    del p, q
    torch.cuda.empty_cache()
    return {"metric": f"spec_verify [{n_req * R} x {V}] fp32 p and q", "value": n_req * R / (ms / 1e3),
            "unit": "rows/s", "ms_per_call": ms, "calls": K, "mean_accepted": a,
            "l2": "inputs (4.98 GB) larger than L2",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": None,
                         "algorithmic_bytes_per_call": nbytes, "peak_source": pk["source"]},
            "clocks": clk.summary()}


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


def step_bytes(cfg, batch, ctx_window, kv_per_token=None):
    """Algorithmic HBM bytes of one iteration: base weights once per pass (the
    embedding table is only gathered), the adapters once (draft pass), each
    request's KV at the window's mean context once per pass in the model's
    precision (kv_per_token overrides: the layout's bytes), and the fp32
    logits written and read once."""
    esz = 2 if cfg["dtype"] == "bf16" else 4
    from lossless_diffusion_draft_b200 import synth
    base = lora = 0
    for name, shp, kind in synth.param_list(cfg):
        n = int(np.prod(shp)) * esz
        if kind in ("lora_a", "lora_b"):
            lora += n
        elif name != "embed":
            base += n
    ctx = sum(ctx_window) / 2
    kv = ctx * (kv_per_token or kv_bytes_algorithmic(cfg)) * 2 * batch
    logits = (2 * cfg["B"] + 1) * cfg["vocab"] * 4 * 2 * batch
    return 2 * base + lora + kv + logits


def reference_arm(args, rank, cfg, metric):
    """The CPU oracle, timed as it stands on the host cores: each step is one
    bounded sample of the workload's iteration (see OracleSample)."""
    if rank != 0:
        return
    ctx_len = cfg["prompt_len"] + cfg["gen_tokens"] // 2
    sample = OracleSample(cfg, ctx_len)
    times, toks = [], []
    for i in range(args.warmup + args.steps):
        t, n = sample.step(i)
        if i >= args.warmup:
            times.append(t)
            toks.append(n)
    step_s = sum(times) / len(times)
    tpi = sum(toks) / len(toks)
    batch = cfg["batch"] or 1
    value = tpi * batch / step_s
    desc = sample.describe(len(times))
    line = {"impl": "reference", "metric": metric, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "batch": cfg["batch"], "B": cfg["B"],
                       "context": ctx_len},
            "tokens_per_step": tpi * batch,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_cores(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def rate(t):
    return t["tokens"] / (t["ms"] / 1e3)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
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
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (profiler captures of a max-batch step on "
                         "fewer layers; the line's config records it)")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the layer count (small cases for profiler captures; the "
                         "line's config records it)")
    ap.add_argument("--est-tokens-per-step", type=float, default=2.6)
    ap.add_argument("--headline-only", action="store_true",
                    help="the batch-1 headline alone (no context sweep, fixed-accept run, "
                         "max-batch line or spec_verify microbenchmark)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-range", action="store_true",
                    help="bracket the headline's timed steps with cudaProfilerStart/Stop, for "
                         "ncu --profile-from-start off")
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
        reference_arm(args, rank, cfg, metric)
        return

    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    from lossless_diffusion_draft_b200 import build
    build.build()

    res = run_uno(args, rank, world, device)
    cfg, pk, head = res["cfg"], res["pk"], res["head"]
    K = head["K"]
    ms_max = reduce_max(head["ms"], world, device)
    tokens_all = reduce_sum(head["tokens"], world, device)
    e2e_ms = reduce_max(res["e2e"]["ms"], world, device)
    e2e_tokens = reduce_sum(res["e2e"]["tokens"], world, device)
    value = tokens_all / (ms_max / 1e3)
    per_step_ms = ms_max / K
    batch = res["batch"]
    sb = step_bytes(cfg, batch, head["ctx_window"])
    step_roof = {"algorithmic_bytes_per_step": sb, "achieved_GBps": sb / (per_step_ms / 1e3) / 1e9,
                 "frac_of_hbm_peak": sb / (per_step_ms / 1e3) / 1e9 / pk["hbm_gbs"],
                 "peak_source": pk["source"],
                 "layout_bytes_per_step": step_bytes(cfg, batch, head["ctx_window"],
                                                     kv_bytes_per_token(cfg)),
                 "note": "algorithmic bytes count the KV cache in the model's precision (bf16 K and V); "
                         "layout_bytes_per_step counts the three fp16 planes the kernels read"}
    kp = res["kprof"]
    g_launch, g_ms, g_bytes = kp["gemm"]
    roofline = gemm_roofline(res["detail"], cfg, pk) or {}
    if g_ms > 0:
        roofline["all_gemm_launches"] = {"achieved_GBps": g_bytes / (g_ms / 1e3) / 1e9,
                                         "launches": g_launch,
                                         "avg_launch_us": g_ms * 1e3 / max(1, g_launch)}
    tps = head["tokens"] / K / batch
    line = {
        "metric": metric, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": per_step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg["dtype"],
        "data": "synthetic (random-init weights, uniform-random prompt tokens)",
        "config": {"workload": args.workload, "n_layers": cfg["n_layers"],
                   "batch": batch, "B": cfg["B"], "pdl": not args.no_pdl,
                   "fused": res["fused"], "graphs": not args.no_graphs,
                   "prompt_len": cfg["prompt_len"], "gen_tokens": cfg["gen_tokens"],
                   "context_window": head["ctx_window"], "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (15+ GB of weights streamed per pass)"},
        "tokens_per_step": tokens_all / K,
        "step_latency_ms": {"median": statistics.median(head["step_ms"]),
                            "min": min(head["step_ms"]), "max": max(head["step_ms"])},
        "mean_accepted_a": tps - 1,
        "tpf": tps / 2,
        "ar_only": {"value": rate(res["ar"]), "unit": "tokens/s",
                    "ms_per_step": res["ar"]["ms"] / res["ar"]["K"],
                    "note": "uno_ar_step on the same requests and kernels, one token per request"},
        "roofline": roofline, "step_roofline": step_roof,
        "kernel_breakdown": {k: {"launches": v[0], "ms_per_step": v[1] / K} for k, v in kp.items()},
        "e2e": {"value": e2e_tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": res["e2e"]["h2d"], "d2h_bytes_per_step": res["e2e"]["d2h"],
                "ms_per_step": e2e_ms / K, "tokens_per_step": e2e_tokens / K},
        "gpu_launches": head["launches"], "clocks": head["clocks"],
        "kernel_detail": res["detail"][:24],
        "prefill_s": res["prefill_s"],
    }
    if "contexts" in res:
        pts = sorted(res["contexts"].items())
        by_ctx = {}
        for c0, t in pts:
            by_ctx[str(c0)] = {"ms_per_step": t["ms"] / t["K"], "tokens_per_step": t["tokens"] / t["K"],
                               "tokens_per_s": rate(t), "context_window": t["ctx_window"],
                               "frac_of_hbm_peak": step_bytes(cfg, batch, t["ctx_window"]) /
                               (t["ms"] / t["K"] / 1e3) / 1e9 / pk["hbm_gbs"]}
        lat = [t["ms"] / t["K"] for _, t in pts]
        tok = sum(t["tokens"] for _, t in pts) / sum(t["K"] for _, t in pts)
        mean_lat = (lat[0] + 4 * lat[1] + lat[2]) / 6          # Simpson over 1K .. 9K
        line["contexts"] = {
            "steps_per_point": K, "points": by_ctx,
            "whole_run_estimate": {
                "tokens_per_s": tok / (mean_lat / 1e3), "mean_ms_per_step": mean_lat,
                "tokens_per_step": tok,
                "note": "the 1K-in / 8K-out run: step latency averaged over the context range by "
                        "Simpson's rule on the three measured points, at the tokens per step "
                        "measured there"}}
        head_lat = per_step_ms
        line["tpf_projection"] = {
            "tokens_per_s": 2 * 2.25 / (head_lat / 1e3), "tpf": 2.25,
            "note": "projection, not a measurement: the measured iteration latency at the mean "
                    "context times the pages' tokens per forward for the Qwen3-8B adapter (2.25), "
                    "as the pages convert decode steps to tokens by TPF"}
        fa = res["fixed_accept"]
        line["fixed_accept"] = {
            "a": fa["a"], "tokens_per_s": rate(fa), "ms_per_step": fa["ms"] / fa["K"],
            "tokens_per_step": fa["tokens"] / fa["K"], "tpf": fa["tokens"] / fa["K"] / batch / 2,
            "note": "measured with the uno_debug_set_fixed_accept tap forcing a = 4 accepted "
                    "tokens (TPF 2.5, the pages' trained-adapter range); not a parity run"}
    if "cohorts" in res:
        line["cohorts"] = res["cohorts"]
    if "tree" in res:
        line["tree"] = res["tree"]
    if "max_batch" in res:
        line["max_batch"] = res["max_batch"]
    if "spec_verify_micro" in res:
        line["spec_verify_micro"] = res["spec_verify_micro"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ctx_len = sum(head["ctx_window"]) // 2
        v, step_s, tpi, desc = oracle_baseline(cfg, ctx_len)
        line["cpu_baseline"] = {"value": v * batch, "unit": "tokens/s", "cores": cpu_cores(),
                                "kind": "oracle", "sample": desc, "s_per_iteration": step_s,
                                "tokens_per_iteration": tpi}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
