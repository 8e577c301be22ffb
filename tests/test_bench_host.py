"""Host side of bench.py (CPU): the reference arm's JSON line, rank-0-only
printing, and the multi-rank aggregation over gloo (world size 2)."""

import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _run_bench(args, env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = _run_bench(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0"],
                   {"WORLD_SIZE": "1", "RANK": "0"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["higher_is_better"] is True and d["steps"] == 1 and d["warmup"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_silently():
    r = _run_bench(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0"],
                   {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]


def test_replica_streams_are_disjoint():
    seen = set()
    for rank in range(8):
        s = bench.replica_streams(rank, 80)
        assert len(s) == 80 and not seen.intersection(s)
        seen.update(s)


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dev = torch.device("cpu")
        # per-rank step times and token counts: time is the max, tokens the sum
        ms = bench.reduce_max(10.0 + 5.0 * rank, world, dev)
        tok = bench.reduce_sum(100 + rank, world, dev)
        bench.barrier(world)
        out[rank] = (ms, tok)
    finally:
        dist.destroy_process_group()


def test_aggregation_over_two_gloo_ranks():
    port = 29500 + os.getpid() % 1000
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        assert out[0] == out[1] == (15.0, 201)


def test_single_rank_aggregation_is_identity():
    assert bench.reduce_max(3.5, 1, None) == 3.5
    assert bench.reduce_sum(7, 1, None) == 7


class _FakeNvml:
    """pynvml stand-in: an SM clock that drops under a power cap after the
    third read."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonHwThermalSlowdown = 0x40

    def __init__(self):
        self.reads = 0
        self.shut = False

    def nvmlInit(self):
        pass

    def nvmlShutdown(self):
        self.shut = True

    def nvmlDeviceGetHandleByUUID(self, uuid):
        return ("uuid", uuid)

    def nvmlDeviceGetHandleByIndex(self, i):
        return ("index", i)

    def nvmlDeviceGetClockInfo(self, h, which):
        assert which == self.NVML_CLOCK_SM
        self.reads += 1
        return 1965 if self.reads <= 3 else 1800

    def nvmlDeviceGetMaxClockInfo(self, h, which):
        return 1965

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return 0x1 | (0x4 if self.reads >= 3 else 0)   # idle bit ignored


def test_clock_sampler_reads_nvml_without_touching_settings():
    import time
    nv = _FakeNvml()
    with bench.ClockSampler(0, nvml=nv) as clk:
        time.sleep(0.2)
    s = clk.summary()
    assert s["source"] == "nvml" and s["samples"] >= 5
    assert s["sm_max_mhz"] == 1965 and s["sm_mhz"] == 1800
    assert s["reasons"] == ["sw_power_cap"]
    assert nv.shut
    # the fake has no setter: any call beyond reads would raise AttributeError


def test_clock_sampler_disabled_records_nothing():
    with bench.ClockSampler(0, enabled=False, nvml=_FakeNvml()) as clk:
        pass
    assert clk.summary() is None


def test_step_bytes_match_the_qwen8b_budget():
    """The per-step roofline's algorithmic bytes for the Qwen3-8B shape at
    batch 1 and context 5120, from the shape's own counts: 6,945,767,424
    body + 622,329,856 LM-head parameters (bf16) per pass, 349,175,808 LoRA
    parameters once, the RMSNorm gains ((2 x 36 + 1) x 4096) per pass,
    147,456 KV bytes per token per pass (36 layers x K and V x 8 heads x 128
    x 2 bytes), fp32 logits of 33 rows written and read."""
    from lossless_diffusion_draft_b200 import synth
    cfg = dict(synth.CONFIGS["qwen8b"])
    assert bench.kv_bytes_algorithmic(cfg) == 147_456
    norms = (2 * 36 + 1) * 4096
    expect = (2 * (6_945_767_424 + 622_329_856 + norms) * 2 + 349_175_808 * 2 + 5120 * 147_456 * 2
              + 33 * 151_936 * 4 * 2)
    assert bench.step_bytes(cfg, 1, [5120, 5120]) == expect
    # the library's three-plane layout reads half as many KV bytes again
    extra = bench.step_bytes(cfg, 1, [5120, 5120], bench.kv_bytes_per_token(cfg)) - expect
    assert extra == 5120 * 147_456 * 2 // 2


def test_gemm_roofline_arithmetic():
    """The dominant GEMM's roofline from per-launch times: the gate|up
    projection of a batch-1 draft pass is HBM-bound (its 203.6 MB over the
    measured copy rate), the max-batch one tensor-bound (2 M N K flops over
    the sustained bf16 rate; the hi/lo inputs double the executed flops)."""
    pk = {"hbm_gbs": 6545.9, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1345.1, "source": "measured"}
    cfg = {"dtype": "bf16"}
    small = [{"cls": "gemm", "m": 17, "n": 24832, "k": 4096, "r": 0, "us_per_call": 40.0,
              "calls_per_step": 36.0, "ms_per_step": 1.44},
             {"cls": "attn", "us_per_call": 15.0, "calls_per_step": 144.0, "ms_per_step": 2.2}]
    r = bench.gemm_roofline(small, cfg, pk)
    b = (24832 * 4096 + 17 * 4096) * 2
    assert r["bound"] == "hbm" and r["algorithmic_bytes"] == b == 203_563_008
    assert abs(r["achieved"] - b / 40e-6 / 1e9) < 1e-6 and abs(r["frac"] - r["achieved"] / 6545.9) < 1e-12
    big = [{"cls": "gemm", "m": 1360, "n": 24576, "k": 4096, "r": 128, "us_per_call": 500.0,
            "calls_per_step": 36.0, "ms_per_step": 18.0}]
    r = bench.gemm_roofline(big, cfg, pk)
    f = 2.0 * 1360 * 24576 * (4096 + 128)
    assert r["bound"] == "tensor" and r["algorithmic_flops"] == f
    assert abs(r["achieved"] - f / 500e-6 / 1e12) < 1e-9 and r["peak"] == 1345.1
    assert abs(r["executed_TFLOPs"] - 2 * r["achieved"]) < 1e-9
