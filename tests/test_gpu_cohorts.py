"""Cohort-interleaved steps (GPU): one forward carries one cohort's draft
rows and another cohort's verify rows, so each weight tile serves both paths
(the gated LoRA computes both in one forward: Walkthrough §Diffusion
Distillation：一步蒸馏 + 块级扩散).  Per request nothing changes - its draft,
its verification and its uniforms are those of a plain Psi-Spec iteration -
so every verified request is checked against the oracle's spec_step on the
same state: logits, sampling decisions (near-ties traced), the emitted
tokens (fp32: the oracle's own iteration), and the KV cache at the end.
"""

import numpy as np
import pytest
import torch

from lossless_diffusion_draft_b200 import synth, uno
from oracle import psispec as ops

import parity
from test_gpu_model import _kv_check, _setup

pytestmark = pytest.mark.gpu


def _cohort_run(name, n_req, prompt_len, n_calls, logit_tol, end_to_end, **over):
    cfg, ctx, ids, model, states = _setup(name, n_req, prompt_len,
                                          prompt_len + (n_calls + 2) * 10, **over)
    B, V, seed, mb = cfg["B"], cfg["vocab"], cfg["seed"], n_req
    half = n_req // 2
    cohorts = [torch.tensor(ids[:half], dtype=torch.int32, device="cuda"),
               torch.tensor(ids[half:], dtype=torch.int32, device="cuda")]
    members = [list(range(half)), list(range(half, n_req))]
    out = torch.zeros((n_req, B + 1), dtype=torch.int32, device="cuda")
    n_new = torch.zeros(n_req, dtype=torch.int32, device="cuda")
    tally, e2e = parity.Tally(), parity.Tally()
    verified = 0
    for call in range(n_calls):
        d = call % 2                     # cohort d drafts, the other verifies (none on call 0)
        v_ids = cohorts[1 - d] if call > 0 else None
        nv = 0 if v_ids is None else v_ids.numel()
        uno.uno_spec_step_cohorts(ctx, cohorts[d], v_ids, out[:max(nv, 1)], n_new[:max(nv, 1)])
        uno.uno_status(ctx)
        if v_ids is None:
            continue
        logits = uno.uno_debug_read(ctx, uno.UNO_DBG_COHORT_LOGITS,
                                    torch.empty((2 * mb, B + 1, V))).double().numpy()
        drafts_all = uno.uno_debug_read(ctx, uno.UNO_DBG_COHORT_DRAFTS,
                                        torch.empty((mb, B), dtype=torch.int32)).numpy()
        o, nn = out.cpu().numpy(), n_new.cpu().numpy()
        for k, i in enumerate(members[1 - d]):
            st = states[i]
            slot = ids[i]
            ld = logits[slot]                  # its draft rows, from the call that drafted it
            lv = logits[mb + k, :B]            # its verify rows, from this call
            drafts = [int(t) for t in drafts_all[slot]]
            emitted = [int(t) for t in o[k, : nn[k]]]
            assert 2 <= nn[k] <= B + 1
            new_st, res = ops.spec_step(model, st, B, seed, drafts=drafts)
            err_d = float(np.max(np.abs(ld - res.logits_draft)))
            err_v = float(np.max(np.abs(lv - res.logits_verify)))
            assert err_d <= logit_tol and err_v <= logit_tol, (call, i, err_d, err_v)
            parity.check_step_sampling(ld, lv, drafts, emitted, st.c, B, seed, st.stream, tally,
                                       f"call {call} req {i}")
            if end_to_end:
                _, own = ops.spec_step(model, st, B, seed)
                e2e.add(own.emitted == emitted, (call, i, own.emitted, emitted))
            states[i] = new_st if res.emitted == emitted else \
                ops.prefill(model, st.tokens + emitted, stream=st.stream)
            c_gpu, pend = uno.uno_request_state(ctx, slot)
            assert c_gpu == states[i].c and pend == states[i].pending
            verified += 1
    assert verified >= (n_calls - 1) * half
    # the cohort drafted by the last call holds scratch keys past its cache
    # only; its committed cache is checked like the others'
    for i in range(n_req):
        _kv_check(ctx, cfg, model, states[i], ids[i], logit_tol)
    ctx.close()
    return tally, e2e


def test_tiny_fp32_cohorts():
    tally, e2e = _cohort_run("tiny", 4, 32, 9, 1e-4, True)
    assert tally.mismatches <= parity.near_tie_budget(tally.positions), tally.notes
    assert e2e.mismatches <= tally.mismatches, e2e.notes


def test_small_bf16_cohorts():
    """bf16, 6 requests in two cohorts: 54 rows per forward (fused pipeline)."""
    tally, _ = _cohort_run("small", 6, 24, 5, 2e-2, False, n_layers=2)
    assert tally.mismatches <= parity.near_tie_budget(tally.positions), tally.notes


def test_cohort_tokens_equal_plain_steps():
    """fp32 (the SIMT kernels add every row in a fixed order whatever the pass
    holds): each request's token stream from interleaved cohorts equals its
    stream from plain uno_spec_step calls, bit for bit."""
    cfg = dict(synth.CONFIGS["tiny"])
    shape = synth.model_shape(cfg)
    shape["dtype"] = "f32"
    params = {k: v.cuda() for k, v in synth.make_params(cfg, "cpu").items()}
    prompts = torch.from_numpy(synth.make_prompts(cfg, 4, 20)).cuda()
    B = cfg["B"]
    streams = []
    for mode in ("plain", "cohort"):
        ctx = uno.uno_init(shape, params, cfg["lora_rank"], cfg["lora_alpha"], B, 4, 200, cfg["seed"],
                           torch.cuda.current_stream())
        ids = uno.uno_prefill(ctx, prompts, [20] * 4, streams=[0, 1, 2, 3])
        seqs = [[] for _ in range(4)]
        out = torch.zeros((4, B + 1), dtype=torch.int32, device="cuda")
        nn = torch.zeros(4, dtype=torch.int32, device="cuda")
        if mode == "plain":
            req = torch.tensor(ids, dtype=torch.int32, device="cuda")
            for _ in range(5):
                uno.uno_spec_step(ctx, req, out, nn)
                torch.cuda.synchronize()
                for i in range(4):
                    seqs[i] += out[i, : int(nn[i])].tolist()
        else:
            a = torch.tensor(ids[:2], dtype=torch.int32, device="cuda")
            b = torch.tensor(ids[2:], dtype=torch.int32, device="cuda")
            uno.uno_spec_step_cohorts(ctx, a, None, out, nn)
            for call in range(10):
                d, v = (b, a) if call % 2 == 0 else (a, b)
                uno.uno_spec_step_cohorts(ctx, d, v, out, nn)
                torch.cuda.synchronize()
                base = 0 if v is a else 2
                for k in range(2):
                    seqs[base + k] += out[k, : int(nn[k])].tolist()
            uno.uno_spec_step_cohorts(ctx, None, a, out, nn)   # a's last draft (call 9's)
            torch.cuda.synchronize()
            for k in range(2):
                seqs[k] += out[k, : int(nn[k])].tolist()
        uno.uno_status(ctx)
        ctx.close()
        streams.append(seqs)
    for i in range(4):
        n = min(len(streams[0][i]), len(streams[1][i]))
        assert n > 10
        assert streams[0][i][:n] == streams[1][i][:n], i


def test_cohort_phase_check():
    """Verifying a request that was not drafted raises the device flag."""
    cfg = dict(synth.CONFIGS["tiny"])
    shape = synth.model_shape(cfg)
    shape["dtype"] = "f32"
    params = {k: v.cuda() for k, v in synth.make_params(cfg, "cpu").items()}
    ctx = uno.uno_init(shape, params, cfg["lora_rank"], cfg["lora_alpha"], cfg["B"], 2, 100,
                       cfg["seed"], torch.cuda.current_stream())
    ids = uno.uno_prefill(ctx, torch.from_numpy(synth.make_prompts(cfg, 2, 10)).cuda(), [10, 10])
    out = torch.zeros((2, cfg["B"] + 1), dtype=torch.int32, device="cuda")
    nn = torch.zeros(2, dtype=torch.int32, device="cuda")
    v = torch.tensor(ids[:1], dtype=torch.int32, device="cuda")
    uno.uno_spec_step_cohorts(ctx, None, v, out, nn)
    with pytest.raises(uno.UnoError) as e:
        uno.uno_status(ctx)
    assert e.value.code == uno.UNO_ERR_DEVICE_CHECK
    ctx.close()
