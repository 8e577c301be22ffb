"""Tree sampler on the GPU against the oracle (GPU).

Per iteration, on the same state (teacher-forced):
  1. draft logits and every chain's verify logits against the oracle's
     forwards of the same chains (fp32 1e-4, bf16 2e-2);
  2. every drafted chain token against the oracle's inverse-CDF draw on the
     GPU's logits with the chain's Philox lane (near-ties traced);
  3. the walk: the oracle's tree_walk on the GPU's logits and uniforms must
     emit the GPU's tokens; a difference is accepted only as a near-tie, i.e.
     when moving one uniform by a relative 1e-5 reproduces the GPU's result;
  4. fp32: the emitted tokens against the oracle's own tree iteration;
  5. the committed KV cache (the accepted chain's keys copied into the
     request's slot) position by position at the end.
"""

import numpy as np
import pytest
import torch

from lossless_diffusion_draft_b200 import synth, uno
from oracle import model as om
from oracle import psispec as ops
from oracle.philox import KIND_DRAFT, KIND_FIRST, uniform

import parity
from test_gpu_model import _kv_check

pytestmark = pytest.mark.gpu

PERTURB = 1e-5


def _walk_matches(p_rows, q_rows, chains, c, ufn, want):
    path, last, _ = ops.tree_walk(p_rows, q_rows, chains, c, ufn)
    if path + [last] == want:
        return True, 0
    keys = []
    def rec(kind, pos, lane):
        keys.append((kind, pos, lane))
        return ufn(kind, pos, lane)
    ops.tree_walk(p_rows, q_rows, chains, c, rec)
    for key in keys:
        for f in (1 - PERTURB, 1 + PERTURB):
            def pert(kind, pos, lane, key=key, f=f):
                u = ufn(kind, pos, lane)
                return min(u * f, 1 - 2.0 ** -24) if (kind, pos, lane) == key else u
            p2, l2, _ = ops.tree_walk(p_rows, q_rows, chains, c, pert)
            if p2 + [l2] == want:
                return False, 1
    raise AssertionError(f"walk differs beyond a near-tie: GPU {want}, oracle {path + [last]}")


def _tree_run(name, n_req, prompt_len, n_steps, k, logit_tol, end_to_end, **over):
    cfg = dict(synth.CONFIGS[name], **over)
    shape = synth.model_shape(cfg)
    shape["dtype"] = cfg["dtype"]
    params_cpu = synth.make_params(cfg, "cpu")
    params = {k_: v.cuda() for k_, v in params_cpu.items()}
    # a spare request slot: its pages hold the chains' scratch pages
    ctx = uno.uno_init(shape, params, cfg["lora_rank"], cfg["lora_alpha"], cfg["B"], n_req + 1, 1400,
                       cfg["seed"], torch.cuda.current_stream())
    uno.uno_set_tree(ctx, k)
    prompts = synth.make_prompts(cfg, n_req, prompt_len)
    ids = uno.uno_prefill(ctx, torch.from_numpy(prompts).cuda(), [prompt_len] * n_req,
                          streams=list(range(n_req)))
    model = om.Model(synth.model_shape(cfg), {k_: v.double().numpy() for k_, v in params_cpu.items()})
    states = [ops.prefill(model, [int(t) for t in prompts[i]], stream=i) for i in range(n_req)]
    B, V, seed = cfg["B"], cfg["vocab"], cfg["seed"]
    req = torch.tensor(ids, dtype=torch.int32, device="cuda")
    out = torch.zeros((n_req, B + 1), dtype=torch.int32, device="cuda")
    n_new = torch.zeros(n_req, dtype=torch.int32, device="cuda")
    draws, walks, e2e = parity.Tally(), parity.Tally(), parity.Tally()
    lengths = []
    for step in range(n_steps):
        uno.uno_spec_step(ctx, req, out, n_new)
        uno.uno_status(ctx)
        ld = uno.uno_debug_read(ctx, uno.UNO_DBG_LOGITS_DRAFT, torch.empty((n_req, B + 1, V))).double().numpy()
        lt = uno.uno_debug_read(ctx, uno.UNO_DBG_TREE_LOGITS, torch.empty((n_req, k, B, V))).double().numpy()
        chs = uno.uno_debug_read(ctx, uno.UNO_DBG_TREE_CHAINS,
                                 torch.empty((n_req, k, B), dtype=torch.int32)).numpy()
        o, nn = out.cpu().numpy(), n_new.cpu().numpy()
        for i in range(n_req):
            st = states[i]
            c = st.c
            chains = [[int(t) for t in chs[i, j]] for j in range(k)]
            emitted = [int(t) for t in o[i, : nn[i]]]
            assert 2 <= nn[i] <= B + 1
            lengths.append(len(emitted))
            new_st, res = ops.tree_spec_step(model, st, B, k, seed, chains=chains)
            assert np.max(np.abs(ld[i] - res.logits_draft)) <= logit_tol
            for j in range(k):
                assert np.max(np.abs(lt[i, j] - res.logits_verify[j])) <= logit_tol, (step, i, j)
            # 2. the chains' draws on the GPU's logits
            u = lambda kind, pos, lane=0: float(uniform(seed, st.stream, pos, kind, lane))
            parity.check_sample(ld[i][0], u(KIND_FIRST, c + 1), chains[0][0], draws, "x1")
            for j in range(k):
                assert chains[j][0] == chains[0][0]
                for d in range(2, B + 1):
                    parity.check_sample(ld[i][d], u(KIND_DRAFT, c + d, j), chains[j][d - 1], draws,
                                        f"chain {j} pos {d}")
            # 3. the walk on the GPU's logits
            q_rows = {d: ld[i][d] for d in range(2, B + 1)}
            p_rows = [lt[i, j] for j in range(k)]
            same, near = _walk_matches(p_rows, q_rows, chains, c, u, emitted)
            walks.add(same, (step, i, emitted))
            if end_to_end:
                _, own = ops.tree_spec_step(model, st, B, k, seed)
                e2e.add(own.emitted == emitted, (step, i, own.emitted, emitted))
            states[i] = new_st if res.emitted == emitted else \
                ops.prefill(model, st.tokens + emitted, stream=st.stream)
            c_gpu, pend = uno.uno_request_state(ctx, ids[i])
            assert c_gpu == states[i].c and pend == states[i].pending, (step, i)
    for i in range(n_req):
        _kv_check(ctx, cfg, model, states[i], ids[i], logit_tol)
    ctx.close()
    return draws, walks, e2e, lengths


def test_tiny_fp32_tree_k3():
    draws, walks, e2e, lengths = _tree_run("tiny", 2, 24, 10, 3, 1e-4, True)
    assert draws.mismatches <= parity.near_tie_budget(draws.positions), draws.notes
    assert walks.mismatches <= max(1, walks.positions // 100), walks.notes
    assert e2e.mismatches <= draws.mismatches + walks.mismatches, e2e.notes
    assert max(lengths) >= 3                      # some block went past its first test


def test_small_bf16_tree_k2():
    draws, walks, _, _ = _tree_run("small", 2, 24, 3, 2, 2e-2, False, n_layers=2)
    assert draws.mismatches <= parity.near_tie_budget(draws.positions), draws.notes
    assert walks.mismatches <= max(1, walks.positions // 100), walks.notes


def test_tree_setting_capacity_and_switch():
    cfg = dict(synth.CONFIGS["tiny"])
    shape = synth.model_shape(cfg)
    shape["dtype"] = "f32"
    params = {k: v.cuda() for k, v in synth.make_params(cfg, "cpu").items()}
    # one request slot of 7 pages; the tree with 2 chains takes 4 of them
    ctx = uno.uno_init(shape, params, cfg["lora_rank"], cfg["lora_alpha"], cfg["B"], 1, 400, 0,
                       torch.cuda.current_stream())
    ids = uno.uno_prefill(ctx, torch.from_numpy(synth.make_prompts(cfg, 1, 10)).cuda(), [10])
    with pytest.raises(uno.UnoError) as e:          # every page is the request's
        uno.uno_set_tree(ctx, 2)
    assert e.value.code == uno.UNO_ERR_CAPACITY
    with pytest.raises(uno.UnoError):
        uno.uno_set_tree(ctx, 5)
    uno.uno_release(ctx, ids[0])
    uno.uno_set_tree(ctx, 2)
    with pytest.raises(uno.UnoError) as e:          # the chains' pages are taken now
        uno.uno_prefill(ctx, torch.from_numpy(synth.make_prompts(cfg, 1, 10)).cuda(), [10])
    assert e.value.code == uno.UNO_ERR_CAPACITY
    uno.uno_set_tree(ctx, 1)                        # gives them back
    uno.uno_prefill(ctx, torch.from_numpy(synth.make_prompts(cfg, 1, 10)).cuda(), [10])
    ctx.close()
