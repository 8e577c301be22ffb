"""The Qwen3-8B-shaped workload (36 layers, d 4096, GQA 32/8 x 128, FFN
12288, vocab 151936, LoRA rank 128 / alpha 256, B = 16, batch 1, 1024-token
prompt) through the C ABI vs the oracle for its first four Psi-Spec
iterations (GPU).

The random-init weights are made on the GPU (the benchmark's weights); the
float64 oracle reads them one tensor at a time, so the host never holds the
model in float64.  Per iteration: draft and verify logits within 2e-2 of the
oracle, draft_sample and spec_verify decisions on the GPU's logits with the
same uniforms (near-ties traced), teacher forcing on the emitted tokens, and
the KV cache of every layer after the last commit.
"""

import collections.abc

import numpy as np
import pytest
import torch

from lossless_diffusion_draft_b200 import synth, uno
from oracle import model as om
from oracle import psispec as ops

import parity

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


class DeviceParams(collections.abc.Mapping):
    """The device weights as host arrays, copied on each access."""

    def __init__(self, params):
        self._p = params

    def __getitem__(self, name):
        return self._p[name].float().cpu().numpy()

    def __iter__(self):
        return iter(self._p)

    def __len__(self):
        return len(self._p)


def _run(n_layers=None, prompt_len=None, n_steps=4, fused=True):
    cfg = dict(synth.CONFIGS["qwen8b"])
    if n_layers:
        cfg["n_layers"] = n_layers
    shape = synth.model_shape(cfg)
    shape["dtype"] = cfg["dtype"]
    params = synth.make_params(cfg, "cuda")
    B, V, seed = cfg["B"], cfg["vocab"], cfg["seed"]
    P = prompt_len or cfg["prompt_len"]
    ctx = uno.uno_init(shape, params, cfg["lora_rank"], cfg["lora_alpha"], B, 1, P + 4 * (B + 1) + 8,
                       seed, torch.cuda.current_stream())
    if not fused:
        uno.uno_set_fused(ctx, False)
    prompt = synth.make_prompts(cfg, 1, P)
    ids = uno.uno_prefill(ctx, torch.from_numpy(prompt).cuda(), [P], streams=[0])
    model = om.Model(synth.model_shape(cfg), DeviceParams(params))
    st = ops.prefill(model, [int(t) for t in prompt[0]], stream=0)

    req = torch.tensor(ids, dtype=torch.int32, device="cuda")
    out = torch.zeros((1, B + 1), dtype=torch.int32, device="cuda")
    n_new = torch.zeros(1, dtype=torch.int32, device="cuda")
    tally = parity.Tally()
    worst = 0.0
    for step in range(n_steps):
        uno.uno_spec_step(ctx, req, out, n_new)
        uno.uno_status(ctx)
        ld = uno.uno_debug_read(ctx, uno.UNO_DBG_LOGITS_DRAFT, torch.empty((1, B + 1, V)))
        lv = uno.uno_debug_read(ctx, uno.UNO_DBG_LOGITS_VERIFY, torch.empty((1, B, V)))
        dr = uno.uno_debug_read(ctx, uno.UNO_DBG_DRAFTS, torch.empty((1, B), dtype=torch.int32))
        drafts = [int(t) for t in dr[0]]
        emitted = [int(t) for t in out[0, : int(n_new[0])].cpu()]
        assert 2 <= len(emitted) <= B + 1
        new_st, res = ops.spec_step(model, st, B, seed, drafts=drafts)
        err_d = float(np.max(np.abs(ld[0].double().numpy() - res.logits_draft)))
        err_v = float(np.max(np.abs(lv[0].double().numpy() - res.logits_verify)))
        worst = max(worst, err_d, err_v)
        print(f"step {step}: draft logits max err {err_d:.3e}, verify {err_v:.3e}")
        assert err_d <= 2e-2 and err_v <= 2e-2, (step, err_d, err_v)
        parity.check_step_sampling(ld[0].double().numpy(), lv[0].double().numpy(), drafts, emitted,
                                   st.c, B, seed, st.stream, tally, f"step {step}")
        st = new_st if res.emitted == emitted else ops.prefill(model, st.tokens + emitted, stream=0)
        c_gpu, pend_gpu = uno.uno_request_state(ctx, ids[0])
        assert c_gpu == st.c and pend_gpu == st.pending
    assert tally.mismatches <= parity.near_tie_budget(tally.positions), tally.notes
    # the cache after the last commit, every layer
    c = st.c
    Hkv, hd = cfg["n_kv_heads"], cfg["head_dim"]
    for l in range(cfg["n_layers"]):
        k = torch.empty((c, Hkv, hd), dtype=torch.float16)   # fp16 cache
        v = torch.empty((c, Hkv, hd), dtype=torch.float16)
        uno.uno_debug_kv(ctx, ids[0], l, 0, c, k, v)
        np.testing.assert_allclose(k.double().numpy(), st.cache.k[l], atol=2e-2, rtol=0)
        np.testing.assert_allclose(v.double().numpy(), st.cache.v[l], atol=2e-2, rtol=0)
    ctx.close()
    print(f"worst logit error {worst:.3e}")


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "unfused"])
def test_qwen8b_shape_two_layers(fused):
    """The Qwen3-8B widths (d 4096: 32 norm tiles per row, hd 128, FFN 12288,
    vocab 151936) on two layers and a 200-token prompt: a quick check of every
    width-dependent index, through both layer pipelines."""
    _run(n_layers=2, prompt_len=200, n_steps=2, fused=fused)


def test_qwen8b_first_four_steps():
    """The full 36-layer model, 1024-token prompt, first four iterations."""
    _run()


@pytest.mark.parametrize("n_req,checked", [(8, (0, 3, 7)), (80, (0, 41, 79))],
                         ids=["8_requests", "80_requests"])
def test_qwen8b_two_layers_many_requests(n_req, checked):
    """Several requests at once on the Qwen3-8B widths (two layers, 80-token
    prompts).  Eight requests: 136 draft rows take the tokens-in-M GEMM form,
    whose last LM-head weight tile is cut by the 151936-token vocabulary
    (593.5 tiles of 256).  Eighty requests: the largest batch's launch
    configuration (1360 draft / 1280 verify rows, m-tile groups, 640
    unsplit attention groups, more than the SMs).  The checked requests'
    draft and verify logits within 2e-2 of the oracle's on the GPU's drafts,
    and their request states after the step."""
    cfg = dict(synth.CONFIGS["qwen8b"], n_layers=2)
    shape = synth.model_shape(cfg)
    shape["dtype"] = cfg["dtype"]
    params = synth.make_params(cfg, "cuda")
    B, V, seed = cfg["B"], cfg["vocab"], cfg["seed"]
    P = 80
    ctx = uno.uno_init(shape, params, cfg["lora_rank"], cfg["lora_alpha"], B, n_req, P + 2 * (B + 1),
                       seed, torch.cuda.current_stream())
    prompts = synth.make_prompts(cfg, n_req, P)
    ids = uno.uno_prefill(ctx, torch.from_numpy(prompts).cuda(), [P] * n_req,
                          streams=list(range(n_req)))
    # two layers: the weights fit the host as fp32 (exact for bf16); the
    # oracle's products upcast them to fp64
    model = om.Model(synth.model_shape(cfg), {k: v.float().cpu().numpy() for k, v in params.items()})
    req = torch.tensor(ids, dtype=torch.int32, device="cuda")
    out = torch.zeros((n_req, B + 1), dtype=torch.int32, device="cuda")
    n_new = torch.zeros(n_req, dtype=torch.int32, device="cuda")
    uno.uno_spec_step(ctx, req, out, n_new)
    uno.uno_status(ctx)
    ld = uno.uno_debug_read(ctx, uno.UNO_DBG_LOGITS_DRAFT, torch.empty((n_req, B + 1, V)))
    lv = uno.uno_debug_read(ctx, uno.UNO_DBG_LOGITS_VERIFY, torch.empty((n_req, B, V)))
    dr = uno.uno_debug_read(ctx, uno.UNO_DBG_DRAFTS, torch.empty((n_req, B), dtype=torch.int32))
    nn = n_new.cpu().numpy()
    # the first request, one in the middle and the last, whose rows end the
    # last token tile
    for i in checked:
        st = ops.prefill(model, [int(t) for t in prompts[i]], stream=i)
        _, res = ops.spec_step(model, st, B, seed, drafts=[int(t) for t in dr[i]])
        err_d = float(np.max(np.abs(ld[i].double().numpy() - res.logits_draft)))
        err_v = float(np.max(np.abs(lv[i].double().numpy() - res.logits_verify)))
        assert err_d <= 2e-2 and err_v <= 2e-2, (i, err_d, err_v)
        c_gpu, _ = uno.uno_request_state(ctx, ids[i])
        assert c_gpu == st.c + int(nn[i])
    ctx.close()
