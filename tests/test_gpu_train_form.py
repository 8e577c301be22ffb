"""The training-form forward [x, z] with the general block-causal mask (GPU).

Walkthrough §Diffusion Distillation：一步蒸馏 + 块级扩散: the input is the
clean sequence x followed by its noised copy z (context 2L); the clean part
is causal, each noised block is causal inside itself and sees every clean
token before the block; the adapter is gated off on x and on on z, so one
forward gives the teacher (AR) logits of x and the student (diffusion)
logits of z.  Checked three ways:
  1. logits of every row against the oracle's forward with its explicit
     mask matrix (the bf16 fused and unfused pipelines, the fp32 kernels);
  2. the GPU's mask itself against the hand-written fixture
     tests/golden/block_causal_mask_x4_z4_B2.txt: in a one-layer model row
     i's logits depend on token j exactly when i may attend to j, so
     perturbing token j must change exactly the fixture's column j (the
     other rows bit-identical);
  3. capacity errors and the slots being free again afterwards.
"""

import os

import numpy as np
import pytest
import torch

from lossless_diffusion_draft_b200 import synth, uno
from oracle import model as om

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _ctx(name, max_batch, max_ctx, **over):
    cfg = dict(synth.CONFIGS[name], **over)
    shape = synth.model_shape(cfg)
    shape["dtype"] = cfg["dtype"]
    params_cpu = synth.make_params(cfg, "cpu")
    params = {k: v.cuda() for k, v in params_cpu.items()}
    ctx = uno.uno_init(shape, params, cfg["lora_rank"], cfg["lora_alpha"], cfg["B"], max_batch,
                       max_ctx, cfg["seed"], torch.cuda.current_stream())
    return cfg, ctx, params_cpu


def _oracle_train_logits(model, cfg, x, z):
    L, B = len(x), cfg["B"]
    pos = np.concatenate([np.arange(L), np.arange(L)])
    noised = np.array([False] * L + [True] * L)
    block = np.concatenate([np.zeros(L, int), (np.arange(L) // B) * B])
    gates = np.concatenate([np.zeros(L), np.ones(L)])
    logits, _, _ = model.forward(om.KVCache(model.shape), list(x) + list(z), pos, gates, noised, block)
    return logits


def _tokens(cfg, n_seq, L, seed, z_mask=True):
    rng = np.random.default_rng(seed)
    V = cfg["vocab"]
    x = rng.integers(0, V - 1, (n_seq, L))
    z = np.full((n_seq, L), V - 1) if z_mask else rng.integers(0, V, (n_seq, L))
    return np.concatenate([x, z], axis=1).astype(np.int32)


def _check(name, n_seq, L, tol, seed, z_mask=True, **over):
    cfg, ctx, params_cpu = _ctx(name, 2 * n_seq + 1, L + 8, **over)
    toks = _tokens(cfg, n_seq, L, seed, z_mask)
    V = cfg["vocab"]
    out = torch.full((n_seq, 2 * L, V), float("nan"), device="cuda")
    uno.uno_train_forward(ctx, torch.from_numpy(toks).cuda(), out)
    uno.uno_status(ctx)
    got = out.cpu().double().numpy()
    model = om.Model(synth.model_shape(cfg), {k: v.double().numpy() for k, v in params_cpu.items()})
    worst = 0.0
    for s in range(n_seq):
        want = _oracle_train_logits(model, cfg, toks[s, :L], toks[s, L:])
        err = float(np.max(np.abs(got[s] - want)))
        worst = max(worst, err)
        assert err <= tol, (s, err)
    ctx.close()
    return worst


def test_train_form_bf16_fused():
    """Small bf16 model (2 layers), 2 sequences of L = 24 with B = 8 (three
    noised blocks each): 96 rows, the fused pipeline."""
    _check("small", 2, 24, 2e-2, 1, n_layers=2)


def test_train_form_bf16_unfused_random_noise():
    """160 rows (past the fused pipeline's 128): the unfused kernels; z holds
    random tokens instead of MASK, and L = 80 is not a multiple of the
    attention's query tile."""
    _check("small", 1, 80, 2e-2, 2, z_mask=False, n_layers=2)


def test_train_form_fp32_simt():
    """The tiny fp32 model on the SIMT attention: L = 18, B = 4 (the last
    block is ragged), logits within 1e-4."""
    _check("tiny", 2, 18, 1e-4, 3)


def test_gpu_mask_equals_fixture():
    """L = 4, B = 2 on a one-layer bf16 model: perturbing token j changes
    exactly the rows the fixture lets attend to key j."""
    want = np.loadtxt(os.path.join(GOLDEN, "block_causal_mask_x4_z4_B2.txt"), dtype=int).astype(bool)
    cfg, ctx, _ = _ctx("small", 3, 16, n_layers=1, B=2)
    V = cfg["vocab"]
    base = _tokens(cfg, 1, 4, 4)
    def run(toks):
        out = torch.empty((1, 8, V), device="cuda")
        uno.uno_train_forward(ctx, torch.from_numpy(toks).cuda(), out)
        uno.uno_status(ctx)
        return out.cpu().numpy()[0]
    ref = run(base)
    for j in range(8):
        t = base.copy()
        t[0, j] = (t[0, j] + 12345) % (V - 1)
        got = run(t)
        changed = np.array([not np.array_equal(got[i], ref[i]) for i in range(8)])
        assert np.array_equal(changed, want[:, j]), (j, changed.astype(int), want[:, j].astype(int))
    ctx.close()


def test_train_form_capacity_and_slots():
    cfg, ctx, _ = _ctx("small", 2, 64, n_layers=1)
    V = cfg["vocab"]
    toks = torch.from_numpy(_tokens(cfg, 1, 40, 5)).cuda()
    out = torch.empty((1, 80, V), device="cuda")
    for _ in range(3):                  # the two slots are free again after each call
        uno.uno_train_forward(ctx, toks, out)
    uno.uno_status(ctx)
    big = torch.from_numpy(_tokens(cfg, 1, 300, 5)).cuda()   # 600 rows > 512
    with pytest.raises(uno.UnoError) as e:
        uno.uno_train_forward(ctx, big, torch.empty((1, 600, V), device="cuda"))
    assert e.value.code == uno.UNO_ERR_CAPACITY
    ids = uno.uno_prefill(ctx, toks[:, :8].contiguous(), [8])   # one slot taken: one left
    with pytest.raises(uno.UnoError) as e:
        uno.uno_train_forward(ctx, toks, out)
    assert e.value.code == uno.UNO_ERR_CAPACITY
    uno.uno_release(ctx, ids[0])
    uno.uno_train_forward(ctx, toks, out)
    uno.uno_status(ctx)
    ctx.close()
