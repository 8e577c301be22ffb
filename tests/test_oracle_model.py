"""Pins of the oracle's model forward (CPU only).

Each elementary operation is checked against an independent formulation:
PyTorch CPU float64 functional ops, a closed form, a hand-written fixture or
a brute-force loop.
"""

import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from lossless_diffusion_draft_b200 import synth
from oracle import model as om
from oracle import psispec as ops

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _tiny_shape(**kw):
    s = dict(n_layers=2, d_model=32, n_heads=4, n_kv_heads=2, head_dim=8, ffn_dim=48, vocab=40,
             mask_id=39, rope_theta=1e4, rms_eps=1e-6, lora_rank=4, lora_alpha=8.0, temperature=1.0)
    s.update(kw)
    return s


def _random_params(shape, seed=0, lora_b_std=0.05):
    rng = np.random.default_rng(seed)
    p = {}
    for name, shp in om.param_names(shape):
        if name.endswith("norm"):
            p[name] = 1.0 + 0.1 * rng.standard_normal(shp)
        elif name.endswith(".B"):
            p[name] = lora_b_std * rng.standard_normal(shp)
        else:
            p[name] = 0.2 * rng.standard_normal(shp)
    return p


def test_rms_norm_matches_torch():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 24))
    g = rng.standard_normal(24)
    want = F.rms_norm(torch.from_numpy(x), (24,), torch.from_numpy(g), eps=1e-6).numpy()
    np.testing.assert_allclose(om.rms_norm(x, g, 1e-6), want, rtol=1e-13, atol=1e-14)


def test_silu_matches_torch():
    z = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(om.silu(z), F.silu(torch.from_numpy(z)).numpy(), rtol=1e-13, atol=1e-300)


def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(2)
    hd, theta = 16, 1e4
    x = rng.standard_normal((6, 3, hd))
    pos = np.array([0, 1, 5, 17, 1000, 9231])
    got = om.rope(x, pos, theta)
    half = hd // 2
    z = x[..., :half] + 1j * x[..., half:]
    freqs = np.array([theta ** (-(2.0 * i) / hd) for i in range(half)])
    rot = np.exp(1j * pos[:, None, None] * freqs[None, None, :])
    want = np.concatenate([(z * rot).real, (z * rot).imag], axis=-1)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(om.rope(x, np.zeros(6, int), theta), x)


def test_rope_relative_position_invariance():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 32))
    k = rng.standard_normal((1, 32))
    dots = [float((om.rope(q, [m + 7], 1e6) @ om.rope(k, [m], 1e6).T)[0, 0]) for m in (0, 11, 500, 8000)]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-9)


def test_attention_matches_torch_sdpa_gqa():
    rng = np.random.default_rng(4)
    n, m, H, Hkv, hd = 7, 11, 8, 2, 16
    q = rng.standard_normal((n, H, hd))
    k = rng.standard_normal((m, Hkv, hd))
    v = rng.standard_normal((m, Hkv, hd))
    allowed = rng.random((n, m)) < 0.6
    allowed[:, 0] = True
    got = om.attention(q, k, v, allowed)
    kk = torch.from_numpy(k).repeat_interleave(H // Hkv, dim=1).permute(1, 0, 2)
    vv = torch.from_numpy(v).repeat_interleave(H // Hkv, dim=1).permute(1, 0, 2)
    qq = torch.from_numpy(q).permute(1, 0, 2)
    want = F.scaled_dot_product_attention(qq, kk, vv, attn_mask=torch.from_numpy(allowed))
    np.testing.assert_allclose(got, want.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)


def test_attention_brute_force_loop_restricted():
    """Explicit -inf masking equals a softmax taken over the allowed keys only."""
    rng = np.random.default_rng(5)
    n, m, H, Hkv, hd = 6, 9, 4, 4, 8
    q = rng.standard_normal((n, H, hd))
    k = rng.standard_normal((m, Hkv, hd))
    v = rng.standard_normal((m, Hkv, hd))
    pos = np.arange(m)
    qpos = np.arange(m - n, m)
    allowed = om.block_causal_allowed(qpos, np.zeros(n, bool), np.zeros(n, int),
                                      pos, np.zeros(m, bool), np.zeros(m, int))
    got = om.attention(q, k, v, allowed)
    for i in range(n):
        keys = [j for j in range(m) if pos[j] <= qpos[i]]
        for h in range(H):
            s = np.array([q[i, h] @ k[j, h] / math.sqrt(hd) for j in keys])
            w = np.exp(s - s.max())
            w /= w.sum()
            o = sum(w[t] * v[j, h] for t, j in enumerate(keys))
            np.testing.assert_allclose(got[i, h], o, rtol=1e-12, atol=1e-13)


def test_block_causal_mask_training_form_fixture():
    want = np.loadtxt(os.path.join(GOLDEN, "block_causal_mask_x4_z4_B2.txt"), dtype=int).astype(bool)
    L, B = 4, 2
    pos = np.concatenate([np.arange(L), np.arange(L)])
    noised = np.array([False] * L + [True] * L)
    block = np.concatenate([np.zeros(L, int), (np.arange(L) // B) * B])
    got = om.block_causal_allowed(pos, noised, block, pos, noised, block)
    np.testing.assert_array_equal(got, want)


def test_block_causal_mask_inference_form_is_causal():
    c, B = 5, 4
    kpos = np.arange(c + B + 1)
    kn = np.array([False] * (c + 1) + [True] * B)
    kb = np.array([0] * (c + 1) + [c + 1] * B)
    qpos, qn, qb = kpos[c:], kn[c:], kb[c:]
    got = om.block_causal_allowed(qpos, qn, qb, kpos, kn, kb)
    np.testing.assert_array_equal(got, qpos[:, None] >= kpos[None, :])


def test_gated_lora_closed_forms():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((4, 12))
    W = rng.standard_normal((10, 12))
    A = rng.standard_normal((3, 12))
    B = rng.standard_normal((10, 3))
    s = 2.0
    y = om.gated_lora_linear(x, W, A, B, [0, 1, 0, 1], s)
    np.testing.assert_array_equal(y[[0, 2]], (x @ W.T)[[0, 2]])
    np.testing.assert_allclose(y[[1, 3]], x[[1, 3]] @ (W + s * B @ A).T, rtol=1e-12, atol=1e-12)


def test_gate_off_identity_bit_exact():
    """With every gate off, the LoRA weights cannot change the logits at all."""
    shape = _tiny_shape()
    p1 = _random_params(shape, 0)
    p2 = dict(p1)
    rng = np.random.default_rng(9)
    for name, shp in om.param_names(shape):
        if ".lora_" in name:
            p2[name] = rng.standard_normal(shp)
    m1, m2 = om.Model(shape, p1), om.Model(shape, p2)
    toks = [3, 7, 1, 38, 38]
    pos = np.arange(5)
    l1, _, _ = m1.forward(om.KVCache(shape), toks, pos, np.zeros(5))
    l2, _, _ = m2.forward(om.KVCache(shape), toks, pos, np.zeros(5))
    np.testing.assert_array_equal(l1, l2)
    g1, _, _ = m1.forward(om.KVCache(shape), toks, pos, np.ones(5))
    g2, _, _ = m2.forward(om.KVCache(shape), toks, pos, np.ones(5))
    assert np.max(np.abs(g1 - g2)) > 1e-3


def test_incremental_cache_equals_full_recompute():
    shape = _tiny_shape()
    m = om.Model(shape, _random_params(shape, 1))
    toks = [5, 9, 2, 11, 30, 4, 17]
    full, _, _ = m.forward(om.KVCache(shape), toks, np.arange(7), np.zeros(7))
    st = ops.prefill(m, toks[:3])
    for t in toks[3:]:
        logits, _, _ = m.forward(st.cache, [st.pending], [st.c], [0.0])
        np.testing.assert_allclose(logits[0], full[st.c], rtol=1e-12, atol=1e-12)
        cache = st.cache.copy()
        _, k, v = m.forward(st.cache, [st.pending], [st.c], [0.0])
        cache.append(k, v, [0])
        st = ops.DecodeState(st.tokens + [t], cache)


def test_draft_row0_is_the_ar_distribution():
    """The block's first token is drawn from AR weights only: the pending row
    of the draft pass equals the AR forward of the same state."""
    shape = _tiny_shape()
    m = om.Model(shape, _random_params(shape, 2))
    st = ops.prefill(m, [1, 2, 3, 4, 5])
    ld, _, _ = ops.draft_pass(m, st, 4)
    _, lar, _ = ops.ar_step(m, st, seed=0)
    np.testing.assert_allclose(ld[0], lar, rtol=1e-12, atol=1e-12)


def test_noised_rows_see_no_later_rows():
    """Causal inside the noised block: changing later MASK rows' gates leaves
    earlier rows' logits unchanged."""
    shape = _tiny_shape()
    m = om.Model(shape, _random_params(shape, 3))
    st = ops.prefill(m, [1, 2, 3])
    c, B = st.c, 4
    toks = [st.pending] + [shape["mask_id"]] * B
    pos = np.arange(c, c + B + 1)
    noised = np.array([False] + [True] * B)
    block = np.array([0] + [c + 1] * B)
    l1, _, _ = m.forward(st.cache, toks, pos, [0, 1, 1, 1, 1], noised, block)
    l2, _, _ = m.forward(st.cache, toks, pos, [0, 1, 1, 0, 0], noised, block)
    np.testing.assert_array_equal(l1[:3], l2[:3])
    assert np.max(np.abs(l1[3:] - l2[3:])) > 0


def test_lora_param_count_qwen8b():
    """Rank 128 on q/k/v/o/gate/up/down of the Qwen3-8B shape is the 0.35B of
    the pages (Walkthrough section on the Qwen3-8B comparison)."""
    s = synth.model_shape(synth.CONFIGS["qwen8b"])
    assert om.lora_param_count(s) == 349_175_808


@pytest.mark.parametrize("name", ["tiny", "small", "qwen8b"])
def test_synth_param_list_matches_oracle(name):
    cfg = synth.CONFIGS[name]
    a = [(n, tuple(s)) for n, s, _ in synth.param_list(cfg)]
    b = [(n, tuple(s)) for n, s in om.param_names(synth.model_shape(cfg))]
    assert a == b


def test_temperature_divides_the_logits():
    """Logits at temperature T are the T = 1 logits divided by T (the model
    forward does not depend on T), and softmax(l / T) sharpens as T falls:
    at T -> 0 the distribution concentrates on the argmax."""
    shape = _tiny_shape()
    p = _random_params(shape, 4)
    toks, pos = [3, 1, 4, 1, 5], np.arange(5)
    l1, _, _ = om.Model(shape, p).forward(om.KVCache(shape), toks, pos, np.zeros(5))
    for t in (0.7, 1.3):
        lt, _, _ = om.Model(_tiny_shape(temperature=t), p).forward(om.KVCache(shape), toks, pos,
                                                                     np.zeros(5))
        np.testing.assert_allclose(lt, l1 / t, rtol=1e-12, atol=1e-14)
    lc, _, _ = om.Model(_tiny_shape(temperature=1e-3), p).forward(om.KVCache(shape), toks, pos,
                                                                  np.zeros(5))
    probs = np.exp(lc - lc.max(axis=-1, keepdims=True))
    probs /= probs.sum(axis=-1, keepdims=True)
    assert np.all(probs.argmax(axis=-1) == l1.argmax(axis=-1))
    assert np.all(probs.max(axis=-1) > 0.99)


# ---------------------------------------------------------------------------
# Layer composition.  The elementary ops above are pinned one by one; these
# closed forms pin how Model.forward puts them together: which RMSNorm feeds
# which block, that the attention and FFN outputs enter only through o and
# down as residual adds, that SiLU acts on the gate projection and multiplies
# the up projection, and the final norm / untied head / temperature.
# (Walkthrough §一句话直觉: one causal Transformer whose frozen AR weights
# carry the diffusion path as a gated LoRA; the decoder layout is the
# Qwen3-style pre-norm block the workloads name.)
# ---------------------------------------------------------------------------

def _one_layer_shape(**kw):
    s = dict(n_layers=1, d_model=4, n_heads=1, n_kv_heads=1, head_dim=4, ffn_dim=2, vocab=4,
             mask_id=3, rope_theta=1e4, rms_eps=0.0, lora_rank=1, lora_alpha=1.0, temperature=1.0)
    s.update(kw)
    return s


def _zero_params(shape):
    return {name: np.zeros(shp) for name, shp in om.param_names(shape)}


def test_composition_skeleton_with_o_and_down_zeroed():
    """w_o = w_down = 0 in every layer: the residual stream keeps the raw
    embedding row, so logits = lm_head . rmsnorm(embed[t], final_norm) / T
    whatever the attention, gate, up weights, gains and LoRA gates are."""
    shape = _tiny_shape(temperature=0.8)
    p = _random_params(shape, 11)
    for l in range(shape["n_layers"]):
        for proj in ("o", "down"):
            p[f"l{l}.w_{proj}"] = np.zeros_like(p[f"l{l}.w_{proj}"])
            p[f"l{l}.lora_{proj}.B"] = np.zeros_like(p[f"l{l}.lora_{proj}.B"])
    m = om.Model(shape, p)
    toks = [5, 9, 2, 11, 30]
    logits, _, _ = m.forward(om.KVCache(shape), toks, np.arange(5), [0, 1, 0, 1, 1])
    e = p["embed"][toks]
    g = p["final_norm"]
    for i in range(5):
        rms = math.sqrt(sum(v * v for v in e[i]) / shape["d_model"] + shape["rms_eps"])
        want = [sum(p["lm_head"][t][j] * e[i][j] / rms * g[j] for j in range(shape["d_model"])) / 0.8
                for t in range(shape["vocab"])]
        np.testing.assert_allclose(logits[i], want, rtol=1e-12, atol=1e-12)


def test_composition_attention_branch_uses_attn_norm():
    """One token, one layer, w_down = 0, W_v = W_o = I, lm_head = I, final
    gain 1, eps 0.  A single key gets softmax weight 1, so the attention
    output is that token's value row and x1 = x + g_attn * x / rms(x).
    x = (3, 0, 4, 0): rms = 2.5, x / rms = (1.2, 0, 1.6, 0); attn_norm gains
    (1, 2, 3, 4) give x1 = (4.2, 0, 8.8, 0).  The ffn_norm gains (5, ...)
    would give (9, 0, 12, 0) if the two norms were swapped."""
    shape = _one_layer_shape()
    p = _zero_params(shape)
    p["embed"][1] = [3.0, 0.0, 4.0, 0.0]
    p["l0.attn_norm"] = np.array([1.0, 2.0, 3.0, 4.0])
    p["l0.ffn_norm"] = np.array([5.0, 5.0, 5.0, 5.0])
    p["l0.w_v"] = np.eye(4)
    p["l0.w_o"] = np.eye(4)
    p["l0.w_q"] = np.eye(4)
    p["l0.w_k"] = np.eye(4)
    p["lm_head"] = np.eye(4)
    p["final_norm"] = np.ones(4)
    logits, k_rows, v_rows = om.Model(shape, p).forward(om.KVCache(shape), [1], [0], [0.0])
    x1 = np.array([4.2, 0.0, 8.8, 0.0])
    rms1 = math.sqrt((4.2 ** 2 + 8.8 ** 2) / 4)
    np.testing.assert_allclose(logits[0], x1 / rms1, rtol=1e-13, atol=1e-15)
    # the cached value row is W_v applied to the attn-normed input
    np.testing.assert_allclose(v_rows[0][0, 0], [1.2, 0.0, 4.8, 0.0], rtol=1e-13, atol=1e-15)


def test_composition_ffn_is_silu_gate_times_up_on_ffn_norm():
    """One token, one layer, w_o = 0 (x1 = x).  x = (2, 2, 2, 2), eps 0:
    x / rms = 1 everywhere; ffn_norm gains 0.5 give n = (0.5, ...).  W_gate
    row 0 = (4, 0, 0, 0) -> gate 2; W_up row 0 = (0, -6, 0, 0) -> up -3;
    W_down column 0 = e_0.  x2 = x + silu(2) * (-3) e_0 with
    silu(2) = 2 / (1 + e^-2).  Swapping the roles would give
    silu(-3) * 2 = -6 / (1 + e^3); the attn_norm gains (7, ...) would give
    gate 28, up -42 if the two norms were swapped."""
    shape = _one_layer_shape()
    p = _zero_params(shape)
    p["embed"][2] = [2.0, 2.0, 2.0, 2.0]
    p["l0.attn_norm"] = np.full(4, 7.0)
    p["l0.ffn_norm"] = np.full(4, 0.5)
    p["l0.w_gate"][0] = [4.0, 0.0, 0.0, 0.0]
    p["l0.w_up"][0] = [0.0, -6.0, 0.0, 0.0]
    p["l0.w_down"][:, 0] = [1.0, 0.0, 0.0, 0.0]
    p["lm_head"] = np.eye(4)
    p["final_norm"] = np.ones(4)
    logits, _, _ = om.Model(shape, p).forward(om.KVCache(shape), [2], [0], [0.0])
    act = -3.0 * 2.0 / (1.0 + math.exp(-2.0))
    x2 = np.array([2.0 + act, 2.0, 2.0, 2.0])
    np.testing.assert_allclose(logits[0], x2 / math.sqrt(np.mean(x2 * x2)), rtol=1e-13, atol=1e-15)
    swapped = np.array([2.0 + 2.0 * (-3.0) / (1.0 + math.exp(3.0)), 2.0, 2.0, 2.0])
    assert np.max(np.abs(logits[0] - swapped / math.sqrt(np.mean(swapped * swapped)))) > 0.1


def test_composition_gated_lora_on_every_projection():
    """With the gate on, each projection is W + (alpha / r) B A: a model with
    adapters and gate 1 equals the adapter-free model whose base weights are
    W + (alpha / r) B A, on every one of the seven projections at once (and
    gate 0 equals the plain base model)."""
    shape = _tiny_shape()
    p = _random_params(shape, 12, lora_b_std=0.3)
    merged = dict(p)
    plain = dict(p)
    scale = shape["lora_alpha"] / shape["lora_rank"]
    for l in range(shape["n_layers"]):
        for proj in om.PROJ:
            A, B = p[f"l{l}.lora_{proj}.A"], p[f"l{l}.lora_{proj}.B"]
            merged[f"l{l}.w_{proj}"] = p[f"l{l}.w_{proj}"] + scale * (B @ A)
            merged[f"l{l}.lora_{proj}.B"] = np.zeros_like(B)
            plain[f"l{l}.lora_{proj}.B"] = np.zeros_like(B)
    toks, pos = [4, 8, 15, 16, 23], np.arange(5)
    on, _, _ = om.Model(shape, p).forward(om.KVCache(shape), toks, pos, np.ones(5))
    want, _, _ = om.Model(shape, merged).forward(om.KVCache(shape), toks, pos, np.zeros(5))
    np.testing.assert_allclose(on, want, rtol=1e-10, atol=1e-10)
    off, _, _ = om.Model(shape, p).forward(om.KVCache(shape), toks, pos, np.zeros(5))
    base, _, _ = om.Model(shape, plain).forward(om.KVCache(shape), toks, pos, np.zeros(5))
    np.testing.assert_array_equal(off, base)
    assert np.max(np.abs(on - off)) > 1e-2
