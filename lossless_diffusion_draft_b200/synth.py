"""Seeded synthetic inputs: model shapes, random-init weights, prompts, logits.

This module holds the workloads' data recipes and nothing of the method's
arithmetic.  The GPU path and the CPU oracle both consume what it makes, so
the two always see the same tensors; neither one's code lives here.

Workloads (sizes as the benchmark configurations state them):

* ``tiny``   - float32, 2 layers, d_model 64, 4 heads x 16 (no GQA), FFN 172,
  vocab 256, LoRA rank 8 / alpha 16, B=4, batch 1, 32-token prompt,
  64 generated tokens, Philox seed 1, weight seed 0.
* ``small``  - bfloat16, 8 layers, d_model 1024, 16 q / 4 kv heads x 64,
  FFN 2816, vocab 32000, LoRA rank 128 / alpha 256, B=8, batch 8,
  1024-token prompts, 512 generated tokens.
* ``qwen8b`` - bfloat16, Qwen3-8B shape: 36 layers, d_model 4096,
  32 q / 8 kv heads x 128, FFN 12288, vocab 151936, RoPE theta 1e6,
  LoRA rank 128 / alpha 256 on all seven projections, B=16, batch 1,
  1024-token prompt, 8192 generated tokens.
* ``qwen8b_maxbatch`` - the same model at the largest batch that fits.
* ``spec_verify`` - logits microbenchmark: p ~ N(0, 3), q = p + N(0, 0.5),
  fp32 [4096 = 256 requests x 16, 151936], Philox seed 7.

Weights: base matrices N(0, 0.02); LoRA A N(0, 0.02); LoRA B N(0, b_std)
(0.01 tiny, 0.002 otherwise); RMSNorm gains 1.  They are drawn tensor by
tensor in the order of :func:`param_list` from one ``torch.Generator``
seeded with the weight seed, on the device the weights are made on.
Prompts: uniform over [0, vocab-1) (the last id is the reserved MASK token),
from numpy's PCG64 seeded with the workload seed and the request index.
"""

import numpy as np
import torch

PROJ = ("q", "k", "v", "o", "gate", "up", "down")

_BASE = dict(rms_eps=1e-6, temperature=1.0, base_std=0.02, lora_a_std=0.02)

CONFIGS = {
    "tiny": dict(_BASE, n_layers=2, d_model=64, n_heads=4, n_kv_heads=4, head_dim=16,
                 ffn_dim=172, vocab=256, rope_theta=1e4, lora_rank=8, lora_alpha=16.0,
                 lora_b_std=0.01, dtype="f32", B=4, batch=1, prompt_len=32, gen_tokens=64,
                 seed=1, weight_seed=0),
    "small": dict(_BASE, n_layers=8, d_model=1024, n_heads=16, n_kv_heads=4, head_dim=64,
                  ffn_dim=2816, vocab=32000, rope_theta=1e4, lora_rank=128, lora_alpha=256.0,
                  lora_b_std=0.002, dtype="bf16", B=8, batch=8, prompt_len=1024,
                  gen_tokens=512, seed=2, weight_seed=0),
    "qwen8b": dict(_BASE, n_layers=36, d_model=4096, n_heads=32, n_kv_heads=8, head_dim=128,
                   ffn_dim=12288, vocab=151936, rope_theta=1e6, lora_rank=128,
                   lora_alpha=256.0, lora_b_std=0.002, dtype="bf16", B=16, batch=1,
                   prompt_len=1024, gen_tokens=8192, seed=3, weight_seed=0),
}
CONFIGS["qwen8b_maxbatch"] = dict(CONFIGS["qwen8b"], batch=0)   # 0: largest that fits

SPEC_VERIFY_BENCH = dict(requests=256, rows_per_request=16, vocab=151936,
                         p_std=3.0, q_noise_std=0.5, seed=7, logits_seed=0)


def model_shape(cfg):
    """The model-shape part of a workload (what ``uno_init`` and the oracle take)."""
    keys = ("n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim", "ffn_dim", "vocab",
            "rope_theta", "rms_eps", "lora_rank", "lora_alpha", "temperature")
    s = {k: cfg[k] for k in keys}
    s["mask_id"] = cfg["vocab"] - 1
    return s


def proj_shape(cfg, proj):
    """(out_features, in_features) of one projection."""
    d, H, Hkv, hd, F = (cfg[k] for k in ("d_model", "n_heads", "n_kv_heads", "head_dim", "ffn_dim"))
    return {"q": (H * hd, d), "k": (Hkv * hd, d), "v": (Hkv * hd, d), "o": (d, H * hd),
            "gate": (F, d), "up": (F, d), "down": (d, F)}[proj]


def param_list(cfg):
    """(name, shape, kind) of every parameter, in generation order.

    kind is one of "base", "gain", "lora_a", "lora_b".
    """
    V, d, r = cfg["vocab"], cfg["d_model"], cfg["lora_rank"]
    out = [("embed", (V, d), "base"), ("lm_head", (V, d), "base"), ("final_norm", (d,), "gain")]
    for l in range(cfg["n_layers"]):
        out.append((f"l{l}.attn_norm", (d,), "gain"))
        out.append((f"l{l}.ffn_norm", (d,), "gain"))
        for p in PROJ:
            out.append((f"l{l}.w_{p}", proj_shape(cfg, p), "base"))
        for p in PROJ:
            o, i = proj_shape(cfg, p)
            out.append((f"l{l}.lora_{p}.A", (r, i), "lora_a"))
            out.append((f"l{l}.lora_{p}.B", (o, r), "lora_b"))
    return out


def torch_dtype(cfg):
    return torch.float32 if cfg["dtype"] == "f32" else torch.bfloat16


def make_params(cfg, device="cpu", seed=None):
    """Random-init weights of a workload as a dict name -> tensor on ``device``."""
    dtype = torch_dtype(cfg)
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg["weight_seed"] if seed is None else seed)
    std = {"base": cfg["base_std"], "lora_a": cfg["lora_a_std"], "lora_b": cfg["lora_b_std"]}
    out = {}
    for name, shape, kind in param_list(cfg):
        if kind == "gain":
            out[name] = torch.ones(shape, dtype=dtype, device=device)
        else:
            t = torch.randn(shape, generator=gen, dtype=torch.float32, device=device)
            out[name] = (t * std[kind]).to(dtype)
    return out


def make_prompts(cfg, n_req=None, prompt_len=None, seed=None):
    """int32 [n_req, prompt_len] prompts, uniform over [0, vocab-1)."""
    n_req = cfg["batch"] if n_req is None else n_req
    prompt_len = cfg["prompt_len"] if prompt_len is None else prompt_len
    seed = cfg["seed"] if seed is None else seed
    rows = [np.random.Generator(np.random.PCG64([seed, i])).integers(0, cfg["vocab"] - 1, prompt_len)
            for i in range(n_req)]
    return np.stack(rows).astype(np.int32) if rows else np.zeros((0, prompt_len), np.int32)


def make_drafts(q_logits, seed=1, chunk=256):
    """int32 [rows] tokens drawn from softmax(q_logits) by the Gumbel-max rule.

    Input generator of the spec_verify microbenchmark (its drafted tokens
    come from q); it runs on q_logits' device with a seeded torch generator.
    """
    gen = torch.Generator(device=q_logits.device)
    gen.manual_seed(seed)
    rows, V = q_logits.shape
    out = torch.empty(rows, dtype=torch.int32, device=q_logits.device)
    for s in range(0, rows, chunk):
        e = min(rows, s + chunk)
        u = torch.rand((e - s, V), generator=gen, device=q_logits.device).clamp_(min=1e-30)
        out[s:e] = torch.argmax(q_logits[s:e] - torch.log(-torch.log(u)), dim=1).to(torch.int32)
    return out


def make_verify_logits(rows, vocab, device, p_std=3.0, q_noise_std=0.5, seed=0):
    """fp32 (p, q) logits [rows, vocab]: p ~ N(0, p_std), q = p + N(0, q_noise_std)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    p = torch.randn((rows, vocab), generator=gen, dtype=torch.float32, device=device) * p_std
    q = p + torch.randn((rows, vocab), generator=gen, dtype=torch.float32, device=device) * q_noise_std
    return p, q
