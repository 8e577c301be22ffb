"""Transformer forward with gated LoRA and an explicit block-causal mask.

This is the model the Psi-Spec sampler runs twice per iteration: once with
the diffusion weights switched on at the noised positions (draft pass) and
once with the AR weights alone (verify pass).

What the pages fix:

* One causal Transformer keeps its AR weights W_base frozen and carries the
  diffusion weights W_diff as a rank-r LoRA (rank 128, alpha 256) on every
  layer (Summary §方法关键点; Walkthrough §一句话直觉).
* A per-position gate switches the LoRA off at clean positions and on at
  noised positions, so one forward computes both paths
  (Walkthrough §Diffusion Distillation：一步蒸馏 + 块级扩散).
* The block-causal mask: the clean sequence is causal; each noised block is
  causal inside itself and attends to all clean tokens before the block
  (Walkthrough §Diffusion Distillation：一步蒸馏 + 块级扩散).

Readings where the pages are silent (the synthetic model shape is the
Qwen3-style decoder the workloads name):

* pre-RMSNorm blocks with gains, eps 1e-6; no biases; no QK-norm;
* rotate-half (NeoX) RoPE on q and k at absolute positions;
* grouped-query attention: q head h reads kv head h // (H / Hkv);
  attention scale 1 / sqrt(head_dim);
* SwiGLU FFN: down(silu(gate(n)) * up(n));
* untied embedding and LM head, the embedding is not scaled;
* every projection is W v + g * (alpha / r) * B (A v), the LoRA on
  q/k/v/o/gate/up/down (349,175,808 LoRA parameters for the Qwen3-8B
  shape, the "0.35B" of Walkthrough §战线二);
* logits are divided by the temperature.

Parameters are a dict of float64 numpy arrays (see :func:`param_names`),
weights row-major [out, in] as in ``torch.nn.Linear``; LoRA ``A`` is
[r, in] and ``B`` is [out, r].
"""

import math

import numpy as np

PROJ = ("q", "k", "v", "o", "gate", "up", "down")


def proj_dims(shape, proj):
    """(out_features, in_features) of a projection of one layer."""
    d, H, Hkv, hd, F = (shape[k] for k in ("d_model", "n_heads", "n_kv_heads", "head_dim", "ffn_dim"))
    return {
        "q": (H * hd, d), "k": (Hkv * hd, d), "v": (Hkv * hd, d), "o": (d, H * hd),
        "gate": (F, d), "up": (F, d), "down": (d, F),
    }[proj]


def param_names(shape):
    """Every parameter of the model, in a fixed order, with its shape.

    Names: ``embed``, ``lm_head``, ``final_norm``; per layer l
    ``l{l}.attn_norm``, ``l{l}.ffn_norm``, ``l{l}.w_{proj}`` for the seven
    projections and ``l{l}.lora_{proj}.A`` / ``.B``.
    """
    V, d = shape["vocab"], shape["d_model"]
    r = shape["lora_rank"]
    out = [("embed", (V, d)), ("lm_head", (V, d)), ("final_norm", (d,))]
    for l in range(shape["n_layers"]):
        out.append((f"l{l}.attn_norm", (d,)))
        out.append((f"l{l}.ffn_norm", (d,)))
        for p in PROJ:
            o, i = proj_dims(shape, p)
            out.append((f"l{l}.w_{p}", (o, i)))
        for p in PROJ:
            o, i = proj_dims(shape, p)
            out.append((f"l{l}.lora_{p}.A", (r, i)))
            out.append((f"l{l}.lora_{p}.B", (o, r)))
    return out


def lora_param_count(shape):
    """Number of LoRA parameters: r * (in + out) per projection, all layers."""
    r = shape["lora_rank"]
    per_layer = sum(r * (o + i) for o, i in (proj_dims(shape, p) for p in PROJ))
    return per_layer * shape["n_layers"]


# ---------------------------------------------------------------------------
# Elementary operations.  Each is pinned in the tests against an independent
# formulation (PyTorch CPU functional ops in float64, or a closed form).
# ---------------------------------------------------------------------------

def rms_norm(x, gain, eps):
    """x / sqrt(mean(x^2) + eps) * gain over the last axis."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * gain


def rope(x, positions, theta):
    """Rotate-half rotary embedding of x [..., n, hd] at integer positions [n].

    Dimension pair (i, i + hd/2) is rotated by the angle pos * theta^(-2i/hd).
    """
    hd = x.shape[-1]
    half = hd // 2
    inv_freq = theta ** (-np.arange(half, dtype=np.float64) * 2.0 / hd)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv_freq[None, :]
    cos, sin = np.cos(ang), np.sin(ang)
    if x.ndim == 3:  # [n, heads, hd]: broadcast over heads
        cos, sin = cos[:, None, :], sin[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def silu(z):
    """z * sigmoid(z)."""
    return z / (1.0 + np.exp(-z))


def gated_lora_linear(x, W, A, B, gate, scale):
    """y = x W^T + (gate * scale) (x A^T) B^T, one gate value per row of x.

    With gate 0 the result is the base projection alone (the AR path); with
    gate 1 it is the diffusion path W_base + W_diff.
    """
    y = x @ W.T
    if A is not None:
        g = (np.asarray(gate, dtype=np.float64) * scale)[:, None]
        y = y + g * ((x @ A.T) @ B.T)
    return y


# ---------------------------------------------------------------------------
# Block-causal mask and attention.
# ---------------------------------------------------------------------------

def block_causal_allowed(q_pos, q_noised, q_block, k_pos, k_noised, k_block):
    """Explicit mask matrix [n_q, n_k]: True where query i may attend key j.

    Every token carries (pos, noised, block) where ``block`` is the start
    position of the noised block it belongs to (ignored for clean tokens).

    * clean query:  clean keys at positions <= its own (causal);
    * noised query: clean keys before its block starts, and noised keys of
      its own block at positions <= its own (causal inside the block).
    """
    qp, qn, qb = (np.asarray(a)[:, None] for a in (q_pos, q_noised, q_block))
    kp, kn, kb = (np.asarray(a)[None, :] for a in (k_pos, k_noised, k_block))
    clean_q = (~qn) & (~kn) & (kp <= qp)
    noised_q = qn & (((~kn) & (kp < qb)) | (kn & (kb == qb) & (kp <= qp)))
    return clean_q | noised_q


def attention(q, k, v, allowed):
    """Masked softmax attention with grouped-query heads.

    q [n, H, hd], k and v [m, Hkv, hd], allowed [n, m] boolean.
    Scores q.k / sqrt(hd) get -inf where not allowed; every query must be
    allowed at least one key.  Returns [n, H, hd].
    """
    n, H, hd = q.shape
    Hkv = k.shape[1]
    group = H // Hkv
    out = np.empty_like(q)
    scale = 1.0 / math.sqrt(hd)
    for h in range(H):
        kvh = h // group
        s = (q[:, h, :] @ k[:, kvh, :].T) * scale
        s = np.where(allowed, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, kvh, :]
    return out


# ---------------------------------------------------------------------------
# KV cache and the forward of a set of rows.
# ---------------------------------------------------------------------------

class KVCache:
    """Committed keys/values of one sequence: clean tokens at positions 0..n-1.

    ``k[l]`` and ``v[l]`` are [n, Hkv, hd] float64 arrays for layer l (keys
    already rotated).
    """

    def __init__(self, shape):
        L, Hkv, hd = shape["n_layers"], shape["n_kv_heads"], shape["head_dim"]
        self.k = [np.zeros((0, Hkv, hd)) for _ in range(L)]
        self.v = [np.zeros((0, Hkv, hd)) for _ in range(L)]

    def __len__(self):
        return self.k[0].shape[0]

    def copy(self):
        c = KVCache.__new__(KVCache)
        c.k = [a.copy() for a in self.k]
        c.v = [a.copy() for a in self.v]
        return c

    def append(self, k_rows, v_rows, take):
        """Commit rows ``take`` (indices into a pass's rows) of a pass's K/V."""
        take = list(take)
        for l in range(len(self.k)):
            self.k[l] = np.concatenate([self.k[l], k_rows[l][take]], axis=0)
            self.v[l] = np.concatenate([self.v[l], v_rows[l][take]], axis=0)


class _Float64View:
    """Read-only float64 view of a parameter mapping, converted per access."""

    def __init__(self, params):
        self._params = params

    def __getitem__(self, name):
        return np.asarray(self._params[name], dtype=np.float64)


class Model:
    """A model of a given shape with float64 parameters.

    ``shape`` keys: n_layers, d_model, n_heads, n_kv_heads, head_dim,
    ffn_dim, vocab, mask_id, rope_theta, rms_eps, lora_rank, lora_alpha,
    temperature.
    """

    def __init__(self, shape, params):
        self.shape = dict(shape)
        if isinstance(params, dict):
            self.p = {k: np.asarray(v, dtype=np.float64) for k, v in params.items()}
        else:
            # any other mapping is read on demand, one parameter at a time (a
            # model too large to hold in float64 at once); same values
            self.p = _Float64View(params)
        self.scale = shape["lora_alpha"] / shape["lora_rank"]

    def _lin(self, l, proj, x, gate):
        p = self.p
        return gated_lora_linear(x, p[f"l{l}.w_{proj}"], p[f"l{l}.lora_{proj}.A"],
                                 p[f"l{l}.lora_{proj}.B"], gate, self.scale)

    def forward(self, cache, tokens, positions, gates, noised=None, block=None):
        """Forward a set of rows on top of the committed cache.

        The keys are the cache (clean, positions 0..len-1) followed by the
        rows themselves; the explicit block-causal mask decides which keys
        each row sees.  Returns (logits [n, V], k_rows, v_rows) where
        k_rows[l] / v_rows[l] are the rows' rotated keys / values of layer l.
        """
        s = self.shape
        H, Hkv, hd = s["n_heads"], s["n_kv_heads"], s["head_dim"]
        tokens = np.asarray(tokens, dtype=np.int64)
        positions = np.asarray(positions, dtype=np.int64)
        gates = np.asarray(gates, dtype=np.float64)
        n = tokens.shape[0]
        noised = np.zeros(n, bool) if noised is None else np.asarray(noised, bool)
        block = np.zeros(n, np.int64) if block is None else np.asarray(block, np.int64)
        m0 = len(cache)
        k_pos = np.concatenate([np.arange(m0), positions])
        k_noised = np.concatenate([np.zeros(m0, bool), noised])
        k_block = np.concatenate([np.zeros(m0, np.int64), block])
        allowed = block_causal_allowed(positions, noised, block, k_pos, k_noised, k_block)

        x = self.p["embed"][tokens]
        k_rows, v_rows = [], []
        for l in range(s["n_layers"]):
            h = rms_norm(x, self.p[f"l{l}.attn_norm"], s["rms_eps"])
            q = self._lin(l, "q", h, gates).reshape(n, H, hd)
            k = self._lin(l, "k", h, gates).reshape(n, Hkv, hd)
            v = self._lin(l, "v", h, gates).reshape(n, Hkv, hd)
            q = rope(q, positions, s["rope_theta"])
            k = rope(k, positions, s["rope_theta"])
            keys = np.concatenate([cache.k[l], k], axis=0)
            vals = np.concatenate([cache.v[l], v], axis=0)
            a = attention(q, keys, vals, allowed).reshape(n, H * hd)
            x = x + self._lin(l, "o", a, gates)
            h2 = rms_norm(x, self.p[f"l{l}.ffn_norm"], s["rms_eps"])
            act = silu(self._lin(l, "gate", h2, gates)) * self._lin(l, "up", h2, gates)
            x = x + self._lin(l, "down", act, gates)
            k_rows.append(k)
            v_rows.append(v)
        hf = rms_norm(x, self.p["final_norm"], s["rms_eps"])
        logits = (hf @ self.p["lm_head"].T) / s.get("temperature", 1.0)
        return logits, k_rows, v_rows
