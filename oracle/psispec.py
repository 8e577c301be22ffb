"""The Psi-Spec linear sampler, AR-only decoding and prefill.

What the pages fix (Walkthrough §Ψ-Spec 采样器：起草、验证、两种模式;
Summary §方法关键点; Walkthrough §一句话直觉):

* the diffusion path drafts a block of B tokens in parallel from a fully
  noised block; the block's first token is sampled from the AR weights only
  and is therefore always accepted;
* the AR path verifies the whole block in parallel; the longest accepted
  prefix is kept and the first rejected position is redrawn from the
  renormalised residual max(0, p_AR - q_diff), which is standard
  speculative rejection sampling, so the output follows the AR distribution;
* two forwards per iteration, 1 <= TPF <= (B+1)/2, at least 2 tokens out.

Readings where the pages are silent or garbled (each one is an input to the
tests; the GPU path follows the same readings):

* State: ``c`` committed tokens have keys/values in the cache (positions
  0..c-1); the last produced token ``pending`` sits at position c and has no
  keys/values yet.  Prefill caches all prompt tokens but the last, which
  becomes the pending token; nothing is sampled at prefill.
* Draft pass: rows [pending (gate 0), MASK x B (gate 1)] at positions
  c..c+B; the MASK rows form one noised block starting at c+1.  The noise
  prior is a reserved MASK token id (absorbing state).  Row 0 gives the AR
  distribution p_1 of position c+1; MASK row i (position c+i) gives the
  diffusion distribution q_i of the token at its own position.  Row 1's
  logits are unused because the first token comes from the AR row.
* Verify pass: rows x_1..x_B at positions c+1..c+B, gate 0, causal.  Row j
  gives p_{j+1}, the AR distribution of position c+j+1.
* Accept test for draft i = 2..B: u < p_i(x_i) / q_i(x_i) with a strict
  inequality, taken in the log domain.  ``a`` counts the first token plus
  the accepted prefix, a in [1, B].  If a < B the token at position c+a+1 is
  redrawn from max(0, p_{a+1} - q_{a+1}) normalised (from p when that mass
  is zero after rounding); otherwise a bonus token is drawn from p_{B+1}.
  a+1 tokens are emitted.
* Commit: the keys/values of positions c..c+a become part of the cache; the
  emitted last token becomes the new pending token at position c+a+1.
* Inverse-CDF sampling: weights w_v = exp(l_v - max l) in vocabulary order;
  the token is the smallest t whose inclusive prefix sum exceeds u * sum(w);
  if rounding leaves none, the last token with positive weight.
* Uniforms are Philox draws keyed by (seed; stream, position, kind); see
  :mod:`oracle.philox`.
"""

import math
from dataclasses import dataclass, field

import numpy as np

from .model import KVCache
from .philox import KIND_ACCEPT, KIND_DRAFT, KIND_FIRST, KIND_RESID, uniform


# ---------------------------------------------------------------------------
# Sampler primitives.  Each is pinned in the tests by measuring, by bisection
# over u, the set of uniforms that produces each outcome and comparing the
# measure with the closed-form probability.
# ---------------------------------------------------------------------------

def _inverse_cdf(weights, u):
    """Smallest t with inclusive prefix sum > u * total; fallback: last w > 0."""
    c = np.cumsum(weights)
    hit = np.nonzero(c > u * c[-1])[0]
    if hit.size:
        return int(hit[0])
    return int(np.nonzero(weights > 0)[0][-1])


def log_softmax(logits):
    """logits - logsumexp(logits), max-shifted."""
    m = np.max(logits)
    return logits - (m + math.log(np.sum(np.exp(logits - m))))


def sample_token(logits, u):
    """Draw a token from softmax(logits) by inverse CDF with uniform u."""
    w = np.exp(logits - np.max(logits))
    return _inverse_cdf(w, u)


def top_p_logits(logits, top_p):
    """Nucleus filter of one row (Walkthrough §我的判断: the lossless claim is
    stated for the sampling distribution with temperature 1 and top-p 0.95).

    Reading: the nucleus is the smallest set of most probable tokens whose
    probability reaches ``top_p`` -- tokens ordered by probability, ties by
    token id, and the token that crosses ``top_p`` is kept; every other
    logit becomes -inf, so softmax of the result is the renormalised
    filtered distribution.  Speculative sampling applies the same filter to
    the AR rows p and to the drafter's rows q, and is then lossless with
    respect to the filtered p.  ``top_p >= 1`` keeps every token.
    """
    logits = np.asarray(logits, dtype=np.float64)
    if top_p >= 1.0:
        return logits.copy()
    p = np.exp(log_softmax(logits))
    order = np.lexsort((np.arange(p.size), -p))      # most probable first, ties by id
    cum = np.cumsum(p[order])
    k = min(int(np.searchsorted(cum, top_p, side="left")), p.size - 1)
    out = np.full_like(logits, -np.inf)
    keep = order[: k + 1]
    out[keep] = logits[keep]
    return out


def accept_draft(p_logits, q_logits, token, u):
    """Accept test: log u < log p(token) - log q(token), i.e. u < p/q."""
    lp = log_softmax(p_logits)[token]
    lq = log_softmax(q_logits)[token]
    return math.log(u) < lp - lq


def residual_token(p_logits, q_logits, u):
    """Draw from max(0, p - q) renormalised; from p if that mass is zero."""
    p = np.exp(log_softmax(p_logits))
    q = np.exp(log_softmax(q_logits))
    r = np.maximum(p - q, 0.0)
    if not np.sum(r) > 0.0:
        return sample_token(p_logits, u)
    return _inverse_cdf(r, u)


def rrs_token(p_logits, q_logits, cands, u_accept, u_resid):
    """Recursive rejection over several candidates drawn i.i.d. from q (the
    tree sampler's step at one position; with one candidate it is the linear
    sampler's accept test and residual draw).

    The target starts as p.  Candidate j is accepted iff
    u_accept[j] < r(y_j) / q(y_j) (log domain, strict) for the current
    target r; on a rejection r becomes max(0, r - q) renormalised (kept as it
    is if that has no mass after rounding).  If every candidate is rejected
    the token is drawn from the last r with u_resid.  Returns (j, token):
    j = index of the accepted candidate, or None with the drawn token.
    Lossless: the returned token follows p (pinned by exact enumeration).
    Uniforms are read only when used: u_accept[j] when candidate j is
    tested, u_resid (a number, or a function of no argument giving it) only
    for the residual draw.
    """
    cands = [int(y) for y in cands]
    resid_u = u_resid if callable(u_resid) else (lambda: u_resid)
    if accept_draft(p_logits, q_logits, cands[0], u_accept[0]):
        return 0, cands[0]
    if len(cands) == 1:
        return None, residual_token(p_logits, q_logits, resid_u())
    q = np.exp(log_softmax(np.asarray(q_logits, np.float64)))
    r = np.exp(log_softmax(np.asarray(p_logits, np.float64)))
    for j, y in enumerate(cands):
        if j > 0 and r[y] > 0 and math.log(u_accept[j]) < math.log(r[y]) - math.log(q[y]):
            return j, y
        res = np.maximum(r - q, 0.0)
        z = float(np.sum(res))
        if z > 0.0:
            r = res / z
    return None, _inverse_cdf(r, resid_u())


def verify_block(p_rows, q_rows, drafts, u_accept, u_resid, bonus_row):
    """Rejection step over a drafted block.

    ``p_rows[j]`` / ``q_rows[j]`` are the AR and diffusion logits of tested
    draft j, ``drafts[j]`` its token, ``u_accept[j]`` its accept uniform,
    ``u_resid[j]`` the uniform used if j is the first rejection.  When every
    test passes, the bonus token is drawn from ``bonus_row`` with
    ``u_resid[len(drafts)]`` (no token when ``bonus_row`` is None).

    Returns (n_accepted, next_token or None, accept_bits); tests after the
    first rejection are evaluated and reported but do not count.
    """
    bits = [accept_draft(p_rows[j], q_rows[j], drafts[j], u_accept[j]) for j in range(len(drafts))]
    n_acc = 0
    while n_acc < len(drafts) and bits[n_acc]:
        n_acc += 1
    if n_acc < len(drafts):
        nxt = residual_token(p_rows[n_acc], q_rows[n_acc], u_resid[n_acc])
    elif bonus_row is not None:
        nxt = sample_token(bonus_row, u_resid[len(drafts)])
    else:
        nxt = None
    return n_acc, nxt, bits


# ---------------------------------------------------------------------------
# Decode state and the decode iterations.
# ---------------------------------------------------------------------------

@dataclass
class DecodeState:
    """One request: committed tokens, cache of positions 0..c-1, pending token."""
    tokens: list                 # every token so far; tokens[-1] is pending
    cache: KVCache
    stream: int = 0

    @property
    def c(self):
        return len(self.cache)

    @property
    def pending(self):
        return self.tokens[-1]

    def copy(self):
        return DecodeState(list(self.tokens), self.cache.copy(), self.stream)


def prefill(model, prompt, stream=0):
    """Cache every prompt token but the last; the last becomes pending."""
    prompt = [int(t) for t in prompt]
    if len(prompt) < 1:
        raise ValueError("prompt must hold at least one token")
    cache = KVCache(model.shape)
    n = len(prompt) - 1
    if n > 0:
        _, k, v = model.forward(cache, prompt[:n], np.arange(n), np.zeros(n))
        cache.append(k, v, range(n))
    return DecodeState(prompt, cache, stream)


@dataclass
class StepResult:
    """Everything one Psi-Spec iteration decided, for stage-by-stage checks."""
    c: int                              # cached tokens before the step
    logits_draft: np.ndarray            # [B+1, V] draft pass rows
    logits_verify: np.ndarray           # [B, V] verify pass rows
    drafts: list                        # x_1..x_B
    accept_bits: list                   # tests of x_2..x_B
    a: int                              # first token + accepted prefix, in [1, B]
    next_token: int                     # resampled or bonus token
    emitted: list = field(default_factory=list)   # x_1..x_a, next_token


def draft_pass(model, state, B):
    """Rows [pending, MASK x B] at positions c..c+B, gates [0, 1 x B]."""
    c = state.c
    mask_id = model.shape["mask_id"]
    tokens = [state.pending] + [mask_id] * B
    pos = np.arange(c, c + B + 1)
    gates = np.array([0.0] + [1.0] * B)
    noised = np.array([False] + [True] * B)
    block = np.array([0] + [c + 1] * B)
    return model.forward(state.cache, tokens, pos, gates, noised, block)


def verify_pass(model, cache_with_pending, c, drafts):
    """Rows x_1..x_B at positions c+1..c+B, gate 0, over cache 0..c."""
    B = len(drafts)
    return model.forward(cache_with_pending, drafts, np.arange(c + 1, c + B + 1), np.zeros(B))


def spec_step(model, state, B, seed, drafts=None, uniform_fn=None, top_p=None):
    """One Psi-Spec iteration; returns (new_state, StepResult).

    ``drafts`` (optional) replaces the sampled block x_1..x_B, so a test can
    verify exactly the block another implementation drafted.
    ``uniform_fn(kind, position)`` (optional) replaces the Philox uniforms.
    ``top_p`` (optional) filters every sampled or verified row, p and q
    alike, with :func:`top_p_logits`; the StepResult keeps the raw logits.
    """
    if uniform_fn is None:
        def uniform_fn(kind, position):
            return float(uniform(seed, state.stream, position, kind))
    filt = (lambda l: l) if top_p is None else (lambda l: top_p_logits(l, top_p))
    c = state.c
    logits_d, kd, vd = draft_pass(model, state, B)
    if drafts is None:
        x = [sample_token(filt(logits_d[0]), uniform_fn(KIND_FIRST, c + 1))]
        for i in range(2, B + 1):
            x.append(sample_token(filt(logits_d[i]), uniform_fn(KIND_DRAFT, c + i)))
    else:
        x = [int(t) for t in drafts]
    cache = state.cache.copy()
    cache.append(kd, vd, [0])                      # pending token's K/V at position c
    logits_v, kv_k, kv_v = verify_pass(model, cache, c, x)

    # tested draft j (0-based) is x_{j+2} at position c+j+2
    p_rows = [filt(logits_v[j]) for j in range(B - 1)]   # p_{j+2} from verify row j
    q_rows = [filt(logits_d[j + 2]) for j in range(B - 1)]
    u_acc = [uniform_fn(KIND_ACCEPT, c + j + 2) for j in range(B - 1)]
    u_res = [uniform_fn(KIND_RESID, c + j + 2) for j in range(B)]
    n_acc, y, bits = verify_block(p_rows, q_rows, x[1:], u_acc, u_res, filt(logits_v[B - 1]))
    a = 1 + n_acc
    cache.append(kv_k, kv_v, range(a))             # positions c+1..c+a
    emitted = x[:a] + [y]
    new_state = DecodeState(state.tokens + emitted, cache, state.stream)
    res = StepResult(c, logits_d, logits_v, x, bits, a, y, emitted)
    return new_state, res


def ar_step(model, state, seed, uniform_fn=None, top_p=None):
    """AR-only decode: one row (pending, gate 0); emits one token (from the
    ``top_p`` nucleus when given)."""
    if uniform_fn is None:
        def uniform_fn(kind, position):
            return float(uniform(seed, state.stream, position, kind))
    c = state.c
    logits, k, v = model.forward(state.cache, [state.pending], [c], [0.0])
    row = logits[0] if top_p is None else top_p_logits(logits[0], top_p)
    y = sample_token(row, uniform_fn(KIND_FIRST, c + 1))
    cache = state.cache.copy()
    cache.append(k, v, [0])
    return DecodeState(state.tokens + [y], cache, state.stream), logits[0], y


# ---------------------------------------------------------------------------
# Tree sampler (Summary §方法关键点: the linear sampler serves system
# throughput, the tree sampler per-request throughput at batch 1; the
# Walkthrough's description of the two candidate-set modes is missing from
# the page).  Reading: the block's first token x_1 is drawn from the AR row
# as in the linear sampler; k chains then draft positions 2..B independently
# from the drafter's rows (chain j draws its token at position c+d with the
# DRAFT uniform of lane j, so chain 0 is the linear sampler's block).  The
# AR path verifies every chain [x_1, y_j2, ..., y_jB] in one verify pass (k B
# rows, each chain seeing the cache and its own earlier tokens).  The walk
# goes down the tree: at position 2 every chain's token is a candidate
# (chain order); at a later position the candidates are the continuing
# chain's token, then the other chains' tokens there (chain order), which,
# if accepted, end the block because no AR row conditions on them.  Each
# position is one recursive rejection (rrs_token) with the ACCEPT uniform of
# the candidate's lane and the RESID uniform of lane 0.  With k = 1 the tree
# sampler is the linear sampler, uniform for uniform.
# ---------------------------------------------------------------------------

class _Lazy:
    """Sequence whose item i is f(i), evaluated when read."""

    def __init__(self, f):
        self.f = f

    def __getitem__(self, i):
        return self.f(i)


def tree_walk(p_rows, q_rows, chains, c, uniform_fn):
    """The tree's verification walk.

    p_rows[j][i]: AR logits of position c+2+i given chain j's tokens up to
    depth i+1 (i = 0..B-1; row 0 is the same for every chain); q_rows[d]:
    drafter logits of position c+d (d = 2..B); chains[j] = [x_1, y_j2, ...,
    y_jB].  uniform_fn(kind, position, lane).
    Returns (path, last, jstar): the accepted tokens along the continuing
    chain (x_1 first), the final emitted token, and that chain (None when
    nothing past x_1 was accepted).
    """
    k, B = len(chains), len(chains[0])
    path, jstar = [chains[0][0]], None
    for d in range(2, B + 1):
        prow = p_rows[0][0] if d == 2 else p_rows[jstar][d - 2]
        order = list(range(k)) if d == 2 else [jstar] + [j for j in range(k) if j != jstar]
        cands = [chains[j][d - 1] for j in order]
        ua = _Lazy(lambda i, d=d, order=order: uniform_fn(KIND_ACCEPT, c + d, order[i]))
        idx, tok = rrs_token(prow, q_rows[d], cands, ua, lambda d=d: uniform_fn(KIND_RESID, c + d, 0))
        if idx is None:
            return path, tok, jstar
        j = order[idx]
        if d == 2 or j == jstar:
            jstar = j
            path.append(tok)
            continue
        return path, tok, jstar
    return path, sample_token(p_rows[jstar][B - 1], uniform_fn(KIND_RESID, c + B + 1, 0)), jstar


@dataclass
class TreeResult:
    c: int
    logits_draft: np.ndarray            # [B+1, V]
    logits_verify: list                 # per chain [B, V]
    chains: list                        # per chain [x_1, y_2, ..., y_B]
    path: list                          # accepted tokens along the continuing chain
    jstar: object                       # that chain, or None
    emitted: list = field(default_factory=list)


def tree_spec_step(model, state, B, k, seed, chains=None, uniform_fn=None):
    """One tree-sampler iteration; returns (new_state, TreeResult).

    ``chains`` (optional) replaces the drafted chains (each [x_1, y_2..y_B])
    so a test can verify exactly what another implementation drafted.
    """
    if uniform_fn is None:
        def uniform_fn(kind, position, lane=0):
            return float(uniform(seed, state.stream, position, kind, lane))
    c = state.c
    logits_d, kd, vd = draft_pass(model, state, B)
    if chains is None:
        x1 = sample_token(logits_d[0], uniform_fn(KIND_FIRST, c + 1, 0))
        chains = [[x1] + [sample_token(logits_d[d], uniform_fn(KIND_DRAFT, c + d, j))
                          for d in range(2, B + 1)] for j in range(k)]
    chains = [[int(t) for t in ch] for ch in chains]
    cache = state.cache.copy()
    cache.append(kd, vd, [0])                      # pending token's K/V at position c
    p_rows, kvs = [], []
    for ch in chains:
        lv, kk, vv = verify_pass(model, cache, c, ch)
        p_rows.append(lv)
        kvs.append((kk, vv))
    q_rows = {d: logits_d[d] for d in range(2, B + 1)}
    path, last, jstar = tree_walk(p_rows, q_rows, chains, c, uniform_fn)
    kk, vv = kvs[0 if jstar is None else jstar]
    cache.append(kk, vv, range(len(path)))         # positions c+1..c+len(path)
    emitted = path + [last]
    new_state = DecodeState(state.tokens + emitted, cache, state.stream)
    return new_state, TreeResult(c, logits_d, p_rows, chains, path, jstar, emitted)
