"""Pins of the oracle's Psi-Spec sampler (CPU only).

The sampler computes a sample, not a closed form, so it is pinned through its
distribution:

* the set of uniforms that yields each outcome of a sampler primitive is
  measured by bisection over u and compared with the closed-form probability;
* one whole iteration (B=2, V=16) is enumerated exactly over its uniforms and
  the distribution of the first two emitted tokens must equal the AR chain's
  p(t1) p(t2 | t1) to 1e-12 (speculative sampling is lossless);
* 10^6 Philox-driven iterations pass a chi-square test against the same law;
* closed forms: uniform logits, one-hot rows, q = p, q on a token with p = 0;
* the per-position accept rate equals 1 - TV(p, q);
* invariants: a in [1, B], 2 <= emitted <= B+1.
"""

import math
import os
from collections import defaultdict
from concurrent.futures import ProcessPoolExecutor
import multiprocessing as mp

import numpy as np
import pytest
from scipy import stats

from oracle import model as om
from oracle import psispec as ops
from oracle.philox import KIND_ACCEPT, KIND_DRAFT, KIND_FIRST, KIND_RESID, uniform

LO, HI = 2.0 ** -60, 1.0 - 2.0 ** -53


def outcome_measures(f, tol=2.0 ** -47, with_points=False):
    """Measure of {u in (0,1): f(u) = o} for a monotone step function f.

    With ``with_points`` also returns, per outcome, a uniform inside its
    interval (checked by evaluating f there).
    """
    flo, fhi = f(LO), f(HI)
    bps = []

    def refine(a, fa, b, fb):
        if fa == fb:
            return
        if b - a <= tol:
            bps.append((0.5 * (a + b), fa))
            return
        m = 0.5 * (a + b)
        fm = f(m)
        refine(a, fa, m, fm)
        refine(m, fm, b, fb)

    refine(LO, flo, HI, fhi)
    meas = defaultdict(float)
    points = {}
    prev = 0.0
    for u, left in bps + [(1.0, fhi)]:
        meas[left] += u - prev
        if with_points and left not in points:
            mid = 0.5 * (max(prev, LO) + min(u, HI))
            if f(mid) == left:
                points[left] = mid
        prev = u
    if with_points:
        return dict(meas), points
    return dict(meas)


def _softmax(l):
    e = np.exp(l - l.max())
    return e / e.sum()


def test_sample_token_measures_equal_softmax():
    rng = np.random.default_rng(0)
    for _ in range(5):
        l = rng.standard_normal(16) * 2
        meas = outcome_measures(lambda u: ops.sample_token(l, u))
        p = _softmax(l)
        got = np.array([meas.get(t, 0.0) for t in range(16)])
        np.testing.assert_allclose(got, p, atol=1e-12)


def test_accept_measure_equals_min_ratio():
    rng = np.random.default_rng(1)
    for _ in range(10):
        lp, lq = rng.standard_normal(16) * 2, rng.standard_normal(16) * 2
        t = int(rng.integers(16))
        meas = outcome_measures(lambda u: not ops.accept_draft(lp, lq, t, u))
        want = min(1.0, _softmax(lp)[t] / _softmax(lq)[t])
        assert abs(meas.get(False, 0.0) - want) < 1e-12


def test_residual_measures_equal_normalised_residual():
    rng = np.random.default_rng(2)
    for _ in range(5):
        lp, lq = rng.standard_normal(16) * 2, rng.standard_normal(16) * 2
        meas = outcome_measures(lambda u: ops.residual_token(lp, lq, u))
        r = np.maximum(_softmax(lp) - _softmax(lq), 0)
        got = np.array([meas.get(t, 0.0) for t in range(16)])
        np.testing.assert_allclose(got, r / r.sum(), atol=1e-12)


def test_uniform_logits_give_floor_u_v():
    V = 256
    l = np.zeros(V)
    rng = np.random.default_rng(3)
    us = list(rng.random(2000)) + [k / V for k in range(1, V)] + [2.0 ** -24, 1 - 2.0 ** -24]
    for u in us:
        assert ops.sample_token(l, u) == math.floor(u * V)


def test_one_hot_rows():
    l = np.full(16, -np.inf)
    l[11] = 0.0
    for u in (1e-7, 0.3, 0.999999):
        assert ops.sample_token(l, u) == 11
    # q one-hot on a token that p gives zero probability: always rejected, and
    # the residual max(0, p - q) is p itself
    lp = np.random.default_rng(4).standard_normal(16)
    lp[5] = -np.inf
    lq = np.full(16, -np.inf)
    lq[5] = 0.0
    for u in (1e-7, 0.5, 1 - 2.0 ** -24):
        assert not ops.accept_draft(lp, lq, 5, u)
    meas = outcome_measures(lambda u: ops.residual_token(lp, lq, u))
    got = np.array([meas.get(t, 0.0) for t in range(16)])
    np.testing.assert_allclose(got, _softmax(lp), atol=1e-12)


def test_q_equal_p_accepts_everything():
    rng = np.random.default_rng(5)
    B = 6
    rows = [rng.standard_normal(32) for _ in range(B)]
    drafts = [int(rng.integers(32)) for _ in range(B - 1)]
    ua = list(1 - 2.0 ** -24 - rng.random(B - 1) * 1e-3)
    n_acc, nxt, bits = ops.verify_block(rows[:-1], rows[:-1], drafts, ua, [0.5] * B, rows[-1])
    assert n_acc == B - 1 and all(bits)
    assert nxt == ops.sample_token(rows[-1], 0.5)


def test_residual_zero_mass_falls_back_to_p():
    l = np.random.default_rng(6).standard_normal(16)
    for u in (0.01, 0.5, 0.99):
        assert ops.residual_token(l, l, u) == ops.sample_token(l, u)


# ---------------------------------------------------------------------------
# A tiny model with V = 16 for whole-iteration checks.
# ---------------------------------------------------------------------------

def _tiny_v16(seed=0):
    shape = dict(n_layers=1, d_model=16, n_heads=2, n_kv_heads=1, head_dim=8, ffn_dim=24,
                 vocab=16, mask_id=15, rope_theta=1e4, rms_eps=1e-6, lora_rank=4,
                 lora_alpha=8.0, temperature=1.0)
    rng = np.random.default_rng(seed)
    p = {}
    for name, shp in om.param_names(shape):
        if name.endswith("norm"):
            p[name] = np.ones(shp)
        elif name in ("embed", "lm_head"):
            p[name] = 0.8 * rng.standard_normal(shp)
        elif name.endswith(".B"):
            p[name] = 0.3 * rng.standard_normal(shp)
        else:
            p[name] = 0.4 * rng.standard_normal(shp)
    return shape, p


class MemoModel(om.Model):
    """Caches forwards by their inputs (valid while the starting state is fixed)."""

    def __init__(self, shape, params):
        super().__init__(shape, params)
        self._memo = {}

    def forward(self, cache, tokens, positions, gates, noised=None, block=None):
        key = (len(cache), tuple(int(t) for t in tokens), tuple(int(x) for x in positions),
               tuple(float(g) for g in gates),
               None if noised is None else tuple(bool(x) for x in noised))
        if key not in self._memo:
            self._memo[key] = super().forward(cache, tokens, positions, gates, noised, block)
        return self._memo[key]


def _ar_two_token_law(m, state):
    """p(t1 | ctx) p(t2 | ctx, t1) from AR forwards of the oracle model."""
    V = m.shape["vocab"]
    c = state.c
    l1, k1, v1 = m.forward(state.cache, [state.pending], [c], [0.0])
    p1 = _softmax(l1[0])
    cache = state.cache.copy()
    cache.append(k1, v1, [0])
    law = np.zeros((V, V))
    for t1 in range(V):
        l2, _, _ = m.forward(cache, [t1], [c + 1], [0.0])
        law[t1] = p1[t1] * _softmax(l2[0])
    return law


def _enumerate_step(m, state, B):
    """Exact law of the emitted tokens of one spec_step, by DFS over uniforms."""
    leaves = defaultdict(float)

    def run(assign, probe_key=None, probe_u=None):
        requested = []

        def ufn(kind, pos):
            key = (kind, pos)
            requested.append(key)
            if key == probe_key:
                return probe_u
            return assign.get(key, 0.5)

        _, res = ops.spec_step(m, state, B, seed=0, uniform_fn=ufn)
        trace = (tuple(res.drafts), tuple(res.accept_bits), res.a, res.next_token)
        return requested, trace, res

    def dfs(assign, weight):
        requested, _, res = run(assign)
        free = [k for k in requested if k not in assign]
        if not free:
            leaves[tuple(res.emitted)] += weight
            return
        key = free[0]
        meas, points = outcome_measures(lambda u: run(assign, key, u)[1], with_points=True)
        for trace, w in meas.items():
            if w < 1e-14:
                continue
            dfs({**assign, key: points[trace]}, weight * w)

    dfs({}, 1.0)
    return leaves


def test_exact_enumeration_is_lossless():
    """Leviathan et al.'s theorem restated on the Walkthrough page: the tokens
    the iteration emits follow the AR chain exactly."""
    shape, p = _tiny_v16(0)
    m = MemoModel(shape, p)
    state = ops.prefill(m, [3, 9, 1, 4])
    B = 2
    leaves = _enumerate_step(m, state, B)
    V = shape["vocab"]
    law = np.zeros((V, V))
    total = 0.0
    for emitted, w in leaves.items():
        assert 2 <= len(emitted) <= B + 1
        law[emitted[0], emitted[1]] += w
        total += w
    assert abs(total - 1.0) < 1e-12
    want = _ar_two_token_law(m, state)
    assert np.max(np.abs(law - want)) < 1e-12
    # the drafter differs from the AR law, so rejections do happen
    assert any(len(e) == 2 for e in leaves) and any(len(e) == 3 for e in leaves)


def _chi_square_chunk(args):
    seed, start, count = args
    shape, p = _tiny_v16(0)
    m = MemoModel(shape, p)
    state = ops.prefill(m, [3, 9, 1, 4])
    c = state.c
    streams = np.arange(start, start + count, dtype=np.uint64)
    table = {}
    for kind, pos in ((KIND_FIRST, c + 1), (KIND_DRAFT, c + 2), (KIND_ACCEPT, c + 2),
                      (KIND_RESID, c + 2), (KIND_RESID, c + 3)):
        table[(kind, pos)] = uniform(seed, streams, pos, kind)
    counts = np.zeros((16, 16), np.int64)
    for i in range(count):
        _, res = ops.spec_step(m, state, 2, seed, uniform_fn=lambda k, q: float(table[(k, q)][i]))
        counts[res.emitted[0], res.emitted[1]] += 1
    return counts


def test_chi_square_one_million_steps():
    n, chunks = 1_000_000, 16
    per = n // chunks
    ctx = mp.get_context("spawn")
    with ProcessPoolExecutor(max_workers=min(8, os.cpu_count() or 1), mp_context=ctx) as ex:
        parts = list(ex.map(_chi_square_chunk, [(11, i * per, per) for i in range(chunks)]))
    counts = sum(parts)
    shape, p = _tiny_v16(0)
    m = om.Model(shape, p)
    state = ops.prefill(m, [3, 9, 1, 4])
    law = _ar_two_token_law(m, state).ravel()
    obs = counts.ravel()
    keep = law * n >= 5
    exp_ = law[keep] * n
    chi2 = float(np.sum((obs[keep] - exp_) ** 2 / exp_))
    # cells with expectation < 5 are pooled into one
    rest_o, rest_e = obs[~keep].sum(), law[~keep].sum() * n
    dof = int(keep.sum()) - 1
    if rest_e > 0:
        chi2 += (rest_o - rest_e) ** 2 / rest_e
        dof += 1
    pval = stats.chi2.sf(chi2, dof)
    assert pval > 0.01, (chi2, dof, pval)


def test_accept_rate_equals_one_minus_tv():
    """Per-position acceptance of a draft from q is sum_v min(p_v, q_v)."""
    rng = np.random.default_rng(8)
    lp, lq = rng.standard_normal(64) * 1.5, rng.standard_normal(64) * 1.5
    p, q = _softmax(lp), _softmax(lq)
    want = np.minimum(p, q).sum()
    n = 20000
    streams = np.arange(n, dtype=np.uint64)
    u_draft = uniform(5, streams, 0, KIND_DRAFT)
    u_acc = uniform(5, streams, 0, KIND_ACCEPT)
    acc = 0
    for i in range(n):
        t = ops.sample_token(lq, float(u_draft[i]))
        acc += ops.accept_draft(lp, lq, t, float(u_acc[i]))
    rate = acc / n
    assert abs(rate - want) < 5 * math.sqrt(want * (1 - want) / n)


def test_step_invariants_over_a_generation():
    shape, p = _tiny_v16(1)
    m = om.Model(shape, p)
    B = 4
    state = ops.prefill(m, [1, 2, 3, 4, 5, 6])
    for step in range(12):
        c0, n0 = state.c, len(state.tokens)
        state, res = ops.spec_step(m, state, B, seed=3)
        assert 1 <= res.a <= B
        assert len(res.emitted) == res.a + 1
        assert 2 <= len(res.emitted) <= B + 1
        assert res.emitted[0] == res.drafts[0]                 # first token always kept
        assert state.c == c0 + res.a + 1
        assert len(state.tokens) == n0 + res.a + 1
        assert state.pending == res.next_token
        # accept bits before the first rejection are all True
        assert all(res.accept_bits[: res.a - 1])
        if res.a < B:
            assert not res.accept_bits[res.a - 1]


# ---------------------------------------------------------------------------
# top-p (nucleus) filtering.
# ---------------------------------------------------------------------------

def _filtered_probs(logits, top_p):
    f = ops.top_p_logits(np.asarray(logits, dtype=np.float64), top_p)
    e = np.exp(f - np.max(f))
    return e / e.sum()


def test_top_p_fixtures():
    """Hand-computed nuclei on exact binary fractions (cumulative sums away
    from the thresholds): the token that crosses top_p is kept, ties go by
    token id, top_p >= 1 keeps everything, a tiny top_p is greedy."""
    l = np.log([0.5, 0.25, 0.125, 0.125])
    np.testing.assert_allclose(_filtered_probs(l, 0.4), [1, 0, 0, 0], atol=1e-15)
    np.testing.assert_allclose(_filtered_probs(l, 0.7), [2 / 3, 1 / 3, 0, 0], rtol=1e-13)
    np.testing.assert_allclose(_filtered_probs(l, 0.8), [4 / 7, 2 / 7, 1 / 7, 0], rtol=1e-13)
    np.testing.assert_array_equal(ops.top_p_logits(l, 1.0), l)
    # ties: the most probable tokens 1, 2, 3 share 0.3; two of them (by id) reach 0.5
    lt = np.log([0.1, 0.3, 0.3, 0.3])
    np.testing.assert_allclose(_filtered_probs(lt, 0.5), [0, 0.5, 0.5, 0], atol=1e-15)
    rng = np.random.default_rng(3)
    for _ in range(20):
        z = rng.standard_normal(50) * 3
        g = _filtered_probs(z, 1e-9)
        assert g[np.argmax(z)] == 1.0 and np.count_nonzero(g) == 1


def test_top_p_nucleus_is_minimal():
    """On random rows: the kept mass reaches top_p, dropping the least
    probable kept token falls below it, and no dropped token is more
    probable than a kept one."""
    rng = np.random.default_rng(4)
    for trial in range(50):
        z = rng.standard_normal(200) * (0.5 + trial / 10)
        top_p = float(rng.uniform(0.05, 0.99))
        p = _softmax(z)
        kept = np.isfinite(ops.top_p_logits(z, top_p))
        assert p[kept].sum() >= top_p
        assert p[kept].sum() - p[kept].min() < top_p
        if (~kept).any():
            assert p[~kept].max() <= p[kept].min()


def test_top_p_one_leaves_the_iteration_unchanged():
    shape, prm = _tiny_v16(2)
    m = MemoModel(shape, prm)
    st = ops.prefill(m, [2, 7, 11])
    for _ in range(4):
        n1, r1 = ops.spec_step(m, st, 3, seed=5)
        n2, r2 = ops.spec_step(m, st, 3, seed=5, top_p=1.0)
        assert r1.emitted == r2.emitted and r1.accept_bits == r2.accept_bits
        st = n1


def test_top_p_enumeration_is_lossless():
    """With p and q filtered alike (top-p 0.9), one iteration's first two
    emitted tokens follow the filtered AR chain p'(t1) p'(t2 | t1) exactly."""
    shape, prm = _tiny_v16(0)
    m = MemoModel(shape, prm)
    state = ops.prefill(m, [3, 9, 1, 4])
    B, V, top_p = 2, shape["vocab"], 0.9
    leaves = defaultdict(float)

    def run(assign, probe_key=None, probe_u=None):
        requested = []

        def ufn(kind, pos):
            key = (kind, pos)
            requested.append(key)
            if key == probe_key:
                return probe_u
            return assign.get(key, 0.5)

        _, res = ops.spec_step(m, state, B, seed=0, uniform_fn=ufn, top_p=top_p)
        return requested, (tuple(res.drafts), tuple(res.accept_bits), res.a, res.next_token), res

    def dfs(assign, weight):
        requested, _, res = run(assign)
        free = [k for k in requested if k not in assign]
        if not free:
            leaves[tuple(res.emitted)] += weight
            return
        key = free[0]
        meas, points = outcome_measures(lambda u: run(assign, key, u)[1], with_points=True)
        for trace, w in meas.items():
            if w >= 1e-14:
                dfs({**assign, key: points[trace]}, weight * w)

    dfs({}, 1.0)
    law = np.zeros((V, V))
    for emitted, w in leaves.items():
        law[emitted[0], emitted[1]] += w
    assert abs(law.sum() - 1.0) < 1e-12
    c = state.c
    l1, k1, v1 = m.forward(state.cache, [state.pending], [c], [0.0])
    p1 = _filtered_probs(l1[0], top_p)
    cache = state.cache.copy()
    cache.append(k1, v1, [0])
    want = np.zeros((V, V))
    for t1 in range(V):
        if p1[t1] > 0:
            l2, _, _ = m.forward(cache, [t1], [c + 1], [0.0])
            want[t1] = p1[t1] * _filtered_probs(l2[0], top_p)
    assert np.max(np.abs(law - want)) < 1e-12
    # the filter removes tokens: some outcomes have zero probability
    assert np.count_nonzero(want) < V * V


def test_top_p_with_masked_logits():
    """Rows that already hold -inf (tokens with no mass): they are never
    kept, and a row with one finite logit keeps exactly that token."""
    z = np.array([0.3, -np.inf, 1.2, -np.inf, -0.5])
    kept = np.isfinite(ops.top_p_logits(z, 0.99))
    assert not kept[1] and not kept[3] and kept[2]
    one = np.array([-np.inf, -np.inf, 0.7, -np.inf])
    np.testing.assert_array_equal(np.isfinite(ops.top_p_logits(one, 0.5)), [False, False, True, False])
    np.testing.assert_allclose(_filtered_probs(one, 0.95), [0, 0, 1, 0])
