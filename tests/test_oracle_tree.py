"""Pins of the oracle's tree sampler (CPU only).

Reading (the Walkthrough's list of the two candidate-set modes is missing
from the page; Summary §方法关键点 names a tree sampler for per-request
throughput): k chains drafted independently from the drafter share the AR
first token; the walk applies recursive rejection over the candidates of
each position.  Pinned by:

* the recursive rejection's output law equals p exactly: an analytic sum
  over all candidate tuples (k = 1..3), and the oracle's own sample paths
  measured by bisection over their uniforms (k = 2);
* k = 1 reproduces the linear sampler token for token (same uniforms);
* the whole walk (B = 3, k = 2, abstract conditionals over V = 3) enumerated
  exactly over drafts and uniforms: the first three tokens follow the AR
  chain to 1e-12 (every emitted sequence extended to B + 1 tokens by the
  AR chain);
* the reading's candidate order (the continuing chain's token first) in a
  closed form where another order would end the block earlier;
* invariants on the model: 2 <= emitted <= B+1, and the committed cache
  equals a recompute of the emitted prefix.
"""

import itertools
import math
from collections import defaultdict

import numpy as np

from oracle import model as om
from oracle import psispec as ops
from oracle.philox import KIND_ACCEPT, KIND_DRAFT, KIND_FIRST, KIND_RESID, uniform

from test_oracle_sampler import MemoModel, _softmax, _tiny_v16, outcome_measures


def test_lane_zero_is_the_linear_uniform():
    pos = np.arange(100)
    np.testing.assert_array_equal(uniform(5, 3, pos, KIND_ACCEPT, 0), uniform(5, 3, pos, KIND_ACCEPT))
    assert np.all(uniform(5, 3, pos, KIND_ACCEPT, 1) != uniform(5, 3, pos, KIND_ACCEPT, 0))


def _rrs_law(p, q, k):
    """Output law of recursive rejection with k i.i.d. candidates from q,
    summed over every candidate tuple (the mathematics, written out)."""
    V = p.size
    out = np.zeros(V)
    for tup in itertools.product(range(V), repeat=k):
        w = float(np.prod([q[y] for y in tup]))
        if w == 0.0:
            continue
        r, reach = p.copy(), 1.0
        for y in tup:
            a = min(1.0, r[y] / q[y])
            out[y] += w * reach * a
            reach *= 1.0 - a
            res = np.maximum(r - q, 0.0)
            if res.sum() > 0:
                r = res / res.sum()
        out += w * reach * r
    return out


def test_rrs_law_is_p():
    rng = np.random.default_rng(0)
    for _ in range(4):
        lp, lq = rng.standard_normal(6) * 1.5, rng.standard_normal(6) * 1.5
        p, q = _softmax(lp), _softmax(lq)
        for k in (1, 2, 3):
            np.testing.assert_allclose(_rrs_law(p, q, k), p, atol=1e-12)


def _rrs_sampled_law(lp, lq, k):
    """Law of the oracle's rrs_token over its uniforms (bisection), summed
    over candidate tuples weighted by q."""
    q = _softmax(lq)
    V = lq.size
    out = np.zeros(V)
    for tup in itertools.product(range(V), repeat=k):
        w = float(np.prod([q[y] for y in tup]))
        def dfs(fixed, weight):
            # uniforms in the order rrs_token consumes them: accept tests, then the residual
            i = len(fixed)
            if i == k + 1:
                _, tok = ops.rrs_token(lp, lq, tup, fixed[:k], fixed[k])
                out[tok] += weight
                return
            def f(u):
                us = list(fixed) + [u] + [0.5] * (k - i)
                j, tok = ops.rrs_token(lp, lq, tup, us[:k], us[k])
                # accept tests: the outcome is where the walk stopped; the draw: the token
                return (j if (j is not None and j <= i) else None, tok if i == k or (j is not None and j <= i) else -1)
            meas, pts = outcome_measures(f, with_points=True)
            for o, m in meas.items():
                if m < 1e-15:
                    continue
                if o[0] is not None:              # accepted at test i: the token is final
                    out[o[1]] += weight * m
                elif i == k:                      # residual draw
                    out[o[1]] += weight * m
                else:
                    dfs(list(fixed) + [pts[o]], weight * m)
        dfs([], w)
    return out


def test_rrs_sampled_law_is_p():
    rng = np.random.default_rng(1)
    for _ in range(2):
        lp, lq = rng.standard_normal(5) * 1.5, rng.standard_normal(5) * 1.5
        np.testing.assert_allclose(_rrs_sampled_law(lp, lq, 2), _softmax(lp), atol=1e-12)


def test_tree_with_one_chain_is_the_linear_sampler():
    shape, p = _tiny_v16(0)
    m = om.Model(shape, p)
    rng = np.random.default_rng(2)
    for trial in range(12):
        prompt = [int(t) for t in rng.integers(0, 15, 4 + trial % 3)]
        st = ops.prefill(m, prompt, stream=trial)
        for B in (2, 4):
            seed = 100 + trial
            lin_state, lin = ops.spec_step(m, st, B, seed)
            tree_state, tree = ops.tree_spec_step(m, st, B, 1, seed)
            assert tree.emitted == lin.emitted, (trial, B)
            for l in range(shape["n_layers"]):
                np.testing.assert_array_equal(tree_state.cache.k[l], lin_state.cache.k[l])
                np.testing.assert_array_equal(tree_state.cache.v[l], lin_state.cache.v[l])


def _abstract(V, seed):
    rng = np.random.default_rng(seed)
    memo = {}
    def p_fn(prefix):
        key = tuple(prefix)
        if key not in memo:
            memo[key] = rng.standard_normal(V) * 1.2
        return memo[key]
    return p_fn


def test_tree_walk_exact_enumeration_is_lossless():
    V, B, k = 3, 3, 2
    p_fn = _abstract(V, 7)
    rng = np.random.default_rng(8)
    q_rows = {d: rng.standard_normal(V) * 1.2 for d in range(2, B + 1)}
    c = 10
    law = defaultdict(float)
    p1 = _softmax(p_fn(()))
    qs = {d: _softmax(q_rows[d]) for d in q_rows}
    for x1 in range(V):
        for ys in itertools.product(range(V), repeat=k * (B - 1)):
            chains = [[x1] + list(ys[j * (B - 1):(j + 1) * (B - 1)]) for j in range(k)]
            w = p1[x1] * float(np.prod([qs[d + 2][chains[j][d + 1]]
                                        for j in range(k) for d in range(B - 1)]))
            p_rows = [[p_fn(ch[: i + 1]) for i in range(B)] for ch in chains]

            def dfs(assign, weight):
                requested = []
                def ufn(kind, pos, lane, probe=None):
                    key = (kind, pos, lane)
                    requested.append(key)
                    if probe is not None and key == probe[0]:
                        return probe[1]
                    return assign.get(key, 0.5)
                path, last, _ = ops.tree_walk(p_rows, q_rows, chains, c, ufn)
                free = [key for key in requested if key not in assign]
                if not free:
                    law[tuple(path + [last])] += weight
                    return
                key = free[0]
                def f(u):
                    req2 = []
                    def ufn2(kind, pos, lane):
                        kk = (kind, pos, lane)
                        req2.append(kk)
                        if kk == key:
                            return u
                        return assign.get(kk, 0.5)
                    path2, last2, _ = ops.tree_walk(p_rows, q_rows, chains, c, ufn2)
                    # outcome of this uniform: the walk's result if it ends without
                    # another free uniform, else the set of uniforms it goes on to
                    later = tuple(kk for kk in req2 if kk not in assign and kk != key)
                    return (tuple(path2 + [last2]) if not later else None, later)
                meas, pts = outcome_measures(f, with_points=True)
                for o, mm in meas.items():
                    if mm < 1e-15:
                        continue
                    dfs({**assign, key: pts[o]}, weight * mm)

            dfs({}, w)
    total = sum(law.values())
    assert abs(total - 1.0) < 1e-12
    # every emitted sequence extended to B + 1 tokens by the AR chain
    full = dict(law)
    for n in range(2, B + 1):
        ext = defaultdict(float)
        for seq, w in full.items():
            if len(seq) > n:
                ext[seq] += w
            else:
                pn = _softmax(p_fn(seq))
                for t in range(V):
                    ext[seq + (t,)] += w * pn[t]
        full = ext
    for seq in itertools.product(range(V), repeat=B + 1):
        want = 1.0
        for i in range(B + 1):
            want *= _softmax(p_fn(seq[:i]))[seq[i]]
        assert abs(full.get(seq, 0.0) - want) < 1e-12, seq


def test_tree_step_invariants_and_commit():
    shape, p = _tiny_v16(1)
    m = om.Model(shape, p)
    st = ops.prefill(m, [2, 7, 11, 5])
    for step in range(6):
        new, res = ops.tree_spec_step(m, st, 4, 3, 40 + step)
        assert 2 <= len(res.emitted) <= 5
        assert res.emitted[: len(res.path)] == res.path
        # the committed cache is what a plain recompute of the tokens gives
        full, k, v = m.forward(om.KVCache(shape), new.tokens[:-1], np.arange(new.c), np.zeros(new.c))
        for l in range(shape["n_layers"]):
            np.testing.assert_allclose(new.cache.k[l], k[l], rtol=1e-10, atol=1e-12)
        st = new


def test_continuing_chain_is_tried_first():
    """p = q at position 3 (every test passes): after chain 1 won position 2,
    its own token is tested first at position 3 and accepted, so the block
    goes on to the bonus token (B + 1 = 4 tokens).  At position 2, chain 0's
    token has p = 0 (always rejected) and chain 1's token is the only one the
    residual keeps (ratio >= 1)."""
    V, c = 4, 20
    p2 = np.array([-np.inf, 0.0, -np.inf, -np.inf])      # position 2: all mass on token 1
    q2 = np.array([0.0, 0.0, 0.0, 0.0])                  # drafter: uniform
    p3 = np.array([0.3, -0.2, 0.5, 0.1])
    chains = [[2, 0, 3], [2, 1, 0]]
    p_rows = [[p2, p3, np.zeros(V)], [p2, p3, np.zeros(V)]]
    q_rows = {2: q2, 3: p3}
    path, last, jstar = ops.tree_walk(p_rows, q_rows, chains, c, lambda kind, pos, lane: 0.5)
    assert jstar == 1 and path == [2, 1, 0], (path, last, jstar)
