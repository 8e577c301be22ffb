"""Nucleus (top-p) sampling on the GPU against the oracle (GPU).

The oracle's filter (oracle.psispec.top_p_logits; Walkthrough §我的判断: the
lossless claim holds for the sampling distribution of temperature 1 and
top-p 0.95) keeps the smallest set of most probable tokens whose probability
reaches top_p, ties by token id.  The GPU computes each row's nucleus with
exact fixed-point mass sums from fp32 weights, so the two kept sets can
differ only where a cumulative probability lies within rounding of top_p:
every difference is traced to such a near-tie (|cum - top_p| < 1e-5) and
counted.  Then every sampling decision is checked against the oracle's
sampler on the filtered rows, and in fp32 mode the emitted tokens against
the oracle's own iteration at the same top_p.
"""

import numpy as np
import pytest
import torch

from lossless_diffusion_draft_b200 import synth, uno
from oracle import model as om
from oracle import psispec as ops

import parity
from test_gpu_model import _kv_check, _setup

pytestmark = pytest.mark.gpu

NUC_TOL = 1e-5


def _keys(logits_f32):
    u = np.ascontiguousarray(logits_f32, dtype=np.float32).view(np.uint32).copy()
    u[u == 0x80000000] = 0
    return np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)


def gpu_kept(logits_f32, entry):
    key = np.uint32(int(entry[0]) & 0xFFFFFFFF)
    k = _keys(logits_f32)
    v = np.arange(k.size)
    return (k > key) | ((k == key) & (v <= int(entry[1])))


def check_nucleus(logits_f32, entry, top_p, tally, what=""):
    """GPU kept set (from its (key, id_cut) entry) against the oracle's.
    Returns True when they are equal."""
    kept = gpu_kept(logits_f32, entry)
    l = np.asarray(logits_f32, np.float64)
    want = np.isfinite(ops.top_p_logits(l, top_p)) & np.isfinite(l)
    if np.array_equal(kept, want):
        tally.add(True)
        return True
    p = np.exp(ops.log_softmax(l))
    order = np.lexsort((np.arange(p.size), -p))
    n_g, n_o = int(kept.sum()), int(want.sum())
    # the GPU's set is a prefix of the same order (probability, then id)
    assert set(order[:n_g].tolist()) == set(np.nonzero(kept)[0].tolist()), what
    cum = np.cumsum(p[order])
    lo, hi = min(n_g, n_o) - 1, max(n_g, n_o) - 1
    m = float(np.max(np.abs(cum[lo:hi] - top_p)))
    assert m < NUC_TOL, f"{what}: GPU keeps {n_g}, oracle {n_o}, margin {m:.3e}"
    tally.add(False, (what, n_g, n_o, m))
    return False


def _filter(rows, top_p):
    rows_d = torch.from_numpy(np.ascontiguousarray(rows, dtype=np.float32)).cuda()
    out = torch.full((rows.shape[0], 2), -7, dtype=torch.int32, device="cuda")
    uno.uno_top_p_filter(rows_d, top_p, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("V", [256, 32000, 151936])
@pytest.mark.parametrize("top_p", [0.3, 0.9, 0.95, 0.999])
def test_filter_random_rows(V, top_p):
    rng = np.random.default_rng(V + int(top_p * 1000))
    rows = np.concatenate([rng.standard_normal((6, V)) * 3.0, rng.standard_normal((4, V)) * 0.3])
    ent = _filter(rows, top_p)
    tally = parity.Tally()
    for i in range(rows.shape[0]):
        check_nucleus(rows[i].astype(np.float32), ent[i], top_p, tally, f"row {i}")
    assert tally.mismatches <= 1, tally.notes


def test_filter_special_rows():
    """Closed forms: all-equal logits keep the first ceil(top_p V) tokens by
    id (the ties are broken by id); a one-hot-like row keeps its peak; -inf
    entries are never kept; a row with its mass in a few tied tokens keeps
    the right count of them."""
    V = 4096
    rows = []
    rows.append(np.zeros(V))                                  # all equal
    r = np.full(V, -5.0); r[1234] = 30.0; rows.append(r)      # one dominant token
    r = np.random.default_rng(1).standard_normal(V); r[::3] = -np.inf; rows.append(r)
    r = np.full(V, -40.0); r[[7, 100, 2000, 4000]] = 3.0; rows.append(r)   # four tied peaks
    r = np.random.default_rng(2).standard_normal(V); r[5] = -0.0; r[6] = 0.0; rows.append(r)
    rows = np.stack(rows).astype(np.float32)
    # top_p values whose crossing is not an exact tie of a cumulative sum
    for top_p in (0.4, 0.95):
        ent = _filter(rows, top_p)
        tally = parity.Tally()
        for i in range(rows.shape[0]):
            assert check_nucleus(rows[i], ent[i], top_p, tally, f"row {i}"), (i, top_p)
        kept0 = gpu_kept(rows[0], ent[0])
        n = int(np.ceil(top_p * V))
        assert kept0[:n].all() and not kept0[n:].any()
        assert np.nonzero(gpu_kept(rows[1], ent[1]))[0].tolist() == [1234]
        assert not gpu_kept(rows[2], ent[2])[::3].any()
        want3 = [7, 100] if top_p == 0.4 else [7, 100, 2000, 4000]
        assert np.nonzero(gpu_kept(rows[3], ent[3]))[0].tolist() == want3


def test_filter_is_deterministic():
    rng = np.random.default_rng(5)
    rows = rng.standard_normal((64, 151936)) * 2.0
    a = _filter(rows, 0.95)
    b = _filter(rows, 0.95)
    assert np.array_equal(a, b)


def _run_top_p(name, n_req, prompt_len, n_steps, top_p, logit_tol, end_to_end, **over):
    cfg, ctx, ids, model, states = _setup(name, n_req, prompt_len,
                                          prompt_len + (n_steps + 1) * 20, **over)
    uno.uno_set_top_p(ctx, top_p)
    B, V, seed = cfg["B"], cfg["vocab"], cfg["seed"]
    req = torch.tensor(ids, dtype=torch.int32, device="cuda")
    out = torch.zeros((n_req, B + 1), dtype=torch.int32, device="cuda")
    n_new = torch.zeros(n_req, dtype=torch.int32, device="cuda")
    nuc, tally, e2e = parity.Tally(), parity.Tally(), parity.Tally()
    for step in range(n_steps):
        uno.uno_spec_step(ctx, req, out, n_new)
        uno.uno_status(ctx)
        ld = uno.uno_debug_read(ctx, uno.UNO_DBG_LOGITS_DRAFT, torch.empty((n_req, B + 1, V)))
        lv = uno.uno_debug_read(ctx, uno.UNO_DBG_LOGITS_VERIFY, torch.empty((n_req, B, V)))
        dr = uno.uno_debug_read(ctx, uno.UNO_DBG_DRAFTS, torch.empty((n_req, B), dtype=torch.int32))
        fd = uno.uno_debug_read(ctx, uno.UNO_DBG_TOPP_DRAFT,
                                torch.empty((n_req, B + 1, 2), dtype=torch.int32)).numpy()
        fv = uno.uno_debug_read(ctx, uno.UNO_DBG_TOPP_VERIFY,
                                torch.empty((n_req, B, 2), dtype=torch.int32)).numpy()
        o, nn = out.cpu().numpy(), n_new.cpu().numpy()
        for i in range(n_req):
            st = states[i]
            drafts = [int(t) for t in dr[i]]
            emitted = [int(t) for t in o[i, : nn[i]]]
            assert 2 <= nn[i] <= B + 1
            new_st, res = ops.spec_step(model, st, B, seed, drafts=drafts, top_p=top_p)
            assert np.max(np.abs(ld[i].double().numpy() - res.logits_draft)) <= logit_tol
            assert np.max(np.abs(lv[i].double().numpy() - res.logits_verify)) <= logit_tol
            ldn, lvn = ld[i].numpy(), lv[i].numpy()
            same = all(check_nucleus(ldn[r], fd[i, r], top_p, nuc, f"step {step} req {i} d{r}")
                       for r in [0] + list(range(2, B + 1)))
            same = all([check_nucleus(lvn[r], fv[i, r], top_p, nuc, f"step {step} req {i} v{r}")
                        for r in range(B)]) and same
            # every drafted token lies in the GPU's nucleus of its row
            assert gpu_kept(ldn[0], fd[i, 0])[drafts[0]]
            for r in range(2, B + 1):
                assert gpu_kept(ldn[r], fd[i, r])[drafts[r - 1]]
            if same:
                # decisions on the oracle-filtered GPU logits
                ldf = np.stack([ops.top_p_logits(ldn[r].astype(np.float64), top_p)
                                for r in range(B + 1)])
                lvf = np.stack([ops.top_p_logits(lvn[r].astype(np.float64), top_p)
                                for r in range(B)])
                parity.check_step_sampling(ldf, lvf, drafts, emitted, st.c, B, seed, st.stream,
                                           tally, f"step {step} req {i}")
            if end_to_end:
                _, own = ops.spec_step(model, st, B, seed, top_p=top_p)
                e2e.add(own.emitted == emitted, (step, i, own.emitted, emitted))
            if res.emitted == emitted:
                states[i] = new_st
            else:
                states[i] = ops.prefill(model, st.tokens + emitted, stream=st.stream)
            c_gpu, pend = uno.uno_request_state(ctx, ids[i])
            assert c_gpu == states[i].c and pend == states[i].pending
    for i in range(n_req):
        _kv_check(ctx, cfg, model, states[i], ids[i], logit_tol)
    ctx.close()
    return nuc, tally, e2e


def test_tiny_fp32_top_p_095():
    """The pages' setting, top-p 0.95, on the tiny fp32 model: kept sets and
    decisions match the oracle (near-ties traced), and the emitted tokens
    equal the oracle's own iteration at top-p 0.95."""
    nuc, tally, e2e = _run_top_p("tiny", 2, 32, 12, 0.95, 1e-4, True)
    assert nuc.mismatches <= parity.near_tie_budget(nuc.positions), nuc.notes
    assert tally.mismatches <= parity.near_tie_budget(tally.positions), tally.notes
    assert e2e.mismatches <= tally.mismatches + nuc.mismatches, e2e.notes


def test_small_bf16_top_p_09():
    """A bf16 model at top-p 0.9: the nucleus of every row and every decision
    against the oracle on the GPU's logits."""
    nuc, tally, _ = _run_top_p("small", 2, 24, 3, 0.9, 2e-2, False, n_layers=2)
    assert nuc.mismatches <= parity.near_tie_budget(nuc.positions), nuc.notes
    assert tally.mismatches <= parity.near_tie_budget(tally.positions), tally.notes


def test_top_p_ar_step_and_switch_off():
    """uno_ar_step draws from the filtered AR row; top_p = 1 turns the filter
    off again (the next step samples the full distribution)."""
    cfg, ctx, ids, model, states = _setup("tiny", 1, 20, 100)
    uno.uno_set_top_p(ctx, 0.8)
    st = states[0]
    req = torch.tensor(ids, dtype=torch.int32, device="cuda")
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    tally, nuc = parity.Tally(), parity.Tally()
    for _ in range(8):
        uno.uno_ar_step(ctx, req, out)
        la = uno.uno_debug_read(ctx, uno.UNO_DBG_LOGITS_AR, torch.empty((1, cfg["vocab"])))[0].numpy()
        fa = uno.uno_debug_read(ctx, uno.UNO_DBG_TOPP_DRAFT, torch.empty((1, 1, 2), dtype=torch.int32)).numpy()
        t = int(out[0])
        assert gpu_kept(la, fa[0, 0])[t]
        check_nucleus(la, fa[0, 0], 0.8, nuc)
        u = float(parity.uniforms(cfg["seed"], st.stream, st.c, cfg["B"])["first"])
        parity.check_sample(ops.top_p_logits(la.astype(np.float64), 0.8), u, t, tally)
        new_st, _, y = ops.ar_step(model, st, cfg["seed"], top_p=0.8)
        st = new_st if y == t else ops.prefill(model, st.tokens + [t], stream=st.stream)
    assert tally.mismatches <= 1 and nuc.mismatches <= 1
    uno.uno_set_top_p(ctx, 1.0)
    uno.uno_ar_step(ctx, req, out)
    uno.uno_status(ctx)
    with pytest.raises(uno.UnoError):
        uno.uno_set_top_p(ctx, 0.0)
    ctx.close()
