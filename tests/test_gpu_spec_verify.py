"""spec_verify kernel vs the oracle's rejection rule (GPU).

Same fp32 logits, same drafted tokens, same Philox uniforms on both sides;
decisions must agree except at traced fp32 near-ties.
"""

import numpy as np
import pytest
import torch

from lossless_diffusion_draft_b200 import synth, uno
from oracle import psispec as ops
from oracle.philox import KIND_ACCEPT, KIND_DRAFT, KIND_RESID, uniform

import parity

pytestmark = pytest.mark.gpu
SEED = 7


def _run_gpu(p, q, drafts, streams, pos0, seed=SEED):
    n_req, n_tests, V = p.shape
    dev = "cuda"
    ws = torch.zeros(uno.uno_spec_verify_workspace_bytes(n_req, n_tests, V), dtype=torch.uint8,
                     device=dev)
    out = torch.full((n_req, n_tests + 1), -1, dtype=torch.int32, device=dev)
    n_out = torch.zeros(n_req, dtype=torch.int32, device=dev)
    uno.uno_spec_verify(p, q, drafts, seed, streams, pos0, out, n_out, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy(), n_out.cpu().numpy(), ws


def _check_request(p_np, q_np, d_np, stream, pos0, out_row, n_out, tally, seed=SEED):
    n_tests = p_np.shape[0]
    u_acc = [float(uniform(seed, stream, pos0 + j, KIND_ACCEPT)) for j in range(n_tests)]
    u_res = [float(uniform(seed, stream, pos0 + j, KIND_RESID)) for j in range(n_tests + 1)]
    a = n_out                                   # accepted prefix length
    assert 0 <= a <= n_tests
    assert list(out_row[:a]) == list(d_np[:a])
    y = int(out_row[a]) if a < n_tests else None
    if a == n_tests:
        assert out_row[a] == -1
    parity.check_verify(list(p_np), list(q_np), list(d_np), u_acc, u_res, None, a, y, tally,
                        f"stream {stream}")


def _make(n_req, n_tests, V, seed=0):
    g = torch.Generator().manual_seed(seed)
    p = torch.randn((n_req, n_tests, V), generator=g) * 3
    q = p + torch.randn((n_req, n_tests, V), generator=g) * 0.5
    streams = np.arange(n_req, dtype=np.uint32) + 100
    pos0 = (np.arange(n_req, dtype=np.int32) * 37) % 5000
    drafts = np.zeros((n_req, n_tests), np.int32)
    qn = q.double().numpy()
    for i in range(n_req):
        for j in range(n_tests):
            u = float(uniform(SEED, int(streams[i]), int(pos0[i]) + j, KIND_DRAFT))
            drafts[i, j] = ops.sample_token(qn[i, j], u)
    return p, q, drafts, streams, pos0


# the last case has more (row, chunk) CTAs than the fused form takes: the
# split reduce / decide kernels run
@pytest.mark.parametrize("n_req,n_tests,V", [(1, 1, 16), (7, 16, 1000), (33, 5, 8196),
                                             (16, 16, 20004), (3, 16, 151936), (40, 16, 65536)])
def test_spec_verify_matches_oracle(n_req, n_tests, V):
    p, q, drafts, streams, pos0 = _make(n_req, n_tests, V)
    out, n_out, ws = _run_gpu(p.cuda(), q.cuda(), torch.from_numpy(drafts).cuda(),
                              torch.from_numpy(streams.view(np.int32)).cuda(),
                              torch.from_numpy(pos0).cuda())
    tally = parity.Tally()
    pn, qn = p.double().numpy(), q.double().numpy()
    for i in range(n_req):
        _check_request(pn[i], qn[i], drafts[i], int(streams[i]), int(pos0[i]), out[i], int(n_out[i]), tally)
    assert tally.mismatches <= parity.near_tie_budget(tally.positions), tally.notes


def test_counters_left_zero_and_repeatable():
    p, q, drafts, streams, pos0 = _make(9, 8, 4100, seed=3)
    args = (p.cuda(), q.cuda(), torch.from_numpy(drafts).cuda(),
            torch.from_numpy(streams.view(np.int32)).cuda(), torch.from_numpy(pos0).cuda())
    n_req, n_tests, V = p.shape
    ws = torch.zeros(uno.uno_spec_verify_workspace_bytes(n_req, n_tests, V), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        out = torch.full((n_req, n_tests + 1), -1, dtype=torch.int32, device="cuda")
        n_out = torch.zeros(n_req, dtype=torch.int32, device="cuda")
        uno.uno_spec_verify(*args[:3], SEED, args[3], args[4], out, n_out, ws)
        torch.cuda.synchronize()
        outs.append((out.cpu().numpy(), n_out.cpu().numpy()))
        # the counter region (first 256-aligned block) is left zeroed
        assert int(ws[: n_req * 2 * n_tests * 4].count_nonzero()) == 0
    for o in outs[1:]:
        np.testing.assert_array_equal(o[0], outs[0][0])
        np.testing.assert_array_equal(o[1], outs[0][1])


def test_special_cases():
    V, n_tests = 64, 6
    g = torch.Generator().manual_seed(5)
    p = torch.randn((2, n_tests, V), generator=g)
    q = p.clone()                      # request 0: q == p, every draft accepted
    q[1] = -float("inf")               # request 1: q one-hot on a token p gives no mass
    q[1, :, 7] = 0.0
    p[1, :, 7] = -float("inf")
    drafts = np.array([[1, 2, 3, 4, 5, 6], [7] * n_tests], np.int32)
    streams = np.array([0, 1], np.uint32)
    pos0 = np.array([10, 20], np.int32)
    out, n_out, _ = _run_gpu(p.cuda(), q.cuda(), torch.from_numpy(drafts).cuda(),
                             torch.from_numpy(streams.view(np.int32)).cuda(), torch.from_numpy(pos0).cuda())
    assert n_out[0] == n_tests and list(out[0, :n_tests]) == list(drafts[0]) and out[0, -1] == -1
    assert n_out[1] == 0            # rejected at once; redraw from the residual = p
    u = float(uniform(SEED, 1, 20, KIND_RESID))
    tally = parity.Tally()
    parity.check_sample(p[1, 0].double().numpy(), u, int(out[1, 0]), tally, "residual=p")
    assert out[1, 0] != 7


def test_special_cases_split_form():
    """The closed forms of test_special_cases at a size that takes the split
    form (8 requests x 32 rows x 19 chunks > 4096 CTAs): q == p accepts every
    draft; q one-hot on a token p gives no mass rejects test 0 and redraws
    from the residual, which is p itself."""
    n_req, n_tests, V = 8, 16, 151936
    g = torch.Generator().manual_seed(9)
    p = torch.randn((n_req, n_tests, V), generator=g) * 3
    q = p.clone()
    for i in range(1, n_req, 2):
        q[i] = -float("inf")
        q[i, :, 11 + i] = 0.0
        p[i, :, 11 + i] = -float("inf")
    drafts = np.array([[(5 * i + j) % V for j in range(n_tests)] if i % 2 == 0 else [11 + i] * n_tests
                       for i in range(n_req)], np.int32)
    streams = np.arange(n_req, dtype=np.uint32) + 40
    pos0 = (np.arange(n_req, dtype=np.int32) * 13) % 1000
    out, n_out, _ = _run_gpu(p.cuda(), q.cuda(), torch.from_numpy(drafts).cuda(),
                             torch.from_numpy(streams.view(np.int32)).cuda(), torch.from_numpy(pos0).cuda())
    tally = parity.Tally()
    for i in range(n_req):
        if i % 2 == 0:
            assert n_out[i] == n_tests and list(out[i, :n_tests]) == list(drafts[i]) and out[i, -1] == -1
        else:
            assert n_out[i] == 0 and out[i, 0] != 11 + i
            u = float(uniform(SEED, int(streams[i]), int(pos0[i]), KIND_RESID))
            parity.check_sample(p[i, 0].double().numpy(), u, int(out[i, 0]), tally, f"residual=p {i}")
    assert tally.mismatches <= 1, tally.notes


def test_microbenchmark_size_sampled():
    """The spec_verify microbenchmark workload at full size: every request's
    output is valid, and sampled requests match the oracle."""
    cfg = synth.SPEC_VERIFY_BENCH
    n_req, R, V = cfg["requests"], cfg["rows_per_request"], cfg["vocab"]
    p, q = synth.make_verify_logits(n_req * R, V, "cuda", cfg["p_std"], cfg["q_noise_std"],
                                    cfg["logits_seed"])
    drafts = synth.make_drafts(q, seed=cfg["logits_seed"] + 1).view(n_req, R)
    p, q = p.view(n_req, R, V), q.view(n_req, R, V)
    streams = torch.arange(n_req, dtype=torch.int32, device="cuda")
    pos0 = torch.zeros(n_req, dtype=torch.int32, device="cuda")
    ws = torch.zeros(uno.uno_spec_verify_workspace_bytes(n_req, R, V), dtype=torch.uint8, device="cuda")
    out = torch.full((n_req, R + 1), -1, dtype=torch.int32, device="cuda")
    n_out = torch.zeros(n_req, dtype=torch.int32, device="cuda")
    uno.uno_spec_verify(p, q, drafts, cfg["seed"], streams, pos0, out, n_out, ws)
    torch.cuda.synchronize()
    o, n, d = out.cpu().numpy(), n_out.cpu().numpy(), drafts.cpu().numpy()
    assert np.all((n >= 0) & (n <= R))
    for i in range(n_req):
        a = int(n[i])
        assert list(o[i, :a]) == list(d[i, :a])
        assert (0 <= o[i, a] < V) if a < R else o[i, a] == -1
    tally = parity.Tally()
    for i in (0, 1, 77, 255):
        pn = p[i].double().cpu().numpy()
        qn = q[i].double().cpu().numpy()
        _check_request(pn, qn, d[i], i, 0, o[i], int(n[i]), tally, seed=cfg["seed"])
    assert tally.mismatches <= 1, tally.notes
