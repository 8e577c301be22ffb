"""uno_spec_verify_noalloc: spec_verify for callers that cannot allocate
device memory (a serving process whose memory is reserved up front by its own
pool, or code that cannot afford cudaMalloc's implicit synchronisation).  It
uses the library's fixed scratch array instead of a workspace; its results
must equal those of uno_spec_verify with a workspace, call after call.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""

import numpy as np
import pytest
import torch

from lossless_diffusion_draft_b200 import build, uno

pytestmark = pytest.mark.gpu


def _inputs(n_req, n_tests, V, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    p = torch.randn((n_req, n_tests, V), generator=g, device="cuda") * 3
    q = p + torch.randn((n_req, n_tests, V), generator=g, device="cuda") * 0.5
    drafts = torch.randint(0, V, (n_req, n_tests), generator=g, device="cuda", dtype=torch.int32)
    streams = torch.arange(n_req, dtype=torch.int32, device="cuda") + seed
    pos0 = torch.randint(0, 5000, (n_req,), generator=g, device="cuda", dtype=torch.int32)
    return p, q, drafts, streams, pos0


def _with_workspace(p, q, drafts, streams, pos0, seed):
    n_req, n_tests, V = p.shape
    ws = torch.zeros(uno.uno_spec_verify_workspace_bytes(n_req, n_tests, V), dtype=torch.uint8,
                     device="cuda")
    out = torch.full((n_req, n_tests + 1), -7, dtype=torch.int32, device="cuda")
    n_out = torch.full((n_req,), -7, dtype=torch.int32, device="cuda")
    uno.uno_spec_verify(p, q, drafts, seed, streams, pos0, out, n_out, ws)
    torch.cuda.synchronize()
    return out.cpu(), n_out.cpu()


def _no_alloc(p, q, drafts, streams, pos0, seed):
    n_req, n_tests, _ = p.shape
    out = torch.full((n_req, n_tests + 1), -7, dtype=torch.int32, device="cuda")
    n_out = torch.full((n_req,), -7, dtype=torch.int32, device="cuda")
    uno.uno_spec_verify_noalloc(p, q, drafts, seed, streams, pos0, out, n_out)
    torch.cuda.synchronize()
    return out.cpu(), n_out.cpu()


def test_noalloc_matches_workspace_entry_two_calls_in_a_row():
    build.build()
    uno.load_library()
    # different workloads back to back: the shared scratch array keeps each
    # call's contents, the next call must not be disturbed by them.  The first
    # two need more than 4096 (row, chunk) CTAs and take the split form; the
    # third (4 x 16 rows x 4 chunks = 256 CTAs) takes the fused form, whose
    # row and request completion counters live in the array and start at
    # zero only because the call clears them.  Before it, a rejected call
    # (vocab not a multiple of 4) must leave the array and the stream alone.
    for call, (n_req, n_tests, V) in enumerate([(64, 16, 32000), (37, 9, 151936), (4, 8, 32000)]):
        seed = 11 + call
        args = _inputs(n_req, n_tests, V, seed)
        if call == 2:
            p, q, drafts, streams, pos0 = args
            out = torch.empty((n_req, n_tests + 1), dtype=torch.int32, device="cuda")
            n_out = torch.empty((n_req,), dtype=torch.int32, device="cuda")
            code = uno.load_library().uno_spec_verify_noalloc(
                p.data_ptr(), q.data_ptr(), drafts.data_ptr(), n_req, n_tests, 6, 0,
                streams.data_ptr(), pos0.data_ptr(), out.data_ptr(), n_out.data_ptr(), None)
            assert code == uno.UNO_ERR_ARG
        need = uno.uno_spec_verify_workspace_bytes(n_req, n_tests, V)
        assert need <= uno.uno_spec_verify_noalloc_max_bytes()
        want_out, want_n = _with_workspace(*args, seed)
        got_out, got_n = _no_alloc(*args, seed)
        # integer outputs: identical (same kernel, same inputs, same uniforms)
        assert torch.equal(got_n, want_n), call
        assert torch.equal(got_out, want_out), call
        assert int((got_n >= 0).sum()) == n_req


def test_noalloc_rejects_sizes_beyond_its_array():
    cap = uno.uno_spec_verify_noalloc_max_bytes()
    n_req, n_tests, V = 1024, 16, 151936          # 16384 rows: > 4 MiB of scratch
    assert uno.uno_spec_verify_workspace_bytes(n_req, n_tests, V) > cap
    dummy = torch.zeros(1, dtype=torch.float32, device="cuda")
    code = uno.load_library().uno_spec_verify_noalloc(
        dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), n_req, n_tests, V, 0,
        dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), None)
    assert code == uno.UNO_ERR_CAPACITY
