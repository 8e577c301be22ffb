"""The C-ABI library loads, exports every declared function, and rejects bad
arguments on the host before touching the GPU (CPU only)."""

import ctypes

import pytest

from lossless_diffusion_draft_b200 import build as B
from lossless_diffusion_draft_b200 import uno


@pytest.fixture(scope="module")
def lib():
    B.build()
    return uno.load_library()


def test_every_declared_function_is_exported(lib):
    names = uno.header_functions()
    assert "uno_spec_step" in names and "uno_init" in names and "uno_spec_verify" in names
    for n in names:
        assert hasattr(lib, n), n


def test_init_rejects_bad_arguments(lib):
    out = ctypes.c_void_p()
    assert lib.uno_init(None, None, 8, 16.0, 4, 1, 64, 0, None, ctypes.byref(out)) == uno.UNO_ERR_ARG
    s = uno.UnoShape(2, 64, 4, 3, 16, 172, 256, 255, 1e4, 1e-6, 1.0, uno.UNO_F32)  # 4 % 3 != 0
    w = uno.UnoWeights()
    assert lib.uno_init(ctypes.byref(s), ctypes.byref(w), 8, 16.0, 4, 1, 64, 0, None,
                        ctypes.byref(out)) == uno.UNO_ERR_ARG
    s = uno.UnoShape(2, 64, 4, 4, 16, 172, 256, 255, 1e4, 1e-6, 1.0, uno.UNO_F32)
    assert lib.uno_init(ctypes.byref(s), ctypes.byref(w), 8, 16.0, 1, 1, 64, 0, None,
                        ctypes.byref(out)) == uno.UNO_ERR_ARG      # B < 2
    s = uno.UnoShape(2, 64, 4, 4, 24, 172, 256, 255, 1e4, 1e-6, 1.0, uno.UNO_F32)
    assert lib.uno_init(ctypes.byref(s), ctypes.byref(w), 8, 16.0, 4, 1, 64, 0, None,
                        ctypes.byref(out)) == uno.UNO_ERR_UNSUPPORTED   # head_dim 24
    s = uno.UnoShape(2, 64, 4, 4, 16, 172, 256, 255, 1e4, 1e-6, 1.0, uno.UNO_F32)
    assert lib.uno_init(ctypes.byref(s), ctypes.byref(w), 8, 16.0, 4, 1, 64, 0, None,
                        ctypes.byref(out)) == uno.UNO_ERR_ARG      # null weight pointers
    assert out.value is None


def test_null_context_calls(lib):
    assert lib.uno_spec_step(None, 1, None, None, None) == uno.UNO_ERR_ARG
    assert lib.uno_prefill(None, 1, None, 1, None, None, None) == uno.UNO_ERR_ARG
    assert lib.uno_destroy(None) == uno.UNO_ERR_ARG
    assert lib.uno_last_error(None) == b"null context"


def test_spec_verify_workspace_and_argument_checks(lib):
    # counters (rows) | request counters | residual counters (requests) |
    # lse (rows) | partial pairs (rows x chunks) | first rejection (requests) |
    # residual chunk sums (requests x chunks)
    n_req, n_tests, V = 256, 16, 151936
    rows = n_req * 2 * n_tests
    nch = -(-V // 8192)
    def a256(x):
        return (x + 255) // 256 * 256
    want = (a256(rows * 4) + a256(n_req * 4) + a256(n_req * 4) + a256(rows * 4) +
            a256(rows * nch * 8) + a256(n_req * 4) + a256(n_req * nch * 4))
    assert uno.uno_spec_verify_workspace_bytes(n_req, n_tests, V) == want
    assert uno.uno_spec_verify_workspace_bytes(0, 16, V) == 0
    null = None
    assert lib.uno_spec_verify(null, null, null, 1, 1, 16, 0, null, null, null, null, null, 0,
                               null) == uno.UNO_ERR_ARG
    fake = 256  # never dereferenced: the size checks fail first
    assert lib.uno_spec_verify(fake, fake, fake, 1, 1, 18, 0, fake, fake, fake, fake, fake, 1 << 20,
                               null) == uno.UNO_ERR_ARG            # vocab % 4 != 0
    assert lib.uno_spec_verify(fake, fake, fake, 1, 1, 16, 0, fake, fake, fake, fake, fake, 8,
                               null) == uno.UNO_ERR_ARG            # workspace too small
