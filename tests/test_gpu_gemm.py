"""gated_lora_linear (tcgen05 and SIMT kernels) vs a plain PyTorch reference
of the same op in float64 on the same inputs (GPU)."""

import pytest
import torch

from lossless_diffusion_draft_b200 import uno

pytestmark = pytest.mark.gpu


def _reference(X, W, A, Bl, gate, scale, cols=None):
    Xd, Wd = X.double().cpu(), W.double().cpu()
    if cols is not None:
        Wd = Wd[cols]
    Y = Xd @ Wd.T
    if A is not None:
        g = torch.ones(X.shape[0], dtype=torch.float64) if gate is None else gate.double().cpu()
        U = (g[:, None] * scale) * (Xd @ A.double().cpu().T)
        U = U.to(X.dtype).double()          # the kernel stores U in the model dtype
        B = Bl.double().cpu()
        if cols is not None:
            B = B[cols]
        Y = Y + U @ B.T
    return Y


def _run(M, N, K, r, dtype, seed=0, cols=None, repeat=1):
    g = torch.Generator(device="cuda").manual_seed(seed)
    dev = "cuda"
    X = torch.randn((M, K), generator=g, device=dev).to(dtype)
    W = (torch.randn((N, K), generator=g, device=dev) * 0.02).to(dtype)
    A = (torch.randn((r, K), generator=g, device=dev) * 0.02).to(dtype) if r else None
    Bl = (torch.randn((N, r), generator=g, device=dev) * 0.05).to(dtype) if r else None
    gate = (torch.rand(M, generator=g, device=dev) < 0.6).float() if r else None
    scale = 2.0
    wsb = uno.uno_gated_lora_linear_workspace_bytes(M, N, K, r, uno.UNO_BF16 if dtype == torch.bfloat16 else uno.UNO_F32)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    outs = []
    for _ in range(repeat):
        Y = torch.full((M, N), float("nan"), device=dev)
        uno.uno_gated_lora_linear(X, W, A, Bl, gate, scale, Y, ws)
        torch.cuda.synchronize()
        outs.append(Y.cpu())
    ref = _reference(X, W, A, Bl, gate, scale, cols)
    Y = outs[0] if cols is None else outs[0][:, cols]
    return Y.double(), ref, outs, ws


@pytest.mark.parametrize("M,N,K,r", [
    (1, 128, 64, 64),          # one tile, one k-block of each kind
    (17, 4096, 4096, 128),     # a draft-pass projection
    (16, 384, 4096, 0),        # LoRA down-projection shape, no adapter
    (33, 1000, 256, 64),       # ragged N: partial last tile
    (130, 512, 1024, 128),     # 256-row token tile
    (300, 640, 512, 128),      # two token tiles
    (17, 12288, 4096, 128),    # gate/up width
    (5, 4096, 12288, 128),     # down-projection depth (many k-blocks per tile)
    (1360, 4224, 4096, 128),   # max-batch rows: six token tiles in m-tile groups, tiles cut
    (600, 24832, 512, 128),    # three token tiles across a wide row of weight tiles
])
def test_bf16_tensor_core(M, N, K, r):
    before = uno.uno_debug_launch_counts()
    Y, ref, _, _ = _run(M, N, K, r, torch.bfloat16)
    after = uno.uno_debug_launch_counts()
    assert after["tc_gemm"] > before["tc_gemm"]          # the tcgen05 kernel ran
    assert torch.isfinite(Y).all()
    err = (Y - ref).abs().max().item()
    assert err <= 2e-3 * ref.abs().max().item() + 1e-4, err


def test_bf16_lm_head_width_sampled():
    cols = torch.arange(0, 151936, 37)
    Y, ref, _, _ = _run(17, 151936, 4096, 0, torch.bfloat16, cols=cols)
    err = (Y - ref).abs().max().item()
    assert err <= 2e-3 * ref.abs().max().item() + 1e-4, err


@pytest.mark.parametrize("M,N,K,r", [(5, 172, 64, 8), (17, 300, 1024, 16), (40, 64, 172, 8)])
def test_fp32_simt(M, N, K, r):
    Y, ref, _, _ = _run(M, N, K, r, torch.float32)
    err = (Y - ref).abs().max().item()
    assert err <= 1e-5 * ref.abs().max().item() + 1e-6, err


def test_bf16_fallback_shape():
    # K = 200 is not a whole number of 64-element blocks: SIMT kernel
    Y, ref, _, _ = _run(9, 256, 200, 16, torch.bfloat16)
    err = (Y - ref).abs().max().item()
    assert err <= 2e-3 * ref.abs().max().item() + 1e-4, err


@pytest.mark.parametrize("M", [17, 1360])
def test_deterministic_and_workspace_left_zero(M):
    _, _, outs, ws = _run(M, 4096, 4096, 128, torch.bfloat16, repeat=3)
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    assert int(ws[: (1 << 16) * 4].count_nonzero()) == 0   # counters left zeroed
