"""The decode kernel's weight-stream GEMV engine run alone (kie_gemv_f16)
against a plain PyTorch reference of the same matrix-vector product.

The engine takes its input vector in fp16 and accumulates fp16 x fp16
products in fp32 (the analogue of a dot2 instruction), so the reference
rounds x to fp16 and sums in fp64; the remaining difference is fp32
accumulation error, bounded by K * eps32 * sum |w x|."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from persistent_sm_decode_monokernel_b200 import build
    build.build()
    return torch


@pytest.mark.parametrize("N,K,chunk", [
    (1, 256, 8192),          # one row, one piece
    (7, 512, 8192),          # fewer rows than CTAs, ragged groups
    (300, 2560, 20480),      # two to three rows per CTA
    (1333, 6912, 20480),     # ragged tail group, K split in chunks
    (4096, 14336, 32768),    # long rows, several k-chunks
    (50304, 2560, 16384),    # LM-head shape
    (9001, 2816, 12800),     # chunk not a power of two, ring wraps unevenly
])
def test_gemv_matches_fp32_reference(torch_cuda, N, K, chunk):
    torch = torch_cuda
    from persistent_sm_decode_monokernel_b200 import _kie
    g = torch.Generator(device="cpu").manual_seed(N * 7 + K)
    W = (torch.randn(N, K, generator=g) * 0.02).half().cuda()
    x = torch.randn(K, generator=g).float().cuda()
    y = torch.full((N,), float("nan"), device="cuda")
    _kie.kie_gemv_f16(W, x, y, iters=2, mode=1, chunk_bytes=chunk,
                      stream=torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    x16 = x.half().double().cpu()
    ref = (W.cpu().double() @ x16).float()
    got = y.cpu()
    assert torch.isfinite(got).all()
    # fp32 accumulation over K terms: bound by K * eps32 * sum|w x|
    bound = (K * 6e-8 * (W.cpu().double().abs() @ x16.abs())).float() + 1e-6
    assert ((got - ref).abs() <= bound).all(), float((got - ref).abs().max())
