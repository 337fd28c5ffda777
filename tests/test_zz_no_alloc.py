"""kie_gemv_f16_noalloc: the GEMV for callers that cannot allocate device
memory (a process whose memory pool already holds the whole GPU, or a loop
that cannot afford the device-wide synchronisation of cudaMalloc/cudaFree).
Its scratch is a fixed array inside the library.

Checked through the C ABI against kie_gemv_f16 (which allocates its own
scratch) on two calls in a row with different shapes, so the second call
runs on the array the first one left behind; the tolerance is the GEMV
tests' fp32-accumulation bound.  The file is named to run last, after every
other test has used the library, and passes alone as well."""
import ctypes

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


def _bound(W, x):
    K = W.shape[1]
    x16 = x.half().double().cpu()
    return (K * 6e-8 * (W.cpu().double().abs() @ x16.abs())).float() + 1e-6


def test_noalloc_matches_allocating_gemv_twice(torch_cuda):
    torch = torch_cuda
    from persistent_sm_decode_monokernel_b200 import _kie
    stream = torch.cuda.current_stream().cuda_stream
    # larger first, then a smaller ragged shape on the leftover scratch
    shapes = [(2560, 3072, 11), (777, 1280, 12)]
    cases = []
    for N, K, seed in shapes:
        g = torch.Generator(device="cpu").manual_seed(seed)
        W = (torch.randn(N, K, generator=g) * 0.02).half().cuda()
        x = torch.randn(K, generator=g).float().cuda()
        assert N * K * 2 <= _kie.KIE_NOALLOC_MAX_WEIGHT_BYTES
        cases.append((W, x))
    torch.cuda.synchronize()
    for i, (W, x) in enumerate(cases):
        N = W.shape[0]
        y_ref = torch.full((N,), float("nan"), device="cuda")
        _kie.kie_gemv_f16(W, x, y_ref, iters=1, mode=1, chunk_bytes=32768, stream=stream)
        y = torch.full((N,), float("nan"), device="cuda")
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        _kie.kie_gemv_f16_noalloc(W, x, y, stream=stream)
        free1, _ = torch.cuda.mem_get_info()
        if i > 0:
            # set-up (first call) done: the call itself takes no device memory
            assert free1 == free0
        got, ref = y.cpu(), y_ref.cpu()
        assert torch.isfinite(got).all()
        assert ((got - ref).abs() <= _bound(W, x)).all(), float((got - ref).abs().max())


def test_noalloc_after_rejected_call_and_after_larger_grid(torch_cuda):
    """A call the entry point rejects (misaligned x) leaves the array as it
    was, and a call on a matrix with fewer rows than the GPU has SMs (a
    smaller grid) after one with more rows must not read the row split or
    offsets the larger call left beyond its own grid."""
    torch = torch_cuda
    from persistent_sm_decode_monokernel_b200 import _kie
    lib = _kie.load_library()
    stream = torch.cuda.current_stream().cuda_stream
    g = torch.Generator(device="cpu").manual_seed(21)
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    big = ((torch.randn(4 * n_sm, 512, generator=g) * 0.02).half().cuda(),
           torch.randn(512, generator=g).float().cuda())
    small = ((torch.randn(n_sm // 3, 768, generator=g) * 0.02).half().cuda(),
             torch.randn(768 + 4, generator=g).float().cuda())
    outs = []
    for W, x in (big, small):
        N, K = W.shape
        xk = x[:K].contiguous()
        y_ref = torch.full((N,), float("nan"), device="cuda")
        _kie.kie_gemv_f16(W, xk, y_ref, iters=1, mode=1, chunk_bytes=32768, stream=stream)
        y = torch.full((N,), float("nan"), device="cuda")
        torch.cuda.synchronize()
        if W is small[0]:
            # x + 1 element is 4-byte but not 16-byte aligned: rejected before
            # the array is touched
            st = lib.kie_gemv_f16_noalloc(ctypes.c_void_p(W.data_ptr()),
                                          ctypes.c_void_p(x.data_ptr() + 4),
                                          ctypes.c_void_p(y.data_ptr()), N, K,
                                          ctypes.c_void_p(stream))
            assert st == _kie.KIE_ERR_INVALID_ARG
        _kie.kie_gemv_f16_noalloc(W, xk, y, stream=stream)
        torch.cuda.synchronize()
        got, ref = y.cpu(), y_ref.cpu()
        assert torch.isfinite(got).all()
        assert ((got - ref).abs() <= _bound(W, xk)).all(), float((got - ref).abs().max())
        outs.append(got)
    assert outs[1].numel() < n_sm


def test_noalloc_rejects_sizes_beyond_its_scratch(torch_cuda):
    from persistent_sm_decode_monokernel_b200 import _kie
    lib = _kie.load_library()
    limit = _kie.KIE_NOALLOC_MAX_WEIGHT_BYTES
    K = 4096
    N = limit // (2 * K) + 1                  # one row more than fits
    fake = ctypes.c_void_p(1 << 20)           # never dereferenced: rejected first
    st = lib.kie_gemv_f16_noalloc(fake, fake, fake, N, K, None)
    assert st == _kie.KIE_ERR_TOO_LARGE
    assert b"scratch" in lib.kie_status_str(st)
