"""w8a8_linear_fwd_noalloc: the forward for callers that cannot give the
library scratch memory (no allocator available, or allocation forbidden on
their path).  Its output must equal w8a8_linear_fwd's, call after call, even
though every call reuses the same built-in scratch array; sizes beyond that
array must be refused before anything runs.

The file name sorts last so that a run stopping at the first failure has
already run every other test; it also passes when run alone."""
import ctypes

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def w8():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w8a8_quantized_linear_b200 import _build
    _build.build()
    import w8a8_quantized_linear_b200 as m
    m.lib()
    return m


def _call_noalloc(w8, x, wq, sw, bias, y):
    """Straight through the C ABI: only the caller's inputs and output."""
    M, K = x.shape
    N = wq.shape[0]
    qt = w8.INT8 if wq.dtype == torch.int8 else w8.E4M3
    g = w8.AXIS if sw.numel() > 1 else w8.TENSOR
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return w8.lib().w8a8_linear_fwd_noalloc(ptr(x), M, N, K, qt, ptr(wq.view(torch.uint8)), ptr(sw), g,
                                            ptr(bias), ptr(y), stream)


CASES = [  # (M, N, K, qtype, granularity, bias) - two calls in a row per case
    [(300, 520, 640, "int8", "tensor", False), (1, 16, 16, "int8", "tensor", False)],
    [(4608, 3072, 3072, "int8", "tensor", False), (129, 257, 96, "int8", "axis", True)],
    [(256, 512, 512, "e4m3", "tensor", True), (2048, 1024, 4096, "e4m3", "tensor", False)],
    # few rows: the one-launch CUDA-core kernels, axis scales and bias
    [(2, 3072, 3072, "int8", "axis", True), (1, 520, 640, "e4m3", "axis", True)],
    [(64, 12288, 3072, "int8", "axis", True), (3, 3072, 3072, "e4m3", "tensor", True)],
]


@pytest.mark.parametrize("calls", CASES)
def test_noalloc_matches_workspace_forward(w8, calls):
    for i, (M, N, K, qt, gran, with_bias) in enumerate(calls):
        x = workloads.with_outlier_channels((M, K), 1.0, seed=M + N + i).to(DEV)
        wq, sw = w8.quantize_weight(workloads.normal((N, K), 0.02, seed=K + i).to(DEV), qt, gran)
        bias = workloads.normal((N,), 0.01, seed=N).to(DEV) if with_bias else None
        y_ref = w8.linear_fwd(x, wq, sw, bias=bias)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _call_noalloc(w8, x, wq, sw, bias, y) == 0, w8.lib().w8a8_last_error()
        torch.cuda.synchronize()
        # bit-exact for both formats: same kernels, same inputs, deterministic order
        assert torch.equal(y, y_ref), (M, N, K, qt)
    assert w8.device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch(w8):
    K = 3072
    M = (64 << 20) // K + 1                    # M*K just above 64 MiB of codes
    x = torch.zeros((M, K), dtype=torch.bfloat16, device=DEV)
    wq, sw = w8.quantize_weight(workloads.normal((16, K), 0.02, 1).to(DEV), "int8", "tensor")
    y = torch.empty((M, 16), dtype=torch.bfloat16, device=DEV)
    assert _call_noalloc(w8, x, wq, sw, None, y) == 4          # W8A8_ERR_WORKSPACE
    assert b"scratch" in w8.lib().w8a8_last_error()
    x2 = torch.zeros((65537, 16), dtype=torch.bfloat16, device=DEV)
    wq2, sw2 = w8.quantize_weight(workloads.normal((16, 16), 0.02, 2).to(DEV), "int8", "tensor")
    y2 = torch.empty((65537, 16), dtype=torch.bfloat16, device=DEV)
    assert _call_noalloc(w8, x2, wq2, sw2, None, y2) == 4      # more rows than row-scale slots
