"""The C-ABI library: it builds for sm_100a, loads, exports every function
include/w8a8.h declares, and rejects bad arguments on the host before any
CUDA call (so these run without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from w8a8_quantized_linear_b200 import _build
    _build.build()
    import w8a8_quantized_linear_b200 as w8
    return w8.lib()


def _header_functions():
    text = open(os.path.join(ROOT, "include", "w8a8.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = _header_functions()
    for want in ("w8a8_quantize_rows", "w8a8_quantize_weight", "q8_0_quantize", "q8_0_dequantize",
                 "q8_0_to_axis_int8", "q8_0_to_axis_e4m3", "w8a8_linear_fwd", "w8a8_linear_dgrad",
                 "svdq_linear_fwd", "svdq_linear_fwd_e4m3"):
        assert want in names


def test_every_declared_symbol_is_exported(L):
    import w8a8_quantized_linear_b200 as w8
    names = _header_functions()
    assert set(names) == set(w8.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_library_is_built_for_sm100a():
    from w8a8_quantized_linear_b200 import _build
    cmd = _build.command()
    assert "arch=compute_100a,code=sm_100a" in cmd


def test_sizes(L):
    assert L.q8_0_bytes(0) == 0
    assert L.q8_0_bytes(1) == 34
    assert L.q8_0_bytes(32) == 34
    assert L.q8_0_bytes(33) == 68
    assert L.q8_0_bytes(1 << 28) == (1 << 23) * 34
    # workspace: codes then row scales, each on a 256-byte boundary
    assert L.w8a8_workspace_bytes(0, 4608, 12288, 3072, 0) == 4608 * 3072 + 4608 * 4
    assert L.w8a8_workspace_bytes(0, 3, 8, 16, 0) == 256 + 256
    assert L.w8a8_workspace_bytes(1, 3, 40, 16, 0) == 256 + 256  # N padded to 48 -> 144 bytes
    # SVDQuant: codes, row scales, T [M, r] bf16, then T's split-K partial sums
    # (36 row tiles over a 3072-long contraction: 4 splits, [4, 4608, 32] fp32)
    # SVDQuant: rows of up to 3072 take the one-pass input kernel (no split
    # partial sums); longer rows the split T product (4 splits at 4608 rows)
    assert L.w8a8_workspace_bytes(2, 4608, 3072, 3072, 32) == 4608 * 3072 + 4608 * 4 + 4608 * 32 * 2
    assert L.w8a8_workspace_bytes(2, 4608, 3072, 6144, 32) == 4608 * 6144 + 4608 * 4 + 4608 * 32 * 2 + 4 * 4608 * 32 * 4
    assert L.w8a8_workspace_bytes(2, 200, 320, 256, 32) == 200 * 256 + 1024 + 200 * 32 * 2   # unsplit
    assert L.w8a8_workspace_bytes(3, 10, 10, 16, 0) == 256
    # few output tiles, long contraction: split-K partial sums follow
    # (48 tiles -> 3 splits of 8 K blocks; [3, 1, 12288] int32)
    assert L.w8a8_workspace_bytes(0, 1, 12288, 3072, 0) == 3072 + 256 + 3 * 12288 * 4
    # dgrad of the up-projection at M=64: 12 tiles over K=3072, 96 K blocks -> 12 splits
    assert L.w8a8_workspace_bytes(1, 64, 12288, 3072, 0) == 64 * 12288 + 256 + 12 * 64 * 3072 * 4
    # output width not a multiple of 8: never split
    assert L.w8a8_workspace_bytes(0, 1, 1001, 4096, 0) == 4096 + 256
    assert L.w8a8_workspace_bytes(9, 1, 1, 16, 0) == 0
    # bf16 Linear: nothing unless split (M = 1, N = 12288: 48 tiles -> 3 splits)
    assert L.w8a8_workspace_bytes(4, 4608, 12288, 3072, 0) == 0
    assert L.w8a8_workspace_bytes(4, 1, 12288, 3072, 0) == 3 * 12288 * 4
    # weight-only: the bf16 weight, then the partial sums
    assert L.w8a8_workspace_bytes(5, 4608, 12288, 3072, 0) == 12288 * 3072 * 2
    assert L.w8a8_workspace_bytes(5, 1, 12288, 3072, 0) == 12288 * 3072 * 2 + 3 * 12288 * 4


A = ctypes.c_void_p(1 << 20)        # a 16-byte aligned stand-in pointer (never dereferenced)
B = ctypes.c_void_p((1 << 20) + 8)  # misaligned


def test_quantize_rows_validation(L):
    # M == 0 is a no-op
    assert L.w8a8_quantize_rows(A, 0, 64, 64, 0, A, 64, A, None) == 0
    assert L.w8a8_quantize_rows(A, 4, 64, 64, 5, A, 64, A, None) == 1         # bad qtype
    assert L.w8a8_quantize_rows(A, 4, 24, 24, 0, A, 32, A, None) == 2         # K % 16
    assert L.w8a8_quantize_rows(A, 4, 0, 0, 0, A, 16, A, None) == 2           # K < 16
    assert L.w8a8_quantize_rows(A, -1, 64, 64, 0, A, 64, A, None) == 2        # M < 0
    assert L.w8a8_quantize_rows(A, 4, 64, 60, 0, A, 64, A, None) == 3         # ldx < K
    assert L.w8a8_quantize_rows(A, 4, 64, 64, 0, A, 72, A, None) == 3         # ldq % 16
    assert L.w8a8_quantize_rows(None, 4, 64, 64, 0, A, 64, A, None) == 1      # null
    assert L.w8a8_quantize_rows(B, 4, 64, 64, 0, A, 64, A, None) == 3         # misaligned
    assert b"16-byte" in L.w8a8_last_error()


def test_linear_validation(L):
    assert L.w8a8_linear_fwd(A, 8, 8, 24, 0, A, A, 0, None, A, A, 1 << 20, None) == 2
    assert L.w8a8_linear_fwd(A, 8, 8, 32, 2, A, A, 0, None, A, A, 1 << 20, None) == 1
    assert L.w8a8_linear_fwd(A, 8, 8, 32, 0, A, A, 0, B, A, A, 1 << 20, None) == 3   # bias misaligned
    assert L.w8a8_linear_fwd(A, 8, 8, 32, 0, A, A, 0, None, A, A, 16, None) == 4     # workspace
    assert L.w8a8_linear_fwd(A, 8, 8, 32, 0, A, A, 0, None, A, None, 0, None) == 4
    assert L.w8a8_linear_fwd(A, 0, 8, 32, 0, A, A, 0, None, A, None, 0, None) == 0   # M == 0
    assert L.w8a8_linear_fwd(A, 8, 0, 32, 0, A, A, 0, None, A, A, 1 << 20, None) == 2
    # dgrad: tensor-wise only, N % 16
    assert L.w8a8_linear_dgrad(A, 8, 32, 32, 0, A, A, 1, A, A, 1 << 20, None) == 1
    assert L.w8a8_linear_dgrad(A, 8, 40, 32, 0, A, A, 0, A, A, 1 << 20, None) == 2
    assert L.w8a8_linear_dgrad(A, 8, 32, 32, 0, A, A, 0, A, A, 8, None) == 4


def test_svdq_validation(L):
    assert L.svdq_linear_fwd(A, 8, 8, 32, A, A, 12, A, A, None, A, A, 1 << 20, None) == 2   # r % 8
    assert L.svdq_linear_fwd(A, 8, 8, 32, A, A, 64, A, A, None, A, A, 1 << 20, None) == 2   # r > 32
    assert L.svdq_linear_fwd(A, 8, 8, 32, A, A, 32, None, A, None, A, A, 1 << 20, None) == 1
    assert L.svdq_linear_fwd(A, 8, 8, 32, A, A, 32, A, A, None, A, A, 64, None) == 4
    assert L.svdq_linear_fwd_e4m3(A, 8, 8, 32, A, A, 12, A, A, None, A, A, 1 << 20, None) == 2   # r % 8
    assert L.svdq_linear_fwd_e4m3(A, 8, 8, 32, A, A, 32, None, A, None, A, A, 1 << 20, None) == 1
    assert L.svdq_linear_fwd_e4m3(A, 8, 8, 32, A, A, 32, A, A, None, A, A, 64, None) == 4
    assert L.svdq_linear_fwd_e4m3(A, 0, 8, 32, A, A, 32, A, A, None, A, A, 0, None) == 0      # M = 0: no-op


def test_linear_fwd_ex_validation(L):
    args = lambda act, xa, ya: (A, 8, 8, 32, 0, A, A, 0, None, act, xa, ya, A, A, 1 << 20, None)
    assert L.w8a8_linear_fwd_ex(*args(3, None, None)) == 1        # unknown activation
    assert L.w8a8_linear_fwd_ex(*args(1, A, A)) == 1              # x_amax aliases y_amax
    assert L.w8a8_linear_fwd_ex(*args(1, B, None)) == 3           # misaligned x_amax
    assert L.w8a8_linear_fwd_ex(A, 0, 8, 32, 0, A, A, 0, None, 1, None, None, A, A, 0, None) == 0   # M = 0


def test_weight_only_validation(L):
    assert L.bf16_linear_fwd(A, 8, 8, 20, A, None, A, A, 1 << 20, None) == 2        # K % 16
    assert L.bf16_linear_fwd(A, 0, 8, 32, None, None, None, None, 0, None) == 0     # M = 0: no-op
    assert L.bf16_linear_fwd(A, 8, 8, 32, None, None, A, A, 1 << 20, None) == 1
    assert L.bf16_linear_fwd(B, 8, 8, 32, A, None, A, A, 1 << 20, None) == 3
    assert L.bf16_linear_fwd(A, 1, 12288, 3072, A, None, A, None, 0, None) == 4     # split needs a workspace
    assert L.float8_linear_fwd(A, 8, 8, 32, A, A, None, A, A, 64, None) == 4        # the bf16 weight needs room
    assert L.float8_linear_fwd(A, 8, 8, 32, A, None, None, A, A, 1 << 20, None) == 1
    assert L.gguf_linear_fwd(A, 8, 8, 32, A, None, A, A, 64, None) == 4
    assert L.gguf_linear_fwd(A, 8, 8, 24, A, None, A, A, 1 << 20, None) == 2
    assert L.w8a8_dequantize_e4m3_bf16(A, 24, A, A, None) == 2                      # n % 16
    assert L.w8a8_dequantize_e4m3_bf16(A, 32, None, A, None) == 1
    assert L.q8_0_dequantize_bf16(A, 3, B, None) == 3
    assert L.bf16_linear_dgrad(A, 8, 12, 32, A, A, A, 1 << 20, None) == 2      # N % 8
    assert L.bf16_linear_dgrad(A, 8, 16, 24, A, A, A, 1 << 20, None) == 2      # K % 16
    assert L.float8_linear_dgrad(A, 8, 16, 32, A, None, A, A, 1 << 20, None) == 1
    assert L.gguf_linear_dgrad(A, 8, 16, 32, A, A, A, 64, None) == 4
    assert L.bf16_linear_dgrad(A, 0, 16, 32, None, None, None, 0, None) == 0     # M = 0


def test_q8_0_validation(L):
    assert L.q8_0_quantize(A, 0, A, None) == 0
    assert L.q8_0_quantize(A, -3, A, None) == 2
    assert L.q8_0_quantize(None, 3, A, None) == 1
    assert L.q8_0_quantize(A, 3, B, None) == 3
    assert L.q8_0_dequantize(A, 3, B, None) == 3
    assert L.q8_0_to_axis_int8(A, 4, 48, A, A, None) == 2      # K % 32
    assert L.q8_0_to_axis_int8(A, 4, 1 << 18, A, A, None) == 2  # K too large
    assert L.q8_0_to_axis_int8(A, 0, 64, A, A, None) == 2
    assert L.q8_0_to_axis_e4m3(A, 4, 48, A, A, None) == 2      # K % 32
    assert L.q8_0_to_axis_e4m3(A, 4, 1 << 18, A, A, None) == 2  # K too large
    assert L.q8_0_to_axis_e4m3(A, 0, 64, A, A, None) == 2
    assert L.q8_0_to_axis_e4m3(A, 4, 64, None, A, None) == 1
    assert L.q8_0_to_axis_e4m3(A, 4, 64, B, A, None) == 3       # misaligned codes
    assert L.w8a8_quantize_weight(A, 4, 64, 0, 0, A, A, None, 0, None) == 4   # tensor needs ws
    assert L.w8a8_quantize_weight(A, 4, 64, 0, 7, A, A, None, 0, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import w8a8_quantized_linear_b200 as w8
    monkeypatch.setattr(w8, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(w8, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        w8.lib()


def test_debug_build_exports_and_reports_its_checks(L):
    """libw8a8_debug.so (device-side index checks that record an error code
    instead of faulting) builds from the same sources, exports the same
    functions, and says it is the checked build; the release build says not."""
    from w8a8_quantized_linear_b200 import _build
    D = ctypes.CDLL(_build.build(debug=True))
    for n in _header_functions():
        assert hasattr(D, n), n
    D.w8a8_debug_checks.restype = ctypes.c_int
    assert D.w8a8_debug_checks() == 1
    assert L.w8a8_debug_checks() == 0
