"""B200-native W8A8 quantized Linear: a thin ctypes binding over libw8a8.so.

Every step of the hot path runs in the library's sm_100a kernels; this module
only checks tensor properties, allocates outputs/workspace with torch on the
tensors' device, and passes pointers and the current CUDA stream through the
C ABI declared in ``include/w8a8.h``.  There is no CPU or PyTorch fallback:
calling any compute function without the built library raises.

Quantization follows OneTrainer wiki "Quantization" (int / float W8A8:
tensor-wise weights, token-wise activations, 8-bit Linear matmul; GGUF A8 int:
GGUF weights re-quantized to int8 axis-wise; SVDQuant), bitsandbytes #1401
(the fused row calibrate-and-quantize op) and entrenar's Q8_0 format.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# W8A8_LIBRARY=debug selects the build with device-side index checks
# (libw8a8_debug.so, see include/w8a8.h); the default is the release build.
LIB_PATH = os.path.join(_PKG, "libw8a8_debug.so" if os.environ.get("W8A8_LIBRARY") == "debug" else "libw8a8.so")

INT8, E4M3 = 0, 1
TENSOR, AXIS = 0, 1
OP_LINEAR_FWD, OP_LINEAR_DGRAD, OP_SVDQ_FWD, OP_QUANTIZE_WEIGHT = 0, 1, 2, 3
OP_BF16_FWD, OP_WEIGHT_ONLY_FWD, OP_BF16_DGRAD, OP_WEIGHT_ONLY_DGRAD = 4, 5, 6, 7
ACTS = {"none": 0, "gelu": 1, "gelu_tanh": 2}

STATUS = {0: "W8A8_OK", 1: "W8A8_ERR_INVALID_ARG", 2: "W8A8_ERR_UNSUPPORTED_SHAPE",
          3: "W8A8_ERR_MISALIGNED", 4: "W8A8_ERR_WORKSPACE", 5: "W8A8_ERR_CUDA",
          6: "W8A8_ERR_DEVICE_TIMEOUT", 7: "W8A8_ERR_UNSUPPORTED_DEVICE", 8: "W8A8_ERR_DEVICE_BOUNDS"}

# Every symbol include/w8a8.h declares (checked by the tests).
EXPORTS = ("w8a8_quantize_rows", "w8a8_quantize_weight", "q8_0_bytes", "q8_0_quantize",
           "q8_0_dequantize", "q8_0_to_axis_int8", "q8_0_to_axis_e4m3", "w8a8_linear_fwd", "w8a8_linear_dgrad",
           "svdq_linear_fwd", "svdq_linear_fwd_e4m3", "w8a8_qgemm_fwd", "w8a8_qgemm_dgrad", "w8a8_workspace_bytes",
           "w8a8_device_status", "w8a8_set_wait_limit_ns", "w8a8_selftest_wait",
           "w8a8_e4m3_encode", "w8a8_last_error", "w8a8_linear_fwd_noalloc", "q8_0_dequantize_bf16",
           "w8a8_dequantize_e4m3_bf16", "bf16_linear_fwd", "float8_linear_fwd", "gguf_linear_fwd",
           "w8a8_linear_fwd_ex", "bf16_linear_dgrad", "float8_linear_dgrad", "gguf_linear_dgrad",
           "w8a8_selftest_bounds", "w8a8_debug_checks")


class W8A8Error(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__("%s: %s" % (STATUS.get(status, str(status)), msg))
        self.status = status


_lib = None
_P, _I64, _I, _SZ, _U64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64


def lib() -> ctypes.CDLL:
    """The loaded libw8a8.so.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("%s is not built (run `python -m w8a8_quantized_linear_b200._build`); "
                               "there is no fallback path" % os.path.basename(LIB_PATH))
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "w8a8_quantize_rows": [_P, _I64, _I64, _I64, _I, _P, _I64, _P, _P],
            "w8a8_quantize_weight": [_P, _I64, _I64, _I, _I, _P, _P, _P, _SZ, _P],
            "q8_0_quantize": [_P, _I64, _P, _P],
            "q8_0_dequantize": [_P, _I64, _P, _P],
            "q8_0_to_axis_int8": [_P, _I64, _I64, _P, _P, _P],
            "q8_0_to_axis_e4m3": [_P, _I64, _I64, _P, _P, _P],
            "w8a8_linear_fwd": [_P, _I64, _I64, _I64, _I, _P, _P, _I, _P, _P, _P, _SZ, _P],
            "w8a8_linear_dgrad": [_P, _I64, _I64, _I64, _I, _P, _P, _I, _P, _P, _SZ, _P],
            "svdq_linear_fwd": [_P, _I64, _I64, _I64, _P, _P, _I, _P, _P, _P, _P, _P, _SZ, _P],
            "svdq_linear_fwd_e4m3": [_P, _I64, _I64, _I64, _P, _P, _I, _P, _P, _P, _P, _P, _SZ, _P],
            "w8a8_qgemm_fwd": [_P, _I64, _P, _I64, _I64, _I64, _I, _P, _P, _I, _P, _P, _P],
            "w8a8_qgemm_dgrad": [_P, _I64, _P, _I64, _I64, _I64, _I, _P, _P, _P, _P],
            "w8a8_device_status": [_P, _I],
            "w8a8_set_wait_limit_ns": [_U64],
            "w8a8_selftest_wait": [_U64, _P],
            "w8a8_selftest_bounds": [_P],
            "w8a8_e4m3_encode": [_P, _I64, _P, _P],
            "w8a8_linear_fwd_noalloc": [_P, _I64, _I64, _I64, _I, _P, _P, _I, _P, _P, _P],
            "q8_0_dequantize_bf16": [_P, _I64, _P, _P],
            "w8a8_linear_fwd_ex": [_P, _I64, _I64, _I64, _I, _P, _P, _I, _P, _I, _P, _P, _P, _P, _SZ, _P],
            "w8a8_dequantize_e4m3_bf16": [_P, _I64, _P, _P, _P],
            "bf16_linear_fwd": [_P, _I64, _I64, _I64, _P, _P, _P, _P, _SZ, _P],
            "float8_linear_fwd": [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _SZ, _P],
            "gguf_linear_fwd": [_P, _I64, _I64, _I64, _P, _P, _P, _P, _SZ, _P],
            "bf16_linear_dgrad": [_P, _I64, _I64, _I64, _P, _P, _P, _SZ, _P],
            "float8_linear_dgrad": [_P, _I64, _I64, _I64, _P, _P, _P, _P, _SZ, _P],
            "gguf_linear_dgrad": [_P, _I64, _I64, _I64, _P, _P, _P, _SZ, _P],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = _I
        L.q8_0_bytes.argtypes = [_I64]
        L.q8_0_bytes.restype = _SZ
        L.w8a8_workspace_bytes.argtypes = [_I, _I64, _I64, _I64, _I]
        L.w8a8_workspace_bytes.restype = _SZ
        L.w8a8_last_error.argtypes = []
        L.w8a8_last_error.restype = ctypes.c_char_p
        L.w8a8_debug_checks.argtypes = []
        L.w8a8_debug_checks.restype = _I
        _lib = L
    return _lib


def _check(status: int):
    if status != 0:
        raise W8A8Error(status, lib().w8a8_last_error().decode(errors="replace"))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _qt(qt) -> int:
    if qt in (INT8, "int8", torch.int8):
        return INT8
    if qt in (E4M3, "e4m3", "fp8", torch.float8_e4m3fn):
        return E4M3
    raise ValueError("qtype must be int8 or e4m3")


def _gran(g) -> int:
    if g in (TENSOR, "tensor"):
        return TENSOR
    if g in (AXIS, "axis"):
        return AXIS
    raise ValueError("granularity must be tensor or axis")


def _code_dtype(qt: int):
    return torch.int8 if qt == INT8 else torch.float8_e4m3fn


def _cuda_2d(t, dtype, name):
    if not (t.is_cuda and t.dtype == dtype and t.dim() == 2 and t.is_contiguous()):
        raise ValueError("%s must be a contiguous 2-D %s CUDA tensor" % (name, dtype))


def _as_bytes(t):
    """View a code tensor (int8 / e4m3 / uint8) as raw bytes for pointer use."""
    return t.view(torch.uint8) if t.dtype != torch.uint8 else t


# --------------------------------------------------------------------------- sizes
def workspace_bytes(op: int, M: int, N: int, K: int, r: int = 0) -> int:
    return int(lib().w8a8_workspace_bytes(op, M, N, K, r))


def q8_0_bytes(n: int) -> int:
    return int(lib().q8_0_bytes(n))


def _workspace(op, M, N, K, r, device, ws):
    need = workspace_bytes(op, M, N, K, r)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
    elif ws.numel() * ws.element_size() < need:
        raise ValueError("workspace of %d bytes is smaller than the %d needed" % (ws.numel(), need))
    return ws


# --------------------------------------------------------------------------- quantizers
def quantize_rows(x: torch.Tensor, qt="int8", out=None, scale=None):
    """Token-wise absmax calibration + quantization of X [M, K] bf16 (one pass).
    Returns (codes [M, K] int8 or float8_e4m3fn, row scales [M] float32)."""
    qt = _qt(qt)
    if not (x.is_cuda and x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1):
        raise ValueError("x must be a 2-D bf16 CUDA tensor with unit column stride")
    M, K = x.shape
    q = torch.empty((M, K), dtype=_code_dtype(qt), device=x.device) if out is None else out
    s = torch.empty((M,), dtype=torch.float32, device=x.device) if scale is None else scale
    _check(lib().w8a8_quantize_rows(_ptr(x), M, K, x.stride(0), qt, _ptr(q), q.stride(0), _ptr(s),
                                    _stream(x.device)))
    return q, s


def quantize_weight(w: torch.Tensor, qt="int8", gran="tensor"):
    """Tensor-wise (scale [1]) or axis-wise (scale [N]) quantization of W [N, K] bf16."""
    qt, g = _qt(qt), _gran(gran)
    _cuda_2d(w, torch.bfloat16, "w")
    N, K = w.shape
    q = torch.empty((N, K), dtype=_code_dtype(qt), device=w.device)
    s = torch.empty((N if g == AXIS else 1,), dtype=torch.float32, device=w.device)
    ws = torch.empty(256, dtype=torch.uint8, device=w.device) if g == TENSOR else None
    _check(lib().w8a8_quantize_weight(_ptr(w), N, K, qt, g, _ptr(q), _ptr(s), _ptr(ws),
                                      0 if ws is None else 256, _stream(w.device)))
    return q, s


def q8_0_quantize(x: torch.Tensor, out=None):
    """fp32 [n] -> GGUF Q8_0 blocks (uint8 [ceil(n/32)*34])."""
    if not (x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()):
        raise ValueError("x must be a contiguous fp32 CUDA tensor")
    n = x.numel()
    b = torch.empty(q8_0_bytes(n), dtype=torch.uint8, device=x.device) if out is None else out
    _check(lib().q8_0_quantize(_ptr(x), n, _ptr(b), _stream(x.device)))
    return b


def q8_0_dequantize(blocks: torch.Tensor, n: int, out=None):
    """GGUF Q8_0 blocks -> fp32 [n] (f16 scale x code)."""
    if not (blocks.is_cuda and blocks.dtype == torch.uint8 and blocks.is_contiguous()):
        raise ValueError("blocks must be a contiguous uint8 CUDA tensor")
    if blocks.numel() < q8_0_bytes(n):
        raise ValueError("blocks hold fewer than n values")
    y = torch.empty(n, dtype=torch.float32, device=blocks.device) if out is None else out
    _check(lib().q8_0_dequantize(_ptr(blocks), n, _ptr(y), _stream(blocks.device)))
    return y


def q8_0_dequantize_bf16(blocks: torch.Tensor, n: int, out=None):
    """GGUF Q8_0 blocks -> bf16 [n] (f16 scale x code, rounded to bf16)."""
    if not (blocks.is_cuda and blocks.dtype == torch.uint8 and blocks.is_contiguous()):
        raise ValueError("blocks must be a contiguous uint8 CUDA tensor")
    if blocks.numel() < q8_0_bytes(n):
        raise ValueError("blocks hold fewer than n values")
    y = torch.empty(n, dtype=torch.bfloat16, device=blocks.device) if out is None else out
    _check(lib().q8_0_dequantize_bf16(_ptr(blocks), n, _ptr(y), _stream(blocks.device)))
    return y


def dequantize_e4m3_bf16(wq: torch.Tensor, scale: torch.Tensor, out=None):
    """e4m3 codes (float8_e4m3fn) -> bf16(value * scale[0]), same shape."""
    if not (wq.is_cuda and wq.dtype == torch.float8_e4m3fn and wq.is_contiguous()):
        raise ValueError("wq must be a contiguous float8_e4m3fn CUDA tensor")
    y = torch.empty(wq.shape, dtype=torch.bfloat16, device=wq.device) if out is None else out
    _check(lib().w8a8_dequantize_e4m3_bf16(_ptr(_as_bytes(wq)), wq.numel(), _ptr(scale), _ptr(y),
                                           _stream(wq.device)))
    return y


def q8_0_to_axis(blocks: torch.Tensor, N: int, K: int, qt="int8", out=None, scale=None):
    """Q8_0 weight [N, K/32 blocks] -> (codes [N, K], per-row scales [N]):
    int8 codes (GGUF A8 int) or float8_e4m3fn codes (GGUF A8 float)."""
    qt = _qt(qt)
    if not (blocks.is_cuda and blocks.dtype == torch.uint8 and blocks.is_contiguous()):
        raise ValueError("blocks must be a contiguous uint8 CUDA tensor")
    if blocks.numel() < q8_0_bytes(N * K):
        raise ValueError("blocks hold fewer than N*K values")
    dt = _code_dtype(qt)
    q = torch.empty((N, K), dtype=dt, device=blocks.device) if out is None else out
    s = torch.empty((N,), dtype=torch.float32, device=blocks.device) if scale is None else scale
    if q.shape != (N, K) or q.dtype != dt or not q.is_contiguous() or s.numel() < N:
        raise ValueError("out must be a contiguous %s [N, K] tensor and scale hold N floats" % dt)
    fn = lib().q8_0_to_axis_int8 if qt == INT8 else lib().q8_0_to_axis_e4m3
    _check(fn(_ptr(blocks), N, K, _ptr(q), _ptr(s), _stream(blocks.device)))
    return q, s


def q8_0_to_axis_int8(blocks: torch.Tensor, N: int, K: int, out=None, scale=None):
    """Q8_0 weight [N, K/32 blocks] -> (int8 codes [N, K], per-row scales [N])."""
    return q8_0_to_axis(blocks, N, K, "int8", out, scale)


def q8_0_to_axis_e4m3(blocks: torch.Tensor, N: int, K: int, out=None, scale=None):
    """Q8_0 weight [N, K/32 blocks] -> (e4m3 codes [N, K] as float8_e4m3fn, per-row scales [N])."""
    return q8_0_to_axis(blocks, N, K, "e4m3", out, scale)


# --------------------------------------------------------------------------- Linear
def linear_fwd(x, wq, w_scale, bias=None, out=None, ws=None):
    """Y = bf16(((Q(X) Q(W)^T) * s_x) * s_w + bias).  x [M, K] bf16, wq [N, K]
    int8 or float8_e4m3fn, w_scale [1] (tensor-wise) or [N] (axis-wise)."""
    _cuda_2d(x, torch.bfloat16, "x")
    qt = _qt(wq.dtype)
    M, K = x.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError("wq must be [N, K]")
    g = AXIS if w_scale.numel() > 1 else TENSOR
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if out is None else out
    ws = _workspace(OP_LINEAR_FWD, M, N, K, 0, x.device, ws)
    _check(lib().w8a8_linear_fwd(_ptr(x), M, N, K, qt, _ptr(_as_bytes(wq)), _ptr(w_scale), g, _ptr(bias),
                                 _ptr(y), _ptr(ws), ws.numel(), _stream(x.device)))
    return y


def bf16_linear_fwd(x, w, bias=None, out=None, ws=None):
    """Y = bf16(X W^T + bias) on the tensor cores: x [M, K], w [N, K] bf16."""
    _cuda_2d(x, torch.bfloat16, "x")
    _cuda_2d(w, torch.bfloat16, "w")
    M, K = x.shape
    N = w.shape[0]
    if w.shape[1] != K:
        raise ValueError("w must be [N, K]")
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if out is None else out
    ws = _workspace(OP_BF16_FWD, M, N, K, 0, x.device, ws)
    _check(lib().bf16_linear_fwd(_ptr(x), M, N, K, _ptr(w), _ptr(bias), _ptr(y), _ptr(ws), ws.numel(),
                                 _stream(x.device)))
    return y


def float8_linear_fwd(x, wq, w_scale, bias=None, out=None, ws=None):
    """Weight-only float8: W = bf16(dec(wq) * w_scale[0]) [N, K], then the bf16
    Linear.  wq float8_e4m3fn [N, K] (tensor-wise), w_scale [1]."""
    _cuda_2d(x, torch.bfloat16, "x")
    if wq.dtype != torch.float8_e4m3fn or wq.dim() != 2 or wq.shape[1] != x.shape[1]:
        raise ValueError("wq must be float8_e4m3fn [N, K]")
    M, K = x.shape
    N = wq.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if out is None else out
    ws = _workspace(OP_WEIGHT_ONLY_FWD, M, N, K, 0, x.device, ws)
    _check(lib().float8_linear_fwd(_ptr(x), M, N, K, _ptr(_as_bytes(wq)), _ptr(w_scale), _ptr(bias), _ptr(y),
                                   _ptr(ws), ws.numel(), _stream(x.device)))
    return y


def gguf_linear_fwd(x, blocks, N, bias=None, out=None, ws=None):
    """GGUF (weight-only): W = bf16(f16(d) q) from the Q8_0 blocks of the
    row-major [N, K] weight, then the bf16 Linear."""
    _cuda_2d(x, torch.bfloat16, "x")
    M, K = x.shape
    if not (blocks.is_cuda and blocks.dtype == torch.uint8 and blocks.is_contiguous()):
        raise ValueError("blocks must be a contiguous uint8 CUDA tensor")
    if blocks.numel() < q8_0_bytes(N * K):
        raise ValueError("blocks hold fewer than N*K values")
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if out is None else out
    ws = _workspace(OP_WEIGHT_ONLY_FWD, M, N, K, 0, x.device, ws)
    _check(lib().gguf_linear_fwd(_ptr(x), M, N, K, _ptr(blocks), _ptr(bias), _ptr(y), _ptr(ws), ws.numel(),
                                 _stream(x.device)))
    return y


def linear_fwd_ex(x, wq, w_scale, bias=None, act="none", x_amax=None, y_amax=None, out=None, ws=None):
    """linear_fwd for a chain of projections: optional activation ("gelu",
    "gelu_tanh") on the fp32 epilogue value; y_amax (int32 [M] CUDA tensor)
    receives the rows' max |y| as fp32 bits; x_amax supplies the rows' max |x|
    (e.g. the previous call's y_amax) so the quantizer skips its reduction."""
    _cuda_2d(x, torch.bfloat16, "x")
    qt = _qt(wq.dtype)
    M, K = x.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError("wq must be [N, K]")
    for name, a in (("x_amax", x_amax), ("y_amax", y_amax)):
        if a is not None and not (a.is_cuda and a.dtype == torch.int32 and a.is_contiguous() and a.numel() >= M):
            raise ValueError("%s must be a contiguous int32 CUDA tensor of at least M entries" % name)
    g = AXIS if w_scale.numel() > 1 else TENSOR
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if out is None else out
    ws = _workspace(OP_LINEAR_FWD, M, N, K, 0, x.device, ws)
    _check(lib().w8a8_linear_fwd_ex(_ptr(x), M, N, K, qt, _ptr(_as_bytes(wq)), _ptr(w_scale), g, _ptr(bias),
                                    ACTS[act], _ptr(x_amax), _ptr(y_amax), _ptr(y), _ptr(ws), ws.numel(),
                                    _stream(x.device)))
    return y


def _dgrad_out(dy, K, out):
    _cuda_2d(dy, torch.bfloat16, "dy")
    M, N = dy.shape
    return M, N, (torch.empty((M, K), dtype=torch.bfloat16, device=dy.device) if out is None else out)


def bf16_linear_dgrad(dy, w, out=None, ws=None):
    """dX = bf16(dY W): dy [M, N], w [N, K] bf16."""
    _cuda_2d(w, torch.bfloat16, "w")
    N, K = w.shape
    M, N2, dx = _dgrad_out(dy, K, out)
    if N2 != N:
        raise ValueError("dy must be [M, N] with w [N, K]")
    ws = _workspace(OP_BF16_DGRAD, M, N, K, 0, dy.device, ws)
    _check(lib().bf16_linear_dgrad(_ptr(dy), M, N, K, _ptr(w), _ptr(dx), _ptr(ws), ws.numel(), _stream(dy.device)))
    return dx


def float8_linear_dgrad(dy, wq, w_scale, out=None, ws=None):
    """Weight-only float8 input gradient: dX = bf16(dY W), W = bf16(dec(wq) w_scale[0])."""
    if wq.dtype != torch.float8_e4m3fn or wq.dim() != 2:
        raise ValueError("wq must be float8_e4m3fn [N, K]")
    N, K = wq.shape
    M, N2, dx = _dgrad_out(dy, K, out)
    if N2 != N:
        raise ValueError("dy must be [M, N] with wq [N, K]")
    ws = _workspace(OP_WEIGHT_ONLY_DGRAD, M, N, K, 0, dy.device, ws)
    _check(lib().float8_linear_dgrad(_ptr(dy), M, N, K, _ptr(_as_bytes(wq)), _ptr(w_scale), _ptr(dx), _ptr(ws),
                                     ws.numel(), _stream(dy.device)))
    return dx


def gguf_linear_dgrad(dy, blocks, K, out=None, ws=None):
    """GGUF input gradient: dX = bf16(dY W), W = bf16(f16(d) q) [N, K] from the Q8_0 blocks."""
    M, N, dx = _dgrad_out(dy, K, out)
    if blocks.numel() < q8_0_bytes(N * K):
        raise ValueError("blocks hold fewer than N*K values")
    ws = _workspace(OP_WEIGHT_ONLY_DGRAD, M, N, K, 0, dy.device, ws)
    _check(lib().gguf_linear_dgrad(_ptr(dy), M, N, K, _ptr(blocks), _ptr(dx), _ptr(ws), ws.numel(),
                                   _stream(dy.device)))
    return dx


def linear_fwd_noalloc(x, wq, w_scale, out, bias=None):
    """linear_fwd for callers that cannot provide scratch memory: the library
    keeps the activation codes in its own fixed device array (M*K and M are
    bounded; see include/w8a8.h).  The output `out` [M, N] bf16 is the caller's."""
    _cuda_2d(x, torch.bfloat16, "x")
    qt = _qt(wq.dtype)
    M, K = x.shape
    N = wq.shape[0]
    g = AXIS if w_scale.numel() > 1 else TENSOR
    _check(lib().w8a8_linear_fwd_noalloc(_ptr(x), M, N, K, qt, _ptr(_as_bytes(wq)), _ptr(w_scale), g,
                                         _ptr(bias), _ptr(out), _stream(x.device)))
    return out


def linear_dgrad(dy, wq, w_scale, out=None, ws=None):
    """dX = bf16((Q(dY) Q(W)) * s_dy * s_w): dy [M, N] bf16, wq [N, K], tensor-wise w_scale."""
    _cuda_2d(dy, torch.bfloat16, "dy")
    qt = _qt(wq.dtype)
    M, N = dy.shape
    K = wq.shape[1]
    if wq.shape[0] != N:
        raise ValueError("wq must be [N, K]")
    dx = torch.empty((M, K), dtype=torch.bfloat16, device=dy.device) if out is None else out
    ws = _workspace(OP_LINEAR_DGRAD, M, N, K, 0, dy.device, ws)
    _check(lib().w8a8_linear_dgrad(_ptr(dy), M, N, K, qt, _ptr(_as_bytes(wq)), _ptr(w_scale), TENSOR,
                                   _ptr(dx), _ptr(ws), ws.numel(), _stream(dy.device)))
    return dx


def qgemm_fwd(xq, x_scale, wq, w_scale, bias=None, out=None):
    """Tensor-core product + epilogue on codes already quantized (xq [M, K])."""
    qt = _qt(wq.dtype)
    M, K = xq.shape
    N = wq.shape[0]
    g = AXIS if w_scale.numel() > 1 else TENSOR
    y = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device) if out is None else out
    _check(lib().w8a8_qgemm_fwd(_ptr(_as_bytes(xq)), xq.stride(0), _ptr(x_scale), M, N, K, qt,
                                _ptr(_as_bytes(wq)), _ptr(w_scale), g, _ptr(bias), _ptr(y), _stream(xq.device)))
    return y


def qgemm_dgrad(dyq, dy_scale, wq, w_scale, out=None):
    """dX = epilogue(dyq wq) on codes already quantized (dyq [M, N], wq [N, K])."""
    qt = _qt(wq.dtype)
    M, N = dyq.shape
    K = wq.shape[1]
    dx = torch.empty((M, K), dtype=torch.bfloat16, device=dyq.device) if out is None else out
    _check(lib().w8a8_qgemm_dgrad(_ptr(_as_bytes(dyq)), dyq.stride(0), _ptr(dy_scale), M, N, K, qt,
                                  _ptr(_as_bytes(wq)), _ptr(w_scale), _ptr(dx), _stream(dyq.device)))
    return dx


def svdq_linear_fwd(x, rq, r_scale, l1, l2, bias=None, out=None, ws=None):
    """SVDQuant forward: Y = epilogue(Q(X) Rq^T) + bf16(X L1) L2.
    x [M, K] bf16, rq [N, K] int8 (int W8A8) or float8_e4m3fn (float W8A8),
    r_scale [1], l1 [K, r] bf16, l2 [r, N] bf16."""
    _cuda_2d(x, torch.bfloat16, "x")
    M, K = x.shape
    N = rq.shape[0]
    r = l1.shape[1]
    if l1.shape[0] != K or tuple(l2.shape) != (r, N):
        raise ValueError("l1 must be [K, r] and l2 [r, N]")
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if out is None else out
    ws = _workspace(OP_SVDQ_FWD, M, N, K, r, x.device, ws)
    if rq.dtype == torch.int8:
        fn = lib().svdq_linear_fwd
    elif rq.dtype == torch.float8_e4m3fn:
        fn = lib().svdq_linear_fwd_e4m3
    else:
        raise ValueError("rq must hold int8 or float8_e4m3fn codes")
    _check(fn(_ptr(x), M, N, K, _ptr(_as_bytes(rq)), _ptr(r_scale), r, _ptr(l1), _ptr(l2),
              _ptr(bias), _ptr(y), _ptr(ws), ws.numel(), _stream(x.device)))
    return y


# The SVDQuant weight split is offline preparation, kept out of this binding:
# see weight_prep.py (svd_split, svdq_prepare).
from .weight_prep import svd_split, svdq_prepare  # noqa: E402,F401


# --------------------------------------------------------------------------- diagnostics
def device_status(reset: bool = True, stream=None) -> int:
    """Synchronize and return the first device-side error code (0 = none)."""
    s = ctypes.c_void_p(stream.cuda_stream) if stream is not None else _stream()
    return int(lib().w8a8_device_status(s, 1 if reset else 0))


def set_wait_limit_ns(limit_ns: int):
    _check(lib().w8a8_set_wait_limit_ns(int(limit_ns)))


def selftest_wait(limit_ns: int):
    _check(lib().w8a8_selftest_wait(int(limit_ns), _stream()))


def selftest_bounds():
    """One failing device-side index check (no memory touched): the debug
    build records W8A8_ERR_DEVICE_BOUNDS, the release build nothing."""
    _check(lib().w8a8_selftest_bounds(_stream()))


def debug_checks() -> bool:
    """True when the loaded library is the debug build with index checks."""
    return bool(lib().w8a8_debug_checks())


def e4m3_encode(x: torch.Tensor):
    """fp32 -> E4M3FN codes with the device conversion the quantizers use."""
    if not (x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()):
        raise ValueError("x must be a contiguous fp32 CUDA tensor")
    y = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(lib().w8a8_e4m3_encode(_ptr(x), x.numel(), _ptr(y), _stream(x.device)))
    return y
