"""Plain CPU oracle for the W8A8 quantized Linear.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg are the only callers.  The product path (the CUDA
library and its binding) never imports this package, and this package never
imports the product.

The scalar arithmetic lives in ``oracle.c`` (plain loops, fp32 operations
rounded one at a time, fp64 where the reading asks for it); this module
composes those steps in the order the pages give them:

* OneTrainer wiki "Quantization", int W8A8 / float W8A8 paragraphs: weights
  quantized tensor-wise, activations token-wise, the Linear matmul in 8 bits.
* OneTrainer wiki "Quantization", float8 and GGUF paragraphs (weight-only):
  the weight dequantized to the train data type (bf16), then a bf16 Linear.
* OneTrainer wiki "Quantization", GGUF A8 int / GGUF A8 float paragraphs:
  GGUF weights re-quantized axis-wise to int8 / to float8 (e4m3).
* bitsandbytes #1401 "LLM.int8() Refactoring: Part 1", Enhancements: the fused
  row calibrate-and-quantize op (int8_vectorwise_quant).
* entrenar 0.7.8 ``src/quant/gguf_quant/q8_0.rs``: the Q8_0 format.
* OneTrainer PR #1034 "SVDQuant" and the wiki's SVDQuant paragraph: the
  low-rank split with bfloat16 factors (``svdquant.py``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

INT8, E4M3 = 0, 1
TENSOR, AXIS = 0, 1
QMAX = {INT8: 127.0, E4M3: 448.0}


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (gcc, OpenMP, no FMA contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= max(os.path.getmtime(_SRC),
                                                    os.path.getmtime(os.path.join(_HERE, "oracle.h")))):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def _declare(L):
    sig = {
        "orc_bf16_to_f32_n": [_P, _P, _I64],
        "orc_f32_to_bf16_n": [_P, _P, _I64],
        "orc_f16_to_f32_n": [_P, _P, _I64],
        "orc_f32_to_f16_n": [_P, _P, _I64],
        "orc_e4m3_to_f32_n": [_P, _P, _I64],
        "orc_f32_to_e4m3_n": [_P, _P, _I64],
        "orc_quantize_rows": [_P, _I64, _I64, _I64, ctypes.c_int, _P, _P],
        "orc_quantize_weight": [_P, _I64, _I64, ctypes.c_int, ctypes.c_int, _P, _P],
        "orc_q8_0_quantize": [_P, _I64, _P, _P],
        "orc_q8_0_dequantize": [_P, _I64, _P],
        "orc_q8_0_dequantize_f32": [_P, _P, _I64, _P],
        "orc_q8_0_to_axis_int8": [_P, _I64, _I64, _P, _P],
        "orc_q8_0_to_axis": [_P, _I64, _I64, ctypes.c_int, _P, _P],
        "orc_dequant_e4m3_bf16": [_P, _I64, ctypes.c_float, _P],
        "orc_act": [_P, _I64, ctypes.c_int, _P],
        "orc_row_absmax_bf16": [_P, _I64, _I64, _P],
        "orc_q8_0_dequantize_bf16": [_P, _I64, _P],
        "orc_linear_bf16": [_P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P],
        "orc_gemm_i8_nt": [_P, _P, _I64, _I64, _I64, _P],
        "orc_gemm_i8_nn": [_P, _P, _I64, _I64, _I64, _P],
        "orc_gemm_e4m3_nt": [_P, _P, _I64, _I64, _I64, _P, _P],
        "orc_gemm_e4m3_nn": [_P, _P, _I64, _I64, _I64, _P, _P],
        "orc_epilogue_i32": [_P, _I64, _I64, _P, _P, ctypes.c_int, _P, _P, _P],
        "orc_epilogue_f64": [_P, _I64, _I64, _P, _P, ctypes.c_int, _P, _P, _P],
        "orc_lowrank_down": [_P, _P, _I64, _I64, _I64, _P, _P],
        "orc_lowrank_up": [_P, _P, _I64, _I64, _I64, _P, _P],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = None
    L.orc_q8_0_bytes.argtypes = [_I64]
    L.orc_q8_0_bytes.restype = _I64
    L.orc_gemm_i8_nt.restype = ctypes.c_int
    L.orc_gemm_i8_nn.restype = ctypes.c_int


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------- codecs
def bf16_to_f32(h):
    h = _c(h, np.uint16)
    out = np.empty(h.shape, np.float32)
    lib().orc_bf16_to_f32_n(_ptr(h), _ptr(out), h.size)
    return out


def f32_to_bf16(f):
    f = _c(f, np.float32)
    out = np.empty(f.shape, np.uint16)
    lib().orc_f32_to_bf16_n(_ptr(f), _ptr(out), f.size)
    return out


def f16_to_f32(h):
    h = _c(h, np.uint16)
    out = np.empty(h.shape, np.float32)
    lib().orc_f16_to_f32_n(_ptr(h), _ptr(out), h.size)
    return out


def f32_to_f16(f):
    f = _c(f, np.float32)
    out = np.empty(f.shape, np.uint16)
    lib().orc_f32_to_f16_n(_ptr(f), _ptr(out), f.size)
    return out


def e4m3_to_f32(c):
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float32)
    lib().orc_e4m3_to_f32_n(_ptr(c), _ptr(out), c.size)
    return out


def f32_to_e4m3(f):
    f = _c(f, np.float32)
    out = np.empty(f.shape, np.uint8)
    lib().orc_f32_to_e4m3_n(_ptr(f), _ptr(out), f.size)
    return out


def decode_codes(q, qt):
    """Code bytes -> float32 values (int8 as signed integers, e4m3 decoded)."""
    q = _c(q, np.uint8)
    if qt == E4M3:
        return e4m3_to_f32(q)
    return q.view(np.int8).astype(np.float32)


# --------------------------------------------------------------------------- quantizers
def quantize_rows(x_bf16, qt=INT8):
    """Token-wise absmax calibration + quantization of X[M,K] (bf16 bits).

    Returns (codes uint8 [M,K], scales float32 [M])."""
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.uint8)
    s = np.empty((M,), np.float32)
    lib().orc_quantize_rows(_ptr(x), M, K, K, qt, _ptr(q), _ptr(s))
    return q, s


def quantize_weight(w_bf16, qt=INT8, gran=TENSOR):
    """Tensor-wise (scale [1]) or axis-wise (scale [N]) weight quantization."""
    w = _c(w_bf16, np.uint16)
    N, K = w.shape
    q = np.empty((N, K), np.uint8)
    s = np.empty((N if gran == AXIS else 1,), np.float32)
    lib().orc_quantize_weight(_ptr(w), N, K, qt, gran, _ptr(q), _ptr(s))
    return q, s


# --------------------------------------------------------------------------- Q8_0
def q8_0_bytes(n):
    return int(lib().orc_q8_0_bytes(n))


def q8_0_quantize(x_f32):
    """Q8_0 blocks (uint8 [ceil(n/32)*34]) and the per-block f32 scales."""
    x = _c(x_f32, np.float32).reshape(-1)
    n = x.size
    blocks = np.empty((q8_0_bytes(n),), np.uint8)
    scales = np.empty(((n + 31) // 32,), np.float32)
    lib().orc_q8_0_quantize(_ptr(x), n, _ptr(blocks), _ptr(scales))
    return blocks, scales


def q8_0_dequantize(blocks, n):
    b = _c(blocks, np.uint8).reshape(-1)
    y = np.empty((n,), np.float32)
    lib().orc_q8_0_dequantize(_ptr(b), n, _ptr(y))
    return y


def q8_0_dequantize_f32(scales_f32, codes, n):
    s = _c(scales_f32, np.float32)
    c = _c(codes, np.int8)
    y = np.empty((n,), np.float32)
    lib().orc_q8_0_dequantize_f32(_ptr(s), _ptr(c), n, _ptr(y))
    return y


def q8_0_codes(blocks, n):
    """The int8 codes of the first n values (block layout: 2-byte scale, 32 codes)."""
    b = _c(blocks, np.uint8).reshape(-1, 34)
    return b[:, 2:].reshape(-1)[:n].view(np.int8).copy()


def q8_0_scales_f16(blocks):
    b = _c(blocks, np.uint8).reshape(-1, 34)
    return np.ascontiguousarray(b[:, :2]).view(np.uint16).reshape(-1).copy()


def q8_0_to_axis(blocks, N, K, qt):
    """Q8_0 [N, K/32 blocks] -> axis-wise codes [N, K] (int8 for qt 0, e4m3
    bytes for qt 1) and the row scales [N]."""
    b = _c(blocks, np.uint8)
    q = np.empty((N, K), np.int8 if qt == 0 else np.uint8)
    s = np.empty((N,), np.float32)
    lib().orc_q8_0_to_axis(_ptr(b), N, K, qt, _ptr(q), _ptr(s))
    return q, s


def q8_0_to_axis_int8(blocks, N, K):
    b = _c(blocks, np.uint8)
    q = np.empty((N, K), np.int8)
    s = np.empty((N,), np.float32)
    lib().orc_q8_0_to_axis_int8(_ptr(b), N, K, _ptr(q), _ptr(s))
    return q, s


# --------------------------------------------------------------------------- GEMMs
def gemm_i8_nt(A, B):
    """acc[m,n] = sum_k A[m,k] B[n,k], int64 sums checked into int32."""
    A = _c(A, np.uint8).view(np.int8)
    B = _c(B, np.uint8).view(np.int8)
    M, K = A.shape
    N = B.shape[0]
    acc = np.empty((M, N), np.int32)
    if lib().orc_gemm_i8_nt(_ptr(A), _ptr(B), M, N, K, _ptr(acc)):
        raise OverflowError("int8 GEMM sum leaves the int32 range")
    return acc


def gemm_i8_nn(A, B):
    """acc[m,k] = sum_n A[m,n] B[n,k] (contraction along B's rows)."""
    A = _c(A, np.uint8).view(np.int8)
    B = _c(B, np.uint8).view(np.int8)
    M, N = A.shape
    K = B.shape[1]
    acc = np.empty((M, K), np.int32)
    if lib().orc_gemm_i8_nn(_ptr(A), _ptr(B), M, N, K, _ptr(acc)):
        raise OverflowError("int8 GEMM sum leaves the int32 range")
    return acc


def gemm_e4m3_nt(A, B):
    A = _c(A, np.uint8)
    B = _c(B, np.uint8)
    M, K = A.shape
    N = B.shape[0]
    acc = np.empty((M, N), np.float64)
    absacc = np.empty((M, N), np.float64)
    lib().orc_gemm_e4m3_nt(_ptr(A), _ptr(B), M, N, K, _ptr(acc), _ptr(absacc))
    return acc, absacc


def gemm_e4m3_nn(A, B):
    A = _c(A, np.uint8)
    B = _c(B, np.uint8)
    M, N = A.shape
    K = B.shape[1]
    acc = np.empty((M, K), np.float64)
    absacc = np.empty((M, K), np.float64)
    lib().orc_gemm_e4m3_nn(_ptr(A), _ptr(B), M, N, K, _ptr(acc), _ptr(absacc))
    return acc, absacc


# --------------------------------------------------------------------------- epilogue
def epilogue(acc, s_row, s_w, bias=None):
    """((acc * s_row) * s_w) (+ bias) -> (y bf16 bits, y fp32).

    int32 acc: fp32 operations rounded one by one.  fp64 acc (the e4m3 path):
    the same in fp64, rounded once to fp32."""
    s_row = _c(s_row, np.float32)
    s_w = _c(s_w, np.float32)
    M, N = acc.shape
    w_axis = 1 if s_w.size > 1 else 0
    if w_axis:
        assert s_w.size == N
    b = None if bias is None else _c(bias, np.uint16)
    y = np.empty((M, N), np.uint16)
    y32 = np.empty((M, N), np.float32)
    if acc.dtype == np.int32:
        a = _c(acc, np.int32)
        lib().orc_epilogue_i32(_ptr(a), M, N, _ptr(s_row), _ptr(s_w), w_axis, _ptr(b), _ptr(y32), _ptr(y))
    else:
        a = _c(acc, np.float64)
        lib().orc_epilogue_f64(_ptr(a), M, N, _ptr(s_row), _ptr(s_w), w_axis, _ptr(b), _ptr(y32), _ptr(y))
    return y, y32


# --------------------------------------------------------------------------- composed ops
ACT_NONE, ACT_GELU, ACT_GELU_TANH = 0, 1, 2


def act_f32(v, act):
    """The activation of fp32 values (double math, one rounding to fp32)."""
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.float32)
    lib().orc_act(_ptr(v), v.size, act, _ptr(out))
    return out


def row_absmax_bf16(y_bf16):
    """max_n |y[m, n]| of bf16 values, fp32 [M]."""
    y = _c(y_bf16, np.uint16)
    M, N = y.shape
    a = np.empty((M,), np.float32)
    lib().orc_row_absmax_bf16(_ptr(y), M, N, _ptr(a))
    return a


def linear_fwd(x_bf16, wq, s_w, qt=INT8, bias=None, act=ACT_NONE):
    """W8A8 Linear forward: Q(X) token-wise, 8-bit matmul with Q(W), epilogue,
    then the optional activation on the fp32 epilogue value.

    Returns a dict: y (bf16 bits), y32, xq, sx, acc and, for e4m3, absacc
    (sum |a*b| per output, for the fp8 tolerance); with an activation also
    pre (the fp32 value it was applied to); amax = the rows' max |y|."""
    xq, sx = quantize_rows(x_bf16, qt)
    out = {"xq": xq, "sx": sx}
    if qt == INT8:
        acc = gemm_i8_nt(xq, wq)
    else:
        acc, absacc = gemm_e4m3_nt(xq, wq)
        out["absacc"] = absacc
    out["acc"] = acc
    out["y"], out["y32"] = epilogue(acc, sx, s_w, bias)
    if act != ACT_NONE:
        out["pre"] = out["y32"]
        out["y32"] = act_f32(out["pre"], act)
        out["y"] = f32_to_bf16(out["y32"])
    out["amax"] = row_absmax_bf16(out["y"])
    return out


def linear_dgrad(dy_bf16, wq, s_w, qt=INT8):
    """dX = Q(dY) Q(W): dY token-wise quantized, contraction over the weight's
    output dimension (the rows of W[N,K]), epilogue with s_dy[m] * s_w."""
    s_w = _c(s_w, np.float32)
    if s_w.size != 1:
        raise ValueError("dgrad reads a tensor-wise weight scale")
    dyq, sdy = quantize_rows(dy_bf16, qt)
    out = {"xq": dyq, "sx": sdy}
    if qt == INT8:
        acc = gemm_i8_nn(dyq, wq)
    else:
        acc, absacc = gemm_e4m3_nn(dyq, wq)
        out["absacc"] = absacc
    out["acc"] = acc
    out["y"], out["y32"] = epilogue(acc, sdy, s_w, None)
    return out


def lowrank_down(x_bf16, l1_bf16):
    x = _c(x_bf16, np.uint16)
    l1 = _c(l1_bf16, np.uint16)
    M, K = x.shape
    r = l1.shape[1]
    t64 = np.empty((M, r), np.float64)
    t = np.empty((M, r), np.uint16)
    lib().orc_lowrank_down(_ptr(x), _ptr(l1), M, K, r, _ptr(t64), _ptr(t))
    return t, t64


def lowrank_up(t_bf16, l2_bf16):
    t = _c(t_bf16, np.uint16)
    l2 = _c(l2_bf16, np.uint16)
    M, r = t.shape
    N = l2.shape[1]
    lr = np.empty((M, N), np.float64)
    lr_abs = np.empty((M, N), np.float64)
    lib().orc_lowrank_up(_ptr(t), _ptr(l2), M, r, N, _ptr(lr), _ptr(lr_abs))
    return lr, lr_abs


def svdq_linear_fwd(x_bf16, rq, s_r, l1_bf16, l2_bf16, bias=None, qt=INT8):
    """SVDQuant forward: Y = epilogue(Q(X) Q(R)) + (X L1) L2, bf16 out, with
    int8 (int W8A8) or e4m3 (float W8A8) codes for X and R.

    T = bf16(X L1) [M,r]; lr = T L2 accumulated exactly (fp64) and rounded to
    fp32 before the add.  Returns the 8-bit part, T, lr and the bound inputs."""
    base = linear_fwd(x_bf16, rq, s_r, qt, bias)
    t, t64 = lowrank_down(x_bf16, l1_bf16)
    lr, lr_abs = lowrank_up(t, l2_bf16)
    y32 = (base["y32"] + lr.astype(np.float32)).astype(np.float32)
    base.update({"t": t, "t64": t64, "lr": lr, "lr_abs": lr_abs,
                 "y32": y32, "y": f32_to_bf16(y32), "y32_int": base["y32"]})
    return base


# --------------------------------------------------------------------------- weight-only types
def dequant_e4m3_bf16(q, s):
    """Weight-only float8: bf16 bits of dec(q) * s (fp32 RN product)."""
    q = _c(q, np.uint8)
    w = np.empty(q.shape, np.uint16)
    lib().orc_dequant_e4m3_bf16(_ptr(q), q.size, float(np.float32(_c(s, np.float32).reshape(-1)[0])), _ptr(w))
    return w


def q8_0_dequantize_bf16(blocks, n):
    """GGUF to the train data type: bf16 bits of f16(d) * q, n values."""
    b = _c(blocks, np.uint8)
    w = np.empty((n,), np.uint16)
    lib().orc_q8_0_dequantize_bf16(_ptr(b), n, _ptr(w))
    return w


def linear_bf16(x_bf16, w_bf16, bias=None):
    """bf16 Linear: returns dict(y bf16 bits, y32, acc fp64, absacc)."""
    x = _c(x_bf16, np.uint16)
    w = _c(w_bf16, np.uint16)
    M, K = x.shape
    N = w.shape[0]
    b = None if bias is None else _c(bias, np.uint16)
    acc = np.empty((M, N), np.float64)
    absacc = np.empty((M, N), np.float64)
    y32 = np.empty((M, N), np.float32)
    y = np.empty((M, N), np.uint16)
    lib().orc_linear_bf16(_ptr(x), _ptr(w), M, N, K, _ptr(b), _ptr(acc), _ptr(absacc), _ptr(y32), _ptr(y))
    return {"y": y, "y32": y32, "acc": acc, "absacc": absacc}


def float8_linear_fwd(x_bf16, wq, s_w, bias=None):
    """Weight-only float8 forward: W = bf16(dec(Wq) s_w), then the bf16 Linear."""
    wq = _c(wq, np.uint8)
    return linear_bf16(x_bf16, dequant_e4m3_bf16(wq, s_w).reshape(wq.shape), bias)


def gguf_linear_fwd(x_bf16, blocks, N, K, bias=None):
    """GGUF (weight-only) forward: W = bf16(f16(d) q) [N, K], then the bf16 Linear."""
    return linear_bf16(x_bf16, q8_0_dequantize_bf16(blocks, N * K).reshape(N, K), bias)


def linear_bf16_dgrad(dy_bf16, w_bf16):
    """dX = bf16(fp32(dY W)): the bf16 Linear with the explicit transposed
    weight W^T [K, N] (the contraction runs over W's rows)."""
    w = _c(w_bf16, np.uint16)
    return linear_bf16(dy_bf16, np.ascontiguousarray(w.T))
