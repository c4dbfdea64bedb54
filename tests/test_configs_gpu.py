"""Parity at the workloads' full sizes, in the launch configuration the bench
times.  Each step is row-local (token scales are per row, weights fixed), so
the oracle recomputes a seeded sample of whole output rows - plus the last
128-row tile - from the same inputs; the GPU computes everything.

With W8A8_FULL_PARITY=1 in the environment every row is compared instead of
a sample: all outputs of every workload here, e.g. the four outputs of the
DiT MLP block and the 16384-token GGUF forward, against the oracle on all
host cores (a few minutes)."""
import os

import numpy as np
import pytest
import torch

import workloads
from _tol import bf16_bits_to_f64, ulp_bf16

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


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def u8(t):
    return t.detach().cpu().contiguous().view(torch.uint8).numpy()


FULL = os.environ.get("W8A8_FULL_PARITY", "") not in ("", "0")


def sample_rows(M, n=192, seed=0):
    """A seeded sample of n rows plus row 0 and the last 128-row tile; every
    row in full-parity mode."""
    if FULL:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(M, size=min(n, M), replace=False).tolist())
    rows |= set(range(max(0, M - 128), M)) | {0}
    return np.array(sorted(rows))


def test_int_tiny_full(w8, orc):
    d = workloads.int_tiny()
    wq, sw = w8.quantize_weight(d["w"].to(DEV), "int8", "tensor")
    y = w8.linear_fwd(d["x"].to(DEV), wq, sw)
    wqr, swr = orc.quantize_weight(workloads.to_u16(d["w"]), 0, 0)
    assert np.array_equal(u8(wq), wqr) and float(sw) == swr[0]
    ref = orc.linear_fwd(workloads.to_u16(d["x"]), wqr, swr)
    assert np.array_equal(u16(y), ref["y"])


def test_float_w8a8_sampled(w8, orc):
    d = workloads.float_w8a8()
    wq, sw = w8.quantize_weight(d["w"].to(DEV), "e4m3", "tensor")
    y = w8.linear_fwd(d["x"].to(DEV), wq, sw, bias=d["bias"].to(DEV))
    wqr, swr = orc.quantize_weight(workloads.to_u16(d["w"]), 1, 0)
    assert np.array_equal(u8(wq), wqr)
    rows = sample_rows(d["x"].shape[0])
    ref = orc.linear_fwd(workloads.to_u16(d["x"])[rows], wqr, swr, qt=1, bias=workloads.to_u16(d["bias"]))
    yr = bf16_bits_to_f64(ref["y"])
    yg = bf16_bits_to_f64(u16(y)[rows])
    bound = 1e-3 * ref["sx"][:, None].astype(np.float64) * swr[0] * ref["absacc"] \
        + ulp_bf16(np.maximum(np.abs(yr), np.abs(yg)))
    assert np.all(np.abs(yg - yr) <= bound)


def test_dit_mlp_block_fwd_dgrad_sampled(w8, orc):
    """up-proj 3072->12288, down-proj 12288->3072, then dgrad through both
    (dX2 = Q(dY2) Q(W2), dX1 = Q(dX2) Q(W1)); int8 codes, tensor-wise W."""
    d = workloads.dit_mlp()
    W1q, s1 = w8.quantize_weight(d["w1"].to(DEV), "int8", "tensor")
    W2q, s2 = w8.quantize_weight(d["w2"].to(DEV), "int8", "tensor")
    y1 = w8.linear_fwd(d["x"].to(DEV), W1q, s1)
    y2 = w8.linear_fwd(y1, W2q, s2)
    dx2 = w8.linear_dgrad(d["dy2"].to(DEV), W2q, s2)
    dx1 = w8.linear_dgrad(dx2, W1q, s1)
    W1r, s1r = orc.quantize_weight(workloads.to_u16(d["w1"]), 0, 0)
    W2r, s2r = orc.quantize_weight(workloads.to_u16(d["w2"]), 0, 0)
    assert np.array_equal(u8(W1q), W1r) and np.array_equal(u8(W2q), W2r)
    rows = sample_rows(d["x"].shape[0], n=160)
    r1 = orc.linear_fwd(workloads.to_u16(d["x"])[rows], W1r, s1r)
    assert np.array_equal(u16(y1)[rows], r1["y"])
    r2 = orc.linear_fwd(r1["y"], W2r, s2r)
    assert np.array_equal(u16(y2)[rows], r2["y"])
    g2 = orc.linear_dgrad(workloads.to_u16(d["dy2"])[rows], W2r, s2r)
    assert np.array_equal(u16(dx2)[rows], g2["y"])
    g1 = orc.linear_dgrad(g2["y"], W1r, s1r)
    assert np.array_equal(u16(dx1)[rows], g1["y"])


def test_svdquant_sampled(w8, orc):
    from test_parity_gpu import _svdq_check
    d = workloads.svdquant()
    _svdq_check(w8, orc, d["x"], d["w"], d["r"], rows=sample_rows(d["x"].shape[0], n=96))


def test_svdquant_e4m3_sampled(w8, orc):
    """The SVDQuant workload with an e4m3 residual (float W8A8 + SVDQuant)."""
    from test_parity_gpu import _svdq_check
    d = workloads.svdquant()
    _svdq_check(w8, orc, d["x"], d["w"], d["r"], rows=sample_rows(d["x"].shape[0], n=96), qt=1)


def test_gguf_q8_0_requant_and_forward_sweep(w8, orc):
    d = workloads.gguf_q8_0(M=max(workloads.GGUF_MS))
    w = d["w_f32"]
    N, K = w.shape
    blocks = w8.q8_0_quantize(w.reshape(-1).to(DEV))
    br, _ = orc.q8_0_quantize(w.numpy().reshape(-1))
    assert np.array_equal(u8(blocks), br)
    wq, sw = w8.q8_0_to_axis_int8(blocks, N, K)
    wqr, swr = orc.q8_0_to_axis_int8(br, N, K)
    assert np.array_equal(u8(wq), wqr.view(np.uint8)) and np.array_equal(sw.cpu().numpy(), swr)
    xall = d["x"]
    for M in workloads.GGUF_MS:
        x = xall[:M]
        y = w8.linear_fwd(x.to(DEV), wq, sw)
        rows = sample_rows(M, n=64, seed=M)
        ref = orc.linear_fwd(workloads.to_u16(x)[rows], wqr.view(np.uint8), swr)
        assert np.array_equal(u16(y)[rows], ref["y"]), M


def test_gguf_a8_float_requant_and_forward_sweep(w8, orc):
    """GGUF A8 float at full size: the Q8_0 weight re-quantized to axis-wise
    e4m3 (bit for bit), then the e4m3 forward over the M sweep (sampled rows,
    the fp8 tolerance of the parity tests)."""
    from test_parity_gpu import _fp8_tol
    d = workloads.gguf_q8_0(M=max(workloads.GGUF_MS))
    w = d["w_f32"]
    N, K = w.shape
    blocks = w8.q8_0_quantize(w.reshape(-1).to(DEV))
    br, _ = orc.q8_0_quantize(w.numpy().reshape(-1))
    wq, sw = w8.q8_0_to_axis_e4m3(blocks, N, K)
    wqr, swr = orc.q8_0_to_axis(br, N, K, 1)
    assert np.array_equal(u8(wq), wqr) and np.array_equal(sw.cpu().numpy(), swr)
    xall = d["x"]
    for M in workloads.GGUF_MS:
        x = xall[:M]
        y = w8.linear_fwd(x.to(DEV), wq, sw)
        rows = sample_rows(M, n=32, seed=M)
        ref = orc.linear_fwd(workloads.to_u16(x)[rows], wqr, swr, qt=1)
        ref["sw"] = swr[None, :]
        err, bound = _fp8_tol(ref, u16(y)[rows])
        assert np.all(err <= bound), (M, float((err / bound).max()))


@pytest.mark.parametrize("kind", ["float8", "gguf"])
def test_weight_only_dit_up_sampled(w8, orc, kind):
    """The weight-only types on the DiT up-projection (X [4608, 3072], W
    [12288, 3072]): the whole product on the GPU, sampled rows by the oracle."""
    from test_parity_gpu import _bf16_tol
    d = workloads.gguf_q8_0(M=4608)
    w32 = d["w_f32"]
    N, K = w32.shape
    x = d["x"]
    rows = sample_rows(4608, n=24, seed=5)
    if kind == "float8":
        wb = w32.to(torch.bfloat16)
        wq, sw = w8.quantize_weight(wb.to(DEV), "e4m3", "tensor")
        y = w8.float8_linear_fwd(x.to(DEV), wq, sw)
        wqr, swr = orc.quantize_weight(workloads.to_u16(wb), 1, 0)
        assert np.array_equal(u8(wq), wqr)
        ref = orc.float8_linear_fwd(workloads.to_u16(x)[rows], wqr, swr)
    else:
        br, _ = orc.q8_0_quantize(w32.numpy().reshape(-1))
        y = w8.gguf_linear_fwd(x.to(DEV), torch.from_numpy(br).to(DEV), N)
        ref = orc.gguf_linear_fwd(workloads.to_u16(x)[rows], br, N, K)
    err, bound = _bf16_tol(ref, u16(y)[rows], K)
    assert np.all(err <= bound), float((err / bound).max())
