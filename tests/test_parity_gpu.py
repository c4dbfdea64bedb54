"""GPU parity: every C-ABI call against the CPU oracle on the same seeded
inputs.  Codes, scales, Q8_0 blocks and int-path outputs are compared bit
for bit; e4m3 and low-rank outputs within the tolerances derived from the
arithmetic (see the helpers below)."""
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


def f32(t):
    return t.detach().cpu().numpy()


QT = {"int8": 0, "e4m3": 1}


# --------------------------------------------------------------------------- codecs
def test_e4m3_device_conversion_matches_oracle(w8, orc):
    grid = orc.bf16_to_f32(np.arange(1 << 16, dtype=np.uint32).astype(np.uint16))
    grid = grid[np.isfinite(grid)]
    scales = np.float32([1.0, 0.37, 3.1e-3, 117.0, 2.0 ** -12, 1e-10, 448.0 / 127.0])
    with np.errstate(over="ignore"):
        vals = [grid / s for s in scales]
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 32, size=1 << 22, dtype=np.uint64).astype(np.uint32).view(np.float32)
    vals.append(bits[np.isfinite(bits)])
    x = np.concatenate(vals).astype(np.float32)
    with np.errstate(all="ignore"):
        x = x[np.isfinite(x)]
    got = u8(w8.e4m3_encode(torch.from_numpy(x).to(DEV)))
    assert np.array_equal(got, orc.f32_to_e4m3(x))


# --------------------------------------------------------------------------- quantize_rows
# rows up to 200 KB take the bulk-copy kernel; (2, 110016) is past that and
# exercises the register kernel
ROW_SHAPES = [(1, 16), (5, 48), (127, 512), (129, 3072), (64, 12288), (3, 40000), (2, 110016)]


@pytest.mark.parametrize("qt", ["int8", "e4m3"])
@pytest.mark.parametrize("M,K", ROW_SHAPES)
def test_quantize_rows_parity(w8, orc, qt, M, K):
    x = workloads.with_outlier_channels((M, K), 1.0, seed=M * 7 + K)
    if M > 2:
        x[1] = 0                       # all-zero row: the 1e-10 floor
        x[2, :] = 1e-3
        x[2, K // 3] = 3.0e4           # one huge value
    q, s = w8.quantize_rows(x.to(DEV), qt)
    qr, sr = orc.quantize_rows(workloads.to_u16(x), QT[qt])
    assert np.array_equal(f32(s).view(np.uint32), sr.view(np.uint32))
    assert np.array_equal(u8(q), qr)


GOLDEN_ROWS = __import__("json").load(open(__import__("os").path.join(
    __import__("os").path.dirname(__file__), "golden", "quantize_rows.json")))["cases"]


@pytest.mark.parametrize("case", GOLDEN_ROWS, ids=lambda c: c["name"])
def test_quantize_rows_golden_on_gpu(w8, case):
    """The hand-derived golden rows (ties, floors, e4m3 grid points) through
    the device kernels, zero-padded to K = 16 (zeros change no absmax)."""
    vals = case["x"] + [0.0] * (16 - len(case["x"]))
    x = torch.tensor([vals], dtype=torch.float32).to(torch.bfloat16).to(DEV)
    q, s = w8.quantize_rows(x, case["qt"])
    assert float(s[0]) == float(np.float32(case["scale"]))
    got = u8(q)[0, :len(case["codes"])]
    want = np.array(case["codes"], dtype=np.int64)
    want = (want & 0xFF).astype(np.uint8)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("qt", ["int8", "e4m3"])
def test_quantize_rows_exact_ties(w8, orc, qt):
    """Rows whose quotients x/s fall exactly on rounding boundaries (every
    half-integer for int8, e4m3 midpoints): the exactness check must route
    them to the exact division."""
    if qt == "int8":
        base = np.arange(-127, 127, dtype=np.float32) + 0.5        # all ties, s = 1 via the 127 entry
        row = np.concatenate([[127.0], base]).astype(np.float32)
        row = np.concatenate([row, np.zeros((-row.size) % 16, np.float32)])
    else:
        grid = orc.e4m3_to_f32(np.arange(1, 126, dtype=np.uint8)).astype(np.float64)
        mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)      # midpoints, s = 1 via 448
        row = np.concatenate([[448.0], mids, -mids]).astype(np.float32)
        row = np.concatenate([row, np.zeros((-row.size) % 16, np.float32)])
    xb = torch.from_numpy(np.tile(row, (40, 1))).to(torch.bfloat16)
    q, s = w8.quantize_rows(xb.to(DEV), qt)
    qr, sr = orc.quantize_rows(workloads.to_u16(xb), QT[qt])
    assert np.array_equal(f32(s), sr) and np.array_equal(u8(q), qr)


@pytest.mark.parametrize("qt", ["int8", "e4m3"])
def test_quantize_rows_every_bf16_value(w8, orc, qt):
    """Each row holds its absmax a and every bf16 value v with |v| <= a, so
    every code of every representable input is compared with the oracle at
    these scales: powers of two (exact products), absmax values whose halves
    land next to ties after the fp32 division (4.0625, 4.125, 3.59375 - the
    common case in N(0,1) rows), and arbitrary ones."""
    grid = orc.bf16_to_f32(np.arange(1 << 16, dtype=np.uint32).astype(np.uint16))
    grid = np.unique(np.abs(grid[np.isfinite(grid)]))
    absmax = [4.0625, 4.125, 3.59375, 3.828125, 4.5, 3.96875, 1.0, 0.7578125, 100.5, 448.0, 57.5,
              1.0e-3, 3.0e-8, 2.5e4, 15.875]
    rows = []   # rows of 12288 (the team kernel), each [a, a chunk of the values, zeros]
    for a in absmax:
        a = float(np.float32(torch.tensor(a).to(torch.bfloat16).float()))
        v = grid[grid <= a]
        v = np.concatenate([v, -v])
        for c in range(0, v.size, 12287):
            rows.append(np.concatenate([[a], v[c:c + 12287]]))
    K = 12288
    x = np.zeros((len(rows), K), np.float32)
    for i, r in enumerate(rows):
        x[i, :r.size] = r
    xb = torch.from_numpy(x).to(torch.bfloat16)
    q, s = w8.quantize_rows(xb.to(DEV), qt)
    qr, sr = orc.quantize_rows(workloads.to_u16(xb), QT[qt])
    assert np.array_equal(f32(s).view(np.uint32), sr.view(np.uint32))
    assert np.array_equal(u8(q), qr)


def test_quantize_rows_strided_input(w8, orc):
    big = workloads.normal((40, 256), 1.0, 3)
    x = big.to(DEV)[:, :160]           # ldx = 256 > K = 160
    q, s = w8.quantize_rows(x, "int8")
    qr, sr = orc.quantize_rows(workloads.to_u16(big[:, :160]), 0)
    assert np.array_equal(u8(q), qr) and np.array_equal(f32(s), sr)


# --------------------------------------------------------------------------- weights
@pytest.mark.parametrize("qt", ["int8", "e4m3"])
@pytest.mark.parametrize("gran", ["tensor", "axis"])
@pytest.mark.parametrize("N,K", [(1, 16), (96, 160), (3072, 3072)])
def test_quantize_weight_parity(w8, orc, qt, gran, N, K):
    w = workloads.normal((N, K), 0.02, seed=N + K)
    q, s = w8.quantize_weight(w.to(DEV), qt, gran)
    qr, sr = orc.quantize_weight(workloads.to_u16(w), QT[qt], 0 if gran == "tensor" else 1)
    assert np.array_equal(f32(s), sr)
    assert np.array_equal(u8(q), qr)


# --------------------------------------------------------------------------- Q8_0
@pytest.mark.parametrize("n", [1, 31, 32, 33, 255, 256, 257, 1000, 65536 + 7, 1 << 22])
def test_q8_0_parity(w8, orc, n):
    x = workloads.q8_0_standalone(n, seed=n).numpy()
    if n > 64:
        x[32:64] = 0.0                 # a floor block
        x[64:96] *= 1e-12
    b = w8.q8_0_quantize(torch.from_numpy(x).to(DEV))
    br, _ = orc.q8_0_quantize(x)
    assert np.array_equal(u8(b), br)
    y = w8.q8_0_dequantize(torch.from_numpy(br).to(DEV), n)
    assert np.array_equal(f32(y).view(np.uint32), orc.q8_0_dequantize(br, n).view(np.uint32))


def test_q8_0_standalone_full_size(w8, orc):
    """2^28 fp32 values ~ N(0,1): every block bit-exact, every value exact."""
    x = workloads.q8_0_standalone()
    xd = x.to(DEV)
    b = w8.q8_0_quantize(xd)
    br, _ = orc.q8_0_quantize(x.numpy())
    assert np.array_equal(u8(b), br)
    del xd
    y = w8.q8_0_dequantize(b, x.numel())
    assert np.array_equal(f32(y).view(np.uint32), orc.q8_0_dequantize(br, x.numel()).view(np.uint32))


# K = 3072, 6144, 12288 and 24576 fill the register-holding kernel's blocks
# exactly (its FULL form); 512 and 4096 do not; 96 and 4128 take the
# one-warp-per-row kernel, 32768 and 131072 the team kernel
RQ_SHAPES = [(1, 32), (37, 96), (64, 512), (12288, 3072), (5, 4096), (4, 6144), (7, 12288), (3, 24576),
             (3, 32768), (2, 131072), (5, 4128)]


@pytest.mark.parametrize("N,K", RQ_SHAPES)
def test_q8_0_to_axis_int8_parity(w8, orc, N, K):
    w = workloads.gguf_q8_0(N=N, K=K, M=1)["w_f32"].numpy().reshape(-1)
    br, _ = orc.q8_0_quantize(w)
    q, s = w8.q8_0_to_axis_int8(torch.from_numpy(br).to(DEV), N, K)
    qr, sr = orc.q8_0_to_axis_int8(br, N, K)
    assert np.array_equal(f32(s), sr)
    assert np.array_equal(u8(q), qr.view(np.uint8))


@pytest.mark.parametrize("N,K", [(13, 256), (50, 3072), (11, 4096), (6, 12288), (4, 32768), (9, 96), (12, 4128),
                                 (5, 6144), (3, 24576)])
def test_q8_0_to_axis_int8_arbitrary_blocks(w8, orc, N, K):
    """Blocks not produced by a quantizer: -128 codes, zero, negative and
    subnormal f16 scales, rows sharing one scale (codes come back unchanged)."""
    br = workloads.raw_q8_0_blocks(N, K, seed=61 + K)
    q, s = w8.q8_0_to_axis_int8(br.to(DEV), N, K)
    qr, sr = orc.q8_0_to_axis_int8(br.numpy(), N, K)
    assert np.array_equal(f32(s).view(np.uint32), sr.view(np.uint32))
    assert np.array_equal(u8(q), qr.view(np.uint8))


# Q8_0 -> axis e4m3 (GGUF A8 float): the same kernels with the e4m3 code
@pytest.mark.parametrize("N,K", RQ_SHAPES)
def test_q8_0_to_axis_e4m3_parity(w8, orc, N, K):
    w = workloads.gguf_q8_0(N=N, K=K, M=1)["w_f32"].numpy().reshape(-1)
    br, _ = orc.q8_0_quantize(w)
    q, s = w8.q8_0_to_axis_e4m3(torch.from_numpy(br).to(DEV), N, K)
    assert q.dtype == torch.float8_e4m3fn
    qr, sr = orc.q8_0_to_axis(br, N, K, 1)
    assert np.array_equal(f32(s), sr)
    assert np.array_equal(u8(q), qr)


@pytest.mark.parametrize("N,K", [(13, 256), (50, 3072), (11, 4096), (6, 12288), (4, 32768), (9, 96), (12, 4128),
                                 (5, 6144), (3, 24576)])
def test_q8_0_to_axis_e4m3_arbitrary_blocks(w8, orc, N, K):
    """Blocks not produced by a quantizer (see raw_q8_0_blocks): -128 codes,
    all-zero and negative scales (so -0 values, code 0x80), f16 subnormal
    scales (quotients in the e4m3 subnormal range)."""
    br = workloads.raw_q8_0_blocks(N, K, seed=71 + K)
    q, s = w8.q8_0_to_axis_e4m3(br.to(DEV), N, K)
    qr, sr = orc.q8_0_to_axis(br.numpy(), N, K, 1)
    assert np.array_equal(f32(s).view(np.uint32), sr.view(np.uint32))
    assert np.array_equal(u8(q), qr)


# --------------------------------------------------------------------------- Linear forward
def _fp8_tol(ref, y):
    """|y - y_ref| <= 1e-3 * s_x * s_w * sum|a*b| + 1 bf16 ulp."""
    yr = bf16_bits_to_f64(ref["y"])
    yg = bf16_bits_to_f64(y)
    bound = 1e-3 * ref["sx"][:, None].astype(np.float64) * ref["sw"] * ref["absacc"]
    bound = bound + ulp_bf16(np.maximum(np.abs(yr), np.abs(yg)))
    return np.abs(yg - yr), bound


# (7, 1000, 4096), (1, 2048, 3072) and (100, 256, 12288) have few output
# tiles and a long contraction: split-K with 8, 6 and 16 splits
LIN_SHAPES = [(256, 512, 512), (300, 520, 640), (1, 16, 16), (129, 257, 96), (7, 1000, 4096),
              (128, 256, 128), (520, 300, 272), (1, 2048, 3072), (100, 256, 12288)]


@pytest.mark.parametrize("M,N,K", LIN_SHAPES)
def test_linear_fwd_int8_parity(w8, orc, M, N, K):
    x = workloads.with_outlier_channels((M, K), 1.0, seed=M + 3 * N + K)
    w = workloads.normal((N, K), 0.02, seed=N + 5)
    wq, sw = w8.quantize_weight(w.to(DEV), "int8", "tensor")
    y = w8.linear_fwd(x.to(DEV), wq, sw)
    wqr, swr = orc.quantize_weight(workloads.to_u16(w), 0, 0)
    ref = orc.linear_fwd(workloads.to_u16(x), wqr, swr)
    assert np.array_equal(u16(y), ref["y"])


@pytest.mark.parametrize("M,N,K", [(200, 384, 256), (77, 130, 512), (33, 520, 2048)])
def test_linear_fwd_int8_axis_bias_parity(w8, orc, M, N, K):
    x = workloads.normal((M, K), 1.0, seed=11)
    w = workloads.normal((N, K), 0.02, seed=12)
    bias = workloads.normal((N,), 0.01, seed=13)
    wq, sw = w8.quantize_weight(w.to(DEV), "int8", "axis")
    y = w8.linear_fwd(x.to(DEV), wq, sw, bias=bias.to(DEV))
    wqr, swr = orc.quantize_weight(workloads.to_u16(w), 0, 1)
    ref = orc.linear_fwd(workloads.to_u16(x), wqr, swr, bias=workloads.to_u16(bias))
    assert np.array_equal(u16(y), ref["y"])


# CTA-pair forwards (M >= 512) with both formats, both weight scale
# granularities and a bias: fewer tiles than pairs at (600, 520, 512),
# (1024, 1024, 1024) and the ragged (777, 264, 384); two full rounds over the
# 74 pairs and a partial third at (4096, 3072, 256)
# CTA-pair forwards; (520, 9000): two rounds of tiles over the 74 pairs, the
# last tile 40 columns wide.
PAIR_SHAPES = [(600, 520, 512), (1024, 1024, 1024), (777, 264, 384), (4096, 3072, 256), (520, 9000, 512)]


@pytest.mark.parametrize("qt", ["int8", "e4m3"])
@pytest.mark.parametrize("gran", ["tensor", "axis"])
@pytest.mark.parametrize("M,N,K", PAIR_SHAPES)
def test_linear_fwd_pair_parity(w8, orc, qt, gran, M, N, K):
    x = workloads.with_outlier_channels((M, K), 1.0, seed=M + 2 * N + K)
    w = workloads.normal((N, K), 0.02, seed=N + 9)
    bias = workloads.normal((N,), 0.01, seed=N + 10)
    q, g = QT[qt], (0 if gran == "tensor" else 1)
    wq, sw = w8.quantize_weight(w.to(DEV), qt, gran)
    xd, bd = x.to(DEV), bias.to(DEV)
    y = w8.linear_fwd(xd, wq, sw, bias=bd)
    assert torch.equal(y, w8.linear_fwd(xd, wq, sw, bias=bd))        # deterministic
    wqr, swr = orc.quantize_weight(workloads.to_u16(w), q, g)
    assert np.array_equal(u8(wq), wqr)
    rows = np.unique(np.concatenate([np.arange(0, M, 7), np.arange(max(0, M - 256), M)]))
    ref = orc.linear_fwd(workloads.to_u16(x)[rows], wqr, swr, qt=q, bias=workloads.to_u16(bias))
    if q == 0:
        assert np.array_equal(u16(y)[rows], ref["y"])
    else:
        ref["sw"] = swr[0] if g == 0 else swr[None, :]
        err, bound = _fp8_tol(ref, u16(y)[rows])
        assert np.all(err <= bound), float((err / bound).max())


@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (300, 520, 640), (1, 16, 16), (129, 257, 96), (5, 264, 4096)])
def test_linear_fwd_e4m3_parity(w8, orc, M, N, K):
    x = workloads.with_outlier_channels((M, K), 1.0, seed=M + N)
    w = workloads.normal((N, K), 0.02, seed=K + 1)
    bias = workloads.normal((N,), 0.01, seed=N + 2)
    wq, sw = w8.quantize_weight(w.to(DEV), "e4m3", "tensor")
    y = w8.linear_fwd(x.to(DEV), wq, sw, bias=bias.to(DEV))
    wqr, swr = orc.quantize_weight(workloads.to_u16(w), 1, 0)
    assert np.array_equal(u8(wq), wqr)
    ref = orc.linear_fwd(workloads.to_u16(x), wqr, swr, qt=1, bias=workloads.to_u16(bias))
    ref["sw"] = swr[0]
    err, bound = _fp8_tol(ref, u16(y))
    assert np.all(err <= bound), float((err / bound).max())


# GGUF A8 float forward: e4m3 weight codes from the Q8_0 re-quantization
# with one scale per output column, e4m3 activations token-wise
@pytest.mark.parametrize("M,N,K", [(1, 12288, 3072), (8, 520, 1024), (64, 1024, 3072), (300, 520, 640),
                                   (600, 1024, 512), (129, 257, 96)])
def test_gguf_a8_float_forward_parity(w8, orc, M, N, K):
    d = workloads.gguf_q8_0(N=N, K=K, M=M)
    br, _ = orc.q8_0_quantize(d["w_f32"].numpy().reshape(-1))
    wq, sw = w8.q8_0_to_axis_e4m3(torch.from_numpy(br).to(DEV), N, K)
    y = w8.linear_fwd(d["x"].to(DEV), wq, sw)
    wqr, swr = orc.q8_0_to_axis(br, N, K, 1)
    assert np.array_equal(u8(wq), wqr)
    ref = orc.linear_fwd(workloads.to_u16(d["x"]), wqr, swr, qt=1)
    ref["sw"] = swr[None, :]
    err, bound = _fp8_tol(ref, u16(y))
    assert np.all(err <= bound), float((err / bound).max())


def test_qgemm_fwd_equals_linear(w8):
    x = workloads.normal((300, 640), 1.0, 21).to(DEV)
    wq, sw = w8.quantize_weight(workloads.normal((520, 640), 0.02, 22).to(DEV), "int8", "tensor")
    xq, sx = w8.quantize_rows(x, "int8")
    assert torch.equal(w8.qgemm_fwd(xq, sx, wq, sw), w8.linear_fwd(x, wq, sw))


def test_linear_fwd_extreme_codes(w8, orc):
    """Every code at +-127 and K = 12288: the int32 accumulator's largest sums."""
    M, N, K = 130, 260, 12288
    x = torch.full((M, K), 1.0)
    x[::2] = -1.0
    w = torch.full((N, K), 0.5)
    w[1::3] = -0.5
    xb, wb = x.to(torch.bfloat16), w.to(torch.bfloat16)
    wq, sw = w8.quantize_weight(wb.to(DEV), "int8", "tensor")
    y = w8.linear_fwd(xb.to(DEV), wq, sw)
    wqr, swr = orc.quantize_weight(workloads.to_u16(wb), 0, 0)
    ref = orc.linear_fwd(workloads.to_u16(xb), wqr, swr)
    assert np.abs(ref["acc"]).max() == 127 * 127 * K
    assert np.array_equal(u16(y), ref["y"])


def test_linear_fwd_m0_noop(w8):
    x = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    wq, sw = w8.quantize_weight(workloads.normal((32, 64), 0.02, 1).to(DEV), "int8", "tensor")
    assert w8.linear_fwd(x, wq, sw).shape == (0, 32)


@pytest.mark.parametrize("M,N,K", [(1, 7, 16), (2, 300, 48), (2, 513, 16384), (2, 64, 16400), (4, 1000, 3072),
                                   (64, 1000, 3072), (128, 264, 4096), (33, 12288, 3072)])
@pytest.mark.parametrize("gran", ["tensor", "axis"])
def test_linear_fwd_few_tokens(w8, orc, M, N, K, gran):
    """M <= 2 int8 forwards run as one weight-streaming launch (dp4a on the
    CUDA cores, the rows quantized inside it; K <= 16384, else the GEMM);
    up to 128 tokens the transposed tensor-core product (weight rows as the
    MMA's M, split along K for few weight tiles): bit-exact with the oracle
    and with the tensor-core product on the same codes."""
    x = workloads.with_outlier_channels((M, K), 1.0, seed=M * 31 + K)
    w = workloads.normal((N, K), 0.02, seed=N + 17)
    bias = workloads.normal((N,), 0.01, seed=N + 18)
    wq, sw = w8.quantize_weight(w.to(DEV), "int8", gran)
    y = w8.linear_fwd(x.to(DEV), wq, sw, bias=bias.to(DEV))
    wqr, swr = orc.quantize_weight(workloads.to_u16(w), 0, 1 if gran == "axis" else 0)
    ref = orc.linear_fwd(workloads.to_u16(x), wqr, swr, bias=workloads.to_u16(bias))
    assert np.array_equal(u16(y), ref["y"])
    xq, sx = w8.quantize_rows(x.to(DEV), "int8")
    assert torch.equal(y, w8.qgemm_fwd(xq, sx, wq, sw, bias=bias.to(DEV)))


# e4m3 few-token forwards: M = 1 runs the CUDA-core kernel (K up to 32768),
# 2..4 the transposed tensor-core product; ragged N, K = 16 and K not a
# multiple of 512, both weight granularities
@pytest.mark.parametrize("M,N,K,gran", [(1, 16, 16, "tensor"), (1, 3000, 4112, "axis"), (2, 257, 1024, "tensor"),
                                        (3, 1000, 3072, "axis"), (4, 520, 8192, "tensor"), (1, 264, 32768, "axis"),
                                        (4, 12288, 3072, "axis")])
def test_linear_fwd_e4m3_few_tokens(w8, orc, M, N, K, gran):
    x = workloads.with_outlier_channels((M, K), 1.0, seed=101 + M + K)
    w = workloads.normal((N, K), 0.02, seed=102 + N)
    bias = workloads.normal((N,), 0.01, seed=103)
    wq, sw = w8.quantize_weight(w.to(DEV), "e4m3", gran)
    y = w8.linear_fwd(x.to(DEV), wq, sw, bias=bias.to(DEV))
    wqr, swr = orc.quantize_weight(workloads.to_u16(w), 1, 1 if gran == "axis" else 0)
    assert np.array_equal(u8(wq), wqr)
    ref = orc.linear_fwd(workloads.to_u16(x), wqr, swr, qt=1, bias=workloads.to_u16(bias))
    ref["sw"] = swr[None, :] if gran == "axis" else swr[0]
    err, bound = _fp8_tol(ref, u16(y))
    assert np.all(err <= bound), float((err / bound).max())
    # the same product through the tensor-core path (the chained entry point
    # does not take the few-token kernel): both within the bound of the oracle
    y2 = w8.linear_fwd_ex(x.to(DEV), wq, sw, bias=bias.to(DEV), y_amax=torch.zeros(M, dtype=torch.int32, device=DEV))
    err2, bound2 = _fp8_tol(ref, u16(y2))
    assert np.all(err2 <= bound2)


def test_linear_fwd_split_equals_unsplit(w8):
    """A forward with few output tiles and a long K (split-K for int8) equals
    the GEMM on the same codes without splitting (qgemm_fwd never splits), bit
    for bit; e4m3 products are not split, so they are equal too."""
    x = workloads.normal((64, 3072), 1.0, 33).to(DEV)
    w = workloads.normal((1024, 3072), 0.02, 34).to(DEV)
    assert w8.workspace_bytes(w8.OP_LINEAR_FWD, 64, 1024, 3072) > 64 * 3072 + 256
    for qt in ("int8", "e4m3"):
        wq, sw = w8.quantize_weight(w, qt, "tensor")
        xq, sx = w8.quantize_rows(x, qt)
        assert torch.equal(w8.linear_fwd(x, wq, sw), w8.qgemm_fwd(xq, sx, wq, sw)), qt


def test_linear_fwd_deterministic(w8):
    x = workloads.normal((1000, 1024), 1.0, 31).to(DEV)
    wq, sw = w8.quantize_weight(workloads.normal((2048, 1024), 0.02, 32).to(DEV), "e4m3", "tensor")
    a = w8.linear_fwd(x, wq, sw)
    b = w8.linear_fwd(x, wq, sw)
    assert torch.equal(a, b)


# --------------------------------------------------------------------------- dgrad
@pytest.mark.parametrize("qt", ["int8", "e4m3"])
@pytest.mark.parametrize("M,N,K", [(64, 256, 512), (129, 96, 80), (300, 512, 272), (1, 16, 16), (50, 2048, 768)])
def test_linear_dgrad_parity(w8, orc, qt, M, N, K):
    dy = workloads.normal((M, N), 1e-3, seed=M + N)
    w = workloads.normal((N, K), 0.02, seed=N * 3 + K)
    wq, sw = w8.quantize_weight(w.to(DEV), qt, "tensor")
    dx = w8.linear_dgrad(dy.to(DEV), wq, sw)
    wqr, swr = orc.quantize_weight(workloads.to_u16(w), QT[qt], 0)
    ref = orc.linear_dgrad(workloads.to_u16(dy), wqr, swr, qt=QT[qt])
    if qt == "int8":
        assert np.array_equal(u16(dx), ref["y"])
    else:
        ref["sw"] = swr[0]
        err, bound = _fp8_tol(ref, u16(dx))
        assert np.all(err <= bound), float((err / bound).max())


def test_qgemm_dgrad_equals_linear(w8):
    dy = workloads.normal((96, 256), 1e-3, 41).to(DEV)
    wq, sw = w8.quantize_weight(workloads.normal((256, 160), 0.02, 42).to(DEV), "int8", "tensor")
    dyq, sdy = w8.quantize_rows(dy, "int8")
    assert torch.equal(w8.qgemm_dgrad(dyq, sdy, wq, sw), w8.linear_dgrad(dy, wq, sw))


# --------------------------------------------------------------------------- SVDQuant
def _svdq_check(w8, orc, x, w, r, bias=None, rows=None, qt=0):
    """The library's own weight preparation (svdq_prepare) feeds both sides:
    the forward on the GPU and the oracle's forward on the same factors and
    residual codes."""
    dp = w8.svdq_prepare(w.to(DEV), r, "int8" if qt == 0 else "e4m3")
    l1, l2, rq, rs = dp["l1"], dp["l2"], dp["rq"], dp["r_scale"]
    prep = {"l1": u16(l1), "l2": u16(l2), "rq": u8(rq), "s_r": f32(rs)}
    M, K = x.shape
    N = w.shape[0]
    ws = torch.empty(w8.workspace_bytes(w8.OP_SVDQ_FWD, M, N, K, r), dtype=torch.uint8, device=DEV)
    y = w8.svdq_linear_fwd(x.to(DEV), rq, rs, l1, l2, bias=None if bias is None else bias.to(DEV), ws=ws)
    # the activation codes, row scales and T = bf16(X L1) as the kernels left
    # them in the workspace (codes [M, K] at 0, scales [M] and T [M, r] each
    # on the next 256-byte boundary)
    off_s = -(-(M * K) // 256) * 256
    off = off_s + -(-(M * 4) // 256) * 256
    t_gpu = ws[off:off + M * r * 2].view(torch.bfloat16).view(M, r)
    rows = np.arange(M) if rows is None else np.asarray(rows)
    xs = workloads.to_u16(x)[rows]
    ref = orc.svdq_linear_fwd(xs, prep["rq"], prep["s_r"], prep["l1"], prep["l2"],
                              bias=None if bias is None else workloads.to_u16(bias), qt=qt)
    assert np.array_equal(u8(ws[:M * K]).reshape(M, K)[rows], ref["xq"])
    assert np.array_equal(f32(ws[off_s:off_s + M * 4].view(torch.float32))[rows].view(np.uint32),
                          ref["sx"].view(np.uint32))
    # T: fp32 accumulation over K on the tensor cores, then one bf16 rounding
    xabs = np.abs(orc.bf16_to_f32(xs).astype(np.float64)) @ np.abs(orc.bf16_to_f32(prep["l1"]).astype(np.float64))
    gam = K * 2.0 ** -23 * xabs
    tg = bf16_bits_to_f64(u16(t_gpu)[rows])
    assert np.all(np.abs(tg - ref["t64"]) <= ulp_bf16(np.abs(ref["t64"]) + gam) + gam)
    # y: the int part is exact (the e4m3 part within the fp8 bound); T may
    # differ by its bound; lr sums in fp32
    dt = ulp_bf16(np.abs(ref["t64"]) + gam) + gam
    l2abs = np.abs(orc.bf16_to_f32(prep["l2"]).astype(np.float64))
    yr = bf16_bits_to_f64(ref["y"])
    yg = bf16_bits_to_f64(u16(y)[rows])
    bound = dt @ l2abs + 2.0 ** -16 * ref["lr_abs"] + ulp_bf16(np.maximum(np.abs(yr), np.abs(yg)))
    if qt == 1:
        bound = bound + 1e-3 * ref["sx"][:, None].astype(np.float64) * float(prep["s_r"][0]) * ref["absacc"]
    assert np.all(np.abs(yg - yr) <= bound), float((np.abs(yg - yr) / bound).max())
    return y, ref


@pytest.mark.parametrize("r", [8, 16, 32])
def test_svdq_parity_small(w8, orc, r):
    x = workloads.with_outlier_channels((200, 256), 1.0, seed=51 + r)
    w = workloads.rank_spike_weight(320, 256, 8, 0.5, 0.02, seed=52)
    bias = workloads.normal((320,), 0.01, seed=53)
    _svdq_check(w8, orc, x, w, r, bias=bias)


@pytest.mark.parametrize("M,N,K,r", [(600, 520, 512, 8), (777, 264, 384, 24), (1024, 1024, 1024, 32),
                                     (520, 136, 256, 16), (530, 300, 256, 16), (601, 264, 272, 16)])
def test_svdq_parity_pairs(w8, orc, M, N, K, r):
    """M >= 512 with N % 8 == 0 runs the CTA-pair kernel, whose low-rank sum
    is a tensor-core product of the pair written, in two halves of the tile's
    columns, into the TMEM the tile's int32 sums occupied (ragged edges, r
    padded to the MMA's K steps); (530, 300) keeps the single-SM form."""
    x = workloads.with_outlier_channels((M, K), 1.0, seed=M + r)
    w = workloads.rank_spike_weight(N, K, 8, 0.5, 0.02, seed=N + K)
    bias = workloads.normal((N,), 0.01, seed=N + 7)
    _svdq_check(w8, orc, x, w, r, bias=bias)


@pytest.mark.parametrize("M,K,r,qt", [(33, 3072, 32, 0), (65, 3072, 24, 1), (33, 3088, 8, 0), (97, 1040, 16, 1),
                                      (1, 16, 8, 0), (31, 48, 32, 1)])
def test_svdq_input_row_lengths(w8, orc, M, K, r, qt):
    """Rows up to 3072 columns: codes, scales and T come from one pass over X
    (32 rows per CTA held on chip; a CTA with one row); K = 3088 takes the
    row quantizer and the T product; K = 1040 ends in a partial block of 64
    columns; K = 16 and 48 give one k-step to one or three of the eight
    k-groups (the others add zero partial sums)."""
    x = workloads.with_outlier_channels((M, K), 1.0, seed=M + K)
    w = workloads.rank_spike_weight(136, K, 8, 0.5, 0.02, seed=K + r)
    _svdq_check(w8, orc, x, w, r, bias=workloads.normal((136,), 0.01, seed=77), qt=qt)


@pytest.mark.parametrize("qt", [0, 1])
def test_svdq_parity_long_rows(w8, orc, qt):
    """Long rows (K = 6400): the T product's split along K and the row
    quantizer's multi-warp teams."""
    x = workloads.with_outlier_channels((130, 6400), 1.0, seed=74)
    w = workloads.rank_spike_weight(264, 6400, 8, 0.5, 0.02, seed=75)
    _svdq_check(w8, orc, x, w, 16, bias=workloads.normal((264,), 0.01, seed=76), qt=qt)


@pytest.mark.parametrize("M", [130, 600])
def test_svdq_zero_factors_equal_int_linear(w8, M):
    x = workloads.normal((M, 256), 1.0, 61).to(DEV)
    wq, sw = w8.quantize_weight(workloads.normal((304, 256), 0.02, 62).to(DEV), "int8", "tensor")
    l1 = torch.zeros((256, 16), dtype=torch.bfloat16, device=DEV)
    l2 = torch.zeros((16, 304), dtype=torch.bfloat16, device=DEV)
    assert torch.equal(w8.svdq_linear_fwd(x, wq, sw, l1, l2), w8.linear_fwd(x, wq, sw))


# SVDQuant on float W8A8: e4m3 residual and activation codes.  Small M and
# N % 8 != 0 take the single-SM low-rank epilogue, the rest the CTA pair.
@pytest.mark.parametrize("M,N,K,r", [(200, 320, 256, 8), (130, 300, 256, 16), (600, 520, 512, 8),
                                     (1024, 1024, 1024, 32), (530, 300, 256, 16), (777, 264, 384, 24)])
def test_svdq_e4m3_parity(w8, orc, M, N, K, r):
    x = workloads.with_outlier_channels((M, K), 1.0, seed=71 + M)
    w = workloads.rank_spike_weight(N, K, 8, 0.5, 0.02, seed=72 + N)
    bias = workloads.normal((N,), 0.01, seed=73)
    _svdq_check(w8, orc, x, w, r, bias=bias, qt=1)


@pytest.mark.parametrize("M", [130, 600])
def test_svdq_e4m3_zero_factors_equal_float_linear(w8, M):
    x = workloads.normal((M, 256), 1.0, 61).to(DEV)
    wq, sw = w8.quantize_weight(workloads.normal((304, 256), 0.02, 62).to(DEV), "e4m3", "tensor")
    l1 = torch.zeros((256, 16), dtype=torch.bfloat16, device=DEV)
    l2 = torch.zeros((16, 304), dtype=torch.bfloat16, device=DEV)
    assert torch.equal(w8.svdq_linear_fwd(x, wq, sw, l1, l2), w8.linear_fwd(x, wq, sw))


# --------------------------------------------------------------------------- fused MLP chain
def _amax_of(y):
    """Row max |y| of a bf16 CUDA tensor, as fp32 bit patterns (int32)."""
    return y.float().abs().amax(dim=1).view(torch.int32)


# pair kernel (600 rows), single-SM (130), split-K (7 x 1000 x 4096, 1 x 2048 x 3072), e4m3
CHAIN_SHAPES = [(600, 520, 512, "int8"), (130, 264, 256, "int8"), (7, 1000, 4096, "int8"), (1, 2048, 3072, "int8"),
                (600, 520, 512, "e4m3"), (33, 256, 1024, "e4m3")]


@pytest.mark.parametrize("M,N,K,qt", CHAIN_SHAPES)
def test_linear_fwd_ex_row_absmax(w8, orc, M, N, K, qt):
    """Without an activation the output is linear_fwd's bit for bit, and
    y_amax holds each row's max |y| exactly (every epilogue form: pair,
    single-SM, split-K)."""
    x = workloads.with_outlier_channels((M, K), 1.0, seed=91 + M).to(DEV)
    wq, sw = w8.quantize_weight(workloads.normal((N, K), 0.02, seed=92).to(DEV), qt, "tensor")
    bias = workloads.normal((N,), 0.01, seed=93).to(DEV)
    amax = torch.full((M,), 12345, dtype=torch.int32, device=DEV)   # the call clears it
    y = w8.linear_fwd_ex(x, wq, sw, bias=bias, y_amax=amax)
    assert torch.equal(y, w8.linear_fwd(x, wq, sw, bias=bias))
    assert torch.equal(amax, _amax_of(y))


@pytest.mark.parametrize("act", ["gelu", "gelu_tanh"])
@pytest.mark.parametrize("M,N,K,qt", CHAIN_SHAPES)
def test_linear_fwd_ex_gelu_parity(w8, orc, M, N, K, qt, act):
    """GELU on the fp32 epilogue value.  Bound: 1 bf16 ulp plus the fp32
    evaluation error of the activation (the erf / tanh of CUDA's math library
    within a few units of 2^-23 absolute, scaled by |v|); for e4m3 also the
    GEMM bound, through GELU's slope (|GELU'| < 1.13)."""
    x = workloads.with_outlier_channels((M, K), 1.0, seed=94 + M)
    w = workloads.normal((N, K), 0.02, seed=95)
    bias = workloads.normal((N,), 0.01, seed=96)
    q = QT[qt]
    wq, sw = w8.quantize_weight(w.to(DEV), qt, "tensor")
    amax = torch.zeros((M,), dtype=torch.int32, device=DEV)
    y = w8.linear_fwd_ex(x.to(DEV), wq, sw, bias=bias.to(DEV), act=act, y_amax=amax)
    assert torch.equal(amax, _amax_of(y))
    wqr, swr = orc.quantize_weight(workloads.to_u16(w), q, 0)
    a = orc.ACT_GELU if act == "gelu" else orc.ACT_GELU_TANH
    ref = orc.linear_fwd(workloads.to_u16(x), wqr, swr, qt=q, bias=workloads.to_u16(bias), act=a)
    v = np.abs(ref["pre"].astype(np.float64))
    yr = bf16_bits_to_f64(ref["y"])
    yg = bf16_bits_to_f64(u16(y))
    bound = ulp_bf16(np.maximum(np.abs(yr), np.abs(yg))) + 2.0 ** -19 * (v + 0.05 * v ** 3)
    if q == 1:
        bound = bound + 1.13 * 1e-3 * ref["sx"][:, None].astype(np.float64) * float(swr[0]) * ref["absacc"]
    err = np.abs(yg - yr)
    assert np.all(err <= bound), float((err / bound).max())


@pytest.mark.parametrize("M", [1, 64, 600])
def test_mlp_chain_given_absmax_equals_unfused(w8, M):
    """Up-projection with GELU hands its row absmax to the down-projection,
    whose quantizer then skips the reduction: the result is the unfused
    chain's bit for bit."""
    x = workloads.normal((M, 512), 1.0, 97).to(DEV)
    w1q, s1 = w8.quantize_weight(workloads.normal((1024, 512), 0.02, 98).to(DEV), "int8", "tensor")
    w2q, s2 = w8.quantize_weight(workloads.normal((512, 1024), 0.02, 99).to(DEV), "int8", "tensor")
    a1 = torch.zeros((M,), dtype=torch.int32, device=DEV)
    y1 = w8.linear_fwd_ex(x, w1q, s1, act="gelu", y_amax=a1)
    y2 = w8.linear_fwd_ex(y1, w2q, s2, x_amax=a1)
    assert torch.equal(y2, w8.linear_fwd(y1, w2q, s2))
    # and with a wrong absmax the codes change: the given value is used
    y2w = w8.linear_fwd_ex(y1, w2q, s2, x_amax=(a1.view(torch.float32) * 2).view(torch.int32).contiguous())
    assert not torch.equal(y2w, y2)


# --------------------------------------------------------------------------- weight-only types
@pytest.mark.parametrize("n,s", [(256, 1.0), (4096 * 16, 0.02 / 448), ((1 << 20) + 48, 3.1e-5)])
def test_dequantize_e4m3_bf16_parity(w8, orc, n, s):
    codes = torch.arange(n, dtype=torch.int64).remainder(256).to(torch.uint8)
    codes[codes == 0x7F] = 0x7E          # no NaN codes: a quantizer never writes them
    codes[codes == 0xFF] = 0xFE
    codes = codes[torch.randperm(n, generator=torch.Generator().manual_seed(n))]
    sc = torch.tensor([s], dtype=torch.float32)
    w = w8.dequantize_e4m3_bf16(codes.to(DEV).view(torch.float8_e4m3fn), sc.to(DEV))
    assert np.array_equal(u16(w), orc.dequant_e4m3_bf16(codes.numpy(), sc.numpy()))


@pytest.mark.parametrize("n", [77, 4096, (1 << 20) + 3])
def test_q8_0_dequantize_bf16_parity(w8, orc, n):
    x = workloads.q8_0_standalone(n, seed=n).numpy()
    br, _ = orc.q8_0_quantize(x)
    y = w8.q8_0_dequantize_bf16(torch.from_numpy(br).to(DEV), n)
    assert np.array_equal(u16(y), orc.q8_0_dequantize_bf16(br, n))


def _bf16_tol(ref, y, K):
    """fp32 sums on the tensor cores: |y - y_ref| <= K 2^-23 sum|x w| + 1 bf16 ulp."""
    yr = bf16_bits_to_f64(ref["y"])
    yg = bf16_bits_to_f64(y)
    bound = K * 2.0 ** -23 * ref["absacc"] + ulp_bf16(np.maximum(np.abs(yr), np.abs(yg)))
    return np.abs(yg - yr), bound


# (600, 520, 512) and (1024, 1024, 1024): the CTA pair; (1, 3072, 4096) and
# (64, 1024, 3072): split along K; the rest single-SM tiles, ragged edges
BF16_SHAPES = [(600, 520, 512), (1024, 1024, 1024), (1, 3072, 4096), (64, 1024, 3072), (129, 257, 96),
               (300, 520, 640), (1, 16, 16), (530, 300, 256)]


@pytest.mark.parametrize("M,N,K", BF16_SHAPES)
def test_bf16_linear_parity(w8, orc, M, N, K):
    x = workloads.with_outlier_channels((M, K), 1.0, seed=81 + M)
    w = workloads.normal((N, K), 0.02, seed=82 + N)
    bias = workloads.normal((N,), 0.01, seed=83)
    y = w8.bf16_linear_fwd(x.to(DEV), w.to(DEV), bias=bias.to(DEV))
    ref = orc.linear_bf16(workloads.to_u16(x), workloads.to_u16(w), workloads.to_u16(bias))
    err, bound = _bf16_tol(ref, u16(y), K)
    assert np.all(err <= bound), float((err / bound).max())


@pytest.mark.parametrize("M,N,K", [(600, 520, 512), (1, 3072, 4096), (129, 257, 96), (64, 1024, 3072)])
def test_float8_weight_only_parity(w8, orc, M, N, K):
    x = workloads.normal((M, K), 1.0, seed=84 + M)
    w = workloads.normal((N, K), 0.02, seed=85 + N)
    bias = workloads.normal((N,), 0.01, seed=86)
    wq, sw = w8.quantize_weight(w.to(DEV), "e4m3", "tensor")
    y = w8.float8_linear_fwd(x.to(DEV), wq, sw, bias=bias.to(DEV))
    wqr, swr = orc.quantize_weight(workloads.to_u16(w), 1, 0)
    assert np.array_equal(u8(wq), wqr)
    ref = orc.float8_linear_fwd(workloads.to_u16(x), wqr, swr, workloads.to_u16(bias))
    err, bound = _bf16_tol(ref, u16(y), K)
    assert np.all(err <= bound), float((err / bound).max())


@pytest.mark.parametrize("M,N,K", [(600, 520, 512), (1, 3072, 4096), (129, 264, 96), (64, 1024, 3072)])
def test_gguf_weight_only_parity(w8, orc, M, N, K):
    d = workloads.gguf_q8_0(N=N, K=K, M=M)
    br, _ = orc.q8_0_quantize(d["w_f32"].numpy().reshape(-1))
    bias = workloads.normal((N,), 0.01, seed=87)
    y = w8.gguf_linear_fwd(d["x"].to(DEV), torch.from_numpy(br).to(DEV), N, bias=bias.to(DEV))
    ref = orc.gguf_linear_fwd(workloads.to_u16(d["x"]), br, N, K, workloads.to_u16(bias))
    err, bound = _bf16_tol(ref, u16(y), K)
    assert np.all(err <= bound), float((err / bound).max())


# input gradients: (600, 520, 512) and (1024, 1024, 3072) the CTA pair (the
# weight read MN-major, two 64-column atoms per CTA), (1, 3072, 4096) and
# (64, 1024, 3072) split along the contraction, the rest single-SM tiles
BF16_DGRAD_SHAPES = [(600, 520, 512), (1024, 1024, 3072), (1, 3072, 4096), (64, 1024, 3072), (130, 264, 96),
                     (300, 520, 640)]


@pytest.mark.parametrize("M,N,K", BF16_DGRAD_SHAPES)
def test_bf16_linear_dgrad_parity(w8, orc, M, N, K):
    dy = workloads.normal((M, N), 1e-3, seed=111 + M)
    w = workloads.normal((N, K), 0.02, seed=112 + N)
    dx = w8.bf16_linear_dgrad(dy.to(DEV), w.to(DEV))
    ref = orc.linear_bf16_dgrad(workloads.to_u16(dy), workloads.to_u16(w))
    err, bound = _bf16_tol(ref, u16(dx), N)
    assert np.all(err <= bound), float((err / bound).max())


@pytest.mark.parametrize("M,N,K", [(600, 520, 512), (64, 1024, 3072), (130, 264, 96)])
@pytest.mark.parametrize("kind", ["float8", "gguf"])
def test_weight_only_dgrad_parity(w8, orc, M, N, K, kind):
    dy = workloads.normal((M, N), 1e-3, seed=113 + M)
    w32 = workloads.normal((N, K), 0.02, seed=114 + N).float()
    if kind == "float8":
        wb = w32.to(torch.bfloat16)
        wq, sw = w8.quantize_weight(wb.to(DEV), "e4m3", "tensor")
        dx = w8.float8_linear_dgrad(dy.to(DEV), wq, sw)
        wqr, swr = orc.quantize_weight(workloads.to_u16(wb), 1, 0)
        wd = orc.dequant_e4m3_bf16(wqr, swr).reshape(N, K)
    else:
        br, _ = orc.q8_0_quantize(w32.numpy().reshape(-1))
        dx = w8.gguf_linear_dgrad(dy.to(DEV), torch.from_numpy(br).to(DEV), K)
        wd = orc.q8_0_dequantize_bf16(br, N * K).reshape(N, K)
    ref = orc.linear_bf16_dgrad(workloads.to_u16(dy), wd)
    err, bound = _bf16_tol(ref, u16(dx), N)
    assert np.all(err <= bound), float((err / bound).max())


def test_weight_only_m0_and_unsplit_equal_split(w8):
    x = workloads.normal((64, 3072), 1.0, 88).to(DEV)
    w = workloads.normal((1024, 3072), 0.02, 89).to(DEV)
    assert w8.bf16_linear_fwd(x[:0], w).shape == (0, 1024)
    # one row through the split path equals itself computed within a
    # larger, unsplit product up to the fp32 summation order
    y_all = w8.bf16_linear_fwd(torch.cat([x] * 10), w)[:64]
    y_small = w8.bf16_linear_fwd(x, w)
    d = (y_all.float() - y_small.float()).abs()
    assert float(d.max()) <= 2 ** -6 * float(y_all.float().abs().max())


# --------------------------------------------------------------------------- diagnostics
def test_device_status_clean_then_bounded_wait_times_out(w8):
    assert w8.device_status(reset=True) == 0
    w8.selftest_wait(50_000_000)                  # 50 ms wait on a barrier nothing completes
    assert w8.device_status(reset=True) == 6      # W8A8_ERR_DEVICE_TIMEOUT, context intact
    assert w8.device_status(reset=True) == 0
    x = workloads.normal((64, 64), 1.0, 71).to(DEV)
    wq, sw = w8.quantize_weight(workloads.normal((64, 64), 0.02, 72).to(DEV), "int8", "tensor")
    w8.linear_fwd(x, wq, sw)
    assert w8.device_status(reset=True) == 0
