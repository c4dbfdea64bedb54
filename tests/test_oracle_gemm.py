"""Pins of the oracle's 8-bit matrix products, the dequantizing epilogue, the
composed Linear forward / dgrad and the SVDQuant branch."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import workloads
from oracle import svdquant


def _rand_i8(shape, seed):
    return np.random.default_rng(seed).integers(-128, 128, size=shape).astype(np.int8)


# --------------------------------------------------------------------------- int GEMM
def test_gemm_i8_bruteforce_tiny(orc):
    A = _rand_i8((3, 5), 1)
    B = _rand_i8((4, 5), 2)
    acc = orc.gemm_i8_nt(A.view(np.uint8), B.view(np.uint8))
    for m in range(3):
        for n in range(4):
            assert acc[m, n] == sum(int(A[m, k]) * int(B[n, k]) for k in range(5))


@pytest.mark.parametrize("M,N,K", [(7, 9, 33), (64, 48, 256), (1, 300, 1024)])
def test_gemm_i8_vs_numpy_int64(orc, M, N, K):
    A = _rand_i8((M, K), M)
    B = _rand_i8((N, K), N)
    ref = A.astype(np.int64) @ B.astype(np.int64).T
    assert np.array_equal(orc.gemm_i8_nt(A.view(np.uint8), B.view(np.uint8)), ref.astype(np.int32))
    # contraction along B's rows (dgrad form): A2 [M,N] x B [N,K]
    A2 = _rand_i8((M, N), K)
    ref2 = A2.astype(np.int64) @ B.astype(np.int64)
    assert np.array_equal(orc.gemm_i8_nn(A2.view(np.uint8), B.view(np.uint8)), ref2.astype(np.int32))


def test_gemm_i8_int32_range_check(orc):
    K = 140000   # 127*127*K > 2^31 - 1
    A = np.full((1, K), 127, np.int8)
    with pytest.raises(OverflowError):
        orc.gemm_i8_nt(A.view(np.uint8), A.view(np.uint8))
    # 12288 (the largest contraction of the DiT shapes) stays well inside
    A = np.full((1, 12288), -127, np.int8)
    assert orc.gemm_i8_nt(A.view(np.uint8), A.view(np.uint8))[0, 0] == 127 * 127 * 12288


# --------------------------------------------------------------------------- e4m3 GEMM
def test_gemm_e4m3_vs_numpy(orc):
    rng = np.random.default_rng(3)
    A = rng.integers(0, 256, size=(20, 96)).astype(np.uint8)
    B = rng.integers(0, 256, size=(12, 96)).astype(np.uint8)
    A[(A & 0x7F) == 0x7F] = 0x38   # no NaN codes
    B[(B & 0x7F) == 0x7F] = 0x38
    a = orc.e4m3_to_f32(A).astype(np.float64)
    b = orc.e4m3_to_f32(B).astype(np.float64)
    acc, absacc = orc.gemm_e4m3_nt(A, B)
    assert np.allclose(acc, a @ b.T, rtol=1e-13, atol=1e-300)
    assert np.allclose(absacc, np.abs(a) @ np.abs(b).T, rtol=1e-13)
    acc2, _ = orc.gemm_e4m3_nn(A[:, :12], B[:, :50])
    assert np.allclose(acc2, a[:, :12] @ b[:, :50], rtol=1e-13, atol=1e-300)


# --------------------------------------------------------------------------- epilogue
def _fp32_round(fr: Fraction) -> np.float32:
    """Exact rational -> nearest fp32 (ties to even), via exact comparison."""
    f = np.float32(float(fr))          # within one ulp; fix by exact comparison
    lo = np.nextafter(f, np.float32(-np.inf))
    hi = np.nextafter(f, np.float32(np.inf))
    best = min((lo, f, hi), key=lambda c: (abs(Fraction(float(c)) - fr),
                                           int(np.float32(c).view(np.uint32)) & 1))
    return np.float32(best)


def test_epilogue_closed_form(orc):
    # powers of two and small integers: exact in every order
    acc = np.array([[1000, -3, 0]], np.int32)
    y, y32 = orc.epilogue(acc, np.float32([0.5]), np.float32([0.25]),
                          workloads.to_u16(torch.tensor([1.0, 2.0, -1.5]).to(torch.bfloat16)))
    assert y32.tolist() == [[126.0, 1.625, -1.5]]
    # the fp64 (e4m3) form: same closed form
    y, y32 = orc.epilogue(np.array([[1000.0, -3.0, 0.0]]), np.float32([0.5]), np.float32([0.25]),
                          workloads.to_u16(torch.tensor([1.0, 2.0, -1.5]).to(torch.bfloat16)))
    assert y32.tolist() == [[126.0, 1.625, -1.5]]


def test_epilogue_rounds_each_operation(orc):
    """((acc * s_row) * s_w) + bias with every step rounded to fp32 on its own:
    checked against exact rational arithmetic rounded step by step."""
    rng = np.random.default_rng(7)
    acc = rng.integers(-2 ** 20, 2 ** 20, size=(16, 8)).astype(np.int32)
    s_row = (rng.random(16).astype(np.float32) / np.float32(127))
    s_w = np.float32([0.0123]) / np.float32(127)
    bias_f = torch.tensor(rng.standard_normal(8) * 0.01, dtype=torch.float32).to(torch.bfloat16)
    y, y32 = orc.epilogue(acc, s_row, s_w, workloads.to_u16(bias_f))
    bias = bias_f.float().numpy()
    for m in range(16):
        for n in range(8):
            t = _fp32_round(Fraction(int(acc[m, n])) * Fraction(float(s_row[m])))
            u = _fp32_round(Fraction(float(t)) * Fraction(float(s_w[0])))
            v = _fp32_round(Fraction(float(u)) + Fraction(float(bias[n])))
            assert y32[m, n] == v, (m, n)
    assert np.array_equal(y, orc.f32_to_bf16(y32))


def test_epilogue_axis_scale_indexes_columns(orc):
    acc = np.ones((2, 3), np.int32)
    _, y32 = orc.epilogue(acc, np.float32([1.0, 2.0]), np.float32([1.0, 4.0, 16.0]))
    assert y32.tolist() == [[1.0, 4.0, 16.0], [2.0, 8.0, 32.0]]


# --------------------------------------------------------------------------- composed Linear
def _integer_operands(M, N, K, seed):
    """bf16 integer matrices whose every X row and W reach |127|: the token
    scales and the tensor scale are exactly 1, so the W8A8 Linear reduces to
    the textbook integer matmul."""
    rng = np.random.default_rng(seed)
    X = rng.integers(-127, 128, size=(M, K)).astype(np.float32)
    X[:, 0] = 127.0
    W = rng.integers(-127, 128, size=(N, K)).astype(np.float32)
    W[0, 1] = -127.0
    to = lambda a: workloads.to_u16(torch.from_numpy(a).to(torch.bfloat16))
    return X, W, to(X), to(W)


def test_linear_fwd_reduces_to_integer_matmul(orc):
    M, N, K = 5, 7, 64      # non-square: a transposed operand cannot pass
    X, W, xu, wu = _integer_operands(M, N, K, 8)
    wq, sw = orc.quantize_weight(wu, orc.INT8, orc.TENSOR)
    assert sw[0] == 1.0
    out = orc.linear_fwd(xu, wq, sw)
    ref = X.astype(np.int64) @ W.astype(np.int64).T
    assert np.array_equal(out["acc"], ref)
    assert np.all(out["sx"] == 1.0)
    assert np.array_equal(out["y"], orc.f32_to_bf16(ref.astype(np.float32)))


def test_linear_fwd_e4m3_reduces_to_float_matmul(orc):
    """e4m3 with unit scales: codes of the e4m3 grid values come back exactly."""
    rng = np.random.default_rng(9)
    grid = orc.e4m3_to_f32(np.arange(0x30, 0x7F, dtype=np.uint8))   # 0.5 .. 448
    X = rng.choice(np.concatenate([grid, -grid]), size=(4, 32)).astype(np.float32)
    X[:, 3] = 448.0
    W = rng.choice(np.concatenate([grid, -grid]), size=(6, 32)).astype(np.float32)
    W[2, 2] = -448.0
    to = lambda a: workloads.to_u16(torch.from_numpy(a).to(torch.bfloat16))
    wq, sw = orc.quantize_weight(to(W), orc.E4M3, orc.TENSOR)
    assert sw[0] == 1.0
    out = orc.linear_fwd(to(X), wq, sw, qt=orc.E4M3)
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    assert np.array_equal(out["acc"], ref)


def test_linear_dgrad_reduces_to_integer_matmul(orc):
    M, N, K = 6, 40, 24
    dY, Wt, dyu, _ = _integer_operands(M, K, N, 10)    # dY [M,N], Wt [K,N]
    W = np.ascontiguousarray(Wt.T)                      # W [N,K]
    wu = workloads.to_u16(torch.from_numpy(W).to(torch.bfloat16))
    wq, sw = orc.quantize_weight(wu, orc.INT8, orc.TENSOR)
    assert sw[0] == 1.0
    out = orc.linear_dgrad(dyu, wq, sw)
    ref = dY.astype(np.int64) @ W.astype(np.int64)     # [M,N] x [N,K]
    assert np.array_equal(out["acc"], ref)


def test_dgrad_equals_forward_with_transposed_weight(orc):
    """dgrad(dY, Wq) == forward GEMM against an explicit copy of Wq^T."""
    dy = workloads.to_u16(workloads.normal((33, 80), 1e-3, 11))
    wu = workloads.to_u16(workloads.normal((80, 48), 0.02, 12))
    wq, sw = orc.quantize_weight(wu, orc.INT8, orc.TENSOR)
    d = orc.linear_dgrad(dy, wq, sw)
    f = orc.linear_fwd(dy, np.ascontiguousarray(wq.T), sw)
    assert np.array_equal(d["acc"], f["acc"]) and np.array_equal(d["y"], f["y"])


def test_linear_fwd_error_vs_bf16_matmul(orc):
    """W8A8 error sanity: relative Frobenius error of the int8 Linear against
    the fp64 product of the bf16 inputs stays at the 8-bit level."""
    x = workloads.normal((64, 512), 1.0, 13)
    w = workloads.normal((96, 512), 0.02, 14)
    wq, sw = orc.quantize_weight(workloads.to_u16(w), orc.INT8, orc.TENSOR)
    out = orc.linear_fwd(workloads.to_u16(x), wq, sw)
    ref = x.double().numpy() @ w.double().numpy().T
    rel = np.linalg.norm(out["y32"] - ref) / np.linalg.norm(ref)
    assert 1e-3 < rel < 3e-2


# --------------------------------------------------------------------------- SVDQuant
def test_lowrank_vs_numpy(orc):
    x = workloads.normal((9, 64), 1.0, 15)
    l1 = workloads.normal((64, 8), 0.1, 16)
    l2 = workloads.normal((8, 40), 0.1, 17)
    t, t64 = orc.lowrank_down(workloads.to_u16(x), workloads.to_u16(l1))
    ref = x.double().numpy() @ l1.double().numpy()
    assert np.allclose(t64, ref, rtol=1e-12, atol=1e-15)
    tb = torch.from_numpy(t.view(np.int16)).view(torch.bfloat16)
    assert torch.equal(tb, torch.from_numpy(t64.astype(np.float32)).to(torch.bfloat16))
    lr, lr_abs = orc.lowrank_up(t, workloads.to_u16(l2))
    ref2 = tb.double().numpy() @ l2.double().numpy()
    assert np.allclose(lr, ref2, rtol=1e-12, atol=1e-15)


def test_svdq_zero_factors_is_int_linear(orc):
    x = workloads.to_u16(workloads.with_outlier_channels((16, 256), 1.0, 18))
    w = workloads.to_u16(workloads.normal((64, 256), 0.02, 19))
    rq, sr = orc.quantize_weight(w, orc.INT8, orc.TENSOR)
    z1 = np.zeros((256, 32), np.uint16)
    z2 = np.zeros((32, 64), np.uint16)
    s = orc.svdq_linear_fwd(x, rq, sr, z1, z2)
    f = orc.linear_fwd(x, rq, sr)
    assert np.array_equal(s["y"], f["y"])


def test_svdq_zero_factors_is_float_linear(orc):
    """SVDQuant on float W8A8 (e4m3 residual codes): zero factors give the
    e4m3 Linear forward exactly."""
    x = workloads.to_u16(workloads.with_outlier_channels((16, 256), 1.0, 18))
    w = workloads.to_u16(workloads.normal((64, 256), 0.02, 19))
    rq, sr = orc.quantize_weight(w, orc.E4M3, orc.TENSOR)
    z1 = np.zeros((256, 32), np.uint16)
    z2 = np.zeros((32, 64), np.uint16)
    s = orc.svdq_linear_fwd(x, rq, sr, z1, z2, qt=orc.E4M3)
    f = orc.linear_fwd(x, rq, sr, qt=orc.E4M3)
    assert np.array_equal(s["y"], f["y"])
    rq8, sr8 = orc.quantize_weight(w, orc.INT8, orc.TENSOR)
    assert not np.array_equal(f["y"], orc.linear_fwd(x, rq8, sr8)["y"])   # the code type is in effect


@pytest.mark.parametrize("qt", [0, 1])
def test_svdq_zero_residual_is_lowrank_product(orc, qt):
    """With all residual codes zero, y is the low-rank product alone: the bf16
    rounding of fp32(T L2), T = bf16(X L1), checked against numpy in fp64."""
    x = workloads.normal((12, 96), 1.0, 23)
    l1 = workloads.normal((96, 16), 0.1, 24)
    l2 = workloads.normal((16, 40), 0.1, 25)
    rq = np.zeros((40, 96), np.uint8)
    sr = np.array([1e-10], np.float32)
    s = orc.svdq_linear_fwd(workloads.to_u16(x), rq, sr, workloads.to_u16(l1), workloads.to_u16(l2), qt=qt)
    t = torch.from_numpy((x.double() @ l1.double()).numpy().astype(np.float32)).to(torch.bfloat16)
    lr = (t.double() @ l2.double()).numpy().astype(np.float32)
    want = torch.from_numpy(lr).to(torch.bfloat16)
    assert np.array_equal(s["y"], workloads.to_u16(want))


def test_svdq_split_reduces_weight_error(orc):
    """With a rank-8 spike, the low-rank branch plus the int8 residual is a
    better approximation of W than plain tensor-wise int8."""
    w = workloads.rank_spike_weight(256, 320, 8, 0.5, 0.02, 20)
    wu = workloads.to_u16(w)
    prep = svdquant.prepare(wu, 32)
    W = w.double().numpy()
    lowrank = (orc.bf16_to_f32(prep["l1"]).astype(np.float64)
               @ orc.bf16_to_f32(prep["l2"]).astype(np.float64)).T
    deq_r = prep["rq"].view(np.int8).astype(np.float64) * prep["s_r"][0]
    err_svd = np.linalg.norm(W - lowrank - deq_r)
    wq, sw = orc.quantize_weight(wu, orc.INT8, orc.TENSOR)
    err_plain = np.linalg.norm(W - wq.view(np.int8).astype(np.float64) * sw[0])
    assert err_svd < 0.5 * err_plain
    # the residual no longer holds the spike: its absmax is at the noise level
    assert np.abs(orc.bf16_to_f32(prep["resid"])).max() < 0.2


def test_svdq_exact_lowrank_weight(orc):
    """A weight that is exactly rank 4 (bf16 factors, products exact) leaves a
    residual at the bf16 rounding level."""
    a = workloads.normal((48, 4), 0.25, 21).double()
    b = workloads.normal((4, 40), 0.25, 22).double()
    w = (a @ b).T.to(torch.bfloat16)     # [N=40, K=48]
    prep = svdquant.prepare(workloads.to_u16(w), 8)
    resid = orc.bf16_to_f32(prep["resid"])
    assert np.abs(resid).max() < 0.02 * np.abs(w.float().numpy()).max()


def test_svdq_split_reduces_weight_error_e4m3(orc):
    """The same with an e4m3 residual (float W8A8 + SVDQuant): the factors
    carry the spike in bf16, and the residual's e4m3 error is that of the
    noise alone."""
    w = workloads.rank_spike_weight(256, 320, 8, 0.5, 0.02, 20)
    wu = workloads.to_u16(w)
    prep = svdquant.prepare(wu, 32, orc.E4M3)
    W = w.double().numpy()
    lowrank = (orc.bf16_to_f32(prep["l1"]).astype(np.float64)
               @ orc.bf16_to_f32(prep["l2"]).astype(np.float64)).T
    deq_r = orc.decode_codes(prep["rq"], orc.E4M3).astype(np.float64) * prep["s_r"][0]
    err_svd = np.linalg.norm(W - lowrank - deq_r)
    wq, sw = orc.quantize_weight(wu, orc.E4M3, orc.TENSOR)
    err_plain = np.linalg.norm(W - orc.decode_codes(wq, orc.E4M3).astype(np.float64) * sw[0])
    assert err_svd < 0.5 * err_plain, (err_svd, err_plain)


# --------------------------------------------------------------------------- weight-only types
@pytest.mark.parametrize("s", [1.0, 0.02 / 448, 3.1e-5, 7.77])
def test_dequant_e4m3_bf16_vs_torch(orc, s):
    """Every e4m3 code (NaN codes excluded) times a scale, through torch's
    float8 -> fp32 cast, one fp32 product and torch's bf16 cast."""
    q = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    s32 = np.float32(s)
    got = orc.dequant_e4m3_bf16(q, np.array([s32]))
    t = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float32) * torch.tensor(s32)
    assert np.array_equal(got, workloads.to_u16(t.to(torch.bfloat16)))


def test_q8_0_dequantize_bf16_vs_torch(orc):
    """GGUF values f16(d) * q through torch (f16 -> fp32 cast, exact product),
    then torch's bf16 cast; 77 values end in a short block."""
    blocks = workloads.raw_q8_0_blocks(4, 96, seed=31).numpy()
    n = 4 * 96 - 19
    got = orc.q8_0_dequantize_bf16(blocks, n)
    b = blocks.reshape(-1, 34)
    d = torch.from_numpy(np.ascontiguousarray(b[:, :2]).view(np.float16).reshape(-1)).to(torch.float32)
    q = torch.from_numpy(b[:, 2:].view(np.int8).astype(np.float32))
    want = (q * d[:, None]).reshape(-1)[:n].to(torch.bfloat16)
    assert np.array_equal(got, workloads.to_u16(want))


def test_linear_bf16_vs_numpy_and_textbook(orc):
    x = workloads.normal((7, 96), 1.0, 32)
    w = workloads.normal((13, 96), 0.05, 33)
    bias = workloads.normal((13,), 0.1, 34)
    r = orc.linear_bf16(workloads.to_u16(x), workloads.to_u16(w), workloads.to_u16(bias))
    ref = x.double().numpy() @ w.double().numpy().T
    assert np.allclose(r["acc"], ref, rtol=1e-13, atol=1e-15)
    assert np.allclose(r["absacc"], np.abs(x.double().numpy()) @ np.abs(w.double().numpy()).T, rtol=1e-13)
    y32 = ref.astype(np.float32) + bias.float().numpy()
    assert np.array_equal(r["y32"], y32.astype(np.float32))
    assert np.array_equal(r["y"], workloads.to_u16(torch.from_numpy(y32).to(torch.bfloat16)))
    # integer operands: the textbook integer matmul, exactly (non-square: a
    # transposed operand cannot pass)
    g = np.random.default_rng(35)
    xi = g.integers(-8, 9, size=(5, 64)).astype(np.float32)
    wi = g.integers(-8, 9, size=(9, 64)).astype(np.float32)
    to = lambda a: workloads.to_u16(torch.from_numpy(a).to(torch.bfloat16))
    ri = orc.linear_bf16(to(xi), to(wi))
    assert np.array_equal(ri["acc"], (xi.astype(np.int64) @ wi.astype(np.int64).T).astype(np.float64))


def test_weight_only_forwards_compose(orc):
    """float8: quantize W tensor-wise to e4m3, dequantize to bf16, bf16 Linear;
    GGUF: the same through Q8_0 blocks.  Both stay close to the bf16 Linear
    on W itself (the quantization error bound of each format)."""
    x = workloads.normal((6, 128), 1.0, 36)
    w = workloads.normal((24, 128), 0.02, 37)
    xu, wu = workloads.to_u16(x), workloads.to_u16(w)
    base = orc.linear_bf16(xu, wu)["acc"]
    wq, sw = orc.quantize_weight(wu, orc.E4M3, orc.TENSOR)
    f8 = orc.float8_linear_fwd(xu, wq, sw)
    assert np.array_equal(f8["y"], orc.linear_bf16(xu, orc.dequant_e4m3_bf16(wq, sw).reshape(24, 128))["y"])
    absx = np.abs(x.double().numpy()) @ np.abs(w.double().numpy()).T
    assert np.all(np.abs(f8["acc"] - base) <= 2 ** -4 * absx + 2 ** -9 * float(sw[0]) * np.abs(x.double().numpy()).sum(1)[:, None] + 2 ** -8 * absx)
    blocks, s32 = orc.q8_0_quantize(w.float().numpy().reshape(-1))
    gg = orc.gguf_linear_fwd(xu, blocks, 24, 128)
    assert np.array_equal(gg["y"], orc.linear_bf16(xu, orc.q8_0_dequantize_bf16(blocks, 24 * 128).reshape(24, 128))["y"])
    # per weight: half a code step of the f32 block scale, the f16 rounding of
    # that scale (127 codes x 2^-11 relative), then one bf16 rounding
    sb = np.repeat(s32.astype(np.float64), 32).reshape(24, 128)
    ew = sb * (0.5 * (1 + 2 ** -20) + 127 * 2 ** -11)
    ew = ew + 2 ** -8 * (np.abs(w.double().numpy()) + ew)
    assert np.all(np.abs(gg["acc"] - base) <= np.abs(x.double().numpy()) @ ew.T)


# --------------------------------------------------------------------------- activation and row absmax
def test_gelu_closed_forms_and_library(orc):
    """GELU(1) = Phi(1) and GELU(-1) = -Phi(-1) (the normal CDF at 1); the odd
    identity GELU(v) - GELU(-v) = v of both forms; the exact form equals
    scipy's erf composed in double, rounded once; the tanh form stays within
    1e-3 of it."""
    from scipy.special import erf
    g = orc.act_f32(np.array([1.0, -1.0, 0.0], np.float32), orc.ACT_GELU)
    assert g[0] == np.float32(0.8413447460685429) and g[1] == np.float32(-0.15865525393145707) and g[2] == 0.0
    v = np.linspace(-6, 6, 4001).astype(np.float32)
    for act in (orc.ACT_GELU, orc.ACT_GELU_TANH):
        a, b = orc.act_f32(v, act).astype(np.float64), orc.act_f32(-v, act).astype(np.float64)
        assert np.all(np.abs(a - b - v) <= 4 * np.spacing(np.maximum(np.abs(v), 1e-30).astype(np.float32)))
    vd = v.astype(np.float64)
    ref = (0.5 * vd * (1.0 + erf(vd / np.sqrt(2.0)))).astype(np.float32)
    assert np.array_equal(orc.act_f32(v, orc.ACT_GELU), ref)
    assert np.all(np.abs(orc.act_f32(v, orc.ACT_GELU_TANH) - ref) <= 1e-3)
    assert np.array_equal(orc.act_f32(v, orc.ACT_NONE), v)


def test_row_absmax_and_activated_forward(orc):
    x = workloads.to_u16(workloads.with_outlier_channels((9, 128), 1.0, 40))
    w = workloads.to_u16(workloads.normal((40, 128), 0.02, 41))
    bias = workloads.to_u16(workloads.normal((40,), 0.01, 42))
    wq, sw = orc.quantize_weight(w, orc.INT8, orc.TENSOR)
    base = orc.linear_fwd(x, wq, sw, bias=bias)
    yb = orc.bf16_to_f32(base["y"])
    assert np.array_equal(base["amax"], np.abs(yb).max(axis=1))
    g = orc.linear_fwd(x, wq, sw, bias=bias, act=orc.ACT_GELU)
    assert np.array_equal(g["pre"], base["y32"])
    assert np.array_equal(g["y"], orc.f32_to_bf16(orc.act_f32(base["y32"], orc.ACT_GELU)))
    assert np.array_equal(g["amax"], np.abs(orc.bf16_to_f32(g["y"])).max(axis=1))
    assert np.all(orc.bf16_to_f32(g["y"]) >= -0.17)     # GELU's minimum is about -0.17
    # maxima placed by hand: last column, first column, negative, all zero
    yh = np.zeros((4, 9), np.float32)
    yh[0, 8], yh[1, 0], yh[2, 4], yh[2, 5] = -3.0, 2.5, 1.0, -0.5
    assert orc.row_absmax_bf16(orc.f32_to_bf16(yh)).tolist() == [3.0, 2.5, 1.0, 0.0]


def test_linear_bf16_dgrad_is_the_textbook_product(orc):
    """dX = dY W with integer operands: exact, and non-square so that a
    transposed operand cannot pass."""
    g = np.random.default_rng(43)
    dy = g.integers(-8, 9, size=(5, 24)).astype(np.float32)
    w = g.integers(-8, 9, size=(24, 40)).astype(np.float32)
    to = lambda a: workloads.to_u16(torch.from_numpy(a).to(torch.bfloat16))
    r = orc.linear_bf16_dgrad(to(dy), to(w))
    assert r["acc"].shape == (5, 40)
    assert np.array_equal(r["acc"], (dy.astype(np.int64) @ w.astype(np.int64)).astype(np.float64))
