"""Pins of the oracle's quantizers: hand-derived golden rows, the absmax
invariant, weight granularities, and the GGUF Q8_0 format and re-quantization."""
import json
import os

import numpy as np
import pytest
import torch

import workloads

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(vals):
    t = torch.tensor(vals, dtype=torch.float32)
    assert torch.equal(t.to(torch.bfloat16).float(), t), "fixture value not bf16-exact"
    return workloads.to_u16(t.to(torch.bfloat16))


# --------------------------------------------------------------------------- rows
@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLD, "quantize_rows.json")))["cases"],
                         ids=lambda c: c["name"])
def test_quantize_rows_golden(orc, case):
    qt = orc.INT8 if case["qt"] == "int8" else orc.E4M3
    x = _bf16(case["x"])[None, :]
    q, s = orc.quantize_rows(x, qt)
    assert s[0] == np.float32(case["scale"])
    if qt == orc.INT8:
        assert q[0].view(np.int8).tolist() == case["codes"]
    else:
        assert q[0].tolist() == case["codes"]


@pytest.mark.parametrize("qt", [0, 1])
def test_quantize_rows_absmax_invariant(orc, qt):
    x = workloads.with_outlier_channels((64, 384), 1.0, 5)
    q, s = orc.quantize_rows(workloads.to_u16(x), qt)
    dec = orc.decode_codes(q, qt)
    qmax = orc.QMAX[qt]
    # the largest |code| of every row is QMAX, all codes within [-QMAX, QMAX]
    assert np.all(np.abs(dec).max(axis=1) == qmax)
    assert np.all(np.abs(dec) <= qmax)
    # s_m = absmax_m / QMAX, fp32 division
    amax = np.abs(x.float().numpy()).max(axis=1).astype(np.float32)
    assert np.array_equal(s, (amax / np.float32(qmax)).astype(np.float32))
    # codes carry the sign of x and reconstruct within half a code step (int8)
    xf = x.float().numpy().astype(np.float64)
    err = np.abs(dec * s[:, None].astype(np.float64) - xf)
    if qt == 0:
        assert np.all(err <= 0.5 * s[:, None] * (1 + 2 ** -20) + 1e-30)
    assert np.all(np.sign(dec) * np.sign(xf) >= 0)


def test_quantize_rows_leading_dimension(orc):
    x = workloads.to_u16(workloads.normal((8, 64), 1.0, 6))
    q1, s1 = orc.quantize_rows(x[:, :48], 0)
    xs = np.ascontiguousarray(x[:, :48])
    q2, s2 = orc.quantize_rows(xs, 0)
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


def test_quantize_rows_each_row_independent(orc):
    """Quantizing a subset of rows gives the same rows as quantizing all: the
    property the sampled full-size parity checks rely on."""
    x = workloads.to_u16(workloads.normal((50, 96), 1.0, 7))
    q, s = orc.quantize_rows(x, 0)
    idx = [3, 17, 49]
    q2, s2 = orc.quantize_rows(x[idx], 0)
    assert np.array_equal(q[idx], q2) and np.array_equal(s[idx], s2)


# --------------------------------------------------------------------------- weights
@pytest.mark.parametrize("qt", [0, 1])
def test_quantize_weight_tensor(orc, qt):
    w = workloads.normal((96, 160), 0.02, 8)
    wu = workloads.to_u16(w)
    q, s = orc.quantize_weight(wu, qt, orc.TENSOR)
    assert s.shape == (1,)
    amax = np.float32(np.abs(w.float().numpy()).max())
    assert s[0] == amax / np.float32(orc.QMAX[qt])
    dec = orc.decode_codes(q, qt)
    assert np.abs(dec).max() == orc.QMAX[qt]
    # only the element(s) holding the global absmax reach QMAX exactly
    wf = np.abs(w.float().numpy())
    assert np.all(np.abs(dec)[wf == amax] == orc.QMAX[qt])


def test_quantize_weight_axis_is_rowwise(orc):
    wu = workloads.to_u16(workloads.normal((40, 64), 0.02, 9))
    q, s = orc.quantize_weight(wu, orc.INT8, orc.AXIS)
    q2, s2 = orc.quantize_rows(wu, orc.INT8)
    assert np.array_equal(q, q2) and np.array_equal(s, s2) and s.shape == (40,)


def test_quantize_weight_tensor_equals_rows_when_one_scale(orc):
    """If every row has the same absmax, tensor-wise and axis-wise agree."""
    w = workloads.normal((16, 64), 0.02, 10).float()
    w[:, 0] = 0.0625
    w = w.clamp(-0.0625, 0.0625)
    wu = workloads.to_u16(w.to(torch.bfloat16))
    qt_, st_ = orc.quantize_weight(wu, orc.INT8, orc.TENSOR)
    qa_, sa_ = orc.quantize_weight(wu, orc.INT8, orc.AXIS)
    assert np.array_equal(qt_, qa_) and np.all(sa_ == st_[0])


# --------------------------------------------------------------------------- Q8_0
Q80 = json.load(open(os.path.join(GOLD, "q8_0_blocks.json")))


@pytest.mark.parametrize("case", Q80["cases"], ids=lambda c: c["name"])
def test_q8_0_golden_blocks(orc, case):
    x = np.float32(case["x"])
    blocks, scales = orc.q8_0_quantize(x)
    assert blocks.size == 34
    codes = blocks[2:].view(np.int8).tolist()
    assert codes == case["codes"]
    if "scale_f32" in case:
        assert scales[0] == np.float32(case["scale_f32"])
    if "scale_f16_bits" in case:
        assert int(blocks[0]) | (int(blocks[1]) << 8) == case["scale_f16_bits"]


@pytest.mark.parametrize("n,packed,gguf", Q80["sizes"]["cases"])
def test_q8_0_sizes(orc, n, packed, gguf):
    assert orc.q8_0_bytes(n) == packed
    nb = (n + 31) // 32
    assert 2 * nb + n == gguf          # gguf_bytes of the Q8_0 struct
    if n % 32 == 0:
        assert abs(4 * n / gguf - 128 / 34) < 1e-12


def test_q8_0_invariants(orc):
    x = workloads.q8_0_standalone(1 << 16, seed=3).numpy()
    x[:32] = 0.0                      # one floor block
    x[32:64] *= 1e-12                 # another floor block (tiny values)
    blocks, s32 = orc.q8_0_quantize(x)
    codes = orc.q8_0_codes(blocks, x.size).astype(np.int32).reshape(-1, 32)
    xb = x.reshape(-1, 32)
    floor = np.abs(xb).max(axis=1) < np.float32(1e-10)
    assert floor[0] and floor[1] and floor.sum() == 2
    assert np.all(s32[floor] == np.float32(1e-10))
    assert np.all(np.abs(codes[floor]) <= 1)
    nf = ~floor
    # the element with the largest |v| of every block gets code +-127; codes in [-127,127]
    arg = np.abs(xb[nf]).argmax(axis=1)
    assert np.all(np.abs(codes[nf][np.arange(arg.size), arg]) == 127)
    assert np.all(np.abs(codes) <= 127)
    # per-element error of the f32-scale dequantization: <= scale/2 (+ rounding of v/scale)
    y32 = orc.q8_0_dequantize_f32(s32, orc.q8_0_codes(blocks, x.size), x.size).reshape(-1, 32)
    bound = s32[:, None].astype(np.float64) * (0.5 + 2 ** -20) + np.abs(xb) * 2 ** -23
    assert np.all(np.abs(y32.astype(np.float64) - xb) <= bound)
    # GGUF (f16 scale) dequantization adds at most 127 * |s32 - s16| per element
    y16 = orc.q8_0_dequantize(blocks, x.size).reshape(-1, 32)
    s16 = orc.f16_to_f32(orc.q8_0_scales_f16(blocks)).astype(np.float64)
    extra = 127 * np.abs(s32.astype(np.float64) - s16)[:, None]
    assert np.all(np.abs(y16.astype(np.float64) - xb) <= bound + extra + 1e-30)
    # f16 scale is the RNE binary16 of the f32 scale
    assert np.array_equal(orc.q8_0_scales_f16(blocks), s32.astype(np.float16).view(np.uint16))


def test_q8_0_short_tail(orc):
    x = workloads.q8_0_standalone(77, seed=4).numpy()
    blocks, s = orc.q8_0_quantize(x)
    assert blocks.size == 3 * 34 and s.size == 3
    tail = blocks.reshape(3, 34)[2, 2:].view(np.int8)
    assert np.all(tail[77 - 64:] == 0)
    # the short block's scale uses only its 13 real values
    assert s[2] == np.abs(x[64:]).max() / np.float32(127)
    y = orc.q8_0_dequantize(blocks, 77)
    assert y.size == 77
    full, _ = orc.q8_0_quantize(np.concatenate([x, np.zeros(19, np.float32)]))
    assert np.array_equal(full, blocks)


def test_q8_0_grid_roundtrip(orc):
    """Values already on a block's power-of-two grid come back exactly."""
    rng = np.random.default_rng(5)
    codes = rng.integers(-127, 128, size=(64, 32)).astype(np.float32)
    codes[:, 0] = 127.0
    step = np.exp2(rng.integers(-12, 2, size=(64, 1))).astype(np.float32)
    x = (codes * step).reshape(-1)
    blocks, s = orc.q8_0_quantize(x)
    assert np.array_equal(orc.q8_0_dequantize(blocks, x.size), x)
    assert np.array_equal(orc.q8_0_codes(blocks, x.size).astype(np.float32), codes.reshape(-1))


# --------------------------------------------------------------------------- Q8_0 -> axis int8
def test_requant_same_scale_rows_are_unchanged(orc):
    """If every block of a row shares one f16 scale d and the row's largest
    |code| is 127, re-quantization returns the codes unchanged with s_n = d."""
    rng = np.random.default_rng(6)
    N, K = 8, 256
    codes = rng.integers(-127, 128, size=(N, K)).astype(np.float32)
    codes[:, 5] = -127.0
    d = np.exp2(rng.integers(-10, -2, size=(N, 1))).astype(np.float32) * np.float32(1.5)
    x = (codes * d).reshape(-1)
    blocks, _ = orc.q8_0_quantize(x)
    # blocks whose own max code is below 127 get a different f16 scale; build
    # the row so that every block contains a +-127 code
    x2 = codes.copy()
    x2[:, ::32] = 127.0
    x = (x2 * d).reshape(-1)
    blocks, s32 = orc.q8_0_quantize(x)
    assert np.all(s32.reshape(N, -1) == d)
    q, s = orc.q8_0_to_axis_int8(blocks, N, K)
    assert np.array_equal(q.astype(np.float32), x2)
    assert np.array_equal(s, d.reshape(-1))


def test_requant_invariants(orc):
    d = workloads.gguf_q8_0(N=64, K=512)
    w = d["w_f32"].numpy()
    blocks, _ = orc.q8_0_quantize(w.reshape(-1))
    q, s = orc.q8_0_to_axis_int8(blocks, 64, 512)
    deq = orc.q8_0_dequantize(blocks, w.size).reshape(64, 512)
    amax = np.abs(deq).max(axis=1)
    assert np.array_equal(s, (amax / np.float32(127)).astype(np.float32))
    assert np.all(np.abs(q).max(axis=1) == 127)
    err = np.abs(q.astype(np.float64) * s[:, None] - deq)
    assert np.all(err <= s[:, None] * (0.5 + 2 ** -20))


# --------------------------------------------------------------------------- Q8_0 -> axis e4m3
def _e4m3_grid():
    """(value, code) of the 127 non-negative finite E4M3FN codes, built from
    the format: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, subnormal
    step 2^-9; S.1111.111 is NaN."""
    out = []
    for c in range(127):
        e, m = c >> 3, c & 7
        v = m * 2.0 ** -9 if e == 0 else (8 + m) * 2.0 ** (e - 10)
        out.append((v, c))
    return out


def _e4m3_nearest(t):
    """Brute force: the grid value nearest to t (exact in fp64), ties to the
    even code, |t| >= 448 saturating to +-448."""
    sign = 0x80 if np.signbit(t) else 0
    a = abs(float(t))
    if a >= 448.0:
        return sign | 0x7E
    best = min(_e4m3_grid(), key=lambda vc: (abs(vc[0] - a), vc[1] & 1))
    return sign | best[1]


def _raw_blocks(d_rows, q_rows):
    """Q8_0 bytes from chosen f16 block scales d [N, nb] (exactly f16) and codes
    q [N, nb, 32]."""
    d = np.asarray(d_rows, np.float32)
    assert np.array_equal(d.astype(np.float16).astype(np.float32), d)
    N, nb = d.shape
    blk = np.zeros((N, nb, 34), np.uint8)
    blk[:, :, :2] = d.astype(np.float16).view(np.uint8).reshape(N, nb, 2)
    blk[:, :, 2:] = np.asarray(q_rows, np.int8).view(np.uint8)
    return blk.reshape(-1)


def test_requant_e4m3_closed_form(orc):
    """Rows whose largest |d q| is 112 * 2^-6 get s = 2^-8 exactly, so every
    quotient is d q / 2^-8, a small multiple of 1/2 (4q, 2q or q/2 for block
    scales 2^-6, 2^-7, 2^-9); its code must be the nearest E4M3 value by brute
    force, ties to the even code, including the midpoints 68, 136, 264, ...
    An all-zero row takes the 1e-10 floor and codes 0."""
    rng = np.random.default_rng(11)
    N, nb = 6, 8
    d = np.full((N, nb), 2.0 ** -6, np.float32)
    d[:, 1::3] = 2.0 ** -7
    d[:, 2::3] = 2.0 ** -9
    q = np.zeros((N, nb, 32), np.int64)
    allq = np.arange(-112, 113)
    q[:4].reshape(-1)[: allq.size] = allq          # every code once in the 2^-6 rows ...
    q[:4] = q[:4].reshape(4, -1)[:, rng.permutation(nb * 32)].reshape(4, nb, 32)
    q[4] = rng.integers(-112, 113, size=(nb, 32))
    q[4, 1, 5] = -128                               # -128 in a 2^-7 block: quotient -256
    q[:5, 0, 0] = 112                               # ... and the row maximum in a 2^-6 block
    q[:5, 0, 1] = -112
    d[:5, 0] = 2.0 ** -6
    d[5] = 2.0 ** -6                                # row 5: all codes zero
    blocks = _raw_blocks(d, q)
    codes, s = orc.q8_0_to_axis(blocks, N, nb * 32, orc.E4M3)
    assert np.all(s[:5] == np.float32(2.0 ** -8)) and s[5] == np.float32(1e-10)
    quot = (q * (d[:, :, None].astype(np.float64) / 2.0 ** -8)).reshape(N, -1)
    want = np.array([[_e4m3_nearest(t) for t in row] for row in quot[:5]], np.uint8)
    assert np.array_equal(codes[:5], want)
    assert np.all(codes[5] == 0)
    assert _e4m3_nearest(68.0) == 0x68 and _e4m3_nearest(-68.0) == 0xE8   # tie 64 | 72 -> 64 (1.000 x 2^6)


@pytest.mark.parametrize("qt", [0, 1])
def test_requant_equals_row_quantizer_on_bf16_exact_rows(orc, qt):
    """With power-of-two block scales every d q (|q| <= 127, 7 bits) is a bf16
    value, so re-quantizing the blocks must equal quantizing the dequantized
    weight axis-wise with the row quantizer (pinned by its own golden rows)."""
    rng = np.random.default_rng(12 + qt)
    N, nb = 12, 6
    d = np.exp2(rng.integers(-14, -2, size=(N, nb))).astype(np.float32)
    q = rng.integers(-127, 128, size=(N, nb, 32))
    blocks = _raw_blocks(d, q)
    deq = orc.q8_0_dequantize(blocks, N * nb * 32).reshape(N, -1)
    wu = workloads.to_u16(torch.from_numpy(deq).to(torch.bfloat16))
    assert np.array_equal(workloads.to_u16(torch.from_numpy(deq).to(torch.bfloat16)).view(np.uint16).astype(np.uint32) << 16,
                          deq.view(np.uint32))
    q1, s1 = orc.q8_0_to_axis(blocks, N, nb * 32, qt)
    q2, s2 = orc.quantize_weight(wu, qt, orc.AXIS)
    assert np.array_equal(s1, s2)
    assert np.array_equal(q1.view(np.uint8), q2)


def test_requant_e4m3_invariants(orc):
    d = workloads.gguf_q8_0(N=64, K=512)
    w = d["w_f32"].numpy()
    blocks, _ = orc.q8_0_quantize(w.reshape(-1))
    q, s = orc.q8_0_to_axis(blocks, 64, 512, orc.E4M3)
    deq = orc.q8_0_dequantize(blocks, w.size).reshape(64, 512)
    amax = np.abs(deq).max(axis=1)
    assert np.array_equal(s, (amax / np.float32(448)).astype(np.float32))
    dec = orc.decode_codes(q, orc.E4M3).astype(np.float64)
    assert np.all(np.abs(dec).max(axis=1) == 448.0)
    v = deq / s[:, None].astype(np.float64)
    # half a code step: 2^-10 below 2^-6 (subnormals), 2^(E-4) in binade E above
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -6)))
    assert np.all(np.abs(dec - v) <= np.exp2(e - 4) * (1 + 2 ** -20))
    assert np.all(np.sign(dec) * np.sign(deq) >= 0)
    # the int8 re-quantization of the same blocks is the generic entry's qt 0
    q8, s8 = orc.q8_0_to_axis_int8(blocks, 64, 512)
    q8b, s8b = orc.q8_0_to_axis(blocks, 64, 512, orc.INT8)
    assert np.array_equal(q8, q8b) and np.array_equal(s8, s8b)
