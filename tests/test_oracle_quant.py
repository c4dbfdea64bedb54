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
