"""Pins of the oracle's number codecs against library conversions and the
formats' closed forms (bf16, IEEE binary16, OCP E4M3FN)."""
import numpy as np
import pytest
import torch


def _all_f32_sample(n=1 << 22, seed=0):
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 1 << 32, size=n, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    return f[np.isfinite(f)]


def test_bf16_decode_exhaustive(orc):
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).float().numpy()
    got = orc.bf16_to_f32(h)
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin].view(np.uint32), ref[fin].view(np.uint32))
    assert np.array_equal(np.isnan(got), np.isnan(ref))


def test_bf16_encode_vs_torch(orc):
    f = _all_f32_sample()
    # add exact ties: low 16 bits == 0x8000 with both parities of the kept half
    rng = np.random.default_rng(1)
    hi = rng.integers(0, 0x7F7F, size=1 << 16, dtype=np.uint32)
    ties = ((hi << 16) | 0x8000).view(np.float32)
    f = np.concatenate([f, ties, -ties, np.float32([0.0, -0.0, 3.0e38, -3.4e38, 1e-40])])
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = orc.f32_to_bf16(f)
    assert np.array_equal(got, ref)


def test_bf16_encode_closed_form(orc):
    # 1 + 2^-8 is exactly halfway between 1 and 1 + 2^-7: ties to even -> 1.
    # 1 + 3*2^-8 is halfway between 1+2^-7 (odd) and 1+2^-6 (even) -> 1+2^-6.
    got = orc.f32_to_bf16(np.float32([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -20]))
    assert list(got) == [0x3F80, 0x3F82, 0x3F81]


def test_f16_decode_exhaustive(orc):
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float32)
    got = orc.f16_to_f32(h)
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin].view(np.uint32), ref[fin].view(np.uint32))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


def test_f16_encode_vs_numpy(orc):
    f = _all_f32_sample(seed=2)
    # dense coverage of the f16 range incl. subnormals and the overflow edge
    rng = np.random.default_rng(3)
    dense = (rng.standard_normal(1 << 20) * np.exp2(rng.integers(-26, 17, 1 << 20))).astype(np.float32)
    edge = np.float32([65504.0, 65519.99, 65520.0, 65536.0, 2 ** -24, 2 ** -25, 1.5 * 2 ** -24,
                       2 ** -14, 2 ** -14 - 2 ** -25, 0.0, -0.0, 1e-10])
    f = np.concatenate([f, dense, edge, -edge])
    with np.errstate(over="ignore"):
        ref = f.astype(np.float16).view(np.uint16)
    got = orc.f32_to_f16(f)
    assert np.array_equal(got, ref)


def test_e4m3_decode_table(orc):
    codes = np.arange(256, dtype=np.uint32).astype(np.uint8)
    got = orc.e4m3_to_f32(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin])
    # closed form independent of torch: 254 finite values, max 448, min 2^-9,
    # positive half strictly increasing
    assert np.isnan(got).sum() == 2
    pos = got[:127]
    assert np.all(np.diff(pos) > 0)
    assert pos.max() == 448.0 and pos[1] == 2.0 ** -9 and got[0x38] == 1.0


def test_e4m3_encode_vs_torch(orc):
    rng = np.random.default_rng(4)
    f = (rng.standard_normal(1 << 21) * np.exp2(rng.integers(-12, 9, 1 << 21))).astype(np.float32)
    f = f[np.abs(f) <= 448.0]
    # every midpoint between consecutive finite codes, and the points themselves
    grid = orc.e4m3_to_f32(np.arange(127, dtype=np.uint8)).astype(np.float64)
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)
    f = np.concatenate([f, mids, -mids, grid.astype(np.float32), -grid.astype(np.float32)])
    ref = torch.from_numpy(f).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = orc.f32_to_e4m3(f)
    assert np.array_equal(got, ref)


def test_e4m3_saturation_closed_form(orc):
    f = np.float32([448.0, 449.0, 463.99, 464.0, 480.0, 1e6, 3.4e38, np.inf])
    assert list(orc.f32_to_e4m3(f)) == [0x7E] * 8
    assert list(orc.f32_to_e4m3(-f)) == [0xFE] * 8


def test_e4m3_all_bf16_values(orc):
    """Every finite bf16 value (the activations' own grid), scaled into range."""
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    v = orc.bf16_to_f32(h)
    v = v[np.isfinite(v) & (np.abs(v) <= 448.0)]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(orc.f32_to_e4m3(v), ref)
