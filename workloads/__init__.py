"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module only draws random numbers and shapes them; it holds none of the
quantization, matmul or epilogue arithmetic.  Values are drawn in fp32 with a
torch CPU generator of a fixed seed and rounded to bf16 by torch, so every run
on every machine sees the same inputs (bitsandbytes #1401, "Deterministic Test
Inputs").  The pages train and run unnamed DiT/LLM models; these shapes stand
in for them: hidden size 3072, MLP width 12288, 4096 image + 512 text tokens.
"""
from __future__ import annotations

import torch

HIDDEN = 3072
MLP = 12288
TOKENS = 4096 + 512


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal(shape, std: float, seed: int, dtype=torch.bfloat16) -> torch.Tensor:
    """N(0, std^2) drawn in fp32, then rounded to ``dtype`` by torch."""
    x = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def with_outlier_channels(shape, std: float, seed: int, frac: float = 0.01,
                          factor: float = 20.0) -> torch.Tensor:
    """N(0, std^2) activations whose round(frac*K) channels (a seeded choice of
    columns) are multiplied by ``factor`` in fp32 before the bf16 rounding."""
    M, K = shape
    x = torch.randn(M, K, generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    n_out = int(round(frac * K))
    cols = torch.randperm(K, generator=_gen(seed + 7919))[:n_out]
    x[:, cols] *= factor
    return x.to(torch.bfloat16)


def rank_spike_weight(N: int, K: int, rank: int, peak: float, std: float,
                      seed: int) -> torch.Tensor:
    """W = N(0, std^2) + S with S = U V^T (U [N,rank], V [K,rank] ~ N(0,1)),
    S scaled so that max |S_ij| = peak; built in fp32, rounded to bf16."""
    base = torch.randn(N, K, generator=_gen(seed), dtype=torch.float32) * std
    u = torch.randn(N, rank, generator=_gen(seed + 1), dtype=torch.float32)
    v = torch.randn(K, rank, generator=_gen(seed + 2), dtype=torch.float32)
    s = u @ v.T
    s *= peak / s.abs().max()
    return (base + s).to(torch.bfloat16)


# --------------------------------------------------------------------------- configurations
def int_tiny():
    """int W8A8 forward, tiny: X [256,512] ~ N(0,1), W [512,512] ~ N(0,0.02)."""
    return {"x": normal((256, 512), 1.0, 1), "w": normal((512, 512), 0.02, 2)}


def float_w8a8(M=4096, N=HIDDEN, K=HIDDEN):
    """float W8A8 forward: X [4096,3072], W [3072,3072], bias [3072]."""
    return {"x": normal((M, K), 1.0, 11), "w": normal((N, K), 0.02, 12),
            "bias": normal((N,), 0.01, 13)}


def dit_mlp(M=TOKENS, H=HIDDEN, F=MLP):
    """int W8A8 DiT MLP block: X [M,H] with 1% x20 outlier channels,
    W1 [F,H], W2 [H,F] ~ N(0,0.02), dY2 [M,H] ~ N(0,1e-3)."""
    return {"x": with_outlier_channels((M, H), 1.0, 21),
            "w1": normal((F, H), 0.02, 22), "w2": normal((H, F), 0.02, 23),
            "dy2": normal((M, H), 1e-3, 24)}


def svdquant(M=TOKENS, N=HIDDEN, K=HIDDEN, r=32):
    """SVDQuant: W [N,K] = N(0,0.02) + rank-8 spike of peak 0.5, X with outliers."""
    return {"x": with_outlier_channels((M, K), 1.0, 31),
            "w": rank_spike_weight(N, K, 8, 0.5, 0.02, 32),
            "bias": None, "r": r}


GGUF_MS = (1, 64, 512, 4608, 16384)


def gguf_q8_0(N=MLP, K=HIDDEN, M=4608):
    """GGUF Q8_0 path: fp32 weight [N,K] ~ N(0,0.02) (bf16-representable values,
    the bf16 weight of the configuration widened to fp32), X [M,K] ~ N(0,1)."""
    w = normal((N, K), 0.02, 41).to(torch.float32)
    return {"w_f32": w, "x": normal((M, K), 1.0, 42)}


def q8_0_standalone(n=1 << 28, seed=51):
    """Standalone Q8_0 quantize/dequantize input: n fp32 values ~ N(0,1)."""
    return torch.randn(n, generator=_gen(seed), dtype=torch.float32)


def raw_q8_0_blocks(N: int, K: int, seed: int) -> torch.Tensor:
    """Arbitrary Q8_0 block bytes for N rows of K values (K % 32 == 0): each
    34-byte block is an f16 scale followed by 32 int8 codes, both drawn at
    random rather than produced by a quantizer.  Row n % 6 picks the kind:
    0 one shared scale with +-127 present, 1 all scales zero, 2 random scales
    of both signs, 3 codes that include -128, 4 all codes zero, 5 scales in
    the f16 subnormal range."""
    nb = K // 32
    g = _gen(seed)
    codes = torch.round(torch.randn(N, nb, 32, generator=g) * 40.0).clamp_(-128, 127)
    scales = torch.rand(N, nb, generator=g) * 2e-3 + 1e-5
    signs = torch.where(torch.rand(N, nb, generator=g) < 0.1, -1.0, 1.0)
    kind = torch.arange(N) % 6
    scales = torch.where((kind == 2)[:, None], scales * signs, scales)
    scales = torch.where((kind == 0)[:, None], torch.full_like(scales, 0.02 / 127), scales)
    scales = torch.where((kind == 1)[:, None], torch.zeros_like(scales), scales)
    scales = torch.where((kind == 5)[:, None], scales * 1e-3, scales)
    idx = torch.arange(nb) % 32
    spike = torch.where(torch.arange(nb) % 2 == 0, 127.0, -127.0)
    rows0 = torch.nonzero(kind == 0).reshape(-1)
    codes[rows0] = codes[rows0].clamp(-126, 126)
    for n in rows0.tolist():
        codes[n, torch.arange(nb), idx] = spike
    neg = torch.rand(N, nb, 32, generator=g) < 1.0 / 64
    codes = torch.where((kind == 3)[:, None, None] & neg, torch.full_like(codes, -128.0), codes)
    codes = torch.where((kind == 4)[:, None, None], torch.zeros_like(codes), codes)
    out = torch.empty(N, nb, 34, dtype=torch.uint8)
    out[:, :, :2] = scales.to(torch.float16).contiguous().view(torch.uint8).view(N, nb, 2)
    out[:, :, 2:] = codes.to(torch.int8).view(torch.uint8)
    return out.reshape(-1)


def to_u16(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (for the oracle)."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")


__all__ = ["normal", "with_outlier_channels", "rank_spike_weight", "int_tiny",
           "float_w8a8", "dit_mlp", "svdquant", "gguf_q8_0", "q8_0_standalone",
           "to_u16", "GGUF_MS", "HIDDEN", "MLP", "TOKENS"]
