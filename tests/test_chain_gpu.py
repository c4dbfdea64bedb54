"""Calls chained on one stream with no host synchronization in between.

A weight preparation (Q8_0 -> axis-wise codes, axis-wise weight quantization)
is followed directly by a forward that reads the weight it wrote, and the
weight-only forwards / input gradients (OneTrainer wiki "Quantization",
float8 and GGUF paragraphs: the weight is dequantized to the train data type
for each product) dequantize into their workspace and multiply in the same
call.  Every chain alternates two weights through the same buffers 50 times
and keeps every output.  Each output must equal, bit for bit, the output for
the same weight computed with the host synchronized between preparation and
product (the kernels are deterministic), and that output is compared with the
oracle on sampled rows.  A product that read the weight before its producer
had finished would see the other weight's values.

The weight is the GGUF configuration's 12288 x 3072 (OneTrainer wiki, GGUF A8
int paragraph), so the producer runs long enough for an early read to land
inside it; M covers the few-token kernels, the transposed product, split-K
and single-SM tiles."""
import numpy as np
import pytest
import torch

import workloads
from _tol import bf16_bits_to_f64, ulp_bf16

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
N, K = 12288, 3072
REPS = 50


@pytest.fixture(scope="module")
def w8():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w8a8_quantized_linear_b200 import _build
    _build.build()
    import w8a8_quantized_linear_b200 as m
    m.lib()
    return m


@pytest.fixture(scope="module")
def weights(orc):
    """Two different bf16 weights [N, K] and their Q8_0 blocks (quantized by
    the oracle: inputs never come from the CUDA path)."""
    out = []
    for seed in (301, 302):
        wb = workloads.normal((N, K), 0.02, seed)
        blocks, _ = orc.q8_0_quantize(wb.float().numpy().reshape(-1))
        out.append({"bf16": wb, "blocks": blocks})
    return out


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def rows_of(M):
    return sorted({0, M // 2, M - 1})


def _run_chain(prepare, product, n_out):
    """REPS rounds of prepare(i % 2) + product(out[i]) without a host sync;
    then the two reference outputs, each with the host synchronized between
    preparation and product."""
    outs = [torch.empty(n_out, dtype=torch.bfloat16, device=DEV) for _ in range(REPS)]
    torch.cuda.synchronize()
    for i in range(REPS):
        prepare(i % 2)
        product(outs[i])
    torch.cuda.synchronize()
    refs = []
    for j in (0, 1):
        prepare(j)
        torch.cuda.synchronize()
        r = torch.empty(n_out, dtype=torch.bfloat16, device=DEV)
        product(r)
        torch.cuda.synchronize()
        refs.append(r)
    assert not torch.equal(refs[0], refs[1]), "the two weights must give different outputs"
    for i, o in enumerate(outs):
        assert torch.equal(o, refs[i % 2]), "chained call %d differs from the synchronized one" % i
    return refs


@pytest.mark.parametrize("qt,M", [("int8", 1), ("int8", 64), ("int8", 200), ("e4m3", 64)])
def test_requant_then_forward_without_sync(w8, orc, weights, qt, M):
    """q8_0_to_axis_{int8,e4m3} writes the codes and scales that the next
    call's forward reads (GGUF A8 int / GGUF A8 float)."""
    blocks = [torch.from_numpy(w["blocks"]).to(DEV) for w in weights]
    dt = torch.int8 if qt == "int8" else torch.float8_e4m3fn
    wq = torch.empty((N, K), dtype=dt, device=DEV)
    sw = torch.empty((N,), dtype=torch.float32, device=DEV)
    x = workloads.normal((M, K), 1.0, 303 + M).to(DEV)
    ws = torch.empty(w8.workspace_bytes(w8.OP_LINEAR_FWD, M, N, K), dtype=torch.uint8, device=DEV)
    prepare = lambda j: w8.q8_0_to_axis(blocks[j], N, K, qt, out=wq, scale=sw)
    product = lambda y: w8.linear_fwd(x, wq, sw, out=y.view(M, N), ws=ws)
    refs = _run_chain(prepare, product, M * N)
    q = 0 if qt == "int8" else 1
    rows = rows_of(M)
    xr = workloads.to_u16(x.cpu())[rows]
    for j, w in enumerate(weights):
        wqr, swr = orc.q8_0_to_axis(w["blocks"], N, K, q)
        ref = orc.linear_fwd(xr, wqr.view(np.uint8), swr, qt=q)
        got = u16(refs[j].view(M, N))[rows]
        if q == 0:
            assert np.array_equal(got, ref["y"])
        else:
            yr, yg = bf16_bits_to_f64(ref["y"]), bf16_bits_to_f64(got)
            bound = 1e-3 * ref["sx"][:, None].astype(np.float64) * swr[None, :].astype(np.float64) * ref["absacc"] \
                + ulp_bf16(np.maximum(np.abs(yr), np.abs(yg)))
            assert np.all(np.abs(yg - yr) <= bound)


def test_axis_weight_quantize_then_forward_without_sync(w8, orc, weights):
    """w8a8_quantize_weight(AXIS) runs the row quantizer on the weight; the
    next call's forward (64 tokens: the transposed product) reads it."""
    M = 64
    wb = [w["bf16"].to(DEV) for w in weights]
    wq = torch.empty((N, K), dtype=torch.int8, device=DEV)
    sw = torch.empty((N,), dtype=torch.float32, device=DEV)
    x = workloads.normal((M, K), 1.0, 304).to(DEV)
    ws = torch.empty(w8.workspace_bytes(w8.OP_LINEAR_FWD, M, N, K), dtype=torch.uint8, device=DEV)
    lib = w8.lib()
    ptr = lambda t: w8._ptr(t)

    def prepare(j):
        w8._check(lib.w8a8_quantize_weight(ptr(wb[j]), N, K, w8.INT8, w8.AXIS, ptr(wq.view(torch.uint8)), ptr(sw),
                                           None, 0, w8._stream()))

    product = lambda y: w8.linear_fwd(x, wq, sw, out=y.view(M, N), ws=ws)
    refs = _run_chain(prepare, product, M * N)
    rows = rows_of(M)
    xr = workloads.to_u16(x.cpu())[rows]
    for j, w in enumerate(weights):
        wqr, swr = orc.quantize_weight(workloads.to_u16(w["bf16"]), orc.INT8, orc.AXIS)
        ref = orc.linear_fwd(xr, wqr, swr, qt=orc.INT8)
        assert np.array_equal(u16(refs[j].view(M, N))[rows], ref["y"])


def _bf16_bound(ref, got, klen):
    yr, yg = bf16_bits_to_f64(ref["y"]), bf16_bits_to_f64(got)
    bound = klen * 2.0 ** -23 * ref["absacc"] + ulp_bf16(np.maximum(np.abs(yr), np.abs(yg)))
    return np.abs(yg - yr), bound


@pytest.mark.parametrize("M", [1, 64, 300])
@pytest.mark.parametrize("kind", ["float8", "gguf"])
def test_weight_only_forward_without_sync(w8, orc, weights, kind, M):
    """float8_linear_fwd / gguf_linear_fwd dequantize the weight into the
    workspace and multiply in one call; consecutive calls alternate weights
    through the same workspace."""
    x = workloads.normal((M, K), 1.0, 305 + M).to(DEV)
    ws = torch.empty(w8.workspace_bytes(w8.OP_WEIGHT_ONLY_FWD, M, N, K), dtype=torch.uint8, device=DEV)
    if kind == "float8":
        q = [w8.quantize_weight(w["bf16"].to(DEV), "e4m3", "tensor") for w in weights]
        torch.cuda.synchronize()
        call = lambda j, y: w8.float8_linear_fwd(x, q[j][0], q[j][1], out=y.view(M, N), ws=ws)
    else:
        blocks = [torch.from_numpy(w["blocks"]).to(DEV) for w in weights]
        call = lambda j, y: w8.gguf_linear_fwd(x, blocks[j], N, out=y.view(M, N), ws=ws)
    state = {"j": 0}

    def prepare(j):
        state["j"] = j

    refs = _run_chain(prepare, lambda y: call(state["j"], y), M * N)
    rows = rows_of(M)
    xr = workloads.to_u16(x.cpu())[rows]
    for j, w in enumerate(weights):
        if kind == "float8":
            wqr, swr = orc.quantize_weight(workloads.to_u16(w["bf16"]), orc.E4M3, orc.TENSOR)
            ref = orc.float8_linear_fwd(xr, wqr, swr)
        else:
            ref = orc.gguf_linear_fwd(xr, w["blocks"], N, K)
        err, bound = _bf16_bound(ref, u16(refs[j].view(M, N))[rows], K)
        assert np.all(err <= bound), float((err / bound).max())


@pytest.mark.parametrize("M", [1, 64, 300])
@pytest.mark.parametrize("kind", ["float8", "gguf"])
def test_weight_only_dgrad_without_sync(w8, orc, weights, kind, M):
    """float8_linear_dgrad / gguf_linear_dgrad: dX [M, K] = dY [M, N] W."""
    dy = workloads.normal((M, N), 1e-3, 306 + M).to(DEV)
    ws = torch.empty(w8.workspace_bytes(w8.OP_WEIGHT_ONLY_DGRAD, M, N, K), dtype=torch.uint8, device=DEV)
    if kind == "float8":
        q = [w8.quantize_weight(w["bf16"].to(DEV), "e4m3", "tensor") for w in weights]
        torch.cuda.synchronize()
        call = lambda j, y: w8.float8_linear_dgrad(dy, q[j][0], q[j][1], out=y.view(M, K), ws=ws)
    else:
        blocks = [torch.from_numpy(w["blocks"]).to(DEV) for w in weights]
        call = lambda j, y: w8.gguf_linear_dgrad(dy, blocks[j], K, out=y.view(M, K), ws=ws)
    state = {"j": 0}

    def prepare(j):
        state["j"] = j

    refs = _run_chain(prepare, lambda y: call(state["j"], y), M * K)
    rows = rows_of(M)
    dyr = workloads.to_u16(dy.cpu())[rows]
    for j, w in enumerate(weights):
        if kind == "float8":
            wqr, swr = orc.quantize_weight(workloads.to_u16(w["bf16"]), orc.E4M3, orc.TENSOR)
            wd = orc.dequant_e4m3_bf16(wqr, swr).reshape(N, K)
        else:
            wd = orc.q8_0_dequantize_bf16(w["blocks"], N * K).reshape(N, K)
        ref = orc.linear_bf16_dgrad(dyr, wd)
        err, bound = _bf16_bound(ref, u16(refs[j].view(M, K))[rows], N)
        assert np.all(err <= bound), float((err / bound).max())
