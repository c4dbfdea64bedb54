"""The SVDQuant weight split of the library (weight_prep.svd_split /
svdq_prepare), pinned against the mathematics of the decomposition rather
than against itself (OneTrainer PR #1034, "SVDQuant"; OneTrainer wiki
"Quantization", SVDQuant paragraph: bfloat16 low-rank factors).

Host tests: factor shapes and types; the factors carry the top r singular
values, shared evenly; an exactly low-rank weight leaves a residual at the
bf16 rounding level; on the rank-8 spike weight the low-rank branch plus the
quantized residual halves the error of plain tensor-wise int8; the split
agrees with the oracle's independent one.  The GPU test checks the residual's
codes against the oracle's quantizer bit for bit."""
import numpy as np
import pytest
import torch

import workloads
from w8a8_quantized_linear_b200.weight_prep import svd_split


def f64(t):
    return t.to(torch.float64).numpy()


def test_shapes_and_types():
    w = workloads.normal((96, 80), 0.02, 401)
    l1, l2, resid = svd_split(w, 16)
    assert l1.shape == (80, 16) and l2.shape == (16, 96) and resid.shape == (96, 80)
    assert l1.dtype == l2.dtype == resid.dtype == torch.bfloat16
    assert l1.is_contiguous() and l2.is_contiguous() and resid.is_contiguous()
    with pytest.raises(ValueError):
        svd_split(w, 0)
    with pytest.raises(ValueError):
        svd_split(w.float(), 8)


def test_factors_carry_the_top_singular_values_evenly():
    """L1 L2 has the r largest singular values of W (to bf16 rounding), and
    column j of L1 and row j of L2 both have norm sqrt(sigma_j): U and V are
    orthonormal, so the split shares each singular value evenly."""
    w = workloads.rank_spike_weight(160, 128, 8, 0.5, 0.02, 402)
    r = 12
    l1, l2, _ = svd_split(w, r)
    sig = np.linalg.svd(f64(w), compute_uv=False)[:r]
    prod = f64(l1) @ f64(l2)
    got = np.linalg.svd(prod, compute_uv=False)[:r]
    assert np.allclose(got, sig, rtol=2.0 ** -7, atol=0)
    assert np.linalg.matrix_rank(prod, tol=1e-9 * sig[0]) == r
    c1 = np.linalg.norm(f64(l1), axis=0)
    c2 = np.linalg.norm(f64(l2), axis=1)
    assert np.allclose(c1, np.sqrt(sig), rtol=2.0 ** -7)
    assert np.allclose(c2, np.sqrt(sig), rtol=2.0 ** -7)


def test_exact_low_rank_weight_leaves_rounding_residual():
    """W = bf16(A B) of rank 6: with r >= 6 the residual R = bf16(W - (L1
    L2)^T) is only what the bf16 factors and W's own rounding leave."""
    a = workloads.normal((112, 6), 0.3, 403).double()
    b = workloads.normal((6, 72), 0.3, 404).double()
    w = (a @ b).to(torch.bfloat16)        # [N=112, K=72]
    l1, l2, resid = svd_split(w, 8)
    W = f64(w)
    assert np.linalg.norm(f64(resid)) <= 2.0 ** -7 * np.linalg.norm(W)
    # and R is W minus the factors' product, rounded (bf16 of the fp64
    # difference, within one bf16 step of it)
    diff = W - (f64(l1) @ f64(l2)).T
    step = np.exp2(np.floor(np.log2(np.maximum(np.abs(diff), 2.0 ** -126))) - 7)
    assert np.all(np.abs(f64(resid) - diff) <= step)


def test_spike_weight_split_halves_int8_error(orc):
    """On the SVDQuant configuration's weight kind (N(0, 0.02) plus a rank-8
    spike of peak 0.5), ||W - (L1 L2)^T - deq(Rq)|| < 0.5 ||W - deq(Q(W))||
    with tensor-wise int8 codes (oracle quantizer) for both."""
    w = workloads.rank_spike_weight(384, 320, 8, 0.5, 0.02, 405)
    l1, l2, resid = svd_split(w, 32)
    W = f64(w)
    rq, sr = orc.quantize_weight(workloads.to_u16(resid), orc.INT8, orc.TENSOR)
    err_svd = np.linalg.norm(W - (f64(l1) @ f64(l2)).T - rq.view(np.int8).astype(np.float64) * sr[0])
    wq, sw = orc.quantize_weight(workloads.to_u16(w), orc.INT8, orc.TENSOR)
    err_plain = np.linalg.norm(W - wq.view(np.int8).astype(np.float64) * sw[0])
    assert err_svd < 0.5 * err_plain, (err_svd, err_plain)
    # the spike left W: the residual's absmax is at the noise level
    assert np.abs(f64(resid)).max() < 0.2


def test_split_agrees_with_the_oracle(orc):
    """The oracle's split (numpy LAPACK) and the library's (torch LAPACK) are
    separate programs of the same formulas; singular vectors may differ in
    sign (which the product cancels) and in the last bits (which bf16
    rounding may move by one step)."""
    from oracle import svdquant
    w = workloads.rank_spike_weight(256, 192, 8, 0.5, 0.02, 406)
    l1, l2, resid = svd_split(w, 16)
    ol1, ol2, oresid = svdquant.svd_split(workloads.to_u16(w), 16)
    to64 = lambda b: orc.bf16_to_f32(b).astype(np.float64)
    p = f64(l1) @ f64(l2)
    po = to64(ol1) @ to64(ol2)
    assert np.linalg.norm(p - po) <= 2.0 ** -8 * np.linalg.norm(p)
    assert np.linalg.norm(f64(resid) - to64(oresid)) <= 2.0 ** -8 * np.linalg.norm(f64(w))


@pytest.mark.gpu
@pytest.mark.parametrize("qt", ["int8", "e4m3"])
def test_prepare_quantizes_the_residual_like_the_oracle(orc, qt):
    """svdq_prepare's codes and scale of R equal the oracle quantizer's on
    the same R, bit for bit, and the factors it returns are svd_split's."""
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w8a8_quantized_linear_b200 import _build
    _build.build()
    import w8a8_quantized_linear_b200 as w8
    w = workloads.rank_spike_weight(520, 384, 8, 0.5, 0.02, 407)
    prep = w8.svdq_prepare(w.to("cuda:0"), 32, qt)
    l1, l2, resid = svd_split(w, 32)
    assert torch.equal(prep["l1"].cpu(), l1) and torch.equal(prep["l2"].cpu(), l2)
    assert torch.equal(prep["resid"].cpu(), resid)
    q = orc.INT8 if qt == "int8" else orc.E4M3
    rq, sr = orc.quantize_weight(workloads.to_u16(resid), q, orc.TENSOR)
    assert np.array_equal(prep["rq"].cpu().view(torch.uint8).numpy(), rq)
    assert np.array_equal(prep["r_scale"].cpu().numpy().view(np.uint32), sr.view(np.uint32))
