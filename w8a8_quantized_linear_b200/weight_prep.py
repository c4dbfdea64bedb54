"""Offline weight preparation for SVDQuant (run once when a weight is loaded,
not on the forward path).

OneTrainer PR #1034, section "SVDQuant", applies SVDQuant to the quantized
types; the OneTrainer wiki "Quantization", SVDQuant paragraph, keeps the
low-rank factors in bfloat16 and finds a small rank enough.  The weight is
split into a rank-r product and a residual, and only the residual is
quantized:

    W^T [K, N] = U diag(sigma) V^T            singular value decomposition
    L1 = bf16(U_r diag(sqrt(sigma_r)))        [K, r]  (the factors share the
    L2 = bf16(diag(sqrt(sigma_r)) V_r^T)      [r, N]   singular values evenly)
    R  = bf16(W - (L1 L2)^T)                  [N, K]  residual of the rounded factors
    Rq, s_R = tensor-wise int8 (int W8A8) or e4m3 (float W8A8) codes of R

so that X W^T ~= X L1 L2 + X R^T, which ``svdq_linear_fwd`` evaluates.  The
decomposition is a library routine (LAPACK through torch, in fp64 on the
host); the residual is formed in fp64 from the rounded factors and rounded
once to fp32, then to bf16.  The quantization of R runs in the library's
kernel (``w8a8_quantize_weight``) on the weight's device, the same call any
other weight goes through.  Activation smoothing from the SVDQuant paper is
not on the pages and is not applied.
"""
from __future__ import annotations

import torch


def svd_split(w: torch.Tensor, r: int):
    """Split W [N, K] (bf16) into (L1 [K, r], L2 [r, N], R [N, K]), all bf16,
    on the host; see the module docstring for the formulas."""
    if w.dim() != 2 or w.dtype != torch.bfloat16:
        raise ValueError("w must be a 2-D bf16 tensor")
    N, K = w.shape
    if not 1 <= r <= min(N, K):
        raise ValueError("rank r must be in [1, min(N, K)]")
    w64 = w.detach().cpu().to(torch.float64)                       # [N, K], exact
    u, sig, vh = torch.linalg.svd(w64.T, full_matrices=False)        # W^T = u diag(sig) vh
    root = sig[:r].sqrt()
    l1 = (u[:, :r] * root[None, :]).to(torch.float32).to(torch.bfloat16)      # [K, r]
    l2 = (root[:, None] * vh[:r, :]).to(torch.float32).to(torch.bfloat16)     # [r, N]
    lowrank = l1.to(torch.float64) @ l2.to(torch.float64)                     # [K, N]
    resid = (w64 - lowrank.T).to(torch.float32).to(torch.bfloat16)            # [N, K]
    return l1.contiguous(), l2.contiguous(), resid.contiguous()


def svdq_prepare(w: torch.Tensor, r: int, qt="int8"):
    """The full SVDQuant weight preparation of W [N, K] bf16 (a CUDA tensor):
    the split of ``svd_split``, then R quantized tensor-wise by the library
    (int8 or e4m3).  Returns dict(l1, l2, resid, rq, r_scale) on w's device."""
    from . import quantize_weight   # the library call; imported here to keep this module loadable alone
    l1, l2, resid = svd_split(w, r)
    dev = w.device
    resid_d = resid.to(dev)
    rq, r_scale = quantize_weight(resid_d, qt, "tensor")
    return {"l1": l1.to(dev), "l2": l2.to(dev), "resid": resid_d, "rq": rq, "r_scale": r_scale}
