"""SVDQuant weight preparation for the oracle (offline, host, fp64).

TEST INFRASTRUCTURE ONLY (see the package docstring).

OneTrainer PR #1034, section "SVDQuant": SVDQuant (arXiv 2411.05007) applied
to the quant types; OneTrainer wiki "Quantization", SVDQuant paragraph: the
low-rank factors are bfloat16 and rank 16 already helps.  The split written
out here:

    W^T [K,N] = U diag(sigma) V^T            (fp64 SVD, a library primitive)
    L1 = bf16(U_r diag(sqrt(sigma_r)))       [K, r]
    L2 = bf16(diag(sqrt(sigma_r)) V_r^T)     [r, N]
    R  = bf16(W - (L1 L2)^T)                 [N, K]   residual, after rounding
    Rq, s_R = tensor-wise quantization of R: int8 (int W8A8), or e4m3 (float
              W8A8: the wiki says SVDQuant combines with all quantized types
              except GGUF)

so that X W^T ~= X L1 L2 + X R^T.  Activation smoothing from the paper is not
on the pages and is not applied.
"""
from __future__ import annotations

import numpy as np

from . import INT8, TENSOR, bf16_to_f32, f32_to_bf16, quantize_weight


def svd_split(w_bf16, r):
    """Return (l1_bf16 [K,r], l2_bf16 [r,N], resid_bf16 [N,K])."""
    w = bf16_to_f32(w_bf16).astype(np.float64)          # [N, K]
    u, sig, vt = np.linalg.svd(w.T, full_matrices=False)  # w.T = u diag(sig) vt
    root = np.sqrt(sig[:r])
    l1 = f32_to_bf16((u[:, :r] * root[None, :]).astype(np.float32))   # [K, r]
    l2 = f32_to_bf16((root[:, None] * vt[:r, :]).astype(np.float32))  # [r, N]
    lowrank = bf16_to_f32(l1).astype(np.float64) @ bf16_to_f32(l2).astype(np.float64)  # [K, N]
    resid = f32_to_bf16((w - lowrank.T).astype(np.float32))
    return l1, l2, resid


def prepare(w_bf16, r, qt=INT8):
    """Full SVDQuant weight prep: factors plus the tensor-wise residual codes
    (qt: INT8 or E4M3)."""
    l1, l2, resid = svd_split(w_bf16, r)
    rq, s_r = quantize_weight(resid, qt, TENSOR)
    return {"l1": l1, "l2": l2, "resid": resid, "rq": rq, "s_r": s_r}
