"""Layer-level error of Residual Activation Compensation -- TEST
INFRASTRUCTURE ONLY (see oracle/__init__.py).

For one dense layer Y = X W^T the rollout engine computes, with NVFP4
weights What (the only weights it holds) and NVFP4 activations,

    Y_RAC(k) = Xhat What^T + s_a rho What[:, S]^T

where S is the k channels of largest residual score and rho the bf16
residual of those channels (gist.science/it 2.2 B; "nvfp4": the residual
re-quantized in a second NVFP4 pass).  The error the correction removes is
that of activation quantization alone, the layer-level counterpart of the
activation error term the pages analyse (gist.science/it section 2):

    err(k) = ||Y_RAC(k) - X What^T||_F / ||X What^T||_F

computed in binary64 from the exact binary32 Xhat, What and the bf16 rho.
"""
from __future__ import annotations

import numpy as np

from . import (quantize, channel_score, select_topk, rac_residual, rac_residual_nvfp4, w4a4_rac_matmul,
               bf16_to_f32)


def rac_layer_error(x: np.ndarray, w: np.ndarray, ks, rac_mode: str = "bf16") -> list[float]:
    """err(k) for each k in ``ks``; x bf16 bits [T, K], w bf16 bits [N, K]."""
    assert rac_mode in ("bf16", "nvfp4")
    what = quantize(w).xhat.astype(np.float64)
    yref = bf16_to_f32(x).astype(np.float64) @ what.T
    nref = np.linalg.norm(yref)
    xq = quantize(x)
    score = channel_score(xq.resid)
    errs = []
    for k in ks:
        if k == 0:
            y = w4a4_rac_matmul(xq.xhat, xq.s_t, None, None, what)
        else:
            S = select_topk(score, k)
            if rac_mode == "nvfp4":
                rho = rac_residual_nvfp4(xq.resid, xq.s_t, S)[0]
            else:
                rho = rac_residual(xq.resid, xq.s_t, S)
            y = w4a4_rac_matmul(xq.xhat, xq.s_t, rho, S, what)
        errs.append(float(np.linalg.norm(y - yref) / nref))
    return errs
