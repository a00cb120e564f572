"""Layer-level error of W4A4 + Residual Activation Compensation on the GPU.

For one dense layer with NVFP4 weights What the rollout product is

    Y_RAC(k) = Xhat What^T + s_a rho What[:, S]^T       (S: k channels of largest residual score)

and the error it leaves against the product with unquantized activations is

    err(k) = ||Y_RAC(k) - X What^T||_F / ||X What^T||_F,

the layer-level counterpart of the activation-quantization error the QUADS
pages analyse (gist.science/it section 2; RAC in section 2.2 B).  Y_RAC(k)
runs through the library (nvfp4_quantize with RAC, the weight-channel gather
and moe_w4a4_grouped_gemm_rac with one expert).  The reference X What^T runs
through the library's BF16 grouped GEMM on X and the weight's e2m1 * sf
values, which bf16 holds exactly (at most 6 significant bits), times the
weight's tensor scale: the only rounding in it is the binary32 accumulation.
The norms are taken in binary64 on the device (measurement, not the product
path).
"""
from __future__ import annotations

import torch

from . import api
from .moe import rac_channels  # noqa: F401  (k as a percentage of the channels)


class LayerErrorProbe:
    """One dense layer's NVFP4 weight and its exact reference operands; err(k)
    for any activation matrix with ``tokens`` rows."""

    def __init__(self, w: torch.Tensor, tokens: int):
        assert w.dtype == torch.bfloat16 and w.dim() == 2 and w.is_cuda
        N, K = w.shape
        dev = w.device
        self.N, self.K, self.T = N, K, tokens
        _, self.s_w, self.c_w, self.sf_w = api.qdq_weights(w.unsqueeze(0).contiguous(), want_qdq=False,
                                                           want_packed=True)
        self.m_pad = api.padded_rows_bound(tokens, 1, 1)
        self.r = api.route(torch.zeros(tokens, 1, dtype=torch.float32, device=dev), 1, self.m_pad)
        every = torch.arange(K, dtype=torch.int32, device=dev)
        self.wq = api.gather_weight_channels(self.c_w, self.sf_w, N, K, every, K, K)     # e2m1 * sf, [1, N, K]
        self.y = torch.empty(self.m_pad, N, dtype=torch.float32, device=dev)

    def reference(self, x: torch.Tensor) -> torch.Tensor:
        """X What^T in binary64 (from the binary32-accumulated BF16 GEMM)."""
        a = api.gather_rows_bf16(x, self.r.dst_row, self.m_pad)
        out = torch.empty(self.m_pad, self.N, dtype=torch.float32, device=x.device)
        api.bf16_grouped_gemm(a, self.m_pad, self.wq, self.N, self.K, 1, self.r.offsets,
                              epilogue=api.EPI_STORE_F32, row_token=self.r.row_token, row_gate=self.r.row_gate,
                              out=out)
        return out[: self.T].double() * self.s_w.double()

    def rac_output(self, x: torch.Tensor, k: int, rac_mode: str = "bf16") -> torch.Tensor:
        """Y_RAC(k), binary32 [T, N]."""
        assert rac_mode in ("bf16", "nvfp4")
        r, N, K = self.r, self.N, self.K
        ld = -(-k // 64) * 64 if k else 0
        xq = api.quantize(x, rac_k=k, rac_ld=ld, dst_rows=r.dst_row, fanout=1, m_out=self.m_pad)
        w_sel = None
        if k:
            if rac_mode == "nvfp4":
                api.rac_residual_nvfp4(x, xq, k, ld, dst_rows=r.dst_row, fanout=1, m_out=self.m_pad)
            w_sel = api.gather_weight_channels(self.c_w, self.sf_w, N, K, xq.sel, k, ld)
        api.grouped_gemm(xq.codes, xq.scales, xq.s_t, self.m_pad, self.c_w, self.sf_w, self.s_w, N, K, 1,
                         r.offsets, rac_ld=ld, rho=xq.r_sel, w_sel=w_sel, epilogue=api.EPI_STORE_F32,
                         row_token=r.row_token, row_gate=r.row_gate, out=self.y)
        return self.y[: self.T]

    def errors(self, x: torch.Tensor, ks, rac_mode: str = "bf16") -> list[float]:
        yref = self.reference(x)
        nref = torch.linalg.vector_norm(yref)
        out = []
        for k in ks:
            d = self.rac_output(x, k, rac_mode).double() - yref
            out.append(float(torch.linalg.vector_norm(d) / nref))
        return out
