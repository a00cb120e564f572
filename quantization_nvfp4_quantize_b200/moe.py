"""The QUADS rollout MoE expert layer on the library's kernels.

One forward = the whole hot path (QUADS pages: gist.science/it sections 1
and 2.2 B; shd-paper.top abstract):

  1. moe_route                 top-k_r routing, expert-grouped padded row layout
  2. nvfp4_quantize(X)         amax -> s_x, codes/scales written to every routed
                               row of each token, channel scores, top-k S_x,
                               RAC residual rho_x for every routed row
  3. gather_weight_channels_cm W13q[:, :, S_x] as bf16 (e2m1 * sf), read from
                               the channel-major weight copy
  4. grouped GEMM (gate/up)    W4A4 + RAC, epilogue SwiGLU -> h bf16 and max |h|
  5. nvfp4_quantize(h)         over the valid routed rows, s_h from the epilogue's
                               max |h| (no amax pass): codes, S_h, rho_h
  6. gather_weight_channels_cm W2q[:, :, S_h]
  7. grouped GEMM (down)       W4A4 + RAC, epilogue router-weighted scatter-add
                               into Y [T x H] fp32

Weights are quantized to NVFP4 once at construction (the rollout engine holds
NVFP4 weights).  All buffers are allocated once; ``forward`` launches only the
library's kernels plus one memset of Y.
"""
from __future__ import annotations

import torch

from . import api


def rac_channels(percent: float, K: int) -> int:
    """RAC channel count for "the top k% of channels" (gist.science/it 2.2 B,
    e.g. 50%): round(percent / 100 * K)."""
    return int(round(percent / 100.0 * K))


class MoELayerW4A4:
    """rac_k: RAC channels of the gate/up input X (and of h unless rac_k_h is
    given); see rac_channels for a percentage.  rac_scope "expert" selects the
    channel sets per expert (nvfp4_quantize_experts): X through its complete
    routed copy, h directly; rac_mode must then be "bf16"."""

    def __init__(self, w13: torch.Tensor, w2: torch.Tensor, tokens: int, topk: int, rac_k: int,
                 seg_align: int = 256, rac_k_h: int | None = None, rac_mode: str = "bf16",
                 rac_scope: str = "tensor"):
        assert w13.dtype == torch.bfloat16 and w2.dtype == torch.bfloat16
        E, N13, H = w13.shape
        E2, H2, I = w2.shape
        assert E2 == E and H2 == H and N13 == 2 * I
        dev = w13.device
        self.E, self.H, self.I, self.T, self.k_r = E, H, I, tokens, topk
        assert rac_mode in ("bf16", "nvfp4") and rac_scope in ("tensor", "expert")
        assert rac_scope == "tensor" or (rac_mode == "bf16" and rac_k > 0 and (rac_k_h is None or rac_k_h > 0))
        self.rac_mode = rac_mode            # "nvfp4": second NVFP4 pass over the selected residual channels
        self.rac_scope = rac_scope
        self.rac_k = rac_k
        self.rac_k_h = rac_k if rac_k_h is None else rac_k_h
        self.rac_ld = -(-rac_k // 64) * 64 if rac_k else 0
        self.rac_ld_h = -(-self.rac_k_h // 64) * 64 if self.rac_k_h else 0
        _, self.s13, self.c13, self.sf13 = api.qdq_weights(w13, want_qdq=False, want_packed=True)
        _, self.s2, self.c2, self.sf2 = api.qdq_weights(w2, want_qdq=False, want_packed=True)
        # channel-major copies: the per-step RAC gathers read only the selected channels
        self.c13_cm, self.sf13_cm = api.weights_channel_major(self.c13, self.sf13, 2 * I, H)
        self.c2_cm, self.sf2_cm = api.weights_channel_major(self.c2, self.sf2, H, I)
        self.seg_align = seg_align          # 256: 2-SM GEMM tiles; 128: one SM per tile
        self.m_pad = api.padded_rows_bound(tokens, topk, E, seg_align)
        mp, ld, ldh = self.m_pad, max(self.rac_ld, 1), max(self.rac_ld_h, 1)
        self.xq = api.Quantized(
            codes=torch.empty(mp, H // 2, dtype=torch.uint8, device=dev),
            scales=torch.empty(api.scale_bytes(mp, H), dtype=torch.uint8, device=dev),
            s_t=torch.empty(1, dtype=torch.float32, device=dev),
            score=torch.empty(H, dtype=torch.float64, device=dev),
            sel=torch.empty(max(rac_k, 1), dtype=torch.int32, device=dev),
            r_sel=torch.empty(mp, ld, dtype=torch.bfloat16, device=dev))
        self.hq = api.Quantized(
            codes=torch.empty(mp, I // 2, dtype=torch.uint8, device=dev),
            scales=torch.empty(api.scale_bytes(mp, I), dtype=torch.uint8, device=dev),
            s_t=torch.empty(1, dtype=torch.float32, device=dev),
            score=torch.empty(I, dtype=torch.float64, device=dev),
            sel=torch.empty(max(self.rac_k_h, 1), dtype=torch.int32, device=dev),
            r_sel=torch.empty(mp, ldh, dtype=torch.bfloat16, device=dev))
        self.w_sel13 = torch.empty(E, 2 * I, ld, dtype=torch.bfloat16, device=dev)
        self.w_sel2 = torch.empty(E, H, ldh, dtype=torch.bfloat16, device=dev)
        self.h = torch.empty(mp, I, dtype=torch.bfloat16, device=dev)
        self.y = torch.empty(tokens, H, dtype=torch.float32, device=dev)
        self.h_amax = torch.empty(1, dtype=torch.float32, device=dev)
        lib = api._lib.load()
        self.ws_x = api._ws(lib.nvfp4_quantize_workspace_size(tokens, H), dev)
        self.ws_h = api._ws(lib.nvfp4_quantize_workspace_size(mp, I), dev)
        self.routing = None
        if rac_scope == "expert":
            # per-expert sets: [E x k] selections, the routed copy of X, and
            # workspaces sized for the routed rows
            self.xq.sel = torch.empty(E, rac_k, dtype=torch.int32, device=dev)
            self.hq.sel = torch.empty(E, self.rac_k_h, dtype=torch.int32, device=dev)
            self.xq.score = self.hq.score = None
            self.x_routed = torch.empty(mp, H, dtype=torch.bfloat16, device=dev)
            self.ws_x = api._ws(lib.nvfp4_quantize_experts_workspace_size(mp, H, E, seg_align), dev)
            self.ws_h = api._ws(lib.nvfp4_quantize_experts_workspace_size(mp, I, E, seg_align), dev)

    def forward(self, x: torch.Tensor, logits: torch.Tensor) -> torch.Tensor:
        if self.rac_scope == "expert":
            return self._forward_experts(x, logits)
        E, H, I, k, kh = self.E, self.H, self.I, self.rac_k, self.rac_k_h
        r = api.route(logits, self.k_r, self.m_pad, self.seg_align) if self.routing is None else self._route_into(logits)
        self.routing = r
        nvfp4_rac = self.rac_mode == "nvfp4"          # the second pass writes the RAC operand
        api.quantize(x, rac_k=k, rac_ld=self.rac_ld, dst_rows=r.dst_row, fanout=self.k_r, m_out=self.m_pad,
                     out=self.xq, workspace=self.ws_x, want_residual=not nvfp4_rac)
        if k and self.rac_mode == "nvfp4":
            api.rac_residual_nvfp4(x, self.xq, k, self.rac_ld, dst_rows=r.dst_row, fanout=self.k_r, m_out=self.m_pad)
        if k:
            api.gather_weight_channels_cm(self.c13_cm, self.sf13_cm, 2 * I, H, self.xq.sel, k, self.rac_ld,
                                          out=self.w_sel13)
        api.grouped_gemm(self.xq.codes, self.xq.scales, self.xq.s_t, self.m_pad, self.c13, self.sf13, self.s13,
                         2 * I, H, E, r.offsets, seg_align=self.seg_align, rac_ld=self.rac_ld if k else 0, rho=self.xq.r_sel,
                         w_sel=self.w_sel13, epilogue=api.EPI_SWIGLU_BF16, row_token=r.row_token,
                         row_gate=r.row_gate, out=self.h, amax_out=self.h_amax)
        api.quantize(self.h, rac_k=kh, rac_ld=self.rac_ld_h, m_out=self.m_pad, m_valid=r.offsets[E:],
                     amax=self.h_amax, out=self.hq, workspace=self.ws_h, want_residual=not nvfp4_rac)
        if kh and self.rac_mode == "nvfp4":
            api.rac_residual_nvfp4(self.h, self.hq, kh, self.rac_ld_h, m_out=self.m_pad, m_valid=r.offsets[E:])
        if kh:
            api.gather_weight_channels_cm(self.c2_cm, self.sf2_cm, H, I, self.hq.sel, kh, self.rac_ld_h,
                                          out=self.w_sel2)
        self.y.zero_()
        api.grouped_gemm(self.hq.codes, self.hq.scales, self.hq.s_t, self.m_pad, self.c2, self.sf2, self.s2,
                         H, I, E, r.offsets, seg_align=self.seg_align, rac_ld=self.rac_ld_h if kh else 0,
                         rho=self.hq.r_sel, w_sel=self.w_sel2,
                         epilogue=api.EPI_SCATTER_ADD_F32, row_token=r.row_token, row_gate=r.row_gate, out=self.y)
        return self.y

    def _forward_experts(self, x: torch.Tensor, logits: torch.Tensor) -> torch.Tensor:
        """The layer with one RAC channel set per expert for X and for h."""
        E, H, I, k, kh, sa = self.E, self.H, self.I, self.rac_k, self.rac_k_h, self.seg_align
        r = api.route(logits, self.k_r, self.m_pad, sa) if self.routing is None else self._route_into(logits)
        self.routing = r
        api.routed_rows_bf16(x, r.row_token, self.m_pad, out=self.x_routed)
        api.quantize_experts(self.x_routed, r.offsets, E, sa, rac_k=k, rac_ld=self.rac_ld, out=self.xq,
                             workspace=self.ws_x)
        api.gather_weight_channels_cm_experts(self.c13_cm, self.sf13_cm, 2 * I, H, self.xq.sel, k, self.rac_ld,
                                              out=self.w_sel13)
        api.grouped_gemm(self.xq.codes, self.xq.scales, self.xq.s_t, self.m_pad, self.c13, self.sf13, self.s13,
                         2 * I, H, E, r.offsets, seg_align=sa, rac_ld=self.rac_ld, rho=self.xq.r_sel,
                         w_sel=self.w_sel13, epilogue=api.EPI_SWIGLU_BF16, row_token=r.row_token,
                         row_gate=r.row_gate, out=self.h, amax_out=self.h_amax)
        api.quantize_experts(self.h, r.offsets, E, sa, rac_k=kh, rac_ld=self.rac_ld_h, amax=self.h_amax,
                             out=self.hq, workspace=self.ws_h)
        api.gather_weight_channels_cm_experts(self.c2_cm, self.sf2_cm, H, I, self.hq.sel, kh, self.rac_ld_h,
                                              out=self.w_sel2)
        self.y.zero_()
        api.grouped_gemm(self.hq.codes, self.hq.scales, self.hq.s_t, self.m_pad, self.c2, self.sf2, self.s2,
                         H, I, E, r.offsets, seg_align=sa, rac_ld=self.rac_ld_h, rho=self.hq.r_sel, w_sel=self.w_sel2,
                         epilogue=api.EPI_SCATTER_ADD_F32, row_token=r.row_token, row_gate=r.row_gate, out=self.y)
        return self.y

    def _route_into(self, logits):
        lib = api._lib.load()
        r = self.routing
        T, E = logits.shape
        ws = getattr(self, "_ws_route", None)
        if ws is None:
            ws = self._ws_route = api._ws(lib.moe_route_workspace_size(T, E), logits.device)
        api.check(lib.moe_route(api._p(logits), T, E, self.k_r, api._p(r.topk_idx), api._p(r.topk_gate),
                                self.seg_align, api._p(r.offsets), api._p(r.dst_row), api._p(r.row_token), api._p(r.row_gate),
                                r.m_pad_max, api._p(ws), ws.numel(), api._stream(logits.device)))
        return r


class MoELayerW4A16:
    """Trainer-side asymmetric QAT layer (gist.science/it 2.2 A): the expert
    weights are fake-quantized to NVFP4 (nvfp4_qdq_weights: bf16 ->
    NVFP4 with each expert tensor's own scale -> bf16), activations stay
    BF16, and both expert GEMMs run as BF16 grouped GEMMs on the tensor cores:

      1. moe_route               as in MoELayerW4A4
      2. moe_gather_rows_bf16    X rows to their routed rows
      3. BF16 grouped GEMM       X Wq13^T, epilogue SwiGLU -> h bf16
      4. BF16 grouped GEMM       h Wq2^T, epilogue router-weighted scatter-add
                                 into Y [T x H] fp32
    """

    def __init__(self, w13: torch.Tensor, w2: torch.Tensor, tokens: int, topk: int, seg_align: int = 256):
        assert w13.dtype == torch.bfloat16 and w2.dtype == torch.bfloat16
        E, N13, H = w13.shape
        E2, H2, I = w2.shape
        assert E2 == E and H2 == H and N13 == 2 * I
        dev = w13.device
        self.E, self.H, self.I, self.T, self.k_r = E, H, I, tokens, topk
        self.wq13 = torch.empty_like(w13)
        self.wq2 = torch.empty_like(w2)
        self.s13 = torch.empty(E, dtype=torch.float32, device=dev)
        self.s2 = torch.empty(E, dtype=torch.float32, device=dev)
        lib = api._lib.load()
        self.ws_qdq = api._ws(max(lib.nvfp4_qdq_workspace_size(E, 2 * I, H), lib.nvfp4_qdq_workspace_size(E, H, I)), dev)
        self.set_weights(w13, w2)
        self.seg_align = seg_align
        self.m_pad = api.padded_rows_bound(tokens, topk, E, seg_align)
        self.xr = torch.zeros(self.m_pad, H, dtype=torch.bfloat16, device=dev)
        self.h = torch.empty(self.m_pad, I, dtype=torch.bfloat16, device=dev)
        self.y = torch.empty(tokens, H, dtype=torch.float32, device=dev)
        self.routing = None

    def set_weights(self, w13: torch.Tensor, w2: torch.Tensor):
        """Fake-quantize new bf16 weights into the layer (the per-step work of
        QAT, where the weights change every optimizer step)."""
        lib = api._lib.load()
        st = api._stream(w13.device)
        for w, wq, s_t in ((w13, self.wq13, self.s13), (w2, self.wq2, self.s2)):
            assert w.shape == wq.shape and w.dtype == torch.bfloat16 and w.is_contiguous()
            G, rows, cols = w.shape
            api.check(lib.nvfp4_qdq_weights(api._p(w), G, rows, cols, api._p(wq), api._p(s_t), None, None,
                                            api._p(self.ws_qdq), self.ws_qdq.numel(), st))

    def forward(self, x: torch.Tensor, logits: torch.Tensor) -> torch.Tensor:
        E, H, I = self.E, self.H, self.I
        r = api.route(logits, self.k_r, self.m_pad, self.seg_align) if self.routing is None else self._route_into(logits)
        self.routing = r
        api.gather_rows_bf16(x, r.dst_row, self.m_pad, out=self.xr)
        api.bf16_grouped_gemm(self.xr, self.m_pad, self.wq13, 2 * I, H, E, r.offsets, seg_align=self.seg_align,
                              epilogue=api.EPI_SWIGLU_BF16, row_token=r.row_token, row_gate=r.row_gate, out=self.h)
        self.y.zero_()
        api.bf16_grouped_gemm(self.h, self.m_pad, self.wq2, H, I, E, r.offsets, seg_align=self.seg_align,
                              epilogue=api.EPI_SCATTER_ADD_F32, row_token=r.row_token, row_gate=r.row_gate,
                              out=self.y)
        return self.y

    _route_into = MoELayerW4A4._route_into


class MoELayerW8A8:
    """The FP8 rollout the pages compare NVFP4 against (gist.science/it
    sections 1 and 4), on the same expert layer: per-tensor E4M3 weights
    (quantized once) and activations (quantized online, X to its routed rows,
    h with the scale from the gate/up epilogue's max |h|), grouped E4M3 GEMMs
    with the SwiGLU and router-weighted combine epilogues.  No RAC."""

    def __init__(self, w13: torch.Tensor, w2: torch.Tensor, tokens: int, topk: int, seg_align: int = 256):
        E, N13, H = w13.shape
        _, _, I = w2.shape
        dev = w13.device
        self.E, self.H, self.I, self.T, self.k_r, self.seg_align = E, H, I, tokens, topk, seg_align
        self.c13, self.s13 = api.fp8_quantize(w13.contiguous())
        self.c2, self.s2 = api.fp8_quantize(w2.contiguous())
        self.m_pad = api.padded_rows_bound(tokens, topk, E, seg_align)
        self.xc = torch.empty(self.m_pad, H, dtype=torch.uint8, device=dev)
        self.xs = torch.empty(1, dtype=torch.float32, device=dev)
        self.h = torch.empty(self.m_pad, I, dtype=torch.bfloat16, device=dev)
        self.hc = torch.empty(self.m_pad, I, dtype=torch.uint8, device=dev)
        self.hs = torch.empty(1, dtype=torch.float32, device=dev)
        self.h_amax = torch.empty(1, dtype=torch.float32, device=dev)
        self.y = torch.empty(tokens, H, dtype=torch.float32, device=dev)
        self.routing = None

    def forward(self, x: torch.Tensor, logits: torch.Tensor) -> torch.Tensor:
        E, H, I = self.E, self.H, self.I
        r = api.route(logits, self.k_r, self.m_pad, self.seg_align) if self.routing is None else self._route_into(logits)
        self.routing = r
        api.fp8_quantize(x, dst_rows=r.dst_row, fanout=self.k_r, m_out=self.m_pad, codes=self.xc, s_out=self.xs)
        api.w8a8_grouped_gemm(self.xc, self.xs, self.m_pad, self.c13, self.s13, 2 * I, H, E, r.offsets,
                              seg_align=self.seg_align, epilogue=api.EPI_SWIGLU_BF16, row_token=r.row_token,
                              row_gate=r.row_gate, out=self.h, amax_out=self.h_amax)
        api.fp8_quantize(self.h, amax=self.h_amax, codes=self.hc, s_out=self.hs)
        self.y.zero_()
        api.w8a8_grouped_gemm(self.hc, self.hs, self.m_pad, self.c2, self.s2, H, I, E, r.offsets,
                              seg_align=self.seg_align, epilogue=api.EPI_SCATTER_ADD_F32, row_token=r.row_token,
                              row_gate=r.row_gate, out=self.y)
        return self.y

    _route_into = MoELayerW4A4._route_into


class DenseLayerW4A4:
    """Single dense W4A4 + RAC layer: Y = Xq Wq^T + RAC, fp32 out (one expert,
    identity routing)."""

    def __init__(self, w: torch.Tensor, tokens: int, rac_k: int):
        N, K = w.shape
        self.N, self.K, self.T, self.rac_k = N, K, tokens, rac_k
        self.rac_ld = -(-rac_k // 64) * 64 if rac_k else 0
        _, self.s_w, self.c_w, self.sf_w = api.qdq_weights(w.unsqueeze(0).contiguous(), want_qdq=False,
                                                           want_packed=True)
        self.m_pad = api.padded_rows_bound(tokens, 1, 1)
        dev = w.device
        self.out = torch.empty(self.m_pad, N, dtype=torch.float32, device=dev)
        self.w_sel = torch.empty(1, N, max(self.rac_ld, 1), dtype=torch.bfloat16, device=dev)
        self.logits = torch.zeros(tokens, 1, dtype=torch.float32, device=dev)

    def forward(self, x: torch.Tensor):
        r = api.route(self.logits, 1, self.m_pad)
        self.routing = r
        xq = api.quantize(x, rac_k=self.rac_k, rac_ld=self.rac_ld, dst_rows=r.dst_row, fanout=1, m_out=self.m_pad)
        self.xq = xq
        if self.rac_k:
            api.gather_weight_channels(self.c_w, self.sf_w, self.N, self.K, xq.sel, self.rac_k, self.rac_ld,
                                       out=self.w_sel)
        api.grouped_gemm(xq.codes, xq.scales, xq.s_t, self.m_pad, self.c_w, self.sf_w, self.s_w, self.N, self.K, 1,
                         r.offsets, rac_ld=self.rac_ld, rho=xq.r_sel, w_sel=self.w_sel,
                         epilogue=api.EPI_STORE_F32, row_token=r.row_token, row_gate=r.row_gate, out=self.out)
        return self.out[: self.T]
