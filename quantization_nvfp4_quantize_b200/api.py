"""Thin PyTorch-facing binding of the C ABI (include/nvfp4_quads.h).

Each function only allocates output buffers with torch (device memory is
PyTorch's), marshals pointers and sizes, and calls the library on the current
CUDA stream; every step of the computation runs in the library's kernels.
There is no CPU or PyTorch fallback.
"""
from __future__ import annotations

import dataclasses

import torch

from . import _lib
from ._lib import check

U8 = torch.uint8
I32 = torch.int32
F32 = torch.float32
F64 = torch.float64
BF16 = torch.bfloat16

EPI_STORE_F32 = 0
EPI_SWIGLU_BF16 = 1
EPI_SCATTER_ADD_F32 = 2


def _p(t):
    return None if t is None else t.data_ptr()


def _stream(device=None):
    if device is not None and torch.device(device).type != "cuda":
        raise ValueError(f"the NVFP4 kernels run on CUDA tensors only (got a tensor on {device}); "
                         "there is no CPU path")
    return torch.cuda.current_stream(device).cuda_stream


def _ws(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(16, int(nbytes)), dtype=U8, device=device)


def scale_bytes(rows: int, K: int) -> int:
    """Bytes of a swizzled scale buffer: rows padded to 128, K/16 scales each."""
    return -(-rows // 128) * 128 * (K // 16)


@dataclasses.dataclass
class Quantized:
    codes: torch.Tensor          # uint8 [M_out, K/2]
    scales: torch.Tensor         # uint8 swizzled
    s_t: torch.Tensor            # float32 [1]
    score: torch.Tensor | None   # float64 [K]
    sel: torch.Tensor | None     # int32 [rac_k]
    r_sel: torch.Tensor | None   # bf16 [M_out, rac_ld]


def quantize(x: torch.Tensor, *, rac_k: int = 0, rac_ld: int | None = None, s_t: torch.Tensor | None = None,
             amax: torch.Tensor | None = None,
             dst_rows: torch.Tensor | None = None, fanout: int = 1, m_out: int | None = None,
             m_valid: torch.Tensor | None = None, want_score: bool = False, out: Quantized | None = None,
             workspace: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
             want_residual: bool = True) -> Quantized:
    """nvfp4_quantize on a bf16 [M, K] tensor (see the header for semantics).
    want_residual=False selects the RAC channels without writing r_sel."""
    lib = _lib.load()
    assert x.dtype == BF16 and x.dim() == 2 and x.stride(1) == 1
    M, K = x.shape
    dev = x.device
    if m_out is None:
        m_out = M
    if rac_ld is None:
        rac_ld = -(-rac_k // 64) * 64 if rac_k else 0
    if out is None:
        out = Quantized(
            codes=torch.empty(m_out, K // 2, dtype=U8, device=dev),
            scales=torch.empty(scale_bytes(m_out, K), dtype=U8, device=dev),
            s_t=torch.empty(1, dtype=F32, device=dev),
            score=torch.empty(K, dtype=F64, device=dev) if (want_score or rac_k) else None,
            sel=torch.empty(max(rac_k, 1), dtype=I32, device=dev) if rac_k else None,
            r_sel=torch.empty(m_out, max(rac_ld, 1), dtype=BF16, device=dev) if rac_k else None,
        )
    if workspace is None:
        workspace = _ws(lib.nvfp4_quantize_workspace_size(M, K), dev)
    check(lib.nvfp4_quantize(_p(x), M, K, x.stride(0), _p(m_valid), _p(s_t), _p(amax), _p(out.s_t), _p(dst_rows),
                             fanout, m_out, _p(out.codes), _p(out.scales), _p(out.score), rac_k, rac_ld,
                             _p(out.sel), _p(out.r_sel) if want_residual else None, _p(dev_status), _p(workspace),
                             workspace.numel(), _stream(dev)))
    return out


def quantize_experts(x: torch.Tensor, offsets: torch.Tensor, E: int, seg_align: int, *, rac_k: int,
                     rac_ld: int | None = None, s_t: torch.Tensor | None = None, amax: torch.Tensor | None = None,
                     want_score: bool = False, out: Quantized | None = None, workspace: torch.Tensor | None = None,
                     dev_status: torch.Tensor | None = None) -> Quantized:
    """nvfp4_quantize_experts on expert-grouped routed rows bf16 [M, K]: one
    RAC channel set per expert (sel [E, rac_k], score [E, K])."""
    lib = _lib.load()
    assert x.dtype == BF16 and x.dim() == 2 and x.stride(1) == 1
    M, K = x.shape
    dev = x.device
    if rac_ld is None:
        rac_ld = -(-rac_k // 64) * 64
    if out is None:
        out = Quantized(
            codes=torch.empty(M, K // 2, dtype=U8, device=dev),
            scales=torch.empty(scale_bytes(M, K), dtype=U8, device=dev),
            s_t=torch.empty(1, dtype=F32, device=dev),
            score=torch.empty(E, K, dtype=F64, device=dev) if want_score else None,
            sel=torch.empty(E, rac_k, dtype=I32, device=dev),
            r_sel=torch.empty(M, rac_ld, dtype=BF16, device=dev),
        )
    if workspace is None:
        workspace = _ws(lib.nvfp4_quantize_experts_workspace_size(M, K, E, seg_align), dev)
    check(lib.nvfp4_quantize_experts(_p(x), M, K, x.stride(0), _p(offsets), E, seg_align, _p(s_t), _p(amax),
                                     _p(out.s_t), _p(out.codes), _p(out.scales), _p(out.score), rac_k, rac_ld,
                                     _p(out.sel), _p(out.r_sel), _p(dev_status), _p(workspace), workspace.numel(),
                                     _stream(dev)))
    return out


def qdq_weights(w: torch.Tensor, *, want_qdq: bool = True, want_packed: bool = False):
    """nvfp4_qdq_weights on bf16 [G, rows, cols] (or [rows, cols]).
    Returns (w_qdq or None, s_t [G], codes or None, scales or None)."""
    lib = _lib.load()
    assert w.dtype == BF16 and w.is_contiguous()
    squeeze = w.dim() == 2
    w3 = w.unsqueeze(0) if squeeze else w
    G, rows, cols = w3.shape
    dev = w.device
    w_qdq = torch.empty_like(w3) if want_qdq else None
    s_t = torch.empty(G, dtype=F32, device=dev)
    codes = torch.empty(G, rows, cols // 2, dtype=U8, device=dev) if want_packed else None
    scales = torch.empty(G, scale_bytes(rows, cols), dtype=U8, device=dev) if want_packed else None
    ws = _ws(lib.nvfp4_qdq_workspace_size(G, rows, cols), dev)
    check(lib.nvfp4_qdq_weights(_p(w3), G, rows, cols, _p(w_qdq), _p(s_t), _p(codes), _p(scales), _p(ws),
                                ws.numel(), _stream(dev)))
    if squeeze and w_qdq is not None:
        w_qdq = w_qdq[0]
    return w_qdq, s_t, codes, scales


@dataclasses.dataclass
class Routing:
    topk_idx: torch.Tensor      # int32 [T, k_r]
    topk_gate: torch.Tensor     # float32 [T, k_r]
    offsets: torch.Tensor       # int32 [E+1]
    dst_row: torch.Tensor       # int32 [T, k_r]
    row_token: torch.Tensor     # int32 [M_pad_max]
    row_gate: torch.Tensor      # float32 [M_pad_max]
    m_pad_max: int
    seg_align: int = 128


def padded_rows_bound(T: int, k_r: int, E: int, seg_align: int = 128) -> int:
    return -(-(T * k_r + E * (seg_align - 1)) // seg_align) * seg_align


def route(logits: torch.Tensor, k_r: int, m_pad_max: int | None = None, seg_align: int = 128) -> Routing:
    lib = _lib.load()
    assert logits.dtype == F32 and logits.is_contiguous()
    T, E = logits.shape
    dev = logits.device
    if m_pad_max is None:
        m_pad_max = padded_rows_bound(T, k_r, E, seg_align)
    r = Routing(torch.empty(T, k_r, dtype=I32, device=dev), torch.empty(T, k_r, dtype=F32, device=dev),
                torch.empty(E + 1, dtype=I32, device=dev), torch.empty(T, k_r, dtype=I32, device=dev),
                torch.empty(m_pad_max, dtype=I32, device=dev), torch.empty(m_pad_max, dtype=F32, device=dev),
                m_pad_max, seg_align)
    ws = _ws(lib.moe_route_workspace_size(T, E), dev)
    check(lib.moe_route(_p(logits), T, E, k_r, _p(r.topk_idx), _p(r.topk_gate), seg_align, _p(r.offsets), _p(r.dst_row),
                        _p(r.row_token), _p(r.row_gate), m_pad_max, _p(ws), ws.numel(), _stream(dev)))
    return r


def gather_weight_channels(codes: torch.Tensor, scales: torch.Tensor, N: int, K: int, sel: torch.Tensor,
                           k: int, ld: int, out: torch.Tensor | None = None) -> torch.Tensor:
    lib = _lib.load()
    E = codes.shape[0]
    if out is None:
        out = torch.empty(E, N, ld, dtype=BF16, device=codes.device)
    check(lib.nvfp4_gather_weight_channels(_p(codes), _p(scales), E, N, K, _p(sel), k, ld, _p(out),
                                           _stream(codes.device)))
    return out


def weights_channel_major(codes: torch.Tensor, scales: torch.Tensor, N: int, K: int):
    """nvfp4_weights_channel_major: (codes_cm [E, K, N/2], scales_cm [E, K/16, N])."""
    lib = _lib.load()
    E = codes.shape[0]
    ccm = torch.empty(E, K, N // 2, dtype=U8, device=codes.device)
    scm = torch.empty(E, K // 16, N, dtype=U8, device=codes.device)
    check(lib.nvfp4_weights_channel_major(_p(codes), _p(scales), E, N, K, _p(ccm), _p(scm), _stream(codes.device)))
    return ccm, scm


def gather_weight_channels_cm(codes_cm: torch.Tensor, scales_cm: torch.Tensor, N: int, K: int, sel: torch.Tensor,
                              k: int, ld: int, out: torch.Tensor | None = None) -> torch.Tensor:
    lib = _lib.load()
    E = codes_cm.shape[0]
    if out is None:
        out = torch.empty(E, N, ld, dtype=BF16, device=codes_cm.device)
    check(lib.nvfp4_gather_weight_channels_cm(_p(codes_cm), _p(scales_cm), E, N, K, _p(sel), k, ld, _p(out),
                                              _stream(codes_cm.device)))
    return out


def gather_weight_channels_cm_experts(codes_cm: torch.Tensor, scales_cm: torch.Tensor, N: int, K: int,
                                      sel: torch.Tensor, k: int, ld: int, out: torch.Tensor | None = None) -> torch.Tensor:
    """nvfp4_gather_weight_channels_cm_experts: expert e gathers sel[e, :k]."""
    lib = _lib.load()
    E = codes_cm.shape[0]
    assert sel.dtype == I32 and sel.numel() >= E * k
    if out is None:
        out = torch.empty(E, N, ld, dtype=BF16, device=codes_cm.device)
    check(lib.nvfp4_gather_weight_channels_cm_experts(_p(codes_cm), _p(scales_cm), E, N, K, _p(sel), k, ld, _p(out),
                                                      _stream(codes_cm.device)))
    return out


def grouped_gemm(a_codes, a_scales, a_s_t, m_pad_max, b_codes, b_scales, b_s_t, N, K, E, offsets, *,
                 seg_align=128, rac_ld=0, rho=None, w_sel=None, epilogue=EPI_STORE_F32, row_token=None, row_gate=None,
                 out=None, ld_out=None, amax_out=None, dev_status=None):
    """moe_w4a4_grouped_gemm_rac (see the header)."""
    lib = _lib.load()
    if ld_out is None:
        ld_out = out.stride(0)
    check(lib.moe_w4a4_grouped_gemm_rac(_p(a_codes), _p(a_scales), _p(a_s_t), m_pad_max, _p(b_codes),
                                        _p(b_scales), _p(b_s_t), N, K, E, _p(offsets), seg_align, rac_ld, _p(rho),
                                        _p(w_sel), epilogue, _p(row_token), _p(row_gate), _p(out), ld_out,
                                        _p(amax_out), _p(dev_status), _stream(out.device)))
    return out


def bf16_grouped_gemm(a, m_pad_max, b, N, K, E, offsets, *, seg_align=128, epilogue=EPI_STORE_F32,
                      row_token=None, row_gate=None, out=None, ld_out=None, amax_out=None, dev_status=None):
    """moe_bf16_grouped_gemm (see the header): bf16 A [m_pad_max x lda] in
    routed order times bf16 B [E x N x K]."""
    lib = _lib.load()
    assert a.dtype == BF16 and b.dtype == BF16 and b.is_contiguous()
    if ld_out is None:
        ld_out = out.stride(0)
    check(lib.moe_bf16_grouped_gemm(_p(a), a.stride(0), m_pad_max, _p(b), N, K, E, _p(offsets), seg_align, epilogue,
                                    _p(row_token), _p(row_gate), _p(out), ld_out, _p(amax_out), _p(dev_status),
                                    _stream(out.device)))
    return out


def gather_rows_bf16(x: torch.Tensor, dst_rows: torch.Tensor, m_out: int, *, out=None):
    """moe_gather_rows_bf16: token rows of x to their routed rows (dst_rows
    int32 [T x fanout]); rows of `out` not named are left as they are."""
    lib = _lib.load()
    assert x.dtype == BF16 and x.dim() == 2 and dst_rows.dtype == I32
    T, K = x.shape
    if out is None:
        out = torch.zeros(m_out, K, dtype=BF16, device=x.device)
    check(lib.moe_gather_rows_bf16(_p(x), T, K, x.stride(0), _p(dst_rows), dst_rows.shape[1], _p(out), out.stride(0),
                                   m_out, _stream(x.device)))
    return out


def routed_rows_bf16(x: torch.Tensor, row_token: torch.Tensor, m_out: int, *, out=None):
    """moe_routed_rows_bf16: out[r] = x[row_token[r]], zero rows for padding."""
    lib = _lib.load()
    assert x.dtype == BF16 and x.dim() == 2 and x.stride(1) == 1
    T, K = x.shape
    if out is None:
        out = torch.empty(m_out, K, dtype=BF16, device=x.device)
    check(lib.moe_routed_rows_bf16(_p(x), T, K, x.stride(0), _p(row_token), _p(out), out.stride(0), m_out,
                                   _stream(x.device)))
    return out


def rac_residual_nvfp4(x: torch.Tensor, q: "Quantized", rac_k: int, rac_ld: int, *, dst_rows=None, fanout=1,
                       m_out=None, m_valid=None, s_r_out=None):
    """nvfp4_rac_residual_nvfp4: replace q.r_sel by the second-pass NVFP4
    residual operand of the channels q.sel (see the header)."""
    lib = _lib.load()
    M, K = x.shape
    if m_out is None:
        m_out = M
    ws = _ws(lib.nvfp4_rac_residual_nvfp4_workspace_size(), x.device)
    check(lib.nvfp4_rac_residual_nvfp4(_p(x), M, K, x.stride(0), _p(m_valid), _p(q.s_t), _p(q.sel), rac_k, rac_ld,
                                       _p(dst_rows), fanout, m_out, _p(q.r_sel), _p(s_r_out), _p(ws), ws.numel(),
                                       _stream(x.device)))
    return q


def fp8_quantize(x: torch.Tensor, *, s: torch.Tensor | None = None, amax: torch.Tensor | None = None,
                 dst_rows: torch.Tensor | None = None, fanout: int = 1, m_out: int | None = None,
                 codes: torch.Tensor | None = None, s_out: torch.Tensor | None = None):
    """fp8_quantize (see the header) on bf16 [M, K] or [G, M, K]: per-tensor
    E4M3 codes (sign in bit 7).  Returns (codes uint8, s float32 [G])."""
    lib = _lib.load()
    assert x.dtype == BF16 and x.stride(-1) == 1
    x3 = x.unsqueeze(0) if x.dim() == 2 else x
    G, M, K = x3.shape
    assert G == 1 or x3.is_contiguous()
    dev = x.device
    if m_out is None:
        m_out = M
    if codes is None:
        codes = torch.empty((G, m_out, K) if x.dim() == 3 else (m_out, K), dtype=U8, device=dev)
    if s_out is None:
        s_out = torch.empty(G, dtype=F32, device=dev)
    ws = _ws(lib.fp8_quantize_workspace_size(G), dev)
    check(lib.fp8_quantize(_p(x3), G, M, K, x3.stride(1), _p(s), _p(amax), _p(s_out), _p(dst_rows), fanout, m_out,
                           _p(codes), _p(ws), ws.numel(), _stream(dev)))
    return codes, s_out


def w8a8_grouped_gemm(a_codes, a_s, m_pad_max, b_codes, b_s, N, K, E, offsets, *, seg_align=128,
                      epilogue=EPI_STORE_F32, row_token=None, row_gate=None, out=None, ld_out=None, amax_out=None,
                      dev_status=None):
    """moe_w8a8_grouped_gemm (see the header): E4M3 A [m_pad_max x K] in
    routed order times E4M3 B [E x N x K] with per-tensor scales."""
    lib = _lib.load()
    if ld_out is None:
        ld_out = out.stride(0)
    check(lib.moe_w8a8_grouped_gemm(_p(a_codes), _p(a_s), m_pad_max, _p(b_codes), _p(b_s), N, K, E, _p(offsets),
                                    seg_align, epilogue, _p(row_token), _p(row_gate), _p(out), ld_out,
                                    _p(amax_out), _p(dev_status), _stream(out.device)))
    return out


def debug_encode(v: torch.Tensor):
    """nvfp4_debug_encode: (E2M1 codes, E4M3 codes) of float32 values."""
    lib = _lib.load()
    assert v.dtype == F32 and v.is_contiguous()
    e2 = torch.empty(v.shape, dtype=U8, device=v.device)
    e4 = torch.empty(v.shape, dtype=U8, device=v.device)
    check(lib.nvfp4_debug_encode(_p(v), v.numel(), _p(e2), _p(e4), _stream(v.device)))
    return e2, e4


def read_status(dev_status: torch.Tensor) -> int:
    lib = _lib.load()
    import ctypes
    out = ctypes.c_int32(0)
    check(lib.nvfp4_read_status(_p(dev_status), ctypes.addressof(out), _stream(dev_status.device)))
    return int(out.value)
