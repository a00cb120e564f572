"""GPU parity of the FP8 comparison path (per-tensor E4M3, the FP8 rollout
the pages compare NVFP4 against): codes and scales bit-exact against the
oracle, the grouped E4M3 GEMM and the W8A8 layer within 2e-3 of the oracle's
binary64 products."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import np_u16, to_bf16_dev, rel_fro
from quantization_nvfp4_quantize_b200 import api, workloads as wl
from quantization_nvfp4_quantize_b200.moe import MoELayerW8A8

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.mark.parametrize("M,K", [(1, 16), (300, 768), (4096, 2048)])
def test_fp8_quantize_parity(cuda, M, K):
    rng = np.random.default_rng(M + K)
    x = oracle.f32_to_bf16((rng.standard_normal((M, K)) * 2.0 ** rng.uniform(-6, 6)).astype(np.float32))
    x[0, 0] = 0x8000
    codes, s = api.fp8_quantize(to_bf16_dev(x, cuda))
    torch.cuda.synchronize()
    rc, rx, rs = oracle.fp8_quantize(x)
    assert s.item() == np.float32(rs)
    assert np.array_equal(codes.cpu().numpy(), rc)


def test_fp8_quantize_boundaries_and_groups(cuda):
    """E4M3 rounding boundaries times the scale (exact ties and their
    neighbours), per-group scales, and routed copies."""
    e4 = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (e4[:-1] + e4[1:]) / 2
    rng = np.random.default_rng(9)
    G, M, K = 3, 32, 256
    w = np.empty((G, M, K), np.uint16)
    for g in range(G):
        s = 2.0 ** rng.integers(-8, 8)
        v = rng.choice(np.concatenate([mids, e4]), (M, K)) * s * np.where(rng.random((M, K)) < 0.5, -1, 1)
        w[g] = oracle.f32_to_bf16(v.astype(np.float32))
    codes, s = api.fp8_quantize(to_bf16_dev(w, cuda))
    torch.cuda.synchronize()
    for g in range(G):
        rc, _, rs = oracle.fp8_quantize(w[g])
        assert s[g].item() == np.float32(rs)
        assert np.array_equal(codes[g].cpu().numpy(), rc)
    dst = np.stack([np.arange(M), M + np.arange(M)[::-1]], axis=1).astype(np.int32)
    out, s1 = api.fp8_quantize(to_bf16_dev(w[0], cuda), dst_rows=torch.from_numpy(dst).to(cuda), fanout=2,
                               m_out=2 * M)
    torch.cuda.synchronize()
    rc, _, _ = oracle.fp8_quantize(w[0])
    o = out.cpu().numpy()
    assert np.array_equal(o[dst[:, 0]], rc) and np.array_equal(o[dst[:, 1]], rc)


@pytest.mark.parametrize("align", [128, 256])
def test_w8a8_grouped_gemm_parity(cuda, align):
    rng = np.random.default_rng(align)
    T, E, kr, N, K = 300, 8, 2, 512, 768
    x = oracle.f32_to_bf16(rng.standard_normal((T, K)).astype(np.float32))
    w = oracle.f32_to_bf16((rng.standard_normal((E, N, K)) * 0.02).astype(np.float32))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    r = api.route(torch.from_numpy(logits).to(cuda), kr, seg_align=align)
    xc, xs = api.fp8_quantize(to_bf16_dev(x, cuda), dst_rows=r.dst_row, fanout=kr, m_out=r.m_pad_max)
    wc, ws = api.fp8_quantize(to_bf16_dev(w, cuda))
    out = torch.zeros(r.m_pad_max, N, dtype=torch.float32, device=cuda)
    api.w8a8_grouped_gemm(xc, xs, r.m_pad_max, wc, ws, N, K, E, r.offsets, seg_align=align,
                          epilogue=api.EPI_STORE_F32, row_token=r.row_token, row_gate=r.row_gate, out=out)
    torch.cuda.synchronize()
    idx, _ = oracle.route(logits, kr)
    _, xh, _ = oracle.fp8_quantize(x)
    dst = r.dst_row.cpu().numpy()
    got = out.cpu().numpy()
    have, want = [], []
    for e in range(E):
        _, wh, _ = oracle.fp8_quantize(w[e])
        toks, slots = np.nonzero(idx == e)
        want.append(xh[toks].astype(np.float64) @ wh.astype(np.float64).T)
        have.append(got[dst[toks, slots]])
    assert rel_fro(np.concatenate(have), np.concatenate(want)) <= TOL


def test_w8a8_layer_matches_oracle(cuda):
    """The FP8 comparison layer end to end on the small MoE layer: per-tensor
    E4M3 X (routed), weights and h (scale from the epilogue's max |h|)."""
    cfg = wl.CONFIGS["moe_t512_e8"]
    x = wl.activations(cfg, 6)
    logits = wl.router_logits(cfg, 6)
    w13, w2 = wl.weights(cfg, 6)
    layer = MoELayerW8A8(w13.to(cuda), w2.to(cuda), cfg.tokens, cfg.topk)
    y = layer.forward(x.to(cuda), logits.to(cuda)).cpu().numpy()
    u = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    idx, gate = oracle.route(logits.numpy(), cfg.topk)
    _, xh, _ = oracle.fp8_quantize(u(x))
    T, kr, I, H = cfg.tokens, cfg.topk, cfg.inter, cfg.hidden
    h = np.zeros((T * kr, I))
    rows_t = np.repeat(np.arange(T), kr)
    flat = idx.reshape(-1)
    w13n, w2n = u(w13), u(w2)
    for e in range(cfg.experts):
        rows = np.nonzero(flat == e)[0]
        _, wh, _ = oracle.fp8_quantize(w13n[e])
        h[rows] = oracle.swiglu(xh[rows_t[rows]].astype(np.float64) @ wh.astype(np.float64).T, I)
    hb = oracle.f32_to_bf16(h.astype(np.float32))
    _, hh, _ = oracle.fp8_quantize(hb)
    Y = np.zeros((T, H))
    for e in range(cfg.experts):
        rows = np.nonzero(flat == e)[0]
        _, wh, _ = oracle.fp8_quantize(w2n[e])
        y2 = hh[rows].astype(np.float64) @ wh.astype(np.float64).T
        np.add.at(Y, rows_t[rows], y2 * gate.reshape(-1)[rows][:, None])
    assert rel_fro(y, Y) <= TOL
