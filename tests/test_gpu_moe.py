"""GPU parity of the whole MoE expert layer (route -> quantize X -> gate/up
W4A4+RAC GEMM with SwiGLU -> quantize h -> down W4A4+RAC GEMM with router
combine) against the oracle, stage by stage:

  * routing, X codes/scales/S_x/rho_x: bit-exact (tie window 1e-6);
  * h (bf16) vs the oracle's h: relative Frobenius <= 2e-3;
  * the down stage is checked on a seeded synthetic h given to both sides as
    an input (codes/scales/S_h/rho_h bit-exact, Y within 2e-3);
  * end-to-end Y from X: relative Frobenius reported and bounded.
Large workloads are checked on a seeded sample of tokens (all their routed
rows), with the quantization statistics (s_t, scores, S) over the full
tensors."""
import numpy as np
import pytest
import torch

import oracle
import oracle.moe as omoe
from gpu_util import np_u16, to_bf16_dev, rel_fro, check_selection, unswizzle
from quantization_nvfp4_quantize_b200 import api, workloads as wl
from quantization_nvfp4_quantize_b200.moe import MoELayerW4A4

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _layer_inputs(name, seed, tokens=None):
    cfg = wl.CONFIGS[name]
    x = wl.activations(cfg, seed)
    logits = wl.router_logits(cfg, seed)
    w13, w2 = wl.weights(cfg, seed)
    return cfg, x, logits, w13, w2


def _run_layer(cuda, name, seed, sample_tokens=None):
    cfg, x, logits, w13, w2 = _layer_inputs(name, seed)
    layer = MoELayerW4A4(w13.to(cuda), w2.to(cuda), cfg.tokens, cfg.topk, cfg.rac_k)
    y = layer.forward(x.to(cuda), logits.to(cuda))
    torch.cuda.synchronize()
    return cfg, x, logits, w13, w2, layer, y.cpu().numpy()


@pytest.mark.parametrize("name", ["moe_t512_e8"])
def test_moe_layer_stagewise(cuda, name):
    cfg, x, logits, w13, w2, layer, y = _run_layer(cuda, name, 0)
    xn, w13n, w2n = _u16(x), _u16(w13), _u16(w2)
    T, kr, E, I, k = cfg.tokens, cfg.topk, cfg.experts, cfg.inter, cfg.rac_k
    r = layer.routing
    # routing
    idx, gate = oracle.route(logits.numpy(), kr)
    assert np.array_equal(r.topk_idx.cpu().numpy(), idx)
    # X quantization + selection + rho, per routed row
    qx = oracle.quantize(xn)
    score = oracle.channel_score(qx.resid)
    S_x = oracle.select_topk(score, k)
    check_selection(layer.xq.sel.cpu().numpy(), score, S_x, k)
    assert np.array_equal(layer.xq.sel.cpu().numpy()[:k], S_x)
    dst = r.dst_row.cpu().numpy()
    codes = layer.xq.codes.cpu().numpy()
    sf = unswizzle(layer.xq.scales, layer.m_pad, cfg.hidden)
    rho = np_u16(layer.xq.r_sel)
    rho_ref = oracle.rac_residual(qx.resid, qx.s_t, S_x)
    for j in range(kr):
        assert np.array_equal(codes[dst[:, j]], qx.codes)
        assert np.array_equal(sf[dst[:, j]], qx.sf)
        assert np.array_equal(rho[dst[:, j], :k], rho_ref)
    # gate/up + SwiGLU
    w13q = omoe.quantize_weights(w13n)
    h64, hb = omoe.gate_up(qx, rho_ref, S_x, idx, w13q, I)
    hg = oracle.bf16_to_f32(np_u16(layer.h))
    have = hg[dst.reshape(-1)]
    assert rel_fro(have, oracle.bf16_to_f32(hb)) <= TOL
    # end to end
    w2q = omoe.quantize_weights(w2n)
    out = omoe.down(hb, idx, gate, w2q, k)
    err = rel_fro(y, out["Y"])
    print(f"{name}: end-to-end relative Frobenius error {err:.2e}")
    assert err <= TOL


def test_moe_down_stage_from_synthetic_h(cuda):
    """The down projection on a seeded synthetic h (routed rows, padding rows
    zero), fed identically to both sides."""
    rng = np.random.default_rng(3)
    T, E, kr, H, I, k = 256, 8, 2, 1024, 768, 32
    logits = rng.standard_normal((T, E)).astype(np.float32)
    r = api.route(torch.from_numpy(logits).to(cuda), kr)
    torch.cuda.synchronize()
    off = r.offsets.cpu().numpy()
    tok = r.row_token.cpu().numpy()
    dst = r.dst_row.cpu().numpy()
    hrows = oracle.f32_to_bf16(rng.standard_normal((T * kr, I)).astype(np.float32) * 0.3)   # (t, j) order
    hpad = np.zeros((r.m_pad_max, I), np.uint16)
    hpad[dst.reshape(-1)] = hrows
    w2 = oracle.f32_to_bf16(rng.standard_normal((E, H, I)).astype(np.float32) * 0.02)
    _, s2, c2, sf2 = api.qdq_weights(to_bf16_dev(w2, cuda), want_qdq=False, want_packed=True)
    hd = to_bf16_dev(hpad, cuda)
    hq = api.quantize(hd, rac_k=k, rac_ld=64, m_valid=r.offsets[E:], m_out=r.m_pad_max)
    w_sel = api.gather_weight_channels(c2, sf2, H, I, hq.sel, k, 64)
    y = torch.zeros(T, H, dtype=torch.float32, device=cuda)
    api.grouped_gemm(hq.codes, hq.scales, hq.s_t, r.m_pad_max, c2, sf2, s2, H, I, E, r.offsets, rac_ld=64,
                     rho=hq.r_sel, w_sel=w_sel, epilogue=api.EPI_SCATTER_ADD_F32, row_token=r.row_token,
                     row_gate=r.row_gate, out=y)
    torch.cuda.synchronize()
    idx, gate = oracle.route(logits, kr)
    # quantization of the valid rows (padding rows are zero: they change nothing)
    valid = hpad[: off[E]]
    qh = oracle.quantize(valid)
    assert hq.s_t.item() == np.float32(qh.s_t)
    assert np.array_equal(hq.codes.cpu().numpy()[: off[E]], qh.codes)
    assert np.array_equal(unswizzle(hq.scales, off[E], I), qh.sf)
    score = oracle.channel_score(qh.resid)
    S_h = oracle.select_topk(score, k)
    check_selection(hq.sel.cpu().numpy(), score, S_h, k)
    out = omoe.down(hrows, idx, gate, omoe.quantize_weights(w2), k)
    assert np.array_equal(out["S_h"], S_h)
    assert rel_fro(y.cpu().numpy(), out["Y"]) <= TOL
    del tok


@pytest.mark.slow
@pytest.mark.parametrize("name,n_sample", [("moe_t4096_e128", 64), ("moe_t16384_e128", 16)])
def test_moe_large_sampled(cuda, name, n_sample):
    """Full-size layers in the bench's launch configuration: quantization
    statistics and X-side outputs checked in full; GEMM outputs on a sample
    of tokens."""
    cfg, x, logits, w13, w2, layer, y = _run_layer(cuda, name, 1)
    xn = _u16(x)
    T, kr, I, k = cfg.tokens, cfg.topk, cfg.inter, cfg.rac_k
    r = layer.routing
    idx, gate = oracle.route(logits.numpy(), kr)
    assert np.array_equal(r.topk_idx.cpu().numpy(), idx)
    qx = oracle.quantize(xn)
    score = oracle.channel_score(qx.resid)
    S_x = oracle.select_topk(score, k)
    assert layer.xq.s_t.item() == np.float32(qx.s_t)
    check_selection(layer.xq.sel.cpu().numpy(), score, S_x, k)
    np.testing.assert_allclose(layer.xq.score.cpu().numpy(), score, rtol=5.5e-7)
    rng = np.random.default_rng(17)
    toks = np.sort(rng.choice(T, n_sample, replace=False))
    dst = r.dst_row.cpu().numpy()
    codes = layer.xq.codes.cpu().numpy()
    rho = np_u16(layer.xq.r_sel)
    rho_ref = oracle.rac_residual(qx.resid[toks], qx.s_t, S_x)
    for j in range(kr):
        assert np.array_equal(codes[dst[toks, j]], qx.codes[toks])
        assert np.array_equal(rho[dst[toks, j], :k], rho_ref)
    # gate/up on the sampled tokens' routed rows, one expert at a time
    w13n = _u16(w13)
    hg = oracle.bf16_to_f32(np_u16(layer.h))
    want, have = [], []
    for e in np.unique(idx[toks]):
        wq = oracle.quantize(w13n[e]).xhat
        for i, t in enumerate(toks):
            for j in range(kr):
                if idx[t, j] != e:
                    continue
                y13 = oracle.w4a4_rac_matmul(qx.xhat[t:t + 1], qx.s_t, rho_ref[i][None], S_x, wq)
                want.append(oracle.bf16_to_f32(oracle.f32_to_bf16(oracle.swiglu(y13, I).astype(np.float32)))[0])
                have.append(hg[dst[t, j]])
        del wq
    assert rel_fro(np.stack(have), np.stack(want)) <= TOL
    del want, have


class _Xhat:
    """A quantized weight reduced to its dequantized values (all the layer
    oracle reads), to keep host memory small on the large layers."""

    def __init__(self, w_bits):
        self.xhat = oracle.quantize(w_bits).xhat


@pytest.mark.slow
@pytest.mark.parametrize("name", ["moe_t4096_e128", "moe_t16384_e128"])
def test_down_stage_full_size(cuda, name):
    """Down projection at full size (rollout-prefill and large layers) on a
    seeded synthetic h given to both sides: h quantization statistics in
    full, the codes of every routed row bit-exact, Y on sampled tokens."""
    cfg = wl.CONFIGS[name]
    T, E, kr, H, I, k = cfg.tokens, cfg.experts, cfg.topk, cfg.hidden, cfg.inter, cfg.rac_k
    logits = wl.router_logits(cfg, 2).numpy()
    r = api.route(torch.from_numpy(logits).to(cuda), kr, seg_align=256)
    torch.cuda.synchronize()
    dst = r.dst_row.cpu().numpy()
    g = torch.Generator().manual_seed(99)
    hrows = _u16((torch.randn(T * kr, I, generator=g) * 0.3).to(torch.bfloat16))
    hpad = np.zeros((r.m_pad_max, I), np.uint16)
    hpad[dst.reshape(-1)] = hrows
    _, w2 = wl.weights(cfg, 2)
    w2n = _u16(w2)
    _, s2, c2, sf2 = api.qdq_weights(w2.to(cuda), want_qdq=False, want_packed=True)
    del w2
    rac_ld = -(-k // 64) * 64
    hq = api.quantize(to_bf16_dev(hpad, cuda), rac_k=k, rac_ld=rac_ld, m_valid=r.offsets[E:], m_out=r.m_pad_max)
    w_sel = api.gather_weight_channels(c2, sf2, H, I, hq.sel, k, rac_ld)
    y = torch.zeros(T, H, dtype=torch.float32, device=cuda)
    api.grouped_gemm(hq.codes, hq.scales, hq.s_t, r.m_pad_max, c2, sf2, s2, H, I, E, r.offsets, seg_align=256,
                     rac_ld=rac_ld, rho=hq.r_sel, w_sel=w_sel, epilogue=api.EPI_SCATTER_ADD_F32,
                     row_token=r.row_token, row_gate=r.row_gate, out=y)
    torch.cuda.synchronize()
    idx, gate = oracle.route(logits, kr)
    qh = oracle.quantize(hrows)                 # (t, j) row order; statistics are order-free
    assert hq.s_t.item() == np.float32(qh.s_t)
    score = oracle.channel_score(qh.resid)
    S_h = oracle.select_topk(score, k)
    check_selection(hq.sel.cpu().numpy(), score, S_h, k)
    np.testing.assert_allclose(hq.score.cpu().numpy(), score, rtol=5.5e-7)
    rows = dst.reshape(-1)
    assert np.array_equal(hq.codes.cpu().numpy()[rows], qh.codes)
    assert np.array_equal(unswizzle(hq.scales, r.m_pad_max, I)[rows], qh.sf)
    rng = np.random.default_rng(5)
    toks = np.sort(rng.choice(T, 64, replace=False))
    rho = oracle.rac_residual(qh.resid, qh.s_t, S_h)
    want = np.zeros((len(toks), H))
    wq = {}
    for i, t in enumerate(toks):
        for j in range(kr):
            e = idx[t, j]
            if e not in wq:
                wq[e] = _Xhat(w2n[e])
            row = t * kr + j
            want[i] += gate[t, j] * oracle.w4a4_rac_matmul(qh.xhat[row:row + 1], qh.s_t, rho[row:row + 1], S_h,
                                                           wq[e].xhat)[0]
    assert rel_fro(y.cpu().numpy()[toks], want) <= TOL


@pytest.mark.slow
def test_moe_t4096_full_layer_x_to_y(cuda):
    """The rollout-prefill layer (T=4096, H=2048, I=768, E=128, top-8, k=64)
    end to end: the GPU's Y from X against the oracle's whole layer
    (its own routing, quantization, channel sets, h and down stage) at the
    2e-3 bar; X-side codes and scale bytes of every routed copy bit-exact."""
    cfg, x, logits, w13, w2, layer, y = _run_layer(cuda, "moe_t4096_e128", 1)
    xn, w13n, w2n = _u16(x), _u16(w13), _u16(w2)
    del w13, w2
    kr, k, E = cfg.topk, cfg.rac_k, cfg.experts
    r = layer.routing
    w13q = [_Xhat(w13n[e]) for e in range(E)]
    w2q = [_Xhat(w2n[e]) for e in range(E)]
    out = omoe.layer(xn, logits.numpy(), w13q, w2q, kr, k, k)
    assert np.array_equal(r.topk_idx.cpu().numpy(), out["idx"])
    dst = r.dst_row.cpu().numpy()
    codes = layer.xq.codes.cpu().numpy()
    sf = unswizzle(layer.xq.scales, layer.m_pad, cfg.hidden)
    for j in range(kr):
        assert np.array_equal(codes[dst[:, j]], out["xq"].codes)
        assert np.array_equal(sf[dst[:, j]], out["xq"].sf)
    assert np.array_equal(layer.xq.sel.cpu().numpy()[:k], out["S_x"])
    err = rel_fro(y, out["Y"])
    print(f"moe_t4096_e128: end-to-end relative Frobenius error {err:.2e}")
    assert err <= TOL


@pytest.mark.slow
def test_moe_t16384_x_to_y_sampled(cuda):
    """The large layer (T=16384, H=4096, I=1536, E=128, top-8 with skew,
    k=128) from X: X statistics in full and the routed copies' codes and
    scale bytes bit-exact on sampled tokens; the oracle computes h for every
    routed row, quantizes it as one tensor (its own s_h and S_h over all
    rows), and the GPU's Y on 256 sampled tokens matches its down stage at
    the 2e-3 bar."""
    cfg, x, logits, w13, w2, layer, y = _run_layer(cuda, "moe_t16384_e128", 1)
    xn, w13n, w2n = _u16(x), _u16(w13), _u16(w2)
    del w13, w2
    T, kr, I, k, E = cfg.tokens, cfg.topk, cfg.inter, cfg.rac_k, cfg.experts
    r = layer.routing
    idx, gate = oracle.route(logits.numpy(), kr)
    assert np.array_equal(r.topk_idx.cpu().numpy(), idx)
    qx = oracle.quantize(xn)
    score = oracle.channel_score(qx.resid)
    S_x = oracle.select_topk(score, k)
    assert layer.xq.s_t.item() == np.float32(qx.s_t)
    check_selection(layer.xq.sel.cpu().numpy(), score, S_x, k)
    rho_x = oracle.rac_residual(qx.resid, qx.s_t, S_x)
    rng = np.random.default_rng(29)
    toks = np.sort(rng.choice(T, 256, replace=False))
    dst = r.dst_row.cpu().numpy()
    codes = layer.xq.codes.cpu().numpy()
    sf = unswizzle(layer.xq.scales, layer.m_pad, cfg.hidden)
    for j in range(kr):
        assert np.array_equal(codes[dst[toks, j]], qx.codes[toks])
        assert np.array_equal(sf[dst[toks, j]], qx.sf[toks])
    # h for every routed row, (t, j) order, one expert at a time
    hb = np.empty((T * kr, I), np.uint16)
    flat = idx.reshape(-1)
    rows_t = np.repeat(np.arange(T), kr)
    for e in range(E):
        rows = np.nonzero(flat == e)[0]
        if rows.size == 0:
            continue
        y13 = oracle.w4a4_rac_matmul(qx.xhat[rows_t[rows]], qx.s_t, rho_x[rows_t[rows]], S_x,
                                     oracle.quantize(w13n[e]).xhat)
        hb[rows] = oracle.f32_to_bf16(oracle.swiglu(y13, I).astype(np.float32))
    del qx, rho_x
    qh = oracle.quantize(hb)
    s_h = oracle.channel_score(qh.resid)
    S_h = oracle.select_topk(s_h, k)
    assert abs(layer.hq.s_t.item() / qh.s_t - 1.0) <= 2.0 ** -7      # h agrees up to bf16 roundings
    overlap = len(set(layer.hq.sel.cpu().numpy()[:k].tolist()) & set(S_h.tolist()))
    print(f"moe_t16384_e128: S_h overlap {overlap}/{k}")
    rho_h = oracle.rac_residual(qh.resid, qh.s_t, S_h)
    want = np.zeros((len(toks), cfg.hidden))
    for e in np.unique(idx[toks]):
        wq = oracle.quantize(w2n[e]).xhat
        for i, t in enumerate(toks):
            for j in np.nonzero(idx[t] == e)[0]:
                row = t * kr + j
                want[i] += gate[t, j] * oracle.w4a4_rac_matmul(qh.xhat[row:row + 1], qh.s_t, rho_h[row:row + 1],
                                                               S_h, wq)[0]
    err = rel_fro(y[toks], want)
    print(f"moe_t16384_e128: sampled end-to-end relative Frobenius error {err:.2e}")
    assert err <= TOL


def test_moe_layer_rac_half_of_channels(cuda):
    """The pages' example of RAC on 50% of the channels (gist.science/it 2.2 B)
    on the small MoE layer: k = 1024 of H = 2048 channels for X and 384 of
    I = 768 for h, Y from X against the oracle's layer at the 2e-3 bar."""
    from quantization_nvfp4_quantize_b200.moe import rac_channels
    cfg = wl.CONFIGS["moe_t512_e8"]
    x = wl.activations(cfg, 4)
    logits = wl.router_logits(cfg, 4)
    w13, w2 = wl.weights(cfg, 4)
    kx, kh = rac_channels(50, cfg.hidden), rac_channels(50, cfg.inter)
    assert (kx, kh) == (1024, 384)
    layer = MoELayerW4A4(w13.to(cuda), w2.to(cuda), cfg.tokens, cfg.topk, kx, rac_k_h=kh)
    y = layer.forward(x.to(cuda), logits.to(cuda)).cpu().numpy()
    out = omoe.layer(_u16(x), logits.numpy(), omoe.quantize_weights(_u16(w13)), omoe.quantize_weights(_u16(w2)),
                     cfg.topk, kx, kh)
    check_selection(layer.xq.sel.cpu().numpy(), oracle.channel_score(out["xq"].resid), out["S_x"], kx)
    err = rel_fro(y, out["Y"])
    print(f"moe_t512_e8, RAC on 50% of channels: relative Frobenius error {err:.2e}")
    assert err <= TOL


def test_moe_layer_rac_second_pass(cuda):
    """The small MoE layer with the second-pass NVFP4 RAC variant end to end
    against the oracle's layer (rac_mode 'nvfp4') at the 2e-3 bar."""
    cfg = wl.CONFIGS["moe_t512_e8"]
    x = wl.activations(cfg, 8)
    logits = wl.router_logits(cfg, 8)
    w13, w2 = wl.weights(cfg, 8)
    layer = MoELayerW4A4(w13.to(cuda), w2.to(cuda), cfg.tokens, cfg.topk, cfg.rac_k, rac_mode="nvfp4")
    y = layer.forward(x.to(cuda), logits.to(cuda)).cpu().numpy()
    out = omoe.layer(_u16(x), logits.numpy(), omoe.quantize_weights(_u16(w13)), omoe.quantize_weights(_u16(w2)),
                     cfg.topk, cfg.rac_k, cfg.rac_k, rac_mode="nvfp4")
    dst = layer.routing.dst_row.cpu().numpy()
    rho = np_u16(layer.xq.r_sel)
    for j in range(cfg.topk):
        assert np.array_equal(rho[dst[:, j], :cfg.rac_k], out["rho_x"])
    err = rel_fro(y, out["Y"])
    print(f"moe_t512_e8, second-pass RAC: relative Frobenius error {err:.2e}")
    assert err <= TOL
