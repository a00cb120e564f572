"""GPU parity of per-expert RAC channel sets (nvfp4_quantize_experts, the
per-expert weight-channel gather and the complete routed copy of X) against
the oracle's per-expert reading (oracle.moe.expert_rac / layer with
rac_scope="expert"; the pages' binary channel mask, gist.science/it 2.2 B,
chosen per expert GEMM input):

  * routed copy: bit-exact, padding rows zero whatever the buffer held;
  * codes, scale bytes, s_t and rho: bit-exact; each expert's set: bit-exact
    outside the 1e-6 tie window of its own scores;
  * the gathered weight channels of every expert: bit-exact;
  * the whole layer from X to Y: within 2e-3 of the oracle's layer."""
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


@pytest.mark.parametrize("seg_align", [128, 256])
def test_routed_rows_copy_is_complete(cuda, seg_align):
    rng = np.random.default_rng(seg_align)
    T, K, E, kr = 300, 192, 6, 2
    x = oracle.f32_to_bf16(rng.standard_normal((T, K)).astype(np.float32))
    logits = torch.from_numpy(rng.standard_normal((T, E)).astype(np.float32)).to(cuda)
    r = api.route(logits, kr, seg_align=seg_align)
    out = torch.full((r.m_pad_max, K), 7.0, dtype=torch.bfloat16, device=cuda)      # stale rows
    api.routed_rows_bf16(to_bf16_dev(x, cuda), r.row_token, r.m_pad_max, out=out)
    got = np_u16(out)
    tok = r.row_token.cpu().numpy()
    for i in range(r.m_pad_max):
        want = x[tok[i]] if tok[i] >= 0 else np.zeros(K, np.uint16)
        assert np.array_equal(got[i], want), i


@pytest.mark.parametrize("E,kr,K,k,seg_align", [(8, 2, 256, 8, 128), (16, 4, 768, 64, 256), (5, 1, 2048, 512, 128)])
def test_quantize_experts_parity(cuda, E, kr, K, k, seg_align):
    rng = np.random.default_rng(E * 1000 + K)
    T = 700
    xf = rng.standard_normal((T, K)).astype(np.float32)
    xf[:, rng.choice(K, 3, replace=False)] *= 25.0
    x = oracle.f32_to_bf16(xf)
    logits_np = rng.standard_normal((T, E)).astype(np.float32)
    r = api.route(torch.from_numpy(logits_np).to(cuda), kr, seg_align=seg_align)
    xr = api.routed_rows_bf16(to_bf16_dev(x, cuda), r.row_token, r.m_pad_max)
    q = api.quantize_experts(xr, r.offsets, E, seg_align, rac_k=k, want_score=True)
    torch.cuda.synchronize()
    offs = r.offsets.cpu().numpy()
    tok = r.row_token.cpu().numpy()
    M = int(offs[E])
    # oracle on the same routed rows (padding rows are zero rows)
    xr_np = np_u16(xr)[:M]
    oq = oracle.quantize(xr_np)
    assert q.s_t.item() == np.float32(oq.s_t)
    assert np.array_equal(q.codes.cpu().numpy()[:M], oq.codes)
    assert np.array_equal(unswizzle(q.scales, r.m_pad_max, K)[:M], oq.sf)
    rho = np_u16(q.r_sel)
    sel = q.sel.cpu().numpy()
    for e in range(E):
        rows = np.arange(offs[e], offs[e + 1])
        valid = rows[tok[rows] >= 0]
        score = oracle.channel_score(oq.resid[valid])
        S = oracle.select_topk(score, k)
        check_selection(sel[e], score, S, k)
        np.testing.assert_allclose(q.score[e].cpu().numpy(), score, rtol=6e-7, atol=0)
        want = oracle.rac_residual(oq.resid[rows], oq.s_t, sel[e][:k])
        assert np.array_equal(rho[rows][:, :k], want)
        assert not rho[rows][:, k:].any()


def test_gather_channels_per_expert(cuda):
    rng = np.random.default_rng(5)
    E, N, K, k, ld = 3, 256, 512, 40, 64
    w = oracle.f32_to_bf16((rng.standard_normal((E, N, K)) * 0.02).astype(np.float32))
    _, s_w, c_w, sf_w = api.qdq_weights(to_bf16_dev(w, cuda), want_qdq=False, want_packed=True)
    ccm, scm = api.weights_channel_major(c_w, sf_w, N, K)
    sel = np.stack([np.sort(rng.choice(K, k, replace=False)) for _ in range(E)]).astype(np.int32)
    out = api.gather_weight_channels_cm_experts(ccm, scm, N, K, torch.from_numpy(sel).to(cuda), k, ld)
    got = np_u16(out)
    for e in range(E):
        wq = oracle.quantize(w[e])
        lo = wq.codes & 0xF
        hi = wq.codes >> 4
        q = np.empty((N, K), np.float64)
        q[:, 0::2] = oracle.e2m1_decode(lo)
        q[:, 1::2] = oracle.e2m1_decode(hi)
        sf = np.repeat(oracle.e4m3_decode(wq.sf).astype(np.float64), 16, axis=1)
        want = oracle.f32_to_bf16((q * sf)[:, sel[e]].astype(np.float32))  # e2m1 * sf, exact in bf16
        assert np.array_equal(got[e][:, :k], want)
        assert not got[e][:, k:].any()


@pytest.mark.parametrize("name", ["moe_t512_e8", "moe_t4096_e128"])
def test_moe_layer_per_expert_sets(cuda, name):
    cfg = wl.CONFIGS[name]
    x = wl.activations(cfg, 6)
    logits = wl.router_logits(cfg, 6)
    w13, w2 = wl.weights(cfg, 6)
    layer = MoELayerW4A4(w13.to(cuda), w2.to(cuda), cfg.tokens, cfg.topk, cfg.rac_k, rac_scope="expert")
    y = layer.forward(x.to(cuda), logits.to(cuda)).cpu().numpy()
    out = omoe.layer(_u16(x), logits.numpy(), omoe.quantize_weights(_u16(w13)), omoe.quantize_weights(_u16(w2)),
                     cfg.topk, cfg.rac_k, cfg.rac_k, rac_scope="expert")
    sel = layer.xq.sel.cpu().numpy()
    rows_t = np.repeat(np.arange(cfg.tokens), cfg.topk)
    flat = out["idx"].reshape(-1)
    for e, S_e in out["S_x"].items():
        toks = rows_t[np.nonzero(flat == e)[0]]
        check_selection(sel[e], oracle.channel_score(out["xq"].resid[toks]), S_e, cfg.rac_k)
    err = rel_fro(y, out["Y"])
    print(f"{name}, per-expert RAC sets: relative Frobenius error {err:.2e}")
    assert err <= TOL
