"""GPU parity of the BF16 grouped GEMM (the trainer-side W4A16 path,
gist.science/it 2.2 A) and of the bf16 routed-row gather, through the C ABI,
against the oracle's binary64 products: relative Frobenius error <= 2e-3
(expected ~1e-6: binary32 accumulation of exact bf16 products)."""
import numpy as np
import pytest
import torch

import oracle
import oracle.moe as omoe
from gpu_util import np_u16, to_bf16_dev, rel_fro
from quantization_nvfp4_quantize_b200 import api
from quantization_nvfp4_quantize_b200.moe import MoELayerW4A16

pytestmark = pytest.mark.gpu

TOL = 2e-3


def gen(rng, shape, scale=1.0):
    return oracle.f32_to_bf16(rng.standard_normal(shape).astype(np.float32) * scale)


def _route(cuda, rng, T, E, kr, align):
    logits = rng.standard_normal((T, E)).astype(np.float32)
    r = api.route(torch.from_numpy(logits).to(cuda), kr, seg_align=align)
    return logits, r


def test_gather_rows_is_exact(cuda):
    rng = np.random.default_rng(3)
    T, K, E, kr = 300, 200, 5, 3
    x = gen(rng, (T, K))
    logits, r = _route(cuda, rng, T, E, kr, 128)
    out = api.gather_rows_bf16(to_bf16_dev(x, cuda), r.dst_row, r.m_pad_max)
    got = np_u16(out)
    dst = r.dst_row.cpu().numpy()
    for t in range(T):
        for j in range(kr):
            assert np.array_equal(got[dst[t, j]], x[t])
    tok = r.row_token.cpu().numpy()
    assert np.all(got[np.nonzero(tok < 0)[0]] == 0)     # untouched rows keep their (zero) contents


@pytest.mark.parametrize("align", [128, 256])
@pytest.mark.parametrize("T,E,kr,N,K", [
    (100, 1, 1, 256, 64),
    (300, 3, 2, 512, 320),
    (700, 8, 2, 256, 1024),
])
def test_bf16_gemm_store_f32(cuda, T, E, kr, N, K, align):
    rng = np.random.default_rng(T + N + K)
    x = gen(rng, (T, K))
    w = gen(rng, (E, N, K), 0.05)
    logits, r = _route(cuda, rng, T, E, kr, align)
    a = api.gather_rows_bf16(to_bf16_dev(x, cuda), r.dst_row, r.m_pad_max)
    out = torch.full((r.m_pad_max, N), float("nan"), dtype=torch.float32, device=cuda)
    api.bf16_grouped_gemm(a, r.m_pad_max, to_bf16_dev(w, cuda), N, K, E, r.offsets, seg_align=align,
                          epilogue=api.EPI_STORE_F32, row_token=r.row_token, row_gate=r.row_gate, out=out)
    torch.cuda.synchronize()
    idx, _ = oracle.route(logits, kr)
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    wf = oracle.bf16_to_f32(w).astype(np.float64)
    dst = r.dst_row.cpu().numpy()
    got = out.cpu().numpy()
    want = np.stack([xf[t] @ wf[idx[t, j]].T for t in range(T) for j in range(kr)])
    have = np.stack([got[dst[t, j]] for t in range(T) for j in range(kr)])
    assert np.all(np.isfinite(have))
    assert rel_fro(have, want) <= TOL
    pad = np.nonzero(r.row_token.cpu().numpy() < 0)[0]
    assert np.all(np.isnan(got[pad]))


@pytest.mark.parametrize("align", [128, 256])
def test_w4a16_layer_small(cuda, align):
    """A whole W4A16 layer (T=300, H=256, I=256, E=6, top-2) against the oracle."""
    rng = np.random.default_rng(5)
    T, H, I, E, kr = 300, 256, 256, 6, 2
    x = gen(rng, (T, H))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    w13 = gen(rng, (E, 2 * I, H), 0.05)
    w2 = gen(rng, (E, H, I), 0.05)
    layer = MoELayerW4A16(to_bf16_dev(w13, cuda), to_bf16_dev(w2, cuda), T, kr, seg_align=align)
    y = layer.forward(to_bf16_dev(x, cuda), torch.from_numpy(logits).to(cuda)).cpu().numpy()
    want = omoe.layer_w4a16(x, logits, w13, w2, kr)
    assert rel_fro(y, want["Y"]) <= TOL
    # h rows against the oracle's bf16 h, and padding rows of h are zero
    hg = oracle.bf16_to_f32(np_u16(layer.h))
    dst = layer.routing.dst_row.cpu().numpy()
    have_h = np.stack([hg[dst[t, j]] for t in range(T) for j in range(kr)])
    assert rel_fro(have_h, oracle.bf16_to_f32(want["h_bf16"])) <= TOL
    off = layer.routing.offsets.cpu().numpy()
    tok = layer.routing.row_token.cpu().numpy()
    assert np.all(hg[np.nonzero(tok[: off[-1]] < 0)[0]] == 0)


def test_w4a16_layer_config_sampled(cuda):
    """qat_w4a16_e128 (T=4096, H=2048, I=768, E=128, top-8) on the GPU; the
    oracle evaluates a seeded sample of 48 tokens (rows are independent)."""
    from quantization_nvfp4_quantize_b200 import workloads as wl
    cfg = wl.CONFIGS["qat_w4a16_e128"]
    x = wl.activations(cfg, 0)
    logits = wl.router_logits(cfg, 0)
    w13, w2 = wl.weights(cfg, 0)
    layer = MoELayerW4A16(w13.to(cuda), w2.to(cuda), cfg.tokens, cfg.topk)
    y = layer.forward(x.to(cuda), logits.to(cuda)).cpu().numpy()
    toks = np.sort(np.random.default_rng(9).choice(cfg.tokens, 48, replace=False))
    xn = x.view(torch.int16).numpy().view(np.uint16)
    w13n = w13.view(torch.int16).numpy().view(np.uint16)
    w2n = w2.view(torch.int16).numpy().view(np.uint16)
    want = omoe.layer_w4a16(xn[toks], logits.numpy()[toks], w13n, w2n, cfg.topk)
    assert rel_fro(y[toks], want["Y"]) <= TOL
