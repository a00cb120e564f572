"""GPU parity of the tcgen05 grouped W4A4 + RAC GEMM (through the C ABI)
against the oracle's binary64 products: relative Frobenius error <= 2e-3
(the expected error is ~1e-6: binary32 accumulation of exact products)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import np_u16, to_bf16_dev, rel_fro
from quantization_nvfp4_quantize_b200 import api
from quantization_nvfp4_quantize_b200.moe import DenseLayerW4A4

pytestmark = pytest.mark.gpu

TOL = 2e-3


def gen(rng, shape, scale=1.0):
    return oracle.f32_to_bf16(rng.standard_normal(shape).astype(np.float32) * scale)


def _setup(cuda, rng, T, E, kr, N, K, rac_k, align=128):
    x = gen(rng, (T, K))
    ch = rng.choice(K, 4, replace=False)
    xf = oracle.bf16_to_f32(x)
    xf[:, ch] *= 20
    x = oracle.f32_to_bf16(xf)
    w = gen(rng, (E, N, K), 0.02)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    r = api.route(torch.from_numpy(logits).to(cuda), kr, seg_align=align)
    rac_ld = -(-rac_k // 64) * 64 if rac_k else 0
    xq = api.quantize(to_bf16_dev(x, cuda), rac_k=rac_k, rac_ld=rac_ld, dst_rows=r.dst_row, fanout=kr,
                      m_out=r.m_pad_max)
    _, s_w, c_w, sf_w = api.qdq_weights(to_bf16_dev(w, cuda), want_qdq=False, want_packed=True)
    w_sel = None
    if rac_k:
        w_sel = api.gather_weight_channels(c_w, sf_w, N, K, xq.sel, rac_k, rac_ld)
    return x, w, logits, r, xq, s_w, c_w, sf_w, w_sel, rac_ld


def _oracle_rows(x, w, logits, kr, rac_k, sel):
    """Oracle y[t, j, :] for every (token, slot) with the GPU's channel set
    replaced by the oracle's own selection (checked equal first)."""
    idx, gate = oracle.route(logits, kr)
    qx = oracle.quantize(x)
    score = oracle.channel_score(qx.resid)
    S = oracle.select_topk(score, rac_k) if rac_k else np.zeros(0, np.int32)
    if rac_k:
        assert np.array_equal(np.asarray(sel)[:rac_k], S), "channel set differs"
    rho = oracle.rac_residual(qx.resid, qx.s_t, S) if rac_k else None
    wq = [oracle.quantize(w[e]) for e in range(w.shape[0])]
    T = x.shape[0]
    ys = {}
    for e in np.unique(idx):
        toks, slots = np.nonzero(idx == e)
        y = oracle.w4a4_rac_matmul(qx.xhat[toks], qx.s_t, None if rho is None else rho[toks], S, wq[e].xhat)
        for i, (t, j) in enumerate(zip(toks, slots)):
            ys[(t, j)] = y[i]
    return idx, gate, ys


@pytest.mark.parametrize("align", [128, 256])
@pytest.mark.parametrize("T,E,kr,N,K,rac_k", [
    (100, 1, 1, 256, 256, 0),
    (64, 1, 1, 256, 256, 8),
    (300, 3, 2, 512, 1024, 64),
    (700, 8, 2, 256, 2048, 32),
    (500, 5, 3, 768, 512, 200),
])
def test_gemm_store_f32(cuda, T, E, kr, N, K, rac_k, align):
    rng = np.random.default_rng(T + N + K + rac_k)
    x, w, logits, r, xq, s_w, c_w, sf_w, w_sel, rac_ld = _setup(cuda, rng, T, E, kr, N, K, rac_k, align)
    out = torch.full((r.m_pad_max, N), float("nan"), dtype=torch.float32, device=cuda)
    api.grouped_gemm(xq.codes, xq.scales, xq.s_t, r.m_pad_max, c_w, sf_w, s_w, N, K, E, r.offsets,
                     seg_align=align, rac_ld=rac_ld, rho=xq.r_sel, w_sel=w_sel, epilogue=api.EPI_STORE_F32,
                     row_token=r.row_token, row_gate=r.row_gate, out=out)
    torch.cuda.synchronize()
    sel = xq.sel.cpu().numpy() if rac_k else None
    idx, gate, ys = _oracle_rows(x, w, logits, kr, rac_k, sel)
    dst = r.dst_row.cpu().numpy()
    got = out.cpu().numpy()
    want = np.stack([ys[(t, j)] for t in range(T) for j in range(kr)])
    have = np.stack([got[dst[t, j]] for t in range(T) for j in range(kr)])
    assert np.all(np.isfinite(have))
    err = rel_fro(have, want)
    assert err <= TOL, err
    # padding rows are never written
    tok = r.row_token.cpu().numpy()
    pad = np.nonzero(tok < 0)[0]
    assert np.all(np.isnan(got[pad]))


@pytest.mark.parametrize("align", [128, 256])
def test_gemm_swiglu_and_scatter(cuda, align):
    rng = np.random.default_rng(11)
    T, E, kr, I, K, rac_k = 400, 6, 2, 256, 512, 32
    N = 2 * I
    x, w, logits, r, xq, s_w, c_w, sf_w, w_sel, rac_ld = _setup(cuda, rng, T, E, kr, N, K, rac_k, align)
    h = torch.full((r.m_pad_max, I), float("nan"), dtype=torch.bfloat16, device=cuda)
    h_amax = torch.full((1,), 123.0, dtype=torch.float32, device=cuda)
    api.grouped_gemm(xq.codes, xq.scales, xq.s_t, r.m_pad_max, c_w, sf_w, s_w, N, K, E, r.offsets,
                     seg_align=align, rac_ld=rac_ld, rho=xq.r_sel, w_sel=w_sel, epilogue=api.EPI_SWIGLU_BF16,
                     row_token=r.row_token, row_gate=r.row_gate, out=h, amax_out=h_amax)
    y = torch.zeros(T, N, dtype=torch.float32, device=cuda)
    api.grouped_gemm(xq.codes, xq.scales, xq.s_t, r.m_pad_max, c_w, sf_w, s_w, N, K, E, r.offsets,
                     seg_align=align, rac_ld=rac_ld, rho=xq.r_sel, w_sel=w_sel, epilogue=api.EPI_SCATTER_ADD_F32,
                     row_token=r.row_token, row_gate=r.row_gate, out=y)
    torch.cuda.synchronize()
    idx, gate, ys = _oracle_rows(x, w, logits, kr, rac_k, xq.sel.cpu().numpy())
    dst = r.dst_row.cpu().numpy()
    hg = oracle.bf16_to_f32(np_u16(h))
    want_h = np.stack([oracle.swiglu(ys[(t, j)][None], I)[0] for t in range(T) for j in range(kr)])
    have_h = np.stack([hg[dst[t, j]] for t in range(T) for j in range(kr)])
    assert rel_fro(have_h, want_h) <= TOL
    tok = r.row_token.cpu().numpy()
    off = r.offsets.cpu().numpy()
    pad = np.nonzero(tok[: off[-1]] < 0)[0]
    assert np.all(hg[pad] == 0), "padding rows of h must be zero"
    want_y = np.stack([sum(gate[t, j] * ys[(t, j)] for j in range(kr)) for t in range(T)])
    assert rel_fro(y.cpu().numpy(), want_y) <= TOL
    # the epilogue's max |h| is exactly the amax of the rows it wrote, and
    # quantizing h with it gives the same result as with the amax pass
    n_valid = int(off[-1])
    assert h_amax.item() == h[:n_valid].float().abs().max().item()
    mv = r.offsets[E:]
    q1 = api.quantize(h, rac_k=16, m_valid=mv, m_out=r.m_pad_max)
    q2 = api.quantize(h, rac_k=16, m_valid=mv, m_out=r.m_pad_max, amax=h_amax)
    torch.cuda.synchronize()
    assert q1.s_t.item() == q2.s_t.item()
    assert torch.equal(q1.codes[:n_valid], q2.codes[:n_valid]) and torch.equal(q1.sel, q2.sel)


def test_dense_layer_config(cuda):
    """Single dense layer: X [64 x 256] N(0,1) with 4 outlier channels x20,
    W [256 x 256] N(0, 0.02), k = 8, fp32 output."""
    from quantization_nvfp4_quantize_b200 import workloads as wl
    cfg = wl.CONFIGS["dense_64x256"]
    x = wl.activations(cfg, 0)
    w, _ = wl.weights(cfg, 0)
    layer = DenseLayerW4A4(w[0].to(cuda), cfg.tokens, cfg.rac_k)
    y = layer.forward(x.to(cuda)).cpu().numpy()
    xn = x.view(torch.int16).numpy().view(np.uint16)
    wn = w[0].view(torch.int16).numpy().view(np.uint16)
    qx = oracle.quantize(xn)
    S = oracle.select_topk(oracle.channel_score(qx.resid), cfg.rac_k)
    assert np.array_equal(layer.xq.sel.cpu().numpy()[: cfg.rac_k], S)
    rho = oracle.rac_residual(qx.resid, qx.s_t, S)
    want = oracle.w4a4_rac_matmul(qx.xhat, qx.s_t, rho, S, oracle.quantize(wn).xhat)
    assert rel_fro(y, want) <= TOL


@pytest.mark.parametrize("align", [128, 256])
def test_gemm_no_routed_rows(cuda, align):
    """T = 0: every expert segment is empty, the GEMMs write nothing (the
    scatter target keeps its contents, store rows stay untouched)."""
    rng = np.random.default_rng(17)
    E, N, K = 4, 256, 256
    logits = torch.empty(0, E, dtype=torch.float32, device=cuda)
    r = api.route(logits, 2, seg_align=align)
    assert r.offsets.cpu().numpy().tolist() == [0] * (E + 1)
    w = gen(rng, (E, N, K), 0.05)
    _, s_w, c_w, sf_w = api.qdq_weights(to_bf16_dev(w, cuda), want_qdq=False, want_packed=True)
    a_codes = torch.zeros(r.m_pad_max, K // 2, dtype=torch.uint8, device=cuda)
    a_scales = torch.zeros(api.scale_bytes(r.m_pad_max, K), dtype=torch.uint8, device=cuda)
    s_a = torch.ones(1, dtype=torch.float32, device=cuda)
    out = torch.full((r.m_pad_max, N), 7.0, dtype=torch.float32, device=cuda)
    api.grouped_gemm(a_codes, a_scales, s_a, r.m_pad_max, c_w, sf_w, s_w, N, K, E, r.offsets, seg_align=align,
                     epilogue=api.EPI_STORE_F32, row_token=r.row_token, row_gate=r.row_gate, out=out)
    y = torch.full((1, N), 3.0, dtype=torch.float32, device=cuda)
    api.grouped_gemm(a_codes, a_scales, s_a, r.m_pad_max, c_w, sf_w, s_w, N, K, E, r.offsets, seg_align=align,
                     epilogue=api.EPI_SCATTER_ADD_F32, row_token=r.row_token, row_gate=r.row_gate, out=y)
    a16 = torch.zeros(r.m_pad_max, K, dtype=torch.bfloat16, device=cuda)
    out16 = torch.full((r.m_pad_max, N), 5.0, dtype=torch.float32, device=cuda)
    api.bf16_grouped_gemm(a16, r.m_pad_max, to_bf16_dev(w, cuda), N, K, E, r.offsets, seg_align=align,
                          epilogue=api.EPI_STORE_F32, row_token=r.row_token, row_gate=r.row_gate, out=out16)
    torch.cuda.synchronize()
    assert torch.all(out == 7.0) and torch.all(y == 3.0) and torch.all(out16 == 5.0)


def test_bounded_wait_expiry_reports_timeout(cuda):
    """A device-side wait that runs out: the test hook withholds the
    accumulator-ready signal of a one-tile GEMM (1-SM shape) with every wait
    bounded by 20 ms.  The status word must read NVFP4_ERR_TIMEOUT, the call
    must return, and the same process must then run the normal GEMM on the
    same inputs to the oracle's result."""
    rng = np.random.default_rng(41)
    T, E, kr, N, K = 128, 1, 1, 256, 256
    x, w, logits, r, xq, s_w, c_w, sf_w, w_sel, rac_ld = _setup(cuda, rng, T, E, kr, N, K, 0)
    out = torch.zeros(r.m_pad_max, N, dtype=torch.float32, device=cuda)
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    lib = api._lib.load()
    api.check(lib.nvfp4_debug_gemm_wait_expiry(
        api._p(xq.codes), api._p(xq.scales), api._p(xq.s_t), r.m_pad_max, api._p(c_w), api._p(sf_w), api._p(s_w),
        N, K, E, api._p(r.offsets), api.EPI_STORE_F32, api._p(r.row_token), api._p(r.row_gate), api._p(out), N,
        api._p(status), 20_000_000, api._stream(cuda)))
    torch.cuda.synchronize()
    assert api.read_status(status) == 5, "expected NVFP4_ERR_TIMEOUT"
    # the context is intact: the normal call on the same inputs is exact
    status.zero_()
    api.grouped_gemm(xq.codes, xq.scales, xq.s_t, r.m_pad_max, c_w, sf_w, s_w, N, K, E, r.offsets,
                     epilogue=api.EPI_STORE_F32, row_token=r.row_token, row_gate=r.row_gate, out=out,
                     dev_status=status)
    torch.cuda.synchronize()
    assert api.read_status(status) == 0
    qx = oracle.quantize(x)
    want = qx.xhat.astype(np.float64) @ oracle.quantize(w[0]).xhat.astype(np.float64).T
    tok = r.row_token.cpu().numpy()[: r.m_pad_max]
    got = out.cpu().numpy()
    rows = np.nonzero(tok >= 0)[0]
    assert rel_fro(got[rows], want[tok[rows]]) <= TOL
