"""GPU parity of the bandwidth kernels (through the C ABI) against the oracle:
encoders, quantize + scores + selection + RAC residual, weight QDQ, routing,
weight channel gather.  Codes, scale bytes, tensor scales, selected channel
sets (outside the 1e-6 tie window), RAC residuals and QDQ values are
bit-exact; scores agree to 5.5e-7 relative (binary32 partial sums of at most
4 rows, binary64 above)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import np_u16, to_bf16_dev, check_selection, unswizzle
from quantization_nvfp4_quantize_b200 import api

pytestmark = pytest.mark.gpu

SCORE_RTOL = 5.5e-7


def gen_x(rng, M, K, outliers=4, scale=1.0):
    x = rng.standard_normal((M, K)).astype(np.float32) * scale
    if outliers and K:
        ch = rng.choice(K, size=min(outliers, K), replace=False)
        x[:, ch] *= np.exp(2.0 + 0.5 * rng.standard_normal(len(ch))).astype(np.float32)
    return oracle.f32_to_bf16(x)


def test_hw_encoders_match_oracle(cuda):
    h = np.arange(65536, dtype=np.uint32)
    f = (h << 16).view(np.float32)
    f = f[np.isfinite(f)]
    rng = np.random.default_rng(0)
    grid = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    mids = np.concatenate([grid, np.nextafter(grid, np.float32(0)), np.nextafter(grid, np.float32(9))])
    r = rng.uniform(-8, 8, 1_000_000).astype(np.float32)
    vals = np.concatenate([f, mids, -mids, r]).astype(np.float32)
    e2, _ = api.debug_encode(torch.from_numpy(vals).to(cuda))
    ref2 = oracle.e2m1_encode(vals)
    bad = np.nonzero(e2.cpu().numpy() != ref2)[0]
    assert bad.size == 0, f"E2M1 mismatch at {vals[bad[:8]]}: gpu {e2.cpu().numpy()[bad[:8]]} oracle {ref2[bad[:8]]}"
    # E4M3 on non-negative inputs: all midpoints +-1 ulp, codes, random
    table = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    m = ((table[:-1] + table[1:]) / 2).astype(np.float32)
    pos = np.concatenate([m, np.nextafter(m, np.float32(1e9)), np.nextafter(m, np.float32(0)),
                          table.astype(np.float32), np.array([448, 464, 465, 1e6, 0, 2.0 ** -10], np.float32),
                          np.exp(rng.uniform(np.log(1e-5), np.log(600), 1_000_000)).astype(np.float32),
                          np.abs(f[np.abs(f) < 1e6])]).astype(np.float32)
    _, e4 = api.debug_encode(torch.from_numpy(pos).to(cuda))
    ref4 = oracle.e4m3_encode(pos)
    bad = np.nonzero(e4.cpu().numpy() != ref4)[0]
    assert bad.size == 0, f"E4M3 mismatch at {pos[bad[:8]]}"


def _quant_parity(cuda, x, rac_k, rtol=SCORE_RTOL):
    M, K = x.shape
    xd = to_bf16_dev(x, cuda)
    q = api.quantize(xd, rac_k=rac_k, want_score=True)
    torch.cuda.synchronize()
    ref = oracle.quantize(x)
    assert q.s_t.item() == np.float32(ref.s_t)
    assert np.array_equal(q.codes.cpu().numpy(), ref.codes)
    assert np.array_equal(unswizzle(q.scales, M, K), ref.sf)
    score = oracle.channel_score(ref.resid)
    np.testing.assert_allclose(q.score.cpu().numpy(), score, rtol=rtol, atol=0)
    if rac_k:
        S = oracle.select_topk(score, rac_k)
        sel = q.sel.cpu().numpy()[:rac_k]
        check_selection(sel, score, S, rac_k)
        rho_ref = oracle.rac_residual(ref.resid, ref.s_t, sel)
        rsel = np_u16(q.r_sel)
        assert np.array_equal(rsel[:, :rac_k], rho_ref)
        assert np.all(rsel[:, rac_k:] == 0)
    return q, ref


@pytest.mark.parametrize("M,K,k", [(64, 256, 8), (1, 64, 1), (300, 768, 32), (129, 1536, 64),
                                   (1000, 2048, 64), (257, 4096, 128), (64, 320, 5), (40, 16384, 256)])
def test_quantize_parity(cuda, M, K, k):
    rng = np.random.default_rng(M * 31 + K)
    _quant_parity(cuda, gen_x(rng, M, K), k)


def test_quantize_zero_and_tiny(cuda):
    x = np.zeros((130, 256), np.uint16)
    q, ref = _quant_parity(cuda, x, 8)
    assert q.s_t.item() == 1.0
    rng = np.random.default_rng(5)
    y = gen_x(rng, 70, 128, scale=1e-3)
    y[:, 16:48] = 0
    y[3, 5] = 0x8000          # -0
    _quant_parity(cuda, y, 16)


def test_quantize_reciprocal_overflow(cuda):
    """A tensor scale and block scales below 2^-128, whose reciprocals overflow
    binary32: every decision there must come from the division.  Codes, scale
    bytes, s_t and rho are bit-exact; scores are not compared (their binary32
    partial sums of R^2 underflow at this magnitude)."""
    rng = np.random.default_rng(11)
    x = gen_x(rng, 200, 512, scale=1e-37)
    x[:, 32:40] = 0
    x[5, :] = 0
    x[:, 64:96] = gen_x(rng, 200, 32, outliers=0, scale=1e-39)
    x[::3, 64:72] = 0
    ref = oracle.quantize(x)
    d = oracle.e4m3_decode(ref.sf.astype(np.uint8)).astype(np.float32) * np.float32(ref.s_t)
    assert np.float32(ref.s_t) < 2.0 ** -128 and np.sum((d > 0) & (d < 2.0 ** -128)) > 0
    k = 24
    q = api.quantize(to_bf16_dev(x, cuda), rac_k=k, want_score=True)
    torch.cuda.synchronize()
    assert q.s_t.item() == np.float32(ref.s_t)
    assert np.array_equal(q.codes.cpu().numpy(), ref.codes)
    assert np.array_equal(unswizzle(q.scales, 200, 512), ref.sf)
    sel = q.sel.cpu().numpy()[:k]
    assert len(set(sel.tolist())) == k and sel.min() >= 0 and sel.max() < 512
    assert np.array_equal(np_u16(q.r_sel)[:, :k], oracle.rac_residual(ref.resid, ref.s_t, sel))


def test_quantize_empty(cuda):
    x = torch.empty(0, 256, dtype=torch.bfloat16, device=cuda)
    q = api.quantize(x, rac_k=0, m_out=0, want_score=True)
    torch.cuda.synchronize()
    assert q.s_t.item() == 1.0 and np.all(q.score.cpu().numpy() == 0)


@pytest.mark.parametrize("k", [16, 48])
def test_quantize_fanout_and_valid_rows(cuda, k):
    """dst_rows fan-out writes every copy; m_valid limits the rows read.  With
    k = 16 the selection touches few of a row's 32 blocks (residuals from the
    selected blocks only); with k = 48 rows are streamed whole."""
    rng = np.random.default_rng(6)
    M, K, F = 200, 512, 3
    x = gen_x(rng, M, K)
    perm = rng.permutation(M * F + 100)[: M * F].astype(np.int32).reshape(M, F)
    perm[7, 1] = -1
    m_out = -(-(M * F + 100) // 128) * 128
    xd = to_bf16_dev(x, cuda)
    q = api.quantize(xd, rac_k=k, dst_rows=torch.from_numpy(perm).to(cuda), fanout=F, m_out=m_out)
    torch.cuda.synchronize()
    ref = oracle.quantize(x)
    codes = q.codes.cpu().numpy()
    sf = unswizzle(q.scales, m_out, K)
    rsel = np_u16(q.r_sel)
    score = oracle.channel_score(ref.resid)
    sel = q.sel.cpu().numpy()[:k]
    check_selection(sel, score, oracle.select_topk(score, k), k)
    rho = oracle.rac_residual(ref.resid, ref.s_t, sel)
    for r in range(M):
        for j in range(F):
            d = perm[r, j]
            if d < 0:
                continue
            assert np.array_equal(codes[d], ref.codes[r])
            assert np.array_equal(sf[d], ref.sf[r])
            assert np.array_equal(rsel[d, :k], rho[r])
    # m_valid: only the first 77 rows count
    mv = torch.tensor([77], dtype=torch.int32, device=cuda)
    q2 = api.quantize(xd, rac_k=k, m_valid=mv, want_score=True)
    torch.cuda.synchronize()
    ref2 = oracle.quantize(x[:77])
    assert q2.s_t.item() == np.float32(ref2.s_t)
    assert np.array_equal(q2.codes.cpu().numpy()[:77], ref2.codes)
    np.testing.assert_allclose(q2.score.cpu().numpy(), oracle.channel_score(ref2.resid), rtol=SCORE_RTOL)


def test_fanout_residual_pieces_and_windows(cuda):
    """Residuals streamed in two row pieces (K = 4096) and two column windows
    (ld = 1152), written to three routed rows each, some of them skipped."""
    rng = np.random.default_rng(12)
    M, K, F, k = 96, 4096, 3, 1100
    x = gen_x(rng, M, K, outliers=40)
    perm = rng.permutation(M * F + 50)[: M * F].astype(np.int32).reshape(M, F)
    perm[4, 2] = -1
    perm[9, 0] = M * F + 10_000          # beyond m_out: skipped
    m_out = M * F + 50
    q = api.quantize(to_bf16_dev(x, cuda), rac_k=k, rac_ld=1152, dst_rows=torch.from_numpy(perm).to(cuda),
                     fanout=F, m_out=m_out)
    torch.cuda.synchronize()
    ref = oracle.quantize(x)
    sel = q.sel.cpu().numpy()[:k]
    score = oracle.channel_score(ref.resid)
    check_selection(sel, score, oracle.select_topk(score, k), k)
    rho = oracle.rac_residual(ref.resid, ref.s_t, sel)
    rsel = np_u16(q.r_sel)
    for r in range(M):
        for j in range(F):
            d = perm[r, j]
            if 0 <= d < m_out:
                assert np.array_equal(rsel[d, :k], rho[r]), (r, j)
                assert np.all(rsel[d, k:] == 0)


def test_select_ties(cuda):
    """Equal channel scores: lower channel index first (all-equal columns)."""
    x = np.tile(gen_x(np.random.default_rng(7), 1, 64), (50, 4))     # K = 256, repeated column groups
    q, ref = _quant_parity(cuda, x, 10)


@pytest.mark.parametrize("G,rows,cols", [(3, 256, 512), (2, 200, 64), (5, 1536, 2048)])
def test_qdq_weights_parity(cuda, G, rows, cols):
    rng = np.random.default_rng(G * rows + cols)
    w = oracle.f32_to_bf16(rng.standard_normal((G, rows, cols)).astype(np.float32) * 0.02)
    wd = to_bf16_dev(w, cuda)
    wq, s_t, codes, scales = api.qdq_weights(wd, want_qdq=True, want_packed=True)
    torch.cuda.synchronize()
    wq = np_u16(wq)
    for g in range(G):
        ref_bf16, ref_s, ref = oracle.qdq(w[g])
        assert s_t[g].item() == np.float32(ref_s)
        assert np.array_equal(wq[g], ref_bf16)
        assert np.array_equal(codes[g].cpu().numpy(), ref.codes)
        assert np.array_equal(unswizzle(scales[g], rows, cols), ref.sf)


@pytest.mark.parametrize("T,E,kr,align", [(512, 8, 2, 128), (1000, 128, 8, 128), (64, 1, 1, 128), (3, 16, 4, 128),
                                          (4096, 256, 8, 128), (1000, 128, 8, 256), (700, 8, 2, 256),
                                          (0, 8, 2, 256), (33, 3, 3, 256), (16384, 128, 8, 256)])
def test_route_parity(cuda, T, E, kr, align):
    rng = np.random.default_rng(T + E)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    if E > 4 and T > 0:
        logits[0, [1, 3]] = 5.0      # tie
    r = api.route(torch.from_numpy(logits).to(cuda), kr, seg_align=align)
    torch.cuda.synchronize()
    idx, gate = oracle.route(logits, kr)
    assert np.array_equal(r.topk_idx.cpu().numpy(), idx)
    np.testing.assert_allclose(r.topk_gate.cpu().numpy(), gate, rtol=2e-6, atol=1e-7)
    off = r.offsets.cpu().numpy()
    counts = np.bincount(idx.reshape(-1), minlength=E)
    padded = -(-counts // align) * align
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(padded)]))
    dst = r.dst_row.cpu().numpy()
    tok = r.row_token.cpu().numpy()
    rg = r.row_gate.cpu().numpy()
    for e in range(E):
        seg = tok[off[e]:off[e + 1]]
        toks = np.nonzero((idx == e).any(axis=1))[0]
        assert np.array_equal(seg[: counts[e]], toks)            # ascending tokens
        assert np.all(seg[counts[e]:] == -1)
        assert np.all(rg[off[e] + counts[e]:off[e + 1]] == 0)   # padding rows carry no gate
    assert np.all(tok[off[E]:] == -1)
    if T:
        tt = np.repeat(np.arange(T), kr)
        d = dst.reshape(-1)
        e = idx.reshape(-1)
        assert np.array_equal(tok[d], tt)
        assert np.all((off[e] <= d) & (d < off[e + 1]))
        assert np.array_equal(rg[d], r.topk_gate.cpu().numpy().reshape(-1))
        assert len(np.unique(d)) == T * kr


def test_gather_weight_channels(cuda):
    rng = np.random.default_rng(8)
    E, N, K = 3, 256, 512
    w = oracle.f32_to_bf16(rng.standard_normal((E, N, K)).astype(np.float32) * 0.02)
    _, s_t, codes, scales = api.qdq_weights(to_bf16_dev(w, cuda), want_qdq=False, want_packed=True)
    sel = np.sort(rng.choice(K, 40, replace=False)).astype(np.int32)
    out = api.gather_weight_channels(codes, scales, N, K, torch.from_numpy(sel).to(cuda), 40, 64)
    torch.cuda.synchronize()
    got = np_u16(out)
    for e in range(E):
        ref = oracle.quantize(w[e])
        q = np.empty((N, K), np.uint8)
        q[:, 0::2] = ref.codes & 0xF
        q[:, 1::2] = ref.codes >> 4
        vals = oracle.e2m1_decode(q) * np.repeat(oracle.e4m3_decode(ref.sf), 16, axis=1)
        want = oracle.f32_to_bf16(vals[:, sel].astype(np.float32))
        assert np.array_equal(got[e, :, :40], want)
        assert np.all(got[e, :, 40:] == 0)


@pytest.mark.parametrize("E,N,K,k,ld", [(3, 256, 512, 40, 64), (2, 1536, 768, 128, 128), (4, 128, 2048, 256, 256)])
def test_channel_major_copy_and_gather(cuda, E, N, K, k, ld):
    """The channel-major weight copy holds the same codes/scales, and the
    gather from it equals the gather from the K-major weight and the oracle."""
    rng = np.random.default_rng(E * N + K)
    w = oracle.f32_to_bf16(rng.standard_normal((E, N, K)).astype(np.float32) * 0.02)
    _, s_t, codes, scales = api.qdq_weights(to_bf16_dev(w, cuda), want_qdq=False, want_packed=True)
    ccm, scm = api.weights_channel_major(codes, scales, N, K)
    sel = np.sort(rng.choice(K, k, replace=False)).astype(np.int32)
    seld = torch.from_numpy(sel).to(cuda)
    a = api.gather_weight_channels(codes, scales, N, K, seld, k, ld)
    b = api.gather_weight_channels_cm(ccm, scm, N, K, seld, k, ld)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    ccm_n, scm_n = ccm.cpu().numpy(), scm.cpu().numpy()
    for e in range(E):
        ref = oracle.quantize(w[e])
        q = np.empty((N, K), np.uint8)
        q[:, 0::2] = ref.codes & 0xF
        q[:, 1::2] = ref.codes >> 4
        assert np.array_equal(ccm_n[e] & 0xF, q[0::2].T)
        assert np.array_equal(ccm_n[e] >> 4, q[1::2].T)
        assert np.array_equal(scm_n[e], ref.sf.T)
        vals = oracle.e2m1_decode(q) * np.repeat(oracle.e4m3_decode(ref.sf), 16, axis=1)
        want = oracle.f32_to_bf16(vals[:, sel].astype(np.float32))
        assert np.array_equal(np_u16(b)[e, :, :k], want)


def test_gather_out_of_range_channels_give_zero_columns(cuda):
    """Channel indices outside [0, K) give zero columns in both weight
    gathers; the valid columns are unchanged."""
    rng = np.random.default_rng(19)
    E, N, K, k, ld = 2, 128, 256, 6, 64
    w = oracle.f32_to_bf16(rng.standard_normal((E, N, K)).astype(np.float32) * 0.02)
    _, s_t, codes, scales = api.qdq_weights(to_bf16_dev(w, cuda), want_qdq=False, want_packed=True)
    codes_cm, scales_cm = api.weights_channel_major(codes, scales, N, K)
    sel = np.array([3, K, 17, -1, 100, 1 << 20], np.int32)
    sel_d = torch.from_numpy(sel).to(cuda)
    a = np_u16(api.gather_weight_channels(codes, scales, N, K, sel_d, k, ld))
    b = np_u16(api.gather_weight_channels_cm(codes_cm, scales_cm, N, K, sel_d, k, ld))
    assert np.array_equal(a, b)
    bad = [1, 3, 5]
    assert np.all(a[:, :, bad] == 0) and np.all(a[:, :, k:] == 0)
    good = np.array([3, 17, 100], np.int32)
    ref = np_u16(api.gather_weight_channels(codes, scales, N, K, torch.from_numpy(good).to(cuda), 3, ld))
    assert np.array_equal(a[:, :, [0, 2, 4]], ref[:, :, :3])


def test_fanout_skips_rows_beyond_m_out(cuda):
    """Destination rows >= M_out are skipped like negative ones: the outputs'
    guard rows past M_out keep their contents, the valid copies are exact."""
    rng = np.random.default_rng(23)
    M, K, F, m_out, guard = 64, 256, 2, 256, 128
    x = gen_x(rng, M, K)
    dst = np.stack([np.arange(M), M + np.arange(M)], axis=1).astype(np.int32)
    dst[3, 0] = m_out                        # first guard row
    dst[9, 1] = m_out + 77                   # deep inside the guard
    out = api.Quantized(
        codes=torch.full((m_out + guard, K // 2), 0xAB, dtype=torch.uint8, device=cuda),
        scales=torch.full((api.scale_bytes(m_out + guard, K),), 0xAB, dtype=torch.uint8, device=cuda),
        s_t=torch.empty(1, dtype=torch.float32, device=cuda),
        score=torch.empty(K, dtype=torch.float64, device=cuda),
        sel=torch.empty(16, dtype=torch.int32, device=cuda),
        r_sel=torch.full((m_out + guard, 64), 7.0, dtype=torch.bfloat16, device=cuda))
    api.quantize(to_bf16_dev(x, cuda), rac_k=16, dst_rows=torch.from_numpy(dst).to(cuda), fanout=F, m_out=m_out,
                 out=out)
    torch.cuda.synchronize()
    codes = out.codes.cpu().numpy()
    assert np.all(codes[m_out:] == 0xAB)
    assert np.all(out.scales.cpu().numpy()[api.scale_bytes(m_out, K):] == 0xAB)
    assert torch.all(out.r_sel[m_out:].float() == 7.0)
    ref = oracle.quantize(x)
    for r in range(M):
        for j in range(F):
            d = dst[r, j]
            if d < m_out:
                assert np.array_equal(codes[d], ref.codes[r])


def _codes16(packed):
    return [int(packed[i // 2] >> (4 * (i % 2)) & 15) for i in range(16)]


def test_division_boundary_blocks_match_oracle(cuda):
    """The stored blocks on which a reciprocal-multiply or double-rounded
    shortcut would give other scale codes, element codes or dequantized
    values (tests/golden/division_cases.txt): the kernels' codes, scales,
    residual operand and fake-quantized values equal the stored ones."""
    from conftest import division_cases
    for c in division_cases():
        x = np.zeros((1, 64), np.uint16)
        x[0, :16] = c["x"]
        s_t = np.array([c["s_t"]], np.uint32).view(np.float32)
        st = torch.from_numpy(s_t.copy()).to(cuda)
        q = api.quantize(to_bf16_dev(x, cuda), rac_k=16, s_t=st, want_score=True)
        torch.cuda.synchronize()
        assert unswizzle(q.scales, 1, 64)[0, 0] == c["sf"]
        assert _codes16(q.codes.cpu().numpy()[0]) == c["codes"]
        ref = oracle.quantize(x, s_t=float(s_t[0]))
        sel = q.sel.cpu().numpy()[:16]
        assert np.array_equal(np_u16(q.r_sel)[:, :16], oracle.rac_residual(ref.resid, ref.s_t, sel))
        xh = np.array(c["xhat"], np.uint32).view(np.float32)
        assert np.array_equal(ref.xhat[0, :16].view(np.uint32), c["xhat"])
        del xh


def _near_boundary_groups(rng, G, rows, cols):
    """G weight tensors whose blocks sit next to the encoders' rounding
    boundaries: each block has a maximum whose scale quotient a/(6 s_t) lies
    near an E4M3 midpoint or value, and elements at the bf16 values nearest
    to an E2M1 threshold times the block scale.  The tensor scale comes from
    one planted maximum per tensor."""
    e4 = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    thr = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    out = np.empty((G, rows, cols), np.uint16)
    nb = rows * cols // 16
    for g in range(G):
        A = float(oracle.bf16_to_f32(oracle.f32_to_bf16(np.array([rng.uniform(1.0, 2.0) * 2.0 ** rng.integers(-8, 8)],
                                                                np.float32)))[0])
        s_t = np.float32(np.float32(A) / np.float32(2688.0))
        c = rng.integers(0x08, 0x7E, nb)
        mid = np.where(rng.random(nb) < 0.5, (e4[c] + e4[c + 1]) / 2, e4[c])
        amax_b = np.minimum(6.0 * mid * float(s_t), A)
        d = (e4[c].astype(np.float32) * s_t).astype(np.float64)
        t = thr[rng.integers(0, 7, (nb, 15))] * np.where(rng.random((nb, 15)) < 0.5, -1.0, 1.0)
        vals = np.concatenate([amax_b[:, None], t * d[:, None]], axis=1)
        blk = oracle.f32_to_bf16(vals.astype(np.float32)).reshape(rows, cols)
        blk[0, 0] = oracle.f32_to_bf16(np.array([A], np.float32))[0]
        out[g] = blk
    return out


def test_near_boundary_sweep_matches_oracle(cuda):
    """About a million blocks built at the encoders' rounding boundaries, as
    per-tensor weight fake quantization (each tensor its own s_t): codes,
    scale bytes and bf16 dequantized values bit-exact against the oracle, and
    the activation path (given s_t, with scores) gives the same codes."""
    rng = np.random.default_rng(123)
    G, rows, cols = 1024, 64, 256
    w = _near_boundary_groups(rng, G, rows, cols)
    wq, s_t, codes, scales = api.qdq_weights(to_bf16_dev(w, cuda), want_qdq=True, want_packed=True)
    torch.cuda.synchronize()
    wq, s_t, codes, scales = np_u16(wq), s_t.cpu().numpy(), codes.cpu().numpy(), scales.cpu().numpy()
    for g in range(G):
        ref_bf16, ref_s, ref = oracle.qdq(w[g])
        assert s_t[g] == np.float32(ref_s)
        assert np.array_equal(codes[g], ref.codes), g
        assert np.array_equal(oracle.unswizzle_scales(scales[g], rows, cols), ref.sf), g
        assert np.array_equal(wq[g], ref_bf16), g
    for g in range(0, G, 97):
        q = api.quantize(to_bf16_dev(w[g], cuda), rac_k=32, s_t=torch.tensor([s_t[g]], device=cuda),
                         want_score=True)
        torch.cuda.synchronize()
        assert np.array_equal(q.codes.cpu().numpy(), codes[g])


@pytest.mark.parametrize("M,K,k", [(300, 2048, 1024), (129, 768, 768), (64, 4096, 2048), (200, 4096, 300),
                                   (40, 16384, 1100)])
def test_quantize_rac_percent_channels(cuda, M, K, k):
    """RAC on "the top k% of channels" (7% to 100%, rows staged in one or
    several pieces and column windows): selection, scores and residual operand
    bit-exact beyond the former 256-channel cap."""
    rng = np.random.default_rng(M + K + k)
    _quant_parity(cuda, gen_x(rng, M, K), k)


def test_channel_major_gather_wide(cuda):
    """The channel-major weight gather with more than 256 channels (chunked
    over channels) equals the K-major gather and the oracle's e2m1 * sf."""
    rng = np.random.default_rng(31)
    E, N, K, k, ld = 2, 256, 1536, 700, 768
    w = oracle.f32_to_bf16(rng.standard_normal((E, N, K)).astype(np.float32) * 0.02)
    _, s_t, codes, scales = api.qdq_weights(to_bf16_dev(w, cuda), want_qdq=False, want_packed=True)
    ccm, scm = api.weights_channel_major(codes, scales, N, K)
    sel = np.sort(rng.choice(K, k, replace=False)).astype(np.int32)
    seld = torch.from_numpy(sel).to(cuda)
    a = np_u16(api.gather_weight_channels(codes, scales, N, K, seld, k, ld))
    b = np_u16(api.gather_weight_channels_cm(ccm, scm, N, K, seld, k, ld))
    assert np.array_equal(a, b)
    assert np.all(b[:, :, k:] == 0)
    for e in range(E):
        ref = oracle.quantize(w[e])
        q = np.empty((N, K), np.uint8)
        q[:, 0::2] = ref.codes & 0xF
        q[:, 1::2] = ref.codes >> 4
        vals = oracle.e2m1_decode(q) * np.repeat(oracle.e4m3_decode(ref.sf), 16, axis=1)
        assert np.array_equal(b[e, :, :k], oracle.f32_to_bf16(vals[:, sel].astype(np.float32)))


@pytest.mark.parametrize("M,K,k,ld", [(300, 768, 32, 64), (129, 2048, 100, 128), (64, 4096, 2048, 2048)])
def test_rac_second_pass_nvfp4_parity(cuda, M, K, k, ld):
    """The second-pass RAC variant: the selected residual channels quantized
    again to NVFP4 (own tensor scale, 16-channel blocks, last block padded);
    the operand bit-exact against the oracle, padding columns zero."""
    rng = np.random.default_rng(M + K + k)
    x = gen_x(rng, M, K)
    xd = to_bf16_dev(x, cuda)
    q = api.quantize(xd, rac_k=k, rac_ld=ld, want_score=True)
    s_r = torch.empty(1, dtype=torch.float32, device=cuda)
    api.rac_residual_nvfp4(xd, q, k, ld, s_r_out=s_r)
    torch.cuda.synchronize()
    ref = oracle.quantize(x)
    sel = q.sel.cpu().numpy()[:k]
    check_selection(sel, oracle.channel_score(ref.resid), oracle.select_topk(oracle.channel_score(ref.resid), k), k)
    rho2, s_r_ref = oracle.rac_residual_nvfp4(ref.resid, ref.s_t, sel)
    assert s_r.item() == np.float32(s_r_ref)
    got = np_u16(q.r_sel)
    assert np.array_equal(got[:, :k], rho2)
    assert np.all(got[:, k:] == 0)


def test_zero_row_chunks_match_oracle(cuda):
    """Rows whose 256-channel chunks are all zero (the padding rows of routed
    segments) take a short path in the kernel: +0 and -0 rows, rows zero in
    only some chunks, and mixed rows give the oracle's codes (-0 -> code 8),
    scale bytes, scores and QDQ values bit for bit."""
    rng = np.random.default_rng(77)
    M, K = 96, 1024
    x = gen_x(rng, M, K)
    x[0:8] = 0                                   # +0 rows
    x[8:16] = 0x8000                             # -0 rows
    x[16:24, :256] = 0                           # first chunk zero
    x[24:32, 512:768] = 0x8000                   # a middle chunk of -0
    x[32:40] = np.where(rng.random((8, K)) < 0.5, 0x8000, 0).astype(np.uint16)   # mixed signed zeros
    x[40:48, 768:] = 0
    x[40:48, 768] = 0x3F80                       # a single 1.0 in an otherwise zero chunk
    _quant_parity(cuda, x, 16)
    # QDQ (one tensor) over the same rows
    w_qdq, s_t, codes, scales = api.qdq_weights(to_bf16_dev(x, cuda), want_packed=True)
    torch.cuda.synchronize()
    wq, s_ref, _ = oracle.qdq(x)
    assert s_t.item() == np.float32(s_ref)
    assert np.array_equal(np_u16(w_qdq), wq)


def test_selection_without_residual(cuda):
    """r_sel NULL with rac_k > 0: the channels are selected exactly as with a
    residual output, and no residual is written."""
    rng = np.random.default_rng(12)
    M, K, k = 300, 1024, 40
    x = gen_x(rng, M, K)
    xd = to_bf16_dev(x, cuda)
    full = api.quantize(xd, rac_k=k, want_score=True)
    q = api.quantize(xd, rac_k=k, want_score=True, want_residual=False)
    sentinel = torch.full_like(q.r_sel, 3.0)
    q.r_sel.copy_(sentinel)
    q = api.quantize(xd, rac_k=k, want_score=True, want_residual=False, out=q)
    torch.cuda.synchronize()
    assert torch.equal(q.sel, full.sel) and torch.equal(q.codes, full.codes)
    assert torch.equal(q.r_sel, sentinel)
