"""Pins of the oracle's second-pass RAC variant (the selected residual
channels quantized again to NVFP4): the binary32 block quantization against
the exact rational model, grid-valued residuals passing through unchanged,
the per-element bound |rhat - R| <= d, and the MoE layer reducing to the
plain RAC layer when the second pass is exact."""
import numpy as np

import oracle
from exact_fp import quantize_block_exact_f32, f32_bits_to_fraction

F = np.float32
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def test_quantize_f32_matches_exact_model():
    rng = np.random.default_rng(21)
    for _ in range(200):
        s_t = F(2.0 ** rng.uniform(-20, 5)) * F(rng.uniform(1, 2))
        x = (rng.standard_normal(16) * float(s_t) * 2688 * 2.0 ** rng.uniform(-10, 0)).astype(F)
        q = oracle.quantize_f32(x.reshape(1, 16), float(s_t))
        codes = [int(q.codes[0, i // 2] >> (4 * (i % 2)) & 15) for i in range(16)]
        sb = int(np.array([s_t], F).view(np.uint32)[0])
        sf_e, codes_e, xhat_e = quantize_block_exact_f32(x.view(np.uint32).tolist(), sb)
        assert (int(q.sf[0, 0]), codes) == (sf_e, codes_e)
        assert [f32_bits_to_fraction(int(b)) for b in q.xhat[0].view(np.uint32)] == xhat_e


def test_second_pass_is_identity_on_grid_residuals():
    """Residuals that already are NVFP4 values of their own blocks pass the
    second quantization unchanged, so the variant's operand equals the plain
    one: every block's maximum is 6 sf_b s_r for an E4M3 value sf_b, and the
    largest block has sf_b = 448, so the tensor scale max/2688 is exactly
    s_r (a power of two) and every step is exact."""
    rng = np.random.default_rng(22)
    M, K, k = 8, 64, 32
    s_r = 2.0 ** -8
    e4 = oracle.e4m3_decode(np.arange(0x08, 0x7F, dtype=np.uint8))   # normal E4M3 values
    sf = rng.choice(e4, (M, k // 16))
    sf[0, 0] = 448.0
    idx = rng.integers(0, 8, (M, k))
    idx[:, 0] = 7
    idx[:, 16] = 7
    R = E2M1[idx] * np.repeat(sf, 16, axis=1) * s_r * np.where(rng.random((M, k)) < 0.5, -1, 1)
    assert np.array_equal(R.astype(F).astype(np.float64), R)
    resid = np.zeros((M, K), F)
    S = np.sort(rng.choice(K, k, replace=False)).astype(np.int32)
    resid[:, S] = R.astype(F)
    rho2, s_r_got = oracle.rac_residual_nvfp4(resid, 0.5, S)
    assert s_r_got == s_r
    rho = oracle.rac_residual(resid, 0.5, S)
    assert np.array_equal(rho2, rho)


def test_second_pass_error_bound():
    rng = np.random.default_rng(23)
    x = oracle.f32_to_bf16(rng.standard_normal((64, 256)).astype(F))
    qz = oracle.quantize(x)
    S = oracle.select_topk(oracle.channel_score(qz.resid), 40)
    RS = np.zeros((64, 48), F)
    RS[:, :40] = qz.resid[:, S]
    q2 = oracle.quantize_f32(RS)
    d = (oracle.e4m3_decode(q2.sf).astype(F) * F(q2.s_t)).astype(np.float64)
    assert np.all(np.abs(q2.xhat.astype(np.float64) - RS) <= np.repeat(d, 16, axis=1) * (1 + 2.0 ** -20))
    assert np.all(q2.xhat[:, 40:] == 0)
