"""Pins of the oracle's NVFP4 block quantization, residual scoring, channel
selection and RAC residual against closed forms, invariants and brute force."""
from fractions import Fraction

import numpy as np
import pytest

import oracle

E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def bf16(a):
    return oracle.f32_to_bf16(np.asarray(a, np.float32))


def randn_bf16(rng, *shape, scale=1.0):
    return bf16(rng.standard_normal(shape).astype(np.float32) * scale)


def test_grid_values_round_trip_exactly():
    """A block of grid values g * sf * s_t (exact in bf16 for s_t a power of
    two) containing 6 * sf * s_t quantizes back to exactly those codes and
    scale, with zero residual."""
    rng = np.random.default_rng(0)
    sf_vals = oracle.e4m3_decode(np.arange(0x08, 0x7F, dtype=np.uint8))   # normal E4M3 scales
    for trial in range(400):
        s_t = np.float32(2.0 ** rng.integers(-20, 10))
        sf_code = rng.integers(0x08, 0x7F)
        sf = oracle.e4m3_decode(np.array([sf_code], np.uint8))[0]
        idx = rng.integers(0, 8, 16)
        idx[rng.integers(0, 16)] = 7
        sign = rng.integers(0, 2, 16)
        vals = np.where(sign == 1, -1.0, 1.0) * E2M1_MAG[idx] * sf * float(s_t)
        x = bf16(vals)
        assert np.array_equal(oracle.bf16_to_f32(x).astype(np.float64), vals), "test values not exact"
        qz = oracle.quantize(x.reshape(1, 16), s_t=float(s_t))
        assert qz.sf[0, 0] == sf_code
        codes = np.empty(16, np.uint8)
        codes[0::2] = qz.codes[0] & 0xF
        codes[1::2] = qz.codes[0] >> 4
        assert np.array_equal(codes & 7, idx)
        nz = idx != 0
        assert np.array_equal((codes[nz] >> 3) & 1, sign[nz])
        assert np.all(qz.resid == 0)
    del sf_vals


def test_block_max_maps_to_six_and_residual_bound():
    rng = np.random.default_rng(1)
    x = randn_bf16(rng, 256, 512)
    x[:, 37] = bf16(oracle.bf16_to_f32(x[:, 37]) * 40)          # an outlier channel
    qz = oracle.quantize(x)
    xf = oracle.bf16_to_f32(x).reshape(256, 32, 16)
    q = np.empty((256, 512), np.uint8)
    q[:, 0::2] = qz.codes & 0xF
    q[:, 1::2] = qz.codes >> 4
    q = q.reshape(256, 32, 16)
    sf = oracle.e4m3_decode(qz.sf)
    d = (sf.astype(np.float32) * np.float32(qz.s_t)).astype(np.float32)
    amax_pos = np.abs(xf).argmax(axis=2)
    qmax = np.take_along_axis(q, amax_pos[..., None], axis=2)[..., 0]
    normal = sf >= 2.0 ** -6
    assert normal.mean() > 0.9
    assert np.all((qmax[normal] & 7) == 7), "block maximum must map to magnitude 6"
    R = qz.resid.reshape(256, 32, 16).astype(np.float64)
    assert np.all(np.abs(R) <= d[..., None].astype(np.float64) * (1 + 2.0 ** -20))
    # xhat = fl(e2m1 * sf * s_t), one rounding of the exact product
    qsf = (oracle.e2m1_decode(q) * sf[..., None]).astype(np.float32)
    xh = (qsf * np.float32(qz.s_t)).astype(np.float32)
    assert np.array_equal(xh.reshape(256, 512), qz.xhat)
    assert np.array_equal((xf - xh).reshape(256, 512), qz.resid)


def test_tensor_scale_puts_largest_block_at_448():
    rng = np.random.default_rng(2)
    x = randn_bf16(rng, 64, 256, scale=3.0)
    qz = oracle.quantize(x)
    A = np.abs(oracle.bf16_to_f32(x)).max()
    assert qz.s_t == np.float32(np.float32(A) / np.float32(2688.0))
    r, c = np.unravel_index(np.abs(oracle.bf16_to_f32(x)).argmax(), x.shape)
    assert qz.sf[r, c // 16] == 0x7E


def test_zero_block_and_zero_tensor():
    x = np.zeros((4, 64), np.uint16)
    qz = oracle.quantize(x)
    assert qz.s_t == 1.0
    assert np.all(qz.codes == 0) and np.all(qz.sf == 0) and np.all(qz.resid == 0)
    rng = np.random.default_rng(3)
    y = randn_bf16(rng, 4, 64)
    y[:, 16:32] = 0
    qy = oracle.quantize(y)
    assert np.all(qy.sf[:, 1] == 0) and np.all(qy.codes[:, 8:16] == 0)
    # negative zeros keep their sign bit
    z = np.zeros((1, 16), np.uint16)
    z[0, 3] = 0x8000
    assert (oracle.quantize(z).codes[0, 1] >> 4) == 0x8


def test_dequantize_matches_quantize_xhat():
    rng = np.random.default_rng(4)
    x = randn_bf16(rng, 33, 128, scale=0.1)
    qz = oracle.quantize(x)
    assert np.array_equal(oracle.dequantize(qz.codes, qz.sf, qz.s_t), qz.xhat)


def test_relative_quantization_error_is_fp4_sized():
    rng = np.random.default_rng(5)
    x = randn_bf16(rng, 512, 256)
    qz = oracle.quantize(x)
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    rel = np.linalg.norm(qz.resid) / np.linalg.norm(xf)
    assert 0.05 < rel < 0.2, rel


def test_channel_score_brute_force_exact():
    rng = np.random.default_rng(6)
    x = randn_bf16(rng, 9, 32)
    qz = oracle.quantize(x)
    valid = np.array([0, 1, -1, 3, 4, -1, 6, 7, 8], np.int32)
    s = oracle.channel_score(qz.resid, valid)
    for c in range(32):
        exact = sum(Fraction(float(qz.resid[r, c])) ** 2 for r in range(9) if valid[r] >= 0)
        assert abs(Fraction(s[c]) - exact) <= exact * Fraction(1, 2 ** 50)


@pytest.mark.parametrize("K,k", [(64, 0), (64, 1), (256, 8), (256, 128), (256, 256), (4096, 128)])
def test_select_topk_matches_full_sort(K, k):
    rng = np.random.default_rng(K + k)
    score = rng.random(K) ** 3
    score[rng.integers(0, K, K // 4)] = 0.5           # ties
    S = oracle.select_topk(score, k)
    order = np.lexsort((np.arange(K), -score))       # score desc, index asc
    assert np.array_equal(S, np.sort(order[:k]))
    assert np.all(np.diff(S) > 0)


def test_select_all_equal_prefers_low_indices():
    S = oracle.select_topk(np.ones(100), 7)
    assert np.array_equal(S, np.arange(7))


def test_rac_residual_is_bf16_of_scaled_residual():
    rng = np.random.default_rng(7)
    x = randn_bf16(rng, 40, 128)
    qz = oracle.quantize(x)
    S = np.array([3, 17, 64, 127], np.int32)
    rho = oracle.rac_residual(qz.resid, qz.s_t, S, k_pad=64)
    assert rho.shape == (40, 64) and np.all(rho[:, 4:] == 0)
    got = oracle.bf16_to_f32(rho[:, :4]).astype(np.float64) * qz.s_t
    want = qz.resid[:, S].astype(np.float64)
    assert np.all(np.abs(got - want) <= np.abs(want) * 2.0 ** -8 + 1e-30)
