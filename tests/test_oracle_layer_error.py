"""Pins of the oracle's layer-error measure (oracle/layer_error.py) against
identities of the definition err(k) = ||Y_RAC(k) - X What^T|| / ||X What^T||
(QUADS, gist.science/it 2.2 B): the residual R = X - Xhat is exact, so the
error is a function of R, the selection and rho alone."""
import numpy as np
import pytest
import torch

import oracle
from oracle.layer_error import rac_layer_error
from quantization_nvfp4_quantize_b200 import workloads as wl


GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).numpy().view(np.uint16)


def _small(alpha=20.0, T=48, K=256, N=64, seed=3):
    x = _bits(wl.outlier_activations(T, K, alpha, seed, frac=0.02))
    w = _bits(wl.dense_weight(N, K, seed))
    return x, w


def test_exactly_representable_input_has_no_error():
    # blocks of E2M1 grid values x 448 x 2^m with a 6 in every block: s_t = 2^m,
    # block scales 448 * 2^-i and the codes are exact, so R = 0 and every err is 0
    rng = np.random.default_rng(0)
    T, K, m = 32, 64, -8
    mag = GRID[rng.integers(0, 8, size=(T, K))]
    mag.reshape(T, K // 16, 16)[:, :, 0] = 6.0
    sign = np.where(rng.random((T, K)) < 0.5, -1.0, 1.0)
    blk = np.repeat(2.0 ** -rng.integers(0, 5, size=(T, K // 16)), 16, axis=1)
    blk[0, :16] = 1.0                                   # the tensor max is 6 * 448 * 2^m
    xf = (sign * mag * blk * 448.0 * 2.0 ** m).astype(np.float32)
    x = oracle.f32_to_bf16(xf)
    assert np.array_equal(oracle.bf16_to_f32(x), xf)
    w = _bits(wl.dense_weight(16, K, 0))
    xq = oracle.quantize(x)
    assert xq.s_t == 2.0 ** m and not xq.resid.any()
    for mode in ("bf16", "nvfp4"):
        assert rac_layer_error(x, w, [0, 1, 8, 64], mode) == [0.0, 0.0, 0.0, 0.0]


def test_no_rac_error_is_the_residual_product():
    # Y_RAC(0) - X What^T = -R What^T exactly (R = x - xhat has no rounding)
    x, w = _small()
    what = oracle.quantize(w).xhat.astype(np.float64)
    X = oracle.bf16_to_f32(x).astype(np.float64)
    R = oracle.quantize(x).resid.astype(np.float64)
    assert np.array_equal(X - oracle.quantize(x).xhat.astype(np.float64), R)
    want = np.linalg.norm(R @ what.T) / np.linalg.norm(X @ what.T)
    got = rac_layer_error(x, w, [0])[0]
    assert got == pytest.approx(want, rel=1e-9)


@pytest.mark.parametrize("mode", ["bf16", "nvfp4"])
def test_all_channels_leave_only_the_operand_rounding(mode):
    # k = K: Y_RAC - X What^T = (s_t rho - R) What^T, rho over every channel
    x, w = _small()
    K = x.shape[1]
    what = oracle.quantize(w).xhat.astype(np.float64)
    X = oracle.bf16_to_f32(x).astype(np.float64)
    xq = oracle.quantize(x)
    S = np.arange(K, dtype=np.int32)
    rho = oracle.rac_residual(xq.resid, xq.s_t, S) if mode == "bf16" else \
        oracle.rac_residual_nvfp4(xq.resid, xq.s_t, S)[0]
    D = xq.s_t * oracle.bf16_to_f32(rho).astype(np.float64) - xq.resid.astype(np.float64)
    want = np.linalg.norm(D @ what.T) / np.linalg.norm(X @ what.T)
    got, e0 = rac_layer_error(x, w, [K, 0], mode)
    assert got == pytest.approx(want, rel=1e-9)
    assert got < (0.02 if mode == "bf16" else 0.5) * e0


def test_scaled_identity_weight_reduces_to_unselected_residual_energy():
    # W = 2688 I is exact in NVFP4 (s_t = 1, sf = 448, code 6), so Y = 2688 X and
    # err(k)^2 ||X||^2 = (energy of the K - k smallest-score channels) + (rounding of rho)
    K, T = 64, 40
    x = _bits(wl.outlier_activations(T, K, 20.0, 5, frac=0.05))
    w = oracle.f32_to_bf16((2688.0 * np.eye(K)).astype(np.float32))
    wq = oracle.quantize(w)
    assert np.array_equal(wq.xhat, (2688.0 * np.eye(K)).astype(np.float32))
    xq = oracle.quantize(x)
    score = oracle.channel_score(xq.resid)
    X = oracle.bf16_to_f32(x).astype(np.float64)
    for k in (0, 3, 16, 40):
        S = oracle.select_topk(score, k)
        rest = np.sort(score)[: K - k].sum()                 # the K - k smallest scores
        rho = oracle.rac_residual(xq.resid, xq.s_t, S) if k else np.zeros((T, 0), np.uint16)
        sel = xq.resid[:, S].astype(np.float64) - xq.s_t * oracle.bf16_to_f32(rho).astype(np.float64)
        want = np.sqrt(rest + (sel ** 2).sum()) / np.linalg.norm(X)
        assert rac_layer_error(x, w, [k])[0] == pytest.approx(want, rel=1e-9)
