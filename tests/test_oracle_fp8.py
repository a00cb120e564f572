"""Pins of the oracle's per-tensor FP8 E4M3 quantization (the comparison
format): an exact rational model, the tensor maximum at 448, grid values
round-tripping, saturation and signed zeros."""
import numpy as np

import oracle
from exact_fp import fp8_quantize_exact, f32_bits_to_fraction

F = np.float32


def test_fp8_matches_exact_model():
    rng = np.random.default_rng(3)
    for trial in range(60):
        scale = 2.0 ** rng.uniform(-20, 20)
        v = (rng.standard_normal(64) * scale).astype(F)
        x = oracle.f32_to_bf16(v).reshape(1, 64)
        if trial % 7 == 0:
            x[0, 5] = 0x8000
        codes, xhat, s = oracle.fp8_quantize(x)
        sb = int(np.array([s], F).view(np.uint32)[0])
        want = fp8_quantize_exact(x[0].tolist(), sb)
        assert [c for c, _ in want] == codes[0].tolist()
        assert [xh for _, xh in want] == [f32_bits_to_fraction(int(b)) for b in xhat[0].view(np.uint32)]


def test_fp8_tensor_max_maps_to_448_and_grid_round_trip():
    rng = np.random.default_rng(4)
    x = oracle.f32_to_bf16((rng.standard_normal((32, 64)) * 3).astype(F))
    codes, xhat, s = oracle.fp8_quantize(x)
    A = np.abs(oracle.bf16_to_f32(x)).max()
    assert s == np.float32(np.float32(A) / np.float32(448))
    r, c = np.unravel_index(np.abs(oracle.bf16_to_f32(x)).argmax(), x.shape)
    assert codes[r, c] & 0x7F == 0x7E
    # E4M3 grid values times a power-of-two scale come back exactly
    grid = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    vals = np.concatenate([grid, -grid[1:]]) * 0.25
    xg = oracle.f32_to_bf16(vals.astype(F)).reshape(1, -1)
    cg, xhg, sg = oracle.fp8_quantize(xg, s=0.25)
    assert np.array_equal(xhg[0], vals.astype(F))


def test_fp8_saturates_and_zero_tensor():
    x = oracle.f32_to_bf16(np.array([[1e4, -1e4, 1.0, -0.0] * 4], F))
    codes, xhat, s = oracle.fp8_quantize(x, s=1.0)
    assert codes[0, 0] == 0x7E and codes[0, 1] == 0xFE and codes[0, 3] == 0x80
    z = np.zeros((2, 16), np.uint16)
    cz, xz, sz = oracle.fp8_quantize(z)
    assert sz == 1.0 and np.all(cz == 0) and np.all(xz == 0)
