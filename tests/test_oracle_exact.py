"""Pins of the oracle's NVFP4 block arithmetic against an exact rational
model (tests/exact_fp.py: binary32 round-to-nearest-even written out, the
OCP E2M1 / E4M3 code tables), on random blocks and on stored blocks
(tests/golden/division_cases.txt) chosen so that a reciprocal-multiply
scale or element step, or a double-rounded dequantization, would give
other codes or values."""
import numpy as np
import pytest

import oracle
from conftest import division_cases
from exact_fp import quantize_block_exact, f32_bits_to_fraction

F = np.float32


CASES = division_cases()


def _oracle_block(x_bits, s_t_bits):
    s_t = float(np.array([s_t_bits], np.uint32).view(F)[0])
    q = oracle.quantize(np.array(x_bits, np.uint16).reshape(1, 16), s_t=s_t)
    codes = [int(q.codes[0, i // 2] >> (4 * (i % 2)) & 15) for i in range(16)]
    return int(q.sf[0, 0]), codes, q.xhat[0].view(np.uint32).tolist(), q.resid[0]


def test_fixture_covers_every_kind():
    kinds = [c["kind"] for c in CASES]
    assert kinds.count("scale") >= 10 and kinds.count("element") >= 20 and kinds.count("dequant") >= 5


@pytest.mark.parametrize("i", range(len(CASES)))
def test_stored_case_oracle_and_exact_model(i):
    c = CASES[i]
    sf, codes, xhat, _ = _oracle_block(c["x"], c["s_t"])
    assert (sf, codes, xhat) == (c["sf"], c["codes"], c["xhat"])
    sf_e, codes_e, xhat_e, _ = quantize_block_exact(c["x"], c["s_t"])
    assert sf_e == c["sf"] and codes_e == c["codes"]
    assert xhat_e == [f32_bits_to_fraction(b) for b in c["xhat"]]


@pytest.mark.parametrize("i", range(len(CASES)))
def test_stored_case_rejects_shortcuts(i):
    """Each stored block separates the plain evaluation from a shortcut, so a
    reversion to the shortcut fails the test above."""
    c = CASES[i]
    s_t = np.array([c["s_t"]], np.uint32).view(F)[0]
    x = oracle.bf16_to_f32(np.array(c["x"], np.uint16))
    a = np.abs(x).max()
    if c["kind"] == "scale":
        recip = oracle.e4m3_encode(np.array([a * F(F(1) / F(F(6) * s_t))], F))[0]
        div6 = oracle.e4m3_encode(np.array([a / F(F(6) * s_t)], F))[0]
        assert recip != c["sf"] or div6 != c["sf"]
    d = F(F(oracle.e4m3_decode(np.array([c["sf"]], np.uint8))[0]) * s_t)
    if c["kind"] == "element":
        alt = oracle.e2m1_encode((x * F(F(1) / d)).astype(F))
        assert not np.array_equal(alt, np.array(c["codes"], np.uint8))
    if c["kind"] == "dequant":
        alt = (oracle.e2m1_decode(np.array(c["codes"], np.uint8)).astype(F) * d).astype(F)
        assert not np.array_equal(alt.view(np.uint32), np.array(c["xhat"], np.uint32))


def _random_blocks(rng, n):
    out = []
    for _ in range(n):
        s_t = F(2.0 ** rng.uniform(-30, 20)) * F(rng.uniform(1, 2))
        scale = float(s_t) * 2688 * 2.0 ** rng.uniform(-24, 0)
        v = rng.standard_normal(16) * scale
        if rng.random() < 0.2:
            v[rng.integers(0, 16, 4)] = 0.0
        bits = oracle.f32_to_bf16(v.astype(F))
        if rng.random() < 0.2:
            bits[rng.integers(0, 16)] = 0x8000              # a negative zero
        out.append((bits.tolist(), int(np.array([s_t], F).view(np.uint32)[0])))
    return out


def test_random_blocks_match_exact_model():
    rng = np.random.default_rng(11)
    for x_bits, s_bits in _random_blocks(rng, 400):
        sf, codes, xhat, resid = _oracle_block(x_bits, s_bits)
        sf_e, codes_e, xhat_e, R_e = quantize_block_exact(x_bits, s_bits)
        assert (sf, codes) == (sf_e, codes_e), (x_bits, s_bits)
        assert [f32_bits_to_fraction(b) for b in xhat] == xhat_e
        assert [f32_bits_to_fraction(int(b)) for b in resid.view(np.uint32)] == R_e
