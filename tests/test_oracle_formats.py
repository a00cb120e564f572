"""Pins of the oracle's E2M1 / E4M3 / bf16 encoders against the format
definitions (golden tables from the OCP specifications) and exhaustive
nearest-value properties."""
import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden

E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def all_finite_bf16_as_f32():
    h = np.arange(65536, dtype=np.uint32)
    f = (h << 16).view(np.float32)
    return f[np.isfinite(f)]


def test_e2m1_decode_matches_golden_table():
    for code, val in read_golden("e2m1_table.txt"):
        c = int(code, 16)
        got = oracle.e2m1_decode(np.array([c], np.uint8))[0]
        assert got == float(val) and np.signbit(got) == val.startswith("-"), (code, got, val)


def test_e2m1_ties_and_saturation_golden():
    for y, code in read_golden("e2m1_ties.txt"):
        got = int(oracle.e2m1_encode(np.array([np.float32(y)]))[0])
        assert got == int(code, 16), (y, hex(got), code)


def test_e2m1_encode_exhaustive_nearest_even():
    y = all_finite_bf16_as_f32()
    q = oracle.e2m1_encode(y)
    a = np.abs(y.astype(np.float64))
    idx = (q & 7).astype(np.int64)
    assert np.all(idx[a > 6.0] == 7), "values above 6 must saturate"
    inr = a <= 6.0                      # distances below are exact in binary64
    a, idx, q, y = a[inr], idx[inr], q[inr], y[inr]
    err = np.abs(a - E2M1_MAG[idx])
    dist = np.abs(a[:, None] - E2M1_MAG[None, :])
    best = dist.min(axis=1)
    assert np.all(err == best), "not a nearest value"
    ties = (dist == best[:, None]).sum(axis=1) > 1
    assert np.all(idx[ties] % 2 == 0), "tie not resolved to the even code"
    assert np.all(((q >> 3) & 1) == np.signbit(y)), "sign bit does not follow the input"
    # monotone in |y|
    order = np.argsort(a, kind="stable")
    assert np.all(np.diff(idx[order]) >= 0)


def test_e4m3_decode_golden_and_monotone():
    for code, val in read_golden("e4m3_table.txt"):
        assert oracle.e4m3_decode(np.array([int(code, 16)], np.uint8))[0] == float(val), code
    v = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    assert np.all(np.diff(v) > 0)
    assert v[-1] == 448.0 and v[1] == 2.0 ** -9


def test_e4m3_roundtrip_all_codes():
    codes = np.arange(0x7F, dtype=np.uint8)
    v = oracle.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(v), codes)


def _e4m3_probe_values(rng):
    v = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (v[:-1] + v[1:]) / 2          # exact in binary32
    m32 = mids.astype(np.float32)
    assert np.all(m32.astype(np.float64) == mids)
    pts = [m32, np.nextafter(m32, np.float32(np.inf)), np.nextafter(m32, np.float32(0)),
           v.astype(np.float32), np.array([448.0, 464.0, 465.0, 480.0, 1e6, 3e38, 0.0, 2.0 ** -10, 2.0 ** -11],
                                          np.float32)]
    r = np.exp(rng.uniform(np.log(1e-5), np.log(600.0), 1_000_000)).astype(np.float32)
    return np.concatenate(pts + [r]).astype(np.float32)


def test_e4m3_encode_nearest_even_saturating():
    rng = np.random.default_rng(0)
    x = _e4m3_probe_values(rng)
    q = oracle.e4m3_encode(x)
    table = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    a = x.astype(np.float64)
    err = np.abs(a - table[q])
    # nearest: compare against both neighbours in the sorted table
    pos = np.clip(np.searchsorted(table, a), 1, len(table) - 1)
    lo, hi = pos - 1, pos
    best = np.minimum(np.abs(a - table[lo]), np.abs(a - table[hi]))
    best = np.where(a >= table[-1], a - table[-1], best)
    assert np.all(err == best)
    tie = (np.abs(a - table[lo]) == np.abs(a - table[hi])) & (a < table[-1])
    assert np.all(q[tie] % 2 == 0)
    assert np.all(q[a >= 448.0] == 0x7E)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    f = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        (np.arange(1 << 16, dtype=np.uint32) << 16 | 0x8000).view(np.float32)])
    f = f[np.isfinite(f)]
    ours = oracle.f32_to_bf16(f)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(oracle.bf16_to_f32(ours), torch.from_numpy(ours.view(np.int16)).view(torch.bfloat16).float().numpy())


# ---------------------------------------------------- scale-factor byte layout
# Structural pins of oracle.swizzle_scales / unswizzle_scales.  The layout
# itself is pinned on the GPU, where the tensor cores consume it and the GEMM
# matches the oracle's products.  Here: it is a bijection onto the padded
# buffer, its inverse is exact, padding rows are zero, and it has the two
# properties the kernels rely on (a row's four scales of one 64-element block
# group are one 32-bit word; rows 32 apart in an atom are 4 bytes apart).

def _sf(M, nkb, seed=0):
    rng = np.random.default_rng(seed)
    return rng.integers(1, 256, size=(M, nkb), dtype=np.uint8)      # never 0


@pytest.mark.parametrize("M,nkb", [(128, 4), (256, 8), (384, 16), (130, 4), (1, 8), (1000, 12)])
def test_swizzle_round_trip_and_padding(M, nkb):
    sf = _sf(M, nkb, M + nkb)
    buf = oracle.swizzle_scales(sf)
    m_pad = -(-M // 128) * 128
    assert buf.size == m_pad * nkb                      # one byte per (padded row, block)
    assert np.array_equal(oracle.unswizzle_scales(buf, M, nkb * 16), sf)
    assert np.count_nonzero(buf) == M * nkb            # padding rows are zero, nothing collides


def test_swizzle_is_a_bijection_on_full_atoms():
    M, nkb = 256, 8
    r = np.arange(M)[:, None]
    c = np.arange(nkb)[None, :]
    # position of (r, c) found by swizzling a one-hot byte per row chunk
    seen = np.zeros(M * nkb, np.int32)
    for rr in range(M):
        for cc in range(nkb):
            one = np.zeros((M, nkb), np.uint8)
            one[rr, cc] = 1
            seen += oracle.swizzle_scales(one).astype(np.int32)
    assert np.all(seen == 1)


def test_swizzle_word_and_quadrant_structure():
    M, nkb = 128, 8
    sf = np.zeros((M, nkb), np.uint8)
    # row 5, blocks 4..7 -> four consecutive bytes (one 32-bit word)
    sf[5, 4:8] = [11, 12, 13, 14]
    buf = oracle.swizzle_scales(sf)
    pos = np.nonzero(buf)[0]
    assert np.array_equal(buf[pos], [11, 12, 13, 14]) and np.array_equal(np.diff(pos), [1, 1, 1])
    assert pos[0] % 4 == 0
    # rows r and r + 32 of an atom, same block: 4 bytes apart
    sf2 = np.zeros((M, nkb), np.uint8)
    sf2[7, 1] = 1
    sf2[39, 1] = 2
    b2 = oracle.swizzle_scales(sf2)
    assert np.nonzero(b2 == 2)[0][0] - np.nonzero(b2 == 1)[0][0] == 4
