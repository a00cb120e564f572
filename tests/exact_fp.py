"""Exact rational model of binary32 round-to-nearest-even and of the NVFP4
element and scale encoders, for pinning the oracle's block arithmetic.

Independent of the oracle: everything here is Python ``fractions.Fraction``
arithmetic with the rounding rule written out (IEEE 754-2019 section 4.3.1,
roundTiesToEven, binary32 with subnormals) and the code tables of OCP MX v1.0
section 5.3.3 (E2M1) and the OCP 8-bit floating point specification (E4M3).
"""
from fractions import Fraction

HALF = Fraction(1, 2)

E2M1_MAG = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4),
            Fraction(6)]


def _e4m3_value(code: int) -> Fraction:
    e, m = (code >> 3) & 0xF, code & 7
    if e == 0:
        return Fraction(m, 8) * Fraction(1, 2 ** 6)
    return (1 + Fraction(m, 8)) * (Fraction(2) ** (e - 7))


E4M3_VAL = [_e4m3_value(c) for c in range(0x7F)]      # 0x7F is NaN


def rn32(v: Fraction) -> Fraction:
    """Nearest binary32 value to v, ties to the even significand (no overflow
    handling: callers stay in range)."""
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = -v if v < 0 else v
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)                                # subnormals share the quantum 2^-149
    quantum = Fraction(2) ** (e - 23)
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > HALF or (rem == HALF and fl % 2 == 1):
        fl += 1
    return sign * fl * quantum


def f32_bits_to_fraction(bits: int) -> Fraction:
    sign = -1 if bits >> 31 else 1
    e = (bits >> 23) & 0xFF
    m = bits & 0x7FFFFF
    assert e != 0xFF
    if e == 0:
        return sign * Fraction(m) * Fraction(2) ** -149
    return sign * Fraction(m | 0x800000) * Fraction(2) ** (e - 150)


def bf16_bits_to_fraction(bits: int) -> Fraction:
    return f32_bits_to_fraction(bits << 16)


def nearest_even(a: Fraction, table) -> int:
    """Index of the table value nearest to a >= 0, ties to the even index."""
    best, best_err = 0, abs(a - table[0])
    for i in range(1, len(table)):
        err = abs(a - table[i])
        if err < best_err or (err == best_err and i % 2 == 0 and best % 2 == 1):
            best, best_err = i, err
    return best


def e4m3_code(v: Fraction) -> int:
    return nearest_even(min(v, E4M3_VAL[0x7E]), E4M3_VAL)


def e2m1_code(y: Fraction, negative: bool) -> int:
    return (8 if negative else 0) | nearest_even(min(abs(y), Fraction(6)), E2M1_MAG)


def quantize_block_exact(x_bits, s_t_bits):
    """The NVFP4 block steps with one binary32 rounding per operation:
    v = fl(fl(a/6)/s_t), sf = E4M3(v), d = fl(sf s_t), q = E2M1(fl(x/d)),
    xhat = fl(e2m1(q) sf s_t), R = fl(x - xhat).
    x_bits: 16 bf16 bit patterns.  Returns (sf_code, codes, xhat, R) with
    xhat and R as Fractions."""
    s_t = f32_bits_to_fraction(s_t_bits)
    xs = [bf16_bits_to_fraction(b) for b in x_bits]
    neg = [bool(b & 0x8000) for b in x_bits]
    a = max(abs(x) for x in xs)
    v = rn32(rn32(a / 6) / s_t)
    sf_code = e4m3_code(v)
    sf = E4M3_VAL[sf_code]
    d = rn32(sf * s_t)
    codes, xhat, R = [], [], []
    for x, n in zip(xs, neg):
        y = rn32(x / d) if d != 0 else Fraction(0)
        q = e2m1_code(y, n)
        mag = E2M1_MAG[q & 7]
        xh = rn32((-mag if q & 8 else mag) * sf * s_t)
        codes.append(q)
        xhat.append(xh)
        R.append(rn32(x - xh))
    return sf_code, codes, xhat, R


def fp8_quantize_exact(x_bits, s_bits):
    """Per-tensor E4M3 quantization with one rounding per operation:
    q = E4M3(fl(x / s)) (sign of x), xhat = fl(e4m3(q) * s)."""
    s = f32_bits_to_fraction(s_bits)
    out = []
    for b in x_bits:
        x = bf16_bits_to_fraction(b)
        y = rn32(x / s)
        c = e4m3_code(abs(y)) | (0x80 if b & 0x8000 else 0)
        out.append((c, rn32((-1 if c & 0x80 else 1) * E4M3_VAL[c & 0x7F] * s)))
    return out


def quantize_block_exact_f32(x_f32_bits, s_t_bits):
    """quantize_block_exact for binary32 inputs (bit patterns)."""
    s_t = f32_bits_to_fraction(s_t_bits)
    xs = [f32_bits_to_fraction(b) for b in x_f32_bits]
    neg = [bool(b >> 31) for b in x_f32_bits]
    a = max(abs(x) for x in xs)
    v = rn32(rn32(a / 6) / s_t)
    sf_code = e4m3_code(v)
    sf = E4M3_VAL[sf_code]
    d = rn32(sf * s_t)
    codes, xhat = [], []
    for x, n in zip(xs, neg):
        y = rn32(x / d) if d != 0 else Fraction(0)
        q = e2m1_code(y, n)
        mag = E2M1_MAG[q & 7]
        codes.append(q)
        xhat.append(rn32((-mag if q & 8 else mag) * sf * s_t))
    return sf_code, codes, xhat
