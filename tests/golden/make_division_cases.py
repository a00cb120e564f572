"""Writes division_cases.txt: NVFP4 blocks on which the oracle's plain
binary32 evaluation of the block steps gives other codes or dequantized
values than the shortcuts an implementation might take:

  scale    E4M3(fl(fl(a/6)/s_t)) differs from E4M3(fl(a * fl(1/fl(6 s_t))))
           or from E4M3(fl(a / fl(6 s_t)));
  element  E2M1(fl(x/d)) differs from E2M1(fl(x * fl(1/d)));
  dequant  fl(e2m1 * sf * s_t) (one rounding) differs from fl(e2m1 * fl(sf * s_t)).

Candidates are searched with numpy binary32 arithmetic; every stored
expected value (scale code, element codes, dequantized values) is the
oracle's own output (oracle.quantize with the given s_t).  Run from the
repository root:  python tests/golden/make_division_cases.py
"""
import os
import sys

import numpy as np

os.environ.setdefault("OMP_NUM_THREADS", "1")     # the oracle is called on single values here

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402

F = np.float32
OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "division_cases.txt")
E4M3 = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
E2M1 = oracle.e2m1_decode(np.arange(16, dtype=np.uint8))


def bf16_of(v):
    return int(oracle.f32_to_bf16(np.array([v], F))[0])


def f32_of_bf16(b):
    return float(oracle.bf16_to_f32(np.array([b], np.uint16))[0])


def e4m3(v):
    return int(oracle.e4m3_encode(np.array([v], F))[0])


def e2m1(v):
    return int(oracle.e2m1_encode(np.array([v], F))[0])


def step(v, k):
    """v moved by k binary32 ulps."""
    b = np.array([v], F).view(np.uint32)[0].astype(np.int64) + k
    return np.array([b], np.uint32).view(F)[0]


def run_block(block_bits, s_t):
    x = np.array(block_bits, np.uint16).reshape(1, 16)
    q = oracle.quantize(x, s_t=float(s_t))
    codes = [int(q.codes[0, i // 2] >> (4 * (i % 2)) & 15) for i in range(16)]
    return int(q.sf[0, 0]), codes, q.xhat[0]


def filler(rng, amax, n):
    return [bf16_of(F(v)) for v in rng.uniform(-0.9, 0.9, n) * amax]


def scale_cases(rng, want):
    out = []
    while len(out) < want:
        a = F(f32_of_bf16(bf16_of(F(rng.uniform(0.5, 300.0)))))
        c = int(rng.integers(1, 0x7D))
        m = (E4M3[c] + E4M3[c + 1]) / 2
        s0 = F(float(a) / (6.0 * m))
        for k in range(-40, 41):
            s_t = step(s0, k)
            plain = e4m3(F(F(a / F(6)) / s_t))
            recip = e4m3(F(a * F(F(1) / F(F(6) * s_t))))
            div6 = e4m3(F(a / F(F(6) * s_t)))
            if plain != recip or plain != div6:
                block = [bf16_of(a)] + filler(rng, float(a), 15)
                sf, codes, xh = run_block(block, s_t)
                assert sf == plain
                out.append(("scale", s_t, block, sf, codes, xh))
                break
    return out


def element_cases(rng, want):
    out = []
    thresholds = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    while len(out) < want:
        c = int(rng.integers(0x10, 0x70))
        t = thresholds[int(rng.integers(0, len(thresholds)))]
        s_base = F(2.0 ** rng.uniform(-12, 4))
        d0 = F(F(E4M3[c]) * s_base)
        xb = bf16_of(F(t * float(d0)))
        x = F(f32_of_bf16(xb))
        found = False
        for k in range(-64, 65):
            s_t = step(s_base, k)
            d = F(F(E4M3[c]) * s_t)
            if e2m1(F(x / d)) == e2m1(F(x * F(F(1) / d))):
                continue
            # a block whose maximum gives scale code c under this s_t
            a = None
            for frac in (0.999, 0.995, 0.99, 0.98, 1.0, 1.001):
                ab = bf16_of(F(6.0 * E4M3[c] * float(s_t) * frac))
                if e4m3(F(F(F(f32_of_bf16(ab)) / F(6)) / s_t)) == c and f32_of_bf16(ab) >= abs(float(x)):
                    a = ab
                    break
            if a is None:
                continue
            block = [xb, a] + filler(rng, f32_of_bf16(a), 14)
            sf, codes, xh = run_block(block, s_t)
            assert sf == c
            out.append(("element", s_t, block, sf, codes, xh))
            found = True
            break
        del found
    return out


def dequant_cases(rng, want):
    out = []
    while len(out) < want:
        s_t = F(2.0 ** rng.uniform(-10, 2))
        block = [bf16_of(F(v)) for v in rng.standard_normal(16) * float(s_t) * 500]
        sf, codes, xh = run_block(block, s_t)
        d = F(F(E4M3[sf]) * s_t)
        alt = np.array([F(F(E2M1[q]) * d) for q in codes], F)
        if not np.array_equal(alt, xh):
            out.append(("dequant", s_t, block, sf, codes, xh))
    return out


def main():
    rng = np.random.default_rng(20260720)
    cases = scale_cases(rng, 12) + element_cases(rng, 24) + dequant_cases(rng, 8)
    with open(OUT, "w") as f:
        f.write("# NVFP4 blocks that tell the plain binary32 block arithmetic apart from\n"
                "# reciprocal-multiply and double-rounding shortcuts (see make_division_cases.py,\n"
                "# which wrote this file from oracle.quantize).  One block per line:\n"
                "# kind s_t(f32 hex) x0..x15(bf16 hex) sf_code codes(16 hex digits, element 0 first)\n"
                "#   xhat0..xhat15(f32 hex)\n")
        for kind, s_t, block, sf, codes, xh in cases:
            s_hex = "%08x" % np.array([s_t], F).view(np.uint32)[0]
            xs = " ".join("%04x" % b for b in block)
            cs = "".join("%x" % q for q in codes)
            xhs = " ".join("%08x" % u for u in np.asarray(xh, F).view(np.uint32))
            f.write(f"{kind} {s_hex} {xs} {sf:02x} {cs} {xhs}\n")
    print(f"wrote {len(cases)} cases to {OUT}")


if __name__ == "__main__":
    main()
