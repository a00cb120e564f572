"""CPU oracle for the QUADS rollout hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never imports,
links or calls it, and it imports nothing from the product package: the two
share no kernels, headers, helpers, tables or constant generators.

Element-wise and block-wise quantization arithmetic lives in plain C
(``nvfp4_oracle.c``, built to ``liboracle.so`` with ``-ffp-contract=off``);
this module adds the layout transforms and the dense algebra (routing glue,
matrix products in binary64, SiLU) on numpy.  Every function cites the passage
of the QUADS pages it follows; readings of what the pages leave open are
marked READING.

Pins (tests/test_oracle_*.py): exhaustive nearest-value checks of the E2M1 and
E4M3 encoders, the format tables in tests/golden/, an exact rational
re-derivation of the block arithmetic (including stored cases where a
reciprocal-multiply or double-rounded variant would give other codes),
closed forms (block maximum maps to +-6, |R| <= d, all-zero tensors),
selection against a full sort, routing against a sort-based top-k, the
matrix products against brute force loops on tiny shapes plus special-case
reductions, and structural pins of the scale-factor byte layout (a bijection
onto the padded buffer with an exact inverse, zero padding rows, one 32-bit
word per row and 64-element group).  The exact byte positions of that layout
are pinned on the GPU, where the tensor-core GEMM consumes it and matches the
brute-force dense product.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None

F32P = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
F64P = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
U8P = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
U16P = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
I32P = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile the C part of the oracle (gcc, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp%d" % os.getpid()
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
            "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        lib.oracle_e2m1_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e2m1_decode.restype = ctypes.c_double
        lib.oracle_e2m1_encode_array.argtypes = [F32P, U8P, I64]
        lib.oracle_e4m3_encode_array.argtypes = [F32P, U8P, I64]
        lib.oracle_e4m3_decode_array.argtypes = [U8P, F64P, I64]
        lib.oracle_e2m1_decode_array.argtypes = [U8P, F64P, I64]
        lib.oracle_bf16_from_f32_array.argtypes = [F32P, U16P, I64]
        lib.oracle_amax.argtypes = [U16P, I64, I64, I64]
        lib.oracle_amax.restype = ctypes.c_float
        lib.oracle_tensor_scale_from_amax.argtypes = [ctypes.c_float]
        lib.oracle_tensor_scale_from_amax.restype = ctypes.c_float
        lib.oracle_quantize.argtypes = [U16P, I64, I64, I64, ctypes.c_float,
                                        ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_channel_score.argtypes = [F32P, I64, I64, ctypes.c_void_p, F64P]
        lib.oracle_select_topk.argtypes = [F64P, I64, I64, I32P]
        lib.oracle_rac_residual.argtypes = [F32P, I64, I64, ctypes.c_float, I32P, I64, U16P]
        lib.oracle_route.argtypes = [F32P, I64, I64, I64, I32P, F64P]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_quantize_f32.argtypes = [F32P, I64, I64, I64, ctypes.c_float,
                                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_fp8_scale_from_amax.argtypes = [ctypes.c_float]
        lib.oracle_fp8_scale_from_amax.restype = ctypes.c_float
        lib.oracle_fp8_quantize.argtypes = [U16P, I64, I64, I64, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    """OpenMP threads the C part runs with."""
    return int(_L().oracle_num_threads())


# --------------------------------------------------------------- formats

def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> binary32 values (exact)."""
    return (np.ascontiguousarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(f: np.ndarray) -> np.ndarray:
    """binary32 -> nearest bfloat16 bit pattern, ties to even."""
    f = np.ascontiguousarray(f, np.float32)
    out = np.empty(f.shape, np.uint16)
    _L().oracle_bf16_from_f32_array(f.reshape(-1), out.reshape(-1), f.size)
    return out


def e2m1_encode(y: np.ndarray) -> np.ndarray:
    """Nearest E2M1 code (ties to even, saturating at 6, sign bit of y)."""
    y = np.ascontiguousarray(y, np.float32)
    q = np.empty(y.shape, np.uint8)
    _L().oracle_e2m1_encode_array(y.reshape(-1), q.reshape(-1), y.size)
    return q


def e2m1_decode(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, np.uint8)
    v = np.empty(q.shape, np.float64)
    _L().oracle_e2m1_decode_array(q.reshape(-1), v.reshape(-1), q.size)
    return v


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Nearest non-negative finite E4M3 code (ties to even, saturating at 448)."""
    v = np.ascontiguousarray(v, np.float32)
    q = np.empty(v.shape, np.uint8)
    _L().oracle_e4m3_encode_array(v.reshape(-1), q.reshape(-1), v.size)
    return q


def e4m3_decode(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, np.uint8)
    v = np.empty(q.shape, np.float64)
    _L().oracle_e4m3_decode_array(q.reshape(-1), v.reshape(-1), q.size)
    return v


# ------------------------------------------------------- quantization

def amax(x: np.ndarray) -> float:
    """max |x| over a bf16 (uint16) matrix."""
    x = np.ascontiguousarray(x, np.uint16)
    if x.size == 0:
        return 0.0
    return float(_L().oracle_amax(x, x.shape[0], x.shape[1], x.shape[1]))


def tensor_scale(A: float) -> float:
    """s_t = A / 2688 in binary32, 1 when A == 0 (READING, see nvfp4_oracle.c)."""
    return float(_L().oracle_tensor_scale_from_amax(ctypes.c_float(A)))


class Quantized:
    """Result of :func:`quantize` (row-major, unswizzled)."""

    def __init__(self, codes, sf, xhat, resid, s_t):
        self.codes = codes      # uint8 [M, K/2]
        self.sf = sf            # uint8 [M, K/16] E4M3 codes
        self.xhat = xhat        # float32 [M, K]
        self.resid = resid      # float32 [M, K]
        self.s_t = s_t          # float


def quantize(x: np.ndarray, s_t: float | None = None) -> Quantized:
    """NVFP4 quantization of a bf16 matrix (QUADS, gist.science/it 2.1: online
    activation quantization onto the coarse E2M1 grid).  ``s_t`` defaults to
    the tensor's own scale."""
    x = np.ascontiguousarray(x, np.uint16)
    M, K = x.shape
    assert K % 16 == 0
    if s_t is None:
        s_t = tensor_scale(amax(x))
    codes = np.empty((M, K // 2), np.uint8)
    sf = np.empty((M, K // 16), np.uint8)
    xhat = np.empty((M, K), np.float32)
    resid = np.empty((M, K), np.float32)
    if M:
        _L().oracle_quantize(x, M, K, K, ctypes.c_float(s_t), _ptr(codes), _ptr(sf),
                             _ptr(xhat), _ptr(resid))
    return Quantized(codes, sf, xhat, resid, float(np.float32(s_t)))


def dequantize(codes: np.ndarray, sf: np.ndarray, s_t: float) -> np.ndarray:
    """xhat = fl(e2m1(q) * sf * s_t) in binary32 from packed codes and
    row-major scale codes (e2m1 * sf is exact, so one rounding)."""
    M = codes.shape[0]
    K = codes.shape[1] * 2
    q = np.empty((M, K), np.uint8)
    q[:, 0::2] = codes & 0xF
    q[:, 1::2] = codes >> 4
    sfv = np.repeat(e4m3_decode(sf).astype(np.float32), 16, axis=1)
    qsf = (e2m1_decode(q).astype(np.float32) * sfv).astype(np.float32)
    return (qsf * np.float32(s_t)).astype(np.float32)


def swizzle_scales(sf: np.ndarray, m_pad: int | None = None) -> np.ndarray:
    """Scale codes [M, K/16] -> the tensor-core scale-factor layout: 512-byte
    atoms of 128 rows x 4 scale columns, atom (rb, cb) at (rb*(K/64) + cb)*512,
    row r / column c of the atom at byte (r%32)*16 + (r//32)*4 + c (PTX ISA,
    tcgen05 block-scaled MMA scale-factor layout).  Rows past M are zero."""
    M, nkb = sf.shape
    assert nkb % 4 == 0
    m_pad = m_pad if m_pad is not None else -(-M // 128) * 128
    out = np.zeros((m_pad // 128) * (nkb // 4) * 512, np.uint8)
    r = np.arange(M)[:, None]
    c = np.arange(nkb)[None, :]
    off = ((r // 128) * (nkb // 4) + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
    out[off] = sf
    return out


def unswizzle_scales(buf: np.ndarray, M: int, K: int) -> np.ndarray:
    """Inverse of :func:`swizzle_scales` for the first M rows."""
    nkb = K // 16
    r = np.arange(M)[:, None]
    c = np.arange(nkb)[None, :]
    off = ((r // 128) * (nkb // 4) + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
    return np.asarray(buf).reshape(-1)[off]


def channel_score(resid: np.ndarray, row_valid: np.ndarray | None = None) -> np.ndarray:
    """score[c] = sum_r R[r,c]^2 in binary64 (READING of "residual magnitude",
    gist.science/it 2.2 B).  Rows with row_valid < 0 are skipped."""
    resid = np.ascontiguousarray(resid, np.float32)
    M, K = resid.shape
    score = np.empty(K, np.float64)
    rv = None if row_valid is None else np.ascontiguousarray(row_valid, np.int32)
    _L().oracle_channel_score(resid, M, K, _ptr(rv), score)
    return score


def select_topk(score: np.ndarray, k: int) -> np.ndarray:
    """Binary top-k channel mask as an ascending index set (gist.science/it
    2.2 B); equal scores prefer the lower channel index."""
    score = np.ascontiguousarray(score, np.float64)
    assert 0 <= k <= score.size
    S = np.empty(k, np.int32)
    _L().oracle_select_topk(score, score.size, k, S)
    return S


def rac_residual(resid: np.ndarray, s_t: float, S: np.ndarray, k_pad: int | None = None) -> np.ndarray:
    """rho[r, j] = bf16(fl(R[r, S_j] / s_t)); columns past len(S) are zero."""
    resid = np.ascontiguousarray(resid, np.float32)
    S = np.ascontiguousarray(S, np.int32)
    M, K = resid.shape
    k = S.size
    rho = np.empty((M, k), np.uint16)
    if M and k:
        _L().oracle_rac_residual(resid, M, K, ctypes.c_float(s_t), S, k, rho)
    if k_pad is not None and k_pad > k:
        rho = np.concatenate([rho, np.zeros((M, k_pad - k), np.uint16)], axis=1)
    return rho


def quantize_f32(x: np.ndarray, s_t: float | None = None) -> Quantized:
    """NVFP4 quantization of a binary32 matrix with the block steps of
    quantize(); s_t defaults to max|x| / 2688."""
    x = np.ascontiguousarray(x, np.float32)
    M, K = x.shape
    assert K % 16 == 0
    if s_t is None:
        s_t = tensor_scale(float(np.abs(x).max()) if x.size else 0.0)
    codes = np.empty((M, K // 2), np.uint8)
    sf = np.empty((M, K // 16), np.uint8)
    xhat = np.empty((M, K), np.float32)
    resid = np.empty((M, K), np.float32)
    if M:
        _L().oracle_quantize_f32(x, M, K, K, ctypes.c_float(s_t), _ptr(codes), _ptr(sf), _ptr(xhat), _ptr(resid))
    return Quantized(codes, sf, xhat, resid, float(np.float32(s_t)))


def rac_residual_nvfp4(resid: np.ndarray, s_t: float, S: np.ndarray, k_pad: int | None = None):
    """RAC with the "second pass of quantization" of the selected channels
    (gist.science/it 2.2 B): the residual R[:, S] (binary32, channels in
    ascending order) is quantized again to NVFP4 as one [M x k] tensor with
    its own tensor scale s_r = max|R_S| / 2688 and 16-element blocks along the
    selected channels (a last partial block zero-padded); the correction uses
    its dequantized value rhat, carried like the plain residual:
    rho2[r, j] = bf16(fl(rhat[r, j] / s_t)).  READING: the pages name the
    second pass but not its format; the block steps are those of quantize().
    Returns (rho2 bf16 bits [M, k or k_pad], s_r)."""
    resid = np.ascontiguousarray(resid, np.float32)
    S = np.ascontiguousarray(S, np.int32)
    M, k = resid.shape[0], S.size
    kb = -(-k // 16) * 16
    RS = np.zeros((M, kb), np.float32)
    RS[:, :k] = resid[:, S]
    A = float(np.abs(RS).max()) if RS.size else 0.0
    q = quantize_f32(RS, tensor_scale(A)) if M and kb else None
    rhat = q.xhat[:, :k] if q is not None else np.zeros((M, k), np.float32)
    rho = f32_to_bf16((rhat / np.float32(s_t)).astype(np.float32)) if k else np.zeros((M, 0), np.uint16)
    if k_pad is not None and k_pad > k:
        rho = np.concatenate([rho, np.zeros((M, k_pad - k), np.uint16)], axis=1)
    return rho, (q.s_t if q is not None else 1.0)


def qdq(w: np.ndarray):
    """Trainer-side weight fake-quantization (gist.science/it 2.2 A, W4A16):
    bf16 -> NVFP4 with the tensor's own scale -> bf16(xhat).  Returns
    (bf16 bits, s_t, Quantized)."""
    qz = quantize(w)
    return f32_to_bf16(qz.xhat), qz.s_t, qz


# ------------------------------------------------------------ routing

def route(logits: np.ndarray, kr: int):
    """Top-k_r experts per token by logit (equal logits prefer the lower
    expert index), descending; gate = softmax over the selected logits in
    binary64."""
    logits = np.ascontiguousarray(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, kr), np.int32)
    gate = np.empty((T, kr), np.float64)
    if T:
        _L().oracle_route(logits, T, E, kr, idx, gate)
    return idx, gate


# ------------------------------------------------------------- products

def w4a4_rac_matmul(xhat: np.ndarray, s_a: float, rho: np.ndarray | None, S: np.ndarray | None,
                    what: np.ndarray) -> np.ndarray:
    """Y = Xhat Wq^T + (s_a rho) Wq[:, S]^T in binary64.

    The first term is the native W4A4 product of the dequantized operands; the
    second is Residual Activation Compensation on the selected channels
    (gist.science/it 2.2 B: the correction is added back to the quantized
    output, the bulk stays on the W4A4 GEMM).  READING: the correction
    multiplies the dequantized NVFP4 weight, the only weight the rollout
    engine holds.  ``what`` is [N, K] (output features x input channels)."""
    Y = xhat.astype(np.float64) @ what.astype(np.float64).T
    if rho is not None and S is not None and len(S):
        r = bf16_to_f32(rho[:, :len(S)]).astype(np.float64) * float(s_a)
        Y += r @ what[:, S].astype(np.float64).T
    return Y


def fp8_quantize(x: np.ndarray, s: float | None = None):
    """Per-tensor FP8 E4M3 quantization of a bf16 matrix (the FP8 rollout the
    pages compare NVFP4 against, gist.science/it sections 1 and 4; READING:
    s = max|x| / 448, q = E4M3(fl(x / s)), xhat = fl(e4m3(q) * s)).
    Returns (codes uint8 [M, K] with the sign in bit 7, xhat float32, s)."""
    x = np.ascontiguousarray(x, np.uint16)
    M, K = x.shape
    if s is None:
        s = float(_L().oracle_fp8_scale_from_amax(ctypes.c_float(amax(x))))
    codes = np.empty((M, K), np.uint8)
    xhat = np.empty((M, K), np.float32)
    if M:
        _L().oracle_fp8_quantize(x, M, K, K, ctypes.c_float(s), _ptr(codes), _ptr(xhat))
    return codes, xhat, float(np.float32(s))


def silu(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, np.float64)
    return z / (1.0 + np.exp(-z))


def swiglu(y: np.ndarray, inter: int) -> np.ndarray:
    """h = silu(gate) * up with gate = columns [0, I), up = columns [I, 2I)
    (READING: gate and up stacked in one [2I x H] weight)."""
    return silu(y[:, :inter]) * y[:, inter:2 * inter]
