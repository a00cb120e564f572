// common.cuh -- shared host/device helpers of the NVFP4 QUADS library.
//
// Device side: the NVFP4 block arithmetic (one definition used by every kernel
// that quantizes, so that codes, scales and residuals agree bit for bit
// between kernels) built on the sm_100a conversion instructions
// cvt.rn.satfinite.{e2m1x2,e4m3x2}.f32 and their widening inverses, and on
// IEEE round-to-nearest intrinsics (__fmul_rn, __frcp_rn, __fdiv_rn) so the
// compiler cannot contract or reassociate the quantization arithmetic.
//
// Host side: error strings, argument checks, launch checks.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <stdio.h>
#include <stdarg.h>

#include "../../include/nvfp4_quads.h"

namespace nvfp4 {

// ----------------------------------------------------------------- host side

nvfp4_status set_error(nvfp4_status st, const char *fmt, ...);
nvfp4_status check_launch(const char *what);
int num_sms();

// Row-major 2D tensor [rows x inner] (row stride row_bytes) with a
// (box_inner x box_rows) TMA box; false if the driver rejects it.
bool make_tmap_2d(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint64_t inner, uint64_t rows,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle);

#define NVFP4_REQUIRE(cond, status, ...)                 \
    do {                                                 \
        if (!(cond)) return ::nvfp4::set_error(status, __VA_ARGS__); \
    } while (0)

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Byte offset of scale entry (row r, scale column c) in the tensor-core
// scale-factor layout (128-row x 4-column atoms of 512 bytes).
__host__ __device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t c, int64_t K)
{
    return ((r >> 7) * (K >> 6) + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

__host__ __device__ __forceinline__ int64_t sf_bytes(int64_t rows, int64_t K) { return ((rows + 127) / 128) * 128 * (K / 16); }

// ----------------------------------------------------------------- device side

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two floats -> one byte of two E2M1 codes: `lo` in bits 0..3, `hi` in 4..7.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi)
{
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "mov.b32 %0, {t, t, t, t};\n\t}"
        : "=r"(r) : "f"(hi), "f"(lo));
    return r & 0xFFu;
}

// Eight floats -> four bytes of E2M1 codes, element 2i in the low nibble of
// byte i.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float y[8])
{
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
    return r;
}

// One byte of two E2M1 codes -> the two values as floats (exact).
__device__ __forceinline__ float2 e2m1x2_to_f32(uint32_t byte)
{
    uint32_t h2;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t}"
        : "=r"(h2) : "r"(byte));
    return __half22float2(*reinterpret_cast<__half2 *>(&h2));   // .x = bits 0..3
}

// Four bytes of E2M1 codes -> eight exact values (element 2i = low nibble of
// byte i).  Each byte is converted from the low byte of its own register.
__device__ __forceinline__ void e2m1x8_to_f32(uint32_t w, float v[8])
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = e2m1x2_to_f32((w >> (8 * i)) & 0xFFu);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

// Non-negative float -> E4M3 code (nearest even, saturating at 448).
__device__ __forceinline__ uint32_t cvt_e4m3(float v)
{
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\t"
        "cvt.u32.u16 %0, t;\n\t}"
        : "=r"(r) : "f"(0.0f), "f"(v));
    return r & 0xFFu;
}

// Two non-negative floats -> their E4M3 codes: `lo` in bits 0..7, `hi` in 8..15.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi)
{
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\t"
        "cvt.u32.u16 %0, t;\n\t}"
        : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// E4M3 code -> value (exact in f16 and f32).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code)
{
    uint32_t h2;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "mov.b32 {lo, hi}, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t}"
        : "=r"(h2) : "r"(code & 0xFFu));
    return __low2float(*reinterpret_cast<__half2 *>(&h2));
}

// E4M3 code -> the value in both halves of an f16x2 (exact).
__device__ __forceinline__ uint32_t e4m3_to_h2(uint32_t code)
{
    uint32_t h2;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "mov.b32 {lo, hi}, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t}"
        : "=r"(h2) : "r"((code & 0xFFu) * 0x101u));
    return h2;
}

// Per-tensor scale from the tensor's max |x|: s_t = A / 2688, 1 if A == 0.
__device__ __forceinline__ float tensor_scale_from_amax(float A)
{
    return A == 0.0f ? 1.0f : __fdiv_rn(A, 2688.0f);
}

// ------------------------------------------------------- NVFP4 block steps
//
// Definitions (binary32, one rounding per operation):
//   block scale   sf = E4M3(fl(fl(a/6) / s_t)), a = max |x| over the block
//   element code  q  = E2M1(fl(x / d)), d = fl(sf * s_t)
//   dequantized   xhat = fl(e2m1(q) * sf * s_t)   (e2m1 * sf is exact)
//   residual      R = fl(x - xhat)
//
// Both encodings are monotone in their (real) argument, so a decision can be
// taken from two multiplications that bracket the exact quotient: with
// lo = fl(fl(1/den) * (1 - 2^-20)) and hi = fl(fl(1/den) * (1 + 2^-20)),
//   num * lo < num / den * (1 - 2^-21) and num * hi > num / den * (1 + 2^-21),
// which encloses every value within a few binary32 roundings of num / den
// (a rounded reciprocal and product move a value by at most 2^-23 relative;
// fl(fl(a/6) / s_t) by at most 2^-23 from a / (6 s_t)).  Rounding to binary32
// is monotone, so fl(num * lo) <= fl(num / den) <= fl(num * hi); when the two
// brackets encode to the same code, that is the code of the exact-division
// definition.  Otherwise (an argument within about 2^-20 of a rounding
// boundary: a few per million elements) the IEEE divisions are evaluated.

// Bracketing multipliers (lo, hi) around 1/den.
__device__ __forceinline__ float2 recip_bracket(float den)
{
    const float r = __frcp_rn(den);
    // 1/den above the binary32 range (den below 2^-128): the pair (0, inf)
    // never encodes to one code for a non-zero argument, so every decision
    // then takes the division
    if (!(r < INFINITY)) return make_float2(0.0f, INFINITY);
    return make_float2(__fmul_rn(r, 1.0f - 0x1p-20f), __fmul_rn(r, 1.0f + 0x1p-20f));
}

// E4M3 code of the block scale fl(fl(a/6) / s_t), a >= 0; r6 = bracket of
// 1/(6 s_t) (recip_bracket(fl(6 s_t)) encloses it: fl(6 s_t) is within 2^-24).
// The division fallbacks are rare (arguments within ~2^-20 of a rounding
// boundary) and kept out of line, so the streaming loops stay small.
static __device__ __noinline__ uint32_t block_scale_code_div(float a, float s_t)
{
    return cvt_e4m3(__fdiv_rn(__fdiv_rn(a, 6.0f), s_t));
}

__device__ __forceinline__ uint32_t block_scale_code(float a, float s_t, float2 r6)
{
    const uint32_t c2 = cvt_e4m3x2(__fmul_rn(a, r6.x), __fmul_rn(a, r6.y));
    const uint32_t c = c2 & 0xFFu;
    if ((c2 >> 8) == c) return c;
    return block_scale_code_div(a, s_t);
}

// Per E4M3 scale code, the per-tensor quantities of a block: its scale
// d = fl(sf * s_t), the bracket of 1/d (both 0 when d == 0: every element
// then maps to a signed zero), and sf in both halves of an f16x2.
struct BlockConst {
    float d, rlo, rhi;
    uint32_t sf_h2;
};

__device__ __forceinline__ BlockConst block_const(uint32_t code, float s_t)
{
    BlockConst b;
    b.d = __fmul_rn(e4m3_to_f32(code), s_t);
    if (b.d == 0.0f) {
        b.rlo = b.rhi = 0.0f;
    } else {
        const float2 r = recip_bracket(b.d);
        b.rlo = r.x;
        b.rhi = r.y;
    }
    b.sf_h2 = e4m3_to_h2(code);
    return b;
}

// Packed binary32 pairs (sm_100a f32x2 arithmetic, round to nearest even).
__device__ __forceinline__ float2 mul2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 a, b, d;\n\t"
        "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "mul.rn.f32x2 d, a, b;\n\t"
        "mov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{\n\t.reg .b64 a, b, c, d;\n\t"
        "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %7};\n\t"
        "fma.rn.f32x2 d, a, b, c;\n\t"
        "mov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// One bf16x2 word -> its two values as a float pair (exact): .x = low half.
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w)
{
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// E2M1 codes of 8 elements by IEEE division (the out-of-line fallback).
static __device__ __noinline__ uint32_t element_codes8_div(float2 v0, float2 v1, float2 v2, float2 v3, float d)
{
    const float y[8] = {__fdiv_rn(v0.x, d), __fdiv_rn(v0.y, d), __fdiv_rn(v1.x, d), __fdiv_rn(v1.y, d),
                        __fdiv_rn(v2.x, d), __fdiv_rn(v2.y, d), __fdiv_rn(v3.x, d), __fdiv_rn(v3.y, d)};
    return cvt_e2m1x8(y);
}

// E2M1 codes of 8 elements (one lane's half of a 16-block; 4 bytes, element
// 2i in the low nibble of byte i) given the block's constants.
__device__ __forceinline__ uint32_t element_codes8(const float2 v[4], const BlockConst &b)
{
    float ylo[8], yhi[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 lo = mul2(v[i], make_float2(b.rlo, b.rlo));
        const float2 hi = mul2(v[i], make_float2(b.rhi, b.rhi));
        ylo[2 * i] = lo.x; ylo[2 * i + 1] = lo.y;
        yhi[2 * i] = hi.x; yhi[2 * i + 1] = hi.y;
    }
    const uint32_t wlo = cvt_e2m1x8(ylo);
    if (wlo == cvt_e2m1x8(yhi)) return wlo;
    return element_codes8_div(v[0], v[1], v[2], v[3], b.d);
}

// Dequantized values of 8 elements from their codes: pairs
// xhat = fl(fl(e2m1 * sf) * s_t), the e2m1 * sf products exact in f16.  The
// final multiply is scalar mul.rn.f32: the code generator fuses a packed
// f32x2 multiply with a following packed subtraction into one fused
// multiply-add, which would skip the rounding of xhat the residual depends on.
__device__ __forceinline__ void dequant8(uint32_t w, uint32_t sf_h2, float s_t, float2 xh[4])
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t q2;
        asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
            "mov.b32 {b0, b1, b2, b3}, %1;\n\t"
            "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t}"
            : "=r"(q2) : "r"(w >> (8 * i)));
        uint32_t p2;
        asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(p2) : "r"(q2), "r"(sf_h2));
        const float2 qsf = __half22float2(*reinterpret_cast<__half2 *>(&p2));
        xh[i] = make_float2(__fmul_rn(qsf.x, s_t), __fmul_rn(qsf.y, s_t));
    }
}

// Residuals R = fl(x - xhat) of 8 elements (scalar sub.rn.f32, see dequant8).
__device__ __forceinline__ void residual8(const float2 v[4], const float2 xh[4], float2 R[4])
{
#pragma unroll
    for (int i = 0; i < 4; ++i) R[i] = make_float2(__fsub_rn(v[i].x, xh[i].x), __fsub_rn(v[i].y, xh[i].y));
}

static __device__ __noinline__ uint32_t element_code1_div(float v, float d)
{
    return cvt_e2m1x2(__fdiv_rn(v, d), 0.0f) & 15u;
}

// Dequantized value fl(fl(e2m1(q) * sf) * s_t) of a single element.
__device__ __forceinline__ float element_xhat1(float v, const BlockConst &b, float s_t)
{
    const uint32_t c2 = cvt_e2m1x2(__fmul_rn(v, b.rlo), __fmul_rn(v, b.rhi));
    uint32_t q = c2 & 15u;
    if ((c2 >> 4) != q) q = element_code1_div(v, b.d);
    const float sf = __low2float(*reinterpret_cast<const __half2 *>(&b.sf_h2));
    return __fmul_rn(__fmul_rn(e2m1x2_to_f32(q).x, sf), s_t);
}

// Status word helpers.
__device__ __forceinline__ void report_status(int32_t *dev_status, int32_t st)
{
    if (dev_status) atomicCAS(dev_status, 0, st);
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

}  // namespace nvfp4
