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

// Per-tensor scale from the tensor's max |x|: s_t = A / 2688, 1 if A == 0.
__device__ __forceinline__ float tensor_scale_from_amax(float A)
{
    return A == 0.0f ? 1.0f : __fdiv_rn(A, 2688.0f);
}

// Block scale factor pieces shared by every quantizing kernel.
struct BlockScale {
    uint32_t sf_code;  // E4M3 code
    float d;           // block dequantization scale fl(sf * s_t)
    float rcp;         // fl(1 / d), 0 when d == 0
};

__device__ __forceinline__ BlockScale block_scale(float amax_b, float s_t, float r6)
{
    BlockScale b;
    b.sf_code = cvt_e4m3(__fmul_rn(amax_b, r6));
    float sf = e4m3_to_f32(b.sf_code);
    b.d = __fmul_rn(sf, s_t);
    b.rcp = (b.d == 0.0f) ? 0.0f : __frcp_rn(b.d);
    return b;
}

// r6 = fl(1 / fl(6 * s_t)), the per-tensor factor mapping a block max to its
// E4M3 scale value.
__device__ __forceinline__ float block_r6(float s_t) { return __frcp_rn(__fmul_rn(6.0f, s_t)); }

// Quantize 8 consecutive elements (one lane's half of a 16-block whose other
// half is held by lane ^ 1) given the block scale.  Returns 4 code bytes
// (little-endian element order) and the dequantized values.
__device__ __forceinline__ uint32_t quant8(const float v[8], const BlockScale &b, float xh[8])
{
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = __fmul_rn(v[i], b.rcp);
    uint32_t w = cvt_e2m1x8(y);
    float q[8];
    e2m1x8_to_f32(w, q);
#pragma unroll
    for (int i = 0; i < 8; ++i) xh[i] = __fmul_rn(q[i], b.d);
    return w;
}

// Dequantized value of a single element given its block scale.
__device__ __forceinline__ float quant1_xhat(float v, const BlockScale &b)
{
    uint32_t byte = cvt_e2m1x2(__fmul_rn(v, b.rcp), 0.0f);
    float2 q = e2m1x2_to_f32(byte);
    return __fmul_rn(q.x, b.d);
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
