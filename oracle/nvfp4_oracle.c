/*
 * nvfp4_oracle.c -- plain, slow CPU oracle for the QUADS rollout hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes
 * or calls this file; only tests/, the smoke check and the CPU-baseline leg of
 * bench.py load it (through oracle/__init__.py).  It shares no code, header,
 * table or constant generator with the CUDA path.
 *
 * Sources (page, section):
 *   - "coarse E2M1 grid" with "fine-grained scaling": QUADS abstract
 *     (shd-paper.top, original English abstract) and gist.science/it, section 1.
 *   - online activation quantization is the dominant error source:
 *     gist.science/it, section 2.1 ("Attivazioni").
 *   - Residual Activation Compensation: channels with the largest FP4
 *     quantization residual are selected by a binary top-k channel mask and a
 *     residual correction is added back: gist.science/it, section 2.2 B.
 *   - trainer-side weight fake-quantization (QDQ, W4A16):
 *     gist.science/it, section 2.2 A.
 *   The NVFP4 bit format itself (E2M1 elements on {0,.5,1,1.5,2,3,4,6}, one
 *   unsigned E4M3 scale per 16 consecutive elements, one FP32 scale per
 *   tensor) is the OCP Microscaling / NVIDIA NVFP4 format; the pages only name
 *   it.  Readings of steps the pages leave open are marked READING below.
 *
 * Arithmetic: IEEE binary32 round-to-nearest-even for every quantization
 * decision (compiled with -ffp-contract=off, no fast-math), binary64 for
 * accumulations.  Encoders are brute-force "nearest representable value,
 * ties to the even code" searches over the format's code table, so that a
 * reader can check them against the format definition by eye.
 *
 * Pins: tests/test_oracle_*.py check these functions against exhaustive
 * nearest-value properties, the format tables in tests/golden/, closed forms
 * (block max -> code 6, |R| <= d, all-zero tensors) and brute force.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ bf16 */

float oracle_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a finite binary32 value to the nearest bfloat16, ties to even. */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lower = u & 0xFFFFu;
    uint32_t upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))
        upper += 1u;
    return (uint16_t)upper;
}

/* ------------------------------------------------------------------ E2M1 */

/* E2M1 magnitudes indexed by the 3 low code bits (exponent:2, mantissa:1,
 * bias 1; index 1 is the subnormal 0.5). */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_decode(uint8_t code)
{
    double m = E2M1_MAG[code & 7u];
    return (code & 8u) ? -m : m;
}

/* Nearest E2M1 value to y, ties to the even code, saturating at +-6; the
 * sign bit follows the sign of y (so a negative value that rounds to zero
 * gives code 0x8).  READING: the pages fix no rounding mode; round to nearest
 * even with saturation is the IEEE default the format inherits. */
uint8_t oracle_e2m1_encode(float y)
{
    double a = fabs((double)y);
    if (a > 6.0) a = 6.0;                          /* saturate before the search */
    int best = 0;
    double best_err = fabs(a - E2M1_MAG[0]);
    for (int i = 1; i < 8; ++i) {
        double err = fabs(a - E2M1_MAG[i]);
        if (err < best_err || (err == best_err && (i & 1) == 0 && (best & 1) == 1)) {
            best = i;
            best_err = err;
        }
    }
    return (uint8_t)((signbit(y) ? 8 : 0) | best);
}

/* ------------------------------------------------------------------ E4M3 */

/* Unsigned use of FP8 E4M3 (sign 1, exponent 4 with bias 7, mantissa 3, no
 * infinities, 0x7F/0xFF are NaN): codes 0x00..0x7E are the non-negative
 * finite values, largest 448, smallest subnormal 2^-9. */
double oracle_e4m3_decode(uint8_t code)
{
    int e = (code >> 3) & 0xF;
    int m = code & 7;
    double v;
    if (e == 0)
        v = ldexp((double)m, -9);                 /* m/8 * 2^-6 */
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return (code & 0x80) ? -v : v;
}

/* Nearest non-negative finite E4M3 value to v >= 0, ties to the even code,
 * values above 448 saturate to 448 (code 0x7E). */
uint8_t oracle_e4m3_encode(float v)
{
    double a = (double)v;
    if (a > 448.0) a = 448.0;                      /* saturate before the search */
    int best = 0;
    double best_err = fabs(a - oracle_e4m3_decode(0));
    for (int c = 1; c <= 0x7E; ++c) {
        double err = fabs(a - oracle_e4m3_decode((uint8_t)c));
        if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_err = err;
        }
    }
    return (uint8_t)best;
}

/* ------------------------------------------------------- per-tensor scale */

/* A = max |x| over a row-major bf16 tensor; s_t = A / 2688 (2688 = 6 * 448,
 * the largest E2M1 magnitude times the largest E4M3 scale), or 1 when A == 0.
 * READING: the pages only say "fine-grained scaling"; this per-tensor FP32
 * scale is the plainest choice that makes the largest block scale land on
 * E4M3's maximum. */
float oracle_amax(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld)
{
    float A = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            float a = fabsf(oracle_bf16_to_f32(x[r * ld + c]));
            if (a > A) A = a;
        }
    return A;
}

float oracle_tensor_scale_from_amax(float A)
{
    if (A == 0.0f) return 1.0f;
    return A / 2688.0f;
}

/* ------------------------------------------------------ block quantization */

/* One 16-element block (see the header comment of oracle_quantize for the
 * steps).  Writes 16 element codes and their dequantized values, returns the
 * E4M3 scale code. */
static uint8_t quantize_block(const float xb[16], float s_t, uint8_t q[16], float xh[16])
{
    float amax_b = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(xb[i]);
        if (a > amax_b) amax_b = a;
    }
    float v = (amax_b / 6.0f) / s_t;                /* amax/6, in units of s_t */
    uint8_t sf_code = oracle_e4m3_encode(v);
    float sf = (float)oracle_e4m3_decode(sf_code);
    float d = sf * s_t;                             /* the block's scale */
    for (int i = 0; i < 16; ++i) {
        /* a zero scale (only when the block is negligible next to the tensor
         * maximum) maps every element to a signed zero */
        float y = (d == 0.0f) ? xb[i] * 0.0f : xb[i] / d;
        q[i] = oracle_e2m1_encode(y);
        float qsf = (float)oracle_e2m1_decode(q[i]) * sf;   /* exact: 2 x 4 significant bits */
        xh[i] = qsf * s_t;
    }
    return sf_code;
}

/*
 * NVFP4 quantization of a row-major bf16 matrix X [M x K] (K % 16 == 0) with
 * a given per-tensor scale s_t.  For each 16-element block along K:
 *   1. a_b = max |x|;  v = fl(fl(a_b / 6) / s_t): the block maximum over the
 *      largest E2M1 magnitude, in units of the tensor scale;
 *   2. sf = E4M3(v) (nearest even, saturating);  d = fl(sf * s_t);
 *   3. q_i = E2M1(fl(x_i / d))  (all codes +-0 when d == 0);
 *   4. xhat_i = fl(e2m1(q_i) * sf * s_t), the dequantized value (the product
 *      e2m1 * sf is exact, so this is one rounding of the exact triple
 *      product);  R_i = fl(x_i - xhat_i).
 * READING: the pages name the format but not its arithmetic; every step is
 * the plain binary32 evaluation of its definition, left to right, one
 * rounding per operation.
 * Outputs (any may be NULL):
 *   codes  [M x K/2]  element 2j in bits 0..3, element 2j+1 in bits 4..7
 *   sf     [M x K/16] E4M3 scale codes, plain row-major (not swizzled)
 *   xhat   [M x K]    binary32 dequantized values
 *   resid  [M x K]    binary32 residual x - xhat
 */
void oracle_quantize(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, float s_t,
                     uint8_t *codes, uint8_t *sf, float *xhat, float *resid)
{
    int64_t nkb = K / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        for (int64_t b = 0; b < nkb; ++b) {
            float xb[16], xh[16];
            uint8_t q[16];
            for (int i = 0; i < 16; ++i)
                xb[i] = oracle_bf16_to_f32(x[r * ldx + b * 16 + i]);
            uint8_t sc = quantize_block(xb, s_t, q, xh);
            if (sf) sf[r * nkb + b] = sc;
            if (codes)
                for (int i = 0; i < 8; ++i)
                    codes[r * (K / 2) + b * 8 + i] = (uint8_t)(q[2 * i] | (q[2 * i + 1] << 4));
            for (int i = 0; i < 16; ++i) {
                if (xhat) xhat[r * K + b * 16 + i] = xh[i];
                if (resid) resid[r * K + b * 16 + i] = xb[i] - xh[i];
            }
        }
    }
}

/*
 * The same block quantization of a binary32 matrix (the residuals that the
 * "second pass of quantization" RAC variant quantizes again).  Outputs as for
 * oracle_quantize; rows of x are ldx floats apart.
 */
void oracle_quantize_f32(const float *x, int64_t M, int64_t K, int64_t ldx, float s_t,
                         uint8_t *codes, uint8_t *sf, float *xhat, float *resid)
{
    int64_t nkb = K / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        for (int64_t b = 0; b < nkb; ++b) {
            float xb[16], xh[16];
            uint8_t q[16];
            for (int i = 0; i < 16; ++i) xb[i] = x[r * ldx + b * 16 + i];
            uint8_t sc = quantize_block(xb, s_t, q, xh);
            if (sf) sf[r * nkb + b] = sc;
            if (codes)
                for (int i = 0; i < 8; ++i)
                    codes[r * (K / 2) + b * 8 + i] = (uint8_t)(q[2 * i] | (q[2 * i + 1] << 4));
            for (int i = 0; i < 16; ++i) {
                if (xhat) xhat[r * K + b * 16 + i] = xh[i];
                if (resid) resid[r * K + b * 16 + i] = xb[i] - xh[i];
            }
        }
    }
}

/*
 * Per-channel residual score: score[c] = sum over rows of R[r,c]^2, with R
 * the binary32 residual of oracle_quantize and the sum in binary64, rows in
 * order.  READING: the pages rank channels by "residual magnitude"
 * (gist.science/it, section 2.2 B); the squared L2 norm over the batch is the
 * plainest magnitude tied to the GEMM output error.
 * Rows whose row_valid entry is negative are skipped (row_valid may be NULL).
 */
void oracle_channel_score(const float *resid, int64_t M, int64_t K,
                          const int32_t *row_valid, double *score)
{
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < K; ++c) {
        double s = 0.0;
        for (int64_t r = 0; r < M; ++r) {
            if (row_valid && row_valid[r] < 0) continue;
            double v = (double)resid[r * K + c];
            s += v * v;
        }
        score[c] = s;
    }
}

/*
 * Top-k channel selection: S = the k channels with the largest score, equal
 * scores ordered by lower channel index first; S is returned in ascending
 * channel order (it is a set: the binary channel mask of gist.science/it,
 * section 2.2 B).  Selection sort, O(k K): slow and obvious.
 */
void oracle_select_topk(const double *score, int64_t K, int64_t k, int32_t *S)
{
    char *taken = (char *)calloc((size_t)K, 1);
    for (int64_t j = 0; j < k; ++j) {
        int64_t best = -1;
        for (int64_t c = 0; c < K; ++c) {
            if (taken[c]) continue;
            if (best < 0 || score[c] > score[best]) best = c;
        }
        if (best < 0) break;                       /* k > K */
        taken[best] = 1;
    }
    int64_t n = 0;
    for (int64_t c = 0; c < K; ++c)
        if (taken[c]) S[n++] = (int32_t)c;
    free(taken);
}

/*
 * RAC residual operand: rho[r, j] = bf16(fl(R[r, S_j] / s_t)), the residual of
 * the selected channels in units of the tensor scale, rounded to bfloat16.
 * READING: the correction is carried in BF16; expressing it in units of s_t
 * lets the correction share the main product's s_a * s_b output scale.
 */
void oracle_rac_residual(const float *resid, int64_t M, int64_t K, float s_t,
                         const int32_t *S, int64_t k, uint16_t *rho)
{
    for (int64_t r = 0; r < M; ++r)
        for (int64_t j = 0; j < k; ++j)
            rho[r * k + j] = oracle_f32_to_bf16(resid[r * K + S[j]] / s_t);
}

/*
 * Router: for each token the k_r experts with the largest logit (equal logits
 * ordered by lower expert index), in descending logit order, and the gate
 * weights g = softmax over the k_r selected logits, in binary64.
 */
void oracle_route(const float *logits, int64_t T, int64_t E, int64_t kr,
                  int32_t *idx, double *gate)
{
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        int32_t *o = idx + t * kr;
        for (int64_t j = 0; j < kr; ++j) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e) {
                int used = 0;
                for (int64_t i = 0; i < j; ++i)
                    if (o[i] == e) used = 1;
                if (used) continue;
                if (best < 0 || l[e] > l[best]) best = e;
            }
            o[j] = (int32_t)best;
        }
        double mx = (double)l[o[0]];
        double z = 0.0;
        for (int64_t j = 0; j < kr; ++j) z += exp((double)l[o[j]] - mx);
        for (int64_t j = 0; j < kr; ++j) gate[t * kr + j] = exp((double)l[o[j]] - mx) / z;
    }
}

/* ---------------------------------------------------- FP8 (comparison) */

/*
 * Per-tensor FP8 E4M3 quantization, the format of the FP8 rollout the pages
 * compare against (gist.science/it, sections 1 and 4: the stable FP8
 * baseline; NVFP4 GEMMs are quoted at ~2x its throughput).  READING: the
 * pages give no FP8 recipe; the plainest one is a per-tensor scale that maps
 * the tensor maximum to E4M3's largest magnitude:
 *   s = A / 448 (1 when A == 0);  q = E4M3(fl(x / s)) with the sign of x,
 *   nearest even, saturating at 448;  xhat = fl(e4m3(q) * s).
 * codes [M x K] (sign in bit 7), xhat [M x K] (either may be NULL).
 */
float oracle_fp8_scale_from_amax(float A)
{
    if (A == 0.0f) return 1.0f;
    return A / 448.0f;
}

void oracle_fp8_quantize(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, float s,
                         uint8_t *codes, float *xhat)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r)
        for (int64_t c = 0; c < K; ++c) {
            float v = oracle_bf16_to_f32(x[r * ldx + c]);
            float y = v / s;
            uint8_t q = oracle_e4m3_encode(fabsf(y));
            if (signbit(y)) q |= 0x80;
            if (codes) codes[r * K + c] = q;
            if (xhat) xhat[r * K + c] = (float)oracle_e4m3_decode(q) * s;
        }
}

/* Number of OpenMP threads the oracle runs with (1 without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------ array forms for tests */

void oracle_e2m1_encode_array(const float *y, uint8_t *q, int64_t n)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) q[i] = oracle_e2m1_encode(y[i]);
}

void oracle_e4m3_encode_array(const float *v, uint8_t *q, int64_t n)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) q[i] = oracle_e4m3_encode(v[i]);
}

void oracle_e4m3_decode_array(const uint8_t *q, double *v, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) v[i] = oracle_e4m3_decode(q[i]);
}

void oracle_e2m1_decode_array(const uint8_t *q, double *v, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) v[i] = oracle_e2m1_decode(q[i]);
}

void oracle_bf16_from_f32_array(const float *f, uint16_t *h, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) h[i] = oracle_f32_to_bf16(f[i]);
}
