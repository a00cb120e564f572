/*
 * nvfp4_quads.h -- C ABI of the B200 (sm_100a) QUADS rollout hot path:
 * NVFP4 online activation quantization with residual channel scoring,
 * top-k high-residual channel selection, the token-permuted grouped W4A4 MoE
 * expert GEMM with Residual Activation Compensation (RAC), and the
 * trainer-side weight quantize-dequantize (QDQ, asymmetric W4A16 QAT).
 *
 * Sources (the QUADS pages; page, section):
 *   gist.science/it, section 1      native W4A4 FP4 GEMMs; coarse E2M1 grid
 *   shd-paper.top, English abstract NVFP4 = fine-grained scaling + native W4A4
 *                                   GEMMs; activations are quantized online
 *   gist.science/it, section 2.1    activations recomputed online are the
 *                                   dominant error source
 *   gist.science/it, section 2.2 A  trainer fake-quantizes weights (W4A16)
 *   gist.science/it, section 2.2 B  RAC: top-k high-residual channels by a
 *                                   binary channel mask, correction added back
 *                                   to the quantized output, bulk stays on the
 *                                   native W4A4 GEMM
 *
 * Conventions (every entry point):
 *   - Pointers named *_dev are device pointers; the caller allocates and owns
 *     every buffer.  The library allocates nothing: scratch memory is a
 *     caller-provided workspace whose size the matching *_workspace_size
 *     function returns.  Workspaces need no initialization.
 *   - Calls are asynchronous on the given cudaStream_t (passed as void*;
 *     NULL = legacy default stream) and return after enqueueing.
 *   - Argument errors are detected synchronously and returned without
 *     enqueueing anything; nvfp4_last_error_string() describes the last one.
 *     NVFP4_ERR_CUDA reports a failed launch or runtime call.
 *   - Device-side bounded waits that run out (a deadlock would otherwise
 *     hang the GPU) write NVFP4_ERR_TIMEOUT into *dev_status when dev_status
 *     is non-NULL; the kernel then drains its copies, frees its tensor memory
 *     and returns.  Read it with nvfp4_read_status().
 *   - Device pointers must be 16-byte aligned.  Tensors are dense row-major.
 *   - Inputs must be finite; a tensor's max |x| must be 0 or >= 2^-90.
 *
 * Data formats (NVFP4):
 *   codes   uint8 [rows x K/2]: element 2j of a row in bits 0..3 of byte j,
 *           element 2j+1 in bits 4..7; code = sign<<3 | i, magnitude
 *           {0,0.5,1,1.5,2,3,4,6}[i] (E2M1).
 *   scales  uint8 E4M3 (sign 0), one per 16 consecutive elements of a row,
 *           in the tensor-core scale-factor layout: 512-byte atoms holding
 *           128 rows x 4 scale columns; atom (r/128, c/4) at byte offset
 *           ((r/128)*(K/64) + c/4)*512, entry (r, c) inside it at
 *           (r%32)*16 + ((r%128)/32)*4 + c%4.  Buffer size:
 *           ceil(rows/128)*128 * K/16 bytes.  Rows are padded to 128.
 *   s_t     float32 per tensor: s_t = max|x| / 2688 (1 for an all-zero tensor).
 *   Per 16-block with amax a (binary32, one rounding per operation):
 *   sf = E4M3_rne(fl(fl(a/6)/s_t)), d = fl(sf*s_t), q = E2M1_rne(fl(x/d)),
 *   dequantized value xhat = fl(e2m1(q)*sf*s_t) (e2m1*sf is exact), residual
 *   R = fl(x - xhat).
 */
#ifndef NVFP4_QUADS_H
#define NVFP4_QUADS_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum */
    NVFP4_ERR_ALIGNMENT = 2,         /* pointer or leading dimension misaligned */
    NVFP4_ERR_UNSUPPORTED_SHAPE = 3, /* shape outside the supported envelope */
    NVFP4_ERR_CUDA = 4,              /* CUDA runtime / launch failure */
    NVFP4_ERR_TIMEOUT = 5,           /* a device-side bounded wait ran out */
    NVFP4_ERR_WORKSPACE = 6          /* workspace missing or too small */
} nvfp4_status;

/* Library version, e.g. 100 for 0.1.0. */
NVFP4_API int nvfp4_version(void);

/* Message for the last error returned on the calling thread ("" if none). */
NVFP4_API const char *nvfp4_last_error_string(void);

/* Synchronously copies a device status word (see dev_status above) to the
 * host; *status_out receives NVFP4_OK or the device-reported status. */
NVFP4_API nvfp4_status nvfp4_read_status(const int32_t *dev_status, int32_t *status_out, void *stream);

/* Number of SMs of the current device (used to size persistent grids). */
NVFP4_API int nvfp4_num_sms(void);

/* --------------------------------------------------------------------------
 * nvfp4_quantize -- online NVFP4 activation quantization, residual channel
 * scoring and RAC channel selection (shd-paper.top abstract: activations are
 * quantized online; gist.science/it 2.2 B: channels with the largest FP4
 * residual are selected by a top-k binary mask).
 *
 * One call runs: (1) per-tensor amax -> s_t (skipped when s_t_in_dev is
 * given), (2) one streaming pass that writes codes and swizzled scales and
 * accumulates score[c] = sum_r R[r,c]^2 (binary64 across rows), (3) selection
 * of the rac_k channels with the largest score (equal scores: lower index
 * first), returned ascending, (4) the RAC residual operand
 * r_sel[dst, j] = bf16(R[r, S_j] / s_t) for every output row.
 *
 *   x_dev        bf16 [M x K], row stride ldx elements (ldx % 8 == 0).
 *   M, K         K % 64 == 0, 64 <= K <= 16384; M >= 0.
 *   m_valid_dev  optional int32 on the device: rows >= *m_valid_dev are
 *                ignored (absent from amax, scores and outputs).  NULL = M.
 *   s_t_in_dev   optional float32: use this tensor scale instead of amax.
 *   amax_in_dev  optional float32: the tensor's max |x| over its valid rows,
 *                already computed by the producer of x (e.g. the SwiGLU
 *                epilogue of moe_w4a4_grouped_gemm_rac); s_t is derived from
 *                it and the amax pass is skipped.  Ignored when s_t_in_dev is
 *                given.
 *   s_t_out_dev  float32 [1]: receives s_t (required).
 *   dst_rows_dev optional int32 [M x fanout]: input row r is written to output
 *                rows dst_rows[r*fanout + j] (j < fanout, 1 <= fanout <= 32);
 *                a negative entry, or one >= M_out, skips that copy.  NULL:
 *                output row = input row, fanout 1.
 *   M_out        rows of the output arrays (every destination < M_out).
 *   codes_dev    uint8 [M_out x K/2].
 *   scales_dev   uint8 swizzled, ceil(M_out/128)*128*K/16 bytes.
 *   score_dev    optional float64 [K]: receives the channel scores.  Required
 *                when rac_k > 0.
 *   rac_k        channels to select, 0 <= rac_k <= K (the pages' "top k% of
 *                channels" is rac_k = k% of K).
 *   rac_ld       row stride (elements) of r_sel, rac_ld >= rac_k,
 *                rac_ld % 64 == 0; columns [rac_k, rac_ld) are written as 0.
 *   sel_dev      int32 [rac_k]: selected channels, ascending.
 *   r_sel_dev    bf16 [M_out x rac_ld], or NULL: the channels are selected
 *                but no residual is written (e.g. when
 *                nvfp4_rac_residual_nvfp4 produces the RAC operand next;
 *                rac_ld is then not checked).
 *   dev_status   optional int32 status word (see conventions).
 *   workspace    nvfp4_quantize_workspace_size(M, K) bytes, 16-byte aligned.
 * Only rows named as destinations are written; other output rows keep their
 * contents.
 * -------------------------------------------------------------------------- */
NVFP4_API size_t nvfp4_quantize_workspace_size(int64_t M, int64_t K);

NVFP4_API nvfp4_status nvfp4_quantize(const void *x_dev, int64_t M, int64_t K, int64_t ldx,
                            const int32_t *m_valid_dev,
                            const float *s_t_in_dev, const float *amax_in_dev, float *s_t_out_dev,
                            const int32_t *dst_rows_dev, int32_t fanout, int64_t M_out,
                            uint8_t *codes_dev, uint8_t *scales_dev,
                            double *score_dev, int32_t rac_k, int32_t rac_ld,
                            int32_t *sel_dev, void *r_sel_dev,
                            int32_t *dev_status, void *workspace, size_t workspace_bytes,
                            void *stream);

/* --------------------------------------------------------------------------
 * nvfp4_quantize_experts -- nvfp4_quantize with one RAC channel set per
 * expert (READING: the pages select one binary mask of the top-k channels by
 * residual magnitude per GEMM input, gist.science/it 2.2 B; here each
 * expert's GEMM input gets the mask of its own rows).  x holds routed rows
 * in the expert-grouped layout of moe_route (expert e owns rows
 * [offsets[e], offsets[e+1]), segments padded to seg_align with zero rows;
 * rows >= offsets[E] are ignored), e.g. h from the gate/up GEMM or X from
 * moe_routed_rows_bf16.
 *   one tensor scale s_t over all rows (s_t_in / amax_in / amax pass as for
 *   nvfp4_quantize); codes and scales for every row (M_out = M, no fan-out);
 *   score_dev   optional float64 [E x K]: score[e,c] = sum over e's rows of
 *               R[r,c]^2 (NULL: kept in the workspace);
 *   sel_dev     int32 [E x rac_k]: expert e's channels, ascending;
 *   r_sel_dev   bf16 [M x rac_ld]: rho[r, j] = bf16(R[r, S_e(r)[j]] / s_t),
 *               zero for j >= rac_k.
 * 1 <= E <= 256, seg_align 128 or 256, M % seg_align == 0, 1 <= rac_k <= K,
 * rac_ld % 64 == 0; K, ldx and alignment as for nvfp4_quantize.
 * workspace: nvfp4_quantize_experts_workspace_size(M, K, E, seg_align).
 * -------------------------------------------------------------------------- */
NVFP4_API size_t nvfp4_quantize_experts_workspace_size(int64_t M, int64_t K, int32_t E, int32_t seg_align);

NVFP4_API nvfp4_status nvfp4_quantize_experts(const void *x_dev, int64_t M, int64_t K, int64_t ldx,
                                    const int32_t *offsets_dev, int32_t E, int32_t seg_align,
                                    const float *s_t_in_dev, const float *amax_in_dev, float *s_t_out_dev,
                                    uint8_t *codes_dev, uint8_t *scales_dev, double *score_dev,
                                    int32_t rac_k, int32_t rac_ld, int32_t *sel_dev, void *r_sel_dev,
                                    int32_t *dev_status, void *workspace, size_t workspace_bytes, void *stream);

/* --------------------------------------------------------------------------
 * nvfp4_quantize_noalloc -- nvfp4_quantize without a caller workspace.  The
 * QUADS pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory at the moment they quantize: a plug-in
 * running inside a host framework that owns every device allocation and gives
 * it no allocator, or a serving loop that reserved all free device memory up
 * front and may not call cudaMalloc (or wait on its implicit synchronization)
 * per request.  Such a caller still passes its inputs and outputs; only the
 * scratch memory moves into the library.
 *
 * Arguments, outputs and errors are those of nvfp4_quantize minus
 * workspace/workspace_bytes.  Scratch is a fixed 4 MiB array in the library's
 * device memory (nvfp4_quantize_noalloc_max_scratch() returns its size), held
 * by every GPU that loads the library until the process exits.  Shapes whose
 * nvfp4_quantize_workspace_size(M, K) exceeds it are rejected with
 * NVFP4_ERR_UNSUPPORTED_SHAPE.  The call allocates nothing (no cudaMalloc,
 * cudaFree or allocating library routine).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls share the one array and it keeps the previous call's
 *     contents; the call clears what must start at zero itself.  Calls whose
 *     executions overlap on the GPU (different streams, or several host
 *     threads) race on the array and give undefined results: serialize them.
 * -------------------------------------------------------------------------- */
NVFP4_API size_t nvfp4_quantize_noalloc_max_scratch(void);

NVFP4_API nvfp4_status nvfp4_quantize_noalloc(const void *x_dev, int64_t M, int64_t K, int64_t ldx,
                                              const int32_t *m_valid_dev,
                                              const float *s_t_in_dev, const float *amax_in_dev,
                                              float *s_t_out_dev,
                                              const int32_t *dst_rows_dev, int32_t fanout, int64_t M_out,
                                              uint8_t *codes_dev, uint8_t *scales_dev,
                                              double *score_dev, int32_t rac_k, int32_t rac_ld,
                                              int32_t *sel_dev, void *r_sel_dev,
                                              int32_t *dev_status, void *stream);

/* --------------------------------------------------------------------------
 * nvfp4_rac_residual_nvfp4 -- the RAC variant with a second pass of NVFP4
 * quantization on the selected channels (gist.science/it 2.2 B).  Given the
 * channel set S (sel_dev, ascending, from nvfp4_quantize) and the tensor
 * scale s_t of x, the residuals R[r, S_j] = fl(x - xhat) of the valid rows
 * are quantized again as one [rows x rac_k] tensor: s_r = max|R_S| / 2688 (1
 * if all zero), 16-element blocks along j (the last block zero-padded), the
 * NVFP4 block steps of nvfp4_quantize, dequantized value rhat; the RAC
 * operand becomes r_sel[dst, j] = bf16(fl(rhat / s_t)) for j < rac_k and 0
 * for rac_k <= j < rac_ld, written like nvfp4_quantize's r_sel (same
 * m_valid, dst_rows, fanout, M_out semantics), replacing the plain residual.
 *   s_r_out_dev  optional float32 [1]: receives s_r.
 *   workspace    nvfp4_rac_residual_nvfp4_workspace_size() bytes.
 * rac_ld % 64 == 0, rac_k <= rac_ld; x as for nvfp4_quantize.
 * -------------------------------------------------------------------------- */
NVFP4_API size_t nvfp4_rac_residual_nvfp4_workspace_size(void);

NVFP4_API nvfp4_status nvfp4_rac_residual_nvfp4(const void *x_dev, int64_t M, int64_t K, int64_t ldx,
                                                const int32_t *m_valid_dev, const float *s_t_dev,
                                                const int32_t *sel_dev, int32_t rac_k, int32_t rac_ld,
                                                const int32_t *dst_rows_dev, int32_t fanout, int64_t M_out,
                                                void *r_sel_dev, float *s_r_out_dev, void *workspace,
                                                size_t workspace_bytes, void *stream);

/* --------------------------------------------------------------------------
 * nvfp4_qdq_weights -- trainer-side asymmetric QAT weight fake-quantization
 * (gist.science/it 2.2 A: weights are quantized to NVFP4 and dequantized on
 * every trainer forward so the trainer sees the rollout's weights; activations
 * stay BF16), and the rollout engine's weight quantizer.
 *
 * G independent tensors w[g] of [rows x cols] bf16 (contiguous, g-major),
 * each with its own s_t[g] = max|w[g]|/2688.
 *   w_qdq_dev   optional bf16 [G x rows x cols]: bf16(xhat), nearest even.
 *   s_t_dev     float32 [G] (required).
 *   codes_dev   optional uint8 [G x rows x cols/2].
 *   scales_dev  optional uint8 [G x ceil(rows/128)*128*cols/16], swizzled per
 *               tensor.
 * cols % 64 == 0, cols <= 16384, ldx = cols.
 * -------------------------------------------------------------------------- */
NVFP4_API size_t nvfp4_qdq_workspace_size(int64_t G, int64_t rows, int64_t cols);

NVFP4_API nvfp4_status nvfp4_qdq_weights(const void *w_dev, int64_t G, int64_t rows, int64_t cols,
                               void *w_qdq_dev, float *s_t_dev,
                               uint8_t *codes_dev, uint8_t *scales_dev,
                               void *workspace, size_t workspace_bytes, void *stream);

/* --------------------------------------------------------------------------
 * moe_route -- top-k_r expert routing of T tokens over E experts and the
 * expert-grouped routed-row layout used by the grouped GEMMs.
 *
 *   logits_dev   float32 [T x E], E <= 256, 1 <= k_r <= min(E, 8); -0 ranks
 *                as +0, and a NaN logit (not a routing input) would rank
 *                above every number.
 *   topk_idx_dev int32 [T x k_r]: experts by descending logit (equal logits:
 *                lower expert first).
 *   topk_gate_dev float32 [T x k_r]: softmax over the k_r selected logits.
 *   seg_align    128 or 256: every expert segment is padded to a multiple of
 *                this many rows (the grouped GEMM's tile height: 256 selects
 *                its 2-SM shape).
 *   offsets_dev  int32 [E+1]: expert e owns routed rows
 *                [offsets[e], offsets[e+1]); offsets[E] = total padded rows.
 *   dst_row_dev  int32 [T x k_r]: routed row of (token t, slot j).  Inside
 *                an expert's segment tokens appear in ascending order.
 *   row_token_dev int32 [M_pad_max]: token of each routed row, -1 for padding
 *                and for rows >= offsets[E].
 *   row_gate_dev float32 [M_pad_max]: gate of each routed row (0 for padding).
 *   M_pad_max    >= T*k_r + E*(seg_align-1) rounded up to seg_align.
 * T may be 0 (the per-token arrays may then be NULL): every segment is empty.
 * workspace: moe_route_workspace_size(T, E) bytes (per-block expert counts).
 * -------------------------------------------------------------------------- */
NVFP4_API size_t moe_route_workspace_size(int64_t T, int32_t E);

NVFP4_API nvfp4_status moe_route(const float *logits_dev, int64_t T, int32_t E, int32_t k_r,
                       int32_t *topk_idx_dev, float *topk_gate_dev,
                       int32_t seg_align, int32_t *offsets_dev, int32_t *dst_row_dev,
                       int32_t *row_token_dev, float *row_gate_dev, int64_t M_pad_max,
                       void *workspace, size_t workspace_bytes, void *stream);

/* --------------------------------------------------------------------------
 * nvfp4_gather_weight_channels -- RAC weight operand: the selected input
 * channels S of every expert's NVFP4 weight, dequantized without the tensor
 * scale (e2m1 * sf is exact in bf16):
 *   w_sel[e, n, j] = bf16(e2m1(q_e[n, S_j]) * sf_e[n, S_j/16])  (j < k)
 *   w_sel[e, n, j] = 0                                          (k <= j < ld)
 * A selected index outside [0, K) also gives a zero column.
 *   codes_dev  uint8 [E x N x K/2], scales_dev swizzled per expert.
 *   w_sel_dev  bf16 [E x N x ld], ld % 64 == 0, k <= ld <= 16384.
 * -------------------------------------------------------------------------- */
NVFP4_API nvfp4_status nvfp4_gather_weight_channels(const uint8_t *codes_dev, const uint8_t *scales_dev,
                                          int32_t E, int64_t N, int64_t K,
                                          const int32_t *sel_dev, int32_t k, int32_t ld,
                                          void *w_sel_dev, void *stream);

/* --------------------------------------------------------------------------
 * nvfp4_weights_channel_major -- one-time channel-major copy of E NVFP4
 * weights [N x K] (made when weights are loaded; they do not change between
 * steps) so that the per-step RAC weight gather reads only the selected
 * channels:
 *   codes_cm_dev  uint8 [E x K x N/2]: row c holds the codes of input
 *                 channel c for all N output features (even n in the low
 *                 nibble).
 *   scales_cm_dev uint8 [E x K/16 x N]: row b holds the E4M3 scale of block
 *                 b of every output feature.
 * N % 64 == 0, K % 64 == 0.
 *
 * nvfp4_gather_weight_channels_cm -- nvfp4_gather_weight_channels from the
 * channel-major copy (identical output: w_sel[e, n, j] = bf16(e2m1 * sf) of
 * channel S_j, zero for k <= j < ld).
 * -------------------------------------------------------------------------- */
NVFP4_API nvfp4_status nvfp4_weights_channel_major(const uint8_t *codes_dev, const uint8_t *scales_dev, int32_t E,
                                                   int64_t N, int64_t K, uint8_t *codes_cm_dev,
                                                   uint8_t *scales_cm_dev, void *stream);

NVFP4_API nvfp4_status nvfp4_gather_weight_channels_cm(const uint8_t *codes_cm_dev, const uint8_t *scales_cm_dev,
                                                       int32_t E, int64_t N, int64_t K, const int32_t *sel_dev,
                                                       int32_t k, int32_t ld, void *w_sel_dev, void *stream);

/* nvfp4_gather_weight_channels_cm_experts -- the same with one channel set
 * per expert (per-expert RAC, see nvfp4_quantize_experts): sel_dev is int32
 * [E x k] and expert e gathers the channels sel[e*k .. e*k + k). */
NVFP4_API nvfp4_status nvfp4_gather_weight_channels_cm_experts(const uint8_t *codes_cm_dev,
                                                               const uint8_t *scales_cm_dev, int32_t E, int64_t N,
                                                               int64_t K, const int32_t *sel_dev, int32_t k,
                                                               int32_t ld, void *w_sel_dev, void *stream);

/* --------------------------------------------------------------------------
 * moe_w4a4_grouped_gemm_rac -- the native W4A4 block-scaled grouped expert
 * GEMM with Residual Activation Compensation folded into the same
 * accumulator (gist.science/it 2.2 B; shd-paper.top abstract: RAC corrects
 * high-error activation channels while keeping native W4A4 GEMMs).
 *
 * For every routed row r of expert e (offsets[e] <= r < offsets[e+1]) and
 * output feature n:
 *   D[r,n] = sum_k (e2m1(a)*sfa)[r,k] (e2m1(b_e)*sfb_e)[n,k]      (FP4 MMA)
 *          + sum_j rho[r,j] w_sel[e,n,j]                          (BF16 MMA)
 *   y[r,n] = s_a * s_b[e] * D[r,n]
 * and the epilogue writes y:
 *   MOE_EPI_STORE_F32    out f32 [M_pad_max x ld_out], rows with
 *                        row_token < 0 not written.
 *   MOE_EPI_SWIGLU_BF16  N = 2I (gate rows [0,I), up rows [I,2I) of B);
 *                        out bf16 [M_pad_max x ld_out]:
 *                        h[r,i] = bf16(silu(y[r,i]) * y[r,I+i]) for i < I;
 *                        rows with row_token < 0 (and < offsets[E]) are
 *                        written as 0.  I % 128 == 0.  If amax_out_dev is
 *                        non-NULL it receives max |h| over every row written
 *                        (the value nvfp4_quantize's amax_in_dev takes).
 *   MOE_EPI_SCATTER_ADD_F32  out f32 [T x ld_out]:
 *                        out[row_token[r], n] += row_gate[r] * y[r,n]
 *                        (atomic; the caller zeroes out first).  Every
 *                        row_token >= 0 must be a row of out (< T), as
 *                        moe_route's are; the kernel does not check it.
 *
 *   a_codes_dev/a_scales_dev  NVFP4 A, rows in routed order, M_pad_max rows.
 *   a_s_t_dev       float32 [1].
 *   b_codes_dev/b_scales_dev  NVFP4 B, E tensors of [N x K] (per-expert
 *                   swizzled scales), b_s_t_dev float32 [E].
 *   offsets_dev     int32 [E+1] from moe_route, multiples of seg_align.
 *   seg_align       128: one CTA per SM computes 128-row x 256-feature tiles;
 *                   256: CTA pairs (2-SM tensor-core tiles, cluster launch)
 *                   compute 256-row x 256-feature tiles.
 *   rac_ld          0 (no RAC) or the row stride of rho / w_sel, % 64 == 0,
 *                   <= 16384 (rac_ld / 64 BF16 stages per tile); rho_dev
 *                   bf16 [M_pad_max x rac_ld] and
 *                   w_sel_dev bf16 [E x N x rac_ld].
 * Shapes: K % 256 == 0, N % 256 == 0 (SWIGLU: I % 128 == 0), M_pad_max a
 * multiple of seg_align, E <= 256; pointers 16-byte aligned.  Persistent
 * kernel: one CTA per SM (seg_align 256: one 2-CTA cluster per SM pair); the
 * tile count is read from offsets[E] on the device (no host sync).
 * Errors: argument, shape and alignment errors are returned synchronously;
 * a device wait that exceeds its bound (1 s) writes NVFP4_ERR_TIMEOUT to
 * dev_status (if given) and the kernel exits cleanly.  Tuning only: the
 * environment variable NVFP4_GEMM_NGROUP (a divisor of the n-tile count)
 * overrides how many n-tiles run as one group in the tile order.
 * -------------------------------------------------------------------------- */
typedef enum {
    MOE_EPI_STORE_F32 = 0,
    MOE_EPI_SWIGLU_BF16 = 1,
    MOE_EPI_SCATTER_ADD_F32 = 2
} moe_epilogue;

NVFP4_API nvfp4_status moe_w4a4_grouped_gemm_rac(
    const uint8_t *a_codes_dev, const uint8_t *a_scales_dev, const float *a_s_t_dev,
    int64_t M_pad_max,
    const uint8_t *b_codes_dev, const uint8_t *b_scales_dev, const float *b_s_t_dev,
    int64_t N, int64_t K, int32_t E,
    const int32_t *offsets_dev, int32_t seg_align,
    int32_t rac_ld, const void *rho_dev, const void *w_sel_dev,
    int32_t epilogue, const int32_t *row_token_dev, const float *row_gate_dev,
    void *out_dev, int64_t ld_out, float *amax_out_dev,
    int32_t *dev_status, void *stream);

/* --------------------------------------------------------------------------
 * moe_bf16_grouped_gemm -- the trainer-side W4A16 expert GEMM
 * (gist.science/it 2.2 A: the trainer fake-quantizes the weights to NVFP4
 * and keeps activations in BF16): BF16 A x BF16 B on the tensor cores
 * (kind::f16, f32 accumulation in TMEM), B normally the nvfp4_qdq_weights
 * output.  For every routed row r of expert e and output feature n:
 *   y[r,n] = sum_k a[r,k] b_e[n,k]
 * with the same three epilogues as moe_w4a4_grouped_gemm_rac (unit tensor
 * scales).
 *   a_dev     bf16 [M_pad_max x lda], rows in routed order (e.g. from
 *             moe_gather_rows_bf16, or the SwiGLU output of the first GEMM).
 *   b_dev     bf16 [E x N x K], contiguous.
 *   offsets_dev, seg_align, epilogue, row_token_dev, row_gate_dev, out_dev,
 *   ld_out, amax_out_dev: as for moe_w4a4_grouped_gemm_rac.
 * Shapes: K % 64 == 0, N % 256 == 0 (SWIGLU: I % 128 == 0), lda >= K and
 * lda % 8 == 0, M_pad_max a multiple of seg_align, E <= 256.  Pointers 16-byte
 * aligned.  Errors as for moe_w4a4_grouped_gemm_rac.
 *
 * moe_gather_rows_bf16 -- the W4A16 path's activation fan-out: token row t of
 * x (bf16 [T x ldx]) is copied to rows dst_rows[t*fanout + j] (j < fanout,
 * 1 <= fanout <= 32, negative entries skipped) of out (bf16 [M_out x ld_out]);
 * other rows of out are not touched.  K % 8 == 0, ldx and ld_out >= K and
 * multiples of 8, pointers 16-byte aligned.
 * -------------------------------------------------------------------------- */
NVFP4_API nvfp4_status moe_bf16_grouped_gemm(
    const void *a_dev, int64_t lda, int64_t M_pad_max, const void *b_dev, int64_t N, int64_t K, int32_t E,
    const int32_t *offsets_dev, int32_t seg_align, int32_t epilogue, const int32_t *row_token_dev,
    const float *row_gate_dev, void *out_dev, int64_t ld_out, float *amax_out_dev, int32_t *dev_status,
    void *stream);

NVFP4_API nvfp4_status moe_gather_rows_bf16(const void *x_dev, int64_t T, int64_t K, int64_t ldx,
                                            const int32_t *dst_rows_dev, int32_t fanout, void *out_dev,
                                            int64_t ld_out, int64_t M_out, void *stream);

/* moe_routed_rows_bf16 -- the complete routed copy of x: every row r < M_out
 * of out (bf16 [M_out x ld_out]) receives token row row_token[r] of x (bf16
 * [T x ldx]), or zeros where row_token[r] < 0 (segment padding), so rows a
 * previous routing left behind never survive.  Used by per-expert RAC on the
 * gate/up input.  K % 8 == 0, ldx and ld_out >= K and multiples of 8,
 * pointers 16-byte aligned, M_out < 2^31. */
NVFP4_API nvfp4_status moe_routed_rows_bf16(const void *x_dev, int64_t T, int64_t K, int64_t ldx,
                                            const int32_t *row_token_dev, void *out_dev, int64_t ld_out,
                                            int64_t M_out, void *stream);

/* --------------------------------------------------------------------------
 * fp8_quantize / moe_w8a8_grouped_gemm -- the FP8 comparison path: the pages
 * compare NVFP4 rollout with a stable FP8 rollout and quote native NVFP4
 * GEMMs at about twice FP8 throughput (gist.science/it sections 1 and 4);
 * these two calls give the same grouped expert GEMM on E4M3 operands so that
 * the ratio can be measured on the same shapes.
 *
 * fp8_quantize: per-tensor E4M3 of G bf16 tensors [M x K] (row stride ldx,
 * group stride M*ldx): s = max|x| / 448 (1 for an all-zero tensor), or
 * s_in_dev[g] when given, or amax_in_dev[0] / 448 (G == 1); codes =
 * E4M3(fl(x / s)) with the sign of x in bit 7, nearest even, saturating.
 *   s_out_dev   float32 [G] (required).
 *   dst_rows_dev optional int32 [M x fanout] (G == 1): routed copies of each
 *               row, negative entries or entries >= M_out skipped.
 *   codes_dev   uint8 [G x M_out x K] (M_out >= M without dst_rows).
 * K % 16 == 0, ldx % 8 == 0, pointers 16-byte aligned.  workspace:
 * fp8_quantize_workspace_size(G) bytes unless s_in_dev or amax_in_dev.
 *
 * moe_w8a8_grouped_gemm: for every routed row r of expert e,
 *   y[r,n] = s_a * s_b[e] * sum_k e4m3(a)[r,k] e4m3(b_e)[n,k]
 * (kind::f8f6f4 MMAs, f32 accumulation in TMEM) with the epilogues of
 * moe_w4a4_grouped_gemm_rac.  a_codes_dev uint8 [M_pad_max x K] in routed
 * order, b_codes_dev uint8 [E x N x K], a_s_dev float32 [1], b_s_dev float32
 * [E].  K % 128 == 0, N % 256 == 0; other shapes and errors as for
 * moe_w4a4_grouped_gemm_rac.
 * -------------------------------------------------------------------------- */
NVFP4_API size_t fp8_quantize_workspace_size(int64_t G);

NVFP4_API nvfp4_status fp8_quantize(const void *x_dev, int64_t G, int64_t M, int64_t K, int64_t ldx,
                                    const float *s_in_dev, const float *amax_in_dev, float *s_out_dev,
                                    const int32_t *dst_rows_dev, int32_t fanout, int64_t M_out, uint8_t *codes_dev,
                                    void *workspace, size_t workspace_bytes, void *stream);

NVFP4_API nvfp4_status moe_w8a8_grouped_gemm(
    const uint8_t *a_codes_dev, const float *a_s_dev, int64_t M_pad_max, const uint8_t *b_codes_dev,
    const float *b_s_dev, int64_t N, int64_t K, int32_t E, const int32_t *offsets_dev, int32_t seg_align,
    int32_t epilogue, const int32_t *row_token_dev, const float *row_gate_dev, void *out_dev, int64_t ld_out,
    float *amax_out_dev, int32_t *dev_status, void *stream);

/* --------------------------------------------------------------------------
 * nvfp4_debug_gemm_wait_expiry -- test hook for the bounded device waits of
 * the grouped GEMM (the pages have no counterpart).  Runs
 * moe_w4a4_grouped_gemm_rac in its 1-SM shape (seg_align 128, no RAC) with
 * every mbarrier wait bounded by wait_limit_ns (1 ms .. 1 s), and with the
 * MMA issuer withholding the "accumulator ready" signal of the first tile
 * (it drains its MMAs itself), so the epilogue's wait runs out.  Expected
 * outcome: *dev_status = NVFP4_ERR_TIMEOUT, every copy and MMA drained, tensor
 * memory freed, the kernel returns and the context stays usable; the output
 * of the withheld tile is not written.  Arguments as for
 * moe_w4a4_grouped_gemm_rac; dev_status is required.
 * -------------------------------------------------------------------------- */
NVFP4_API nvfp4_status nvfp4_debug_gemm_wait_expiry(
    const uint8_t *a_codes_dev, const uint8_t *a_scales_dev, const float *a_s_t_dev, int64_t M_pad_max,
    const uint8_t *b_codes_dev, const uint8_t *b_scales_dev, const float *b_s_t_dev, int64_t N, int64_t K, int32_t E,
    const int32_t *offsets_dev, int32_t epilogue, const int32_t *row_token_dev, const float *row_gate_dev,
    void *out_dev, int64_t ld_out, int32_t *dev_status, int64_t wait_limit_ns, void *stream);

/* --------------------------------------------------------------------------
 * nvfp4_debug_encode -- runs the library's element and scale encoders on n
 * arbitrary floats (for validation against an independent definition):
 *   e2m1_dev[i] = E2M1 code of in[i] (nearest even, saturating, sign bit
 *                 of in[i]); e4m3_dev[i] = E4M3 code of in[i] >= 0 (nearest
 *                 even, saturating at 448).  Either output may be NULL.
 * -------------------------------------------------------------------------- */
NVFP4_API nvfp4_status nvfp4_debug_encode(const float *in_dev, int64_t n, uint8_t *e2m1_dev, uint8_t *e4m3_dev,
                                void *stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_QUADS_H */
