// route.cu -- MoE top-k routing and the expert-grouped routed-row layout.
//
//   k_route_topk    one warp per token: k_r rounds of warp argmax over the E
//                   logits (equal logits: lower expert), softmax over the
//                   selected logits, per-expert counts (atomics).
//   k_route_assign  one CTA per expert: padded segment offset (segments are
//                   multiples of 128 or 256 rows, the GEMM's tile height) from the
//                   counts, then a block-wide scan over tokens in ascending
//                   order assigns each (token, slot) routed to the expert its
//                   row; writes dst_row, row_token, row_gate and the padding.
// Rows inside an expert's segment are in ascending token order, so the layout
// is deterministic.
#include "common.cuh"

#include <algorithm>

namespace nvfp4 {

constexpr int MAX_EXPERTS = 256;
constexpr int MAX_TOPK = 8;

__global__ void __launch_bounds__(256) k_route_topk(const float *__restrict__ logits, int64_t T, int E, int kr,
                                                    int32_t *__restrict__ topk_idx, float *__restrict__ topk_gate,
                                                    int32_t *__restrict__ counts)
{
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    float l[MAX_EXPERTS / 32];
#pragma unroll
    for (int i = 0; i < MAX_EXPERTS / 32; ++i) {
        int e = lane + 32 * i;
        l[i] = (e < E) ? logits[t * E + e] : -INFINITY;
    }
    unsigned taken = 0;      // bit i: expert lane + 32 i already selected
    float sel_l[MAX_TOPK];   // fully unrolled below: stays in registers
    int sel_e[MAX_TOPK];
#pragma unroll
    for (int j = 0; j < MAX_TOPK; ++j) {
        sel_l[j] = -INFINITY;
        sel_e[j] = 0;
        if (j < kr) {
            float bv = -INFINITY;
            int be = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < MAX_EXPERTS / 32; ++i) {
                int e = lane + 32 * i;
                if (e < E && !((taken >> i) & 1u)) {
                    if (be == 0x7fffffff || l[i] > bv) { bv = l[i]; be = e; }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                int oe = __shfl_xor_sync(0xffffffffu, be, o);
                if (oe != 0x7fffffff && (be == 0x7fffffff || ov > bv || (ov == bv && oe < be))) { bv = ov; be = oe; }
            }
            sel_l[j] = bv;
            sel_e[j] = be;
            if ((be & 31) == lane) taken |= 1u << (be >> 5);
        }
    }
    if (lane == 0) {
        const float mx = sel_l[0];
        float z = 0.0f;
        float ex[MAX_TOPK];
#pragma unroll
        for (int j = 0; j < MAX_TOPK; ++j) {
            ex[j] = j < kr ? expf(sel_l[j] - mx) : 0.0f;
            z += ex[j];
        }
#pragma unroll
        for (int j = 0; j < MAX_TOPK; ++j) {
            if (j < kr) {
                topk_idx[t * kr + j] = sel_e[j];
                topk_gate[t * kr + j] = ex[j] / z;
                atomicAdd(counts + sel_e[j], 1);
            }
        }
    }
}

__global__ void __launch_bounds__(1024) k_route_assign(const int32_t *__restrict__ topk_idx,
                                                       const float *__restrict__ topk_gate, int64_t T, int E, int kr,
                                                       const int32_t *__restrict__ counts, int align,
                                                       int32_t *__restrict__ offsets, int32_t *__restrict__ dst_row,
                                                       int32_t *__restrict__ row_token, float *__restrict__ row_gate)
{
    __shared__ int s_base, s_cnt, s_running;
    __shared__ int warp_sums[32];
    const int e = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        int base = 0, total = 0;
        for (int i = 0; i < E; ++i) {
            int padded = (counts[i] + align - 1) / align * align;
            if (i < e) base += padded;
            total += padded;
        }
        s_base = base;
        s_cnt = counts[e];
        s_running = 0;
        offsets[e] = base;
        if (e == E - 1) offsets[E] = total;
    }
    __syncthreads();
    const int base = s_base;
    for (int64_t t0 = 0; t0 < T; t0 += blockDim.x) {
        int64_t t = t0 + tid;
        int slot = -1;
        if (t < T) {
            for (int j = 0; j < kr; ++j)
                if (topk_idx[t * kr + j] == e) slot = j;
        }
        unsigned ballot = __ballot_sync(0xffffffffu, slot >= 0);
        int within = __popc(ballot & ((1u << lane) - 1u));
        if (lane == 0) warp_sums[warp] = __popc(ballot);
        __syncthreads();
        int before = 0, chunk_total = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            int s = warp_sums[w];
            if (w < warp) before += s;
            chunk_total += s;
        }
        if (slot >= 0) {
            int row = base + s_running + before + within;
            dst_row[t * kr + slot] = row;
            row_token[row] = (int32_t)t;
            row_gate[row] = topk_gate[t * kr + slot];
        }
        __syncthreads();
        if (tid == 0) s_running += chunk_total;
        __syncthreads();
    }
    const int cnt = s_cnt;
    const int padded = (cnt + align - 1) / align * align;
    for (int i = cnt + tid; i < padded; i += blockDim.x) {
        row_token[base + i] = -1;
        row_gate[base + i] = 0.0f;
    }
}

// One CTA per (token row, 2048-column chunk): each thread loads 8 bf16 of the
// row once and stores them to every destination row.
__global__ void __launch_bounds__(256) k_gather_rows_bf16(const uint4 *__restrict__ x, int64_t K, int64_t ldx,
                                                          const int32_t *__restrict__ dst_rows, int fanout,
                                                          uint4 *__restrict__ out, int64_t ld_out, int64_t M_out)
{
    const int64_t t = blockIdx.x;
    const int64_t col = ((int64_t)blockIdx.y * 256 + threadIdx.x) * 8;
    if (col >= K) return;
    const uint4 v = x[(t * ldx + col) >> 3];
    for (int j = 0; j < fanout; ++j) {
        const int64_t d = dst_rows[t * fanout + j];
        if (d >= 0 && d < M_out) out[(d * ld_out + col) >> 3] = v;
    }
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status moe_gather_rows_bf16(const void *x_dev, int64_t T, int64_t K, int64_t ldx,
                                             const int32_t *dst_rows_dev, int32_t fanout, void *out_dev,
                                             int64_t ld_out, int64_t M_out, void *stream)
{
    NVFP4_REQUIRE(T >= 0 && K >= 0 && M_out >= 0, NVFP4_ERR_INVALID_ARG, "moe_gather_rows_bf16: negative size");
    if (T == 0 || K == 0) return NVFP4_OK;
    NVFP4_REQUIRE(x_dev && dst_rows_dev && out_dev, NVFP4_ERR_INVALID_ARG, "moe_gather_rows_bf16: null pointer");
    NVFP4_REQUIRE(fanout >= 1 && fanout <= 32, NVFP4_ERR_INVALID_ARG, "moe_gather_rows_bf16: fanout must be in [1, 32]");
    NVFP4_REQUIRE(K % 8 == 0 && ldx >= K && ldx % 8 == 0 && ld_out >= K && ld_out % 8 == 0, NVFP4_ERR_ALIGNMENT,
                  "moe_gather_rows_bf16: K, ldx and ld_out must be multiples of 8 with ldx, ld_out >= K");
    NVFP4_REQUIRE(aligned16(x_dev) && aligned16(out_dev), NVFP4_ERR_ALIGNMENT,
                  "moe_gather_rows_bf16: pointers must be 16-byte aligned");
    NVFP4_REQUIRE(T < (1ll << 31), NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_gather_rows_bf16: too many rows");
    dim3 grid((unsigned)T, (unsigned)((K + 2047) / 2048));
    k_gather_rows_bf16<<<grid, 256, 0, (cudaStream_t)stream>>>(reinterpret_cast<const uint4 *>(x_dev), K, ldx,
                                                               dst_rows_dev, fanout, reinterpret_cast<uint4 *>(out_dev),
                                                               ld_out, M_out);
    return check_launch("k_gather_rows_bf16");
}

extern "C" size_t moe_route_workspace_size(int64_t T, int32_t E)
{
    (void)T;
    if (E <= 0) return 0;
    return (size_t)((E * 4 + 255) / 256 * 256);
}

extern "C" nvfp4_status moe_route(const float *logits_dev, int64_t T, int32_t E, int32_t k_r,
                                  int32_t *topk_idx_dev, float *topk_gate_dev,
                                  int32_t seg_align, int32_t *offsets_dev, int32_t *dst_row_dev,
                                  int32_t *row_token_dev, float *row_gate_dev, int64_t M_pad_max,
                                  void *workspace, size_t workspace_bytes, void *stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    NVFP4_REQUIRE(logits_dev && topk_idx_dev && topk_gate_dev && offsets_dev && dst_row_dev && row_token_dev &&
                  row_gate_dev, NVFP4_ERR_INVALID_ARG, "moe_route: null pointer");
    NVFP4_REQUIRE(T >= 0 && E >= 1 && E <= MAX_EXPERTS && k_r >= 1 && k_r <= MAX_TOPK && k_r <= E,
                  NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_route: need 1 <= E <= 256, 1 <= k_r <= min(8, E)");
    NVFP4_REQUIRE(seg_align == 128 || seg_align == 256, NVFP4_ERR_INVALID_ARG, "moe_route: seg_align must be 128 or 256");
    int64_t need_rows = (T * k_r + (int64_t)E * (seg_align - 1) + seg_align - 1) / seg_align * seg_align;
    NVFP4_REQUIRE(M_pad_max >= need_rows, NVFP4_ERR_INVALID_ARG,
                  "moe_route: M_pad_max must be >= %lld", (long long)need_rows);
    NVFP4_REQUIRE(M_pad_max < (int64_t)1 << 31, NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_route: too many rows");
    size_t need = moe_route_workspace_size(T, E);
    NVFP4_REQUIRE(workspace && workspace_bytes >= need, NVFP4_ERR_WORKSPACE,
                  "moe_route: workspace of %zu bytes required", need);
    int32_t *counts = reinterpret_cast<int32_t *>(workspace);
    if (cudaMemsetAsync(counts, 0, (size_t)E * 4, st) != cudaSuccess) return check_launch("moe_route memset");
    if (cudaMemsetAsync(row_token_dev, 0xFF, (size_t)M_pad_max * 4, st) != cudaSuccess)
        return check_launch("moe_route memset");
    if (T > 0) {
        k_route_topk<<<(unsigned)((T + 7) / 8), 256, 0, st>>>(logits_dev, T, E, k_r, topk_idx_dev, topk_gate_dev,
                                                             counts);
        if (check_launch("k_route_topk") != NVFP4_OK) return NVFP4_ERR_CUDA;
    }
    k_route_assign<<<(unsigned)E, 1024, 0, st>>>(topk_idx_dev, topk_gate_dev, T, E, k_r, counts, seg_align, offsets_dev,
                                                dst_row_dev, row_token_dev, row_gate_dev);
    return check_launch("k_route_assign");
}
