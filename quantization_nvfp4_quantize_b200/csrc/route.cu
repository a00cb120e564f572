// route.cu -- MoE top-k routing and the expert-grouped routed-row layout.
//
//   k_route_topk   one warp per token, 32 tokens per CTA ("routing block"):
//                  k_r rounds of warp argmax over the E logits (warp max of
//                  order-preserving keys, then warp min of the experts holding
//                  it: equal logits go to the lower expert), softmax over the
//                  selected logits; the
//                  block's per-expert counts in shared memory -> blkcnt.
//   k_route_scan   one warp per expert: an exclusive scan of its counts over
//                  the routing blocks, and the expert's total.
//   k_route_place  one CTA (32 warps) per routing block: the padded segment
//                  starts from the totals (segments are multiples of 128 or 256
//                  rows, the GEMM's tile height; CTA 0 also writes offsets and
//                  the padding rows' gates); each warp takes experts in turn
//                  and gives every (token, slot) routed to that expert its row
//                  = segment start + earlier blocks' count + rank in the block
//                  (ballot + popcount over the block's tokens in order).
// Rows inside an expert's segment are in ascending token order, so the layout
// is deterministic.
#include "common.cuh"

#include <algorithm>

namespace nvfp4 {

constexpr int MAX_EXPERTS = 256;
constexpr int MAX_TOPK = 8;
constexpr int RB = 32;                   // tokens per routing block (one warp per token)

__global__ void __launch_bounds__(1024) k_route_topk(const float *__restrict__ logits, int64_t T, int E, int kr,
                                                    int32_t *__restrict__ topk_idx, float *__restrict__ topk_gate,
                                                    int32_t *__restrict__ blkcnt)
{
    __shared__ int cnt[MAX_EXPERTS];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < E; i += blockDim.x) cnt[i] = 0;
    __syncthreads();
    for (int tt = warp; tt < RB; tt += (int)(blockDim.x >> 5)) {
        const int64_t t = (int64_t)blockIdx.x * RB + tt;
        if (t >= T) break;                                    // warp-uniform
        const int nslots = (E + 31) >> 5;                    // populated 32-expert slots
        // order-preserving keys of the logits (-0 taken as +0, so equal
        // logits have equal keys); 0 marks an empty slot
        uint32_t key[MAX_EXPERTS / 32];
#pragma unroll
        for (int i = 0; i < MAX_EXPERTS / 32; ++i) {
            const int e = lane + 32 * i;
            key[i] = 0u;
            if (i < nslots && e < E) {
                const uint32_t u = __float_as_uint(logits[t * E + e] + 0.0f);
                key[i] = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
            }
        }
        float sel_l[MAX_TOPK];   // fully unrolled below: stays in registers
        int sel_e[MAX_TOPK];
#pragma unroll
        for (int j = 0; j < MAX_TOPK; ++j) {
            sel_l[j] = -INFINITY;
            sel_e[j] = 0;
            if (j < kr) {
                // the largest remaining key, then the lowest expert holding it
                uint32_t lm = 0u;
#pragma unroll
                for (int i = 0; i < MAX_EXPERTS / 32; ++i) lm = max(lm, key[i]);
                const uint32_t m = __reduce_max_sync(0xffffffffu, lm);
                uint32_t le = 0xffffffffu;
#pragma unroll
                for (int i = MAX_EXPERTS / 32 - 1; i >= 0; --i)
                    if (key[i] == m) le = (uint32_t)(lane + 32 * i);
                const int be = (int)__reduce_min_sync(0xffffffffu, le);
                sel_e[j] = be;
                sel_l[j] = __uint_as_float((m & 0x80000000u) ? (m & 0x7FFFFFFFu) : ~m);
#pragma unroll
                for (int i = 0; i < MAX_EXPERTS / 32; ++i)
                    if (be == lane + 32 * i) key[i] = 0u;         // taken
            }
        }
        // softmax over the selected logits: lane j < k_r handles slot j; z is
        // summed in slot order (the same order as a serial loop)
        float my_l = sel_l[0];
        int my_e = sel_e[0];
#pragma unroll
        for (int j = 1; j < MAX_TOPK; ++j)
            if (lane == j) { my_l = sel_l[j]; my_e = sel_e[j]; }
        const float ex = lane < kr ? expf(my_l - sel_l[0]) : 0.0f;
        float z = 0.0f;
#pragma unroll
        for (int j = 0; j < MAX_TOPK; ++j) z += __shfl_sync(0xffffffffu, ex, j);
        if (lane < kr) {
            topk_idx[t * kr + lane] = my_e;
            topk_gate[t * kr + lane] = ex / z;
            atomicAdd(&cnt[my_e], 1);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += blockDim.x) blkcnt[(int64_t)i * gridDim.x + blockIdx.x] = cnt[i];   // [E][nblk]
}

// One warp per expert (4 per CTA).  blkcnt [E x nblk] (expert-major, so each
// expert's counts are contiguous) is turned in place into each block's
// exclusive prefix within its expert; tot[e] = the expert's routed rows.
__global__ void __launch_bounds__(128) k_route_scan(int32_t *__restrict__ blkcnt, int nblk, int E,
                                                    int32_t *__restrict__ tot)
{
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * 4 + (threadIdx.x >> 5);
    if (e >= E) return;                                      // warp-uniform
    int running = 0;
    for (int b0 = 0; b0 < nblk; b0 += 32 * 8) {
        // lane l takes 8 consecutive blocks: independent loads, a
        // thread-local prefix, then a warp scan of the lane sums
        int c[8], sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int b = b0 + lane * 8 + i;
            c[i] = b < nblk ? blkcnt[(int64_t)e * nblk + b] : 0;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) sum += c[i];
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int pre = running + incl - sum;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int b = b0 + lane * 8 + i;
            if (b < nblk) blkcnt[(int64_t)e * nblk + b] = pre;
            pre += c[i];
        }
        running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) tot[e] = running;
}

__global__ void __launch_bounds__(1024) k_route_place(const int32_t *__restrict__ topk_idx,
                                                     const float *__restrict__ topk_gate, int64_t T, int E, int kr,
                                                     const int32_t *__restrict__ blkoff,
                                                     const int32_t *__restrict__ tot, int align,
                                                     int32_t *__restrict__ offsets,
                                                     int32_t *__restrict__ dst_row, int32_t *__restrict__ row_token,
                                                     float *__restrict__ row_gate)
{
    __shared__ int32_t sidx[MAX_TOPK * RB];          // [slot][token in block]
    __shared__ int sbase[MAX_EXPERTS + 1];           // padded segment starts
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = (int)(blockDim.x >> 5);
    const int64_t t0 = (int64_t)blockIdx.x * RB;
    const int nt = (int)std::min<int64_t>(RB, T - t0);
    for (int i = threadIdx.x; i < MAX_TOPK * RB; i += blockDim.x) {
        const int j = i / RB, tt = i - j * RB;
        sidx[i] = (j < kr && tt < nt) ? topk_idx[(t0 + tt) * kr + j] : -1;
    }
    if (warp == 0) {
        // padded exclusive scan of the expert totals: lane l takes 8 experts
        int c[MAX_EXPERTS / 32], sum = 0;
#pragma unroll
        for (int i = 0; i < MAX_EXPERTS / 32; ++i) {
            const int e = lane * (MAX_EXPERTS / 32) + i;
            c[i] = e < E ? (tot[e] + align - 1) / align * align : 0;
            sum += c[i];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int pre = incl - sum;
#pragma unroll
        for (int i = 0; i < MAX_EXPERTS / 32; ++i) {
            const int e = lane * (MAX_EXPERTS / 32) + i;
            if (e < E) sbase[e] = pre;
            pre += c[i];
        }
        if (lane == 31) sbase[E] = incl;                     // total padded rows
    }
    __syncthreads();
    if (blockIdx.x == 0) {
        for (int e = threadIdx.x; e <= E; e += blockDim.x) offsets[e] = sbase[e];
        // gates of the padding rows at the end of each segment
        for (int i = threadIdx.x; i < E * align; i += blockDim.x) {
            const int e = i / align, r = sbase[e] + tot[e] + (i - e * align);
            if (r < sbase[e + 1]) row_gate[r] = 0.0f;
        }
    }
    // the warp's experts are e = warp + nwarps * i; lane i prefetches the
    // row base of expert i of the warp (segment start + earlier blocks)
    int mybase = 0;
    {
        const int e = warp + nwarps * lane;
        if (e < E) mybase = sbase[e] + blkoff[(int64_t)e * gridDim.x + blockIdx.x];
    }
    static_assert(RB == 32, "one ballot per expert covers the block");
    for (int i = 0, e = warp; e < E; ++i, e += nwarps) {
        const int run = __shfl_sync(0xffffffffu, mybase, i);
        const int tt = lane;
        int slot = -1;
#pragma unroll
        for (int j = 0; j < MAX_TOPK; ++j)
            if (sidx[j * RB + tt] == e) slot = j;
        const unsigned bal = __ballot_sync(0xffffffffu, slot >= 0);
        if (slot >= 0) {
            const int row = run + __popc(bal & ((1u << lane) - 1u));
            const int64_t t = t0 + tt;
            dst_row[t * kr + slot] = row;
            row_token[row] = (int32_t)t;
            row_gate[row] = topk_gate[t * kr + slot];
        }
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

// Every routed row r < M_out gets token row_token[r] of x, or zeros for a
// padding row (row_token < 0): the copy is complete whatever the routing
// left in the buffer before.
__global__ void __launch_bounds__(256) k_routed_rows_bf16(const uint4 *__restrict__ x, int64_t T, int64_t K,
                                                          int64_t ldx, const int32_t *__restrict__ row_token,
                                                          uint4 *__restrict__ out, int64_t ld_out)
{
    const int64_t r = blockIdx.x;
    const int64_t col = ((int64_t)blockIdx.y * 256 + threadIdx.x) * 8;
    if (col >= K) return;
    const int32_t t = row_token[r];
    const uint4 v = (t >= 0 && t < T) ? x[((int64_t)t * ldx + col) >> 3] : make_uint4(0u, 0u, 0u, 0u);
    out[(r * ld_out + col) >> 3] = v;
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
    if (E <= 0 || T < 0) return 0;
    const int64_t nblk = std::max<int64_t>(1, (T + RB - 1) / RB);
    return (size_t)(((nblk + 1) * E * 4 + 255) / 256 * 256);          // block counts [E x nblk] + totals [E]
}

extern "C" nvfp4_status moe_route(const float *logits_dev, int64_t T, int32_t E, int32_t k_r,
                                  int32_t *topk_idx_dev, float *topk_gate_dev,
                                  int32_t seg_align, int32_t *offsets_dev, int32_t *dst_row_dev,
                                  int32_t *row_token_dev, float *row_gate_dev, int64_t M_pad_max,
                                  void *workspace, size_t workspace_bytes, void *stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    NVFP4_REQUIRE(offsets_dev && row_token_dev && row_gate_dev &&
                  (T == 0 || (logits_dev && topk_idx_dev && topk_gate_dev && dst_row_dev)), NVFP4_ERR_INVALID_ARG,
                  "moe_route: null pointer");
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
    int32_t *blkcnt = reinterpret_cast<int32_t *>(workspace);
    const int nblk = (int)((T + RB - 1) / RB);
    if (cudaMemsetAsync(row_token_dev, 0xFF, (size_t)M_pad_max * 4, st) != cudaSuccess)
        return check_launch("moe_route memset");
    if (nblk > 0) {
        k_route_topk<<<(unsigned)nblk, 1024, 0, st>>>(logits_dev, T, E, k_r, topk_idx_dev, topk_gate_dev, blkcnt);
        if (check_launch("k_route_topk") != NVFP4_OK) return NVFP4_ERR_CUDA;
    }
    int32_t *tot = blkcnt + (int64_t)nblk * E;
    if (nblk == 0) {
        // no tokens: every expert segment is empty
        if (cudaMemsetAsync(offsets_dev, 0, (size_t)(E + 1) * 4, st) != cudaSuccess) return check_launch("moe_route memset");
        return NVFP4_OK;
    }
    k_route_scan<<<(unsigned)((E + 3) / 4), 128, 0, st>>>(blkcnt, nblk, E, tot);
    if (check_launch("k_route_scan") != NVFP4_OK) return NVFP4_ERR_CUDA;
    k_route_place<<<(unsigned)nblk, 1024, 0, st>>>(topk_idx_dev, topk_gate_dev, T, E, k_r, blkcnt, tot, seg_align,
                                                  offsets_dev, dst_row_dev, row_token_dev, row_gate_dev);
    return check_launch("k_route_place");
}

extern "C" nvfp4_status moe_routed_rows_bf16(const void *x_dev, int64_t T, int64_t K, int64_t ldx,
                                             const int32_t *row_token_dev, void *out_dev, int64_t ld_out,
                                             int64_t M_out, void *stream)
{
    NVFP4_REQUIRE(T >= 0 && K >= 0 && M_out >= 0, NVFP4_ERR_INVALID_ARG, "moe_routed_rows_bf16: negative size");
    if (M_out == 0 || K == 0) return NVFP4_OK;
    NVFP4_REQUIRE(row_token_dev && out_dev && (T == 0 || x_dev), NVFP4_ERR_INVALID_ARG,
                  "moe_routed_rows_bf16: null pointer");
    NVFP4_REQUIRE(K % 8 == 0 && ldx >= K && ldx % 8 == 0 && ld_out >= K && ld_out % 8 == 0, NVFP4_ERR_ALIGNMENT,
                  "moe_routed_rows_bf16: K, ldx and ld_out must be multiples of 8 with ldx, ld_out >= K");
    NVFP4_REQUIRE((T == 0 || aligned16(x_dev)) && aligned16(out_dev), NVFP4_ERR_ALIGNMENT,
                  "moe_routed_rows_bf16: pointers must be 16-byte aligned");
    NVFP4_REQUIRE(M_out < (1ll << 31), NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_routed_rows_bf16: too many rows");
    dim3 grid((unsigned)M_out, (unsigned)((K + 2047) / 2048));
    k_routed_rows_bf16<<<grid, 256, 0, (cudaStream_t)stream>>>(reinterpret_cast<const uint4 *>(x_dev), T, K, ldx,
                                                               row_token_dev, reinterpret_cast<uint4 *>(out_dev), ld_out);
    return check_launch("k_routed_rows_bf16");
}
