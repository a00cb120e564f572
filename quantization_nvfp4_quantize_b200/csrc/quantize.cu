// quantize.cu -- bandwidth-bound NVFP4 kernels of the QUADS rollout path.
//
//   k_amax              per-tensor (per-group) max |x|          (HBM read, 2 B/elem)
//   k_quantize          one streaming pass: E2M1 codes + swizzled E4M3 scales
//                       (+ bf16 QDQ values, + per-channel residual score
//                       partials), fanned out to routed rows   (2 B read,
//                       0.5625 B/elem written per destination)
//   k_score_reduce      partial scores -> score[K] (binary64, fixed order)
//   k_select_topk       radix select of the rac_k largest scores, compacted in
//                       ascending channel order (one CTA)
//   k_rac_residual      rho[dst, j] = bf16(R[r, S_j] / s_t)
//   k_gather_w_channels w_sel[e, n, j] = bf16(e2m1 * sf) of selected channels
//
// Layout of k_quantize: a CTA is 8 warps on one 256-channel column chunk and
// one range of rows.  Each lane owns 8 consecutive channels (one 16-byte
// load), two lanes form a 16-element block (amax by one xor-shuffle), a warp
// reads 512 contiguous bytes of a row.  Lanes keep their channels' residual
// sums across rows (binary32 for up to 4 rows, then binary64; each warp keeps
// 4 rows' loads in flight), the CTA reduces its
// 8 warps in shared memory and writes one partial per channel; partials are
// summed in a fixed order by k_score_reduce, so scores are deterministic.
#include "common.cuh"
#include "ptx.cuh"

#include <algorithm>
#include <mutex>

namespace nvfp4 {

constexpr int QWORKERS = 8;           // quantizing warps per CTA
constexpr int QTHREADS = (QWORKERS + 1) * 32;   // + one TMA producer warp
constexpr int QCHUNK = 256;           // channels per CTA column chunk (one 512-byte tile row)
constexpr int QCTAS_PER_SM = 3;       // resident CTAs per SM the grid is sized for (one wave)
constexpr int QSTAGES = 4;            // TMA tile ring depth
constexpr int QROWS = 32;             // rows per TMA tile
constexpr int QRPW = QROWS / QWORKERS;   // tile rows per worker warp
constexpr uint32_t QPITCH = QCHUNK * 2;  // bytes per tile row
constexpr uint32_t QTILE = QPITCH * QROWS;
constexpr uint32_t QSMEM = QSTAGES * QTILE;   // 64 KB of tiles per CTA
constexpr int MAX_EXPERTS = 256;      // expert sets of nvfp4_quantize_experts

__device__ __forceinline__ __nv_bfloat162 bf162_bits(uint32_t w) { return *reinterpret_cast<__nv_bfloat162 *>(&w); }
__device__ __forceinline__ __nv_bfloat16 bf16_from_bits(uint32_t w) { return __ushort_as_bfloat16((unsigned short)w); }

// -------------------------------------------------------------------- amax

// max |x| per group.  |bf16| bit patterns order like their values, so the
// maximum is taken on pairs of 16-bit integers; every thread keeps 4
// independent 16-byte loads in flight.  Contiguous tensors (ldx == K) are
// swept as one flat array; otherwise warps take whole rows.
__device__ __forceinline__ uint32_t absmax_pairs(uint32_t m2, uint4 u)
{
    const uint32_t a = __vmaxu2(u.x & 0x7FFF7FFFu, u.y & 0x7FFF7FFFu);
    const uint32_t b = __vmaxu2(u.z & 0x7FFF7FFFu, u.w & 0x7FFF7FFFu);
    return __vmaxu2(m2, __vmaxu2(a, b));
}

__global__ void __launch_bounds__(256) k_amax(const __nv_bfloat16 *__restrict__ x, int64_t ldx,
                                              int64_t M, int64_t K, const int32_t *__restrict__ m_valid,
                                              int64_t group_stride, unsigned int *__restrict__ amax_bits)
{
    int64_t Me = M;
    if (m_valid) Me = min(Me, (int64_t)max(*m_valid, 0));
    const __nv_bfloat16 *xg = x + (int64_t)blockIdx.y * group_stride;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
    uint32_t m2 = 0u;
    if (ldx == K) {
        const uint4 *v = reinterpret_cast<const uint4 *>(xg);
        const int64_t total = Me * (K / 8);
        int64_t i = tid;
        for (; i + 3 * nthr < total; i += 4 * nthr) {
            const uint4 u0 = __ldg(v + i), u1 = __ldg(v + i + nthr), u2 = __ldg(v + i + 2 * nthr),
                        u3 = __ldg(v + i + 3 * nthr);
            m2 = absmax_pairs(absmax_pairs(absmax_pairs(absmax_pairs(m2, u0), u1), u2), u3);
        }
        for (; i < total; i += nthr) m2 = absmax_pairs(m2, __ldg(v + i));
    } else {
        const int lane = threadIdx.x & 31;
        const int vpr = (int)(K / 8);
        for (int64_t r = tid >> 5; r < Me; r += nthr >> 5) {
            const uint4 *row = reinterpret_cast<const uint4 *>(xg + r * ldx);
            for (int j = lane; j < vpr; j += 32) m2 = absmax_pairs(m2, __ldg(row + j));
        }
    }
    float m = fmaxf(bf16lo(m2), bf16hi(m2));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float wm[8];
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = wm[0];
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) b = fmaxf(b, wm[w]);
        // non-negative floats order like their bit patterns
        atomicMax(amax_bits + blockIdx.y, __float_as_uint(b));
    }
}

// --------------------------------------------------------------- quantize

struct QuantParams {
    int64_t ldx, M, K;
    const int32_t *m_valid;
    const float *s_t_in;             // per group, or null
    const unsigned int *amax_bits;   // per group (max |x| as float bits), used when s_t_in is null
    float *s_t_out;                  // per group
    const int32_t *dst_rows;
    int fanout;
    int64_t M_out;                   // rows of the outputs: destination rows >= M_out are skipped
    uint8_t *codes;
    uint8_t *scales;
    __nv_bfloat16 *qdq;
    double *partials;                // [gridDim.y x K]
    int64_t rows_per_cta;
    int64_t codes_gstride, scales_gstride, qdq_gstride;
    int box_inner;                   // channels per TMA box row (min(256, K))
    int32_t *dev_status;
};

// Bounded mbarrier wait for the streaming kernels (1 s); false on timeout or
// when another thread of the CTA has given up.
__device__ __forceinline__ bool qwait(uint32_t bar, uint32_t parity, volatile int *abort_flag, int32_t *dev_status,
                                      bool ignore_abort = false)
{
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 63u) {
            if (!ignore_abort && *abort_flag) return false;
            const uint64_t now = globaltimer_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > 1000000000ull) {
                *abort_flag = 1;
                report_status(dev_status, NVFP4_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// Byte offset of scale entry (r, c) in the scale-factor layout, 32-bit
// (callers keep rows x K/16 below 2^31).
__device__ __forceinline__ uint32_t sf_off32(uint32_t r, uint32_t c, uint32_t K)
{
    return ((r >> 7) * (K >> 6) + (c >> 2)) * 512u + (r & 31u) * 16u + ((r >> 5) & 3u) * 4u + (c & 3u);
}

// One CTA = 8 worker warps on one 256-channel column chunk and one range of
// rows, plus a producer warp whose lane 0 streams 32-row x 256-channel bf16
// tiles (16 KB, zero-filled past K) through a 4-stage shared-memory ring with
// TMA.  Worker w quantizes tile rows w, w+8, w+16, w+24, each lane 8 channels
// (a lane pair is one 16-element block).
//   SCORE  accumulate the channels' residual sums of squares
//   QDQ    write bf16(xhat) (weight fake quantization)
//   FAN    write the codes and scales to the routed rows dst_rows instead
// With dst_rows, each destination row gets the warp's codes as one coalesced
// 128-byte line (a 4-byte store per lane) and its 4 scale words as 4-byte
// stores, one per lane; the destinations' row offsets are looked up once per
// tile.
// Offsets inside a tensor are 32-bit (the host checks the sizes).
template <bool SCORE, bool QDQ, bool FAN>
__global__ void __launch_bounds__(QTHREADS, QCTAS_PER_SM) k_quantize(const __grid_constant__ CUtensorMap tm_x,
                                                                     QuantParams p)
{
    extern __shared__ __align__(128) uint8_t qsm[];              // QSTAGES x QROWS x 256 bf16
    __shared__ uint64_t full_bar[QSTAGES], empty_bar[QSTAGES];
    __shared__ int abort_sm;
    __shared__ float4 btab[128];                                  // per E4M3 code: d, rlo, rhi, sf_h2
    __shared__ int32_t fdst[QWORKERS][QRPW][32];                  // fan-out rows of a warp's 4 rows (-1: none)
    __shared__ uint32_t fsrow[QWORKERS][QRPW][32];                // their row parts of the scale-atom offset
    volatile int *abort_flag = &abort_sm;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = blockIdx.z;
    const uint32_t K = (uint32_t)p.K;
    const uint32_t c0 = blockIdx.x * QCHUNK;
    const uint32_t c = c0 + lane * 8;                             // first channel of this lane
    const bool active = c < K;

    const float s_t = p.s_t_in ? p.s_t_in[g] : tensor_scale_from_amax(__uint_as_float(p.amax_bits[g]));
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 && p.s_t_out) p.s_t_out[g] = s_t;
    const float2 r6 = recip_bracket(__fmul_rn(6.0f, s_t));

    int64_t Me = p.M;
    if (p.m_valid) Me = min(Me, (int64_t)max(*p.m_valid, 0));
    const int64_t r0l = (int64_t)blockIdx.y * p.rows_per_cta;
    const int64_t r1l = min(Me, r0l + p.rows_per_cta);
    const int n_iter = r1l > r0l ? (int)((r1l - r0l + QROWS - 1) / QROWS) : 0;
    const uint32_t r0 = (uint32_t)r0l, r1 = (uint32_t)max(r1l, r0l);
    const int64_t row_base = (int64_t)g * p.M;                   // row of this group in the tensor map

    uint8_t *codes = p.codes ? p.codes + g * p.codes_gstride : nullptr;
    uint8_t *scales = p.scales ? p.scales + g * p.scales_gstride : nullptr;
    __nv_bfloat16 *qdq = QDQ ? p.qdq + g * p.qdq_gstride : nullptr;
    const int fanout = FAN ? p.fanout : 0;
    const uint32_t M_out = (uint32_t)p.M_out;

    // E4M3 code -> the block's constants: a block scale takes at most 127
    // values per tensor, so each is computed once here rather than per block.
    if (threadIdx.x < 128) {
        const BlockConst b = block_const(threadIdx.x, s_t);
        btab[threadIdx.x] = make_float4(b.d, b.rlo, b.rhi, __uint_as_float(b.sf_h2));
    }
    if (threadIdx.x == 0) {
        for (int st = 0; st < QSTAGES; ++st) {
            ptx::mbar_init(ptx::smem_u32(&full_bar[st]), 1);
            ptx::mbar_init(ptx::smem_u32(&empty_bar[st]), QWORKERS);
        }
        abort_sm = 0;
        ptx::fence_mbar_init();
        ptx::fence_proxy_async_smem();
    }
    __syncthreads();

    float2 acc32[4];
    double acc64[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc32[i] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc64[i] = 0.0;

    if (warp == QWORKERS) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            ptx::prefetch_tmap(&tm_x);
            int issued = 0;
            for (int it = 0; it < n_iter; ++it) {
                const int st = it % QSTAGES;
                // the stage's previous tile has been released by every worker
                if (it >= QSTAGES &&
                    !qwait(ptx::smem_u32(&empty_bar[st]), ((uint32_t)(it / QSTAGES) & 1u) ^ 1u, abort_flag,
                           p.dev_status))
                    break;
                const uint32_t fb = ptx::smem_u32(&full_bar[st]);
                ptx::mbar_arrive_expect_tx(fb, QTILE);
                ptx::tma_load_2d(ptx::smem_u32(qsm + st * QTILE), &tm_x, (int32_t)c0,
                                 (int32_t)(row_base + r0l + (int64_t)it * QROWS), fb);
                ++issued;
            }
            // every issued copy lands before the CTA ends (each stage's last
            // tile: its phase is the barrier's latest)
            for (int j = max(0, issued - QSTAGES); j < issued; ++j)
                qwait(ptx::smem_u32(&full_bar[j % QSTAGES]), (uint32_t)(j / QSTAGES) & 1u, abort_flag, p.dev_status,
                      true);
        }
    } else {
        // -------------------------------------------------------- workers
        const uint32_t kb0 = c >> 4;            // first block of the lane octet's 4-block group (lanes 8j)
        const uint32_t wcol = (c0 >> 4) + 4 * (lane & 3);          // fan-out: first scale column of word lane % 4
        const bool wcol_ok = wcol < (K >> 4);
        const uint32_t wcol_off = sf_off32(0u, wcol, K);             // column part of the word's offset
        const uint32_t code_col = c >> 1;
        for (int it = 0; it < n_iter; ++it) {
            const int st = it % QSTAGES;
            const uint32_t ph = (uint32_t)(it / QSTAGES) & 1u;
            bool ok = true;
            if (lane == 0) ok = qwait(ptx::smem_u32(&full_bar[st]), ph, abort_flag, p.dev_status);
            if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) == 0) break;
            const uint8_t *tile = qsm + st * QTILE + warp * QPITCH + lane * 16;
            const uint32_t rt = r0 + (uint32_t)it * QROWS + (uint32_t)warp;   // this warp's first row of the tile
            if (FAN) {
#pragma unroll
                for (int i = 0; i < QRPW; ++i) {
                    const uint32_t r = rt + (uint32_t)(i * QWORKERS);
                    if (lane < fanout) {
                        int32_t dst = r < r1 ? p.dst_rows[(int64_t)r * fanout + lane] : -1;
                        if (dst >= 0 && (uint32_t)dst >= M_out) dst = -1;
                        fdst[warp][i][lane] = dst;
                        fsrow[warp][i][lane] = dst >= 0 ? sf_off32((uint32_t)dst, 0u, K) : 0u;
                    }
                }
                __syncwarp();
            }
            // the fan-out instance runs smaller as a rolled loop
            constexpr int ROW_UNROLL = FAN ? 1 : QRPW;
#pragma unroll ROW_UNROLL
            for (int i = 0; i < QRPW; ++i) {
                const uint32_t r = rt + (uint32_t)(i * QWORKERS);
                if (r >= r1) break;                                   // warp-uniform
                const uint4 u = active ? *reinterpret_cast<const uint4 *>(tile + i * QWORKERS * QPITCH)
                                       : make_uint4(0u, 0u, 0u, 0u);
                const float2 v[4] = {bf16x2_to_f2(u.x), bf16x2_to_f2(u.y), bf16x2_to_f2(u.z), bf16x2_to_f2(u.w)};
                float m = fmaxf(fmaxf(fmaxf(fabsf(v[0].x), fabsf(v[0].y)), fmaxf(fabsf(v[1].x), fabsf(v[1].y))),
                                fmaxf(fmaxf(fabsf(v[2].x), fabsf(v[2].y)), fmaxf(fabsf(v[3].x), fabsf(v[3].y))));
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
                const uint32_t sf_code = block_scale_code(m, s_t, r6);
                const float4 bt = btab[sf_code];
                const BlockConst b{bt.x, bt.y, bt.z, __float_as_uint(bt.w)};
                const uint32_t cw = element_codes8(v, b);
                if (SCORE || QDQ) {
                    float2 xh[4];
                    dequant8(cw, b.sf_h2, s_t, xh);
                    if (SCORE) {
                        float2 R[4];
                        residual8(v, xh, R);
#pragma unroll
                        for (int k = 0; k < 4; ++k) acc32[k] = fma2(R[k], R[k], acc32[k]);
                    }
                    if (QDQ && active) {
                        uint4 o;
                        __nv_bfloat162 h;
                        h = __floats2bfloat162_rn(xh[0].x, xh[0].y); o.x = *reinterpret_cast<uint32_t *>(&h);
                        h = __floats2bfloat162_rn(xh[1].x, xh[1].y); o.y = *reinterpret_cast<uint32_t *>(&h);
                        h = __floats2bfloat162_rn(xh[2].x, xh[2].y); o.z = *reinterpret_cast<uint32_t *>(&h);
                        h = __floats2bfloat162_rn(xh[3].x, xh[3].y); o.w = *reinterpret_cast<uint32_t *>(&h);
                        *reinterpret_cast<uint4 *>(qdq + r * K + c) = o;
                    }
                }
                if (!codes) continue;
                // the 4 scale codes of blocks kb0..kb0+3 on lanes 8j
                uint32_t sw = sf_code | (__shfl_down_sync(0xffffffffu, sf_code, 2) << 8);
                sw |= __shfl_down_sync(0xffffffffu, sw, 4) << 16;
                if (!FAN) {
                    if (active) {
                        *reinterpret_cast<uint32_t *>(codes + r * (K >> 1) + (c >> 1)) = cw;
                        if ((lane & 7) == 0) *reinterpret_cast<uint32_t *>(scales + sf_off32(r, kb0, K)) = sw;
                    }
                } else {
                    // fan-out: the row's codes, one 128-byte line per destination
                    for (int d = 0; d < fanout; ++d) {
                        const int32_t dst = fdst[warp][i][d];
                        if (dst >= 0 && active)
                            *reinterpret_cast<uint32_t *>(codes + (uint64_t)(uint32_t)dst * (K >> 1) + code_col) = cw;
                    }
                    // scale words: lane l writes word l % 4 of destination l / 4 (+ 8 per round)
                    const uint32_t word = __shfl_sync(0xffffffffu, sw, (lane & 3) * 8);
                    for (int d = lane >> 2; d < fanout; d += 8) {
                        if (fdst[warp][i][d] >= 0 && wcol_ok)
                            *reinterpret_cast<uint32_t *>(scales + fsrow[warp][i][d] + wcol_off) = word;
                    }
                }
            }
            if (SCORE) {
                // at most QRPW = 4 rows were summed in binary32
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    acc64[2 * k] += (double)acc32[k].x;
                    acc64[2 * k + 1] += (double)acc32[k].y;
                    acc32[k] = make_float2(0.0f, 0.0f);
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&empty_bar[st]));
        }
    }

    if (SCORE) {
        __syncthreads();                                          // the stage ring is free: reuse it
        double *red = reinterpret_cast<double *>(qsm);            // [8 workers][256 channels]
        if (warp < QWORKERS) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                red[warp * QCHUNK + lane * 8 + i] = acc64[i] + (double)((i & 1) ? acc32[i >> 1].y : acc32[i >> 1].x);
        }
        __syncthreads();
        const uint32_t ch = c0 + threadIdx.x;
        if (threadIdx.x < QCHUNK && ch < K) {
            double sum = 0.0;
#pragma unroll
            for (int w = 0; w < QWORKERS; ++w) sum += red[w * QCHUNK + threadIdx.x];
            p.partials[(int64_t)blockIdx.y * K + ch] = sum;
        }
    }
}

// ----------------------------------------------------------- score reduce

// score[c] = sum over the P row-range partials of channel c.  A CTA takes 32
// channels (one per lane); its 8 warps sum interleaved eighths of the
// partials (warp w: q = w, w + 8, ...), then warp 0 adds the 8 sums in warp
// order: a fixed order, so the scores are deterministic.
constexpr int SR_WARPS = 8;

__global__ void __launch_bounds__(SR_WARPS * 32) k_score_reduce(const double *__restrict__ partials, int64_t P,
                                                               int64_t K, double *__restrict__ score)
{
    __shared__ double part[SR_WARPS][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t c = (int64_t)blockIdx.x * 32 + lane;
    double s = 0.0;
    if (c < K)
        for (int64_t q = warp; q < P; q += SR_WARPS) s += partials[q * K + c];
    part[warp][lane] = s;
    __syncthreads();
    if (warp == 0 && c < K) {
        double t = part[0][lane];
#pragma unroll
        for (int w = 1; w < SR_WARPS; ++w) t += part[w][lane];
        score[c] = t;
    }
}

// Per-expert scores from row-group partials: row group q covers rows
// [q*rpc, (q+1)*rpc), inside one expert segment (segments are multiples of
// rpc); score[e, c] sums expert e's groups in order.
__global__ void k_score_reduce_experts(const double *__restrict__ partials, const int32_t *__restrict__ offsets,
                                      int64_t rpc, int64_t K, double *__restrict__ score)
{
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int e = blockIdx.y;
    if (c >= K) return;
    const int64_t q0 = offsets[e] / rpc, q1 = offsets[e + 1] / rpc;
    double s = 0.0;
    for (int64_t q = q0; q < q1; ++q) s += partials[q * K + c];
    score[(int64_t)e * K + c] = s;
}

// ---------------------------------------------------------------- top-k

__device__ __forceinline__ int block_exclusive_scan(int v, int *smem_warp, int &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    __syncthreads();
    if (lane == 31) smem_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? smem_warp[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int t = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += t;
        }
        if (lane < nw) smem_warp[lane] = wi - w;     // exclusive warp offsets
        if (lane == nw - 1) smem_warp[32] = wi;      // total
    }
    __syncthreads();
    int r = smem_warp[warp] + incl - v;
    total = smem_warp[32];
    return r;
}

// One CTA of 1024 threads.  Scores are non-negative binary64, whose bit
// patterns order like their values; an MSB-first radix select over 8-bit
// digits finds the k-th largest key (stopping early once a single key holds
// the selected prefix: that key is the k-th), then channels are taken in
// ascending index order: every key above it, and the lowest-index keys equal
// to it.
__global__ void __launch_bounds__(1024) k_select_topk(const double *__restrict__ score, int K, int k,
                                                      int32_t *__restrict__ sel)
{
    extern __shared__ unsigned long long keys[];
    __shared__ unsigned int hist[256];
    __shared__ int scan_tmp[33];
    __shared__ int s_digit, s_rem, s_cnt;
    __shared__ unsigned long long s_key;
    const int tid = threadIdx.x;
    if (k <= 0) return;
    score += (int64_t)blockIdx.x * K;                 // one score vector (and set) per block
    sel += (int64_t)blockIdx.x * k;
    for (int i = tid; i < K; i += blockDim.x) keys[i] = (unsigned long long)__double_as_longlong(score[i]);
    if (tid == 0) s_rem = k;
    __syncthreads();

    unsigned long long prefix = 0ull, mask = 0ull;
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < K; i += blockDim.x) {
            unsigned long long key = keys[i];
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255ull], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            // warp 0 finds the digit: lane l owns bins 255-8l .. 248-8l (descending)
            const int rem = s_rem;
            unsigned int cnt[8], tot = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) { cnt[b] = hist[255 - 8 * tid - b]; tot += cnt[b]; }
            unsigned int incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                unsigned int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (tid >= o) incl += v;
            }
            unsigned int above = incl - tot;          // keys in higher bins than this lane's
            bool mine = above < (unsigned)rem && (unsigned)rem <= incl;
            if (mine) {
                unsigned int a = above;
                int b = 0;
                for (; b < 7; ++b) {
                    if (a + cnt[b] >= (unsigned)rem) break;
                    a += cnt[b];
                }
                s_digit = 255 - 8 * tid - b;
                s_rem = rem - (int)a;
                s_cnt = (int)cnt[b];
            }
        }
        __syncthreads();
        prefix |= (unsigned long long)s_digit << shift;
        mask |= 0xFFull << shift;
        if (s_cnt == 1 && shift > 0) {
            // one key holds the prefix: it is the k-th largest (s_rem == 1)
            for (int i = tid; i < K; i += blockDim.x)
                if ((keys[i] & mask) == prefix) s_key = keys[i];
            __syncthreads();
            prefix = s_key;
            break;
        }
    }
    const unsigned long long kth = prefix;
    const int take_eq = s_rem;          // keys equal to kth to take, lowest index first

    // contiguous ranges per thread
    const int per = (K + blockDim.x - 1) / blockDim.x;
    const int i0 = min(K, tid * per), i1 = min(K, i0 + per);
    int n_eq = 0;
    for (int i = i0; i < i1; ++i) n_eq += (keys[i] == kth);
    int tot;
    int eq_before = block_exclusive_scan(n_eq, scan_tmp, tot);
    int n_take = 0;
    {
        int e = eq_before;
        for (int i = i0; i < i1; ++i) {
            unsigned long long key = keys[i];
            if (key > kth) ++n_take;
            else if (key == kth) { if (e < take_eq) ++n_take; ++e; }
        }
    }
    int take_before = block_exclusive_scan(n_take, scan_tmp, tot);
    {
        int e = eq_before, pos = take_before;
        for (int i = i0; i < i1; ++i) {
            unsigned long long key = keys[i];
            bool t = false;
            if (key > kth) t = true;
            else if (key == kth) { t = e < take_eq; ++e; }
            if (t && pos < k) sel[pos++] = i;
        }
    }
}

// --------------------------------------------------------- RAC residual

// Block constants of the E4M3 scale codes 0..127 (every code a non-negative
// block scale takes) for tensor scale s_t, filled by the CTA's first 128
// threads; the caller synchronizes before reading.
__device__ __forceinline__ void fill_block_table(float4 *tab, float s_t)
{
    if (threadIdx.x < 128) {
        const BlockConst b = block_const(threadIdx.x, s_t);
        tab[threadIdx.x] = make_float4(b.d, b.rlo, b.rhi, __uint_as_float(b.sf_h2));
    }
}

// E4M3 scale code of a 16-block given as its two 16-byte halves, with the
// arithmetic of k_quantize.  The block max is taken on bf16 pairs
// (max.bf16x2 ignores a NaN operand, as fmaxf does).
__device__ __forceinline__ uint32_t block_code16(uint4 u0, uint4 u1, float s_t, float2 r6)
{
    const uint32_t mk = 0x7FFF7FFFu;
    const __nv_bfloat162 m2 = __hmax2(
        __hmax2(__hmax2(bf162_bits(u0.x & mk), bf162_bits(u0.y & mk)), __hmax2(bf162_bits(u0.z & mk), bf162_bits(u0.w & mk))),
        __hmax2(__hmax2(bf162_bits(u1.x & mk), bf162_bits(u1.y & mk)), __hmax2(bf162_bits(u1.z & mk), bf162_bits(u1.w & mk))));
    const uint32_t mb = *reinterpret_cast<const uint32_t *>(&m2);
    return block_scale_code(fmaxf(bf16lo(mb), bf16hi(mb)), s_t, r6);
}

static __device__ __noinline__ uint32_t rho_bf16_div(float R, float s_t)
{
    const __nv_bfloat16 h = __float2bfloat16_rn(__fdiv_rn(R, s_t));
    return *reinterpret_cast<const uint16_t *>(&h);
}

// bf16(fl(R / s_t)) as a 16-bit pattern; rs = recip_bracket(s_t).  Both
// roundings are monotone, so when the bracketing products round to the same
// bf16 that is the value of the division (else the division is evaluated).
__device__ __forceinline__ uint32_t rho_bf16(float R, float s_t, float2 rs)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(R, rs.x), __fmul_rn(R, rs.y));
    const uint32_t w = *reinterpret_cast<const uint32_t *>(&h);
    if ((w & 0xFFFFu) == (w >> 16)) return w & 0xFFFFu;
    return rho_bf16_div(R, s_t);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// E2M1 codes of (lo, hi) in bits 0..3 / 4..7.
__device__ __forceinline__ uint32_t e2m1x2_bits(float lo, float hi)
{
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "cvt.u32.u8 %0, t;\n\t}"
        : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// R = fl(x - xhat) of one element of a block with constants b: the code of
// fl(x / d) from the bracketing products (the division when they differ),
// xhat = fl(fl(e2m1 * sf) * s_t) with the e2m1 * sf product exact in f16.
__device__ __forceinline__ float element_residual(float xv, const BlockConst &b, float s_t)
{
    uint32_t c = e2m1x2_bits(__fmul_rn(xv, b.rlo), __fmul_rn(xv, b.rhi));
    if ((c >> 4) != (c & 15u)) {
        const uint32_t q = element_code1_div(xv, b.d);
        c = q * 0x11u;
    }
    uint32_t h2;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.u8.u32 t, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, t;\n\t"
        "mul.rn.f16x2 %0, %0, %2;\n\t}"
        : "=r"(h2) : "r"(c), "r"(b.sf_h2));
    const float qsf = __low2float(*reinterpret_cast<const __half2 *>(&h2));
    return __fsub_rn(xv, __fmul_rn(qsf, s_t));
}

constexpr int RC_WARPS = 8;            // warps per CTA, each streaming its own rows
constexpr int RC_CHUNK = 2048;         // channels of a row staged at a time (4 KB)
constexpr int RC_GROUPS = 8;           // 4-column output groups a lane holds: windows of 1024 columns
constexpr int RC_WIN = RC_GROUPS * 128;

// Dynamic shared memory of k_rac_residual: two row pieces per warp.
static size_t rac_residual_smem(int64_t K)
{
    return (size_t)RC_WARPS * 2 * (size_t)std::min<int64_t>(K, RC_CHUNK) * 2;
}

// rho[dst, j] = bf16(R[r, S_j] / s_t) for every valid row r and each of its
// destination rows.  The selected channels cover most 32-byte sectors of a
// row, so rows are streamed whole: each warp owns a sequence of rows, taken
// in pieces of up to 2048 channels, and copies the next piece into shared
// memory (cp.async, 16 bytes a lane) while it works on the current one.  Per
// piece the warp first takes the scale codes of all of the piece's 16-blocks
// (k_quantize's arithmetic, so R matches the quantized tensor bit for bit);
// then lane l handles the output columns 4 l .. 4 l + 3 of every 128, for the
// selected channels that fall in the piece, keeping a window of 1024 columns
// in registers until the row's last piece and storing them as 8-byte words
// (a row with more columns passes over its pieces once per window).
// Per-expert sets: row r uses the set of expert e with
// offsets[e] <= r < offsets[e + 1].  Columns [k, ld) are written as zeros.
__global__ void __launch_bounds__(RC_WARPS * 32) k_rac_residual(
    const __nv_bfloat16 *__restrict__ x, int64_t ldx, int64_t M, int64_t K,
    const int32_t *__restrict__ m_valid, const float *__restrict__ s_t_ptr,
    const int32_t *__restrict__ sel, int k, int ld,
    const int32_t *__restrict__ dst_rows, int fanout, int64_t M_out, __nv_bfloat16 *__restrict__ r_sel,
    const int32_t *__restrict__ expert_offsets, int E)
{
    extern __shared__ __align__(16) uint8_t rsm[];               // [RC_WARPS][2][piece]
    __shared__ float4 tab[128];
    __shared__ uint8_t bcode[RC_WARPS][RC_CHUNK / 16];
    __shared__ int32_t offs[MAX_EXPERTS + 1];
    const float s_t = *s_t_ptr;
    fill_block_table(tab, s_t);
    if (expert_offsets)
        for (int i = threadIdx.x; i <= E; i += blockDim.x) offs[i] = expert_offsets[i];
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t Me = M;
    if (m_valid) Me = min(Me, (int64_t)max(*m_valid, 0));
    const float2 r6 = recip_bracket(__fmul_rn(6.0f, s_t));
    const float2 rs = recip_bracket(s_t);
    const int piece = (int)min(K, (int64_t)RC_CHUNK);
    const int npiece = (int)((K + piece - 1) / piece);
    const int nwin = (ld + RC_WIN - 1) / RC_WIN;
    const int64_t nw = (int64_t)gridDim.x * RC_WARPS;
    uint8_t *wbuf = rsm + (size_t)warp * 2 * piece * 2;
    uint8_t *codes = bcode[warp];

    // a warp's units in order: rows gw, gw + nw, ...; per row its windows,
    // per window its pieces
    auto issue = [&](int64_t r, int p, int s) {
        if (r < Me) {
            const int c0 = p * piece;
            const int nv = (int)min((int64_t)piece, K - c0) / 8;      // 16-byte vectors of the piece
            const uint8_t *src = reinterpret_cast<const uint8_t *>(x + r * ldx + c0);
            const uint32_t dst = ptx::smem_u32(wbuf + s * piece * 2);
            for (int v = lane; v < nv; v += 32) cp_async16(dst + v * 16, src + v * 16);
        }
        cp_async_commit();                           // possibly empty: one group per unit keeps the count
    };

    int64_t r = (int64_t)blockIdx.x * RC_WARPS + warp;
    int win = 0, p = 0;
    int64_t rn = r;
    int winn = 0, pn = 0;
    uint2 acc[RC_GROUPS];
    issue(r, p, 0);
    for (int s = 0; r < Me; s ^= 1) {
        if (++pn == npiece) {
            pn = 0;
            if (++winn == nwin) { winn = 0; rn += nw; }
        }
        issue(rn, pn, s ^ 1);
        cp_async_wait1();                            // this lane's copies of the unit have landed
        __syncwarp();                                // ... and every lane's
        const int c0 = p * piece;
        const int w = (int)min((int64_t)piece, K - c0);
        const __nv_bfloat16 *row = reinterpret_cast<const __nv_bfloat16 *>(wbuf + s * piece * 2);
        for (int bi = lane; bi < w / 16; bi += 32) {
            const uint4 *bp = reinterpret_cast<const uint4 *>(row + bi * 16);
            codes[bi] = (uint8_t)block_code16(bp[0], bp[1], s_t, r6);
        }
        __syncwarp();
        const int32_t *srow = sel;
        if (expert_offsets) {
            int lo = 0, hi = E;
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (offs[mid] <= r) lo = mid; else hi = mid;
            }
            srow += (int64_t)lo * k;
        }
        if (p == 0) {
#pragma unroll
            for (int g = 0; g < RC_GROUPS; ++g) acc[g] = make_uint2(0u, 0u);
        }
#pragma unroll
        for (int g = 0; g < RC_GROUPS; ++g) {
            const int j0 = win * RC_WIN + g * 128 + lane * 4;
            if (win * RC_WIN + g * 128 >= ld) break;     // warp-uniform
            if (j0 < ld && j0 < k) {                     // a group lies wholly inside or outside [0, ld)
                uint32_t o[4] = {acc[g].x & 0xFFFFu, acc[g].x >> 16, acc[g].y & 0xFFFFu, acc[g].y >> 16};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    if (j0 + t < k) {
                        const int ch = srow[j0 + t] - c0;
                        if (ch >= 0 && ch < w) {
                            const float4 bt = tab[codes[ch >> 4]];
                            const BlockConst b{bt.x, bt.y, bt.z, __float_as_uint(bt.w)};
                            o[t] = rho_bf16(element_residual(__bfloat162float(row[ch]), b, s_t), s_t, rs);
                        }
                    }
                }
                acc[g] = make_uint2(o[0] | (o[1] << 16), o[2] | (o[3] << 16));
            }
        }
        if (p == npiece - 1) {                          // the window is complete: store it
            const int32_t *drow = dst_rows ? dst_rows + r * fanout : nullptr;
            const int nd = drow ? fanout : 1;
            for (int d = 0; d < nd; ++d) {
                const int64_t dst = drow ? (int64_t)drow[d] : r;
                if (dst < 0 || dst >= M_out) continue;
                uint2 *out = reinterpret_cast<uint2 *>(r_sel + dst * ld);
#pragma unroll
                for (int g = 0; g < RC_GROUPS; ++g) {
                    const int j0 = win * RC_WIN + g * 128 + lane * 4;
                    if (win * RC_WIN + g * 128 >= ld) break;
                    if (j0 < ld) out[j0 >> 2] = acc[g];
                }
            }
        }
        __syncwarp();                                // the piece is read: its buffer may be refilled
        r = rn;
        win = winn;
        p = pn;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// The same rho for a selection that touches few of a row's blocks: one warp
// per input row, lane j handles selected channel S_j and loads only S_j's
// 32-byte block, re-quantized with the arithmetic of k_quantize (one lane
// takes the whole 16-block max), giving the residual bit for bit.
__global__ void __launch_bounds__(256) k_rac_residual_sparse(
    const __nv_bfloat16 *__restrict__ x, int64_t ldx, int64_t M, int64_t K,
    const int32_t *__restrict__ m_valid, const float *__restrict__ s_t_ptr,
    const int32_t *__restrict__ sel, int k, int ld,
    const int32_t *__restrict__ dst_rows, int fanout, int64_t M_out, __nv_bfloat16 *__restrict__ r_sel,
    const int32_t *__restrict__ expert_offsets, int E)
{
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    int64_t Me = M;
    if (m_valid) Me = min(Me, (int64_t)max(*m_valid, 0));
    if (r >= Me) return;
    if (expert_offsets) {
        // per-expert sets: row r belongs to expert e, offsets[e] <= r < offsets[e+1]
        int lo = 0, hi = E;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (expert_offsets[mid] <= r) lo = mid; else hi = mid;
        }
        sel += (int64_t)lo * k;
    }
    const float s_t = *s_t_ptr;
    const float2 r6 = recip_bracket(__fmul_rn(6.0f, s_t));
    const int nd = dst_rows ? fanout : 1;
    for (int j = lane; j < ld; j += 32) {
        __nv_bfloat16 outv = __float2bfloat16_rn(0.0f);
        if (j < k) {
            const int64_t ch = sel[j];
            const __nv_bfloat16 *blk = x + r * ldx + (ch & ~15ll);
            uint4 u0 = __ldg(reinterpret_cast<const uint4 *>(blk));
            uint4 u1 = __ldg(reinterpret_cast<const uint4 *>(blk + 8));
            uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            float m = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) m = fmaxf(m, fmaxf(fabsf(bf16lo(w[i])), fabsf(bf16hi(w[i]))));
            const BlockConst b = block_const(block_scale_code(m, s_t, r6), s_t);
            int idx = (int)(ch & 15);
            uint32_t word = w[idx >> 1];
            float xv = (idx & 1) ? bf16hi(word) : bf16lo(word);
            float R = __fsub_rn(xv, element_xhat1(xv, b, s_t));
            outv = __float2bfloat16_rn(__fdiv_rn(R, s_t));
        }
        for (int d = 0; d < nd; ++d) {
            int64_t dst = dst_rows ? (int64_t)dst_rows[r * fanout + d] : r;
            if (dst >= 0 && dst < M_out) r_sel[dst * ld + j] = outv;
        }
    }
}

// Launch of the RAC residual: the streaming kernel (one wave of resident
// CTAs, fewer for small M) when the selected channels are at least as many as
// a row's 16-blocks, else the per-channel kernel.
static nvfp4_status launch_rac_residual(const __nv_bfloat16 *x, int64_t ldx, int64_t M, int64_t K,
                                        const int32_t *m_valid, const float *s_t, const int32_t *sel, int k, int ld,
                                        const int32_t *dst_rows, int fanout, int64_t M_out, __nv_bfloat16 *r_sel,
                                        const int32_t *expert_offsets, int E, cudaStream_t st)
{
    if ((int64_t)k * 16 < K) {
        // fewer selected channels than blocks: most of a row's sectors are not needed
        k_rac_residual_sparse<<<(unsigned)((M + 7) / 8), 256, 0, st>>>(x, ldx, M, K, m_valid, s_t, sel, k, ld, dst_rows,
                                                                     fanout, M_out, r_sel, expert_offsets, E);
        return check_launch("k_rac_residual_sparse");
    }
    const size_t smem = rac_residual_smem(K);
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return set_error(NVFP4_ERR_CUDA, "k_rac_residual: no device");
    std::call_once(once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(k_rac_residual, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)rac_residual_smem(RC_CHUNK));
    });
    if (attr_err[dev] != cudaSuccess)
        return set_error(NVFP4_ERR_CUDA, "k_rac_residual: smem attribute: %s", cudaGetErrorString(attr_err[dev]));
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_rac_residual, RC_WARPS * 32, smem) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const unsigned blocks = (unsigned)std::max<int64_t>(
        1, std::min<int64_t>((M + RC_WARPS - 1) / RC_WARPS, (int64_t)num_sms() * per_sm));
    k_rac_residual<<<blocks, RC_WARPS * 32, smem, st>>>(x, ldx, M, K, m_valid, s_t, sel, k, ld, dst_rows, fanout,
                                                        M_out, r_sel, expert_offsets, E);
    return check_launch("k_rac_residual");
}

// ----------------------------------------- RAC second-pass (NVFP4) variant

// Residual R = fl(x - xhat) of input channel ch of one row (the element's
// 16-block is re-quantized with the arithmetic of k_quantize).
__device__ __forceinline__ float residual1(const __nv_bfloat16 *__restrict__ xrow, int64_t ch, float s_t, float2 r6)
{
    const __nv_bfloat16 *blk = xrow + (ch & ~15ll);
    const uint4 u0 = __ldg(reinterpret_cast<const uint4 *>(blk));
    const uint4 u1 = __ldg(reinterpret_cast<const uint4 *>(blk + 8));
    const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fmaxf(fabsf(bf16lo(w[i])), fabsf(bf16hi(w[i]))));
    const BlockConst b = block_const(block_scale_code(m, s_t, r6), s_t);
    const int idx = (int)(ch & 15);
    const uint32_t word = w[idx >> 1];
    const float xv = (idx & 1) ? bf16hi(word) : bf16lo(word);
    return __fsub_rn(xv, element_xhat1(xv, b, s_t));
}

// Pass 1: max |R| over the selected channels of the valid rows (one warp per row).
__global__ void __launch_bounds__(256) k_rac_amax(const __nv_bfloat16 *__restrict__ x, int64_t ldx, int64_t M,
                                                  const int32_t *__restrict__ m_valid, const float *__restrict__ s_t_ptr,
                                                  const int32_t *__restrict__ sel, int k, unsigned int *amax_bits)
{
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    int64_t Me = M;
    if (m_valid) Me = min(Me, (int64_t)max(*m_valid, 0));
    if (r >= Me) return;
    const float s_t = *s_t_ptr;
    const float2 r6 = recip_bracket(__fmul_rn(6.0f, s_t));
    float m = 0.0f;
    for (int j = lane; j < k; j += 32) m = fmaxf(m, fabsf(residual1(x + r * ldx, sel[j], s_t, r6)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0 && m > 0.0f) atomicMax(amax_bits, __float_as_uint(m));
}

// Pass 2: the selected residuals quantized again to NVFP4 as one tensor
// (scale s_r from pass 1, 16-channel blocks along the selection, the last
// block zero-padded): rho2 = bf16(fl(rhat / s_t)), written to every
// destination row.  One warp per row; a half-warp is one block.
__global__ void __launch_bounds__(256) k_rac_residual_nvfp4(
    const __nv_bfloat16 *__restrict__ x, int64_t ldx, int64_t M, const int32_t *__restrict__ m_valid,
    const float *__restrict__ s_t_ptr, const int32_t *__restrict__ sel, int k, int ld,
    const unsigned int *__restrict__ amax_bits, float *s_r_out, const int32_t *__restrict__ dst_rows, int fanout,
    int64_t M_out, __nv_bfloat16 *__restrict__ r_sel)
{
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const float s_r = tensor_scale_from_amax(__uint_as_float(*amax_bits));
    if (r == 0 && lane == 0 && s_r_out) *s_r_out = s_r;
    int64_t Me = M;
    if (m_valid) Me = min(Me, (int64_t)max(*m_valid, 0));
    if (r >= Me) return;
    const float s_t = *s_t_ptr;
    const float2 r6 = recip_bracket(__fmul_rn(6.0f, s_t));
    const float2 r6r = recip_bracket(__fmul_rn(6.0f, s_r));
    const int nd = dst_rows ? fanout : 1;
    for (int j0 = 0; j0 < ld; j0 += 32) {
        const int j = j0 + lane;
        const float R = j < k ? residual1(x + r * ldx, sel[j], s_t, r6) : 0.0f;
        float a = fabsf(R);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        const BlockConst b = block_const(block_scale_code(a, s_r, r6r), s_r);
        const float rhat = element_xhat1(R, b, s_r);
        const __nv_bfloat16 outv = __float2bfloat16_rn(j < k ? __fdiv_rn(rhat, s_t) : 0.0f);
        if (j < ld) {
            for (int d = 0; d < nd; ++d) {
                const int64_t dst = dst_rows ? (int64_t)dst_rows[r * fanout + d] : r;
                if (dst >= 0 && dst < M_out) r_sel[dst * ld + j] = outv;
            }
        }
    }
}

// --------------------------------------------------- weight channel gather

__global__ void k_gather_w_channels(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales,
                                    int64_t E, int64_t N, int64_t K, const int32_t *__restrict__ sel,
                                    int k, int ld, __nv_bfloat16 *__restrict__ out)
{
    const int64_t total = E * N * ld;
    const int64_t sf_per_e = sf_bytes(N, K);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        int64_t j = i % ld;
        int64_t en = i / ld;
        int64_t n = en % N, e = en / N;
        float v = 0.0f;
        const int64_t ch = j < k ? (int64_t)sel[j] : -1;
        if (ch >= 0 && ch < K) {                        // channels outside [0, K) give zeros
            uint32_t byte = codes[en * (K >> 1) + (ch >> 1)];
            uint32_t nib = (ch & 1) ? (byte >> 4) : (byte & 15u);
            float q = e2m1x2_to_f32(nib).x;
            float sf = e4m3_to_f32(scales[e * sf_per_e + sf_offset(n, ch >> 4, K)]);
            v = __fmul_rn(q, sf);   // exact: <= 6 significant bits
        }
        out[i] = __float2bfloat16_rn(v);
    }
}

// ------------------------------------------- channel-major weight copies

// codes_cm[e][c][n/2] (element (n, c), even n in the low nibble) and
// scales_cm[e][c/16][n] from the K-major NVFP4 weight.  One thread per output
// code byte; the scale row is written by the threads whose c % 16 == 0.
__global__ void k_weights_channel_major(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales,
                                        int64_t E, int64_t N, int64_t K, uint8_t *__restrict__ codes_cm,
                                        uint8_t *__restrict__ scales_cm)
{
    const int64_t total = E * K * (N / 2);
    const int64_t sf_per_e = sf_bytes(N, K);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t np = i % (N / 2);           // pair of n
        const int64_t ec = i / (N / 2);
        const int64_t c = ec % K, e = ec / K;
        const int64_t n0 = 2 * np;
        const uint8_t *row0 = codes + (e * N + n0) * (K / 2);
        const uint8_t *row1 = row0 + K / 2;
        uint32_t b0 = row0[c >> 1], b1 = row1[c >> 1];
        uint32_t q0 = (c & 1) ? (b0 >> 4) : (b0 & 15u);
        uint32_t q1 = (c & 1) ? (b1 >> 4) : (b1 & 15u);
        codes_cm[i] = (uint8_t)(q0 | (q1 << 4));
        if ((c & 15) == 0) {
            const uint8_t *se = scales + e * sf_per_e;
            uint8_t *dst = scales_cm + (e * (K / 16) + (c >> 4)) * N + n0;
            dst[0] = se[sf_offset(n0, c >> 4, K)];
            dst[1] = se[sf_offset(n0 + 1, c >> 4, K)];
        }
    }
}

// RAC weight operand from the channel-major copy: one CTA per (expert, 64
// output features).  Each selected channel's 64 codes (32 bytes) and scales
// (64 bytes) are read as contiguous runs, dequantized (e2m1 * sf, exact in
// bf16) into a shared [channel][feature] tile, then written out transposed as
// [feature][ld] rows.
constexpr int GCM_N = 128;                           // output features per CTA
constexpr int GCM_J = 256;                           // output channels per CTA (blockIdx.z chunks of ld)

__global__ void __launch_bounds__(256) k_gather_w_channels_cm(const uint8_t *__restrict__ codes_cm,
                                                              const uint8_t *__restrict__ scales_cm, int64_t N,
                                                              int64_t K, const int32_t *__restrict__ sel, int k,
                                                              int ld, __nv_bfloat16 *__restrict__ out, int sel_stride)
{
    extern __shared__ __align__(16) uint16_t gtile[];  // bf16 [GCM_N features][cw channels of this chunk]
    __shared__ float e4[128];                          // E4M3 code -> value (weight scales are non-negative)
    __shared__ int32_t ssel[GCM_J];
    const int64_t e = blockIdx.y;
    const int64_t n0 = (int64_t)blockIdx.x * GCM_N;
    // this CTA's chunk of output channels [j0, j0 + cw); out and sel are
    // addressed through the chunk-local views below
    const int j0 = blockIdx.z * GCM_J;
    const int cw = min(GCM_J, ld - j0);
    const int kc = max(0, min(k - j0, cw));
    sel += e * sel_stride + j0;                          // sel_stride 0: one set for every expert
    if (threadIdx.x < 128) e4[threadIdx.x] = e4m3_to_f32(threadIdx.x);
    for (int j = threadIdx.x; j < kc; j += blockDim.x) ssel[j] = sel[j];
    __syncthreads();
    // phase 1: item (channel j, 32 features): 16 B of codes, 32 B of scales;
    // consecutive threads take consecutive channels, so the 32 shared-memory
    // stores of an item hit 32 consecutive words across the warp
    const int groups = GCM_N / 32;
    for (int idx = threadIdx.x; idx < cw * groups; idx += blockDim.x) {
        const int jj = idx % cw;
        const int f0 = (idx / cw) * 32;
        uint16_t v[32];
        const int64_t ch = jj < kc ? (int64_t)ssel[jj] : -1;
        if (ch >= 0 && ch < K && n0 + f0 < N) {        // channels outside [0, K) give zeros
            const uint4 w = *reinterpret_cast<const uint4 *>(codes_cm + (e * K + ch) * (N / 2) + (n0 + f0) / 2);
            const uint4 *sp = reinterpret_cast<const uint4 *>(scales_cm + (e * (K / 16) + (ch >> 4)) * N + n0 + f0);
            const uint4 s0 = sp[0], s1 = sp[1];
            const uint32_t cw[4] = {w.x, w.y, w.z, w.w};
            const uint32_t sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float c8[8];
                e2m1x8_to_f32(cw[q], c8);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int f = q * 8 + i;
                    // e2m1 * sf has at most 6 significant bits: exact in bf16
                    v[f] = __bfloat16_as_ushort(__float2bfloat16_rn(
                        __fmul_rn(c8[i], e4[(sw[f >> 2] >> (8 * (f & 3))) & 0x7Fu])));
                }
            }
        } else {
#pragma unroll
            for (int f = 0; f < 32; ++f) v[f] = 0;
        }
#pragma unroll
        for (int f = 0; f < 32; ++f) gtile[(f0 + f) * cw + jj] = v[f];
    }
    __syncthreads();
    // phase 2: 16 B (8 channels) per thread, ld / 8 threads per output row:
    // each row of out[e, n0 + f, :] is written as one contiguous run
    const int cpr = cw / 8;
    for (int idx = threadIdx.x; idx < GCM_N * cpr; idx += blockDim.x) {
        const int f = idx / cpr;
        const int jc = (idx - f * cpr) * 8;
        if (n0 + f >= N) break;                        // rows are monotone in idx
        *reinterpret_cast<uint4 *>(out + (e * N + n0 + f) * ld + j0 + jc) =
            *reinterpret_cast<const uint4 *>(gtile + f * cw + jc);
    }
}

// --------------------------------------------------------------- helpers

static int64_t pick_rows_per_cta(int64_t M, int64_t nchunks, int64_t groups)
{
    // one full wave: QCTAS_PER_SM resident CTAs per SM, at least 8 rows per CTA
    int64_t target = (int64_t)num_sms() * QCTAS_PER_SM;
    int64_t per_group = std::max<int64_t>(1, target / std::max<int64_t>(1, nchunks * groups));
    int64_t rpc = (M + per_group - 1) / per_group;
    rpc = std::max<int64_t>(rpc, 8);
    return rpc;
}

static int64_t row_groups(int64_t M, int64_t rpc) { return std::max<int64_t>(1, (M + rpc - 1) / rpc); }

// Builds the TMA map over x ([rows_total x K] bf16, row stride ldx) and
// launches k_quantize.  `fallback` is any valid 16-byte aligned device
// address, used as the map's base when x has no rows (no copy is issued then).
template <bool SCORE, bool QDQ, bool FAN>
static nvfp4_status launch_quantize_t(const CUtensorMap &tm, const QuantParams &p, dim3 grid, size_t smem,
                                      cudaStream_t st)
{
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return check_launch("k_quantize: device");
    std::call_once(once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(k_quantize<SCORE, QDQ, FAN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)QSMEM);
    });
    if (attr_err[dev] != cudaSuccess) return set_error(NVFP4_ERR_CUDA, "k_quantize: smem attribute: %s",
                                                       cudaGetErrorString(attr_err[dev]));
    k_quantize<SCORE, QDQ, FAN><<<grid, QTHREADS, smem, st>>>(tm, p);
    return check_launch("k_quantize");
}

static nvfp4_status launch_quantize(bool score, const void *x, int64_t rows_total, const void *fallback,
                                    QuantParams &p, dim3 grid, cudaStream_t st)
{
    // every tile row is 256 channels (512 bytes): the box reads zeros past K
    p.box_inner = QCHUNK;
    NVFP4_REQUIRE((int64_t)std::max<int64_t>(p.M_out, p.M) * (p.K / 2) < (1ll << 31) &&
                      (int64_t)p.M * p.K < (1ll << 31),
                  NVFP4_ERR_UNSUPPORTED_SHAPE, "k_quantize: rows x K must stay below 2^31 elements per tensor");
    CUtensorMap tm;
    const bool empty = rows_total <= 0 || x == nullptr;
    if (!make_tmap_2d(&tm, empty ? fallback : x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)p.K,
                      (uint64_t)(empty ? 1 : rows_total), (uint64_t)p.ldx * 2, (uint32_t)p.box_inner, QROWS,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
        return set_error(NVFP4_ERR_CUDA, "k_quantize: tensor map encoding failed");
    const size_t smem = QSMEM;
    const bool fan = p.dst_rows != nullptr;
    if (p.qdq) {
        NVFP4_REQUIRE(!fan, NVFP4_ERR_INVALID_ARG, "k_quantize: the QDQ output has no routed-row form");
        return launch_quantize_t<false, true, false>(tm, p, grid, smem, st);
    }
    if (score) return fan ? launch_quantize_t<true, false, true>(tm, p, grid, smem, st)
                          : launch_quantize_t<true, false, false>(tm, p, grid, smem, st);
    return fan ? launch_quantize_t<false, false, true>(tm, p, grid, smem, st)
               : launch_quantize_t<false, false, false>(tm, p, grid, smem, st);
}

}  // namespace nvfp4

using namespace nvfp4;

// Workspace: [0,256) amax slots (64 groups of 4 B... one slot used), then the
// score partials [P x K] binary64, then score[K] when the caller gave none.
extern "C" size_t nvfp4_quantize_workspace_size(int64_t M, int64_t K)
{
    if (M < 0 || K <= 0) return 0;
    int64_t nch = (K + QCHUNK - 1) / QCHUNK;
    int64_t rpc = pick_rows_per_cta(M, nch, 1);
    int64_t P = row_groups(M, rpc);
    return 256 + (size_t)(P * K + K) * sizeof(double);
}

extern "C" nvfp4_status nvfp4_quantize(const void *x_dev, int64_t M, int64_t K, int64_t ldx,
                                       const int32_t *m_valid_dev,
                                       const float *s_t_in_dev, const float *amax_in_dev, float *s_t_out_dev,
                                       const int32_t *dst_rows_dev, int32_t fanout, int64_t M_out,
                                       uint8_t *codes_dev, uint8_t *scales_dev,
                                       double *score_dev, int32_t rac_k, int32_t rac_ld,
                                       int32_t *sel_dev, void *r_sel_dev,
                                       int32_t *dev_status, void *workspace, size_t workspace_bytes,
                                       void *stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    NVFP4_REQUIRE(M >= 0 && K > 0 && M_out >= 0, NVFP4_ERR_INVALID_ARG, "nvfp4_quantize: bad sizes");
    NVFP4_REQUIRE(s_t_out_dev && (M == 0 || x_dev) && (M_out == 0 || (codes_dev && scales_dev)),
                  NVFP4_ERR_INVALID_ARG, "nvfp4_quantize: x, s_t_out, codes and scales are required");
    NVFP4_REQUIRE(K % 64 == 0 && K <= 16384, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "nvfp4_quantize: K must be a multiple of 64 and <= 16384 (K=%lld)", (long long)K);
    NVFP4_REQUIRE(ldx >= K && ldx % 8 == 0, NVFP4_ERR_ALIGNMENT, "nvfp4_quantize: ldx must be >= K and a multiple of 8");
    NVFP4_REQUIRE(aligned16(x_dev) && aligned16(codes_dev) && aligned16(scales_dev),
                  NVFP4_ERR_ALIGNMENT,
                  "nvfp4_quantize: x, codes and scales must be 16-byte aligned");
    NVFP4_REQUIRE(dst_rows_dev == nullptr || (fanout >= 1 && fanout <= 32), NVFP4_ERR_INVALID_ARG,
                  "nvfp4_quantize: fanout must be in [1, 32] with dst_rows");
    NVFP4_REQUIRE(dst_rows_dev != nullptr || M_out >= M, NVFP4_ERR_INVALID_ARG,
                  "nvfp4_quantize: M_out must be >= M without dst_rows");
    NVFP4_REQUIRE(rac_k >= 0 && rac_k <= K, NVFP4_ERR_UNSUPPORTED_SHAPE, "nvfp4_quantize: rac_k must be in [0, K]");
    if (rac_k > 0) {
        NVFP4_REQUIRE(sel_dev, NVFP4_ERR_INVALID_ARG, "nvfp4_quantize: rac_k > 0 needs sel");
        if (r_sel_dev) {
            NVFP4_REQUIRE(rac_ld >= rac_k && rac_ld % 64 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
                          "nvfp4_quantize: rac_ld must be >= rac_k and a multiple of 64");
            NVFP4_REQUIRE(aligned16(r_sel_dev), NVFP4_ERR_ALIGNMENT, "nvfp4_quantize: r_sel must be 16-byte aligned");
        }
    }
    const bool want_score = score_dev != nullptr || rac_k > 0;
    size_t need = nvfp4_quantize_workspace_size(M, K);
    NVFP4_REQUIRE(workspace && workspace_bytes >= need && aligned16(workspace), NVFP4_ERR_WORKSPACE,
                  "nvfp4_quantize: workspace of %zu bytes (16-byte aligned) required", need);

    // non-negative floats order like their bit patterns: a precomputed max |x|
    // is read through the same unsigned view as the amax pass's result
    const unsigned int *amax_bits = amax_in_dev ? reinterpret_cast<const unsigned int *>(amax_in_dev)
                                                : reinterpret_cast<unsigned int *>(workspace);
    const int64_t nch = (K + QCHUNK - 1) / QCHUNK;
    const int64_t rpc = pick_rows_per_cta(M, nch, 1);
    const int64_t P = row_groups(M, rpc);
    double *partials = reinterpret_cast<double *>(reinterpret_cast<char *>(workspace) + 256);
    double *score = score_dev ? score_dev : partials + P * K;

    if (!s_t_in_dev && !amax_in_dev) {
        unsigned int *slot = reinterpret_cast<unsigned int *>(workspace);
        if (cudaMemsetAsync(slot, 0, 4, st) != cudaSuccess) return check_launch("nvfp4_quantize: memset");
        if (M > 0) {
            int blocks = (int)std::min<int64_t>((int64_t)num_sms() * 8, std::max<int64_t>(1, (M * K / 8 + 255) / 256));
            k_amax<<<dim3(blocks, 1), 256, 0, st>>>((const __nv_bfloat16 *)x_dev, ldx, M, K, m_valid_dev, 0, slot);
            if (check_launch("k_amax") != NVFP4_OK) return NVFP4_ERR_CUDA;
        }
    }
    QuantParams p{};
    p.ldx = ldx; p.M = M; p.K = K;
    p.m_valid = m_valid_dev;
    p.s_t_in = s_t_in_dev;
    p.amax_bits = amax_bits;
    p.s_t_out = s_t_out_dev;
    p.dst_rows = dst_rows_dev;
    p.fanout = dst_rows_dev ? fanout : 1;
    p.M_out = M_out;
    p.codes = codes_dev;
    p.scales = scales_dev;
    p.qdq = nullptr;
    p.partials = partials;
    p.rows_per_cta = rpc;
    p.dev_status = dev_status;
    dim3 grid((unsigned)nch, (unsigned)P, 1);
    if (launch_quantize(want_score, x_dev, M, workspace, p, grid, st) != NVFP4_OK) return NVFP4_ERR_CUDA;

    if (want_score) {
        k_score_reduce<<<(unsigned)((K + 31) / 32), SR_WARPS * 32, 0, st>>>(partials, P, K, score);
        if (check_launch("k_score_reduce") != NVFP4_OK) return NVFP4_ERR_CUDA;
    }
    if (rac_k > 0) {
        size_t smem = (size_t)K * sizeof(unsigned long long);
        static std::once_flag once[64];
        static cudaError_t attr_err[64];
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return check_launch("nvfp4_quantize: device");
        std::call_once(once[dev], [&] {
            attr_err[dev] = cudaFuncSetAttribute(k_select_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, 16384 * 8);
        });
        if (attr_err[dev] != cudaSuccess)
            return set_error(NVFP4_ERR_CUDA, "nvfp4_quantize: smem attribute: %s", cudaGetErrorString(attr_err[dev]));
        k_select_topk<<<1, 1024, smem, st>>>(score, (int)K, rac_k, sel_dev);
        if (check_launch("k_select_topk") != NVFP4_OK) return NVFP4_ERR_CUDA;
        if (M > 0 && r_sel_dev) {                         // no r_sel: the selection only
            const float *s_t_used = s_t_in_dev ? s_t_in_dev : s_t_out_dev;
            if (launch_rac_residual((const __nv_bfloat16 *)x_dev, ldx, M, K, m_valid_dev, s_t_used, sel_dev, rac_k,
                                    rac_ld, dst_rows_dev, dst_rows_dev ? fanout : 1, M_out,
                                    (__nv_bfloat16 *)r_sel_dev, nullptr, 0, st) != NVFP4_OK)
                return NVFP4_ERR_CUDA;
        }
    }
    return NVFP4_OK;
}

extern "C" size_t nvfp4_quantize_experts_workspace_size(int64_t M, int64_t K, int32_t E, int32_t seg_align)
{
    if (M < 0 || K <= 0 || E < 1 || (seg_align != 128 && seg_align != 256)) return 0;
    const int64_t P = std::max<int64_t>(1, (M + seg_align - 1) / seg_align);
    return 256 + (size_t)(P * K + (int64_t)E * K) * sizeof(double);
}

extern "C" nvfp4_status nvfp4_quantize_experts(const void *x_dev, int64_t M, int64_t K, int64_t ldx,
                                               const int32_t *offsets_dev, int32_t E, int32_t seg_align,
                                               const float *s_t_in_dev, const float *amax_in_dev,
                                               float *s_t_out_dev, uint8_t *codes_dev, uint8_t *scales_dev,
                                               double *score_dev, int32_t rac_k, int32_t rac_ld,
                                               int32_t *sel_dev, void *r_sel_dev, int32_t *dev_status,
                                               void *workspace, size_t workspace_bytes, void *stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    NVFP4_REQUIRE(M >= 0 && K > 0, NVFP4_ERR_INVALID_ARG, "nvfp4_quantize_experts: bad sizes");
    NVFP4_REQUIRE(E >= 1 && E <= 256 && offsets_dev, NVFP4_ERR_INVALID_ARG,
                  "nvfp4_quantize_experts: need 1 <= E <= 256 and the expert offsets");
    NVFP4_REQUIRE(seg_align == 128 || seg_align == 256, NVFP4_ERR_INVALID_ARG,
                  "nvfp4_quantize_experts: seg_align must be 128 or 256");
    NVFP4_REQUIRE(M % seg_align == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "nvfp4_quantize_experts: M must be a multiple of seg_align");
    NVFP4_REQUIRE(s_t_out_dev && (M == 0 || (x_dev && codes_dev && scales_dev)), NVFP4_ERR_INVALID_ARG,
                  "nvfp4_quantize_experts: x, s_t_out, codes and scales are required");
    NVFP4_REQUIRE(K % 64 == 0 && K <= 16384, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "nvfp4_quantize_experts: K must be a multiple of 64 and <= 16384");
    NVFP4_REQUIRE(ldx >= K && ldx % 8 == 0, NVFP4_ERR_ALIGNMENT,
                  "nvfp4_quantize_experts: ldx must be >= K and a multiple of 8");
    NVFP4_REQUIRE(aligned16(x_dev) && aligned16(codes_dev) && aligned16(scales_dev), NVFP4_ERR_ALIGNMENT,
                  "nvfp4_quantize_experts: x, codes and scales must be 16-byte aligned");
    NVFP4_REQUIRE(rac_k >= 1 && rac_k <= K && sel_dev && r_sel_dev && rac_ld >= rac_k && rac_ld % 64 == 0,
                  NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "nvfp4_quantize_experts: need 1 <= rac_k <= K, sel, r_sel, rac_ld >= rac_k, rac_ld % 64 == 0");
    NVFP4_REQUIRE(aligned16(r_sel_dev), NVFP4_ERR_ALIGNMENT, "nvfp4_quantize_experts: r_sel must be 16-byte aligned");
    const size_t need = nvfp4_quantize_experts_workspace_size(M, K, E, seg_align);
    NVFP4_REQUIRE(workspace && workspace_bytes >= need && aligned16(workspace), NVFP4_ERR_WORKSPACE,
                  "nvfp4_quantize_experts: workspace of %zu bytes (16-byte aligned) required", need);
    const int32_t *m_valid_dev = offsets_dev + E;               // rows past the last segment are not routed
    const unsigned int *amax_bits = amax_in_dev ? reinterpret_cast<const unsigned int *>(amax_in_dev)
                                                : reinterpret_cast<unsigned int *>(workspace);
    const int64_t nch = (K + QCHUNK - 1) / QCHUNK;
    const int64_t P = std::max<int64_t>(1, M / seg_align);
    double *partials = reinterpret_cast<double *>(reinterpret_cast<char *>(workspace) + 256);
    double *score = score_dev ? score_dev : partials + P * K;
    if (!s_t_in_dev && !amax_in_dev) {
        unsigned int *slot = reinterpret_cast<unsigned int *>(workspace);
        if (cudaMemsetAsync(slot, 0, 4, st) != cudaSuccess) return check_launch("nvfp4_quantize_experts: memset");
        if (M > 0) {
            int blocks = (int)std::min<int64_t>((int64_t)num_sms() * 8, std::max<int64_t>(1, (M * K / 8 + 255) / 256));
            k_amax<<<dim3(blocks, 1), 256, 0, st>>>((const __nv_bfloat16 *)x_dev, ldx, M, K, m_valid_dev, 0, slot);
            if (check_launch("k_amax") != NVFP4_OK) return NVFP4_ERR_CUDA;
        }
    }
    // one row group per seg_align rows: every group lies in one expert's segment
    QuantParams p{};
    p.ldx = ldx; p.M = M; p.K = K;
    p.m_valid = m_valid_dev;
    p.s_t_in = s_t_in_dev;
    p.amax_bits = amax_bits;
    p.s_t_out = s_t_out_dev;
    p.dst_rows = nullptr;
    p.fanout = 1;
    p.M_out = M;
    p.codes = codes_dev;
    p.scales = scales_dev;
    p.qdq = nullptr;
    p.partials = partials;
    p.rows_per_cta = seg_align;
    p.dev_status = dev_status;
    if (launch_quantize(true, x_dev, M, workspace, p, dim3((unsigned)nch, (unsigned)P, 1), st) != NVFP4_OK)
        return NVFP4_ERR_CUDA;
    k_score_reduce_experts<<<dim3((unsigned)((K + 255) / 256), (unsigned)E), 256, 0, st>>>(partials, offsets_dev,
                                                                                          seg_align, K, score);
    if (check_launch("k_score_reduce_experts") != NVFP4_OK) return NVFP4_ERR_CUDA;
    {
        static std::once_flag once[64];
        static cudaError_t attr_err[64];
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
            return check_launch("nvfp4_quantize_experts: device");
        std::call_once(once[dev], [&] {
            attr_err[dev] = cudaFuncSetAttribute(k_select_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, 16384 * 8);
        });
        if (attr_err[dev] != cudaSuccess)
            return set_error(NVFP4_ERR_CUDA, "nvfp4_quantize_experts: smem attribute: %s",
                             cudaGetErrorString(attr_err[dev]));
    }
    k_select_topk<<<(unsigned)E, 1024, (size_t)K * sizeof(unsigned long long), st>>>(score, (int)K, rac_k, sel_dev);
    if (check_launch("k_select_topk") != NVFP4_OK) return NVFP4_ERR_CUDA;
    if (M > 0) {
        const float *s_t_used = s_t_in_dev ? s_t_in_dev : s_t_out_dev;
        if (launch_rac_residual((const __nv_bfloat16 *)x_dev, ldx, M, K, m_valid_dev, s_t_used, sel_dev, rac_k, rac_ld,
                                nullptr, 1, M, (__nv_bfloat16 *)r_sel_dev, offsets_dev, E, st) != NVFP4_OK)
            return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

extern "C" size_t nvfp4_rac_residual_nvfp4_workspace_size(void) { return 256; }

extern "C" nvfp4_status nvfp4_rac_residual_nvfp4(const void *x_dev, int64_t M, int64_t K, int64_t ldx,
                                                 const int32_t *m_valid_dev, const float *s_t_dev,
                                                 const int32_t *sel_dev, int32_t rac_k, int32_t rac_ld,
                                                 const int32_t *dst_rows_dev, int32_t fanout, int64_t M_out,
                                                 void *r_sel_dev, float *s_r_out_dev, void *workspace,
                                                 size_t workspace_bytes, void *stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    NVFP4_REQUIRE(M >= 0 && K > 0 && M_out >= 0, NVFP4_ERR_INVALID_ARG, "nvfp4_rac_residual_nvfp4: bad sizes");
    NVFP4_REQUIRE(s_t_dev && (M == 0 || x_dev) && (rac_k == 0 || sel_dev) && r_sel_dev, NVFP4_ERR_INVALID_ARG,
                  "nvfp4_rac_residual_nvfp4: x, s_t, sel and r_sel are required");
    NVFP4_REQUIRE(K % 64 == 0 && K <= 16384, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "nvfp4_rac_residual_nvfp4: K must be a multiple of 64 and <= 16384");
    NVFP4_REQUIRE(ldx >= K && ldx % 8 == 0 && aligned16(x_dev), NVFP4_ERR_ALIGNMENT,
                  "nvfp4_rac_residual_nvfp4: x must be 16-byte aligned with ldx >= K, ldx % 8 == 0");
    NVFP4_REQUIRE(rac_k >= 0 && rac_k <= K && rac_ld >= rac_k && rac_ld % 64 == 0 && rac_ld > 0,
                  NVFP4_ERR_UNSUPPORTED_SHAPE, "nvfp4_rac_residual_nvfp4: need 0 <= rac_k <= rac_ld, rac_ld % 64 == 0");
    NVFP4_REQUIRE(dst_rows_dev == nullptr || (fanout >= 1 && fanout <= 32), NVFP4_ERR_INVALID_ARG,
                  "nvfp4_rac_residual_nvfp4: fanout must be in [1, 32] with dst_rows");
    NVFP4_REQUIRE(workspace && workspace_bytes >= 256 && aligned16(workspace), NVFP4_ERR_WORKSPACE,
                  "nvfp4_rac_residual_nvfp4: workspace of 256 bytes required");
    unsigned int *slot = reinterpret_cast<unsigned int *>(workspace);
    if (cudaMemsetAsync(slot, 0, 4, st) != cudaSuccess) return check_launch("nvfp4_rac_residual_nvfp4: memset");
    const unsigned blocks = (unsigned)std::max<int64_t>(1, (M + 7) / 8);
    if (M > 0 && rac_k > 0) {
        k_rac_amax<<<blocks, 256, 0, st>>>((const __nv_bfloat16 *)x_dev, ldx, M, m_valid_dev, s_t_dev, sel_dev, rac_k,
                                           slot);
        if (check_launch("k_rac_amax") != NVFP4_OK) return NVFP4_ERR_CUDA;
    }
    k_rac_residual_nvfp4<<<blocks, 256, 0, st>>>((const __nv_bfloat16 *)x_dev, ldx, M, m_valid_dev, s_t_dev, sel_dev,
                                                 rac_k, rac_ld, slot, s_r_out_dev, dst_rows_dev,
                                                 dst_rows_dev ? fanout : 1, M_out, (__nv_bfloat16 *)r_sel_dev);
    return check_launch("k_rac_residual_nvfp4");
}

extern "C" size_t nvfp4_qdq_workspace_size(int64_t G, int64_t rows, int64_t cols)
{
    (void)rows; (void)cols;
    if (G <= 0) return 0;
    return (size_t)(((G * 4) + 255) / 256 * 256);
}

extern "C" nvfp4_status nvfp4_qdq_weights(const void *w_dev, int64_t G, int64_t rows, int64_t cols,
                                          void *w_qdq_dev, float *s_t_dev,
                                          uint8_t *codes_dev, uint8_t *scales_dev,
                                          void *workspace, size_t workspace_bytes, void *stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    NVFP4_REQUIRE(w_dev && s_t_dev, NVFP4_ERR_INVALID_ARG, "nvfp4_qdq_weights: w and s_t are required");
    NVFP4_REQUIRE(G >= 1 && G <= 65535 && rows >= 1 && cols >= 1, NVFP4_ERR_INVALID_ARG,
                  "nvfp4_qdq_weights: bad sizes");
    NVFP4_REQUIRE(cols % 64 == 0 && cols <= 16384, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "nvfp4_qdq_weights: cols must be a multiple of 64 and <= 16384");
    NVFP4_REQUIRE((codes_dev == nullptr) == (scales_dev == nullptr), NVFP4_ERR_INVALID_ARG,
                  "nvfp4_qdq_weights: codes and scales go together");
    NVFP4_REQUIRE(aligned16(w_dev) && (!w_qdq_dev || aligned16(w_qdq_dev)) &&
                  (!codes_dev || (aligned16(codes_dev) && aligned16(scales_dev))), NVFP4_ERR_ALIGNMENT,
                  "nvfp4_qdq_weights: pointers must be 16-byte aligned");
    size_t need = nvfp4_qdq_workspace_size(G, rows, cols);
    NVFP4_REQUIRE(workspace && workspace_bytes >= need && aligned16(workspace), NVFP4_ERR_WORKSPACE,
                  "nvfp4_qdq_weights: workspace of %zu bytes required", need);
    unsigned int *amax_bits = reinterpret_cast<unsigned int *>(workspace);
    if (cudaMemsetAsync(amax_bits, 0, (size_t)G * 4, st) != cudaSuccess) return check_launch("qdq memset");
    const int64_t per_group = rows * cols;
    {
        int64_t want = std::max<int64_t>(1, (int64_t)num_sms() * 8 / G);
        int blocks = (int)std::min<int64_t>(want, std::max<int64_t>(1, (per_group / 8 + 255) / 256));
        k_amax<<<dim3(blocks, (unsigned)G), 256, 0, st>>>((const __nv_bfloat16 *)w_dev, cols, rows, cols,
                                                          nullptr, per_group, amax_bits);
        if (check_launch("k_amax (qdq)") != NVFP4_OK) return NVFP4_ERR_CUDA;
    }
    const int64_t nch = (cols + QCHUNK - 1) / QCHUNK;
    const int64_t rpc = pick_rows_per_cta(rows, nch, G);
    QuantParams p{};
    p.ldx = cols; p.M = rows; p.K = cols;
    p.amax_bits = amax_bits;
    p.s_t_out = s_t_dev;
    p.fanout = 1;
    p.M_out = rows;
    p.codes = codes_dev;
    p.scales = scales_dev;
    p.qdq = (__nv_bfloat16 *)w_qdq_dev;
    p.rows_per_cta = rpc;
    p.codes_gstride = per_group / 2;
    p.scales_gstride = sf_bytes(rows, cols);
    p.qdq_gstride = per_group;
    dim3 grid((unsigned)nch, (unsigned)row_groups(rows, rpc), (unsigned)G);
    return launch_quantize(false, w_dev, G * rows, workspace, p, grid, st);
}

extern "C" nvfp4_status nvfp4_gather_weight_channels(const uint8_t *codes_dev, const uint8_t *scales_dev,
                                                     int32_t E, int64_t N, int64_t K,
                                                     const int32_t *sel_dev, int32_t k, int32_t ld,
                                                     void *w_sel_dev, void *stream)
{
    cudaStream_t st = (cudaStream_t)stream;
    NVFP4_REQUIRE(codes_dev && scales_dev && w_sel_dev && (k == 0 || sel_dev), NVFP4_ERR_INVALID_ARG,
                  "nvfp4_gather_weight_channels: null pointer");
    NVFP4_REQUIRE(E >= 1 && N >= 1 && K >= 64 && K % 64 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "nvfp4_gather_weight_channels: bad shape");
    NVFP4_REQUIRE(k >= 0 && k <= ld && ld % 64 == 0 && ld <= 16384 && k <= K, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "nvfp4_gather_weight_channels: need 0 <= k <= ld <= 16384, ld % 64 == 0");
    int64_t total = (int64_t)E * N * ld;
    int blocks = (int)std::min<int64_t>((int64_t)num_sms() * 16, (total + 255) / 256);
    k_gather_w_channels<<<blocks, 256, 0, st>>>(codes_dev, scales_dev, E, N, K, sel_dev, k, ld,
                                                (__nv_bfloat16 *)w_sel_dev);
    return check_launch("k_gather_w_channels");
}

extern "C" nvfp4_status nvfp4_weights_channel_major(const uint8_t *codes_dev, const uint8_t *scales_dev, int32_t E,
                                                    int64_t N, int64_t K, uint8_t *codes_cm_dev,
                                                    uint8_t *scales_cm_dev, void *stream)
{
    NVFP4_REQUIRE(codes_dev && scales_dev && codes_cm_dev && scales_cm_dev, NVFP4_ERR_INVALID_ARG,
                  "nvfp4_weights_channel_major: null pointer");
    NVFP4_REQUIRE(E >= 1 && N >= 2 && N % 64 == 0 && K >= 64 && K % 64 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "nvfp4_weights_channel_major: need N % 64 == 0, K % 64 == 0");
    int64_t total = (int64_t)E * K * (N / 2);
    int blocks = (int)std::min<int64_t>((int64_t)num_sms() * 16, (total + 255) / 256);
    k_weights_channel_major<<<blocks, 256, 0, (cudaStream_t)stream>>>(codes_dev, scales_dev, E, N, K, codes_cm_dev,
                                                                     scales_cm_dev);
    return check_launch("k_weights_channel_major");
}

static nvfp4_status gather_cm(const uint8_t *codes_cm_dev, const uint8_t *scales_cm_dev, int32_t E, int64_t N,
                              int64_t K, const int32_t *sel_dev, int32_t k, int32_t ld, void *w_sel_dev,
                              int sel_stride, void *stream)
{
    NVFP4_REQUIRE(codes_cm_dev && scales_cm_dev && w_sel_dev && (k == 0 || sel_dev), NVFP4_ERR_INVALID_ARG,
                  "nvfp4_gather_weight_channels_cm: null pointer");
    NVFP4_REQUIRE(E >= 1 && E <= 65535 && N >= 64 && N % 64 == 0 && K >= 64 && K % 64 == 0,
                  NVFP4_ERR_UNSUPPORTED_SHAPE, "nvfp4_gather_weight_channels_cm: need N % 64 == 0, K % 64 == 0");
    NVFP4_REQUIRE(k >= 0 && k <= ld && ld % 64 == 0 && ld <= 16384 && k <= K, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "nvfp4_gather_weight_channels_cm: need 0 <= k <= ld <= 16384, ld % 64 == 0");
    NVFP4_REQUIRE(aligned16(w_sel_dev) && aligned16(codes_cm_dev) && aligned16(scales_cm_dev), NVFP4_ERR_ALIGNMENT,
                  "nvfp4_gather_weight_channels_cm: pointers must be 16-byte aligned");
    size_t smem = (size_t)std::min(ld, GCM_J) * GCM_N * sizeof(uint16_t);
    {
        static std::once_flag once[64];
        static cudaError_t attr_err[64];
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
            return check_launch("nvfp4_gather_weight_channels_cm: device");
        std::call_once(once[dev], [&] {
            attr_err[dev] = cudaFuncSetAttribute(k_gather_w_channels_cm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)(GCM_J * GCM_N * sizeof(uint16_t)));
        });
        if (attr_err[dev] != cudaSuccess)
            return set_error(NVFP4_ERR_CUDA, "nvfp4_gather_weight_channels_cm: smem attribute: %s",
                             cudaGetErrorString(attr_err[dev]));
    }
    dim3 grid((unsigned)((N + GCM_N - 1) / GCM_N), (unsigned)E, (unsigned)((ld + GCM_J - 1) / GCM_J));
    k_gather_w_channels_cm<<<grid, 256, smem, (cudaStream_t)stream>>>(codes_cm_dev, scales_cm_dev, N, K, sel_dev, k,
                                                                    ld, (__nv_bfloat16 *)w_sel_dev, sel_stride);
    return check_launch("k_gather_w_channels_cm");
}

extern "C" nvfp4_status nvfp4_gather_weight_channels_cm(const uint8_t *codes_cm_dev, const uint8_t *scales_cm_dev,
                                                        int32_t E, int64_t N, int64_t K, const int32_t *sel_dev,
                                                        int32_t k, int32_t ld, void *w_sel_dev, void *stream)
{
    return gather_cm(codes_cm_dev, scales_cm_dev, E, N, K, sel_dev, k, ld, w_sel_dev, 0, stream);
}

extern "C" nvfp4_status nvfp4_gather_weight_channels_cm_experts(const uint8_t *codes_cm_dev,
                                                                const uint8_t *scales_cm_dev, int32_t E, int64_t N,
                                                                int64_t K, const int32_t *sel_dev, int32_t k,
                                                                int32_t ld, void *w_sel_dev, void *stream)
{
    return gather_cm(codes_cm_dev, scales_cm_dev, E, N, K, sel_dev, k, ld, w_sel_dev, k, stream);
}

// ------------------------------------------------ FP8 E4M3 (comparison)
//
// Per-tensor E4M3 quantization, the format of the FP8 rollout the QUADS pages
// compare against: s = A / 448 (1 for an all-zero tensor), q = E4M3(fl(x/s))
// with the sign of x, nearest even, saturating.  Each decision is taken from
// the bracketing multiplications (see the NVFP4 block steps in common.cuh),
// the IEEE division being evaluated when they disagree.  16 elements per
// thread; G groups (one scale each) or, for G = 1, routed copies.

namespace nvfp4 {

__global__ void __launch_bounds__(256) k_fp8_quantize(const __nv_bfloat16 *__restrict__ x, int64_t ldx, int64_t M,
                                                      int64_t K, int64_t group_stride, const float *__restrict__ s_in,
                                                      const unsigned int *__restrict__ amax_bits, float *s_out,
                                                      const int32_t *__restrict__ dst_rows, int fanout, int64_t M_out,
                                                      uint8_t *__restrict__ codes, int64_t codes_gstride)
{
    const int g = blockIdx.y;
    float s;
    if (s_in) {
        s = s_in[g];
    } else {
        const float A = __uint_as_float(amax_bits[g]);
        s = A == 0.0f ? 1.0f : __fdiv_rn(A, 448.0f);
    }
    if (blockIdx.x == 0 && threadIdx.x == 0 && s_out) s_out[g] = s;
    const float2 rb = recip_bracket(s);
    const __nv_bfloat16 *xg = x + (int64_t)g * group_stride;
    uint8_t *cg = codes + (int64_t)g * codes_gstride;
    const int64_t cpr = K / 16;
    const int64_t total = M * cpr;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / cpr, c = (i - r * cpr) * 16;
        const uint4 *src = reinterpret_cast<const uint4 *>(xg + r * ldx + c);
        const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
        const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        uint32_t lo[4], hi[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 a = bf16x2_to_f2(w[2 * k]), b = bf16x2_to_f2(w[2 * k + 1]);
            const float2 al = mul2(a, make_float2(rb.x, rb.x)), ah = mul2(a, make_float2(rb.y, rb.y));
            const float2 bl = mul2(b, make_float2(rb.x, rb.x)), bh = mul2(b, make_float2(rb.y, rb.y));
            lo[k] = (cvt_e4m3x2(al.x, al.y) & 0xFFFFu) | (cvt_e4m3x2(bl.x, bl.y) << 16);
            hi[k] = (cvt_e4m3x2(ah.x, ah.y) & 0xFFFFu) | (cvt_e4m3x2(bh.x, bh.y) << 16);
        }
        if (lo[0] != hi[0] || lo[1] != hi[1] || lo[2] != hi[2] || lo[3] != hi[3]) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 a = bf16x2_to_f2(w[2 * k]), b = bf16x2_to_f2(w[2 * k + 1]);
                lo[k] = (cvt_e4m3x2(__fdiv_rn(a.x, s), __fdiv_rn(a.y, s)) & 0xFFFFu) |
                        (cvt_e4m3x2(__fdiv_rn(b.x, s), __fdiv_rn(b.y, s)) << 16);
            }
        }
        const uint4 out = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        if (!dst_rows) {
            *reinterpret_cast<uint4 *>(cg + r * K + c) = out;
        } else {
            for (int j = 0; j < fanout; ++j) {
                const int64_t d = dst_rows[r * fanout + j];
                if (d >= 0 && d < M_out) *reinterpret_cast<uint4 *>(cg + d * K + c) = out;
            }
        }
    }
}

}  // namespace nvfp4

extern "C" size_t fp8_quantize_workspace_size(int64_t G)
{
    if (G <= 0) return 0;
    return (size_t)(((G * 4) + 255) / 256 * 256);
}

extern "C" nvfp4_status fp8_quantize(const void *x_dev, int64_t G, int64_t M, int64_t K, int64_t ldx,
                                     const float *s_in_dev, const float *amax_in_dev, float *s_out_dev,
                                     const int32_t *dst_rows_dev,
                                     int32_t fanout, int64_t M_out, uint8_t *codes_dev, void *workspace,
                                     size_t workspace_bytes, void *stream)
{
    using namespace nvfp4;
    cudaStream_t st = (cudaStream_t)stream;
    NVFP4_REQUIRE(G >= 1 && G <= 65535 && M >= 0 && K > 0 && M_out >= 0, NVFP4_ERR_INVALID_ARG, "fp8_quantize: bad sizes");
    NVFP4_REQUIRE(s_out_dev && (M == 0 || x_dev) && (M_out == 0 || codes_dev), NVFP4_ERR_INVALID_ARG,
                  "fp8_quantize: x, s_out and codes are required");
    NVFP4_REQUIRE(K % 16 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE, "fp8_quantize: K must be a multiple of 16");
    NVFP4_REQUIRE(ldx >= K && ldx % 8 == 0, NVFP4_ERR_ALIGNMENT, "fp8_quantize: ldx must be >= K and a multiple of 8");
    NVFP4_REQUIRE(aligned16(x_dev) && aligned16(codes_dev), NVFP4_ERR_ALIGNMENT,
                  "fp8_quantize: x and codes must be 16-byte aligned");
    NVFP4_REQUIRE(dst_rows_dev == nullptr || (G == 1 && fanout >= 1 && fanout <= 32), NVFP4_ERR_INVALID_ARG,
                  "fp8_quantize: dst_rows needs G == 1 and 1 <= fanout <= 32");
    NVFP4_REQUIRE(dst_rows_dev != nullptr || M_out >= M, NVFP4_ERR_INVALID_ARG,
                  "fp8_quantize: M_out must be >= M without dst_rows");
    NVFP4_REQUIRE(amax_in_dev == nullptr || G == 1, NVFP4_ERR_INVALID_ARG, "fp8_quantize: amax_in needs G == 1");
    const size_t need = fp8_quantize_workspace_size(G);
    const bool need_amax = !s_in_dev && !amax_in_dev;
    NVFP4_REQUIRE(!need_amax || (workspace && workspace_bytes >= need && aligned16(workspace)), NVFP4_ERR_WORKSPACE,
                  "fp8_quantize: workspace of %zu bytes (16-byte aligned) required", need);
    // non-negative floats order like their bit patterns
    const unsigned int *amax_bits = amax_in_dev ? reinterpret_cast<const unsigned int *>(amax_in_dev)
                                                : reinterpret_cast<unsigned int *>(workspace);
    if (need_amax) {
        unsigned int *slots = reinterpret_cast<unsigned int *>(workspace);
        if (cudaMemsetAsync(slots, 0, (size_t)G * 4, st) != cudaSuccess) return check_launch("fp8_quantize: memset");
        if (M > 0) {
            const int64_t want = std::max<int64_t>(1, (int64_t)num_sms() * 8 / G);
            const int blocks = (int)std::min<int64_t>(want, std::max<int64_t>(1, (M * K / 8 + 255) / 256));
            k_amax<<<dim3(blocks, (unsigned)G), 256, 0, st>>>((const __nv_bfloat16 *)x_dev, ldx, M, K, nullptr,
                                                              M * ldx, slots);
            if (check_launch("k_amax (fp8)") != NVFP4_OK) return NVFP4_ERR_CUDA;
        }
    }
    const int64_t chunks = M * (K / 16);
    const int64_t want = std::max<int64_t>(1, (int64_t)num_sms() * 8 / G);
    const int blocks = (int)std::min<int64_t>(want, std::max<int64_t>(1, (chunks + 255) / 256));
    k_fp8_quantize<<<dim3(blocks, (unsigned)G), 256, 0, st>>>((const __nv_bfloat16 *)x_dev, ldx, M, K, M * ldx,
                                                              s_in_dev, amax_bits, s_out_dev, dst_rows_dev,
                                                              dst_rows_dev ? fanout : 1, M_out, codes_dev, M_out * K);
    return check_launch("k_fp8_quantize");
}

// ------------------------------------------------------- conversion probe

namespace nvfp4 {
__global__ void k_debug_encode(const float *__restrict__ in, int64_t n, uint8_t *__restrict__ e2m1,
                               uint8_t *__restrict__ e4m3)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        float v = in[i];
        if (e2m1) e2m1[i] = (uint8_t)cvt_e2m1x2(v, 0.0f);
        if (e4m3) e4m3[i] = (uint8_t)cvt_e4m3(v);
    }
}
}  // namespace nvfp4

extern "C" nvfp4_status nvfp4_debug_encode(const float *in_dev, int64_t n, uint8_t *e2m1_dev, uint8_t *e4m3_dev,
                                           void *stream)
{
    NVFP4_REQUIRE(in_dev && n >= 0, NVFP4_ERR_INVALID_ARG, "nvfp4_debug_encode: bad arguments");
    if (n == 0) return NVFP4_OK;
    int blocks = (int)std::min<int64_t>((int64_t)num_sms() * 8, (n + 255) / 256);
    k_debug_encode<<<blocks, 256, 0, (cudaStream_t)stream>>>(in_dev, n, e2m1_dev, e4m3_dev);
    return check_launch("k_debug_encode");
}

// ------------------------------------------------- allocation-free variant
//
// nvfp4_quantize_noalloc serves callers that cannot allocate device memory
// when they call in (see the header).  Its scratch space -- the amax slot and
// the per-CTA score partials that nvfp4_quantize keeps in the caller's
// workspace -- lives in this file-scope device array instead, which every
// GPU that loads the library holds until the process exits.  In host code
// the array's name is only a host-side stand-in, so its device address is
// looked up once per device with cudaGetSymbolAddress (on the first call made
// with that device current) and passed to the kernels.

namespace nvfp4 {

constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(4) << 20;     // 4 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

static void *noalloc_scratch_ptr(nvfp4_status *st)
{
    static void *ptrs[64];
    static std::mutex mu;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        *st = set_error(NVFP4_ERR_CUDA, "nvfp4_quantize_noalloc: no usable current device");
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            *st = set_error(NVFP4_ERR_CUDA, "nvfp4_quantize_noalloc: cudaGetSymbolAddress failed: %s",
                            cudaGetErrorString(e));
            return nullptr;
        }
        ptrs[dev] = p;
    }
    *st = NVFP4_OK;
    return ptrs[dev];
}

}  // namespace nvfp4

extern "C" size_t nvfp4_quantize_noalloc_max_scratch(void) { return nvfp4::NOALLOC_SCRATCH_BYTES; }

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void *x_dev, int64_t M, int64_t K, int64_t ldx,
                                               const int32_t *m_valid_dev,
                                               const float *s_t_in_dev, const float *amax_in_dev,
                                               float *s_t_out_dev,
                                               const int32_t *dst_rows_dev, int32_t fanout, int64_t M_out,
                                               uint8_t *codes_dev, uint8_t *scales_dev,
                                               double *score_dev, int32_t rac_k, int32_t rac_ld,
                                               int32_t *sel_dev, void *r_sel_dev,
                                               int32_t *dev_status, void *stream)
{
    size_t need = nvfp4_quantize_workspace_size(M, K);
    NVFP4_REQUIRE(need > 0, NVFP4_ERR_INVALID_ARG, "nvfp4_quantize_noalloc: bad sizes");
    NVFP4_REQUIRE(need <= nvfp4::NOALLOC_SCRATCH_BYTES, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "nvfp4_quantize_noalloc: M=%lld, K=%lld needs %zu bytes of scratch, above the fixed %zu-byte "
                  "device array; call nvfp4_quantize with a workspace instead",
                  (long long)M, (long long)K, need, nvfp4::NOALLOC_SCRATCH_BYTES);
    nvfp4_status st;
    void *scratch = nvfp4::noalloc_scratch_ptr(&st);
    if (!scratch) return st;
    return nvfp4_quantize(x_dev, M, K, ldx, m_valid_dev, s_t_in_dev, amax_in_dev, s_t_out_dev, dst_rows_dev, fanout,
                          M_out,
                          codes_dev, scales_dev, score_dev, rac_k, rac_ld, sel_dev, r_sel_dev, dev_status, scratch,
                          nvfp4::NOALLOC_SCRATCH_BYTES, stream);
}
