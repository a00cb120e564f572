// gemm.cu -- persistent grouped W4A4 (NVFP4) expert GEMM with Residual
// Activation Compensation on the sm_100a tensor cores.
//
// One CTA per SM, 10 warps:
//   warp 0      TMA producer (one lane): per 256-element K step it loads the
//               A tile (128 rows x 128 B of packed E2M1), the B tile (two
//               128-row boxes), and the matching 512-byte scale atoms (bulk
//               copies) into a 4-stage shared-memory ring; then the RAC
//               stages (bf16 rho and w_sel tiles, 64 channels each).
//   warp 1      MMA issuer (one lane): copies the stage's scale atoms to TMEM
//               (tcgen05.cp 32x128b.warpx4) and issues 4 block-scaled
//               tcgen05.mma kind::mxf4nvf4 (M128 N256 K64) per stage into one
//               TMEM accumulator; after the FP4 K loop it drains (commit +
//               wait) and accumulates the RAC stages with kind::f16 BF16 MMAs
//               (M128 N256 K16) into the same accumulator.
//   warps 2..9  epilogue: each warp copies its TMEM slice (32-lane quadrant
//               w % 4, one half of the columns) into registers and releases
//               the accumulator at once, so the next tile's MMAs overlap the
//               math and stores: y = s_a s_b D, then store f32 / SwiGLU ->
//               bf16 / router-weighted atomic scatter-add into the token-major
//               output.
// Tiles: 128 routed rows x 256 output features (SwiGLU: 128 gate + the 128
// matching up features).  Every expert's routed-row segment is a multiple of
// 128, so a tile never spans two experts; the tile count comes from the
// device-side offsets (no host synchronization).
//
// Shared memory: a 4-stage ring of 54 KB stages for the SwiGLU (bf16) epilogue;
// the f32 epilogues use 3 stages and a 34 KB staging area from which each lane
// writes 64 contiguous floats of its row with one 256-byte bulk store or bulk
// add-reduction (cp.reduce.async.bulk .add.f32) -- full-line traffic instead
// of per-thread 16-byte stores or atomics.
// TMEM: 512 columns = accumulator [0,256) + scale factors of A [256,272)
// (4 atoms x 4 columns) + scale factors of B [272,304) (4 x 8 columns).
// Every mbarrier wait is bounded (1 s); on expiry the kernel records
// NVFP4_ERR_TIMEOUT, all roles stop, in-flight copies and MMAs are drained
// (bounded) and TMEM is freed before exit.
#include "common.cuh"
#include "ptx.cuh"

#include <cuda.h>
#include <algorithm>
#include <mutex>

namespace nvfp4 {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int MAX_STAGES = 4;
constexpr uint32_t A_BYTES = BM * 128;          // 16 KB
constexpr uint32_t B_BYTES = BN * 128;          // 32 KB
constexpr uint32_t SFA_BYTES = 4 * 512;         // 4 atoms (K=256 / 64)
constexpr uint32_t SFB_BYTES = 8 * 512;         // 2 row blocks x 4 atoms
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr uint32_t RAC_STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 320;           // producer, MMA, 8 epilogue warps
constexpr int EPI_WARPS = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0, SFA_COL = 256, SFB_COL = 272;
constexpr int MAX_E = 256;
constexpr uint64_t TIMEOUT_NS = 1000000000ull;
// f32 epilogues stage rows in shared memory and write them with 256-byte bulk
// copies / bulk add-reductions: per epilogue warp 16 row slots of 64 floats,
// padded to 68 floats so the 16 writing lanes spread over the banks.
constexpr uint32_t SLOT_FLOATS = 68;
constexpr uint32_t STAGING_BYTES = EPI_WARPS * 16 * SLOT_FLOATS * 4;

template <int STAGES>
struct Cfg {
    static constexpr bool STAGING = STAGES < MAX_STAGES;      // f32 epilogues give up one stage for staging
    static constexpr uint32_t SMEM = STAGES * STAGE_BYTES + (STAGING ? STAGING_BYTES : 0) + 1024 /*align*/ +
                                     2048 /*barriers, offsets*/;
};

struct Params {
    const uint8_t *a_scales;
    const float *a_s_t;
    const uint8_t *b_scales;
    const float *b_s_t;
    int64_t N, K;
    int E;
    const int32_t *offsets;
    int rac_ld;
    int epilogue;
    int inter;                 // SwiGLU: I (= N/2)
    const int32_t *row_token;
    const float *row_gate;
    void *out;
    int64_t ld_out;
    unsigned int *amax_out;    // SwiGLU: max |h| (float bits), or null
    int32_t *dev_status;
};

struct Shared {
    uint64_t full[MAX_STAGES];
    uint64_t empty[MAX_STAGES];
    uint64_t tmem_full;
    uint64_t tmem_empty;
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int offsets[MAX_E + 1];
};

// Bounded wait; returns false on abort or timeout (then sets the abort flag).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                         int32_t *dev_status, bool ignore_abort = false)
{
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 63u) {
            if (!ignore_abort && *abort_flag) return false;
            uint64_t now = globaltimer_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > TIMEOUT_NS) {
                *abort_flag = 1;
                report_status(dev_status, NVFP4_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

__device__ __forceinline__ int find_expert(const int *off, int E, int m0)
{
    int lo = 0, hi = E;                   // off[lo] <= m0 < off[hi]
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (off[mid] <= m0) lo = mid; else hi = mid;
    }
    return lo;
}

__device__ __forceinline__ float silu(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

template <int STAGES>
__global__ void __launch_bounds__(NUM_THREADS, 1)
k_moe_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
           const __grid_constant__ CUtensorMap tm_ra, const __grid_constant__ CUtensorMap tm_rb, Params p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *stage_base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *staging = reinterpret_cast<float *>(stage_base + STAGES * STAGE_BYTES);
    Shared *sh = reinterpret_cast<Shared *>(stage_base + STAGES * STAGE_BYTES +
                                            (Cfg<STAGES>::STAGING ? STAGING_BYTES : 0));
    volatile int *abort_flag = &sh->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(ptx::smem_u32(&sh->full[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&sh->empty[s]), 1);
        }
        ptx::mbar_init(ptx::smem_u32(&sh->tmem_full), 1);
        ptx::mbar_init(ptx::smem_u32(&sh->tmem_empty), EPI_WARPS);
        ptx::mbar_init(ptx::smem_u32(&sh->drain), 1);
        sh->abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::fence_proxy_async_smem();
    }
    for (int i = threadIdx.x; i <= E; i += NUM_THREADS) sh->offsets[i] = p.offsets[i];
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(&sh->tmem_base), TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sh->tmem_base;

    const int swiglu = p.epilogue == MOE_EPI_SWIGLU_BF16;
    const int n_tiles = swiglu ? p.inter / 128 : (int)(p.N / BN);
    const int m_tiles = sh->offsets[E] / BM;
    const int total = m_tiles * n_tiles;
    const int nkb = (int)(p.K / 256);
    const int nrk = p.rac_ld / 64;
    const int64_t sf_per_expert = ((p.N + 127) / 128) * 128 * (p.K / 16);

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------- producer
            ptx::prefetch_tmap(&tm_a);
            ptx::prefetch_tmap(&tm_b);
            uint32_t stage = 0, phase = 0;
            uint32_t issued_phase[STAGES];
            bool issued[STAGES];
            for (int s = 0; s < STAGES; ++s) issued[s] = false, issued_phase[s] = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
                const int mt = t / n_tiles, nt = t % n_tiles;
                const int m0 = mt * BM;
                const int e = find_expert(sh->offsets, E, m0);
                int nrow0, nrow1;  // rows inside expert e's [N x K] weight
                if (swiglu) { nrow0 = nt * 128; nrow1 = p.inter + nt * 128; }
                else { nrow0 = nt * BN; nrow1 = nt * BN + 128; }
                const int brow0 = (int)(e * p.N) + nrow0, brow1 = (int)(e * p.N) + nrow1;
                const uint8_t *sfa_src = p.a_scales + (int64_t)(m0 / 128) * (p.K / 64) * 512;
                const uint8_t *sfb_e = p.b_scales + (int64_t)e * sf_per_expert;
                const uint8_t *sfb_src0 = sfb_e + (int64_t)(nrow0 / 128) * (p.K / 64) * 512;
                const uint8_t *sfb_src1 = sfb_e + (int64_t)(nrow1 / 128) * (p.K / 64) * 512;
                for (int kb = 0; kb < nkb + nrk; ++kb) {
                    if (!wait_bar(ptx::smem_u32(&sh->empty[stage]), phase ^ 1u, abort_flag, p.dev_status)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = stage_base + stage * STAGE_BYTES;
                    uint8_t *sb = sa + A_BYTES;
                    const uint32_t fb = ptx::smem_u32(&sh->full[stage]);
                    if (kb < nkb) {
                        uint8_t *ssfa = sb + B_BYTES;
                        uint8_t *ssfb = ssfa + SFA_BYTES;
                        ptx::mbar_arrive_expect_tx(fb, STAGE_BYTES);
                        ptx::tma_load_2d(ptx::smem_u32(sa), &tm_a, kb * 128, m0, fb);
                        ptx::tma_load_2d(ptx::smem_u32(sb), &tm_b, kb * 128, brow0, fb);
                        ptx::tma_load_2d(ptx::smem_u32(sb + B_BYTES / 2), &tm_b, kb * 128, brow1, fb);
                        ptx::bulk_load(ptx::smem_u32(ssfa), sfa_src + kb * 2048, SFA_BYTES, fb);
                        ptx::bulk_load(ptx::smem_u32(ssfb), sfb_src0 + kb * 2048, SFB_BYTES / 2, fb);
                        ptx::bulk_load(ptx::smem_u32(ssfb + SFB_BYTES / 2), sfb_src1 + kb * 2048, SFB_BYTES / 2, fb);
                    } else {
                        const int rk = kb - nkb;
                        ptx::mbar_arrive_expect_tx(fb, RAC_STAGE_BYTES);
                        ptx::tma_load_2d(ptx::smem_u32(sa), &tm_ra, rk * 64, m0, fb);
                        ptx::tma_load_2d(ptx::smem_u32(sb), &tm_rb, rk * 64, brow0, fb);
                        ptx::tma_load_2d(ptx::smem_u32(sb + B_BYTES / 2), &tm_rb, rk * 64, brow1, fb);
                    }
                    issued[stage] = true;
                    issued_phase[stage] = phase;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                // drain copies still in flight before the CTA's memory is released
                for (int s = 0; s < STAGES; ++s)
                    if (issued[s])
                        wait_bar(ptx::smem_u32(&sh->full[s]), issued_phase[s], abort_flag, p.dev_status, true);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // --------------------------------------------------- MMA issuer
            const uint32_t idesc4 = ptx::idesc_mxf4nvf4(BM, BN);
            const uint32_t idesc16 = ptx::idesc_bf16(BM, BN);
            uint32_t stage = 0, phase = 0, drain_phase = 0;
            bool ok = true;
            bool issued_any = false;
            int iter = 0;
            for (int t = blockIdx.x; ok && t < total; t += gridDim.x, ++iter) {
                if (!wait_bar(ptx::smem_u32(&sh->tmem_empty), (uint32_t)(iter & 1) ^ 1u, abort_flag, p.dev_status)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                for (int kb = 0; kb < nkb && ok; ++kb) {
                    if (!wait_bar(ptx::smem_u32(&sh->full[stage]), phase, abort_flag, p.dev_status)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t sa = ptx::smem_u32(stage_base + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
                    const uint32_t ssfa = sb + B_BYTES;
                    const uint32_t ssfb = ssfa + SFA_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        ptx::tmem_cp_32x128b_warpx4(tmem + SFA_COL + 4 * kk, ptx::make_sdesc(ssfa + 512 * kk, 0, 128, 0));
                        ptx::tmem_cp_32x128b_warpx4(tmem + SFB_COL + 8 * kk, ptx::make_sdesc(ssfb + 512 * kk, 0, 128, 0));
                        ptx::tmem_cp_32x128b_warpx4(tmem + SFB_COL + 8 * kk + 4,
                                                    ptx::make_sdesc(ssfb + SFB_BYTES / 2 + 512 * kk, 0, 128, 0));
                    }
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        uint64_t ad = ptx::make_sdesc(sa + 32 * kk, 16, 1024, 2);
                        uint64_t bd = ptx::make_sdesc(sb + 32 * kk, 16, 1024, 2);
                        ptx::mma_mxf4nvf4(tmem + ACC_COL, ad, bd, idesc4, tmem + SFA_COL + 4 * kk,
                                          tmem + SFB_COL + 8 * kk, (kb | kk) != 0);
                    }
                    ptx::tc_commit(ptx::smem_u32(&sh->empty[stage]));
                    issued_any = true;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (ok && nrk > 0) {
                    // the BF16 MMAs accumulate into the same TMEM tile: wait for
                    // the FP4 MMAs to complete first
                    ptx::tc_commit(ptx::smem_u32(&sh->drain));
                    if (!wait_bar(ptx::smem_u32(&sh->drain), drain_phase, abort_flag, p.dev_status)) { ok = false; }
                    drain_phase ^= 1u;
                    ptx::tc_fence_after();
                    for (int rk = 0; rk < nrk && ok; ++rk) {
                        if (!wait_bar(ptx::smem_u32(&sh->full[stage]), phase, abort_flag, p.dev_status)) { ok = false; break; }
                        ptx::tc_fence_after();
                        const uint32_t sa = ptx::smem_u32(stage_base + stage * STAGE_BYTES);
                        const uint32_t sb = sa + A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            uint64_t ad = ptx::make_sdesc(sa + 32 * kk, 16, 1024, 2);
                            uint64_t bd = ptx::make_sdesc(sb + 32 * kk, 16, 1024, 2);
                            ptx::mma_bf16(tmem + ACC_COL, ad, bd, idesc16, 1u);
                        }
                        ptx::tc_commit(ptx::smem_u32(&sh->empty[stage]));
                        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                    }
                }
                if (ok) ptx::tc_commit(ptx::smem_u32(&sh->tmem_full));
            }
            if (!ok && issued_any) {
                // let every issued MMA finish before TMEM is released
                ptx::tc_commit(ptx::smem_u32(&sh->drain));
                wait_bar(ptx::smem_u32(&sh->drain), drain_phase, abort_flag, p.dev_status, true);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------- epilogue
        // Warp w owns TMEM lane quadrant w % 4 (32 rows) and one half of the
        // tile's columns; it copies its whole slice to registers, frees the
        // accumulator for the next tile's MMAs, then computes and stores.
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const int row_in_tile = q * 32 + lane;
        const float s_a = *p.a_s_t;
        int iter = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++iter) {
            bool ok = true;
            if (lane == 0) ok = wait_bar(ptx::smem_u32(&sh->tmem_full), (uint32_t)(iter & 1), abort_flag, p.dev_status);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            ptx::tc_fence_after();
            const int mt = t / n_tiles, nt = t % n_tiles;
            const int m0 = mt * BM;
            const int e = find_expert(sh->offsets, E, m0);
            const uint32_t tbase = tmem + ACC_COL + ((uint32_t)(q * 32) << 16);
            uint32_t v[128];
            if (swiglu) {
                // gate columns [64 half, +64) and the matching up columns
                ptx::tmem_ld_32x32b_x32(tbase + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
                ptx::tmem_ld_32x32b_x32(tbase + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
                ptx::tmem_ld_32x32b_x32(tbase + 128 + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&v[64]));
                ptx::tmem_ld_32x32b_x32(tbase + 128 + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[96]));
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    ptx::tmem_ld_32x32b_x32(tbase + half * 128 + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
            }
            ptx::tmem_ld_wait();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&sh->tmem_empty));

            const float scale = __fmul_rn(s_a, p.b_s_t[e]);
            const int64_t r = (int64_t)m0 + row_in_tile;
            const int token = p.row_token[r];
            if (p.epilogue == MOE_EPI_SWIGLU_BF16) {
                uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.out) + r * p.ld_out +
                                                       nt * 128 + half * 64);
                float hmax = 0.0f;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t w4[4];
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int j = c * 8 + jj * 2;
                        float h0 = 0.0f, h1 = 0.0f;
                        if (token >= 0) {
                            h0 = silu(scale * __uint_as_float(v[j])) * (scale * __uint_as_float(v[64 + j]));
                            h1 = silu(scale * __uint_as_float(v[j + 1])) * (scale * __uint_as_float(v[64 + j + 1]));
                        }
                        const __nv_bfloat16 b0 = __float2bfloat16_rn(h0), b1 = __float2bfloat16_rn(h1);
                        hmax = fmaxf(hmax, fmaxf(fabsf(__bfloat162float(b0)), fabsf(__bfloat162float(b1))));
                        w4[jj] = (uint32_t)__bfloat16_as_ushort(b0) | ((uint32_t)__bfloat16_as_ushort(b1) << 16);
                    }
                    dst[c] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
                if (p.amax_out) {
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) hmax = fmaxf(hmax, __shfl_xor_sync(0xffffffffu, hmax, o));
                    if (lane == 0) atomicMax(p.amax_out, __float_as_uint(hmax));
                }
            } else if (Cfg<STAGES>::STAGING) {
                // f32 out: each lane stages 64 contiguous floats of its row and
                // moves them with one 256-byte bulk store / bulk add-reduction;
                // lanes 0-15 then 16-31 share the warp's 16 slots.
                const bool scatter = p.epilogue == MOE_EPI_SCATTER_ADD_F32;
                const float mul = scatter ? (token >= 0 ? __fmul_rn(scale, p.row_gate[r]) : 0.0f) : scale;
                float *orow = reinterpret_cast<float *>(p.out) +
                              (scatter ? (int64_t)(token >= 0 ? token : 0) : r) * p.ld_out + nt * BN + half * 128;
                float *slot = staging + ((warp - 2) * 16 + (lane & 15)) * SLOT_FLOATS;
                const uint32_t slot_s = ptx::smem_u32(slot);
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        if ((lane >> 4) == rr && token >= 0) {
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                reinterpret_cast<float4 *>(slot)[j] =
                                    make_float4(mul * __uint_as_float(v[cc * 64 + 4 * j]),
                                                mul * __uint_as_float(v[cc * 64 + 4 * j + 1]),
                                                mul * __uint_as_float(v[cc * 64 + 4 * j + 2]),
                                                mul * __uint_as_float(v[cc * 64 + 4 * j + 3]));
                            ptx::fence_proxy_async_smem();
                            if (scatter) ptx::bulk_reduce_add_f32(orow + cc * 64, slot_s, 256);
                            else ptx::bulk_store(orow + cc * 64, slot_s, 256);
                            ptx::bulk_commit();
                            ptx::bulk_wait_read();          // the slot is reused by the other half-warp
                        }
                        __syncwarp();
                    }
                }
            } else if (p.epilogue == MOE_EPI_STORE_F32) {
                if (token >= 0) {
                    float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.out) + r * p.ld_out +
                                                             nt * BN + half * 128);
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        dst[j] = make_float4(scale * __uint_as_float(v[4 * j]), scale * __uint_as_float(v[4 * j + 1]),
                                             scale * __uint_as_float(v[4 * j + 2]), scale * __uint_as_float(v[4 * j + 3]));
                }
            } else if (token >= 0) {
                const float gw = __fmul_rn(scale, p.row_gate[r]);
                float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.out) + (int64_t)token * p.ld_out +
                                                         nt * BN + half * 128);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    atomicAdd(dst + j, make_float4(gw * __uint_as_float(v[4 * j]), gw * __uint_as_float(v[4 * j + 1]),
                                                   gw * __uint_as_float(v[4 * j + 2]), gw * __uint_as_float(v[4 * j + 3])));
            }
        }
        if (Cfg<STAGES>::STAGING) ptx::bulk_wait_all();     // this lane's bulk writes are complete
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ----------------------------------------------------------------- host side

static bool smem_attr_done[2][64];

}  // namespace gemm
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status moe_w4a4_grouped_gemm_rac(
    const uint8_t *a_codes_dev, const uint8_t *a_scales_dev, const float *a_s_t_dev, int64_t M_pad_max,
    const uint8_t *b_codes_dev, const uint8_t *b_scales_dev, const float *b_s_t_dev, int64_t N, int64_t K, int32_t E,
    const int32_t *offsets_dev, int32_t rac_ld, const void *rho_dev, const void *w_sel_dev, int32_t epilogue,
    const int32_t *row_token_dev, const float *row_gate_dev, void *out_dev, int64_t ld_out, float *amax_out_dev,
    int32_t *dev_status, void *stream)
{
    using namespace nvfp4::gemm;
    cudaStream_t st = (cudaStream_t)stream;
    NVFP4_REQUIRE(a_codes_dev && a_scales_dev && a_s_t_dev && b_codes_dev && b_scales_dev && b_s_t_dev &&
                  offsets_dev && row_token_dev && out_dev, NVFP4_ERR_INVALID_ARG,
                  "moe_w4a4_grouped_gemm_rac: null pointer");
    NVFP4_REQUIRE(epilogue >= 0 && epilogue <= 2, NVFP4_ERR_INVALID_ARG, "moe_w4a4_grouped_gemm_rac: bad epilogue");
    NVFP4_REQUIRE(epilogue != MOE_EPI_SCATTER_ADD_F32 || row_gate_dev, NVFP4_ERR_INVALID_ARG,
                  "moe_w4a4_grouped_gemm_rac: scatter-add needs row_gate");
    NVFP4_REQUIRE(E >= 1 && E <= MAX_E, NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_w4a4_grouped_gemm_rac: 1 <= E <= 256");
    NVFP4_REQUIRE(K >= 256 && K % 256 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "moe_w4a4_grouped_gemm_rac: K must be a positive multiple of 256 (K=%lld)", (long long)K);
    NVFP4_REQUIRE(N >= 256 && N % 256 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "moe_w4a4_grouped_gemm_rac: N must be a positive multiple of 256 (N=%lld)", (long long)N);
    NVFP4_REQUIRE(M_pad_max >= 128 && M_pad_max % 128 == 0 && M_pad_max < (1ll << 31), NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "moe_w4a4_grouped_gemm_rac: M_pad_max must be a positive multiple of 128");
    NVFP4_REQUIRE((int64_t)E * N < (1ll << 31), NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_w4a4_grouped_gemm_rac: E*N too large");
    NVFP4_REQUIRE(rac_ld >= 0 && rac_ld <= 256 && rac_ld % 64 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "moe_w4a4_grouped_gemm_rac: rac_ld must be 0..256 and a multiple of 64");
    NVFP4_REQUIRE(rac_ld == 0 || (rho_dev && w_sel_dev), NVFP4_ERR_INVALID_ARG,
                  "moe_w4a4_grouped_gemm_rac: rac_ld > 0 needs rho and w_sel");
    const int inter = (int)(N / 2);
    if (epilogue == MOE_EPI_SWIGLU_BF16) {
        NVFP4_REQUIRE(inter % 128 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_w4a4_grouped_gemm_rac: SwiGLU needs I % 128 == 0");
        NVFP4_REQUIRE(ld_out >= inter && ld_out % 8 == 0, NVFP4_ERR_ALIGNMENT,
                      "moe_w4a4_grouped_gemm_rac: SwiGLU ld_out must be >= N/2 and a multiple of 8");
    } else {
        NVFP4_REQUIRE(ld_out >= N && ld_out % 4 == 0, NVFP4_ERR_ALIGNMENT,
                      "moe_w4a4_grouped_gemm_rac: ld_out must be >= N and a multiple of 4");
    }
    NVFP4_REQUIRE(aligned16(a_codes_dev) && aligned16(a_scales_dev) && aligned16(b_codes_dev) &&
                  aligned16(b_scales_dev) && aligned16(out_dev) && (rac_ld == 0 || (aligned16(rho_dev) && aligned16(w_sel_dev))),
                  NVFP4_ERR_ALIGNMENT, "moe_w4a4_grouped_gemm_rac: pointers must be 16-byte aligned");

    CUtensorMap tm_a, tm_b, tm_ra, tm_rb;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    bool ok = make_tmap_2d(&tm_a, a_codes_dev, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)K / 2, (uint64_t)M_pad_max,
                           (uint64_t)K / 2, 128, 128, sw) &&
              make_tmap_2d(&tm_b, b_codes_dev, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)K / 2, (uint64_t)E * N,
                           (uint64_t)K / 2, 128, 128, sw);
    if (ok && rac_ld > 0) {
        ok = make_tmap_2d(&tm_ra, rho_dev, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)rac_ld, (uint64_t)M_pad_max,
                          (uint64_t)rac_ld * 2, 64, 128, sw) &&
             make_tmap_2d(&tm_rb, w_sel_dev, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)rac_ld, (uint64_t)E * N,
                          (uint64_t)rac_ld * 2, 64, 128, sw);
    } else {
        tm_ra = tm_a;
        tm_rb = tm_b;
    }
    NVFP4_REQUIRE(ok, NVFP4_ERR_CUDA, "moe_w4a4_grouped_gemm_rac: tensor map encoding failed");

    // SwiGLU (bf16 out) keeps 4 stages; the f32 epilogues trade one for staging
    const bool four = epilogue == MOE_EPI_SWIGLU_BF16;
    auto kern = four ? k_moe_gemm<4> : k_moe_gemm<3>;
    const uint32_t smem = four ? Cfg<4>::SMEM : Cfg<3>::SMEM;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !smem_attr_done[four][dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return check_launch("moe_w4a4_grouped_gemm_rac: smem attribute");
        smem_attr_done[four][dev] = true;
    }
    Params p{};
    p.a_scales = a_scales_dev;
    p.a_s_t = a_s_t_dev;
    p.b_scales = b_scales_dev;
    p.b_s_t = b_s_t_dev;
    p.N = N;
    p.K = K;
    p.E = E;
    p.offsets = offsets_dev;
    p.rac_ld = rac_ld;
    p.epilogue = epilogue;
    p.inter = inter;
    p.row_token = row_token_dev;
    p.row_gate = row_gate_dev;
    p.out = out_dev;
    p.ld_out = ld_out;
    p.amax_out = (epilogue == MOE_EPI_SWIGLU_BF16) ? reinterpret_cast<unsigned int *>(amax_out_dev) : nullptr;
    p.dev_status = dev_status;
    if (p.amax_out && cudaMemsetAsync(p.amax_out, 0, sizeof(float), st) != cudaSuccess)
        return check_launch("moe_w4a4_grouped_gemm_rac: memset");
    int64_t n_tiles = epilogue == MOE_EPI_SWIGLU_BF16 ? inter / 128 : N / BN;
    int64_t max_tiles = (M_pad_max / BM) * n_tiles;
    int grid = (int)std::min<int64_t>(num_sms(), max_tiles);
    kern<<<grid, NUM_THREADS, smem, st>>>(tm_a, tm_b, tm_ra, tm_rb, p);
    return check_launch("k_moe_gemm");
}
