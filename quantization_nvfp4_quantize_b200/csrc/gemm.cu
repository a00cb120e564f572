// gemm.cu -- persistent grouped W4A4 (NVFP4) expert GEMM with Residual
// Activation Compensation on the sm_100a tensor cores.
//
// Two shapes of the same kernel:
//   single  one CTA per SM computes 128 routed rows x 256 output features;
//           expert segments padded to 128 rows.
//   pair    a 2-CTA cluster (tcgen05 .cta_group::2) computes 256 routed rows
//           x 256 features: each CTA holds 128 rows of A, half of B (128
//           features) and the scale factors its half needs; the even CTA
//           ("leader") issues every scale-factor copy and MMA for both SMs.
//           Per SM the MMA and scale-copy work per stage is unchanged, but
//           each SM stages only half the B bytes, which leaves room for a
//           fifth stage.  Expert segments padded to 256 rows.
// The same kernel serves the BF16 grouped GEMM (moe_bf16_grouped_gemm): no
// FP4 stage, K / 64 BF16 stages over the whole contraction, unit tensor
// scales.
//
// Warps (384 threads per CTA):
//   warps 0, 2  TMA producers (one lane each): per 256-element K step warp 0
//               loads the A tile (128 rows x 128 B packed E2M1, 128-byte
//               swizzle) and A's 512-byte scale atoms, warp 2 this CTA's B
//               tile(s) and B's scale atoms, into a ring of stages; then the
//               RAC stages (bf16 rho and w_sel tiles, 64 channels).  TMA
//               copies issued by one thread are processed largely one after
//               another, so two issuing threads keep more bytes in flight.
//               In the pair shape both CTAs load their halves and every copy
//               completes on the leader's barrier.
//   warp 3      scale-factor copier (one lane, leader only in the pair shape):
//               once a stage has landed, copies its 12 scale atoms into that
//               stage's own TMEM scale buffer (tcgen05.cp 32x128b.warpx4) and
//               commits to the stage's sf_full barrier.  Issued from their own
//               thread, the copies overlap the MMAs of earlier stages; issued
//               from the MMA thread they would serialize with them (12 copies
//               cost about as much tensor-pipe time as the stage's 4 MMAs).
//               A stage's buffer is free again when the stage is: the
//               producers refill a stage only after the MMAs reading it are
//               done.
//   warp 1      MMA issuer (one lane, leader only in the pair shape): per
//               stage 4 block-scaled tcgen05.mma kind::mxf4nvf4 (K64) into
//               one TMEM accumulator; after the FP4 K loop it drains (commit +
//               wait) and accumulates the RAC stages with kind::f16 BF16 MMAs
//               (K16) into the same accumulator.
//   warps 4..11 epilogue: each warp copies its TMEM slice (32-lane quadrant
//               w % 4, one half of the columns) into registers and releases
//               the accumulator at once, so the next tile's MMAs overlap the
//               math and stores: y = s_a s_b D, then store f32 / SwiGLU ->
//               bf16 / router-weighted scatter-add into the token-major
//               output.
// Tiles never span two experts (segments are multiples of the tile height);
// the tile count comes from the device-side offsets (no host sync).  Tile
// order: m-major, except that the scatter-add epilogue runs the n-tiles in
// groups of 2, so the band of output being reduced into is an eighth of Y
// (much of it still leaves L2 between a row's contributions).
//
// Shared memory: a ring of stages (single 54 KB, pair 38 KB: 4 / 5 stages for
// the bf16 epilogue, 3 / 5 for the f32 ones) plus, for the f32 epilogues, a
// 4 KB 32 x 32 transpose tile per epilogue warp: a warp's rows leave as 16-byte
// vector stores or add-reductions that cover 4 rows x 128 contiguous bytes per
// instruction, without the TMA unit that feeds the operands.
// TMEM: 512 columns = accumulator [0,256) + one 48-column scale buffer per
// stage at 256 + 48 s: A's scale factors in its first 16 columns (4 atoms x 4
// columns), B's in the next 32 (4 x 8 columns); at most 5 stages.
// Every mbarrier wait is bounded (1 s); on expiry the kernel records
// NVFP4_ERR_TIMEOUT, all roles stop, in-flight copies and MMAs are drained
// (bounded) and TMEM is freed before exit.  Every TMA load writes only the
// issuing CTA's own shared memory.
#include "common.cuh"
#include "ptx.cuh"

#include <cuda.h>
#include <algorithm>
#include <mutex>
#include <cstdlib>

namespace nvfp4 {
namespace gemm {

constexpr int BN = 256;
constexpr int MAX_STAGES = 5;
constexpr uint32_t A_BYTES = 128 * 128;         // 16 KB: 128 rows x 256 FP4
constexpr uint32_t SFA_BYTES = 4 * 512;         // 4 atoms (K=256 / 64)
constexpr uint32_t SFB_BYTES = 8 * 512;         // 2 row blocks x 4 atoms (all 256 features)
constexpr int NUM_THREADS = 384;                // 4 control warps + 8 epilogue warps
constexpr int EPI_WARPS = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0, SF_COL = 256, SF_STRIDE = 48;  // scale buffer of stage s: SF_COL + 48 s
constexpr int PROD_A_WARP = 0, MMA_WARP = 1, PROD_B_WARP = 2, COPY_WARP = 3, EPI_WARP0 = 4;
constexpr int MAX_E = 256;
constexpr uint64_t TIMEOUT_NS = 1000000000ull;    // default bound of every mbarrier wait (1 s)
constexpr uint32_t STAGING_BYTES = EPI_WARPS * 32 * 32 * 4;   // one 32 x 32 f32 transpose tile per epilogue warp
constexpr int BOX_ROWS = 128;                   // rows per operand TMA box (128-byte rows)

template <bool PAIR>
struct Geo {
    static constexpr int TILE_M = PAIR ? 256 : 128;                        // routed rows per tile
    static constexpr uint32_t B_LOCAL = (PAIR ? 128 : 256) * 128;           // B bytes this CTA stages
    static constexpr uint32_t STAGE = A_BYTES + B_LOCAL + SFA_BYTES + SFB_BYTES;
    static constexpr uint32_t RAC_STAGE = A_BYTES + B_LOCAL;
    static constexpr uint32_t TX = (PAIR ? 2 : 1) * STAGE;                  // bytes the full barrier expects
    static constexpr uint32_t RAC_TX = (PAIR ? 2 : 1) * RAC_STAGE;
};

template <int STAGES, bool PAIR, bool STAGING>
struct Cfg {
    static constexpr uint32_t SMEM = STAGES * Geo<PAIR>::STAGE + (STAGING ? STAGING_BYTES : 0) +
                                     1024 /*align*/ + 2048 /*barriers, offsets*/;
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(SF_COL + SF_STRIDE * STAGES <= TMEM_COLS, "TMEM budget");
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
    int n_group;               // tile order: n-tiles per group (divides the n-tile count)
    const int32_t *row_token;
    const float *row_gate;
    void *out;
    int64_t ld_out;
    unsigned int *amax_out;    // SwiGLU: max |h| (float bits), or null
    int l2_hints;              // scatter-add: stream A with evict-first loads, reduce into the output with evict-last
    int fp8;                   // 1: A and B are E4M3 codes (the FP8 kernel instance: kind::f8f6f4 MMAs, no scale factors)
    uint64_t wait_limit_ns;    // bound of every mbarrier wait
    int debug_withhold_acc;    // test hook: no "accumulator ready" signal for the first tile (1-SM shape)
    int32_t *dev_status;
};

struct Shared {
    uint64_t full[MAX_STAGES];
    uint64_t sf_full[MAX_STAGES];
    uint64_t empty[MAX_STAGES];
    uint64_t tmem_full;
    uint64_t tmem_empty;
    uint64_t drain;
    uint64_t cp_drain;
    uint32_t tmem_base;
    int abort_flag;
    int offsets[MAX_E + 1];
};

// Bounded wait; returns false on abort or timeout (then sets the abort flag).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                         int32_t *dev_status, uint64_t limit_ns, bool ignore_abort = false)
{
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 63u) {
            if (!ignore_abort && *abort_flag) return false;
            uint64_t now = globaltimer_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > limit_ns) {
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

// Tile t -> (m-tile, n-tile).  n-tiles run in groups of n_group; inside a
// group the tiles are m-major with the group's n-tiles innermost, so the
// output columns in flight stay within one group's band (n_group = n_tiles:
// plain m-major order, each A tile reused by all n-tiles back to back).
__device__ __forceinline__ void tile_coords(int t, int m_tiles, int n_group, int &mt, int &nt)
{
    const int per_group = m_tiles * n_group;
    const int g = t / per_group, rem = t - g * per_group;
    mt = rem / n_group;
    nt = g * n_group + (rem - mt * n_group);
}

__device__ __forceinline__ float silu(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// Scale-atom row of the 2D [bytes/256 x 256] view of a scale buffer.
__device__ __forceinline__ int32_t sf_row(int64_t byte_off) { return (int32_t)(byte_off >> 8); }

template <int STAGES, bool PAIR, bool STAGING, bool FP8>
__global__ void __launch_bounds__(NUM_THREADS, 1)
k_moe_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
           const __grid_constant__ CUtensorMap tm_ra, const __grid_constant__ CUtensorMap tm_rb,
           const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb, Params p)
{
    using G = Geo<PAIR>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *stage_base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *staging = reinterpret_cast<float *>(stage_base + STAGES * G::STAGE);
    Shared *sh = reinterpret_cast<Shared *>(stage_base + STAGES * G::STAGE + (STAGING ? STAGING_BYTES : 0));
    volatile int *abort_flag = &sh->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    const uint32_t rank = PAIR ? ptx::cluster_ctarank() : 0u;       // 0 = leader
    const bool leader = rank == 0;
    const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;   // tile-scheduling unit
    const int n_units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(ptx::smem_u32(&sh->full[s]), 2);      // both producers arrive
            ptx::mbar_init(ptx::smem_u32(&sh->sf_full[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&sh->empty[s]), 1);
        }
        ptx::mbar_init(ptx::smem_u32(&sh->tmem_full), 1);
        ptx::mbar_init(ptx::smem_u32(&sh->tmem_empty), PAIR ? 2 * EPI_WARPS : EPI_WARPS);
        ptx::mbar_init(ptx::smem_u32(&sh->drain), 1);
        ptx::mbar_init(ptx::smem_u32(&sh->cp_drain), 1);
        sh->abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::fence_proxy_async_smem();
    }
    for (int i = threadIdx.x; i <= E; i += NUM_THREADS) sh->offsets[i] = p.offsets[i];
    if (warp == 0) {
        if (PAIR) {
            ptx::tmem_alloc_pair(ptx::smem_u32(&sh->tmem_base), TMEM_COLS);
            ptx::tmem_relinquish_pair();
        } else {
            ptx::tmem_alloc(ptx::smem_u32(&sh->tmem_base), TMEM_COLS);
            ptx::tmem_relinquish();
        }
    }
    ptx::tc_fence_before();
    if (PAIR) ptx::cluster_sync();         // barriers of both CTAs initialized before any remote use
    else __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sh->tmem_base;

    const int swiglu = p.epilogue == MOE_EPI_SWIGLU_BF16;
    const int n_tiles = swiglu ? p.inter / 128 : (int)(p.N / BN);
    const int m_tiles = sh->offsets[E] / G::TILE_M;
    const int total = m_tiles * n_tiles;
    const int nkb = (int)(p.K / (FP8 ? 128 : 256));   // main stages: 128 bytes of K per row
    const int nrk = p.rac_ld / 64;
    const int64_t sf_per_expert = ((p.N + 127) / 128) * 128 * (p.K / 16);

    if (warp == PROD_A_WARP || warp == PROD_B_WARP) {
        if (lane == 0) {
            // -------------------------------------------------- producers
            // Two issuing threads: TMA copies from one thread are processed
            // largely one after another, so A (+ its scale atoms) and B (+
            // its scale atoms) are issued from separate warps.  Each arrives
            // on the stage's full barrier with the bytes it will deliver
            // (both CTAs' bytes in the pair shape, where only the leader
            // arrives and every copy completes on the leader's barrier).
            const bool role_a = warp == PROD_A_WARP;
            ptx::prefetch_tmap(role_a ? &tm_a : &tm_b);
            if (PAIR) ptx::prefetch_tmap(role_a ? &tm_sfa : &tm_sfb);
            if (p.rac_ld > 0) ptx::prefetch_tmap(role_a ? &tm_ra : &tm_rb);
            const uint32_t mult = PAIR ? 2u : 1u;
            const uint32_t tx_fp4 = mult * (role_a ? (A_BYTES + (FP8 ? 0u : SFA_BYTES))
                                                   : (G::B_LOCAL + (FP8 ? 0u : SFB_BYTES)));
            const uint32_t tx_rac = mult * (role_a ? A_BYTES : G::B_LOCAL);
            // the scatter-add GEMM reads each A tile once per group of n-tiles:
            // let those lines leave L2 first so the output band stays resident
            const bool hint_a = p.l2_hints != 0;
            const uint64_t pol_a = ptx::policy_evict_first();
            uint32_t stage = 0, phase = 0;
            uint32_t issued_phase[STAGES];
            bool issued[STAGES];
            for (int s = 0; s < STAGES; ++s) issued[s] = false, issued_phase[s] = 0;
            bool ok = true;
            for (int t = unit; ok && t < total; t += n_units) {
                int mt, nt;
                tile_coords(t, m_tiles, p.n_group, mt, nt);
                const int m0 = mt * G::TILE_M;
                const int e = find_expert(sh->offsets, E, m0);
                const int arow = m0 + (int)rank * 128;      // this CTA's 128 rows of A
                int nrow0, nrow1;  // rows inside expert e's [N x K] weight (the two 128-feature halves)
                if (swiglu) { nrow0 = nt * 128; nrow1 = p.inter + nt * 128; }
                else { nrow0 = nt * BN; nrow1 = nt * BN + 128; }
                const int brow0 = (int)(e * p.N) + nrow0, brow1 = (int)(e * p.N) + nrow1;
                const int64_t sfa_off = (int64_t)(arow / 128) * (p.K / 64) * 512;
                const int64_t sfb_e = (int64_t)e * sf_per_expert;
                const int64_t sfb_off0 = sfb_e + (int64_t)(nrow0 / 128) * (p.K / 64) * 512;
                const int64_t sfb_off1 = sfb_e + (int64_t)(nrow1 / 128) * (p.K / 64) * 512;
                for (int kb = 0; kb < nkb + nrk; ++kb) {
                    if (!wait_bar(ptx::smem_u32(&sh->empty[stage]), phase ^ 1u, abort_flag, p.dev_status, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = stage_base + stage * G::STAGE;
                    uint8_t *sb = sa + A_BYTES;
                    uint8_t *ssfa = sb + G::B_LOCAL;
                    uint8_t *ssfb = ssfa + SFA_BYTES;
                    const uint32_t fb = ptx::smem_u32(&sh->full[stage]);
                    const bool fp4 = kb < nkb;
                    const int rk = kb - nkb;
                    if (leader) ptx::mbar_arrive_expect_tx(fb, fp4 ? tx_fp4 : tx_rac);
                    if (PAIR) {
                        const uint32_t lfb = ptx::mapa_shared(fb, 0);     // the leader's barrier
                        const int browr = rank ? brow1 : brow0;
                        if (role_a && hint_a) {
                            if (fp4) {
                                ptx::tma_load_2d_pair_hint(ptx::smem_u32(sa), &tm_a, kb * 128, arow, lfb, pol_a);
                                if (!FP8)
                                    ptx::tma_load_2d_pair_hint(ptx::smem_u32(ssfa), &tm_sfa, 0,
                                                               sf_row(sfa_off + kb * 2048), lfb, pol_a);
                            } else {
                                ptx::tma_load_2d_pair_hint(ptx::smem_u32(sa), &tm_ra, rk * 64, arow, lfb, pol_a);
                            }
                        } else if (role_a) {
                            if (fp4) {
                                ptx::tma_load_2d_pair(ptx::smem_u32(sa), &tm_a, kb * 128, arow, lfb);
                                if (!FP8)
                                    ptx::tma_load_2d_pair(ptx::smem_u32(ssfa), &tm_sfa, 0, sf_row(sfa_off + kb * 2048),
                                                          lfb);
                            } else {
                                ptx::tma_load_2d_pair(ptx::smem_u32(sa), &tm_ra, rk * 64, arow, lfb);
                            }
                        } else if (fp4) {
                            ptx::tma_load_2d_pair(ptx::smem_u32(sb), &tm_b, kb * 128, browr, lfb);
                            if (!FP8) {
                                ptx::tma_load_2d_pair(ptx::smem_u32(ssfb), &tm_sfb, 0, sf_row(sfb_off0 + kb * 2048),
                                                      lfb);
                                ptx::tma_load_2d_pair(ptx::smem_u32(ssfb + SFB_BYTES / 2), &tm_sfb, 0,
                                                      sf_row(sfb_off1 + kb * 2048), lfb);
                            }
                        } else {
                            ptx::tma_load_2d_pair(ptx::smem_u32(sb), &tm_rb, rk * 64, browr, lfb);
                        }
                    } else if (role_a) {
                        if (fp4) {
                            if (hint_a) ptx::tma_load_2d_hint(ptx::smem_u32(sa), &tm_a, kb * 128, m0, fb, pol_a);
                            else ptx::tma_load_2d(ptx::smem_u32(sa), &tm_a, kb * 128, m0, fb);
                            if (!FP8)
                                ptx::bulk_load(ptx::smem_u32(ssfa), p.a_scales + sfa_off + kb * 2048, SFA_BYTES, fb);
                        } else if (hint_a) {
                            ptx::tma_load_2d_hint(ptx::smem_u32(sa), &tm_ra, rk * 64, m0, fb, pol_a);
                        } else {
                            ptx::tma_load_2d(ptx::smem_u32(sa), &tm_ra, rk * 64, m0, fb);
                        }
                    } else if (fp4) {
                        ptx::tma_load_2d(ptx::smem_u32(sb), &tm_b, kb * 128, brow0, fb);
                        ptx::tma_load_2d(ptx::smem_u32(sb + G::B_LOCAL / 2), &tm_b, kb * 128, brow1, fb);
                        if (!FP8) {
                            ptx::bulk_load(ptx::smem_u32(ssfb), p.b_scales + sfb_off0 + kb * 2048, SFB_BYTES / 2, fb);
                            ptx::bulk_load(ptx::smem_u32(ssfb + SFB_BYTES / 2), p.b_scales + sfb_off1 + kb * 2048,
                                           SFB_BYTES / 2, fb);
                        }
                    } else {
                        ptx::tma_load_2d(ptx::smem_u32(sb), &tm_rb, rk * 64, brow0, fb);
                        ptx::tma_load_2d(ptx::smem_u32(sb + G::B_LOCAL / 2), &tm_rb, rk * 64, brow1, fb);
                    }
                    issued[stage] = true;
                    issued_phase[stage] = phase;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                // drain copies still in flight before the CTA's memory is released
                if (!PAIR || leader) {
                    for (int s = 0; s < STAGES; ++s)
                        if (issued[s])
                            wait_bar(ptx::smem_u32(&sh->full[s]), issued_phase[s], abort_flag, p.dev_status, p.wait_limit_ns, true);
                } else {
                    // the peer's copies complete on the leader's barriers: give them 100 us
                    const uint64_t t0 = globaltimer_ns();
                    while (globaltimer_ns() - t0 < 100000ull) { }
                }
            }
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        if (lane == 0 && leader) {
            // --------------------------------------------------- MMA issuer
            const uint32_t idesc4 = ptx::idesc_mxf4nvf4(PAIR ? 256 : 128, BN);
            const uint32_t idesc8 = ptx::idesc_e4m3(PAIR ? 256 : 128, BN);
            const uint32_t idesc16 = ptx::idesc_bf16(PAIR ? 256 : 128, BN);
            uint32_t stage = 0, phase = 0, drain_phase = 0;
            bool ok = true;
            bool issued_any = false;
            int iter = 0;
            for (int t = unit; ok && t < total; t += n_units, ++iter) {
                if (!wait_bar(ptx::smem_u32(&sh->tmem_empty), (uint32_t)(iter & 1) ^ 1u, abort_flag, p.dev_status, p.wait_limit_ns)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                for (int kb = 0; kb < nkb && ok; ++kb) {
                    // the stage's data has landed and its scale factors are in TMEM
                    if (!wait_bar(ptx::smem_u32(&sh->full[stage]), phase, abort_flag, p.dev_status, p.wait_limit_ns) ||
                        !wait_bar(ptx::smem_u32(&sh->sf_full[stage]), phase, abort_flag, p.dev_status, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t sa = ptx::smem_u32(stage_base + stage * G::STAGE);
                    const uint32_t sb = sa + A_BYTES;
                    const uint32_t sfa = tmem + SF_COL + SF_STRIDE * stage, sfb = sfa + 16;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        // 32 bytes of K per MMA: 64 FP4 or 32 E4M3 elements
                        uint64_t ad = ptx::make_sdesc(sa + 32 * kk, 16, 1024, 2);
                        uint64_t bd = ptx::make_sdesc(sb + 32 * kk, 16, 1024, 2);
                        if (FP8) {
                            if (PAIR) ptx::mma_e4m3_pair(tmem + ACC_COL, ad, bd, idesc8, (kb | kk) != 0);
                            else ptx::mma_e4m3(tmem + ACC_COL, ad, bd, idesc8, (kb | kk) != 0);
                        } else if (PAIR) {
                            ptx::mma_mxf4nvf4_pair(tmem + ACC_COL, ad, bd, idesc4, sfa + 4 * kk, sfb + 8 * kk,
                                                   (kb | kk) != 0);
                        } else {
                            ptx::mma_mxf4nvf4(tmem + ACC_COL, ad, bd, idesc4, sfa + 4 * kk, sfb + 8 * kk,
                                              (kb | kk) != 0);
                        }
                    }
                    if (PAIR) ptx::tc_commit_pair_mc(ptx::smem_u32(&sh->empty[stage]), 3);
                    else ptx::tc_commit(ptx::smem_u32(&sh->empty[stage]));
                    issued_any = true;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (ok && nrk > 0 && nkb > 0) {
                    // the BF16 MMAs accumulate into the same TMEM tile: wait for
                    // the FP4 MMAs to complete first
                    if (PAIR) ptx::tc_commit_pair_mc(ptx::smem_u32(&sh->drain), 1);
                    else ptx::tc_commit(ptx::smem_u32(&sh->drain));
                    if (!wait_bar(ptx::smem_u32(&sh->drain), drain_phase, abort_flag, p.dev_status, p.wait_limit_ns)) { ok = false; }
                    drain_phase ^= 1u;
                    ptx::tc_fence_after();
                }
                if (ok && nrk > 0) {
                    for (int rk = 0; rk < nrk && ok; ++rk) {
                        if (!wait_bar(ptx::smem_u32(&sh->full[stage]), phase, abort_flag, p.dev_status, p.wait_limit_ns) ||
                            !wait_bar(ptx::smem_u32(&sh->sf_full[stage]), phase, abort_flag, p.dev_status, p.wait_limit_ns)) {
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after();
                        const uint32_t sa = ptx::smem_u32(stage_base + stage * G::STAGE);
                        const uint32_t sb = sa + A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            uint64_t ad = ptx::make_sdesc(sa + 32 * kk, 16, 1024, 2);
                            uint64_t bd = ptx::make_sdesc(sb + 32 * kk, 16, 1024, 2);
                            // without an FP4 part (BF16-only GEMM) the tile's first MMA overwrites
                            const uint32_t acc = (nkb > 0 || rk > 0 || kk > 0) ? 1u : 0u;
                            if (PAIR) ptx::mma_bf16_pair(tmem + ACC_COL, ad, bd, idesc16, acc);
                            else ptx::mma_bf16(tmem + ACC_COL, ad, bd, idesc16, acc);
                        }
                        if (PAIR) ptx::tc_commit_pair_mc(ptx::smem_u32(&sh->empty[stage]), 3);
                        else ptx::tc_commit(ptx::smem_u32(&sh->empty[stage]));
                        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                    }
                }
                if (ok && !PAIR && p.debug_withhold_acc && iter == 0) {
                    // test hook: withhold the tile's "accumulator ready" signal so
                    // the epilogue's bounded wait runs out; the MMAs are drained
                    // here instead, before any thread can release TMEM
                    ptx::tc_commit(ptx::smem_u32(&sh->drain));
                    if (!wait_bar(ptx::smem_u32(&sh->drain), drain_phase, abort_flag, p.dev_status, p.wait_limit_ns))
                        ok = false;
                    drain_phase ^= 1u;
                } else if (ok) {
                    if (PAIR) ptx::tc_commit_pair_mc(ptx::smem_u32(&sh->tmem_full), 3);
                    else ptx::tc_commit(ptx::smem_u32(&sh->tmem_full));
                }
            }
            if (!ok && issued_any) {
                // let every issued MMA finish before TMEM is released
                if (PAIR) ptx::tc_commit_pair_mc(ptx::smem_u32(&sh->drain), 1);
                else ptx::tc_commit(ptx::smem_u32(&sh->drain));
                wait_bar(ptx::smem_u32(&sh->drain), drain_phase, abort_flag, p.dev_status, p.wait_limit_ns, true);
            }
        }
        __syncwarp();
    } else if (warp == COPY_WARP) {
        if (lane == 0 && leader) {
            // ------------------------------------------- scale-factor copier
            // Follows the producer's stage sequence; per stage one commit to
            // sf_full (RAC stages carry no scale factors: an empty commit
            // keeps the barrier's phase in step with full).
            uint32_t stage = 0, phase = 0;
            bool ok = true, issued_any = false;
            for (int t = unit; ok && t < total; t += n_units) {
                for (int kb = 0; kb < nkb + nrk; ++kb) {
                    if (!wait_bar(ptx::smem_u32(&sh->full[stage]), phase, abort_flag, p.dev_status, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    if (kb < nkb && !FP8) {
                        const uint32_t ssfa = ptx::smem_u32(stage_base + stage * G::STAGE) + A_BYTES + G::B_LOCAL;
                        const uint32_t ssfb = ssfa + SFA_BYTES;
                        const uint32_t sfa = tmem + SF_COL + SF_STRIDE * stage, sfb = sfa + 16;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t da = ptx::make_sdesc(ssfa + 512 * kk, 0, 128, 0);
                            const uint64_t db0 = ptx::make_sdesc(ssfb + 512 * kk, 0, 128, 0);
                            const uint64_t db1 = ptx::make_sdesc(ssfb + SFB_BYTES / 2 + 512 * kk, 0, 128, 0);
                            if (PAIR) {
                                ptx::tmem_cp_32x128b_warpx4_pair(sfa + 4 * kk, da);
                                ptx::tmem_cp_32x128b_warpx4_pair(sfb + 8 * kk, db0);
                                ptx::tmem_cp_32x128b_warpx4_pair(sfb + 8 * kk + 4, db1);
                            } else {
                                ptx::tmem_cp_32x128b_warpx4(sfa + 4 * kk, da);
                                ptx::tmem_cp_32x128b_warpx4(sfb + 8 * kk, db0);
                                ptx::tmem_cp_32x128b_warpx4(sfb + 8 * kk + 4, db1);
                            }
                        }
                    }
                    if (PAIR) ptx::tc_commit_pair_mc(ptx::smem_u32(&sh->sf_full[stage]), 1);
                    else ptx::tc_commit(ptx::smem_u32(&sh->sf_full[stage]));
                    issued_any = true;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok && issued_any) {
                // copies still in flight complete before TMEM is released
                if (PAIR) ptx::tc_commit_pair_mc(ptx::smem_u32(&sh->cp_drain), 1);
                else ptx::tc_commit(ptx::smem_u32(&sh->cp_drain));
                wait_bar(ptx::smem_u32(&sh->cp_drain), 0, abort_flag, p.dev_status, p.wait_limit_ns, true);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------- epilogue
        // Warp w owns TMEM lane quadrant w % 4 (32 rows) and one half of the
        // tile's columns; it copies its whole slice to registers, frees the
        // accumulator for the next tile's MMAs, then computes and stores.
        const int q = warp & 3;
        const int half = (warp - EPI_WARP0) >> 2;
        const int row_in_tile = (int)rank * 128 + q * 32 + lane;
        const float s_a = p.a_s_t ? *p.a_s_t : 1.0f;       // null: unit tensor scales (BF16 GEMM)
        const uint32_t empty_bar = PAIR ? ptx::mapa_shared(ptx::smem_u32(&sh->tmem_empty), 0)
                                        : ptx::smem_u32(&sh->tmem_empty);
        int iter = 0;
        for (int t = unit; t < total; t += n_units, ++iter) {
            bool ok = true;
            if (lane == 0) ok = wait_bar(ptx::smem_u32(&sh->tmem_full), (uint32_t)(iter & 1), abort_flag, p.dev_status, p.wait_limit_ns);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            ptx::tc_fence_after();
            int mt, nt;
            tile_coords(t, m_tiles, p.n_group, mt, nt);
            const int m0 = mt * G::TILE_M;
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
            if (lane == 0) {
                if (PAIR) ptx::mbar_arrive_cluster(empty_bar);
                else ptx::mbar_arrive(empty_bar);
            }

            const float scale = __fmul_rn(s_a, p.b_s_t ? p.b_s_t[e] : 1.0f);
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
            } else if (STAGING) {
                // f32 out through a per-warp 32-row x 32-column transpose tile
                // (16-byte chunks XOR-swizzled by row, conflict-free both
                // ways): each lane writes 32 floats of its row, then each
                // instruction moves 4 rows x 128 contiguous bytes, as plain
                // vector stores (store) or vector add-reductions (scatter-add
                // into the token rows).  Padding rows are never written.
                const bool scatter = p.epilogue == MOE_EPI_SCATTER_ADD_F32;
                const bool hint_y = p.l2_hints != 0;
                const uint64_t pol_y = ptx::policy_evict_last();
                const bool has_row = token >= 0;
                const float mul = scatter ? (has_row ? __fmul_rn(scale, p.row_gate[r]) : 0.0f) : scale;
                const int32_t orow = scatter ? token : (int32_t)r;
                float4 *tile = reinterpret_cast<float4 *>(staging) + (warp - EPI_WARP0) * 256;
                float *out_base = reinterpret_cast<float *>(p.out) + nt * BN + half * 128;
                const int jj = lane & 7;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        tile[lane * 8 + (j ^ (lane & 7))] =
                            make_float4(mul * __uint_as_float(v[ch * 32 + 4 * j]),
                                        mul * __uint_as_float(v[ch * 32 + 4 * j + 1]),
                                        mul * __uint_as_float(v[ch * 32 + 4 * j + 2]),
                                        mul * __uint_as_float(v[ch * 32 + 4 * j + 3]));
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int rr = i * 4 + (lane >> 3);
                        const int32_t orow_r = __shfl_sync(0xffffffffu, orow, rr);
                        const bool valid_r = __shfl_sync(0xffffffffu, has_row ? 1 : 0, rr) != 0;
                        const float4 val = tile[rr * 8 + (jj ^ (rr & 7))];
                        if (valid_r) {
                            float *dst = out_base + (int64_t)orow_r * p.ld_out + ch * 32 + jj * 4;
                            if (scatter && hint_y) ptx::red_add_v4_f32_hint(dst, val, pol_y);
                            else if (scatter) ptx::red_add_v4_f32(dst, val);
                            else ptx::st_v4_f32(dst, val);
                        }
                    }
                    __syncwarp();
                }
            }
        }
    }

    ptx::tc_fence_before();
    if (PAIR) ptx::cluster_sync();         // neither CTA leaves while the pair still uses its memory
    else __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        if (PAIR) ptx::tmem_dealloc_pair(tmem, TMEM_COLS);
        else ptx::tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ----------------------------------------------------------------- host side

template <int STAGES, bool PAIR, bool STAGING, bool FP8>
static nvfp4_status launch(const CUtensorMap &tm_a, const CUtensorMap &tm_b, const CUtensorMap &tm_ra,
                           const CUtensorMap &tm_rb, const CUtensorMap &tm_sfa, const CUtensorMap &tm_sfb,
                           const Params &p, int units, cudaStream_t st)
{
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    auto kern = k_moe_gemm<STAGES, PAIR, STAGING, FP8>;
    const uint32_t smem = Cfg<STAGES, PAIR, STAGING>::SMEM;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return check_launch("k_moe_gemm: device");
    std::call_once(once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    if (attr_err[dev] != cudaSuccess)
        return set_error(NVFP4_ERR_CUDA, "k_moe_gemm: smem attribute: %s", cudaGetErrorString(attr_err[dev]));
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3((unsigned)(PAIR ? 2 * units : units));
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    if (PAIR) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    if (cudaLaunchKernelEx(&cfg, kern, tm_a, tm_b, tm_ra, tm_rb, tm_sfa, tm_sfb, p) != cudaSuccess)
        return check_launch("k_moe_gemm");
    return check_launch("k_moe_gemm");
}


// Tile order and launch shape (1-SM or 2-SM tiles, stages), then launch.
static nvfp4_status dispatch(const CUtensorMap &tm_a, const CUtensorMap &tm_b, const CUtensorMap &tm_ra,
                             const CUtensorMap &tm_rb, const CUtensorMap &tm_sfa, const CUtensorMap &tm_sfb,
                             Params &p, int64_t M_pad_max, int seg_align, cudaStream_t st)
{
    const int epilogue = p.epilogue;
    const bool pair = seg_align == 256;
    const int64_t n_tiles = epilogue == MOE_EPI_SWIGLU_BF16 ? p.inter / 128 : p.N / BN;
    // Tile order: the scatter-add epilogue reduces into token rows that every
    // expert touches; grouping 2 n-tiles (512 output columns) keeps the band
    // of output being reduced into small (16384 tokens x 4096 f32: 1114 us in
    // plain order, 937 us in groups of 2; groups of 1, 4 or 8 and a token-phase
    // order of the m-tiles measured no better).
    int n_group = (int)n_tiles;
    if (epilogue == MOE_EPI_SCATTER_ADD_F32 && n_tiles % 2 == 0) n_group = 2;
    p.n_group = n_group;
    p.l2_hints = epilogue == MOE_EPI_SCATTER_ADD_F32 ? 1 : 0;
    const int64_t max_tiles = (M_pad_max / seg_align) * n_tiles;
    const bool swiglu = epilogue == MOE_EPI_SWIGLU_BF16;
    if (pair) {
        // 5 stages; the f32 epilogues add their transpose tiles
        const int units = (int)std::min<int64_t>(num_sms() / 2, max_tiles);
        if (p.fp8)
            return swiglu ? launch<5, true, false, true>(tm_a, tm_b, tm_ra, tm_rb, tm_sfa, tm_sfb, p, units, st)
                          : launch<5, true, true, true>(tm_a, tm_b, tm_ra, tm_rb, tm_sfa, tm_sfb, p, units, st);
        return swiglu ? launch<5, true, false, false>(tm_a, tm_b, tm_ra, tm_rb, tm_sfa, tm_sfb, p, units, st)
                      : launch<5, true, true, false>(tm_a, tm_b, tm_ra, tm_rb, tm_sfa, tm_sfb, p, units, st);
    }
    // SwiGLU (bf16 out): 4 stages; f32 epilogues: 3 stages + transpose tiles
    const int units = (int)std::min<int64_t>(num_sms(), max_tiles);
    if (p.fp8)
        return swiglu ? launch<4, false, false, true>(tm_a, tm_b, tm_ra, tm_rb, tm_sfa, tm_sfb, p, units, st)
                      : launch<3, false, true, true>(tm_a, tm_b, tm_ra, tm_rb, tm_sfa, tm_sfb, p, units, st);
    return swiglu ? launch<4, false, false, false>(tm_a, tm_b, tm_ra, tm_rb, tm_sfa, tm_sfb, p, units, st)
                  : launch<3, false, true, false>(tm_a, tm_b, tm_ra, tm_rb, tm_sfa, tm_sfb, p, units, st);
}

}  // namespace gemm
}  // namespace nvfp4

using namespace nvfp4;

static nvfp4_status gemm_rac(
    const uint8_t *a_codes_dev, const uint8_t *a_scales_dev, const float *a_s_t_dev, int64_t M_pad_max,
    const uint8_t *b_codes_dev, const uint8_t *b_scales_dev, const float *b_s_t_dev, int64_t N, int64_t K, int32_t E,
    const int32_t *offsets_dev, int32_t seg_align, int32_t rac_ld, const void *rho_dev, const void *w_sel_dev,
    int32_t epilogue, const int32_t *row_token_dev, const float *row_gate_dev, void *out_dev, int64_t ld_out,
    float *amax_out_dev, int32_t *dev_status, void *stream, uint64_t wait_limit_ns, int debug_withhold_acc)
{
    using namespace nvfp4::gemm;
    cudaStream_t st = (cudaStream_t)stream;
    NVFP4_REQUIRE(a_codes_dev && a_scales_dev && a_s_t_dev && b_codes_dev && b_scales_dev && b_s_t_dev &&
                  offsets_dev && row_token_dev && out_dev, NVFP4_ERR_INVALID_ARG,
                  "moe_w4a4_grouped_gemm_rac: null pointer");
    NVFP4_REQUIRE(epilogue >= 0 && epilogue <= 2, NVFP4_ERR_INVALID_ARG, "moe_w4a4_grouped_gemm_rac: bad epilogue");
    NVFP4_REQUIRE(seg_align == 128 || seg_align == 256, NVFP4_ERR_INVALID_ARG,
                  "moe_w4a4_grouped_gemm_rac: seg_align must be 128 or 256");
    NVFP4_REQUIRE(epilogue != MOE_EPI_SCATTER_ADD_F32 || row_gate_dev, NVFP4_ERR_INVALID_ARG,
                  "moe_w4a4_grouped_gemm_rac: scatter-add needs row_gate");
    NVFP4_REQUIRE(E >= 1 && E <= MAX_E, NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_w4a4_grouped_gemm_rac: 1 <= E <= 256");
    NVFP4_REQUIRE(K >= 256 && K % 256 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "moe_w4a4_grouped_gemm_rac: K must be a positive multiple of 256 (K=%lld)", (long long)K);
    NVFP4_REQUIRE(N >= 256 && N % 256 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "moe_w4a4_grouped_gemm_rac: N must be a positive multiple of 256 (N=%lld)", (long long)N);
    NVFP4_REQUIRE(M_pad_max >= seg_align && M_pad_max % seg_align == 0 && M_pad_max < (1ll << 31),
                  NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "moe_w4a4_grouped_gemm_rac: M_pad_max must be a positive multiple of seg_align");
    NVFP4_REQUIRE((int64_t)E * N < (1ll << 31), NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_w4a4_grouped_gemm_rac: E*N too large");
    NVFP4_REQUIRE(rac_ld >= 0 && rac_ld <= 16384 && rac_ld % 64 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "moe_w4a4_grouped_gemm_rac: rac_ld must be 0..16384 and a multiple of 64");
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

    CUtensorMap tm_a, tm_b, tm_ra, tm_rb, tm_sfa, tm_sfb;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    bool ok = make_tmap_2d(&tm_a, a_codes_dev, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)K / 2, (uint64_t)M_pad_max,
                           (uint64_t)K / 2, 128, BOX_ROWS, sw) &&
              make_tmap_2d(&tm_b, b_codes_dev, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)K / 2, (uint64_t)E * N,
                           (uint64_t)K / 2, 128, BOX_ROWS, sw);
    if (ok && rac_ld > 0) {
        ok = make_tmap_2d(&tm_ra, rho_dev, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)rac_ld, (uint64_t)M_pad_max,
                          (uint64_t)rac_ld * 2, 64, BOX_ROWS, sw) &&
             make_tmap_2d(&tm_rb, w_sel_dev, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)rac_ld, (uint64_t)E * N,
                          (uint64_t)rac_ld * 2, 64, BOX_ROWS, sw);
    } else {
        tm_ra = tm_a;
        tm_rb = tm_b;
    }
    const bool pair = seg_align == 256;
    if (ok && pair) {
        // scale buffers viewed as [bytes/256 x 256] for 2 KB (4-atom) TMA boxes
        const uint64_t sfa_bytes = (uint64_t)M_pad_max * (uint64_t)(K / 16);
        const uint64_t sfb_bytes = (uint64_t)E * (uint64_t)(((N + 127) / 128) * 128) * (uint64_t)(K / 16);
        ok = make_tmap_2d(&tm_sfa, a_scales_dev, CU_TENSOR_MAP_DATA_TYPE_UINT8, 256, sfa_bytes / 256, 256, 256, 8,
                          CU_TENSOR_MAP_SWIZZLE_NONE) &&
             make_tmap_2d(&tm_sfb, b_scales_dev, CU_TENSOR_MAP_DATA_TYPE_UINT8, 256, sfb_bytes / 256, 256, 256, 8,
                          CU_TENSOR_MAP_SWIZZLE_NONE);
    } else {
        tm_sfa = tm_a;
        tm_sfb = tm_b;
    }
    NVFP4_REQUIRE(ok, NVFP4_ERR_CUDA, "moe_w4a4_grouped_gemm_rac: tensor map encoding failed");

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
    p.wait_limit_ns = wait_limit_ns;
    p.debug_withhold_acc = debug_withhold_acc;
    p.dev_status = dev_status;
    if (p.amax_out && cudaMemsetAsync(p.amax_out, 0, sizeof(float), st) != cudaSuccess)
        return check_launch("moe_w4a4_grouped_gemm_rac: memset");
    return dispatch(tm_a, tm_b, tm_ra, tm_rb, tm_sfa, tm_sfb, p, M_pad_max, seg_align, st);
}

extern "C" nvfp4_status moe_w4a4_grouped_gemm_rac(
    const uint8_t *a_codes_dev, const uint8_t *a_scales_dev, const float *a_s_t_dev, int64_t M_pad_max,
    const uint8_t *b_codes_dev, const uint8_t *b_scales_dev, const float *b_s_t_dev, int64_t N, int64_t K, int32_t E,
    const int32_t *offsets_dev, int32_t seg_align, int32_t rac_ld, const void *rho_dev, const void *w_sel_dev,
    int32_t epilogue, const int32_t *row_token_dev, const float *row_gate_dev, void *out_dev, int64_t ld_out,
    float *amax_out_dev, int32_t *dev_status, void *stream)
{
    return gemm_rac(a_codes_dev, a_scales_dev, a_s_t_dev, M_pad_max, b_codes_dev, b_scales_dev, b_s_t_dev, N, K, E,
                    offsets_dev, seg_align, rac_ld, rho_dev, w_sel_dev, epilogue, row_token_dev, row_gate_dev, out_dev,
                    ld_out, amax_out_dev, dev_status, stream, nvfp4::gemm::TIMEOUT_NS, 0);
}

extern "C" nvfp4_status nvfp4_debug_gemm_wait_expiry(
    const uint8_t *a_codes_dev, const uint8_t *a_scales_dev, const float *a_s_t_dev, int64_t M_pad_max,
    const uint8_t *b_codes_dev, const uint8_t *b_scales_dev, const float *b_s_t_dev, int64_t N, int64_t K, int32_t E,
    const int32_t *offsets_dev, int32_t epilogue, const int32_t *row_token_dev, const float *row_gate_dev,
    void *out_dev, int64_t ld_out, int32_t *dev_status, int64_t wait_limit_ns, void *stream)
{
    NVFP4_REQUIRE(dev_status && wait_limit_ns >= 1000000 && wait_limit_ns <= 1000000000ll, NVFP4_ERR_INVALID_ARG,
                  "nvfp4_debug_gemm_wait_expiry: needs dev_status and 1 ms <= wait_limit_ns <= 1 s");
    return gemm_rac(a_codes_dev, a_scales_dev, a_s_t_dev, M_pad_max, b_codes_dev, b_scales_dev, b_s_t_dev, N, K, E,
                    offsets_dev, 128, 0, nullptr, nullptr, epilogue, row_token_dev, row_gate_dev, out_dev, ld_out,
                    nullptr, dev_status, stream, (uint64_t)wait_limit_ns, 1);
}

extern "C" nvfp4_status moe_bf16_grouped_gemm(
    const void *a_dev, int64_t lda, int64_t M_pad_max, const void *b_dev, int64_t N, int64_t K, int32_t E,
    const int32_t *offsets_dev, int32_t seg_align, int32_t epilogue, const int32_t *row_token_dev,
    const float *row_gate_dev, void *out_dev, int64_t ld_out, float *amax_out_dev, int32_t *dev_status, void *stream)
{
    using namespace nvfp4::gemm;
    cudaStream_t st = (cudaStream_t)stream;
    NVFP4_REQUIRE(a_dev && b_dev && offsets_dev && row_token_dev && out_dev, NVFP4_ERR_INVALID_ARG,
                  "moe_bf16_grouped_gemm: null pointer");
    NVFP4_REQUIRE(epilogue >= 0 && epilogue <= 2, NVFP4_ERR_INVALID_ARG, "moe_bf16_grouped_gemm: bad epilogue");
    NVFP4_REQUIRE(seg_align == 128 || seg_align == 256, NVFP4_ERR_INVALID_ARG,
                  "moe_bf16_grouped_gemm: seg_align must be 128 or 256");
    NVFP4_REQUIRE(epilogue != MOE_EPI_SCATTER_ADD_F32 || row_gate_dev, NVFP4_ERR_INVALID_ARG,
                  "moe_bf16_grouped_gemm: scatter-add needs row_gate");
    NVFP4_REQUIRE(E >= 1 && E <= MAX_E, NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_bf16_grouped_gemm: 1 <= E <= 256");
    NVFP4_REQUIRE(K >= 64 && K % 64 == 0 && K < (1 << 20), NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "moe_bf16_grouped_gemm: K must be a positive multiple of 64 (K=%lld)", (long long)K);
    NVFP4_REQUIRE(N >= 256 && N % 256 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "moe_bf16_grouped_gemm: N must be a positive multiple of 256 (N=%lld)", (long long)N);
    NVFP4_REQUIRE(lda >= K && lda % 8 == 0, NVFP4_ERR_ALIGNMENT,
                  "moe_bf16_grouped_gemm: lda must be >= K and a multiple of 8");
    NVFP4_REQUIRE(M_pad_max >= seg_align && M_pad_max % seg_align == 0 && M_pad_max < (1ll << 31),
                  NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_bf16_grouped_gemm: M_pad_max must be a positive multiple of seg_align");
    NVFP4_REQUIRE((int64_t)E * N < (1ll << 31), NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_bf16_grouped_gemm: E*N too large");
    const int inter = (int)(N / 2);
    if (epilogue == MOE_EPI_SWIGLU_BF16) {
        NVFP4_REQUIRE(inter % 128 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_bf16_grouped_gemm: SwiGLU needs I % 128 == 0");
        NVFP4_REQUIRE(ld_out >= inter && ld_out % 8 == 0, NVFP4_ERR_ALIGNMENT,
                      "moe_bf16_grouped_gemm: SwiGLU ld_out must be >= N/2 and a multiple of 8");
    } else {
        NVFP4_REQUIRE(ld_out >= N && ld_out % 4 == 0, NVFP4_ERR_ALIGNMENT,
                      "moe_bf16_grouped_gemm: ld_out must be >= N and a multiple of 4");
    }
    NVFP4_REQUIRE(aligned16(a_dev) && aligned16(b_dev) && aligned16(out_dev), NVFP4_ERR_ALIGNMENT,
                  "moe_bf16_grouped_gemm: pointers must be 16-byte aligned");

    // A and B travel the kernel's BF16 (kind::f16) stages, K / 64 of them per
    // tile, with no FP4 stage and unit tensor scales.
    CUtensorMap tm_ra, tm_rb;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    const bool ok = make_tmap_2d(&tm_ra, a_dev, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)K, (uint64_t)M_pad_max,
                                 (uint64_t)lda * 2, 64, BOX_ROWS, sw) &&
                    make_tmap_2d(&tm_rb, b_dev, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)K, (uint64_t)E * N,
                                 (uint64_t)K * 2, 64, BOX_ROWS, sw);
    NVFP4_REQUIRE(ok, NVFP4_ERR_CUDA, "moe_bf16_grouped_gemm: tensor map encoding failed");

    Params p{};
    p.N = N;
    p.K = 0;                          // no FP4 stages
    p.E = E;
    p.offsets = offsets_dev;
    p.rac_ld = (int)K;                // the BF16 stages cover all of K
    p.epilogue = epilogue;
    p.inter = inter;
    p.row_token = row_token_dev;
    p.row_gate = row_gate_dev;
    p.out = out_dev;
    p.ld_out = ld_out;
    p.amax_out = (epilogue == MOE_EPI_SWIGLU_BF16) ? reinterpret_cast<unsigned int *>(amax_out_dev) : nullptr;
    p.wait_limit_ns = TIMEOUT_NS;
    p.dev_status = dev_status;
    if (p.amax_out && cudaMemsetAsync(p.amax_out, 0, sizeof(float), st) != cudaSuccess)
        return check_launch("moe_bf16_grouped_gemm: memset");
    return dispatch(tm_ra, tm_rb, tm_ra, tm_rb, tm_ra, tm_rb, p, M_pad_max, seg_align, st);
}

extern "C" nvfp4_status moe_w8a8_grouped_gemm(
    const uint8_t *a_codes_dev, const float *a_s_dev, int64_t M_pad_max, const uint8_t *b_codes_dev,
    const float *b_s_dev, int64_t N, int64_t K, int32_t E, const int32_t *offsets_dev, int32_t seg_align,
    int32_t epilogue, const int32_t *row_token_dev, const float *row_gate_dev, void *out_dev, int64_t ld_out,
    float *amax_out_dev, int32_t *dev_status, void *stream)
{
    using namespace nvfp4::gemm;
    cudaStream_t st = (cudaStream_t)stream;
    NVFP4_REQUIRE(a_codes_dev && a_s_dev && b_codes_dev && b_s_dev && offsets_dev && row_token_dev && out_dev,
                  NVFP4_ERR_INVALID_ARG, "moe_w8a8_grouped_gemm: null pointer");
    NVFP4_REQUIRE(epilogue >= 0 && epilogue <= 2, NVFP4_ERR_INVALID_ARG, "moe_w8a8_grouped_gemm: bad epilogue");
    NVFP4_REQUIRE(seg_align == 128 || seg_align == 256, NVFP4_ERR_INVALID_ARG,
                  "moe_w8a8_grouped_gemm: seg_align must be 128 or 256");
    NVFP4_REQUIRE(epilogue != MOE_EPI_SCATTER_ADD_F32 || row_gate_dev, NVFP4_ERR_INVALID_ARG,
                  "moe_w8a8_grouped_gemm: scatter-add needs row_gate");
    NVFP4_REQUIRE(E >= 1 && E <= MAX_E, NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_w8a8_grouped_gemm: 1 <= E <= 256");
    NVFP4_REQUIRE(K >= 128 && K % 128 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "moe_w8a8_grouped_gemm: K must be a positive multiple of 128 (K=%lld)", (long long)K);
    NVFP4_REQUIRE(N >= 256 && N % 256 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
                  "moe_w8a8_grouped_gemm: N must be a positive multiple of 256 (N=%lld)", (long long)N);
    NVFP4_REQUIRE(M_pad_max >= seg_align && M_pad_max % seg_align == 0 && M_pad_max < (1ll << 31),
                  NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_w8a8_grouped_gemm: M_pad_max must be a positive multiple of seg_align");
    NVFP4_REQUIRE((int64_t)E * N < (1ll << 31), NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_w8a8_grouped_gemm: E*N too large");
    const int inter = (int)(N / 2);
    if (epilogue == MOE_EPI_SWIGLU_BF16) {
        NVFP4_REQUIRE(inter % 128 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE, "moe_w8a8_grouped_gemm: SwiGLU needs I % 128 == 0");
        NVFP4_REQUIRE(ld_out >= inter && ld_out % 8 == 0, NVFP4_ERR_ALIGNMENT,
                      "moe_w8a8_grouped_gemm: SwiGLU ld_out must be >= N/2 and a multiple of 8");
    } else {
        NVFP4_REQUIRE(ld_out >= N && ld_out % 4 == 0, NVFP4_ERR_ALIGNMENT,
                      "moe_w8a8_grouped_gemm: ld_out must be >= N and a multiple of 4");
    }
    NVFP4_REQUIRE(aligned16(a_codes_dev) && aligned16(b_codes_dev) && aligned16(out_dev), NVFP4_ERR_ALIGNMENT,
                  "moe_w8a8_grouped_gemm: pointers must be 16-byte aligned");
    CUtensorMap tm_a, tm_b;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    const bool ok = make_tmap_2d(&tm_a, a_codes_dev, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)K, (uint64_t)M_pad_max,
                                 (uint64_t)K, 128, BOX_ROWS, sw) &&
                    make_tmap_2d(&tm_b, b_codes_dev, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)K, (uint64_t)E * N,
                                 (uint64_t)K, 128, BOX_ROWS, sw);
    NVFP4_REQUIRE(ok, NVFP4_ERR_CUDA, "moe_w8a8_grouped_gemm: tensor map encoding failed");
    Params p{};
    p.a_s_t = a_s_dev;
    p.b_s_t = b_s_dev;
    p.N = N;
    p.K = K;
    p.E = E;
    p.offsets = offsets_dev;
    p.rac_ld = 0;
    p.epilogue = epilogue;
    p.inter = inter;
    p.row_token = row_token_dev;
    p.row_gate = row_gate_dev;
    p.out = out_dev;
    p.ld_out = ld_out;
    p.amax_out = (epilogue == MOE_EPI_SWIGLU_BF16) ? reinterpret_cast<unsigned int *>(amax_out_dev) : nullptr;
    p.wait_limit_ns = TIMEOUT_NS;
    p.fp8 = 1;
    p.dev_status = dev_status;
    if (p.amax_out && cudaMemsetAsync(p.amax_out, 0, sizeof(float), st) != cudaSuccess)
        return check_launch("moe_w8a8_grouped_gemm: memset");
    return dispatch(tm_a, tm_b, tm_a, tm_b, tm_a, tm_b, p, M_pad_max, seg_align, st);
}
