// Block-scaled FP4 GEMM with the low-rank tail, computed by CTA pairs (cta_group::2).
//
// Same result as gemm_fp4_lowrank_kernel (ft_gemm.cu: FourTune Eq. (2) forward and the
// backbone pathway of Eq. (3), low-rank branches added in the same accumulator), with
// less data moved per SM: two CTAs on neighbouring SMs form a cluster and compute one
// 256 x 256 output tile with tcgen05.mma.cta_group::2, issued by the even CTA.  Each CTA
// loads its own 128 rows of A and its own 128 rows of B (the MMA reads the pair's shared
// memories together).
//
// Per CTA and stage: A [128 x 128 B], B [128 x 128 B] (its half of the tile's N) and the
// k step's scales.  The scales are those of 16x16 blocks, so a k step needs only the
// compact grid rows of its blocks -- 8 x 16 bytes for the CTA's A rows, 16 x 16 bytes for
// the pair tile's 256 B rows (every CTA's part of the MMA reads the scales of the full N
// from its own tensor memory) -- instead of the per-row tensor-core layout (2 KB + 4 KB),
// which is read only for 1x16 groups (A) and for a Q(R)^T transposed on the fly (B).
// Each CTA's loads complete on its own FULL barrier; its four scale warps expand the
// scales into its own tensor memory (tcgen05.st: each 16-byte grid row becomes one word
// of four atom rows) and arrive on the even CTA's SF_READY barrier, which the MMA issuer
// waits on, so SF_READY also certifies that both CTAs' operands have landed.  The MMA
// issuer's commits arrive on both CTAs' EMPTY barriers and on both TMEM_FULL barriers
// (one commit each, multicast to the pair: half the tensor-pipe time of a commit per
// CTA); each CTA drains its own 128 x 256 accumulator and releases it on the even CTA's
// TMEM_EMPTY.  No load is multicast.  Tiles are visited with the smaller operand swept by
// the tiles in flight (p.n_inner), so that it stays in L2.
//
// Five stages and four epilogue warps (eight for the GELU epilogues): a sixth stage (room
// for it once the scales are compact, with the scale-factor slots in tensor memory then
// reused five k steps apart) and eight plain epilogue warps each measured slower on the
// FLUX single-stream layers.
//
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer (even CTA) and TMEM owner, then
// the epilogue warps (4, or 8 for the GELU epilogues: two per TMEM lane quarter, 128
// columns each), then 4 scale writers.
//
// With XP (the dX GEMM of section 3.2 without a stored Q(R)^T) the producer loads B's
// untransposed slab, 256 reduction rows x 64 bytes, into the B slot, and the scale
// writers turn it into the K-major tile in place (ft_xpose.cuh) before they arrive on
// SF_READY: all four read their share first, meet on the XREAD barrier, then write.
#include "ft_internal.h"
#include "ft_ptx.cuh"
#include "ft_sidejobs.cuh"
#include "ft_xpose.cuh"

namespace ft {
namespace gemm2 {

constexpr int BM = 128;                  // rows per CTA (256 per pair)
constexpr int BN = 256;                  // output columns per pair
constexpr int BN_CTA = 128;              // B rows held by one CTA
constexpr int BK_BYTES = 128;
constexpr int STAGES = 5;
constexpr int A_BYTES = BM * BK_BYTES;      // 16 KB
constexpr int B_BYTES = BN_CTA * BK_BYTES;  // 16 KB
constexpr int SFA_BYTES = 4 * 512;
constexpr int SFB_BYTES = 2 * 4 * 512;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;  // 38912
// the compact grids of 16x16-block scales one k step needs (they fit in the atoms' regions)
constexpr int SFA_GRID_BYTES = 8 * 16;   // 8 block-rows x 16 block-columns
constexpr int SFB_GRID_BYTES = 16 * 16;  // the pair tile's 16 block-rows
constexpr int OFF_B = A_BYTES;
constexpr int OFF_SFA = A_BYTES + B_BYTES;
constexpr int OFF_SFB = OFF_SFA + SFA_BYTES;
constexpr int EPI_BYTES = 32 * 64;
constexpr int OFF_EPI = STAGES * STAGE_BYTES;
constexpr int BAR_BYTES = 256;
constexpr int EPI_BUFS = 2;              // staging buffers per epilogue warp (one store in flight)
// Epilogue warps per variant: 4 (one per TMEM lane quarter, all 256 columns) for the plain
// GEMM; 8 (two per quarter, 128 columns each) for the GELU epilogues, whose arithmetic
// needs two warps per scheduler to hide its latency.
__host__ __device__ constexpr int epi_warps(int epi) { return epi == kEpiPlain ? 4 : 8; }
__host__ __device__ constexpr int epi_region(int epi) { return epi_warps(epi) * EPI_BUFS * EPI_BYTES; }
__host__ __device__ constexpr int smem_bytes(int epi) { return OFF_EPI + epi_region(epi) + BAR_BYTES + 1024; }
__host__ __device__ constexpr int threads(int epi) { return 32 * (2 + epi_warps(epi) + 4); }

constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_ACC = 0;
constexpr uint32_t COL_SFA = 256;                    // STAGES x 16 columns
constexpr uint32_t COL_SFB = COL_SFA + STAGES * 16;  // STAGES x 32 columns

static_assert(STAGE_BYTES % 1024 == 0, "stage must keep 1024-byte alignment");
static_assert(smem_bytes(kEpiGelu) <= 232448, "exceeds 227 KB of dynamic shared memory");
static_assert(COL_SFB + STAGES * 32 <= TMEM_COLS, "tensor memory overflow");

__host__ __device__ constexpr int BAR_FULL(int s) { return s; }
__host__ __device__ constexpr int BAR_EMPTY(int s) { return STAGES + s; }
__host__ __device__ constexpr int BAR_SF_READY(int s) { return 2 * STAGES + s; }
constexpr int BAR_TMEM_FULL = 3 * STAGES;
constexpr int BAR_TMEM_EMPTY = 3 * STAGES + 1;
constexpr int BAR_FINAL = 3 * STAGES + 2;
constexpr int BAR_XREAD = 3 * STAGES + 3;  // XP: the scale warps have read the raw B slab
constexpr int NUM_BARS = 3 * STAGES + 4;
constexpr int OFF_TMEM_SLOT = 8 * NUM_BARS;
constexpr int OFF_ABORT = OFF_TMEM_SLOT + 4;
static_assert(OFF_ABORT + 4 <= BAR_BYTES, "barrier area overflow");

// XP: one scale warp's share of the in-place transposition of the B slab at `slab`.
// False if the wait for the other scale warps' reads gave up (the abort flag and status
// are then set).
__device__ __forceinline__ bool xpose_share(uint32_t slab, int q, int lane, uint32_t xread, uint32_t& xr,
                                            volatile int* abort_flag, int* status) {
    xpose::Regs<64> rg;
    xpose::load<64>(slab, q, lane, rg);
    __syncwarp();
    if (lane == 0) mbar_arrive(xread);
    xpose::transpose<64>(lane, rg);
    if (!mbar_wait(xread, xr & 1, abort_flag, status)) return false;
    ++xr;
    xpose::store<64>(slab, q, lane, rg);
    // The stores are complete in this CTA's shared memory once the proxy fence returns;
    // the MMA reading them (issued by the even CTA) starts only after SF_READY completes,
    // which needs this warp's arrival below, so the cta-scope arrival suffices (a
    // cluster-scope release would cost several hundred cycles per stage).
    fence_proxy_async_smem();
    return true;
}

// SFC bit 0: A's scales come from its compact 16x16-block grid (tmSA), bit 1: B's (tmSB);
// otherwise from the tensor-core scale layout (p.sfa / p.sfb).
template <int EPI, bool XP, int SFC>
__global__ void __launch_bounds__(threads(EPI), 1)
    gemm_fp4_lowrank_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                                 const __grid_constant__ CUtensorMap tmB,
                                 const __grid_constant__ CUtensorMap tmLA,
                                 const __grid_constant__ CUtensorMap tmLB,
                                 const __grid_constant__ CUtensorMap tmOut,
                                 const __grid_constant__ CUtensorMap tmAct,
                                 const __grid_constant__ CUtensorMap tmSA,
                                 const __grid_constant__ CUtensorMap tmSB, const GemmFp4Args p) {
    constexpr bool kGridA = (SFC & 1) != 0;
    constexpr bool kGridB = (SFC & 2) != 0;
    // bytes one k step's scales add to a stage: a 128-row band's grid rows (8 x 16 B) or its
    // four 512-byte atoms; the pair tile's 256 B rows: 16 x 16 B or eight atoms
    constexpr uint32_t kSfBytes = (kGridA ? SFA_GRID_BYTES : SFA_BYTES) + (kGridB ? SFB_GRID_BYTES : SFB_BYTES);
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t pad = (1024 - (raw_u32 & 1023)) & 1023;
    uint8_t* base = smem_raw + pad;
    const uint32_t base_u32 = raw_u32 + pad;
    constexpr int EPI_WARPS = epi_warps(EPI);
    constexpr int EPI_COLS = BN / (EPI_WARPS / 4);  // tile columns per epilogue warp
    uint8_t* bar_area = base + OFF_EPI + epi_region(EPI);
    auto bar = [&](int i) { return base_u32 + OFF_EPI + epi_region(EPI) + 8 * i; };
    auto stage = [&](int s) { return base_u32 + s * STAGE_BYTES; };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(bar_area + OFF_TMEM_SLOT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_area + OFF_ABORT);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: the pair's MMA issuer
    const int pair = blockIdx.x >> 1;
    const int num_pairs = gridDim.x >> 1;
    const int MB2 = p.M / (2 * BM);
    const int NB = p.N / BN;
    const int num_tiles = MB2 * NB;
    const int KT = p.K / 256;
    const int KLS = (p.KL + 63) / 64;  // low-rank stages (the last one may be partly past KL:
                                       // TMA fills those columns with zeros, no MMA reads them)
    const int k64 = p.K / 64;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(bar(BAR_FULL(i)), 1);       // this CTA's producer (+ its bytes)
            mbar_init(bar(BAR_EMPTY(i)), 1);      // the MMA issuer's commit
            mbar_init(bar(BAR_SF_READY(i)), 8);   // 4 scale warps x 2 CTAs (even CTA's copy used)
        }
        mbar_init(bar(BAR_TMEM_FULL), 1);
        mbar_init(bar(BAR_TMEM_EMPTY), 2 * EPI_WARPS);  // epilogue warps x 2 CTAs (even CTA's copy used)
        mbar_init(bar(BAR_FINAL), 1);
        mbar_init(bar(BAR_XREAD), 4);  // XP: this CTA's 4 scale warps
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if constexpr (kGridA) tma_prefetch_desc(&tmSA);
        if constexpr (kGridB) tma_prefetch_desc(&tmSB);
        if (KLS > 0) {
            tma_prefetch_desc(&tmLA);
            tma_prefetch_desc(&tmLB);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(const_cast<uint32_t*>(tmem_slot)), TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // barriers initialised and TMEM allocated in both CTAs
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // TMEM is allocated before dependents may be scheduled on this SM (a waiting
    // dependent never holds tensor memory this CTA still needs).
    pdl_trigger();
    pdl_wait();

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            int it = 0;
            int s = 0;        // it % STAGES
            uint32_t ph = 0;  // (it / STAGES) & 1
            auto acquire = [&]() { return mbar_wait(bar(BAR_EMPTY(s)), ph ^ 1, abort_flag, p.status); };
            auto advance = [&]() {
                ++it;
                if (++s == STAGES) { s = 0; ph ^= 1; }
            };
            for (int t = pair; t < num_tiles && !*abort_flag; t += num_pairs) {
                const int mb2 = p.n_inner ? t / NB : t % MB2, nb = p.n_inner ? t % NB : t / MB2;
                const int m_band = mb2 * 2 + static_cast<int>(rank);            // this CTA's A rows
                const int n_rows = nb * BN + BN_CTA * static_cast<int>(rank);  // this CTA's B rows
                for (int kt = 0; kt < KT; ++kt, advance()) {
                    if (!acquire()) break;
                    const uint32_t full = bar(BAR_FULL(s));
                    const uint32_t st = stage(s);
                    mbar_arrive_expect_tx(full, A_BYTES + B_BYTES + kSfBytes);
                    tma_load_2d(st, &tmA, full, kt * BK_BYTES, m_band * BM);
                    if constexpr (XP)  // B^T rows kt*256.., bytes of this CTA's 128 columns
                        tma_load_2d(st + OFF_B, &tmB, full, n_rows / 2, kt * 256);
                    else
                        tma_load_2d(st + OFF_B, &tmB, full, kt * BK_BYTES, n_rows);
                    if constexpr (kGridA)  // block-rows of this CTA's 128 A rows, 16 block-columns
                        tma_load_2d(st + OFF_SFA, &tmSA, full, kt * 16, m_band * (BM / 16));
                    else
                        bulk_load(st + OFF_SFA, p.sfa + (static_cast<size_t>(m_band) * k64 + kt * 4) * 512,
                                  SFA_BYTES, full);
                    if constexpr (kGridB) {  // the pair tile's 16 block-rows of B
                        tma_load_2d(st + OFF_SFB, &tmSB, full, kt * 16, nb * (BN / 16));
                    } else {
#pragma unroll
                        for (int rb = 0; rb < 2; ++rb)
                            bulk_load(st + OFF_SFB + rb * 2048,
                                      p.sfb + (static_cast<size_t>(nb * 2 + rb) * k64 + kt * 4) * 512, 2048,
                                      full);
                    }
                }
                if (*abort_flag) break;
                for (int kl = 0; kl < KLS; ++kl, advance()) {
                    if (!acquire()) break;
                    const uint32_t full = bar(BAR_FULL(s));
                    const uint32_t st = stage(s);
                    mbar_arrive_expect_tx(full, A_BYTES + B_BYTES);
                    tma_load_2d(st, &tmLA, full, kl * 64, m_band * BM);
                    tma_load_2d(st + OFF_B, &tmLB, full, kl * 64, n_rows);
                }
            }
            // Drain: every copy this thread issued has landed before the CTA may exit.
            for (int j = it - 1; j >= 0 && j >= it - STAGES; --j) {
                volatile int no_abort = 0;
                mbar_wait(bar(BAR_FULL(j % STAGES)), (j / STAGES) & 1, &no_abort, p.status);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer (even CTA)
        if (rank == 0 && lane == 0) {
            const uint32_t idesc4 = idesc_fp4_block16(2 * BM, BN);
            const uint32_t idesc16 = idesc_bf16(2 * BM, BN);
            // Every instruction of this thread between MMAs delays the tensor pipe: the loop
            // keeps running stage / parity counters instead of dividing.
            int ti = 0;
            int s = 0;        // stage of the next k step
            uint32_t ph = 0;  // its use parity
            for (int t = pair; t < num_tiles && !*abort_flag; t += num_pairs, ++ti) {
                if (!mbar_wait(bar(BAR_TMEM_EMPTY), (ti & 1) ^ 1, abort_flag, p.status)) break;
                tc_fence_after();
                bool ok = true;
                for (int j = 0; j < KT + KLS; ++j) {
                    // one plain try_wait first: the bounded wait costs more even when the
                    // phase is already complete
                    const uint32_t rdy = bar(BAR_SF_READY(s));
                    if (!mbar_try_wait(rdy, ph) && !mbar_wait(rdy, ph, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = stage(s);
                    const uint64_t ad = sdesc_kmajor_sw128(st);
                    const uint64_t bd = sdesc_kmajor_sw128(st + OFF_B);
                    if (j < KT) {
                        const uint32_t sfa_t = tmem + COL_SFA + 16 * s;
                        const uint32_t sfb_t = tmem + COL_SFB + 32 * s;
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            mma_fp4_block16_pair(tmem + COL_ACC, ad + 2 * i, bd + 2 * i, idesc4, sfa_t + 4 * i,
                                                 sfb_t + 8 * i, (j | i) != 0);
                    } else {
                        const int nk16 = min(4, (p.KL - 64 * (j - KT)) / 16);  // K=16 steps inside KL
                        for (int i = 0; i < nk16; ++i)
                            mma_bf16_pair(tmem + COL_ACC, ad + 2 * i, bd + 2 * i, idesc16, 1);
                    }
                    tc_commit_pair_both(bar(BAR_EMPTY(s)));
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (!ok) break;
                tc_commit_pair_both(bar(BAR_TMEM_FULL));
            }
            // every MMA has retired (in both CTAs' tensor memory) before the pair tears down
            tc_commit_pair(bar(BAR_FINAL));
            volatile int no_abort = 0;
            mbar_wait(bar(BAR_FINAL), 0, &no_abort, p.status);
        }
    } else if (warp >= 2 + EPI_WARPS) {
        // ---------------------------------------------------------------- scale writers
        // Same tensor-memory layout as the single-CTA kernel: lane l of quarter q holds row
        // l of every 512-byte scale atom (4 columns per A k-block, 8 per B k-block).
        const int q = warp & 3;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
        int it = 0;
        uint32_t xr = 0;  // XREAD phases passed
        for (int t = pair; t < num_tiles && !*abort_flag; t += num_pairs) {
            bool ok = true;
            for (int j = 0; j < KT + KLS; ++j, ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                if (!mbar_wait(bar(BAR_FULL(s)), ph, abort_flag, p.status)) { ok = false; break; }
                if (j < KT) {
                    const uint8_t* st = base + s * STAGE_BYTES;
                    // va[4 i + w]: word w (rows lane + 32 w) of A's atom i (k-blocks 4i..4i+3);
                    // vb0 / vb1: B's atoms 0-1 / 2-3, each as [rows 0-127: 4 words, rows 128-255: 4]
                    uint32_t va[16], vb0[16], vb1[16];
                    if constexpr (kGridA) {
                        // rows lane + 32 w lie in block-row lane / 16 + 2 w: its 16 block scales
                        // (one 16-byte grid row) give word w of all four atoms
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            const uint4 g = *reinterpret_cast<const uint4*>(st + OFF_SFA + ((lane >> 4) + 2 * w) * 16);
                            va[w] = g.x; va[4 + w] = g.y; va[8 + w] = g.z; va[12 + w] = g.w;
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint4 a = *reinterpret_cast<const uint4*>(st + OFF_SFA + 512 * i + 16 * lane);
                            va[4 * i] = a.x; va[4 * i + 1] = a.y; va[4 * i + 2] = a.z; va[4 * i + 3] = a.w;
                        }
                    }
                    if constexpr (kGridB) {
#pragma unroll
                        for (int rb = 0; rb < 2; ++rb) {
#pragma unroll
                            for (int w = 0; w < 4; ++w) {
                                const uint4 g = *reinterpret_cast<const uint4*>(
                                    st + OFF_SFB + (8 * rb + (lane >> 4) + 2 * w) * 16);
                                vb0[4 * rb + w] = g.x;
                                vb0[8 + 4 * rb + w] = g.y;
                                vb1[4 * rb + w] = g.z;
                                vb1[8 + 4 * rb + w] = g.w;
                            }
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint4 b0 = *reinterpret_cast<const uint4*>(st + OFF_SFB + 512 * i + 16 * lane);
                            const uint4 b1 =
                                *reinterpret_cast<const uint4*>(st + OFF_SFB + 2048 + 512 * i + 16 * lane);
                            uint32_t* vb = i < 2 ? vb0 : vb1;
                            const int o = 8 * (i & 1);
                            vb[o] = b0.x; vb[o + 1] = b0.y; vb[o + 2] = b0.z; vb[o + 3] = b0.w;
                            vb[o + 4] = b1.x; vb[o + 5] = b1.y; vb[o + 6] = b1.z; vb[o + 7] = b1.w;
                        }
                    }
                    tmem_st_32x32b_x16(lane_base + COL_SFA + 16 * s, va);
                    tmem_st_32x32b_x16(lane_base + COL_SFB + 32 * s, vb0);
                    tmem_st_32x32b_x16(lane_base + COL_SFB + 32 * s + 16, vb1);
                    if constexpr (XP) {
                        if (!xpose_share(stage(s) + OFF_B, q, lane, bar(BAR_XREAD), xr, abort_flag, p.status)) {
                            tmem_st_wait();
                            ok = false;
                            break;
                        }
                    }
                    tmem_st_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(bar(BAR_SF_READY(s)), 0));
            }
            if (!ok) break;
        }
    } else {
        // ---------------------------------------------------------------- epilogue (both CTAs)
        const int q = warp & 3;
        if (p.side0.out || p.side1.out)
            lora_split_sums(p.side0, p.side1, blockIdx.x * (32 * EPI_WARPS) + (threadIdx.x - 64),
                            gridDim.x * (32 * EPI_WARPS));
        const int cbase = EPI_COLS * ((warp - 2) >> 2);  // this warp's first tile column
        const float ga = *p.ga, gb = *p.gb;
        const float c = 1.0f / (ga * gb);
        const uint32_t empty_even = mapa_shared(bar(BAR_TMEM_EMPTY), 0);
        float hmax = 0.0f;  // max |gelu output| of this thread's elements (GELU epilogue)
        int sc = 0;         // stores staged by this warp (staging buffer sc % 2)
        int ti = 0;
        for (int t = pair; t < num_tiles && !*abort_flag; t += num_pairs, ++ti) {
            const int mb2 = p.n_inner ? t / NB : t % MB2, nb = p.n_inner ? t % NB : t / MB2;
            if (!mbar_wait(bar(BAR_TMEM_FULL), ti & 1, abort_flag, p.status)) break;
            tc_fence_after();
            if constexpr (EPI == kEpiGeluBwd) {
                // this thread's 512 bytes of gelu_in for the tile, into L2 while the drain runs
                const __nv_bfloat16* r = p.gelu_in +
                    static_cast<size_t>((mb2 * 2 + static_cast<int>(rank)) * BM + 32 * q + lane) * p.ldo + nb * BN +
                    cbase;
#pragma unroll
                for (int i = 0; i < EPI_COLS / 64; ++i) prefetch_l2(r + 64 * i);
            }
            const uint32_t lane_addr = tmem + COL_ACC + cbase + (static_cast<uint32_t>(32 * q) << 16);
            const uint32_t stage0_u32 = base_u32 + OFF_EPI + (warp - 2) * EPI_BUFS * EPI_BYTES;
            uint8_t* stage0_ptr = base + OFF_EPI + (warp - 2) * EPI_BUFS * EPI_BYTES;
            uint32_t pk[EPI_COLS / 2];
#pragma unroll
            for (int ch = 0; ch < EPI_COLS / 32; ++ch) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(lane_addr + ch * 32, v);
                tmem_ld_wait();
#pragma unroll
                for (int jj = 0; jj < 16; ++jj)
                    pk[ch * 16 + jj] = pack_bf16x2(__uint_as_float(v[2 * jj]) * c,
                                                   __uint_as_float(v[2 * jj + 1]) * c);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(empty_even);
            const int row0 = (mb2 * 2 + static_cast<int>(rank)) * BM + 32 * q;
            // GELU-backward epilogue: this thread's row of gelu_in, one 32-column chunk ahead
            const __nv_bfloat16* prow =
                EPI == kEpiGeluBwd ? p.gelu_in + static_cast<size_t>(row0 + lane) * p.ldo + nb * BN + cbase : nullptr;
            uint4 pin[4];
            if constexpr (EPI == kEpiGeluBwd) {
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) pin[c4] = *reinterpret_cast<const uint4*>(prow + 8 * c4);
            }
#pragma unroll
            for (int ch = 0; ch < EPI_COLS / 32; ++ch) {
                uint32_t stage_u32 = stage0_u32 + (sc & 1) * EPI_BYTES;
                uint8_t* stage_ptr = stage0_ptr + (sc & 1) * EPI_BYTES;
                ++sc;
                if (lane == 0) bulk_wait_group_read1();  // this buffer's last store has read it
                __syncwarp();
                if constexpr (EPI == kEpiGeluBwd) {
                    uint4 cur[4];
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) cur[c4] = pin[c4];
                    if (ch + 1 < EPI_COLS / 32) {
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4)
                            pin[c4] = *reinterpret_cast<const uint4*>(prow + 32 * (ch + 1) + 8 * c4);
                    }
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        pk[ch * 16 + 4 * c4] = gelu_bwd_bf16x2(pk[ch * 16 + 4 * c4], cur[c4].x);
                        pk[ch * 16 + 4 * c4 + 1] = gelu_bwd_bf16x2(pk[ch * 16 + 4 * c4 + 1], cur[c4].y);
                        pk[ch * 16 + 4 * c4 + 2] = gelu_bwd_bf16x2(pk[ch * 16 + 4 * c4 + 2], cur[c4].z);
                        pk[ch * 16 + 4 * c4 + 3] = gelu_bwd_bf16x2(pk[ch * 16 + 4 * c4 + 3], cur[c4].w);
                    }
                }
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const int phys = c4 ^ ((lane >> 1) & 3);
                    *reinterpret_cast<uint4*>(stage_ptr + lane * 64 + phys * 16) =
                        make_uint4(pk[ch * 16 + 4 * c4], pk[ch * 16 + 4 * c4 + 1], pk[ch * 16 + 4 * c4 + 2],
                                   pk[ch * 16 + 4 * c4 + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmOut, stage_u32, nb * BN + cbase + ch * 32, row0);
                    bulk_commit_group();
                }
                if constexpr (EPI == kEpiGelu) {
                    // the same chunk through GELU, staged in the other buffer
                    stage_u32 = stage0_u32 + (sc & 1) * EPI_BYTES;
                    stage_ptr = stage0_ptr + (sc & 1) * EPI_BYTES;
                    ++sc;
                    if (lane == 0) bulk_wait_group_read1();
                    __syncwarp();
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const int phys = c4 ^ ((lane >> 1) & 3);
                        *reinterpret_cast<uint4*>(stage_ptr + lane * 64 + phys * 16) =
                            make_uint4(gelu_bf16x2(pk[ch * 16 + 4 * c4], hmax),
                                       gelu_bf16x2(pk[ch * 16 + 4 * c4 + 1], hmax),
                                       gelu_bf16x2(pk[ch * 16 + 4 * c4 + 2], hmax),
                                       gelu_bf16x2(pk[ch * 16 + 4 * c4 + 3], hmax));
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmAct, stage_u32, nb * BN + cbase + ch * 32, row0);
                        bulk_commit_group();
                    }
                }
            }
        }
        if (EPI == kEpiGelu && p.act_amax) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) hmax = fmaxf(hmax, __shfl_xor_sync(0xffffffffu, hmax, o));
            if (lane == 0) atomicMax(p.act_amax, __float_as_uint(hmax));
        }
        if (lane == 0) bulk_wait_group0();
        __syncwarp();
    }

    // Both CTAs are done issuing (remote arrives, loads, MMAs retired) before the pair's
    // tensor memory is released and either CTA exits.
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, TMEM_COLS);
}

}  // namespace gemm2

namespace {

// One variant: its own instantiation, its shared-memory opt-in set once.
template <int EPI, bool XP, int SFC>
cudaError_t launch_variant(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmLA,
                           const CUtensorMap& tmLB, const CUtensorMap& tmOut, const CUtensorMap& tmAct,
                           const CUtensorMap& tmSA, const CUtensorMap& tmSB, const GemmFp4Args& args,
                           cudaLaunchConfig_t cfg) {
    using namespace gemm2;
    static const cudaError_t attr = cudaFuncSetAttribute(
        gemm_fp4_lowrank_pair_kernel<EPI, XP, SFC>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes(EPI));
    if (attr != cudaSuccess) return attr;
    cfg.blockDim = dim3(threads(EPI));
    cfg.dynamicSmemBytes = smem_bytes(EPI);
    return cudaLaunchKernelEx(&cfg, gemm_fp4_lowrank_pair_kernel<EPI, XP, SFC>, tmA, tmB, tmLA, tmLB, tmOut, tmAct,
                              tmSA, tmSB, args);
}

}  // namespace

cudaError_t launch_gemm_fp4_lowrank_pair(const CUtensorMap& tmA, const CUtensorMap& tmB,
                                         const CUtensorMap& tmLA, const CUtensorMap& tmLB,
                                         const CUtensorMap& tmOut, const CUtensorMap& tmAct,
                                         const CUtensorMap& tmSA, const CUtensorMap& tmSB,
                                         const GemmFp4Args& args, int num_sms, cudaStream_t stream) {
    using namespace gemm2;
    const int tiles = (args.M / (2 * BM)) * (args.N / BN);
    int pairs = num_sms / 2;
    if (pairs > tiles) pairs = tiles;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    cfg.stream = stream;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_k
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    before_launch(K_GEMM, stream);
    // Instantiations: the transposing variants serve the backward's dX GEMM (plain or
    // GELU-backward epilogue; Q(R)^T's scales from its tensor-core layout); A's scales come
    // from the tensor-core layout only for 1x16 groups (the plain forward).
    cudaError_t e = cudaErrorInvalidValue;
#define FT_PAIR(E, X, S) launch_variant<E, X, S>(tmA, tmB, tmLA, tmLB, tmOut, tmAct, tmSA, tmSB, args, cfg)
    const int sfc = args.sfc;
    if (args.xpose) {
        if (sfc == 1 && !args.act_out) e = args.gelu_in ? FT_PAIR(kEpiGeluBwd, true, 1) : FT_PAIR(kEpiPlain, true, 1);
    } else if (sfc == 3) {
        e = args.gelu_in ? FT_PAIR(kEpiGeluBwd, false, 3)
            : args.act_out ? FT_PAIR(kEpiGelu, false, 3) : FT_PAIR(kEpiPlain, false, 3);
    } else if (sfc == 2 && !args.gelu_in && !args.act_out) {
        e = FT_PAIR(kEpiPlain, false, 2);
    }
#undef FT_PAIR
    after_launch(K_GEMM, stream);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace ft
