// Block-scaled FP4 GEMM with the low-rank branches added in the same accumulator.
//
//   OUT[M, N] = bf16( ( sum_k a(m,k) sfa(m,k/16) * b(n,k) sfb(n,k/16)        (E2M1 x E2M1)
//                      + sum_j LA(m, j) LB(n, j) ) * 1/(g_a g_b) )            (bf16 x bf16)
//
// FourTune (arXiv 2607.05711), Eq. (2) forward: a = Q(X), b = Q(R), and the low-rank
// operands carry X [Ls_down; A]^T and [Ls_up, B] (section 3.3 "LoRA Fusion": the up-
// projections are fused into the 4-bit GEMM).  Eq. (3) backward: a = Q(G), b = Q(R)^T,
// low-rank operands G [Ls_up, B] and [Ls_down; A]^T.  The caller pre-multiplies the
// low-rank A operand by g_a g_b and splits it into a bf16 high and low part (both
// multiplied by the same B operand), so the branch keeps ~16 mantissa bits.
//
// B200 design: persistent CTAs (one per SM), 128x256 output tile per CTA, a 4-stage
// shared-memory ring fed by TMA (128-byte swizzle), tcgen05.mma with the fp32
// accumulator in tensor memory, scale factors written into tensor memory by four scale
// warps with tcgen05.st (a tcgen05.cp costs the tensor pipe about as much as half an MMA,
// and a stage would need twelve of them), and an epilogue that drains TMEM into
// registers before storing so the next tile's MMAs start while the stores are still in
// flight.
//
// Warp roles (320 threads): warp 0 = TMA producer, warp 1 = MMA issuer (and TMEM
// owner), warps 2..5 = epilogue, warps 6..9 = scale writers (warp w reaches TMEM lanes
// 32 (w % 4) .. +31).
//
// With XP (the dX GEMM of section 3.2 without a stored Q(R)^T) the producer loads B's
// untransposed slab, 256 reduction rows x 128 bytes, into the B slot and the scale writers
// transpose it in place (ft_xpose.cuh) before they arrive on SF_READY.
#include "ft_internal.h"
#include "ft_ptx.cuh"
#include "ft_sidejobs.cuh"
#include "ft_xpose.cuh"

namespace ft {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK_BYTES = 128;            // one 128-byte swizzle row: 256 fp4 or 64 bf16
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK_BYTES;   // 16 KB
constexpr int B_BYTES = BN * BK_BYTES;   // 32 KB
constexpr int SFA_BYTES = 4 * 512;       // 4 k-blocks of 64 x 128 rows
constexpr int SFB_BYTES = 2 * 4 * 512;   // 2 row bands of 128
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;  // 55296
constexpr int OFF_B = A_BYTES;
constexpr int OFF_SFA = A_BYTES + B_BYTES;
constexpr int OFF_SFB = OFF_SFA + SFA_BYTES;
constexpr int EPI_BYTES = 32 * 64;        // per epilogue warp: 32 rows x 32 bf16 columns
constexpr int OFF_EPI = STAGES * STAGE_BYTES;
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 4 * EPI_BYTES + BAR_BYTES + 1024;  // + alignment slack
constexpr int THREADS = 320;

// Tensor memory columns: accumulator [0,256), scale slots per stage after it.
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_ACC = 0;
constexpr uint32_t COL_SFA = 256;  // 4 stages x 16 columns
constexpr uint32_t COL_SFB = 320;  // 4 stages x 32 columns

static_assert(STAGE_BYTES % 1024 == 0, "stage must keep 1024-byte alignment");
static_assert(SMEM_BYTES <= 232448, "exceeds 227 KB of dynamic shared memory");

struct Smem {
    uint8_t* base;    // 1024-aligned
    uint32_t base_u32;
    __device__ uint32_t stage(int s) const { return base_u32 + s * STAGE_BYTES; }
    __device__ uint32_t bar(int i) const { return base_u32 + OFF_EPI + 4 * EPI_BYTES + 8 * i; }
};
// barrier indices
__host__ __device__ constexpr int BAR_FULL(int s) { return s; }
__host__ __device__ constexpr int BAR_EMPTY(int s) { return STAGES + s; }
constexpr int BAR_TMEM_FULL = 2 * STAGES;
constexpr int BAR_TMEM_EMPTY = 2 * STAGES + 1;
constexpr int BAR_FINAL = 2 * STAGES + 2;
__host__ __device__ constexpr int BAR_SF_READY(int s) { return 2 * STAGES + 3 + s; }
constexpr int BAR_XREAD = 3 * STAGES + 3;  // XP: the scale warps have read the raw B slab
constexpr int NUM_BARS = 3 * STAGES + 4;
constexpr int OFF_TMEM_SLOT = 8 * 16;   // inside the barrier area
constexpr int OFF_ABORT = 8 * 16 + 4;
static_assert(8 * NUM_BARS <= OFF_TMEM_SLOT, "barriers overlap the TMEM slot");

template <int EPI, bool XP>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_fp4_lowrank_kernel(const __grid_constant__ CUtensorMap tmA,
                            const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmLA,
                            const __grid_constant__ CUtensorMap tmLB,
                            const __grid_constant__ CUtensorMap tmOut,
                            const __grid_constant__ CUtensorMap tmAct, const GemmFp4Args p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t pad = (1024 - (raw_u32 & 1023)) & 1023;
    Smem sm{smem_raw + pad, raw_u32 + pad};
    uint8_t* bar_area = sm.base + OFF_EPI + 4 * EPI_BYTES;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(bar_area + OFF_TMEM_SLOT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_area + OFF_ABORT);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int MB = p.M / BM;
    const int NB = p.N / BN;
    const int num_tiles = MB * NB;
    const int KT = p.K / 256;      // fp4 stages
    const int KLS = (p.KL + 63) / 64;  // low-rank stages (the last one may be partly past KL:
                                       // TMA fills those columns with zeros, no MMA reads them)
    const int k64 = p.K / 64;      // scale atoms per 128-row band

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(sm.bar(BAR_FULL(i)), 1);
            mbar_init(sm.bar(BAR_EMPTY(i)), 1);
            mbar_init(sm.bar(BAR_SF_READY(i)), 4);
        }
        mbar_init(sm.bar(BAR_TMEM_FULL), 1);
        mbar_init(sm.bar(BAR_TMEM_EMPTY), 4);
        mbar_init(sm.bar(BAR_FINAL), 1);
        mbar_init(sm.bar(BAR_XREAD), 4);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (KLS > 0) {
            tma_prefetch_desc(&tmLA);
            tma_prefetch_desc(&tmLB);
        }
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // TMEM is allocated before dependents may be scheduled on this SM (a waiting
    // dependent never holds tensor memory this CTA still needs).
    pdl_trigger();
    pdl_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int it = 0;
            for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
                const int mb = t % MB, nb = t / MB;
                const int m0 = mb * BM, n0 = nb * BN;
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(sm.bar(BAR_EMPTY(s)), ph ^ 1, abort_flag, p.status)) break;
                    const uint32_t full = sm.bar(BAR_FULL(s));
                    const uint32_t st = sm.stage(s);
                    mbar_arrive_expect_tx(full, STAGE_BYTES);
                    tma_load_2d(st, &tmA, full, kt * BK_BYTES, m0);
                    if constexpr (XP)  // B^T rows kt*256.., the bytes of the tile's 256 columns
                        tma_load_2d(st + OFF_B, &tmB, full, n0 / 2, kt * 256);
                    else
                        tma_load_2d(st + OFF_B, &tmB, full, kt * BK_BYTES, n0);
                    bulk_load(st + OFF_SFA, p.sfa + (static_cast<size_t>(mb) * k64 + kt * 4) * 512,
                              SFA_BYTES, full);
#pragma unroll
                    for (int rb = 0; rb < 2; ++rb)
                        bulk_load(st + OFF_SFB + rb * 2048,
                                  p.sfb + (static_cast<size_t>(nb * 2 + rb) * k64 + kt * 4) * 512,
                                  2048, full);
                }
                if (*abort_flag) break;
                for (int kl = 0; kl < KLS; ++kl, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(sm.bar(BAR_EMPTY(s)), ph ^ 1, abort_flag, p.status)) break;
                    const uint32_t full = sm.bar(BAR_FULL(s));
                    const uint32_t st = sm.stage(s);
                    mbar_arrive_expect_tx(full, A_BYTES + B_BYTES);
                    tma_load_2d(st, &tmLA, full, kl * 64, m0);
                    tma_load_2d(st + OFF_B, &tmLB, full, kl * 64, n0);
                }
            }
            // Drain: every copy this thread issued has landed before the CTA may exit.
            // (Already true on the normal path; on an abort it bounds the wait.)
            for (int j = it - 1; j >= 0 && j >= it - STAGES; --j) {
                volatile int no_abort = 0;
                mbar_wait(sm.bar(BAR_FULL(j % STAGES)), (j / STAGES) & 1, &no_abort, p.status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc4 = idesc_fp4_block16(BM, BN);
            const uint32_t idesc16 = idesc_bf16(BM, BN);
            int it = 0, ti = 0;
            for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x, ++ti) {
                if (!mbar_wait(sm.bar(BAR_TMEM_EMPTY), (ti & 1) ^ 1, abort_flag, p.status)) break;
                tc_fence_after();
                const uint32_t acc = tmem + COL_ACC;
                bool ok = true;
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(sm.bar(BAR_FULL(s)), ph, abort_flag, p.status) ||
                        !mbar_wait(sm.bar(BAR_SF_READY(s)), ph, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = sm.stage(s);
                    const uint32_t sfa_t = tmem + COL_SFA + 16 * s;
                    const uint32_t sfb_t = tmem + COL_SFB + 32 * s;
                    const uint64_t ad = sdesc_kmajor_sw128(st);
                    const uint64_t bd = sdesc_kmajor_sw128(st + OFF_B);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        mma_fp4_block16(acc, ad + 2 * i, bd + 2 * i, idesc4, sfa_t + 4 * i,
                                        sfb_t + 8 * i, (kt | i) != 0);
                    tc_commit(sm.bar(BAR_EMPTY(s)));
                }
                if (!ok) break;
                for (int kl = 0; kl < KLS; ++kl, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(sm.bar(BAR_FULL(s)), ph, abort_flag, p.status) ||
                        !mbar_wait(sm.bar(BAR_SF_READY(s)), ph, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = sm.stage(s);
                    const uint64_t ad = sdesc_kmajor_sw128(st);
                    const uint64_t bd = sdesc_kmajor_sw128(st + OFF_B);
                    const int nk16 = min(4, (p.KL - 64 * kl) / 16);  // K=16 steps inside KL
                    for (int i = 0; i < nk16; ++i) mma_bf16(acc, ad + 2 * i, bd + 2 * i, idesc16, 1);
                    tc_commit(sm.bar(BAR_EMPTY(s)));
                }
                if (!ok) break;
                tc_commit(sm.bar(BAR_TMEM_FULL));
            }
            // Every MMA issued by this thread has retired before TMEM is released.
            tc_commit(sm.bar(BAR_FINAL));
            volatile int no_abort = 0;
            mbar_wait(sm.bar(BAR_FINAL), 0, &no_abort, p.status);
        }
    } else if (warp >= 6) {
        // ------------------------------------------------------------ scale writers
        // Lane l of warp w owns TMEM lane 32 (w % 4) + l.  The block-scaled MMA reads the
        // scales of a 64-wide k block from 4 columns (A) and 8 columns (B) per lane, holding
        // the 16-byte row (l) of each 512-byte scale atom (the tcgen05.cp 32x128b.warpx4
        // layout: the same 32 x 16 bytes in every 32-lane quarter).  Every ring item gets an
        // arrival, so the MMA issuer can wait on SF_READY with the ring's own phase.
        const int q = warp & 3;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
        int it = 0;
        uint32_t xr = 0;  // XREAD phases passed
        for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
            bool ok = true;
            for (int j = 0; j < KT + KLS; ++j, ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                if (!mbar_wait(sm.bar(BAR_FULL(s)), ph, abort_flag, p.status)) { ok = false; break; }
                if (j < KT) {
                    const uint8_t* st = sm.base + s * STAGE_BYTES;
                    uint32_t va[16], vb0[16], vb1[16];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint4 a = *reinterpret_cast<const uint4*>(st + OFF_SFA + 512 * i + 16 * lane);
                        const uint4 b0 = *reinterpret_cast<const uint4*>(st + OFF_SFB + 512 * i + 16 * lane);
                        const uint4 b1 =
                            *reinterpret_cast<const uint4*>(st + OFF_SFB + 2048 + 512 * i + 16 * lane);
                        uint32_t* vb = i < 2 ? vb0 : vb1;
                        const int o = 8 * (i & 1);
                        va[4 * i] = a.x; va[4 * i + 1] = a.y; va[4 * i + 2] = a.z; va[4 * i + 3] = a.w;
                        vb[o] = b0.x; vb[o + 1] = b0.y; vb[o + 2] = b0.z; vb[o + 3] = b0.w;
                        vb[o + 4] = b1.x; vb[o + 5] = b1.y; vb[o + 6] = b1.z; vb[o + 7] = b1.w;
                    }
                    tmem_st_32x32b_x16(lane_base + COL_SFA + 16 * s, va);
                    tmem_st_32x32b_x16(lane_base + COL_SFB + 32 * s, vb0);
                    tmem_st_32x32b_x16(lane_base + COL_SFB + 32 * s + 16, vb1);
                    if constexpr (XP) {
                        const uint32_t slab = sm.stage(s) + OFF_B;
                        xpose::Regs<128> rg;
                        xpose::load<128>(slab, q, lane, rg);
                        __syncwarp();
                        if (lane == 0) mbar_arrive(sm.bar(BAR_XREAD));
                        xpose::transpose<128>(lane, rg);
                        if (!mbar_wait(sm.bar(BAR_XREAD), xr & 1, abort_flag, p.status)) {
                            tmem_st_wait();
                            ok = false;
                            break;
                        }
                        ++xr;
                        xpose::store<128>(slab, q, lane, rg);
                        fence_proxy_async_smem();  // ordinary stores, read next by the MMA
                    }
                    tmem_st_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(sm.bar(BAR_SF_READY(s)));
            }
            if (!ok) break;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        if (p.side0.out || p.side1.out)  // epilogue warps 2..5: 128 threads per CTA
            lora_split_sums(p.side0, p.side1, blockIdx.x * 128 + (threadIdx.x - 64), gridDim.x * 128);
        const float ga = *p.ga, gb = *p.gb;
        const float c = 1.0f / (ga * gb);
        float hmax = 0.0f;  // max |gelu output| of this thread's elements (GELU epilogue)
        int ti = 0;
        for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x, ++ti) {
            const int mb = t % MB, nb = t / MB;
            if (!mbar_wait(sm.bar(BAR_TMEM_FULL), ti & 1, abort_flag, p.status)) break;
            tc_fence_after();
            // Drain the accumulator into registers (scaled, rounded to bf16) and give the
            // tensor memory back to the MMA warp at once; then stage each 32 x 32 block in
            // shared memory (64-byte swizzle, the layout of the output tensor map) and
            // hand it to a TMA store while the next tile's MMAs already run.
            const uint32_t lane_addr = tmem + COL_ACC + (static_cast<uint32_t>(32 * q) << 16);
            const uint32_t stage_u32 = sm.base_u32 + OFF_EPI + (warp - 2) * EPI_BYTES;
            uint8_t* stage_ptr = sm.base + OFF_EPI + (warp - 2) * EPI_BYTES;
            uint32_t pk[BN / 2];
#pragma unroll
            for (int ch = 0; ch < BN / 32; ++ch) {
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
            if (lane == 0) mbar_arrive(sm.bar(BAR_TMEM_EMPTY));
            // GELU-backward epilogue: this thread's row of gelu_in, one 32-column chunk ahead
            const __nv_bfloat16* prow =
                EPI == kEpiGeluBwd ? p.gelu_in + static_cast<size_t>(mb * BM + 32 * q + lane) * p.ldo + nb * BN : nullptr;
            uint4 pin[4];
            if constexpr (EPI == kEpiGeluBwd) {
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) pin[c4] = *reinterpret_cast<const uint4*>(prow + 8 * c4);
            }
#pragma unroll
            for (int ch = 0; ch < BN / 32; ++ch) {
                if (lane == 0) bulk_wait_group_read0();  // previous store has read the buffer
                __syncwarp();
                if constexpr (EPI == kEpiGeluBwd) {
                    uint4 cur[4];
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) cur[c4] = pin[c4];
                    if (ch + 1 < BN / 32) {
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
                    tma_store_2d(&tmOut, stage_u32, nb * BN + ch * 32, mb * BM + 32 * q);
                    bulk_commit_group();
                }
                if constexpr (EPI == kEpiGelu) {
                    // the same chunk through GELU, once the store above has read the buffer
                    if (lane == 0) bulk_wait_group_read0();
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
                        tma_store_2d(&tmAct, stage_u32, nb * BN + ch * 32, mb * BM + 32 * q);
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

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace gemm

namespace {

// One variant: its own instantiation, its shared-memory opt-in set once.
template <int EPI, bool XP>
cudaError_t launch_variant(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmLA,
                           const CUtensorMap& tmLB, const CUtensorMap& tmOut, const CUtensorMap& tmAct,
                           const GemmFp4Args& args, int grid, cudaStream_t stream) {
    using namespace gemm;
    static const cudaError_t attr = cudaFuncSetAttribute(
        gemm_fp4_lowrank_kernel<EPI, XP>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (attr != cudaSuccess) return attr;
    return launch_k(gemm_fp4_lowrank_kernel<EPI, XP>, dim3(grid), dim3(THREADS), SMEM_BYTES, stream, tmA, tmB,
                    tmLA, tmLB, tmOut, tmAct, args);
}

}  // namespace

cudaError_t launch_gemm_fp4_lowrank(const CUtensorMap& tmA, const CUtensorMap& tmB,
                                    const CUtensorMap& tmLA, const CUtensorMap& tmLB,
                                    const CUtensorMap& tmOut, const CUtensorMap& tmAct,
                                    const GemmFp4Args& args, int num_sms, cudaStream_t stream) {
    using namespace gemm;
    const int tiles = (args.M / BM) * (args.N / BN);
    const int grid = tiles < num_sms ? tiles : num_sms;
    before_launch(K_GEMM, stream);
    // the transposing variants serve the backward's dX GEMM (plain or GELU-backward epilogue)
    cudaError_t le;
    if (args.xpose)
        le = args.act_out ? cudaErrorInvalidValue
             : args.gelu_in
                 ? launch_variant<kEpiGeluBwd, true>(tmA, tmB, tmLA, tmLB, tmOut, tmAct, args, grid, stream)
                 : launch_variant<kEpiPlain, true>(tmA, tmB, tmLA, tmLB, tmOut, tmAct, args, grid, stream);
    else
        le = args.gelu_in
                 ? launch_variant<kEpiGeluBwd, false>(tmA, tmB, tmLA, tmLB, tmOut, tmAct, args, grid, stream)
             : args.act_out
                 ? launch_variant<kEpiGelu, false>(tmA, tmB, tmLA, tmLB, tmOut, tmAct, args, grid, stream)
                 : launch_variant<kEpiPlain, false>(tmA, tmB, tmLA, tmLB, tmOut, tmAct, args, grid, stream);
    if (le != cudaSuccess) return le;
    after_launch(K_GEMM, stream);
    return cudaGetLastError();
}

}  // namespace ft
