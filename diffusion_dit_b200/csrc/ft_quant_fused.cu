// Fused 16x16-block quantizer + low-rank down-projection (FourTune, arXiv 2607.05711,
// section 3.3 "LoRA Fusion": the quantizer and the stabilizer / LoRA down-projections
// share the same input, so they run as one kernel that reads it once).
//
// For a bf16 input X [rows, cols] and a bf16 down factor W [Rp, cols] (Rp = the rank
// rounded up to 16, extra rows zero) one CTA takes a 128-row band and a slice of the
// columns.  Each 128 x 64 tile arrives by TMA (128-byte swizzle) into a shared-memory
// ring and is consumed twice:
//   * an MMA issuer multiplies it with the matching W tile on the tensor cores
//     (tcgen05.mma kind::f16, [128 x Rp] fp32 in TMEM), giving a partial of T = X W^T.
//     Two issuers in separate warps take alternate stages, each into its own
//     accumulator: one thread issues a 128 x Rp x 16 MMA no faster than a 128 x 128 x 16
//     one, so a single issuer would pace the ring;
//   * a set of four quantizer warps (two 16-row block-rows each) copies the tile out of
//     shared memory into registers, releases the stage, and emits the E2M1 codes, the
//     compact block scales and the tensor-core scale layout (same arithmetic, bit for
//     bit, as quant_block16_kernel in ft_quant.cu).  Four sets take the stages in turn.
// A stage is released when its MMAs have finished reading it (tcgen05.commit) and the
// four warps of its set hold its data.  At the end four warps add the two accumulators
// (in a fixed order) into partials[split][row][Rp]; ft_lowrank.cu sums the splits in a
// fixed order.
#include "ft_internal.h"
#include "ft_ptx.cuh"

namespace ft {
namespace qf {

constexpr int BM = 128;
constexpr int BKE = 64;                 // bf16 columns per stage (one 128-byte row)
constexpr int X_BYTES = BM * 128;       // 16 KB
#ifndef FT_QUANT_SETS
#define FT_QUANT_SETS 4
#endif
#ifndef FT_QUANT_SET_WARPS
#define FT_QUANT_SET_WARPS 4
#endif
constexpr int NQ_SET = FT_QUANT_SET_WARPS;  // quantizer warps per set (one set per stage)
constexpr int BR = 8 / NQ_SET;              // 16-row block-rows per quantizer warp
constexpr int NSETS = FT_QUANT_SETS;        // sets take the stages in turn (k % NSETS)
constexpr int NQ = NQ_SET * NSETS;         // quantizer warps
#ifndef FT_QUANT_MMA_WARPS
#define FT_QUANT_MMA_WARPS 2
#endif
// A bf16 MMA of 128 x Rp x 16 costs the issuing thread about as much as one of 128 x 128 x 16,
// so the down-projection's four MMAs per stage are issued by MW threads in separate warps
// (stages alternate between them), each into its own accumulator; the epilogue adds them.
constexpr int MW = FT_QUANT_MMA_WARPS;
constexpr int QW0 = 1 + MW;                 // first quantizer warp
constexpr int THREADS = 32 * (QW0 + NQ);    // producer, MMA issuers, quantizers
constexpr int MAX_STAGES = 8;
constexpr int BAR_BYTES = 768;           // barriers, TMEM slot, abort flag, inv table at +160, max scratch at +672
static_assert(160 + 512 + 4 * NQ <= BAR_BYTES, "barrier area overflow");

struct Layout {
    int stages;
    int stage_bytes;
    int smem_bytes;
};

__host__ __device__ inline Layout layout_for(int Rp) {
    Layout L;
    L.stage_bytes = X_BYTES + Rp * 128;
    // A stage is always consumed by the same quantizer set and the same MMA issuer (the
    // stage count is a multiple of both): each then waits on a stage's phases one after
    // another, so a parity wait cannot be satisfied by the phase before the one it wants.
    constexpr int unit = (NSETS % MW == 0) ? NSETS : (MW % NSETS == 0 ? MW : NSETS * MW);
    // as many stages as the 227 KB of dynamic shared memory hold next to the barrier area
    int s = (232448 - BAR_BYTES - 1024) / L.stage_bytes;
    if (s > MAX_STAGES) s = MAX_STAGES;
    s -= s % unit;
    if (s < unit) s = unit;
    L.stages = s;
    L.smem_bytes = s * L.stage_bytes + BAR_BYTES + 1024;
    return L;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <int GRAN>
__global__ void __launch_bounds__(THREADS, 1)
    quant_down_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                      const QuantDownArgs p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t pad = (1024 - (raw_u32 & 1023)) & 1023;
    uint8_t* base = smem_raw + pad;
    const uint32_t base_u32 = raw_u32 + pad;
    const Layout L = layout_for(p.Rp);
    const int S = L.stages;
    uint8_t* bar_area = base + S * L.stage_bytes;
    auto bar = [&](int i) { return base_u32 + S * L.stage_bytes + 8 * i; };
    // barriers: full[0..S), empty[S..2S), tmem_full 2S, final 2S+1
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(bar_area + 8 * (2 * MAX_STAGES + 2));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_area + 8 * (2 * MAX_STAGES + 2) + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int band = blockIdx.x;
    const int split = blockIdx.y;
    const int64_t row0 = static_cast<int64_t>(band) * BM;
    const int64_t col0 = static_cast<int64_t>(split) * p.cols_per_split;
    const int nk = p.cols_per_split / BKE;
    const bool has_mma = p.Rp > 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(bar(i), 1);
            mbar_init(bar(S + i), NQ_SET + (has_mma ? 1 : 0));  // one set of quantizer warps + MMA
        }
        mbar_init(bar(2 * S), MW);
        mbar_init(bar(2 * S + 1), MW);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmX);
        if (has_mma) tma_prefetch_desc(&tmW);
    }
    if (warp == 1 && has_mma) {
        tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = has_mma ? *tmem_slot : 0;
    // TMEM is allocated before dependents may be scheduled on this SM (a waiting
    // dependent never holds tensor memory this CTA still needs).
    pdl_trigger();
    pdl_wait();

    if (warp == 0) {
        if (lane == 0) {
            const uint32_t tx = X_BYTES + p.Rp * 128;
            int k = 0;
            for (; k < nk; ++k) {
                const int s = k % S;
                if (!mbar_wait(bar(S + s), ((k / S) & 1) ^ 1, abort_flag, p.status)) break;
                const uint32_t st = base_u32 + s * L.stage_bytes;
                mbar_arrive_expect_tx(bar(s), tx);
                const int c = static_cast<int>(col0) + k * BKE;
                tma_load_2d(st, &tmX, bar(s), c, static_cast<int>(row0));
                if (has_mma) tma_load_2d(st + X_BYTES, &tmW, bar(s), c, 0);
            }
            for (int j = k - 1; j >= 0 && j >= k - S; --j) {
                volatile int no_abort = 0;
                mbar_wait(bar(j % S), (j / S) & 1, &no_abort, p.status);
            }
        }
    } else if (warp < QW0) {
        if (has_mma && lane == 0) {
            const int m = warp - 1;  // this issuer takes stages k with k % MW == m
            const uint32_t acc = tmem + m * (p.tmem_cols / MW);
            const uint32_t idesc = idesc_bf16(BM, p.Rp);
            for (int k = m; k < nk; k += MW) {
                const int s = k % S;
                if (!mbar_wait(bar(s), (k / S) & 1, abort_flag, p.status)) break;
                tc_fence_after();
                const uint32_t st = base_u32 + s * L.stage_bytes;
                const uint64_t ad = sdesc_kmajor_sw128(st);
                const uint64_t bd = sdesc_kmajor_sw128(st + X_BYTES);
#pragma unroll
                for (int i = 0; i < 4; ++i) mma_bf16(acc, ad + 2 * i, bd + 2 * i, idesc, k >= MW || i != 0);
                tc_commit(bar(S + s));
            }
            tc_commit(bar(2 * S));
            tc_commit(bar(2 * S + 1));
            volatile int no_abort = 0;
            mbar_wait(bar(2 * S + 1), 0, &no_abort, p.status);
        }
    } else {
        // ---------------------------------------------------------------- quantizers
        // A set of NQ_SET warps quantizes one stage; warp qw of the set owns BR = 8 / NQ_SET
        // consecutive 16-row block-rows of the band.  Lane L works on column block
        // j = L / 8 of the stage and holds, in each of its block-rows, rows l8 and l8 + 8
        // (l8 = L % 8), 16 elements each: a block max takes three shuffle steps inside the
        // 8-lane group, and each lane derives its block's scale once.  The warp copies its
        // rows out of the stage and releases the stage at once (the arithmetic runs on
        // registers), so the ring refills while the sets compute.  The per-tensor table
        // inv[sb] = fl32(g / val(sb)) replaces the division per block; the block max / 6
        // uses div6_bf16 (exact for bf16 inputs).
        const int qw = (warp - QW0) % NQ_SET;
        const int set = (warp - QW0) / NQ_SET;  // this warp takes stages k with k % NSETS == set
        float g = 1.0f;
        bool degenerate = true;
        {
            float amax;
            if (p.amax_parts) {  // max of the per-CTA maxima (exact in any order)
                float m = 0.0f;
                for (int i = threadIdx.x - 32 * QW0; i < p.amax_nparts; i += 32 * NQ) m = fmaxf(m, p.amax_parts[i]);
                m = warp_max(m);
                float* red = reinterpret_cast<float*>(bar_area + 160 + 512);  // after the inv table
                if (lane == 0) red[warp - QW0] = m;
                asm volatile("bar.sync 1, %0;" ::"n"(32 * NQ) : "memory");  // quantizer warps only
                m = 0.0f;
                for (int w = 0; w < NQ; ++w) m = fmaxf(m, red[w]);
                amax = m;
            } else {
                amax = *p.amax;
            }
            if (amax > 0.0f) {
                const float gg = __fdiv_rn(2688.0f, amax);
                if (isfinite(gg) && gg > 0.0f) {
                    g = gg;
                    degenerate = false;
                }
            }
        }
        if (band == 0 && split == 0 && threadIdx.x == 32 * QW0) *p.g_out = g;
        float* inv_lut = reinterpret_cast<float*>(bar_area + 160);  // 128 floats
        {
            const int t = threadIdx.x - 32 * QW0;
            if (t < 128) inv_lut[t] = (t > 0 && t < 127) ? __fdiv_rn(g, ue4m3_to_f32(t)) : 0.0f;
            asm volatile("bar.sync 1, %0;" ::"n"(32 * NQ) : "memory");  // quantizer warps only
        }
        const int j = lane >> 3;  // column block of the stage
        const int l8 = lane & 7;
        // the lane's rows inside the band: rows[2b] = block-row b's row l8, rows[2b+1] = row l8 + 8
        int rows[2 * BR];
#pragma unroll
        for (int b = 0; b < BR; ++b) {
            rows[2 * b] = (qw * BR + b) * 16 + l8;
            rows[2 * b + 1] = rows[2 * b] + 8;
        }
        const int64_t cbs = p.cols / 16;
        const int64_t atoms_per_band = p.cols / 64;
        // bf16 bits of max |x| over a row's 16 elements (two 16-byte chunks): a tree of
        // packed magnitude maxima, then the sign bits cleared (the quantizer's inputs are
        // finite or infinite, never NaN)
        auto row_max = [](const uint4& a, const uint4& b) -> uint32_t {
            const uint32_t m = absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(a.x, a.y), absmax_bf16x2(a.z, a.w)),
                                             absmax_bf16x2(absmax_bf16x2(b.x, b.y), absmax_bf16x2(b.z, b.w))) &
                               0x7FFF7FFFu;
            return max(m & 0xFFFFu, m >> 16);
        };
        auto scale_of = [&](uint32_t amb) -> uint32_t {  // amb: bf16 bits of the block max
            return degenerate ? 0u : cvt_ue4m3(__fmul_rn(div6_bf16(__uint_as_float(amb << 16)), g));
        };
        auto encode8 = [&](const uint4& u, float inv) {
            float v[8];  // x * inv, each rounded to nearest in fp32 (two per instruction)
            mul2_rn(bf16lo_to_f32(u.x), bf16hi_to_f32(u.x), inv, v[0], v[1]);
            mul2_rn(bf16lo_to_f32(u.y), bf16hi_to_f32(u.y), inv, v[2], v[3]);
            mul2_rn(bf16lo_to_f32(u.z), bf16hi_to_f32(u.z), inv, v[4], v[5]);
            mul2_rn(bf16lo_to_f32(u.w), bf16hi_to_f32(u.w), inv, v[6], v[7]);
            return cvt_e2m1x8(v);
        };
        // the four blocks' scale bytes of one row, gathered from the lanes with the same
        // l8: l8, l8 + 8, l8 + 16, l8 + 24 hold blocks 0..3
        auto gather4 = [&](uint32_t sbv) {
            return __shfl_sync(0xffffffffu, sbv, l8) | (__shfl_sync(0xffffffffu, sbv, l8 + 8) << 8) |
                   (__shfl_sync(0xffffffffu, sbv, l8 + 16) << 16) |
                   (__shfl_sync(0xffffffffu, sbv, l8 + 24) << 24);
        };
        for (int k = set; k < nk; k += NSETS) {
            const int s = k % S;
            if (!mbar_wait(bar(s), (k / S) & 1, abort_flag, p.status)) break;
            const uint8_t* tile = base + s * L.stage_bytes;
            uint4 w[2 * BR][2];  // per row: 16-byte chunks 2j, 2j + 1
#pragma unroll
            for (int i = 0; i < 2 * BR; ++i) {
                const int r = rows[i];
                w[i][0] = *reinterpret_cast<const uint4*>(tile + r * 128 + (((2 * j) ^ (r & 7)) << 4));
                w[i][1] = *reinterpret_cast<const uint4*>(tile + r * 128 + (((2 * j + 1) ^ (r & 7)) << 4));
            }
            uint32_t rmax[2 * BR];  // per row: max |x| over its 16 elements (bf16 bits)
#pragma unroll
            for (int i = 0; i < 2 * BR; ++i) rmax[i] = row_max(w[i][0], w[i][1]);
            // every loaded word has been consumed: the stage goes back to the producer
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(S + s));

            const int64_t c0 = col0 + k * BKE;
            uint8_t* atom = p.sf_mma ? p.sf_mma + (static_cast<int64_t>(band) * atoms_per_band + c0 / 64) * 512
                                     : nullptr;
            uint32_t sb[2 * BR];  // per row: its block's (16x16) or its group's (1x16) scale
            if constexpr (GRAN == 16) {
#pragma unroll
                for (int b = 0; b < BR; ++b) {
                    uint32_t amb = max(rmax[2 * b], rmax[2 * b + 1]);
                    amb = max(amb, __shfl_xor_sync(0xffffffffu, amb, 1));
                    amb = max(amb, __shfl_xor_sync(0xffffffffu, amb, 2));
                    amb = max(amb, __shfl_xor_sync(0xffffffffu, amb, 4));
                    sb[2 * b] = sb[2 * b + 1] = scale_of(amb);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 2 * BR; ++i) sb[i] = scale_of(rmax[i]);
            }
#pragma unroll
            for (int i = 0; i < 2 * BR; ++i) {
                const float inv = inv_lut[sb[i]];
                const uint32_t lo = sb[i] ? encode8(w[i][0], inv) : 0u;
                const uint32_t hi = sb[i] ? encode8(w[i][1], inv) : 0u;
                *reinterpret_cast<uint2*>(p.codes + (row0 + rows[i]) * (p.cols / 2) + c0 / 2 + 8 * j) =
                    make_uint2(lo, hi);
            }
            // scale words (the four blocks of a row): row i of the lane's 2 * BR rows is
            // stored by the lanes of group j = i % 4
#pragma unroll
            for (int i = 0; i < 2 * BR; ++i) {
                if (GRAN == 16 && (i & 1)) continue;  // both rows of a block-row share one word
                const uint32_t w4 = gather4(sb[i]);
                if constexpr (GRAN == 16) {
                    if (lane == i / 2)
                        *reinterpret_cast<uint32_t*>(p.scales + (row0 / 16 + qw * BR + i / 2) * cbs + c0 / 16) = w4;
                }
#pragma unroll
                for (int h = 0; h < (GRAN == 16 ? 2 : 1); ++h) {
                    const int ii = i + h;
                    if ((ii & 3) != j) continue;
                    const int r = rows[ii];
                    if constexpr (GRAN == 1)
                        *reinterpret_cast<uint32_t*>(p.scales + (row0 + r) * cbs + c0 / 16) = w4;
                    if (atom) *reinterpret_cast<uint32_t*>(atom + 16 * (r % 32) + 4 * (r / 32)) = w4;
                }
            }
        }
        // ------------------------------------------------------------ T partial epilogue
        if (has_mma && warp >= QW0 && warp < QW0 + 4) {
            const int q = warp & 3;  // the TMEM lane quarter this warp may read
            if (mbar_wait(bar(2 * S), 0, abort_flag, p.status)) {
                tc_fence_after();
                const int64_t orow = row0 + 32 * q + lane;
                float* dst = p.partial + (static_cast<int64_t>(split) * p.rows + orow) * p.Rp;
                const int used = nk < MW ? nk : MW;  // accumulators that received stages
                auto ld16 = [&](uint32_t col, uint32_t (&v)[16]) {
                    asm volatile(
                        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                          "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),
                          "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
                        : "r"(tmem + (static_cast<uint32_t>(32 * q) << 16) + col));
                };
                for (int c = 0; c < p.Rp; c += 16) {
                    float t[16];
                    for (int m = 0; m < used; ++m) {  // accumulators added in order
                        uint32_t v[16];
                        ld16(m * (p.tmem_cols / MW) + c, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 16; ++e) t[e] = m ? __fadd_rn(t[e], __uint_as_float(v[e])) : __uint_as_float(v[e]);
                    }
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4*>(dst + c + e) = make_float4(t[e], t[e + 1], t[e + 2], t[e + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1 && has_mma) tmem_dealloc(tmem, p.tmem_cols);
}

}  // namespace qf

int quant_down_splits(int64_t rows, int64_t cols, int num_sms) {
    // Enough CTAs to cover the SMs once: split the columns of each 128-row band into
    // slices of whole 64-column tiles.
    const int64_t bands = rows / 128;
    const int64_t tiles = cols / 64;
    if (num_sms > 160) num_sms = 160;  // the workspace queries size partials for at most 160 SMs
    int64_t s = bands > 0 ? num_sms / bands : 1;
    if (s < 1) s = 1;
    if (s > 16) s = 16;
    while (s > 1 && tiles % s) --s;
    return static_cast<int>(s);
}

uint32_t quant_down_tmem_cols(int Rp) {
    // MW accumulators, each at a multiple of 32 columns; a power of two >= 32 in all
    uint32_t per = 32;
    while (per < static_cast<uint32_t>(Rp)) per += 32;
    uint32_t c = 32;
    while (c < per * qf::MW) c <<= 1;
    return c;
}

size_t quant_down_smem_bytes(int Rp) { return static_cast<size_t>(qf::layout_for(Rp).smem_bytes); }

cudaError_t launch_quant_down(const CUtensorMap& tmX, const CUtensorMap& tmW, const QuantDownArgs& a,
                              int splits, cudaStream_t stream) {
    const qf::Layout L = qf::layout_for(a.Rp);
    // the opt-in limits are raised once to the device maximum (no per-launch host calls)
    static const cudaError_t attr16 = cudaFuncSetAttribute(
        qf::quant_down_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
    static const cudaError_t attr1 = cudaFuncSetAttribute(
        qf::quant_down_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
    if (attr16 != cudaSuccess) return attr16;
    if (attr1 != cudaSuccess) return attr1;
    dim3 grid(static_cast<unsigned>(a.rows / 128), static_cast<unsigned>(splits));
    before_launch(K_QUANT, stream);
    const cudaError_t le =
        a.block_rows == 1 ? launch_k(qf::quant_down_kernel<1>, dim3(grid), dim3(qf::THREADS), L.smem_bytes, stream,
                                     tmX, tmW, a)
                          : launch_k(qf::quant_down_kernel<16>, dim3(grid), dim3(qf::THREADS), L.smem_bytes,
                                     stream, tmX, tmW, a);
    if (le != cudaSuccess) return le;
    after_launch(K_QUANT, stream);
    return cudaGetLastError();
}

}  // namespace ft
