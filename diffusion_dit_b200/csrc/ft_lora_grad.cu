// Adapter weight gradients on the tensor cores (FourTune, arXiv 2607.05711, section
// 3.2: weight gradients exist only for the adapter branch):
//   dB [N, r] = s G^T T_lora          (T_lora = X A^T, saved by the forward)
//   dA [r, K] = s U_lora^T X          (U_lora = G B, from the backward down-projection)
// Both are contractions over the tokens m of a big bf16 operand P [M, F] (G or X,
// row-major: F contiguous) with a small operand V [M, r]:
//   D[f, c] = sum_m P[m, f] V'[m, c]
// The 128 x 64 tile of P that TMA puts in shared memory (rows = tokens) is exactly
// the MN-major layout the MMA wants for an A operand indexed (f, m), so P is read once,
// straight, with no transpose.  V' = [hi(V), lo(V), 0] (bf16, width NBW = 2r rounded
// up to 64) is MN-major too; the hi and lo halves land in separate accumulator
// columns and are added in the final sum, keeping ~16 mantissa bits of V.
//
// Schedule (lora_grad_schedule): one CTA per SM at a time, in lockstep over the tokens
// -- the CTAs running together read the same 64-token rows of P, each its own 128
// features, so every row of P streams from HBM whole.  Phase 1: q = T / P rounds of whole
// tiles (T tiles of 128 features, P SMs), CTA b < qP taking tile b over all tokens.
// Phase 2: the R = T - qP remaining tiles, each split over S2 = P / R token ranges (at
// most 16), CTA qP + s R + i taking range s of tile qP + i, so that the CTAs of one range
// run together.  CTA b leaves its sum in partial slot b, [128 features][NBW] fp32;
// lora_split_sums (ft_sidejobs.cuh) adds a tile's slots in token order (deterministic).
// The dX GEMM's epilogue warps run those sums while they wait for their first
// accumulator, or a launch of its own does.
//
// When asked (amax_out), the four epilogue warps, idle until the final drain, also take
// max |P| over every tile that lands: with dB computed first in the backward pass this
// gives the tensor max of G for Q(G) without a separate pass over G.
#include "ft_internal.h"
#include "ft_ptx.cuh"
#include "ft_sidejobs.cuh"

namespace ft {
namespace lg {

constexpr int BF = 128;                 // features per CTA (MMA M)
constexpr int BMT = 64;                 // tokens per stage
constexpr int A_BYTES = BMT * BF * 2;   // 16 KB: two 64-feature boxes of [64 tokens x 128 B]
constexpr int THREADS = 192;            // producer, MMA, 4 epilogue warps
constexpr int MAX_STAGES = 8;
constexpr int BAR_BYTES = 256;

struct Layout {
    int stages, stage_bytes, smem_bytes;
};

__host__ __device__ inline Layout layout_for(int NBW) {
    Layout L;
    L.stage_bytes = A_BYTES + BMT * NBW * 2;
    int s = (192 * 1024) / L.stage_bytes;
    if (s > 6) s = 6;
    if (s < 2) s = 2;
    L.stages = s;
    L.smem_bytes = s * L.stage_bytes + BAR_BYTES + 1024;
    return L;
}

__global__ void __launch_bounds__(THREADS, 1)
    lora_grad_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmV,
                     const LoraGradArgs p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t pad = (1024 - (raw_u32 & 1023)) & 1023;
    const uint32_t base_u32 = raw_u32 + pad;
    uint8_t* base = smem_raw + pad;
    const Layout L = layout_for(p.NBW);
    const int S = L.stages;
    uint8_t* bar_area = base + S * L.stage_bytes;
    auto bar = [&](int i) { return base_u32 + S * L.stage_bytes + 8 * i; };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(bar_area + 8 * (2 * MAX_STAGES + 2));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_area + 8 * (2 * MAX_STAGES + 2) + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // this CTA's tile and token range (see the schedule above)
    int tile, c0, c1;
    {
        const int b = blockIdx.x;
        if (b < p.full_tiles) {
            tile = b;
            c0 = 0;
            c1 = p.chunks;
        } else {
            const int rr = b - p.full_tiles;
            const int s = rr / p.rem_tiles;
            tile = p.full_tiles + (rr - s * p.rem_tiles);
            c0 = static_cast<int>(static_cast<int64_t>(s) * p.chunks / p.rem_splits);
            c1 = static_cast<int>(static_cast<int64_t>(s + 1) * p.chunks / p.rem_splits);
        }
    }
    const int f0 = tile * BF;
    const int m0 = c0 * BMT;
    const int nk = c1 - c0;
    const int nchunk = p.NBW / 64;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(bar(i), 1);
            mbar_init(bar(S + i), 1 + (p.amax_out ? 4 : 0));  // MMA commit (+ 4 max warps)
        }
        mbar_init(bar(2 * S), 1);
        mbar_init(bar(2 * S + 1), 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmP);
        tma_prefetch_desc(&tmV);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), p.tmem_cols);
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
        if (lane == 0) {
            const uint32_t tx = L.stage_bytes;
            int k = 0;
            for (; k < nk; ++k) {
                const int s = k % S;
                if (!mbar_wait(bar(S + s), ((k / S) & 1) ^ 1, abort_flag, p.status)) break;
                const uint32_t st = base_u32 + s * L.stage_bytes;
                mbar_arrive_expect_tx(bar(s), tx);
                const int mm = m0 + k * BMT;
                tma_load_2d(st, &tmP, bar(s), f0, mm);
                tma_load_2d(st + A_BYTES / 2, &tmP, bar(s), f0 + 64, mm);
                for (int c = 0; c < nchunk; ++c)
                    tma_load_2d(st + A_BYTES + c * (BMT * 128), &tmV, bar(s), 64 * c, mm);
            }
            for (int j = k - 1; j >= 0 && j >= k - S; --j) {
                volatile int no_abort = 0;
                mbar_wait(bar(j % S), (j / S) & 1, &no_abort, p.status);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(BF, p.NBW, /*a_mn=*/true, /*b_mn=*/true);
            for (int k = 0; k < nk; ++k) {
                const int s = k % S;
                if (!mbar_wait(bar(s), (k / S) & 1, abort_flag, p.status)) break;
                tc_fence_after();
                const uint32_t st = base_u32 + s * L.stage_bytes;
                // MN-major, 128-byte swizzle: 8-token groups 1024 B apart (SBO); the two
                // 64-feature halves of A (and the 64-column chunks of V) 8 KB apart (LBO).
                const uint64_t ad = sdesc_mnmajor_sw128(st, A_BYTES / 2, 1024);
                const uint64_t bd = sdesc_mnmajor_sw128(st + A_BYTES, BMT * 128, 1024);
#pragma unroll
                for (int i = 0; i < BMT / 16; ++i)  // 16 tokens per MMA = two 8-row groups
                    mma_bf16(tmem, ad + (2048 >> 4) * i, bd + (2048 >> 4) * i, idesc, (k | i) != 0);
                tc_commit(bar(S + s));
            }
            tc_commit(bar(2 * S));
            tc_commit(bar(2 * S + 1));
            volatile int no_abort = 0;
            mbar_wait(bar(2 * S + 1), 0, &no_abort, p.status);
        }
    } else {
        const int q = warp & 3;
        if (p.amax_out) {
            // max |x| of each landed P tile (16 KB: 8 x 16 bytes per thread), fp32 fmaxf
            // as in amax_kernel (a NaN never wins); the stage is released after the read
            float m = 0.0f;
            const int t = threadIdx.x - 64;  // 0..127
            for (int k = 0; k < nk; ++k) {
                const int s = k % S;
                if (!mbar_wait(bar(s), (k / S) & 1, abort_flag, p.status)) break;
                const uint8_t* tile = base + s * L.stage_bytes;
#pragma unroll
                for (int i = 0; i < A_BYTES / (128 * 16); ++i) {
                    const uint4 w = *reinterpret_cast<const uint4*>(tile + (i * 128 + t) * 16);
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        m = fmaxf(m, fmaxf(fabsf(bf16lo_to_f32(ws[e])), fabsf(bf16hi_to_f32(ws[e]))));
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(S + s));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) atomicMax(p.amax_out, __float_as_uint(m));
        }
        if (mbar_wait(bar(2 * S), 0, abort_flag, p.status)) {
            tc_fence_after();
            float* dst = p.partial + (static_cast<int64_t>(blockIdx.x) * BF + 32 * q + lane) * p.NBW;
            for (int c = 0; c < p.NBW; c += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * q) << 16) + c, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4*>(dst + c + e) =
                        make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                    __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, p.tmem_cols);
}

// The split sums in a launch of their own (when the dX GEMM's epilogue warps could not
// finish them within its first tile): the same routine, so the same sums bit for bit.
__global__ void lora_grad_finalize_kernel(const LoraFinalizeJob j0, const LoraFinalizeJob j1) {
    pdl_trigger();
    pdl_wait();
    lora_split_sums(j0, j1, blockIdx.x * blockDim.x + threadIdx.x, gridDim.x * blockDim.x);
}

}  // namespace lg

LoraSchedule lora_grad_schedule(int64_t M, int64_t F, int num_sms) {
    if (num_sms > 160) num_sms = 160;  // the workspace queries size the slots for at most 160 SMs
    LoraSchedule sc{};
    const int T = static_cast<int>(F / lg::BF);
    const int C = static_cast<int>(M / lg::BMT);
    sc.full_tiles = (T / num_sms) * num_sms;
    sc.rem_tiles = T - sc.full_tiles;
    int s2 = sc.rem_tiles ? num_sms / sc.rem_tiles : 0;
    if (sc.rem_tiles && s2 < 1) s2 = 1;
    if (s2 > 16) s2 = 16;
    if (s2 > C) s2 = C;
    sc.rem_splits = s2;
    sc.ctas = sc.full_tiles + sc.rem_tiles * s2;
    return sc;
}

cudaError_t launch_lora_grad(const CUtensorMap& tmP, const CUtensorMap& tmV, const LoraGradArgs& a, int kind,
                             cudaStream_t stream) {
    const lg::Layout L = lg::layout_for(a.NBW);
    // the opt-in limit is raised once to the device maximum (no per-launch host calls)
    static const cudaError_t attr = cudaFuncSetAttribute(
        lg::lora_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
    if (attr != cudaSuccess) return attr;
    dim3 grid(static_cast<unsigned>(a.full_tiles + a.rem_tiles * a.rem_splits));
    before_launch(kind, stream);
    const cudaError_t le = launch_k(lg::lora_grad_kernel, dim3(grid), dim3(lg::THREADS),
                                    L.smem_bytes, stream, tmP, tmV, a);
    if (le != cudaSuccess) return le;
    after_launch(kind, stream);
    return cudaGetLastError();
}

cudaError_t launch_lora_grad_finalize(const LoraFinalizeJob& j0, const LoraFinalizeJob& j1, cudaStream_t stream) {
    // one worker per block of 4 features x 4 columns
    int64_t g = ((j0.out ? static_cast<int64_t>(j0.F) * j0.r / 16 : 0) +
                 (j1.out ? static_cast<int64_t>(j1.F) * j1.r / 16 : 0) + 255) / 256;
    if (g > 148 * 8) g = 148 * 8;
    if (g < 1) g = 1;
    before_launch(K_OTHER, stream);
    const cudaError_t le = launch_k(lg::lora_grad_finalize_kernel, dim3(static_cast<unsigned>(g)), dim3(256), 0,
                                    stream, j0, j1);
    if (le != cudaSuccess) return le;
    after_launch(K_OTHER, stream);
    return cudaGetLastError();
}

}  // namespace ft
