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
// Work is balanced over persistent CTAs (at most one per SM): the units (128-feature
// tile t, 64-token chunk c) are numbered u = t C + c (C chunks per tile) and CTA p of P
// takes the run [p U / P, (p + 1) U / P) of the U = T C units.  A run is cut into
// segments where it crosses a tile boundary; each segment's sum over its tokens goes to
// partial slot p + t (unique: a CTA's tiles t0..t1 give slots p + t0 .. p + t1, and the
// next CTA starts at tile t1 or later), [128 features][NBW] fp32.  The accumulator is
// double-buffered in tensor memory so that one segment drains while the next fills.
// lora_split_sums (ft_sidejobs.cuh) adds, for each tile, the slots of the CTAs that
// covered it, in token order (deterministic); the dX GEMM's epilogue warps run it while
// they wait for their first accumulator, or a launch of its own does.
//
// When asked (amax_out), the four epilogue warps also take max |P| over every tile that
// lands: with dB computed first in the backward pass this gives the tensor max of G for
// Q(G) without a separate pass over G.
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
    // barriers: FULL [0, S), EMPTY [S, 2S), ACC_FULL 2S + b, ACC_EMPTY 2S + 2 + b (b = the
    // accumulator buffer), FINAL 2S + 4
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(bar_area + 8 * (2 * MAX_STAGES + 5));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_area + 8 * (2 * MAX_STAGES + 5) + 4);
    const int ACC_FULL = 2 * S, ACC_EMPTY = 2 * S + 2, FINAL = 2 * S + 4;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // this CTA's run of units and the tile it starts in
    const int64_t U = static_cast<int64_t>(p.F / BF) * p.chunks;
    const int64_t u0 = static_cast<int64_t>(blockIdx.x) * U / gridDim.x;
    const int64_t u1 = static_cast<int64_t>(blockIdx.x + 1) * U / gridDim.x;
    const int nk = static_cast<int>(u1 - u0);
    const int t_first = static_cast<int>(u0 / p.chunks);
    const int nchunk = p.NBW / 64;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(bar(i), 1);
            mbar_init(bar(S + i), 1 + (p.amax_out ? 4 : 0));  // MMA commit (+ 4 max warps)
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(ACC_FULL + b), 1);   // the MMA issuer's commit after a segment's last unit
            mbar_init(bar(ACC_EMPTY + b), 4);  // the four drain warps
        }
        mbar_init(bar(FINAL), 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmP);
        tma_prefetch_desc(&tmV);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), 2 * p.tmem_cols);  // two accumulators
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
                const int64_t u = u0 + k;
                const int f0 = static_cast<int>(u / p.chunks) * BF;
                const int mm = static_cast<int>(u % p.chunks) * BMT;
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
            int seg = 0;  // segment of this CTA the next unit belongs to
            for (int k = 0; k < nk; ++k) {
                const int s = k % S;
                const int64_t u = u0 + k;
                const bool first = k == 0 || u % p.chunks == 0;
                const bool last = k == nk - 1 || (u + 1) % p.chunks == 0;
                if (first && k > 0) ++seg;
                const uint32_t acc = tmem + static_cast<uint32_t>(seg & 1) * p.tmem_cols;
                // a buffer is reused two segments later, once its drain has finished
                if (first && seg >= 2 &&
                    !mbar_wait(bar(ACC_EMPTY + (seg & 1)), ((seg >> 1) - 1) & 1, abort_flag, p.status))
                    break;
                if (!mbar_wait(bar(s), (k / S) & 1, abort_flag, p.status)) break;
                tc_fence_after();
                const uint32_t st = base_u32 + s * L.stage_bytes;
                // MN-major, 128-byte swizzle: 8-token groups 1024 B apart (SBO); the two
                // 64-feature halves of A (and the 64-column chunks of V) 8 KB apart (LBO).
                const uint64_t ad = sdesc_mnmajor_sw128(st, A_BYTES / 2, 1024);
                const uint64_t bd = sdesc_mnmajor_sw128(st + A_BYTES, BMT * 128, 1024);
#pragma unroll
                for (int i = 0; i < BMT / 16; ++i)  // 16 tokens per MMA = two 8-row groups
                    mma_bf16(acc, ad + (2048 >> 4) * i, bd + (2048 >> 4) * i, idesc, !first || i != 0);
                tc_commit(bar(S + s));
                if (last) tc_commit(bar(ACC_FULL + (seg & 1)));
            }
            tc_commit(bar(FINAL));
            volatile int no_abort = 0;
            mbar_wait(bar(FINAL), 0, &no_abort, p.status);
        }
    } else {
        // ---------------------------------------------------------------- max + drains
        const int q = warp & 3;  // the TMEM lane quarter this warp reads: features 32 q ..
        // a finished segment: its 128 features x NBW sums go to partial slot blockIdx.x + t
        auto drain = [&](int seg) -> bool {
            if (!mbar_wait(bar(ACC_FULL + (seg & 1)), (seg >> 1) & 1, abort_flag, p.status)) return false;
            tc_fence_after();
            const int64_t slot = static_cast<int64_t>(blockIdx.x) + t_first + seg;
            float* dst = p.partial + (slot * BF + 32 * q + lane) * p.NBW;
            const uint32_t acc = tmem + static_cast<uint32_t>(seg & 1) * p.tmem_cols;
            for (int c = 0; c < p.NBW; c += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(acc + (static_cast<uint32_t>(32 * q) << 16) + c, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4*>(dst + c + e) =
                        make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                    __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(ACC_EMPTY + (seg & 1)));
            return true;
        };
        float m = 0.0f;
        const int t = threadIdx.x - 64;  // 0..127
        int seg = 0;
        for (int k = 0; k < nk; ++k) {
            const int64_t u = u0 + k;
            if (p.amax_out) {
                // max |x| of each landed P tile (16 KB: 8 x 16 bytes per thread), fp32 fmaxf
                // as in amax_kernel (a NaN never wins); the stage is released after the read
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
            if (k == nk - 1 || (u + 1) % p.chunks == 0) {
                if (!drain(seg)) break;
                ++seg;
            }
        }
        if (p.amax_out) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) atomicMax(p.amax_out, __float_as_uint(m));
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 2 * p.tmem_cols);
}

// The split sums in a launch of their own (when the dX GEMM's epilogue warps could not
// finish them within its first tile): the same routine, so the same sums bit for bit.
__global__ void lora_grad_finalize_kernel(const LoraFinalizeJob j0, const LoraFinalizeJob j1) {
    pdl_trigger();
    pdl_wait();
    lora_split_sums(j0, j1, blockIdx.x * blockDim.x + threadIdx.x, gridDim.x * blockDim.x);
}

}  // namespace lg

int lora_grad_ctas(int64_t M, int64_t F, int num_sms) {
    // one persistent CTA per SM (at most kMaxSms, which the workspace query assumes), never
    // more than there are units
    if (num_sms > 160) num_sms = 160;
    const int64_t units = (F / lg::BF) * (M / lg::BMT);
    return static_cast<int>(units < num_sms ? units : num_sms);
}

cudaError_t launch_lora_grad(const CUtensorMap& tmP, const CUtensorMap& tmV, const LoraGradArgs& a, int ctas,
                             int kind, cudaStream_t stream) {
    const lg::Layout L = lg::layout_for(a.NBW);
    // the opt-in limit is raised once to the device maximum (no per-launch host calls)
    static const cudaError_t attr = cudaFuncSetAttribute(
        lg::lora_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
    if (attr != cudaSuccess) return attr;
    dim3 grid(static_cast<unsigned>(ctas));
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
