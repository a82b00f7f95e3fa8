// The high-precision low-rank branches of the triple-branch linear and the adapter
// gradients (FourTune, arXiv 2607.05711, Eq. (2)-(3) and section 3.2):
//   forward   T = X [Ls_down; A]^T                  (down-projection, fp32)
//   backward  U = G [Ls_up, B]                      (down-projection of the gradient)
//             dB = s G^T T_lora,  dA = s U_lora^T X  (weight gradients, adapter only)
// and the concatenated factors the FP4 GEMM's low-rank tail multiplies by.
//
// These kernels accumulate in fp32 on the CUDA cores with a fixed summation order
// (deterministic).  The down-projection also emits the GEMM's low-rank operand:
//   cat[m, :] = [ hi(g v'(m, :)), lo(g v'(m, :)), 0 ... ]   bf16,  width KL,
// where v' is the product with the LoRA columns (>= r_s) scaled by s, g = g_a g_b is
// the product of the two tensor factors of the following 4-bit GEMM, hi = bf16(.) and
// lo = bf16(. - hi): hi + lo carries ~16 mantissa bits, so multiplying both by the same
// bf16 factor keeps the branch far more precise than the bf16 output it feeds.
#include "ft_internal.h"
#include "ft_ptx.cuh"

namespace ft {
namespace {

constexpr int TM = 32;   // rows per CTA
constexpr int TK = 32;   // reduction chunk

// out[m, j] = sum_k x[m, k] w[j, k]; one CTA per 32 rows, all R columns.
__global__ void __launch_bounds__(256) lowrank_down_kernel(const LowRankDownArgs a) {
    extern __shared__ float sh[];
    float* xs = sh;                   // [TM][TK + 1]
    float* wsm = sh + TM * (TK + 1);  // [R][TK + 1]
    const int m0 = blockIdx.x * TM;
    const int tid = threadIdx.x;
    const int R = a.R;
    // each thread owns outputs (row = tid % 32, j = tid / 32 + 8 t)
    const int row = tid & 31;
    const int j0 = tid >> 5;
    constexpr int MAXJ = 32;  // R <= 256
    float acc[MAXJ];
#pragma unroll
    for (int t = 0; t < MAXJ; ++t) acc[t] = 0.0f;
    for (int k0 = 0; k0 < a.K; k0 += TK) {
        for (int i = tid; i < TM * TK; i += blockDim.x) {
            const int r = i / TK, c = i % TK;
            xs[r * (TK + 1) + c] = __bfloat162float(a.x[(int64_t)(m0 + r) * a.ldx + k0 + c]);
        }
        for (int i = tid; i < R * TK; i += blockDim.x) {
            const int r = i / TK, c = i % TK;
            wsm[r * (TK + 1) + c] = __bfloat162float(a.w[(int64_t)r * a.K + k0 + c]);
        }
        __syncthreads();
#pragma unroll
        for (int t = 0; t < MAXJ; ++t) {
            const int j = j0 + 8 * t;
            if (j < R) {
                float s = acc[t];
#pragma unroll 8
                for (int c = 0; c < TK; ++c) s = fmaf(xs[row * (TK + 1) + c], wsm[j * (TK + 1) + c], s);
                acc[t] = s;
            }
        }
        __syncthreads();
    }
    const int64_t m = m0 + row;
    if (!a.cat) {
#pragma unroll
        for (int t = 0; t < MAXJ; ++t) {
            const int j = j0 + 8 * t;
            if (j < R) a.out[m * R + j] = acc[t];
        }
        return;
    }
    const float g = __fmul_rn(*a.ga, *a.gb);
#pragma unroll
    for (int t = 0; t < MAXJ; ++t) {
        const int j = j0 + 8 * t;
        if (j < R) {
            const float v = acc[t];
            if (a.out) a.out[m * R + j] = v;
            const float vs = (j >= a.r_s) ? __fmul_rn(v, a.s) : v;
            const float gv = __fmul_rn(vs, g);
            const __nv_bfloat16 hi = __float2bfloat16_rn(gv);
            const __nv_bfloat16 lo = __float2bfloat16_rn(gv - __bfloat162float(hi));
            a.cat[m * a.KL + j] = hi;
            a.cat[m * a.KL + R + j] = lo;
        }
    }
    for (int j = 2 * R + j0; j < a.KL; j += 8) a.cat[m * a.KL + j] = __float2bfloat16_rn(0.0f);
}

// Concatenated factors, per call (A and B change every optimizer step):
//   dn     [R, K]  = [Ls_down; A]
//   upcat  [N, KL] = [Up, Up, 0]     with Up = [Ls_up, B]   (forward GEMM B operand)
//   upt    [R, N]  = Up^T                                   (backward down-projection)
//   dntcat [K, KL] = [Dn^T, Dn^T, 0]                        (backward GEMM B operand)
__global__ void build_factors_kernel(const __nv_bfloat16* __restrict__ ls_down,
                                     const __nv_bfloat16* __restrict__ lora_a,
                                     const __nv_bfloat16* __restrict__ ls_up,
                                     const __nv_bfloat16* __restrict__ lora_b, int64_t N, int64_t K,
                                     int r_s, int r, int KL, __nv_bfloat16* __restrict__ dn,
                                     __nv_bfloat16* __restrict__ upcat, __nv_bfloat16* __restrict__ upt,
                                     __nv_bfloat16* __restrict__ dntcat) {
    const int R = r_s + r;
    const __nv_bfloat16 zero = __float2bfloat16_rn(0.0f);
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t t0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    auto dn_at = [&](int j, int64_t k) {
        return j < r_s ? ls_down[(int64_t)j * K + k] : lora_a[(int64_t)(j - r_s) * K + k];
    };
    auto up_at = [&](int64_t n, int j) {
        return j < r_s ? ls_up[n * r_s + j] : lora_b[n * r + (j - r_s)];
    };
    if (dn)
        for (int64_t i = t0; i < (int64_t)R * K; i += stride) dn[i] = dn_at(static_cast<int>(i / K), i % K);
    if (upcat)
        for (int64_t i = t0; i < N * KL; i += stride) {
            const int64_t n = i / KL;
            const int c = static_cast<int>(i % KL);
            upcat[i] = c < R ? up_at(n, c) : (c < 2 * R ? up_at(n, c - R) : zero);
        }
    if (upt)
        for (int64_t i = t0; i < (int64_t)R * N; i += stride) upt[i] = up_at(i % N, static_cast<int>(i / N));
    if (dntcat)
        for (int64_t i = t0; i < K * KL; i += stride) {
            const int64_t k = i / KL;
            const int c = static_cast<int>(i % KL);
            dntcat[i] = c < R ? dn_at(c, k) : (c < 2 * R ? dn_at(c - R, k) : zero);
        }
}

// db[n, j] = s sum_m g[m, n] t[m, r_s + j]; one CTA per 64 columns n, fixed m order.
__global__ void __launch_bounds__(256) lora_db_kernel(const __nv_bfloat16* __restrict__ g, int64_t M,
                                                      int64_t N, const float* __restrict__ t, int R,
                                                      int r_s, int r, float s, float* __restrict__ db) {
    extern __shared__ float sh[];
    float* gs = sh;               // [TK][64]
    float* ts = sh + TK * 64;     // [TK][r]
    const int n0 = blockIdx.x * 64;
    const int tid = threadIdx.x;
    const int n = tid & 63;
    const int j0 = tid >> 6;      // 0..3, j = j0 + 4 q
    constexpr int MAXQ = 16;      // r <= 64
    float acc[MAXQ];
#pragma unroll
    for (int q = 0; q < MAXQ; ++q) acc[q] = 0.0f;
    for (int64_t m0 = 0; m0 < M; m0 += TK) {
        for (int i = tid; i < TK * 64; i += blockDim.x)
            gs[i] = __bfloat162float(g[(m0 + i / 64) * N + n0 + (i % 64)]);
        for (int i = tid; i < TK * r; i += blockDim.x) ts[i] = t[(m0 + i / r) * R + r_s + (i % r)];
        __syncthreads();
#pragma unroll
        for (int q = 0; q < MAXQ; ++q) {
            const int j = j0 + 4 * q;
            if (j < r) {
                float a = acc[q];
#pragma unroll 8
                for (int mm = 0; mm < TK; ++mm) a = fmaf(gs[mm * 64 + n], ts[mm * r + j], a);
                acc[q] = a;
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int q = 0; q < MAXQ; ++q) {
        const int j = j0 + 4 * q;
        if (j < r) db[(int64_t)(n0 + n) * r + j] = s * acc[q];
    }
}

// da[j, k] = s sum_m u[m, r_s + j] x[m, k]; one CTA per 64 columns k, fixed m order.
__global__ void __launch_bounds__(256) lora_da_kernel(const float* __restrict__ u, int R, int r_s, int r,
                                                      const __nv_bfloat16* __restrict__ x, int64_t M,
                                                      int64_t K, float s, float* __restrict__ da) {
    extern __shared__ float sh[];
    float* xs = sh;               // [TK][64]
    float* us = sh + TK * 64;     // [TK][r]
    const int k0 = blockIdx.x * 64;
    const int tid = threadIdx.x;
    const int k = tid & 63;
    const int j0 = tid >> 6;
    constexpr int MAXQ = 16;
    float acc[MAXQ];
#pragma unroll
    for (int q = 0; q < MAXQ; ++q) acc[q] = 0.0f;
    for (int64_t m0 = 0; m0 < M; m0 += TK) {
        for (int i = tid; i < TK * 64; i += blockDim.x)
            xs[i] = __bfloat162float(x[(m0 + i / 64) * K + k0 + (i % 64)]);
        for (int i = tid; i < TK * r; i += blockDim.x) us[i] = u[(m0 + i / r) * R + r_s + (i % r)];
        __syncthreads();
#pragma unroll
        for (int q = 0; q < MAXQ; ++q) {
            const int j = j0 + 4 * q;
            if (j < r) {
                float a = acc[q];
#pragma unroll 8
                for (int mm = 0; mm < TK; ++mm) a = fmaf(us[mm * r + j], xs[mm * 64 + k], a);
                acc[q] = a;
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int q = 0; q < MAXQ; ++q) {
        const int j = j0 + 4 * q;
        if (j < r) da[(int64_t)j * K + k0 + k] = s * acc[q];
    }
}

}  // namespace

cudaError_t launch_lowrank_down(const LowRankDownArgs& a, cudaStream_t stream) {
    const size_t smem = sizeof(float) * (TM + a.R) * (TK + 1);
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(lowrank_down_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    before_launch(K_LOWRANK, stream);
    lowrank_down_kernel<<<static_cast<unsigned>(a.M / TM), 256, smem, stream>>>(a);
    after_launch(K_LOWRANK, stream);
    return cudaGetLastError();
}

cudaError_t launch_build_factors(const __nv_bfloat16* ls_down, const __nv_bfloat16* lora_a,
                                 const __nv_bfloat16* ls_up, const __nv_bfloat16* lora_b, int64_t N,
                                 int64_t K, int r_s, int r, int KL, __nv_bfloat16* dn,
                                 __nv_bfloat16* upcat, __nv_bfloat16* upt, __nv_bfloat16* dntcat,
                                 cudaStream_t stream) {
    before_launch(K_OTHER, stream);
    build_factors_kernel<<<148 * 4, 256, 0, stream>>>(ls_down, lora_a, ls_up, lora_b, N, K, r_s, r, KL,
                                                      dn, upcat, upt, dntcat);
    after_launch(K_OTHER, stream);
    return cudaGetLastError();
}

cudaError_t launch_lora_db(const __nv_bfloat16* g, int64_t M, int64_t N, const float* t, int R,
                           int r_s, int r, float s, float* db, cudaStream_t stream) {
    const size_t smem = sizeof(float) * TK * (64 + r);
    before_launch(K_LORA_DB, stream);
    lora_db_kernel<<<static_cast<unsigned>(N / 64), 256, smem, stream>>>(g, M, N, t, R, r_s, r, s, db);
    after_launch(K_LORA_DB, stream);
    return cudaGetLastError();
}

cudaError_t launch_lora_da(const float* u, int R, int r_s, int r, const __nv_bfloat16* x, int64_t M,
                           int64_t K, float s, float* da, cudaStream_t stream) {
    const size_t smem = sizeof(float) * TK * (64 + r);
    before_launch(K_LORA_DA, stream);
    lora_da_kernel<<<static_cast<unsigned>(K / 64), 256, smem, stream>>>(u, R, r_s, r, x, M, K, s, da);
    after_launch(K_LORA_DA, stream);
    return cudaGetLastError();
}

}  // namespace ft
