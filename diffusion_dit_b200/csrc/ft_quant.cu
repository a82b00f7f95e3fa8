// The 16x16-block NVFP4 quantizer Q(.) and its helpers.
//
// FourTune (arXiv 2607.05711): section 2.3 (Round(W / s) with a scale s), section 3.1
// (NVFP4 for the frozen residual and the activations), section 3.2 and Table 5 (16x16
// blocks, so that the transposed matrix reuses the same codes and scales).  The
// arithmetic, fixed here so results are reproducible bit for bit:
//   g     = fl32(2688 / amax_t)       (g = 1 and all-zero output if amax_t == 0 or g is
//                                       not finite)
//   sb    = UE4M3_rn_satfinite( fl32( fl32(amax_b / 6) * g ) )
//   inv   = fl32(g / val(sb))
//   code  = E2M1_rn_satfinite( fl32(x * inv) )  with the sign bit of x; 0 when sb == 0
// Every fp32 operation is an explicitly rounded intrinsic (__fdiv_rn / __fmul_rn).
#include "ft_internal.h"
#include "ft_ptx.cuh"

namespace ft {

namespace {

__device__ __forceinline__ void tensor_scale(float amax, float& g, bool& degenerate) {
    g = 1.0f;
    degenerate = true;
    if (amax > 0.0f) {
        const float gg = __fdiv_rn(2688.0f, amax);
        if (isfinite(gg) && gg > 0.0f) {
            g = gg;
            degenerate = false;
        }
    }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Loads 8 consecutive elements as fp32.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    v[0] = bf16lo_to_f32(w.x); v[1] = bf16hi_to_f32(w.x);
    v[2] = bf16lo_to_f32(w.y); v[3] = bf16hi_to_f32(w.y);
    v[4] = bf16lo_to_f32(w.z); v[5] = bf16hi_to_f32(w.z);
    v[6] = bf16lo_to_f32(w.w); v[7] = bf16hi_to_f32(w.w);
}

__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// ---------------------------------------------------------------------------
// amax_t = max |x|: per-thread max over 8-element vectors, warp/CTA reduction, one
// atomicMax per CTA on the bit pattern (valid ordering for non-negative floats).
template <typename T>
__global__ void __launch_bounds__(256) amax_kernel(const T* __restrict__ x, int64_t rows, int64_t cols,
                                                   int64_t ld, unsigned* __restrict__ out) {
    pdl_trigger();
    pdl_wait();
    const int64_t vec_per_row = cols / 8;
    const int64_t nvec = rows * vec_per_row;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    float m = 0.0f;
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    // a dense matrix (ld == cols) is one flat run of 8-element vectors: no index division
    const bool flat = ld == cols;
    auto at = [&](int64_t iv) { return flat ? x + iv * 8 : x + (iv / vec_per_row) * ld + (iv % vec_per_row) * 8; };
    // four independent 8-element loads in flight per thread per trip
    for (; i + 3 * stride < nvec; i += 4 * stride) {
        float v[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u) load8(at(i + u * stride), v[u]);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[u][j]));
    }
    for (; i < nvec; i += stride) {
        float v[8];
        load8(at(i), v);
#pragma unroll
        for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
    }
    m = warp_max(m);
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
        v = warp_max(v);
        if (threadIdx.x == 0) atomicMax(out, __float_as_uint(v));
    }
}

// ---------------------------------------------------------------------------
// One warp per 16x16 block: lane l holds row l/2, columns 8 (l%2) .. +7 of the block.
template <typename T>
__global__ void __launch_bounds__(256) quant_block16_kernel(const T* __restrict__ x, int64_t rows,
                                                            int64_t cols, int64_t ld,
                                                            const float* __restrict__ amax_ptr,
                                                            uint8_t* __restrict__ codes,
                                                            uint8_t* __restrict__ scales,
                                                            float* __restrict__ g_out) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t nbc = cols / 16;
    const int64_t nblocks = (rows / 16) * nbc;
    float g;
    bool degenerate;
    tensor_scale(*amax_ptr, g, degenerate);
    if (blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;
    const int r = lane >> 1, h = lane & 1;
    const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t b = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); b < nblocks;
         b += warps_total) {
        const int64_t bi = b / nbc, bj = b % nbc;
        const int64_t row = bi * 16 + r, col = bj * 16 + 8 * h;
        float v[8];
        load8(x + row * ld + col, v);
        float am = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) am = fmaxf(am, fabsf(v[j]));
        am = warp_max(am);
        uint32_t sb = 0, packed = 0;
        if (!degenerate) {
            sb = cvt_ue4m3(__fmul_rn(__fdiv_rn(am, 6.0f), g));
            if (sb != 0) {
                const float inv = __fdiv_rn(g, ue4m3_to_f32(sb));
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    packed |= cvt_e2m1x2(__fmul_rn(v[2 * j], inv), __fmul_rn(v[2 * j + 1], inv))
                              << (8 * j);
            }
        }
        *reinterpret_cast<uint32_t*>(codes + row * (cols / 2) + col / 2) = packed;
        if (lane == 0) scales[bi * nbc + bj] = static_cast<uint8_t>(sb);
    }
}

// Tensor-core scale layout: one byte per (row, 16 columns), 512-byte atoms covering
// 128 rows x 64 columns, atoms of a 128-row band consecutive along the columns; in an
// atom, (row m, column block b) sits at 16 (m % 32) + 4 ((m % 128) / 32) + b % 4.
__global__ void expand_scales_kernel(const uint8_t* __restrict__ scales, int64_t rows, int64_t cols,
                                     uint8_t* __restrict__ sf) {
    pdl_trigger();
    pdl_wait();
    const int64_t total = rows * (cols / 16);
    const int64_t atoms_per_band = cols / 64;
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total;
         o += (int64_t)gridDim.x * blockDim.x) {
        const int64_t atom = o / 512;
        const int within = static_cast<int>(o % 512);
        const int64_t band = atom / atoms_per_band, cb4 = atom % atoms_per_band;
        const int m = (within / 16) + 32 * ((within % 16) / 4);
        const int64_t row = band * 128 + m;
        const int64_t cblk = cb4 * 4 + (within % 4);
        sf[o] = scales[(row / 16) * (cols / 16) + cblk];
    }
}

// Q^T from Q without requantization: code (i, j) -> (j, i); block scale (a, b) -> (b, a).
__global__ void transpose_q_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                   int64_t rows, int64_t cols, uint8_t* __restrict__ codes_t,
                                   uint8_t* __restrict__ scales_t) {
    pdl_trigger();
    pdl_wait();
    // output codes_t [cols, rows/2]
    const int64_t total = cols * (rows / 2);
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total;
         o += (int64_t)gridDim.x * blockDim.x) {
        const int64_t a = o / (rows / 2);        // output row = input column
        const int64_t b2 = (o % (rows / 2)) * 2; // output column pair = input rows b2, b2+1
        const int shift = (a & 1) ? 4 : 0;
        const uint32_t lo = (codes[b2 * (cols / 2) + a / 2] >> shift) & 15u;
        const uint32_t hi = (codes[(b2 + 1) * (cols / 2) + a / 2] >> shift) & 15u;
        codes_t[o] = static_cast<uint8_t>(lo | (hi << 4));
    }
    const int64_t nsc = (rows / 16) * (cols / 16);
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < nsc;
         o += (int64_t)gridDim.x * blockDim.x) {
        const int64_t bt = o / (rows / 16), at = o % (rows / 16);  // scales_t[bt][at]
        scales_t[o] = scales[at * (cols / 16) + bt];
    }
}

__global__ void copy_scalar_kernel(const float* src, float* dst) {
    pdl_trigger();
    pdl_wait();
    *dst = *src;
}

__global__ void encode_e2m1_kernel(const float* __restrict__ v, int64_t n, uint8_t* __restrict__ out) {
    pdl_trigger();
    pdl_wait();
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        out[i] = static_cast<uint8_t>(cvt_e2m1x2(v[i], 0.0f) & 15u);
}

__global__ void encode_ue4m3_kernel(const float* __restrict__ v, int64_t n, uint8_t* __restrict__ out) {
    pdl_trigger();
    pdl_wait();
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        out[i] = static_cast<uint8_t>(cvt_ue4m3(v[i]));
}

// The stand-alone GELU passes compute with the same pair functions as the GEMM epilogues
// (gelu_bf16x2, gelu_bwd_bf16x2), so the unfused and fused MLP paths agree bit for bit.
__global__ void gelu_fwd_kernel(const __nv_bfloat16* __restrict__ p, __nv_bfloat16* __restrict__ h,
                                int64_t n) {
    pdl_trigger();
    pdl_wait();
    float unused_max = 0.0f;
    for (int64_t i = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) * 8; i < n;
         i += (int64_t)gridDim.x * blockDim.x * 8) {
        const uint4 w = *reinterpret_cast<const uint4*>(p + i);
        *reinterpret_cast<uint4*>(h + i) = make_uint4(gelu_bf16x2(w.x, unused_max), gelu_bf16x2(w.y, unused_max),
                                                      gelu_bf16x2(w.z, unused_max), gelu_bf16x2(w.w, unused_max));
    }
}

__global__ void gelu_bwd_kernel(const __nv_bfloat16* __restrict__ p, const __nv_bfloat16* __restrict__ dh,
                                __nv_bfloat16* __restrict__ dp, int64_t n) {
    pdl_trigger();
    pdl_wait();
    for (int64_t i = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) * 8; i < n;
         i += (int64_t)gridDim.x * blockDim.x * 8) {
        const uint4 w = *reinterpret_cast<const uint4*>(p + i);
        const uint4 d = *reinterpret_cast<const uint4*>(dh + i);
        *reinterpret_cast<uint4*>(dp + i) = make_uint4(gelu_bwd_bf16x2(d.x, w.x), gelu_bwd_bf16x2(d.y, w.y),
                                                       gelu_bwd_bf16x2(d.z, w.z), gelu_bwd_bf16x2(d.w, w.w));
    }
}

int grid_for(int64_t work, int threads, int cap) {
    int64_t g = (work + threads - 1) / threads;
    if (g < 1) g = 1;
    if (g > cap) g = cap;
    return static_cast<int>(g);
}

}  // namespace

cudaError_t launch_amax(const void* x, bool is_f32, int64_t rows, int64_t cols, int64_t ld,
                        float* amax_out, bool slot_cleared, int num_sms, cudaStream_t stream) {
    if (!slot_cleared) {
        const cudaError_t e = cudaMemsetAsync(amax_out, 0, sizeof(float), stream);
        if (e != cudaSuccess) return e;
    }
    const int grid = grid_for(rows * cols / 32, 256, num_sms * 4);
    before_launch(K_AMAX, stream);
    unsigned* out = reinterpret_cast<unsigned*>(amax_out);
    const cudaError_t le =
        is_f32 ? launch_k(amax_kernel<float>, dim3(grid), dim3(256), 0, stream, static_cast<const float*>(x),
                          rows, cols, ld, out)
               : launch_k(amax_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, stream,
                          static_cast<const __nv_bfloat16*>(x), rows, cols, ld, out);
    if (le != cudaSuccess) return le;
    after_launch(K_AMAX, stream);
    return cudaGetLastError();
}

cudaError_t launch_quant_block16(const void* x, bool is_f32, int64_t rows, int64_t cols, int64_t ld,
                                 const float* amax, uint8_t* codes, uint8_t* scales, float* g_out,
                                 int num_sms, cudaStream_t stream) {
    const int64_t nblocks = (rows / 16) * (cols / 16);
    const int grid = grid_for(nblocks * 32, 256, num_sms * 8);
    before_launch(K_QUANT, stream);
    const cudaError_t le =
        is_f32 ? launch_k(quant_block16_kernel<float>, dim3(grid), dim3(256), 0, stream,
                          static_cast<const float*>(x), rows, cols, ld, amax, codes, scales, g_out)
               : launch_k(quant_block16_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, stream,
                          static_cast<const __nv_bfloat16*>(x), rows, cols, ld, amax, codes, scales, g_out);
    if (le != cudaSuccess) return le;
    after_launch(K_QUANT, stream);
    return cudaGetLastError();
}

cudaError_t launch_expand_scales(const uint8_t* scales, int64_t rows, int64_t cols, uint8_t* sf_mma,
                                 cudaStream_t stream) {
    const int grid = grid_for(rows * cols / 16, 256, 148 * 8);
    before_launch(K_OTHER, stream);
    const cudaError_t le = launch_k(expand_scales_kernel, dim3(grid), dim3(256), 0, stream, scales,
                                    rows, cols, sf_mma);
    if (le != cudaSuccess) return le;
    after_launch(K_OTHER, stream);
    return cudaGetLastError();
}

cudaError_t launch_transpose_q(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                               uint8_t* codes_t, uint8_t* scales_t, cudaStream_t stream) {
    const int grid = grid_for(rows * cols / 2, 256, 148 * 8);
    before_launch(K_OTHER, stream);
    const cudaError_t le = launch_k(transpose_q_kernel, dim3(grid), dim3(256), 0, stream, codes,
                                    scales, rows, cols, codes_t, scales_t);
    if (le != cudaSuccess) return le;
    after_launch(K_OTHER, stream);
    return cudaGetLastError();
}

cudaError_t launch_copy_scalar(const float* src, float* dst, cudaStream_t stream) {
    before_launch(K_OTHER, stream);
    const cudaError_t le = launch_k(copy_scalar_kernel, dim3(1), dim3(1), 0, stream, src, dst);
    if (le != cudaSuccess) return le;
    after_launch(K_OTHER, stream);
    return cudaGetLastError();
}

cudaError_t launch_encode_e2m1(const float* v, int64_t n, uint8_t* out, cudaStream_t stream) {
    before_launch(K_OTHER, stream);
    const cudaError_t le = launch_k(encode_e2m1_kernel, dim3(grid_for(n, 256, 148 * 16)), dim3(256),
                                    0, stream, v, n, out);
    if (le != cudaSuccess) return le;
    after_launch(K_OTHER, stream);
    return cudaGetLastError();
}

cudaError_t launch_encode_ue4m3(const float* v, int64_t n, uint8_t* out, cudaStream_t stream) {
    before_launch(K_OTHER, stream);
    const cudaError_t le = launch_k(encode_ue4m3_kernel, dim3(grid_for(n, 256, 148 * 16)),
                                    dim3(256), 0, stream, v, n, out);
    if (le != cudaSuccess) return le;
    after_launch(K_OTHER, stream);
    return cudaGetLastError();
}

cudaError_t launch_gelu_fwd(const __nv_bfloat16* p, __nv_bfloat16* h, int64_t n, cudaStream_t stream) {
    before_launch(K_OTHER, stream);
    const cudaError_t le = launch_k(gelu_fwd_kernel, dim3(grid_for(n / 8, 256, 148 * 8)), dim3(256),
                                    0, stream, p, h, n);
    if (le != cudaSuccess) return le;
    after_launch(K_OTHER, stream);
    return cudaGetLastError();
}

cudaError_t launch_gelu_bwd(const __nv_bfloat16* p, const __nv_bfloat16* dh, __nv_bfloat16* dp,
                            int64_t n, cudaStream_t stream) {
    before_launch(K_OTHER, stream);
    const cudaError_t le = launch_k(gelu_bwd_kernel, dim3(grid_for(n / 8, 256, 148 * 8)), dim3(256),
                                    0, stream, p, dh, dp, n);
    if (le != cudaSuccess) return le;
    after_launch(K_OTHER, stream);
    return cudaGetLastError();
}

}  // namespace ft

namespace ft {
namespace {

// Self-test of the bounded wait every pipelined kernel uses: wait on an mbarrier that
// nothing will ever complete, give up after limit_ns, report FT_ERR_TIMEOUT.
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns, int* status) {
    pdl_trigger();
    pdl_wait();
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, status, limit_ns);
    __syncthreads();
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, int* status, cudaStream_t stream) {
    before_launch(K_OTHER, stream);
    const cudaError_t le = launch_k(bounded_wait_selftest_kernel, dim3(1), dim3(32), 0, stream,
                                    limit_ns, status);
    if (le != cudaSuccess) return le;
    after_launch(K_OTHER, stream);
    return cudaGetLastError();
}

}  // namespace ft
