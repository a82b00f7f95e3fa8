// The high-precision low-rank branches of the triple-branch linear and the adapter
// gradients (FourTune, arXiv 2607.05711, Eq. (2)-(3) and section 3.2):
//   forward   T = X [Ls_down; A]^T                  (down-projection, fp32)
//   backward  U = G [Ls_up, B]                      (down-projection of the gradient)
//             dB = s G^T T_lora,  dA = s U_lora^T X  (weight gradients, adapter only)
// and the concatenated factors the FP4 GEMM's low-rank tail multiplies by.
//
// The down-projections themselves run on the tensor cores inside the fused quantizer
// (ft_quant_fused.cu) and the adapter gradients in ft_lora_grad.cu; this file sums the
// down-projection's per-slice partials in a fixed order and builds the concatenated
// factors.  The split sum also emits the GEMM's low-rank operand:
//   cat[m, :] = [ hi(g v'(m, :)), lo(g v'(m, :)), 0 ... ]   bf16,  width KL,
// where v' is the product with the LoRA columns (>= r_s) scaled by s, g = g_a g_b is
// the product of the two tensor factors of the following 4-bit GEMM, hi = bf16(.) and
// lo = bf16(. - hi): hi + lo carries ~16 mantissa bits, so multiplying both by the same
// bf16 factor keeps the branch far more precise than the bf16 output it feeds.
#include "ft_internal.h"
#include "ft_ptx.cuh"

namespace ft {
namespace {

// One thread per (row, 4 consecutive j < R): fixed-order sum over the splits (16-byte
// loads), then the hi/lo operands (8-byte stores).  R, r_s and Rp are multiples of 8, so
// a group of four never straddles the stabilizer / adapter boundary.
__device__ __forceinline__ uint32_t bf16x2_bits(__nv_bfloat16 lo, __nv_bfloat16 hi) {
    return static_cast<uint32_t>(__bfloat16_as_ushort(lo)) | (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
}

__global__ void lowrank_finalize_kernel(const LowRankFinalizeArgs a) {
    pdl_trigger();
    pdl_wait();
    const int rows = static_cast<int>(a.rows);
    const int R4 = a.R / 4;
    const int total = rows * R4;
    const float g = (a.cat != nullptr) ? __fmul_rn(*a.ga, *a.gb) : 1.0f;
    const int r = a.R - a.r_s;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
        const int m = i / R4;
        const int j = (i - m * R4) * 4;
        float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int sp = 0; sp < a.splits; ++sp) {
            const float4 pv =
                *reinterpret_cast<const float4*>(a.partial + (static_cast<int64_t>(sp) * rows + m) * a.Rp + j);
            v[0] += pv.x;
            v[1] += pv.y;
            v[2] += pv.z;
            v[3] += pv.w;
        }
        if (a.out) *reinterpret_cast<float4*>(a.out + static_cast<int64_t>(m) * a.R + j) = make_float4(v[0], v[1], v[2], v[3]);
        if (a.cat) {
            __nv_bfloat16 hi[4], lo[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float vs = (j >= a.r_s) ? __fmul_rn(v[q], a.s) : v[q];
                const float gv = __fmul_rn(vs, g);
                hi[q] = __float2bfloat16_rn(gv);
                lo[q] = __float2bfloat16_rn(gv - __bfloat162float(hi[q]));
            }
            __nv_bfloat16* row = a.cat + static_cast<int64_t>(m) * a.KL;
            *reinterpret_cast<uint2*>(row + j) = make_uint2(bf16x2_bits(hi[0], hi[1]), bf16x2_bits(hi[2], hi[3]));
            *reinterpret_cast<uint2*>(row + a.R + j) = make_uint2(bf16x2_bits(lo[0], lo[1]), bf16x2_bits(lo[2], lo[3]));
            if (j < a.KL - 2 * a.R) *reinterpret_cast<uint2*>(row + 2 * a.R + j) = make_uint2(0u, 0u);
        }
        if (a.lora_cat && j >= a.r_s) {  // adapter-gradient operand [hi(v), lo(v), 0] of the LoRA columns
            const int c = j - a.r_s;
            __nv_bfloat16 hi[4], lo[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                hi[q] = __float2bfloat16_rn(v[q]);
                lo[q] = __float2bfloat16_rn(v[q] - __bfloat162float(hi[q]));
            }
            __nv_bfloat16* row = a.lora_cat + static_cast<int64_t>(m) * a.NBW;
            *reinterpret_cast<uint2*>(row + c) = make_uint2(bf16x2_bits(hi[0], hi[1]), bf16x2_bits(hi[2], hi[3]));
            *reinterpret_cast<uint2*>(row + r + c) = make_uint2(bf16x2_bits(lo[0], lo[1]), bf16x2_bits(lo[2], lo[3]));
            for (int z = 2 * r + c; z < a.NBW; z += r) *reinterpret_cast<uint2*>(row + z) = make_uint2(0u, 0u);
        }
    }
    if (a.cat && a.KL - 2 * a.R > a.R) {  // zero padding wider than R columns
        const int w = a.KL - 2 * a.R;
        for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < rows * w; i += gridDim.x * blockDim.x)
            a.cat[(i / w) * a.KL + 2 * a.R + (i % w)] = __float2bfloat16_rn(0.0f);
    }
}

// Shared tile of the transposed factor pieces: 64 rows of up to 256 + 8 bf16, or up to
// 256 rows of 64 + 8 (r_s + r <= 256).
constexpr int kTransposeSmemElems = 256 * 72 > 64 * 264 ? 256 * 72 : 64 * 264;

// Concatenated factors, per call (A and B change every optimizer step):
//   dn     [Rp, K] = [Ls_down; A; 0]
//   upcat  [N, KL] = [Up, Up, 0]     with Up = [Ls_up, B]   (forward GEMM B operand)
//   upt    [Rp, N] = [Up^T; 0]                                  (backward down-projection)
//   dntcat [K, KL] = [Dn^T, Dn^T, 0]                        (backward GEMM B operand)
__global__ void build_factors_kernel(const __nv_bfloat16* __restrict__ ls_down,
                                     const __nv_bfloat16* __restrict__ lora_a,
                                     const __nv_bfloat16* __restrict__ ls_up,
                                     const __nv_bfloat16* __restrict__ lora_b, int N, int K, int r_s,
                                     int r, int Rp, int KL, __nv_bfloat16* __restrict__ dn,
                                     __nv_bfloat16* __restrict__ upcat, __nv_bfloat16* __restrict__ upt,
                                     __nv_bfloat16* __restrict__ dntcat, const PrologueExtras x) {
    pdl_trigger();
    pdl_wait();
    // With the tensor-max job the CTAs split the work: the first kFactorCtas build the
    // factors (and run the side jobs), the others stream the input for its max, so the two
    // latency-bound halves overlap instead of running one after the other in each thread.
    const bool max_job = x.max_src != nullptr;
    const int fctas = max_job ? kFactorCtas : static_cast<int>(gridDim.x);
    if (max_job && static_cast<int>(blockIdx.x) >= fctas) {
        // max |x| of the call's input, one partial per CTA; a dense matrix (row stride ==
        // columns, as the layer calls pass it) is one flat run of 16-byte vectors
        const int64_t vpr = x.max_cols / 8;
        const int64_t nvec = x.max_rows * vpr;
        const int64_t gstride = static_cast<int64_t>(gridDim.x - fctas) * blockDim.x;
        float m = 0.0f;
        auto vmax = [&](const uint4& u) {
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                m = fmaxf(m, fmaxf(fabsf(bf16lo_to_f32(w[e])), fabsf(bf16hi_to_f32(w[e]))));
        };
        const bool flat = x.max_ld == x.max_cols;
        const uint4* flat_src = reinterpret_cast<const uint4*>(x.max_src);
        auto at = [&](int64_t iv) {
            return flat ? flat_src[iv]
                        : *reinterpret_cast<const uint4*>(x.max_src + (iv / vpr) * x.max_ld + (iv % vpr) * 8);
        };
        int64_t i = static_cast<int64_t>(blockIdx.x - fctas) * blockDim.x + threadIdx.x;
        for (; i + 7 * gstride < nvec; i += 8 * gstride) {  // eight independent loads in flight
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = at(i + u * gstride);
#pragma unroll
            for (int u = 0; u < 8; ++u) vmax(v[u]);
        }
        for (; i < nvec; i += gstride) vmax(at(i));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        __shared__ float red[8];
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
        __syncthreads();
        if (threadIdx.x == 0) {
            float v = 0.0f;
            for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) v = fmaxf(v, red[w]);
            x.max_parts[blockIdx.x] = v;
        }
        return;
    }
    if (max_job && threadIdx.x == 0) x.max_parts[blockIdx.x] = 0.0f;  // a factor CTA's partial

    const int R = r_s + r;
    const int stride = fctas * blockDim.x;
    const int t0 = blockIdx.x * blockDim.x + threadIdx.x;
    auto pack8 = [](const __nv_bfloat16 (&e)[8]) {
        uint4 v;
        v.x = static_cast<uint32_t>(__bfloat16_as_ushort(e[0])) | (static_cast<uint32_t>(__bfloat16_as_ushort(e[1])) << 16);
        v.y = static_cast<uint32_t>(__bfloat16_as_ushort(e[2])) | (static_cast<uint32_t>(__bfloat16_as_ushort(e[3])) << 16);
        v.z = static_cast<uint32_t>(__bfloat16_as_ushort(e[4])) | (static_cast<uint32_t>(__bfloat16_as_ushort(e[5])) << 16);
        v.w = static_cast<uint32_t>(__bfloat16_as_ushort(e[6])) | (static_cast<uint32_t>(__bfloat16_as_ushort(e[7])) << 16);
        return v;
    };
    const __nv_bfloat16 zero = __float2bfloat16_rn(0.0f);
    // Every piece moves 8 elements (16 bytes) per thread and step: r_s, r, K, N and the
    // padded widths are multiples of 8, so a chunk never straddles two sources.
    // The row copies issue four independent 16-byte loads before their stores (a thread's
    // chunks are otherwise one L2 round trip each, one after the other).
    if (dn) {
        const int kc = K / 8;
        const int total = Rp * kc;
        for (int i0 = t0; i0 < total; i0 += 4 * stride) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * stride;
                v[u] = make_uint4(0, 0, 0, 0);
                if (i < total) {
                    const int j = i / kc, k = (i % kc) * 8;
                    if (j < r_s) v[u] = *reinterpret_cast<const uint4*>(ls_down + j * K + k);
                    else if (j < R) v[u] = *reinterpret_cast<const uint4*>(lora_a + (j - r_s) * K + k);
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * stride;
                if (i < total) *reinterpret_cast<uint4*>(dn + (i / kc) * K + (i % kc) * 8) = v[u];
            }
        }
    }
    if (upcat) {
        const int cc = KL / 8;
        const int total = N * cc;
        for (int i0 = t0; i0 < total; i0 += 4 * stride) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * stride;
                v[u] = make_uint4(0, 0, 0, 0);
                if (i < total) {
                    const int n = i / cc;
                    int c = (i % cc) * 8;
                    if (c < 2 * R) {
                        if (c >= R) c -= R;
                        v[u] = c < r_s ? *reinterpret_cast<const uint4*>(ls_up + n * r_s + c)
                                       : *reinterpret_cast<const uint4*>(lora_b + n * r + (c - r_s));
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * stride;
                if (i < total) *reinterpret_cast<uint4*>(upcat + (i / cc) * KL + (i % cc) * 8) = v[u];
            }
        }
    }
    // Transposed pieces, through shared memory in tiles of 64 rows: each tile is read with
    // 16-byte loads along its source rows and written with 16-byte stores along the
    // destination rows (a thread gathers its 8 elements from the shared tile), so both
    // sides stay coalesced.  One tile per CTA and trip; upt's tiles come first.
    //   upt    [Rp, N] = [Up^T; 0]           from Up [N, R] = [Ls_up | B]
    //   dntcat [K, KL] = [Dn^T, Dn^T, 0]     from Dn [R, K] = [Ls_down; A]
    __shared__ __align__(16) __nv_bfloat16 tsm[kTransposeSmemElems];
    const int upt_tiles = upt ? N / 64 : 0;
    const int dnt_tiles = dntcat ? K / 64 : 0;
    for (int tile = blockIdx.x; tile < upt_tiles + dnt_tiles; tile += fctas) {
        __syncthreads();  // the previous tile's reads of tsm are done
        if (tile < upt_tiles) {
            const int n0 = tile * 64;
            const int ld = R + 8;  // tsm[n][j], padded rows
            const int rc = R / 8;
            for (int i = threadIdx.x; i < 64 * rc; i += blockDim.x) {
                const int n = i / rc, c = (i % rc) * 8;
                const uint4 v = c < r_s ? *reinterpret_cast<const uint4*>(ls_up + (n0 + n) * r_s + c)
                                        : *reinterpret_cast<const uint4*>(lora_b + (n0 + n) * r + (c - r_s));
                *reinterpret_cast<uint4*>(tsm + n * ld + c) = v;
            }
            __syncthreads();
            for (int i = threadIdx.x; i < Rp * 8; i += blockDim.x) {
                const int j = i / 8, n = (i % 8) * 8;
                __nv_bfloat16 e[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) e[q] = j < R ? tsm[(n + q) * ld + j] : zero;
                *reinterpret_cast<uint4*>(upt + j * N + n0 + n) = pack8(e);
            }
        } else {
            const int k0 = (tile - upt_tiles) * 64;
            const int ld = 64 + 8;  // tsm[j][k], padded rows
            for (int i = threadIdx.x; i < R * 8; i += blockDim.x) {
                const int j = i / 8, k = (i % 8) * 8;
                const uint4 v = j < r_s ? *reinterpret_cast<const uint4*>(ls_down + j * K + k0 + k)
                                        : *reinterpret_cast<const uint4*>(lora_a + (j - r_s) * K + k0 + k);
                *reinterpret_cast<uint4*>(tsm + j * ld + k) = v;
            }
            __syncthreads();
            const int cc = KL / 8;
            for (int i = threadIdx.x; i < 64 * cc; i += blockDim.x) {
                const int k = i / cc, c = (i % cc) * 8;
                __nv_bfloat16 e[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int cq = c + q;
                    e[q] = cq < R ? tsm[cq * ld + k] : (cq < 2 * R ? tsm[(cq - R) * ld + k] : zero);
                }
                *reinterpret_cast<uint4*>(dntcat + (k0 + k) * KL + c) = pack8(e);
            }
        }
    }
    // side jobs: V' = [hi(V), lo(V), 0] for dB (8 columns per thread: one group of hi, of
    // lo, or of zeros, since r is a multiple of 8), and the cleared tensor-max slots
    if (x.hilo_dst) {
        const int w = x.hilo_NBW, rr = x.hilo_r;
        const int wc = w / 8;
        for (int i = t0; i < x.hilo_M * wc; i += stride) {
            const int m = i / wc, c = (i - m * wc) * 8;
            uint4 o = make_uint4(0, 0, 0, 0);
            if (c < 2 * rr) {
                const int cs = c < rr ? c : c - rr;
                const float* src = x.hilo_src + static_cast<int64_t>(m) * x.hilo_ld + x.hilo_c0 + cs;
                const float4 a = *reinterpret_cast<const float4*>(src);
                const float4 b = *reinterpret_cast<const float4*>(src + 4);
                const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                __nv_bfloat16 e[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const __nv_bfloat16 hi = __float2bfloat16_rn(v[q]);
                    e[q] = c < rr ? hi : __float2bfloat16_rn(v[q] - __bfloat162float(hi));
                }
                o = pack8(e);
            }
            *reinterpret_cast<uint4*>(x.hilo_dst + static_cast<int64_t>(m) * w + c) = o;
        }
    }
    if (x.zero_slot && t0 == 0) *x.zero_slot = 0.0f;
    if (x.zero_slot2 && t0 == 0) *x.zero_slot2 = 0.0f;
}

}  // namespace

static int grid_cap(int64_t work, int threads, int cap) {
    int64_t g = (work + threads - 1) / threads;
    if (g < 1) g = 1;
    if (g > cap) g = cap;
    return static_cast<int>(g);
}

cudaError_t launch_lowrank_finalize(const LowRankFinalizeArgs& a, cudaStream_t stream) {
    before_launch(K_LOWRANK, stream);
    const cudaError_t le = launch_k(lowrank_finalize_kernel,
                                    dim3(grid_cap(a.rows * (a.R / 4), 256, 148 * 8)), dim3(256), 0,
                                    stream, a);
    if (le != cudaSuccess) return le;
    after_launch(K_LOWRANK, stream);
    return cudaGetLastError();
}

cudaError_t launch_build_factors(const __nv_bfloat16* ls_down, const __nv_bfloat16* lora_a,
                                 const __nv_bfloat16* ls_up, const __nv_bfloat16* lora_b, int64_t N,
                                 int64_t K, int r_s, int r, int Rp, int KL, __nv_bfloat16* dn,
                                 __nv_bfloat16* upcat, __nv_bfloat16* upt, __nv_bfloat16* dntcat,
                                 const PrologueExtras* extra, cudaStream_t stream) {
    const PrologueExtras x = extra ? *extra : PrologueExtras{};
    // with the tensor-max job the launch is the call's max pass (timed as such)
    const int kind = x.max_src ? K_AMAX : K_OTHER;
    before_launch(kind, stream);
    const cudaError_t le = launch_k(build_factors_kernel, dim3(kPrologueCtas), dim3(256), 0, stream,
                                    ls_down, lora_a, ls_up, lora_b, static_cast<int>(N),
                                    static_cast<int>(K), r_s, r, Rp, KL, dn, upcat, upt, dntcat, x);
    if (le != cudaSuccess) return le;
    after_launch(kind, stream);
    return cudaGetLastError();
}

}  // namespace ft
