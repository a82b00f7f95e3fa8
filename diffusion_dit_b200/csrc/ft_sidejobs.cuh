// Small reductions that run on otherwise idle threads of a later, larger kernel instead
// of in a launch of their own (a launch of latency-bound work costs its full duration
// on the step's critical path even with programmatic dependent launch).
#pragma once
#include "ft_internal.h"

namespace ft {

// The adapter gradients' split sums (FourTune, arXiv 2607.05711, section 3.2: dA and dB
// are the only weight gradients): for output (f, j) of tile t = f / 128, the CTAs p that
// covered tile t are those whose unit runs [p U / P, (p + 1) U / P) meet
// [t C, (t + 1) C) (C = chunks, U = (F / 128) C, P = ctas): p_lo .. p_hi below, in token
// order, each with its slot p + t;
//   out = s * sum over them, in order, of (D[f][j] + D[f][r + j])
// stored as out[f][j], or out[j][f] with transpose_out.  Thread `worker` of `nworkers`
// takes every nworkers-th block of 4 features x 4 columns of the two jobs (j.out ==
// nullptr: no job): per slot it issues eight independent 16-byte loads (four features'
// high and low halves), so an output costs a fraction of an L2 round trip, and it stores
// 16-byte rows (along j for out[f][j], along f for out[j][f]).  The sums are those of a
// separate pass bit for bit.
__device__ __forceinline__ void lora_split_sums(const LoraFinalizeJob& j0, const LoraFinalizeJob& j1,
                                                int worker, int nworkers) {
    const int n0 = j0.out ? (j0.F / 4) * (j0.r / 4) : 0;
    const int total = n0 + (j1.out ? (j1.F / 4) * (j1.r / 4) : 0);
    for (int i = worker; i < total; i += nworkers) {
        const LoraFinalizeJob& jb = i < n0 ? j0 : j1;
        const int ii = i < n0 ? i : i - n0;
        const int fq_n = jb.F / 4, jq_n = jb.r / 4;
        int fq, jq;
        if (jb.transpose_out) {  // consecutive workers walk f: coalesced stores into out[j][f]
            jq = ii / fq_n;
            fq = ii - jq * fq_n;
        } else {
            fq = ii / jq_n;
            jq = ii - fq * jq_n;
        }
        const int f = 4 * fq, j = 4 * jq;
        const int t = f >> 7;
        const int64_t P = jb.ctas;
        const int64_t U = static_cast<int64_t>(jb.F >> 7) * jb.chunks;
        // the largest p with p U / P <= x is ceil((x + 1) P / U) - 1
        const int64_t lo_x = static_cast<int64_t>(t) * jb.chunks, hi_x = lo_x + jb.chunks - 1;
        const int p_lo = static_cast<int>(((lo_x + 1) * P + U - 1) / U - 1);
        const int p_hi = static_cast<int>(((hi_x + 1) * P + U - 1) / U - 1);
        const float* d0 = jb.partial + (static_cast<int64_t>(t) * 128 + (f & 127)) * jb.NBW + j;
        const int64_t slot_stride = static_cast<int64_t>(128) * jb.NBW;
        float v[4][4];  // [feature f + a][column j + b]
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) v[a][b] = 0.0f;
        for (int p = p_lo; p <= p_hi; ++p) {
            const float* d = d0 + static_cast<int64_t>(p) * slot_stride;
            float4 h[4], l[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                h[a] = *reinterpret_cast<const float4*>(d + a * jb.NBW);
                l[a] = *reinterpret_cast<const float4*>(d + a * jb.NBW + jb.r);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                v[a][0] += h[a].x + l[a].x;
                v[a][1] += h[a].y + l[a].y;
                v[a][2] += h[a].z + l[a].z;
                v[a][3] += h[a].w + l[a].w;
            }
        }
        if (jb.transpose_out) {
#pragma unroll
            for (int b = 0; b < 4; ++b)
                *reinterpret_cast<float4*>(jb.out + static_cast<int64_t>(j + b) * jb.F + f) =
                    make_float4(v[0][b] * jb.s, v[1][b] * jb.s, v[2][b] * jb.s, v[3][b] * jb.s);
        } else {
#pragma unroll
            for (int a = 0; a < 4; ++a)
                *reinterpret_cast<float4*>(jb.out + static_cast<int64_t>(f + a) * jb.r + j) =
                    make_float4(v[a][0] * jb.s, v[a][1] * jb.s, v[a][2] * jb.s, v[a][3] * jb.s);
        }
    }
}

}  // namespace ft
