// Small reductions that run on otherwise idle threads of a later, larger kernel instead
// of in a launch of their own (a launch of latency-bound work costs its full duration
// on the step's critical path even with programmatic dependent launch).
#pragma once
#include "ft_internal.h"

namespace ft {

// The adapter gradients' split sums (FourTune, arXiv 2607.05711, section 3.2: dA and dB
// are the only weight gradients).  A tile t < full_tiles has one slot (t); a later tile
// has rem_splits slots, full_tiles + s * rem_tiles + (t - full_tiles) for token range s
// (LoraSchedule in ft_internal.h).  Then
//   out = s * sum over the tile's slots, in token order, of (D[f][j] + D[f][r + j])
// stored as out[f][j], or out[j][f] with transpose_out.  Thread `worker` of `nworkers`
// takes every nworkers-th block of 4 features x 4 columns of the two jobs (j.out ==
// nullptr: no job): per slot it issues eight independent 16-byte loads (four features'
// high and low halves), and it stores 16-byte rows (along j for out[f][j], along f for
// out[j][f]).  The sums are those of a separate pass bit for bit.
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
        int slot0, nslots, slot_step;
        if (t < jb.full_tiles) {
            slot0 = t;
            nslots = 1;
            slot_step = 0;
        } else {
            slot0 = t;  // full_tiles + 0 * rem_tiles + (t - full_tiles)
            nslots = jb.rem_splits;
            slot_step = jb.rem_tiles;
        }
        const int64_t slot_stride = static_cast<int64_t>(128) * jb.NBW;
        const float* d0 = jb.partial + (static_cast<int64_t>(slot0) * 128 + (f & 127)) * jb.NBW + j;
        float v[4][4];  // [feature f + a][column j + b]
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) v[a][b] = 0.0f;
        for (int k = 0; k < nslots; ++k) {
            const float* d = d0 + static_cast<int64_t>(k) * slot_step * slot_stride;
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
