// Small reductions that run on otherwise idle threads of a later, larger kernel instead
// of in a launch of their own (a launch of latency-bound work costs its full duration
// on the step's critical path even with programmatic dependent launch).
#pragma once
#include "ft_internal.h"

namespace ft {

// The adapter gradients' split sums (FourTune, arXiv 2607.05711, section 3.2: dA and dB
// are the only weight gradients):
//   out = s * sum over the splits, in order, of (D[f][j] + D[f][r + j])
// stored as out[f][j], or out[j][f] with transpose_out.  Thread `worker` of `nworkers`
// takes every nworkers-th output of the two jobs (j.out == nullptr: no job).  A thread
// issues all of an output's loads before adding them in split order, so an output costs
// one L2 round trip, and the sums are those of a separate pass bit for bit.
__device__ __forceinline__ void lora_split_sums(const LoraFinalizeJob& j0, const LoraFinalizeJob& j1,
                                                int worker, int nworkers) {
    constexpr int kMaxSplits = 16;
    const int total0 = j0.out ? j0.F * j0.r : 0;
    const int total = total0 + (j1.out ? j1.F * j1.r : 0);
    for (int i = worker; i < total; i += nworkers) {
        const LoraFinalizeJob& jb = i < total0 ? j0 : j1;
        const int ii = i < total0 ? i : i - total0;
        int f, j;
        if (jb.transpose_out) {  // consecutive threads walk f: coalesced stores into out[j][f]
            j = ii / jb.F;
            f = ii - j * jb.F;
        } else {
            f = ii / jb.r;
            j = ii - f * jb.r;
        }
        float hi[kMaxSplits], lo[kMaxSplits];
#pragma unroll
        for (int sp = 0; sp < kMaxSplits; ++sp) {
            if (sp < jb.splits) {
                const float* d = jb.partial + (static_cast<int64_t>(sp) * jb.F + f) * jb.NBW;
                hi[sp] = d[j];
                lo[sp] = d[jb.r + j];
            }
        }
        float v = 0.0f;
#pragma unroll
        for (int sp = 0; sp < kMaxSplits; ++sp)
            if (sp < jb.splits) v += hi[sp] + lo[sp];
        v *= jb.s;
        if (jb.transpose_out)
            jb.out[static_cast<int64_t>(j) * jb.F + f] = v;
        else
            jb.out[static_cast<int64_t>(f) * jb.r + j] = v;
    }
}

}  // namespace ft
