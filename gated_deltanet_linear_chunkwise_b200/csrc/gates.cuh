// gates.cuh -- per-frame gate prefix shared by the kernels.
//
// G_i = sum_{m <= i} log alpha_m over one logical frame (the decay of the
// gated delta rule in log space; SANA-WM summary, "Memory-Efficient
// Long-Context Modeling (Section 3.2)", the decay gate of the GDN update).
// log alpha is clamped at kLogAlphaFloor so alpha = 0 stays finite.
#pragma once

#include "gdn_internal.h"

namespace gdn {

template <typename TG> __device__ __forceinline__ TG log_gate(float a) {
    TG lg = a > 0.f ? (TG)log((TG)a) : (TG)kLogAlphaFloor;
    return lg < (TG)kLogAlphaFloor ? (TG)kLogAlphaFloor : lg;
}

// Inclusive prefix of log(alpha) over logical frame f of chain (b,h) into
// sG[0..L), and the frame's beta into sB[0..L).  Block-wide scan: each
// thread takes a contiguous run, warps scan their totals with shuffles.
template <typename TG>
__device__ void frame_gates(const Problem &p, int b, int h, long long f, TG *sG, float *sB, TG *sScr) {
    const int L = p.L, tid = threadIdx.x, nt = blockDim.x;
    const int per = (L + nt - 1) / nt;
    const int i0 = tid * per, i1 = min(i0 + per, L);
    TG run = 0;
    for (int i = i0; i < i1; ++i) {
        const long long row = tok_row(p, b, h, phys_token(p, f, i));
        run += log_gate<TG>(p.alpha[row]);
        sG[i] = run;
        sB[i] = p.beta[row];
    }
    const int lane = tid & 31, warp = tid >> 5, nw = (nt + 31) >> 5;
    TG x = run;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        TG y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) sScr[warp] = x;
    __syncthreads();
    if (warp == 0) {
        TG w = lane < nw ? sScr[lane] : (TG)0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            TG y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
        }
        if (lane < nw) sScr[lane] = w;
    }
    __syncthreads();
    const TG offset = (x - run) + (warp > 0 ? sScr[warp - 1] : (TG)0);
    for (int i = i0; i < i1; ++i) sG[i] += offset;
    __syncthreads();
}

}  // namespace gdn
