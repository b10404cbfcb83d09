// tc_u.cu -- pseudo-values U = Ub - W Sig on the tensor cores.
//
// With the state Sig entering a frame known, the frame's pseudo-values are
// U = Ub - W Sig (U = T (beta V - decayed K S) in the UT form of the delta
// rule; SANA-WM summary, "Memory-Efficient Long-Context Modeling
// (Section 3.2)", frame-wise GDN).  One CTA per frame-head walks its
// 128-row blocks: A = W (K-major, the last d_k columns of the [Ub | W]
// rows), B = Sig in bf16 (MN-major), D = W Sig in a TMEM double buffer;
// the epilogue subtracts it from Ub (read straight from global) and writes
// U in bf16, the B operand layout of the output kernel.
// The same kernel is the frame-wise operator's output (SANA-WM summary,
// "Memory-Efficient Long-Context Modeling (Section 3.2)", paragraph
// "Adaptation to video: frame-wise recurrence"): A = the frame's queries,
// Sig the state after the frame's update, and o = Q Sig written to o.
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kThreads = 192;

struct Smem {
    static constexpr uint32_t SIG = 0;                     // 2 slabs x d_k rows (<= 32 KB)
    static constexpr uint32_t W = SIG + 2 * SLAB_BYTES;    // 2 stages x 2 slabs x 128 rows
    static constexpr uint32_t END = W + 4 * SLAB_BYTES;
};

enum Bar { SIGFULL, WFULL0, WFULL1, WEMPTY0, WEMPTY1, DFULL0, DFULL1, DEMPTY0, DEMPTY1, QREADY0, QREADY1, NBAR };

__global__ void __launch_bounds__(kThreads, 2)  // two CTAs per SM
k_u_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_q,
       const __grid_constant__ CUtensorMap tm_sig, const UParams prm) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int L = prm.L, dk = prm.dk, dv = prm.dv, nc = dk + dv, nblk = prm.nblk;
    const long long fh = blockIdx.x;
    unsigned char *sSig = smem + Smem::SIG;
    unsigned char *sW = smem + Smem::W;
    uint64_t *bars = (uint64_t *)(smem + Smem::END);
    uint32_t *tmem_slot = (uint32_t *)(bars + NBAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int *err = prm.err;
    const int nslab_k = (dk + SLAB - 1) / SLAB, nslab_v = (dv + SLAB - 1) / SLAB;
    const bool frame = prm.frame != 0;
    const bool normq = frame && prm.norm_q;
    const long long f = frame ? fh % prm.F : 0, chain = frame ? fh / prm.F : 0;
    const int h = frame ? (int)(chain % prm.H) : 0, b = frame ? (int)(chain / prm.H) : 0;

    if (pass_failed(prm.err)) return;  // an earlier stage of this pass gave up
    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i)
            sm100::mbar_init(&bars[i], (i == DEMPTY0 || i == DEMPTY1 || i == QREADY0 || i == QREADY1) ? 128 : 1);
        sm100::fence_barrier_init();
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, 256);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t t_d = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            sm100::tma_prefetch_desc(frame ? &tm_q : &tm_x);
            sm100::tma_prefetch_desc(&tm_sig);
            sm100::mbar_arrive_expect_tx(&bars[SIGFULL], (uint32_t)(nslab_v * dk * 128));
            for (int sl = 0; sl < nslab_v; ++sl)
                sm100::tma_load_3d(sSig + sl * dk * 128, &tm_sig, &bars[SIGFULL], sl * SLAB, 0, (int)fh);
            bool ok = true;
            for (int i = 0; i < nblk && ok; ++i) {
                const int st = i & 1;
                if (i >= 2) ok = sm100::mbar_wait(&bars[WEMPTY0 + st], ((i - 2) >> 1) & 1, err);
                if (!ok) break;
                sm100::mbar_arrive_expect_tx(&bars[WFULL0 + st], (uint32_t)(nslab_k * SLAB_BYTES));
                for (int sl = 0; sl < nslab_k; ++sl) {
                    if (frame)  // the frame's queries
                        sm100::tma_load_4d(sW + (st * 2 + sl) * SLAB_BYTES, &tm_q, &bars[WFULL0 + st], sl * SLAB, h,
                                           i * BM, (int)(b * prm.F + f));
                    else  // W = columns dv .. dv + dk of the [Ub | W] rows
                        sm100::tma_load_3d(sW + (st * 2 + sl) * SLAB_BYTES, &tm_x, &bars[WFULL0 + st],
                                           dv + sl * SLAB, i * BM, (int)fh);
                }
            }
            for (int i = (nblk >= 2 ? nblk - 2 : 0); ok && i < nblk; ++i)
                ok = sm100::mbar_wait(&bars[WEMPTY0 + (i & 1)], (i >> 1) & 1, err);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id = sm100::idesc_bf16(BM, dv, 0, 1);
            bool ok = sm100::mbar_wait(&bars[SIGFULL], 0, err);
            for (int i = 0; i < nblk && ok; ++i) {
                const int st = i & 1;
                // the operand is ready when it has landed, or (query feature map) once the
                // epilogue has normalised it in place
                ok = sm100::mbar_wait(&bars[(normq ? QREADY0 : WFULL0) + st], (i >> 1) & 1, err);
                if (ok && i >= 2) ok = sm100::mbar_wait(&bars[DEMPTY0 + st], ((i - 2) >> 1) & 1, err);
                if (!ok) break;
                sm100::tc_fence_after();
                const unsigned char *wt = sW + st * 2 * SLAB_BYTES;
                for (int ks = 0; ks < dk / 16; ++ks)
                    sm100::mma_bf16_ss(t_d + st * 128, desc_kmajor(wt, ks, BM), desc_mnmajor(sSig, ks, dk), id,
                                       ks > 0);
                sm100::mma_commit(&bars[DFULL0 + st]);
                sm100::mma_commit(&bars[WEMPTY0 + st]);
            }
        }
    } else {
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        bool ok = true;
        // query feature map of the frame-wise operator (SANA-WM summary, section 3.2, "Algebraic
        // Stabilization for Spatial Token Explosion"): row r of block i's staged Q becomes
        // max(RMSNorm(q) w, 0) in place before the product reads it
        auto normalize = [&](int i) -> bool {
            const int st = i & 1;
            if (!sm100::mbar_wait(&bars[WFULL0 + st], (i >> 1) & 1, err)) return false;
            float ss = 0.f;
            for (int sl = 0; sl < nslab_k; ++sl) {
                const uint4 *rowp = reinterpret_cast<const uint4 *>(sW + (st * 2 + sl) * SLAB_BYTES + r * 128);
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const uint4 v = rowp[cc];
                    const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x = __bfloat1622float2(p2[e]);
                        ss = fmaf(x.x, x.x, fmaf(x.y, x.y, ss));
                    }
                }
            }
            const float inv = 1.f / sqrtf(ss / (float)dk + kRmsEps);
            for (int sl = 0; sl < nslab_k; ++sl) {
                uint4 *rowp = reinterpret_cast<uint4 *>(sW + (st * 2 + sl) * SLAB_BYTES + r * 128);
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    uint4 v = rowp[cc];
                    __nv_bfloat162 *p2 = reinterpret_cast<__nv_bfloat162 *>(&v);
                    const int c0 = sl * 64 + ((cc ^ (r & 7)) << 3);  // logical column of the chunk
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x = __bfloat1622float2(p2[e]);
                        const int ca = c0 + 2 * e;
                        const float wa = (prm.q_w && ca < dk) ? prm.q_w[ca] : 1.f;
                        const float wb = (prm.q_w && ca + 1 < dk) ? prm.q_w[ca + 1] : 1.f;
                        p2[e] = __floats2bfloat162_rn(fmaxf(x.x * inv * wa, 0.f), fmaxf(x.y * inv * wb, 0.f));
                    }
                    rowp[cc] = v;
                }
            }
            sm100::fence_proxy_async_smem();
            sm100::mbar_arrive(&bars[QREADY0 + st]);
            return true;
        };
        if (normq && nblk > 0) ok = normalize(0);
        for (int i = 0; i < nblk && ok; ++i) {
            if (normq && i + 1 < nblk && !(ok = normalize(i + 1))) break;
            const int st = i & 1;
            const int row = i * BM + r;
            const bool valid = row < L;
            // chunkwise: U = Ub - D over the row's [Ub | W]; frame-wise: o (+)= D
            const __nv_bfloat16 *xrow =
                frame ? prm.o + (((long long)b * prm.T + f * L + (valid ? row : 0)) * prm.H + h) * dv
                      : prm.X + (fh * (long long)L + (valid ? row : 0)) * nc;
            __nv_bfloat16 *urow = frame ? const_cast<__nv_bfloat16 *>(xrow)
                                        : prm.U + (fh * (long long)L + (valid ? row : 0)) * dv;
            const bool load_row = !frame || prm.accumulate;
            const float sgn = frame ? 1.f : -1.f;
            // this row's Ub (or the o being accumulated into) in registers before the wait, so
            // its latency hides behind the MMA
            uint4 ub[16];
#pragma unroll
            for (int c8 = 0; c8 < 16; ++c8)
                ub[c8] = (valid && load_row && c8 < dv / 8) ? __ldg(reinterpret_cast<const uint4 *>(xrow) + c8)
                                                            : make_uint4(0, 0, 0, 0);
            ok = sm100::mbar_wait(&bars[DFULL0 + st], (i >> 1) & 1, err);
            if (!ok) break;
            sm100::tc_fence_after();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int c0 = 16 * j;
                if (c0 >= dv) break;
                float d[16];
                sm100::tmem_ld16(t_d + st * 128 + lane_off + c0, d);
                sm100::tmem_ld_wait();
                if (valid) {
                    uint4 out[2];
#pragma unroll
                    for (int w = 0; w < 2; ++w) {
                        uint4 xv = ub[2 * j + w];
                        __nv_bfloat162 *p2 = reinterpret_cast<__nv_bfloat162 *>(&xv);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 u = __bfloat1622float2(p2[e]);
                            p2[e] = __floats2bfloat162_rn(u.x + sgn * d[w * 8 + 2 * e], u.y + sgn * d[w * 8 + 2 * e + 1]);
                        }
                        out[w] = xv;
                    }
                    reinterpret_cast<uint4 *>(urow + c0)[0] = out[0];
                    reinterpret_cast<uint4 *>(urow + c0)[1] = out[1];
                }
            }
            sm100::tc_fence_before();
            sm100::mbar_arrive(&bars[DEMPTY0 + st]);
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(t_d, 256);
    }
}

}  // namespace

cudaError_t launch_u_tc(const CUtensorMap &tm_x, const CUtensorMap &tm_q, const CUtensorMap &tm_sig,
                        const UParams &prm, long long n_fh, cudaStream_t s) {
    const size_t smem = 1024 + Smem::END + sizeof(uint64_t) * NBAR + 16;
    cudaError_t e = cudaFuncSetAttribute(k_u_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_u_tc<<<(unsigned)n_fh, kThreads, smem, s>>>(tm_x, tm_q, tm_sig, prm);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace gdn
