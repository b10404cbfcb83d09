// tc_transition.cu -- the frame-wise operator's per-frame map on the tensor cores.
//
// The frame-wise operator (SANA-WM summary, "Memory-Efficient Long-Context
// Modeling (Section 3.2)", paragraph "Adaptation to video: frame-wise
// recurrence") carries the state across frame f by the affine map
//   Sig_next = M Sig + N,   M = gamma (I - K^T B K),   N = K^T B V,   B = diag(beta)
// (the pages compose such maps with a prefix sum over frames: cliffmar.tech
// article, "NVIDIA SANA-WM", the training section on context parallelism).
// The chunked (token-wise) pass does not use this kernel: its maps come out of
// the intra-frame kernel.
// One CTA per frame-head accumulates K^T B [V | K] over 64-token chunks that
// stream through a 2-deep ring, two CTAs per SM so that one CTA's loads
// overlap the other's start-up and final stores (the kernel is bound by the
// rate at which the chunks arrive from HBM): A = B K as an MN-major operand
// (the K chunk's rows are tokens, i.e. the contraction index), B = the [V | K]
// chunk (V in the first 64-column slabs, K after them; MN-major), D in TMEM
// with one lane per key dimension.  The epilogue warps scale the K rows in
// shared memory by beta (a per-row factor, so the swizzle does not matter),
// apply the key feature map when asked, and finally write M and N in fp32
// (and/or the scan's bf16 operand images of M).
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kThreads = 192;
constexpr int CH = 64;                         // tokens per chunk
constexpr int NST = 2;                         // ring depth (two CTAs per SM)
constexpr int CSLAB = CH * 128;                // one 64-row slab
constexpr int STAGE = 6 * CSLAB;               // K (2 slabs) + [Ub | W] (4 slabs)

struct Smem {
    static constexpr uint32_t RING = 0;
    static constexpr uint32_t END = RING + NST * STAGE;
};

enum Bar { FULL = 0, SCALED = FULL + NST, EMPTY = SCALED + NST, DONE = EMPTY + NST, NBAR };

__global__ void __launch_bounds__(kThreads, 2)
k_transition_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const TransParams prm) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int L = prm.L, dk = prm.dk, dv = prm.dv;
    const long long fh = blockIdx.x;
    const long long F = prm.F;
    const long long f = fh % F, chain = fh / F;
    const int h = (int)(chain % prm.H), b = (int)(chain / prm.H);
    const int bf = (int)(b * F + f);
    unsigned char *sRing = smem + Smem::RING;
    uint64_t *bars = (uint64_t *)(smem + Smem::END);
    uint32_t *tmem_slot = (uint32_t *)(bars + NBAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int *err = prm.err;
    const int nslab_k = (dk + SLAB - 1) / SLAB, nslab_v = (dv + SLAB - 1) / SLAB;
    // B operand columns: [V | K], slab-aligned
    const int nslab_x = nslab_v + nslab_k;
    const int ncols = SLAB * nslab_x;
    const int mcol0 = SLAB * nslab_v;  // first column of the M part

    if (pass_failed(prm.err)) return;  // an earlier stage of this pass gave up
    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i) sm100::mbar_init(&bars[i], (i >= SCALED && i < SCALED + NST) ? 128 : 1);
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

    const int nch = (L + CH - 1) / CH;
    if (warp == 0) {
        if (lane == 0) {
            sm100::tma_prefetch_desc(&tm_k);
            sm100::tma_prefetch_desc(&tm_v);
            bool ok = true;
            for (int c = 0; c < nch && ok; ++c) {
                const int st = c % NST;
                if (c >= NST) ok = sm100::mbar_wait(&bars[EMPTY + st], ((c / NST) - 1) & 1, err);
                if (!ok) break;
                unsigned char *stage = sRing + st * STAGE;
                sm100::mbar_arrive_expect_tx(&bars[FULL + st], (uint32_t)((nslab_k + nslab_x) * CSLAB));
                for (int sl = 0; sl < nslab_k; ++sl)
                    sm100::tma_load_4d(stage + sl * CSLAB, &tm_k, &bars[FULL + st], sl * SLAB, h, c * CH, bf);
                for (int sl = 0; sl < nslab_v; ++sl)
                    sm100::tma_load_4d(stage + (2 + sl) * CSLAB, &tm_v, &bars[FULL + st], sl * SLAB, h, c * CH, bf);
                for (int sl = 0; sl < nslab_k; ++sl)
                    sm100::tma_load_4d(stage + (2 + nslab_v + sl) * CSLAB, &tm_k, &bars[FULL + st], sl * SLAB, h,
                                       c * CH, bf);
            }
            if (ok) sm100::mbar_wait(&bars[DONE], 0, err);  // no copy left in flight
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id = sm100::idesc_bf16(BM, ncols, 1, 1);
            bool ok = true;
            for (int c = 0; c < nch && ok; ++c) {
                const int st = c % NST;
                ok = sm100::mbar_wait(&bars[SCALED + st], (c / NST) & 1, err);
                if (!ok) break;
                sm100::tc_fence_after();
                const unsigned char *kt = sRing + st * STAGE;
                const unsigned char *xt = kt + 2 * CSLAB;
                for (int ks = 0; ks < CH / 16; ++ks)
                    sm100::mma_bf16_ss(t_d, desc_mnmajor(kt, ks, CH), desc_mnmajor(xt, ks, CH), id,
                                       (c > 0 || ks > 0) ? 1u : 0u);
                sm100::mma_commit(&bars[EMPTY + st]);
            }
            if (ok) sm100::mma_commit(&bars[DONE]);
        }
    } else {
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;  // the epilogue's 128 threads; at the end, key dimension m
        bool ok = true;
        // thread r scales row r % 64 of the chunk's K, slab r / 64
        const int row_in = r & (CH - 1), sl = r >> 6;
        float *sSS = reinterpret_cast<float *>(bars + NBAR + 1);  // [2][64] partial sums of squares
        const bool normk = prm.norm_k != 0;
        // the K row's factor beta_r, read one chunk ahead so the load's latency stays off the
        // scaling step
        auto row_gate = [&](int c) -> float {
            const int row = c * CH + row_in;
            if (c >= nch || row >= L) return 0.f;
            return prm.beta[((long long)b * prm.T + f * L + row) * prm.H + h];
        };
        float g_next = row_gate(0);
        for (int c = 0; c < nch && ok; ++c) {
            const int st = c % NST;
            const int row = c * CH + row_in;
            const float g_row = g_next;
            g_next = row_gate(c + 1);
            const float sc = row >= L ? 0.f : g_row;
            ok = sm100::mbar_wait(&bars[FULL + st], (c / NST) & 1, err, prm.wait_ns);
            if (normk) ok = named_sync_and(1, 128, ok);  // the row's two halves meet below
            if (!ok) break;
            if (normk) {
                // key feature map of the frame-wise operator (SANA-WM summary, section 3.2,
                // "Algebraic Stabilization for Spatial Token Explosion"): y = max(RMSNorm(k) w, 0)
                // / sqrt(d_k S); the row's mean square is summed over both 64-column halves
                uint4 *rowp = reinterpret_cast<uint4 *>(sRing + st * STAGE + sl * CSLAB + row_in * 128);
                float ss = 0.f;
                if (sl < nslab_k) {
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
                sSS[sl * CH + row_in] = ss;
                named_sync(1, 128);
                const float inv = 1.f / sqrtf((sSS[row_in] + sSS[CH + row_in]) / (float)dk + kRmsEps);
                named_sync(1, 128);  // both halves read before the next chunk writes sSS
                if (sl < nslab_k) {
                    uint4 *rowb = reinterpret_cast<uint4 *>(sRing + st * STAGE + (2 + nslab_v + sl) * CSLAB +
                                                            row_in * 128);
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        uint4 v = rowp[cc], vb;
                        __nv_bfloat162 *p2 = reinterpret_cast<__nv_bfloat162 *>(&v);
                        __nv_bfloat162 *b2 = reinterpret_cast<__nv_bfloat162 *>(&vb);
                        const int c0 = sl * 64 + ((cc ^ (row_in & 7)) << 3);  // logical column of the chunk
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 x = __bfloat1622float2(p2[e]);
                            const int ca = c0 + 2 * e;
                            const float wa = (prm.k_w && ca < dk) ? prm.k_w[ca] : 1.f;
                            const float wb = (prm.k_w && ca + 1 < dk) ? prm.k_w[ca + 1] : 1.f;
                            const float ya = fmaxf(x.x * inv * wa, 0.f) * prm.k_post;
                            const float yb = fmaxf(x.y * inv * wb, 0.f) * prm.k_post;
                            b2[e] = __floats2bfloat162_rn(ya, yb);            // K (the B operand's copy)
                            p2[e] = __floats2bfloat162_rn(sc * ya, sc * yb);  // beta K (the A operand)
                        }
                        rowp[cc] = v;
                        rowb[cc] = vb;
                    }
                }
            } else if (sl < nslab_k) {
                uint4 *rowp = reinterpret_cast<uint4 *>(sRing + st * STAGE + sl * CSLAB + row_in * 128);
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    uint4 v = rowp[cc];
                    __nv_bfloat162 *p2 = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float2 x = __bfloat1622float2(p2[e]);
                        p2[e] = __floats2bfloat162_rn(sc * x.x, sc * x.y);
                    }
                    rowp[cc] = v;
                }
            }
            sm100::fence_proxy_async_smem();
            sm100::mbar_arrive(&bars[SCALED + st]);
        }
        if (ok) ok = sm100::mbar_wait(&bars[DONE], 0, err);
        if (ok) {
            sm100::tc_fence_after();
            const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
            // M = gamma I - gamma (K^T B K)
            const float gam = prm.gamma[((long long)b * F + f) * prm.H + h];
            const float eGL = gam;
            const int m = r;
            for (int c4 = 0; c4 < ncols; c4 += 64) {  // four 16-column loads per wait (the last group may
                float v4[4][16];                      // read past ncols, inside the 256-column buffer, unused)
#pragma unroll
                for (int g = 0; g < 4; ++g) sm100::tmem_ld16(t_d + lane_off + c4 + 16 * g, v4[g]);
                sm100::tmem_ld_wait();
                if (m >= dk) continue;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int c0 = c4 + 16 * g;
                    if (c0 >= ncols) break;
                    float *v = v4[g];
                    float *dst;  // dv is a multiple of 16: a chunk lies wholly in N, in M or in padding
                    if (c0 < dv) {
                        dst = prm.N + (fh * dk + m) * (long long)dv + c0;
                    } else if (c0 >= mcol0 && c0 - mcol0 < dk) {
                        const int j0 = c0 - mcol0;
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = (m == j0 + e ? eGL : 0.f) - gam * v[e];
                        if (prm.Mimg) {  // hi + lo bf16 images of the scan's A operand
                            const int nslab = (dk + SLAB - 1) / SLAB;
                            unsigned char *img = reinterpret_cast<unsigned char *>(prm.Mimg) +
                                                 fh * (long long)(2 * nslab * dk * 128);
#pragma unroll
                            for (int h8 = 0; h8 < 2; ++h8) {
                                uint32_t hi[4], lo[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float a = v[8 * h8 + 2 * e], bb = v[8 * h8 + 2 * e + 1];
                                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(a, bb);
                                    const float2 hf = __bfloat1622float2(h2);
                                    hi[e] = *reinterpret_cast<const uint32_t *>(&h2);
                                    lo[e] = pack_bf16(a - hf.x, bb - hf.y);
                                }
                                const uint32_t off = sm100::sw128_kmajor_offset(m, j0 + 8 * h8, dk);
                                *reinterpret_cast<uint4 *>(img + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                                *reinterpret_cast<uint4 *>(img + nslab * dk * 128 + off) =
                                    make_uint4(lo[0], lo[1], lo[2], lo[3]);
                            }
                        }
                        if (!prm.M) continue;
                        dst = prm.M + (fh * dk + m) * (long long)dk + j0;
                    } else {
                        continue;
                    }
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4 *>(dst + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                }
            }
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

cudaError_t launch_transition_tc(const CUtensorMap &tm_k, const CUtensorMap &tm_v, const TransParams &prm,
                                 long long n_fh, cudaStream_t s) {
    const size_t smem = 1024 + Smem::END + sizeof(uint64_t) * NBAR + 16 + 2 * CH * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(k_transition_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_transition_tc<<<(unsigned)n_fh, kThreads, smem, s>>>(tm_k, tm_v, prm);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace gdn
