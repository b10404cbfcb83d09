// tc_transition.cu -- per-frame affine map of the state on the tensor cores.
//
// Carrying the state across a frame is the affine map
//   Sig_next = M Sig + N,   M = e^{G_L} I - Kt^T W,   N = Kt^T Ub,
//   Kt = diag(e^{G_L - G}) K
// (the per-frame transition of the chunk = frame decomposition; the pages
// compose these maps with a prefix sum over frames: cliffmar.tech article,
// "NVIDIA SANA-WM", the training section on context parallelism).
// One CTA per frame-head accumulates Kt^T [Ub | W] over 128-token blocks:
// A = Kt as an MN-major operand (the K tile's rows are tokens, i.e. the
// contraction index), B = the [Ub | W] block (MN-major), D in TMEM with one
// lane per key dimension.  The epilogue warps scale the K rows in shared
// memory by e^{G_L - G_r} (a per-row factor, so the swizzle does not
// matter) and finally write M and N in fp32.
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kThreads = 192;

struct Smem {
    static constexpr uint32_t K = 0;                       // 2 stages x 2 slabs x 128 rows
    static constexpr uint32_t X = K + 4 * SLAB_BYTES;      // 2 stages x 4 slabs x 128 rows
    static constexpr uint32_t END = X + 8 * SLAB_BYTES;
};

enum Bar { FULL0, FULL1, SCALED0, SCALED1, EMPTY0, EMPTY1, DONE, NBAR };

__global__ void __launch_bounds__(kThreads, 1)
k_transition_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_x,
                const TransParams prm) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int L = prm.L, dk = prm.dk, dv = prm.dv, nc = dk + dv, nblk = prm.nblk;
    const long long fh = blockIdx.x;
    const long long F = prm.F;
    const long long f = fh % F, chain = fh / F;
    const int h = (int)(chain % prm.H), b = (int)(chain / prm.H);
    const int bf = (int)(b * F + f);
    unsigned char *sK = smem + Smem::K;
    unsigned char *sX = smem + Smem::X;
    uint64_t *bars = (uint64_t *)(smem + Smem::END);
    uint32_t *tmem_slot = (uint32_t *)(bars + NBAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int *err = prm.err;
    const int nslab_k = (dk + SLAB - 1) / SLAB, nslab_x = (nc + SLAB - 1) / SLAB;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i) sm100::mbar_init(&bars[i], (i == SCALED0 || i == SCALED1) ? 128 : 1);
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
            sm100::tma_prefetch_desc(&tm_k);
            sm100::tma_prefetch_desc(&tm_x);
            bool ok = true;
            for (int i = 0; i < nblk && ok; ++i) {
                const int st = i & 1;
                if (i >= 2) ok = sm100::mbar_wait(&bars[EMPTY0 + st], ((i - 2) >> 1) & 1, err);
                if (!ok) break;
                sm100::mbar_arrive_expect_tx(&bars[FULL0 + st], (uint32_t)((nslab_k + nslab_x) * SLAB_BYTES));
                for (int sl = 0; sl < nslab_k; ++sl)
                    sm100::tma_load_4d(sK + (st * 2 + sl) * SLAB_BYTES, &tm_k, &bars[FULL0 + st], sl * SLAB, h,
                                       i * BM, bf);
                for (int sl = 0; sl < nslab_x; ++sl)
                    sm100::tma_load_3d(sX + (st * 4 + sl) * SLAB_BYTES, &tm_x, &bars[FULL0 + st], sl * SLAB, i * BM,
                                       (int)fh);
            }
            if (ok) sm100::mbar_wait(&bars[DONE], 0, err);  // no copy left in flight
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id = sm100::idesc_bf16(BM, nc, 1, 1);
            bool ok = true;
            for (int i = 0; i < nblk && ok; ++i) {
                const int st = i & 1;
                ok = sm100::mbar_wait(&bars[SCALED0 + st], (i >> 1) & 1, err);
                if (!ok) break;
                sm100::tc_fence_after();
                const unsigned char *kt = sK + st * 2 * SLAB_BYTES;
                const unsigned char *xt = sX + st * 4 * SLAB_BYTES;
                for (int ks = 0; ks < BM / 16; ++ks)
                    sm100::mma_bf16_ss(t_d, desc_mnmajor(kt, ks, BM), desc_mnmajor(xt, ks, BM), id,
                                       (i > 0 || ks > 0) ? 1u : 0u);
                sm100::mma_commit(&bars[EMPTY0 + st]);
            }
            if (ok) sm100::mma_commit(&bars[DONE]);
        }
    } else {
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;  // token row of each block; at the end, key dimension m
        const float *Gf = prm.G + fh * (long long)((L + 3) & ~3);  // G rows are padded to 16 bytes
        const float GL = Gf[L - 1];
        bool ok = true;
        for (int i = 0; i < nblk && ok; ++i) {
            const int st = i & 1;
            const int row = i * BM + r;
            const float sc = row < L ? __expf(GL - Gf[row]) : 0.f;
            ok = sm100::mbar_wait(&bars[FULL0 + st], (i >> 1) & 1, err);
            if (!ok) break;
            unsigned char *kt = sK + st * 2 * SLAB_BYTES;
            for (int sl = 0; sl < nslab_k; ++sl) {
                uint4 *rowp = reinterpret_cast<uint4 *>(kt + sl * SLAB_BYTES + r * 128);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint4 v = rowp[c];
                    __nv_bfloat162 *p2 = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float2 x = __bfloat1622float2(p2[e]);
                        p2[e] = __floats2bfloat162_rn(sc * x.x, sc * x.y);
                    }
                    rowp[c] = v;
                }
            }
            sm100::fence_proxy_async_smem();
            sm100::mbar_arrive(&bars[SCALED0 + st]);
        }
        if (ok) ok = sm100::mbar_wait(&bars[DONE], 0, err);
        if (ok) {
            sm100::tc_fence_after();
            const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
            const float eGL = __expf(GL);
            const int m = r;
            for (int c0 = 0; c0 < nc; c0 += 16) {
                float v[16];
                sm100::tmem_ld16(t_d + lane_off + c0, v);
                sm100::tmem_ld_wait();
                if (m < dk) {  // dv is a multiple of 16: a chunk lies wholly in N or in M
                    float *dst;
                    if (c0 < dv) {
                        dst = prm.N + (fh * dk + m) * (long long)dv + c0;
                    } else {
                        const int j0 = c0 - dv;
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = (m == j0 + e ? eGL : 0.f) - v[e];
                        dst = prm.M + (fh * dk + m) * (long long)dk + j0;
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

cudaError_t launch_transition_tc(const CUtensorMap &tm_k, const CUtensorMap &tm_x, const TransParams &prm,
                                 long long n_fh, cudaStream_t s) {
    const size_t smem = 1024 + Smem::END + sizeof(uint64_t) * NBAR + 16;
    cudaError_t e = cudaFuncSetAttribute(k_transition_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_transition_tc<<<(unsigned)n_fh, kThreads, smem, s>>>(tm_k, tm_x, prm);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace gdn
