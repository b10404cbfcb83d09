// tc_output.cu -- output stage on the 5th-generation tensor cores.
//
// For one 128-row block I of one frame-head (rows r, columns s of the frame):
//   O_I = diag(e^G) Q_I Sig + sum_{J <= I} P_IJ U_J,
//   P_IJ[r][s] = (q_r . k_s) e^{G_r - G_s}  for s <= r (inclusive: o_r reads S_r)
// (the intra-frame term of the chunkwise gated delta rule; SANA-WM summary,
// "Memory-Efficient Long-Context Modeling (Section 3.2)", frame-wise GDN).
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues tcgen05.mma from one thread, warps 2-5 are the epilogue (one tile
// row per thread, TMEM lane quadrant = warp % 4).
//   TMEM: S_J double buffer (2 x 128 cols), O (dv cols), Q.Sig (dv cols).
//   SMEM: Q_I, K_J x2, U_J x2 (bf16, 128B-swizzled), P (aliases Sig).
// Off-diagonal decay factors are split around the anchor A = G[I*128 - 1]:
// e^{G_r - G_s} = e^{G_r - A} e^{A - G_s}, both <= 1; the diagonal tile
// takes e^{G_r - G_s} per element.  Every wait is bounded (sm100::mbar_wait).
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kThreads = 192;

struct Smem {
    static constexpr uint32_t Q = 0;                       // 2 slabs
    static constexpr uint32_t K = Q + 2 * SLAB_BYTES;      // 2 stages x 2 slabs
    static constexpr uint32_t U = K + 4 * SLAB_BYTES;      // 2 stages x 2 slabs
    static constexpr uint32_t P = U + 4 * SLAB_BYTES;      // P tile; Sig shares it
    static constexpr uint32_t G = P + 2 * SLAB_BYTES;      // nblk*128 floats follow
};

enum Bar { QFULL, QSDONE, KVFULL0, KVFULL1, KVEMPTY0, KVEMPTY1, SFULL0, SFULL1, SEMPTY0, SEMPTY1,
           PFULL, PEMPTY, OFULL, NBAR };

__global__ void __launch_bounds__(kThreads, 1)
k_output_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_sig,
            const OutParams prm) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int L = prm.L, dk = prm.dk, dv = prm.dv, nblk = prm.nblk;
    const long long fh = blockIdx.x / nblk;
    const int I = nblk - 1 - (int)(blockIdx.x % nblk);  // heaviest tiles first
    const long long F = prm.F;
    const long long f = fh % F, chain = fh / F;
    const int h = (int)(chain % prm.H), b = (int)(chain / prm.H);

    unsigned char *sQ = smem + Smem::Q;
    unsigned char *sK = smem + Smem::K;
    unsigned char *sU = smem + Smem::U;
    unsigned char *sP = smem + Smem::P;
    unsigned char *sSig = sP;
    float *sG = (float *)(smem + Smem::G);
    float *sCf = sG + nblk * BM;                    // nblk*128 column decay factors
    uint64_t *bars = (uint64_t *)(sCf + nblk * BM);
    uint32_t *tmem_slot = (uint32_t *)(bars + NBAR);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int *err = prm.err;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i) {
            uint32_t cnt = 1;
            if (i == SEMPTY0 || i == SEMPTY1 || i == PFULL) cnt = 128;
            sm100::mbar_init(&bars[i], cnt);
        }
        sm100::fence_barrier_init();
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, 512);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t t_s0 = tbase, t_o = tbase + 256, t_qs = tbase + 384;

    const int nks_d = dk / 16;                 // K steps over the head dim
    const int nslab_k = (dk + SLAB - 1) / SLAB, nslab_v = (dv + SLAB - 1) / SLAB;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            sm100::tma_prefetch_desc(&tm_q);
            sm100::tma_prefetch_desc(&tm_k);
            sm100::tma_prefetch_desc(&tm_u);
            sm100::tma_prefetch_desc(&tm_sig);
            const int bf = (int)(b * F + f);
            sm100::mbar_arrive_expect_tx(&bars[QFULL], (uint32_t)(nslab_k * SLAB_BYTES + nslab_v * dk * 128));
            for (int sl = 0; sl < nslab_k; ++sl)
                sm100::tma_load_4d(sQ + sl * SLAB_BYTES, &tm_q, &bars[QFULL], sl * SLAB, h, I * BM, bf);
            for (int sl = 0; sl < nslab_v; ++sl)
                sm100::tma_load_3d(sSig + sl * dk * 128, &tm_sig, &bars[QFULL], sl * SLAB, 0, (int)fh);
            bool ok = true;
            for (int J = 0; J <= I && ok; ++J) {
                const int st = J & 1;
                if (J >= 2) ok = sm100::mbar_wait(&bars[KVEMPTY0 + st], ((J - 2) >> 1) & 1, err);
                if (!ok) break;
                sm100::mbar_arrive_expect_tx(&bars[KVFULL0 + st], (uint32_t)((nslab_k + nslab_v) * SLAB_BYTES));
                for (int sl = 0; sl < nslab_k; ++sl)
                    sm100::tma_load_4d(sK + (st * 2 + sl) * SLAB_BYTES, &tm_k, &bars[KVFULL0 + st], sl * SLAB, h,
                                       J * BM, bf);
                for (int sl = 0; sl < nslab_v; ++sl)
                    sm100::tma_load_3d(sU + (st * 2 + sl) * SLAB_BYTES, &tm_u, &bars[KVFULL0 + st], sl * SLAB,
                                       J * BM, (int)fh);
            }
            // do not leave with copies in flight: the last stages' loads must land
            for (int J = (I >= 1 ? I - 1 : 0); J <= I; ++J)
                sm100::mbar_wait(&bars[KVFULL0 + (J & 1)], (J >> 1) & 1, err);
            sm100::mbar_wait(&bars[QFULL], 0, err);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_s = sm100::idesc_bf16(BM, BM, 0, 0);
            const uint32_t id_o = sm100::idesc_bf16(BM, dv, 0, 1);
            bool ok = sm100::mbar_wait(&bars[QFULL], 0, err);
            if (ok) {
                sm100::tc_fence_after();
                for (int ks = 0; ks < nks_d; ++ks)
                    sm100::mma_bf16_ss(t_qs, desc_kmajor(sQ, ks, BM), desc_mnmajor(sSig, ks, dk), id_o, ks > 0);
                sm100::mma_commit(&bars[QSDONE]);
            }
            auto issue_pu = [&](int Jp) -> bool {
                if (!sm100::mbar_wait(&bars[PFULL], Jp & 1, err)) return false;
                sm100::tc_fence_after();
                const unsigned char *u = sU + (Jp & 1) * 2 * SLAB_BYTES;
                for (int ks = 0; ks < BM / 16; ++ks)
                    sm100::mma_bf16_ss(t_o, desc_kmajor(sP, ks, BM), desc_mnmajor(u, ks, BM), id_o,
                                       (Jp > 0 || ks > 0) ? 1u : 0u);
                sm100::mma_commit(&bars[PEMPTY]);
                sm100::mma_commit(&bars[KVEMPTY0 + (Jp & 1)]);
                return true;
            };
            for (int J = 0; J <= I && ok; ++J) {
                const int st = J & 1;
                ok = sm100::mbar_wait(&bars[KVFULL0 + st], (J >> 1) & 1, err);
                if (ok && J >= 2) ok = sm100::mbar_wait(&bars[SEMPTY0 + st], ((J - 2) >> 1) & 1, err);
                if (!ok) break;
                sm100::tc_fence_after();
                const unsigned char *kt = sK + st * 2 * SLAB_BYTES;
                for (int ks = 0; ks < nks_d; ++ks)
                    sm100::mma_bf16_ss(t_s0 + st * 128, desc_kmajor(sQ, ks, BM), desc_kmajor(kt, ks, BM), id_s,
                                       ks > 0);
                sm100::mma_commit(&bars[SFULL0 + st]);
                if (J >= 1) ok = issue_pu(J - 1);
            }
            if (ok) ok = issue_pu(I);
            if (ok) sm100::mma_commit(&bars[OFULL]);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 64;          // 0..127
        const int q4 = warp & 3;                  // TMEM lane quadrant
        const int r = q4 * 32 + lane;             // tile row owned by this thread
        const int row = I * BM + r;               // row within the frame
        const float *Gf = prm.G + fh * (long long)L;
        const int ncols = (I + 1) * BM;
        const float A = I > 0 ? Gf[I * BM - 1] : 0.f;  // anchor: G just before the block
        for (int s = et; s < ncols; s += 128) {
            const float g = Gf[s < L ? s : L - 1];
            sG[s] = g;
            sCf[s] = (s < I * BM) ? __expf(A - g) : 0.f;  // column factors of the off-diagonal tiles
        }
        named_sync(1, 128);  // the only epilogue-wide barrier: before any bounded wait
        const float Gr = sG[row < L ? row : L - 1];
        const float rf = __expf(Gr - A);
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;

        bool ok = sm100::mbar_wait(&bars[QSDONE], 0, err);  // P aliases Sig
        for (int J = 0; J <= I && ok; ++J) {
            const int st = J & 1;
            const bool diag = (J == I);
            const float *cf = sCf + J * BM;
            ok = sm100::mbar_wait(&bars[SFULL0 + st], (J >> 1) & 1, err);
            if (ok && J >= 1) ok = sm100::mbar_wait(&bars[PEMPTY], (J - 1) & 1, err);
            if (!ok) break;
            sm100::tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                float v[32];
                sm100::tmem_ld32(t_s0 + st * 128 + lane_off + c * 32, v);
                sm100::tmem_ld_wait();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int s = J * BM + c * 32 + e;
                    float p0, p1;
                    if (!diag) {
                        p0 = v[e] * rf * cf[c * 32 + e];
                        p1 = v[e + 1] * rf * cf[c * 32 + e + 1];
                    } else {
                        p0 = (s <= row && s < L) ? v[e] * __expf(Gr - sG[s]) : 0.f;
                        p1 = (s + 1 <= row && s + 1 < L) ? v[e + 1] * __expf(Gr - sG[s + 1]) : 0.f;
                    }
                    pk[e >> 1] = pack_bf16(p0, p1);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int chunk = c * 4 + u;  // 8 columns each
                    const int slab = chunk >> 3, cc = chunk & 7;
                    uint4 val = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                    *reinterpret_cast<uint4 *>(sP + slab * SLAB_BYTES + r * 128 + ((cc ^ (r & 7)) << 4)) = val;
                }
            }
            sm100::tc_fence_before();
            sm100::mbar_arrive(&bars[SEMPTY0 + st]);
            sm100::fence_proxy_async_smem();
            sm100::mbar_arrive(&bars[PFULL]);
        }
        if (ok) ok = sm100::mbar_wait(&bars[OFULL], 0, err);
        if (ok) {
            sm100::tc_fence_after();
            const float eg = __expf(Gr);
            const long long t = f * L + row;
            __nv_bfloat16 *o = (__nv_bfloat16 *)prm.o + ((((long long)b * prm.T + t) * prm.H + h) * dv);
            for (int c = 0; c < dv; c += 16) {
                float vo[16], vq[16];
                sm100::tmem_ld16(t_o + lane_off + c, vo);
                sm100::tmem_ld16(t_qs + lane_off + c, vq);
                sm100::tmem_ld_wait();
                if (row < L) {
                    float acc[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) acc[e] = eg * vq[e] + vo[e];
                    if (prm.accumulate) {
                        const uint4 *old = reinterpret_cast<const uint4 *>(o + c);
#pragma unroll
                        for (int w = 0; w < 2; ++w) {
                            uint4 x = old[w];
                            const __nv_bfloat162 *xb = reinterpret_cast<const __nv_bfloat162 *>(&x);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                float2 fl = __bfloat1622float2(xb[e]);
                                acc[w * 8 + 2 * e] += fl.x;
                                acc[w * 8 + 2 * e + 1] += fl.y;
                            }
                        }
                    }
                    uint4 w0 = make_uint4(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]),
                                          pack_bf16(acc[4], acc[5]), pack_bf16(acc[6], acc[7]));
                    uint4 w1 = make_uint4(pack_bf16(acc[8], acc[9]), pack_bf16(acc[10], acc[11]),
                                          pack_bf16(acc[12], acc[13]), pack_bf16(acc[14], acc[15]));
                    reinterpret_cast<uint4 *>(o + c)[0] = w0;
                    reinterpret_cast<uint4 *>(o + c)[1] = w1;
                }
            }
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tbase, 512);
    }
}

}  // namespace

size_t output_tc_smem_bytes(int nblk) {
    return 1024 + Smem::G + sizeof(float) * (2 * nblk * BM) + sizeof(uint64_t) * NBAR + 16;
}

cudaError_t launch_output_tc(const CUtensorMap &tm_q, const CUtensorMap &tm_k, const CUtensorMap &tm_u,
                             const CUtensorMap &tm_sig, const OutParams &prm, long long n_fh, cudaStream_t s) {
    const size_t smem = output_tc_smem_bytes(prm.nblk);
    cudaError_t e = cudaFuncSetAttribute(k_output_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long grid = n_fh * prm.nblk;
    k_output_tc<<<(unsigned)grid, kThreads, smem, s>>>(tm_q, tm_k, tm_u, tm_sig, prm);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace gdn
