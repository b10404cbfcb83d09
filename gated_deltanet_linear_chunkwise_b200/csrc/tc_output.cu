// tc_output.cu -- output stage on the 5th-generation tensor cores.
//
// For one 128-row block I of one frame-head (rows r, columns s of the frame):
//   O_I = diag(e^G) Q_I Sig + sum_{J <= I} P_IJ U_J,
//   P_IJ[r][s] = (q_r . k_s) e^{G_r - G_s}  for s <= r (inclusive: o_r reads S_r)
// (the intra-frame term of the chunkwise gated delta rule; SANA-WM summary,
// "Memory-Efficient Long-Context Modeling (Section 3.2)", frame-wise GDN).
//
// Persistent kernel: one CTA per SM walks (frame-head, block) items in
// frame-head order (neighbouring CTAs share a frame's K and U tiles in L2),
// with TMEM and barriers set up once.
// Warp roles (320 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues tcgen05.mma from one thread, warps 2-9 are the epilogue: two
// warpgroups, each thread owning one tile row (TMEM lane quadrant =
// warp % 4) and one half of the tile's columns.
//   TMEM: two S/P buffers (128 columns each) and two O buffers (128 each).
//         The epilogue turns S (fp32) into P (bf16) in place -- each
//         column half into the first 32 TMEM columns of its own range --
//         and the O += P U product reads P straight from tensor memory.
//   SMEM: Q_I double buffer; a 2-stage ring of (K_J, U_J, G_J, cf_J) tiles.
// The state term is a pseudo-tile in front of the J tiles: the epilogue
// writes Q~ = diag(e^G) Q_I into an S/P buffer and the ring delivers Sig
// (bf16, MN-major) in the U slot, so O starts as Q~ Sig.  Off-diagonal
// decay factors are e^{G_r - a} cf_s with cf_s = e^{a - G_s} (a = G at the
// end of s's 64-token tile, both <= 1); the diagonal tile takes
// e^{G_r - G_s} per element.  Every wait is bounded (sm100::mbar_wait).
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kThreads = 320;
constexpr int kEpi = 256;  // epilogue threads
constexpr int GC_BYTES = 2 * BM * 4;  // G and cf of one 128-column tile

struct Smem {
    static constexpr uint32_t Q = 0;                       // 2 stages x 2 slabs
    static constexpr uint32_t K = Q + 4 * SLAB_BYTES;      // 2 stages x 2 slabs
    static constexpr uint32_t U = K + 4 * SLAB_BYTES;      // 2 stages x 2 slabs (Sig in the pseudo-tile)
    static constexpr uint32_t GC = U + 4 * SLAB_BYTES;     // 2 stages x (G[128], cf[128])
    static constexpr uint32_t END = GC + 2 * GC_BYTES;
};

enum Bar { QFULL0, QFULL1, QEMPTY0, QEMPTY1, RFULL0, RFULL1, REMPTY0, REMPTY1, SFULL0, SFULL1, SFREE0, SFREE1,
           PFULL0, PFULL1, OFULL0, OFULL1, OEMPTY0, OEMPTY1, NBAR };

__global__ void __launch_bounds__(kThreads, 1)
k_output_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_sig,
            const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_cf,
            const OutParams prm) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int L = prm.L, dk = prm.dk, dv = prm.dv, nblk = prm.nblk;
    const long long F = prm.F, nfh = prm.n_fh, nitems = nfh * nblk;
    const int gs = (L + 3) & ~3;  // row stride of G and cf

    unsigned char *sQ = smem + Smem::Q;
    unsigned char *sK = smem + Smem::K;
    unsigned char *sU = smem + Smem::U;
    float *sGC = (float *)(smem + Smem::GC);
    uint64_t *bars = (uint64_t *)(smem + Smem::END);
    uint32_t *tmem_slot = (uint32_t *)(bars + NBAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int *err = prm.err;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i) {
            uint32_t cnt = 1;
            if (i == PFULL0 || i == PFULL1 || i == OEMPTY0 || i == OEMPTY1) cnt = kEpi;
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
    const uint32_t t_s0 = tbase, t_o0 = tbase + 256;

    const int nks_d = dk / 16;
    const int nslab_k = (dk + SLAB - 1) / SLAB, nslab_v = (dv + SLAB - 1) / SLAB;

    // item w: frame-head w / nblk, block nblk-1 - w % nblk (heaviest block of a frame first)
    auto item_blk = [&](long long w) { return nblk - 1 - (int)(w % nblk); };
    auto item_fh = [&](long long w) { return w / nblk; };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            sm100::tma_prefetch_desc(&tm_q);
            sm100::tma_prefetch_desc(&tm_k);
            sm100::tma_prefetch_desc(&tm_u);
            sm100::tma_prefetch_desc(&tm_sig);
            sm100::tma_prefetch_desc(&tm_g);
            sm100::tma_prefetch_desc(&tm_cf);
            bool ok = true;
            int n = 0, t = 0;
            for (long long w = blockIdx.x; w < nitems && ok; w += gridDim.x, ++t) {
                const int I = item_blk(w);
                const long long fh = item_fh(w);
                const long long f = fh % F, chain = fh / F;
                const int h = (int)(chain % prm.H), b = (int)(chain / prm.H);
                const int bf = (int)(b * F + f);
                const int qb = t & 1;
                if (t >= 2) ok = sm100::mbar_wait(&bars[QEMPTY0 + qb], ((t - 2) >> 1) & 1, err);
                if (!ok) break;
                sm100::mbar_arrive_expect_tx(&bars[QFULL0 + qb], (uint32_t)(nslab_k * SLAB_BYTES));
                for (int sl = 0; sl < nslab_k; ++sl)
                    sm100::tma_load_4d(sQ + (qb * 2 + sl) * SLAB_BYTES, &tm_q, &bars[QFULL0 + qb], sl * SLAB, h,
                                       I * BM, bf);
                for (int J = -1; J <= I && ok; ++J, ++n) {
                    const int st = n & 1;
                    if (n >= 2) ok = sm100::mbar_wait(&bars[REMPTY0 + st], ((n - 2) >> 1) & 1, err);
                    if (!ok) break;
                    unsigned char *ut = sU + st * 2 * SLAB_BYTES;
                    if (J < 0) {  // the state term: Sig in the U slot
                        sm100::mbar_arrive_expect_tx(&bars[RFULL0 + st], (uint32_t)(nslab_v * dk * 128));
                        for (int sl = 0; sl < nslab_v; ++sl)
                            sm100::tma_load_3d(ut + sl * dk * 128, &tm_sig, &bars[RFULL0 + st], sl * SLAB, 0,
                                               (int)fh);
                    } else {
                        sm100::mbar_arrive_expect_tx(&bars[RFULL0 + st],
                                                     (uint32_t)((nslab_k + nslab_v) * SLAB_BYTES + GC_BYTES));
                        for (int sl = 0; sl < nslab_k; ++sl)
                            sm100::tma_load_4d(sK + (st * 2 + sl) * SLAB_BYTES, &tm_k, &bars[RFULL0 + st], sl * SLAB,
                                               h, J * BM, bf);
                        for (int sl = 0; sl < nslab_v; ++sl)
                            sm100::tma_load_3d(ut + sl * SLAB_BYTES, &tm_u, &bars[RFULL0 + st], sl * SLAB, J * BM,
                                               (int)fh);
                        float *gc = sGC + st * 2 * BM;
                        sm100::tma_load_2d(gc, &tm_g, &bars[RFULL0 + st], J * BM, (int)fh);
                        sm100::tma_load_2d(gc + BM, &tm_cf, &bars[RFULL0 + st], J * BM, (int)fh);
                    }
                }
            }
            // leave with no copy in flight: the last item's MMAs consumed everything
            if (ok && t >= 1) sm100::mbar_wait(&bars[QEMPTY0 + ((t - 1) & 1)], ((t - 1) >> 1) & 1, err);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_s = sm100::idesc_bf16(BM, BM, 0, 0);
            const uint32_t id_o = sm100::idesc_bf16(BM, dv, 0, 1);
            bool ok = true;
            int n = 0, sc = 0, t = 0;
            for (long long w = blockIdx.x; w < nitems && ok; w += gridDim.x, ++t) {
                const int I = item_blk(w);
                const int ob = t & 1, qb = t & 1;
                const uint32_t t_o = t_o0 + ob * 128;
                const unsigned char *qt = sQ + qb * 2 * SLAB_BYTES;
                // ---- state pseudo-tile: hand an S/P buffer to the epilogue, then O = Q~ Sig
                int sb = sc & 1, st = n & 1;
                if (sc >= 2) ok = sm100::mbar_wait(&bars[SFREE0 + sb], ((sc - 2) >> 1) & 1, err);
                if (!ok) break;
                sm100::mma_commit(&bars[SFULL0 + sb]);
                ok = sm100::mbar_wait(&bars[RFULL0 + st], (n >> 1) & 1, err) &&
                     sm100::mbar_wait(&bars[PFULL0 + sb], (sc >> 1) & 1, err);
                if (ok && t >= 2) ok = sm100::mbar_wait(&bars[OEMPTY0 + ob], ((t - 2) >> 1) & 1, err);
                if (!ok) break;
                sm100::tc_fence_after();
                for (int ks = 0; ks < nks_d; ++ks)
                    sm100::mma_bf16_ts(t_o, t_s0 + sb * 128 + ks * 8, desc_mnmajor(sU + st * 2 * SLAB_BYTES, ks, dk),
                                       id_o, ks > 0);
                sm100::mma_commit(&bars[SFREE0 + sb]);
                sm100::mma_commit(&bars[REMPTY0 + st]);
                ++n;
                ++sc;
                // ---- J tiles: S = Q K^T, then O += P U one tile behind
                int psb = 0, pst = 0, psc = 0;
                auto issue_pu = [&]() -> bool {
                    if (!sm100::mbar_wait(&bars[PFULL0 + psb], (psc >> 1) & 1, err)) return false;
                    sm100::tc_fence_after();
                    const unsigned char *u = sU + pst * 2 * SLAB_BYTES;
                    // P columns k = 0..63 sit in TMEM columns 0..31, k = 64..127 in columns 64..95
                    for (int ks = 0; ks < BM / 16; ++ks)
                        sm100::mma_bf16_ts(t_o, t_s0 + psb * 128 + ks * 8 + (ks >> 2) * 32, desc_mnmajor(u, ks, BM),
                                           id_o, 1u);
                    sm100::mma_commit(&bars[SFREE0 + psb]);
                    sm100::mma_commit(&bars[REMPTY0 + pst]);
                    return true;
                };
                if (ok) ok = sm100::mbar_wait(&bars[QFULL0 + qb], (t >> 1) & 1, err);
                for (int J = 0; J <= I && ok; ++J, ++n, ++sc) {
                    sb = sc & 1;
                    st = n & 1;
                    ok = sm100::mbar_wait(&bars[RFULL0 + st], (n >> 1) & 1, err);
                    if (ok && sc >= 2) ok = sm100::mbar_wait(&bars[SFREE0 + sb], ((sc - 2) >> 1) & 1, err);
                    if (!ok) break;
                    sm100::tc_fence_after();
                    const unsigned char *kt = sK + st * 2 * SLAB_BYTES;
                    for (int ks = 0; ks < nks_d; ++ks)
                        sm100::mma_bf16_ss(t_s0 + sb * 128, desc_kmajor(qt, ks, BM), desc_kmajor(kt, ks, BM), id_s,
                                           ks > 0);
                    sm100::mma_commit(&bars[SFULL0 + sb]);
                    if (J >= 1) ok = issue_pu();
                    psb = sb;
                    pst = st;
                    psc = sc;
                }
                if (ok) ok = issue_pu();
                if (!ok) break;
                sm100::mma_commit(&bars[OFULL0 + ob]);
                sm100::mma_commit(&bars[QEMPTY0 + qb]);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Order: pseudo(0), tiles(0), pseudo(1), drain(0), tiles(1), pseudo(2), drain(1), ...
        // so one item's O drains while the tensor cores work on the next.
        const int q4 = warp & 3;                  // TMEM lane quadrant
        const int r = q4 * 32 + lane;             // tile row owned by this thread
        const int half = (warp - 2) >> 2;         // which half of the tile's columns
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        int sc = 0, n = 0;
        struct Item {
            int I, h, b, row;
            long long fh, f;
            bool valid;
            float Gr;
        };
        auto item_of = [&](long long w) {
            Item it;
            it.I = item_blk(w);
            it.fh = item_fh(w);
            it.f = it.fh % F;
            const long long chain = it.fh / F;
            it.h = (int)(chain % prm.H);
            it.b = (int)(chain / prm.H);
            it.row = it.I * BM + r;
            it.valid = it.row < L;
            it.Gr = prm.G[it.fh * (long long)gs + (it.valid ? it.row : L - 1)];
            return it;
        };
        // one 16-column group of Q~ = e^G q_r (32 bf16 of this thread's row), read from the swizzled Q tile
        auto q_group = [&](int qb, int c16, float eg, uint32_t (&pk)[16]) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int lc = c16 * 4 + u;  // logical 8-column chunk
                if (lc * 8 < dk) {
                    const int sl = lc >> 3, cc = lc & 7;
                    uint4 v = *reinterpret_cast<const uint4 *>(sQ + (qb * 2 + sl) * SLAB_BYTES + r * 128 +
                                                               ((cc ^ (r & 7)) << 4));
                    __nv_bfloat162 *p2 = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x = __bfloat1622float2(p2[e]);
                        pk[u * 4 + e] = pack_bf16(eg * x.x, eg * x.y);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) pk[u * 4 + e] = 0u;
                }
            }
        };
        // state pseudo-tile: P <- diag(e^G) Q_I, written into the S/P buffer as bf16
        auto pseudo = [&](const Item &it, int t) -> bool {
            const int qb = t & 1, sb = sc & 1;
            if (!sm100::mbar_wait(&bars[SFULL0 + sb], (sc >> 1) & 1, err)) return false;
            if (!sm100::mbar_wait(&bars[QFULL0 + qb], (t >> 1) & 1, err)) return false;
            sm100::tc_fence_after();
            const float eg = it.valid ? __expf(it.Gr) : 0.f;
            for (int c16 = half; c16 * 32 < dk; c16 += 2) {  // 32 bf16 -> 16 TMEM columns per group
                uint32_t pk[16];
                q_group(qb, c16, eg, pk);
                sm100::tmem_st16(t_s0 + sb * 128 + lane_off + c16 * 16, pk);
            }
            sm100::tmem_st_wait();
            sm100::tc_fence_before();
            sm100::mbar_arrive(&bars[PFULL0 + sb]);
            ++sc;
            ++n;  // the pseudo-tile's ring slot
            return true;
        };
        auto tiles = [&](const Item &it) -> bool {
            for (int J = 0; J <= it.I; ++J, ++sc, ++n) {
                const int sb = sc & 1, st = n & 1;
                const bool diag = (J == it.I);
                if (!sm100::mbar_wait(&bars[SFULL0 + sb], (sc >> 1) & 1, err)) return false;
                if (!sm100::mbar_wait(&bars[RFULL0 + st], (n >> 1) & 1, err)) return false;  // this tile's G, cf
                sm100::tc_fence_after();
                const float *gJ = sGC + st * 2 * BM, *cfJ = gJ + BM;
                // this half's 64 columns share one 64-token anchor
                const float rf = it.valid ? __expf(it.Gr - gJ[64 * half + 63]) : 0.f;
#pragma unroll 1
                for (int c = 2 * half; c < 2 * half + 2; ++c) {
                    float v[32];
                    sm100::tmem_ld32(t_s0 + sb * 128 + lane_off + c * 32, v);
                    sm100::tmem_ld_wait();
                    uint32_t pk[16];
                    if (!diag) {
#pragma unroll
                        for (int e = 0; e < 32; e += 2)
                            pk[e >> 1] = pack_bf16(v[e] * rf * cfJ[c * 32 + e], v[e + 1] * rf * cfJ[c * 32 + e + 1]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const int s = J * BM + c * 32 + e;
                            const float f0 = (s <= it.row && s < L) ? __expf(it.Gr - gJ[c * 32 + e]) : 0.f;
                            const float f1 = (s + 1 <= it.row && s + 1 < L) ? __expf(it.Gr - gJ[c * 32 + e + 1]) : 0.f;
                            pk[e >> 1] = pack_bf16(v[e] * f0, v[e + 1] * f1);
                        }
                    }
                    // P (bf16 pairs) of this half's 64 columns goes to TMEM columns
                    // [64 half, 64 half + 32): S columns this half has already read
                    sm100::tmem_st16(t_s0 + sb * 128 + lane_off + 64 * half + (c - 2 * half) * 16, pk);
                }
                sm100::tmem_st_wait();
                sm100::tc_fence_before();
                sm100::mbar_arrive(&bars[PFULL0 + sb]);
            }
            return true;
        };
        auto drain = [&](const Item &it, int t) -> bool {
            const int ob = t & 1;
            if (!sm100::mbar_wait(&bars[OFULL0 + ob], (t >> 1) & 1, err)) return false;
            sm100::tc_fence_after();
            const long long tt = it.f * L + it.row;
            __nv_bfloat16 *o = (__nv_bfloat16 *)prm.o + ((((long long)it.b * prm.T + tt) * prm.H + it.h) * dv);
            for (int c = 16 * half; c < dv; c += 32) {
                float acc[16];
                sm100::tmem_ld16(t_o0 + ob * 128 + lane_off + c, acc);
                sm100::tmem_ld_wait();
                if (it.valid) {
                    if (prm.accumulate) {
                        const uint4 *old = reinterpret_cast<const uint4 *>(o + c);
#pragma unroll
                        for (int w2 = 0; w2 < 2; ++w2) {
                            uint4 x = old[w2];
                            const __nv_bfloat162 *xb = reinterpret_cast<const __nv_bfloat162 *>(&x);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 fl = __bfloat1622float2(xb[e]);
                                acc[w2 * 8 + 2 * e] += fl.x;
                                acc[w2 * 8 + 2 * e + 1] += fl.y;
                            }
                        }
                    }
                    reinterpret_cast<uint4 *>(o + c)[0] =
                        make_uint4(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]), pack_bf16(acc[4], acc[5]),
                                   pack_bf16(acc[6], acc[7]));
                    reinterpret_cast<uint4 *>(o + c)[1] =
                        make_uint4(pack_bf16(acc[8], acc[9]), pack_bf16(acc[10], acc[11]),
                                   pack_bf16(acc[12], acc[13]), pack_bf16(acc[14], acc[15]));
                }
            }
            sm100::tc_fence_before();
            sm100::mbar_arrive(&bars[OEMPTY0 + ob]);
            return true;
        };
        long long w = blockIdx.x;
        bool ok = w < nitems;
        Item cur;
        if (ok) {
            cur = item_of(w);
            ok = pseudo(cur, 0);
        }
        for (int t = 0; ok; ++t) {
            ok = tiles(cur);
            if (!ok) break;
            const long long wn = w + gridDim.x;
            Item nxt;
            if (wn < nitems) {
                nxt = item_of(wn);
                ok = pseudo(nxt, t + 1);
                if (!ok) break;
            }
            ok = drain(cur, t);
            if (!ok || wn >= nitems) break;
            w = wn;
            cur = nxt;
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

cudaError_t launch_output_tc(const CUtensorMap &tm_q, const CUtensorMap &tm_k, const CUtensorMap &tm_u,
                             const CUtensorMap &tm_sig, const CUtensorMap &tm_g, const CUtensorMap &tm_cf,
                             const OutParams &prm, int num_sms, cudaStream_t s) {
    const size_t smem = 1024 + Smem::END + sizeof(uint64_t) * NBAR + 16;
    cudaError_t e = cudaFuncSetAttribute(k_output_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long nitems = prm.n_fh * prm.nblk;
    const long long grid = nitems < num_sms ? nitems : num_sms;
    k_output_tc<<<(unsigned)grid, kThreads, smem, s>>>(tm_q, tm_k, tm_u, tm_sig, tm_g, tm_cf, prm);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace gdn
