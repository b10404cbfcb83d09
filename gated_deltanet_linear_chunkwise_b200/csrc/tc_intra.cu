// tc_intra.cu -- intra-frame blocked forward substitution on the tensor cores.
//
// Solves, per frame-head, the unit lower triangular system of the chunkwise
// gated delta rule (one chunk per frame; SANA-WM summary,
// "Memory-Efficient Long-Context Modeling (Section 3.2)", frame-wise GDN):
//   (I + A) X = R,   X = [Ub | W],   R = [beta V | beta e^G K],
//   A_rs = beta_r e^{G_r - G_s} k_r.k_s  (s < r)
// over 128-row blocks i, in order:
//   acc_i = sum_{64-token tiles j before block i} P_ij X_j,  P_ij = -A_ij
//   Y_i   = R_i + acc_i
//   X_i   = T_ii Y_i,   T_ii = (I + A_ii)^{-1}  (from tc_diag_inverse.cu)
// X_i is staged in shared memory (over K_i and T_ii, both dead by then) and
// stored by TMA to the [n_fh][L][d_v + d_k] bf16 workspace, from where later
// blocks load it again (L2-resident).
//
// Warp roles (320 threads): warp 0 TMA, warp 1 TMEM owner + MMA issuer,
// warps 2-9 epilogue (two warpgroups; one block row and one column half
// per thread).
//   TMEM: four S/P buffers (64 columns each; the epilogue turns S into the
//         bf16 P in place and acc += P X_j reads P from tensor memory) and
//         acc / X_i (d_v + d_k columns).
//   SMEM: K_i, T_ii, and a 3-deep ring of (K_j, X_j, G_j, cf_j) tiles; Y_i
//         aliases the first two ring slots during the diagonal step, the
//         bf16 X_i the K_i and T_ii buffers until its TMA store has read it.
// Decay factors use a per-tile anchor a = G at the tile's last token:
// e^{G_r - G_s} = e^{G_r - a} e^{a - G_s}, both <= 1.
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kThreads = 320;
constexpr int kEpi = 256;                    // epilogue threads
constexpr int JT = 64;                       // tokens per off-diagonal tile
constexpr int NSLOT = 3;                     // ring depth
constexpr int NSB = 4;                       // S/P buffers in TMEM
constexpr int KJ_SLAB = JT * 128;            // 64-row slab
constexpr int SLOT_BYTES = 6 * KJ_SLAB;      // K_j (2 slabs) + X_j (4 slabs)
constexpr int GC_BYTES = 2 * JT * 4;         // G and cf of one tile

struct Smem {
    static constexpr uint32_t KI = 0;                          // 2 slabs x 128 rows
    static constexpr uint32_t T = KI + 2 * SLAB_BYTES;         // 2 slabs x 128 rows
    static constexpr uint32_t RING = T + 2 * SLAB_BYTES;       // NSLOT x 48 KB; Y_i (64 KB) aliases the start
    static constexpr uint32_t GC = RING + NSLOT * SLOT_BYTES;  // NSLOT x (G[64], cf[64])
    static constexpr uint32_t END = GC + NSLOT * GC_BYTES;
};
static_assert(2 * SLOT_BYTES >= 4 * SLAB_BYTES, "Y_i must fit in the first two ring slots");

enum Bar {
    KIFULL = 0, TFULL, ACCFULL, YFULL, XFULL, ACCFREE, XSTAGED,
    KXFULL, KXEMPTY = KXFULL + NSLOT, SFULL = KXEMPTY + NSLOT, SFREE = SFULL + NSB, PFULL = SFREE + NSB,
    NBAR = PFULL + NSB
};

__global__ void __launch_bounds__(kThreads, 1)
k_intra_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_x,
           const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_g,
           const __grid_constant__ CUtensorMap tm_cf, const __grid_constant__ CUtensorMap tm_xs,
           const IntraParams prm) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int L = prm.L, dk = prm.dk, dv = prm.dv, nc = dk + dv, nblk = prm.nblk;
    const long long fh = blockIdx.x;
    const long long F = prm.F;
    const long long f = fh % F, chain = fh / F;
    const int h = (int)(chain % prm.H), b = (int)(chain / prm.H);
    const int bf = (int)(b * F + f);

    unsigned char *sKi = smem + Smem::KI;
    unsigned char *sT = smem + Smem::T;
    unsigned char *sRing = smem + Smem::RING;
    unsigned char *sY = sRing;
    unsigned char *sXs = smem + Smem::KI;  // X_i staging: K_i and T_ii, 4 slabs of 128 rows
    static_assert(Smem::T == Smem::KI + 2 * SLAB_BYTES, "the staging slabs must be contiguous");
    float *sGC = (float *)(smem + Smem::GC);
    uint64_t *bars = (uint64_t *)(smem + Smem::END);
    uint32_t *tmem_slot = (uint32_t *)(bars + NBAR);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int *err = prm.err;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i) {
            const bool epi = i == YFULL || i == ACCFREE || i == XSTAGED || (i >= PFULL && i < PFULL + NSB);
            sm100::mbar_init(&bars[i], epi ? kEpi : 1);
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
    const uint32_t t_s0 = tbase, t_acc = tbase + 256;
    const int nks_d = dk / 16;
    const int nslab_k = (dk + SLAB - 1) / SLAB;
    const int nslab_x = (nc + SLAB - 1) / SLAB;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            sm100::tma_prefetch_desc(&tm_k);
            sm100::tma_prefetch_desc(&tm_x);
            sm100::tma_prefetch_desc(&tm_t);
            sm100::tma_prefetch_desc(&tm_g);
            sm100::tma_prefetch_desc(&tm_cf);
            sm100::tma_prefetch_desc(&tm_xs);
            bool ok = true;
            int n = 0;
            auto load_tile = [&](int jt, int i) -> bool {
                const int st = n % NSLOT;
                if (n >= NSLOT && !sm100::mbar_wait(&bars[KXEMPTY + st], ((n / NSLOT) - 1) & 1, err)) return false;
                if (jt == 2 * (i - 1)) sm100::bulk_wait0();  // the rows of X_{i-1} are in global memory
                unsigned char *slot = sRing + st * SLOT_BYTES;
                sm100::mbar_arrive_expect_tx(&bars[KXFULL + st], (uint32_t)((nslab_k + nslab_x) * KJ_SLAB + GC_BYTES));
                for (int sl = 0; sl < nslab_k; ++sl)
                    sm100::tma_load_4d(slot + sl * KJ_SLAB, &tm_k, &bars[KXFULL + st], sl * SLAB, h, jt * JT, bf);
                for (int sl = 0; sl < nslab_x; ++sl)
                    sm100::tma_load_3d(slot + (2 + sl) * KJ_SLAB, &tm_x, &bars[KXFULL + st], sl * SLAB, jt * JT,
                                       (int)fh);
                float *gc = sGC + st * 2 * JT;
                sm100::tma_load_2d(gc, &tm_g, &bars[KXFULL + st], jt * JT, (int)fh);
                sm100::tma_load_2d(gc + JT, &tm_cf, &bars[KXFULL + st], jt * JT, (int)fh);
                ++n;
                return true;
            };
            // store the staged X_{i}: rows past the frame and columns past d_v + d_k are clipped
            auto store_x = [&](int i) -> bool {
                if (!sm100::mbar_wait(&bars[XSTAGED], i & 1, err)) return false;
                for (int sl = 0; sl < nslab_x; ++sl)
                    sm100::tma_store_3d(&tm_xs, sXs + sl * SLAB_BYTES, sl * SLAB, i * BM, (int)fh);
                sm100::bulk_commit();
                sm100::bulk_wait_read0();
                return true;
            };
            for (int i = 0; i < nblk && ok; ++i) {
                int jt = 0;
                if (i >= 1) {
                    // Y_{i-1} is consumed once X_{i-1} = T Y is in TMEM: the ring may refill
                    ok = sm100::mbar_wait(&bars[XFULL], (i - 1) & 1, err);
                    const int pre = min(2 * i - 2, NSLOT);  // tiles that do not read X_{i-1}
                    for (; jt < pre && ok; ++jt) ok = load_tile(jt, i);
                    // K_i and T_ii overwrite the staging buffer once the store has read it
                    if (ok) ok = store_x(i - 1);
                }
                if (!ok) break;
                sm100::mbar_arrive_expect_tx(&bars[KIFULL], (uint32_t)(nslab_k * SLAB_BYTES));
                for (int sl = 0; sl < nslab_k; ++sl)
                    for (int hf = 0; hf < 2; ++hf)
                        sm100::tma_load_4d(sKi + sl * SLAB_BYTES + hf * KJ_SLAB, &tm_k, &bars[KIFULL], sl * SLAB, h,
                                           i * BM + hf * JT, bf);
                sm100::mbar_arrive_expect_tx(&bars[TFULL], (uint32_t)(2 * SLAB_BYTES));
                for (int sl = 0; sl < 2; ++sl)
                    sm100::tma_load_3d(sT + sl * SLAB_BYTES, &tm_t, &bars[TFULL], sl * SLAB, 0, (int)(fh * nblk + i));
                for (; jt < 2 * i && ok; ++jt) ok = load_tile(jt, i);
            }
            if (ok) ok = store_x(nblk - 1);
            sm100::bulk_wait0();  // leave with no store in flight
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_s = sm100::idesc_bf16(BM, JT, 0, 0);
            const uint32_t id_x = sm100::idesc_bf16(BM, nc, 0, 1);
            bool ok = true;
            int n = 0;
            auto issue_px = [&](int m, bool first_of_block, int i) -> bool {
                const int pb = m % NSB, st = m % NSLOT;
                if (!sm100::mbar_wait(&bars[PFULL + pb], (m / NSB) & 1, err)) return false;
                // the first product of a block overwrites acc: X_{i-1} must have been read out
                if (first_of_block && i >= 1 && !sm100::mbar_wait(&bars[ACCFREE], (i - 1) & 1, err)) return false;
                sm100::tc_fence_after();
                const unsigned char *xt = sRing + st * SLOT_BYTES + 2 * KJ_SLAB;
                // P columns k = 0..31 sit in TMEM columns 0..15, k = 32..63 in columns 32..47
                for (int ks = 0; ks < JT / 16; ++ks)
                    sm100::mma_bf16_ts(t_acc, t_s0 + pb * JT + ks * 8 + (ks >> 1) * 16, desc_mnmajor(xt, ks, JT),
                                       id_x, (first_of_block && ks == 0) ? 0u : 1u);
                sm100::mma_commit(&bars[SFREE + pb]);
                sm100::mma_commit(&bars[KXEMPTY + st]);
                return true;
            };
            for (int i = 0; i < nblk && ok; ++i) {
                ok = sm100::mbar_wait(&bars[KIFULL], i & 1, err);
                const int first = n;
                for (int jt = 0; jt < 2 * i && ok; ++jt, ++n) {
                    const int st = n % NSLOT, sb = n % NSB;
                    ok = sm100::mbar_wait(&bars[KXFULL + st], (n / NSLOT) & 1, err);
                    if (ok && n >= NSB) ok = sm100::mbar_wait(&bars[SFREE + sb], ((n / NSB) - 1) & 1, err);
                    if (!ok) break;
                    sm100::tc_fence_after();
                    const unsigned char *kt = sRing + st * SLOT_BYTES;
                    for (int ks = 0; ks < nks_d; ++ks)
                        sm100::mma_bf16_ss(t_s0 + sb * JT, desc_kmajor(sKi, ks, BM), desc_kmajor(kt, ks, JT), id_s,
                                           ks > 0);
                    sm100::mma_commit(&bars[SFULL + sb]);
                    if (jt >= 1) ok = issue_px(n - 1, n - 1 == first, i);
                }
                if (ok && i >= 1) ok = issue_px(n - 1, n - 1 == first, i);
                if (!ok) break;
                sm100::mma_commit(&bars[ACCFULL]);
                ok = sm100::mbar_wait(&bars[YFULL], i & 1, err) && sm100::mbar_wait(&bars[TFULL], i & 1, err);
                if (!ok) break;
                sm100::tc_fence_after();
                for (int ks = 0; ks < BM / 16; ++ks)
                    sm100::mma_bf16_ss(t_acc, desc_kmajor(sT, ks, BM), desc_mnmajor(sY, ks, BM), id_x, ks > 0);
                sm100::mma_commit(&bars[XFULL]);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Two warpgroups: each thread owns one block row (TMEM lane quadrant =
        // warp % 4) and one half of the columns -- 32 of the 64 columns of an
        // off-diagonal tile, and in the diagonal step the Ub columns (half 0,
        // which needs v) or the W columns (half 1, which needs k).
        const int q4 = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r = q4 * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const float *Gf = prm.G + fh * (long long)((L + 3) & ~3);  // G rows are padded to 16 bytes

        bool ok = true;
        int n = 0;
        for (int i = 0; i < nblk && ok; ++i) {
            const int row = i * BM + r;
            const bool valid = row < L;
            const float Gr = valid ? Gf[row] : 0.f;
            const long long t = f * L + row;
            const long long tok = ((long long)b * prm.T + t) * prm.H + h;
            const float be = valid ? prm.beta[tok] : 0.f;
            // half 0 needs this row's values in the diagonal step: pull them into L2 now
            const __nv_bfloat16 *vp = prm.v + tok * dv;
            if (half == 0 && valid)
                for (int by = 0; by < dv * 2; by += 128)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"((const char *)vp + by));
            if (half == 0 && valid) asm volatile("prefetch.global.L2 [%0];" ::"l"((const char *)vp + dv * 2 - 1));

            for (int jt = 0; jt < 2 * i && ok; ++jt, ++n) {
                const int sb = n % NSB, st = n % NSLOT;
                ok = sm100::mbar_wait(&bars[SFULL + sb], (n / NSB) & 1, err) &&
                     sm100::mbar_wait(&bars[KXFULL + st], (n / NSLOT) & 1, err);  // G_j, cf_j
                if (!ok) break;
                sm100::tc_fence_after();
                // the tile is full (it lies before block i): its anchor is G at token 63
                const float *gj = sGC + st * 2 * JT;
                const float rf = valid ? -be * __expf(Gr - gj[JT - 1]) : 0.f;
                const float *cf = gj + JT + 32 * half;
                float v[32];
                sm100::tmem_ld32(t_s0 + sb * JT + lane_off + 32 * half, v);
                sm100::tmem_ld_wait();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) pk[e >> 1] = pack_bf16(rf * cf[e] * v[e], rf * cf[e + 1] * v[e + 1]);
                // this half's P goes to TMEM columns [32 half, 32 half + 16): S columns it has read
                sm100::tmem_st16(t_s0 + sb * JT + lane_off + 32 * half, pk);
                sm100::tmem_st_wait();
                sm100::tc_fence_before();
                sm100::mbar_arrive(&bars[PFULL + sb]);
            }
            if (!ok) break;
            // ---- Y_i = R_i + acc_i  -> sY (MN-major: row = K index of the T_ii Y_i product)
            ok = sm100::mbar_wait(&bars[ACCFULL], i & 1, err);
            if (!ok) break;
            sm100::tc_fence_after();
            auto store_y = [&](int c, const float (&y)[8]) {
                const uint4 val = valid ? make_uint4(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]),
                                                     pack_bf16(y[4], y[5]), pack_bf16(y[6], y[7]))
                                        : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(sY + (c >> 6) * SLAB_BYTES + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4)) = val;
            };
            if (half == 0) {  // Ub columns: beta_r v_r + acc
                uint4 vrow[16];
#pragma unroll
                for (int c8 = 0; c8 < 16; ++c8)
                    vrow[c8] = (valid && c8 < dv / 8) ? __ldg(reinterpret_cast<const uint4 *>(vp) + c8)
                                                      : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int c16 = 16 * j;
                    if (c16 >= dv) break;
                    float acc[16];
                    if (i > 0) {
                        sm100::tmem_ld16(t_acc + lane_off + c16, acc);
                        sm100::tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) acc[e] = 0.f;
                    }
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const __nv_bfloat162 *vb = reinterpret_cast<const __nv_bfloat162 *>(&vrow[2 * j + u]);
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 fv = __bfloat1622float2(vb[e]);
                            y[2 * e] = be * fv.x + acc[u * 8 + 2 * e];
                            y[2 * e + 1] = be * fv.y + acc[u * 8 + 2 * e + 1];
                        }
                        store_y(c16 + 8 * u, y);
                    }
                }
            } else {  // W columns: beta_r e^{G_r} k_r + acc
                const float rk = be * __expf(Gr);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int kc16 = 16 * j;
                    if (kc16 >= dk) break;
                    float acc[16];
                    if (i > 0) {
                        sm100::tmem_ld16(t_acc + lane_off + dv + kc16, acc);
                        sm100::tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) acc[e] = 0.f;
                    }
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int kc = kc16 + 8 * u;
                        const uint4 kv = *reinterpret_cast<const uint4 *>(
                            sKi + (kc >> 6) * SLAB_BYTES + r * 128 + ((((kc & 63) >> 3) ^ (r & 7)) << 4));
                        const __nv_bfloat162 *kb = reinterpret_cast<const __nv_bfloat162 *>(&kv);
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 fk = __bfloat1622float2(kb[e]);
                            y[2 * e] = rk * fk.x + acc[u * 8 + 2 * e];
                            y[2 * e + 1] = rk * fk.y + acc[u * 8 + 2 * e + 1];
                        }
                        store_y(dv + kc, y);
                    }
                }
            }
            sm100::tc_fence_before();
            sm100::fence_proxy_async_smem();
            sm100::mbar_arrive(&bars[YFULL]);
            // ---- X_i = T_ii Y_i  -> bf16 staging (same layout as Y; half 0 the Ub columns, half 1 the W columns)
            ok = sm100::mbar_wait(&bars[XFULL], i & 1, err);
            if (!ok) break;
            sm100::tc_fence_after();
            const int c_lo = half ? dv : 0, c_hi = half ? nc : dv;
            for (int c16 = c_lo; c16 < c_hi; c16 += 16) {
                float x[16];
                sm100::tmem_ld16(t_acc + lane_off + c16, x);
                sm100::tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int c = c16 + 8 * u;
                    *reinterpret_cast<uint4 *>(sXs + (c >> 6) * SLAB_BYTES + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4)) =
                        make_uint4(pack_bf16(x[8 * u], x[8 * u + 1]), pack_bf16(x[8 * u + 2], x[8 * u + 3]),
                                   pack_bf16(x[8 * u + 4], x[8 * u + 5]), pack_bf16(x[8 * u + 6], x[8 * u + 7]));
                }
            }
            sm100::tc_fence_before();
            sm100::mbar_arrive(&bars[ACCFREE]);
            sm100::fence_proxy_async_smem();
            sm100::mbar_arrive(&bars[XSTAGED]);
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

cudaError_t launch_intra_tc(const CUtensorMap &tm_k, const CUtensorMap &tm_x, const CUtensorMap &tm_t,
                            const CUtensorMap &tm_g, const CUtensorMap &tm_cf, const CUtensorMap &tm_xs,
                            const IntraParams &prm, long long n_fh, cudaStream_t s) {
    const size_t smem = 1024 + Smem::END + sizeof(uint64_t) * NBAR + 16;
    cudaError_t e = cudaFuncSetAttribute(k_intra_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_intra_tc<<<(unsigned)n_fh, kThreads, smem, s>>>(tm_k, tm_x, tm_t, tm_g, tm_cf, tm_xs, prm);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace gdn
