// tc_diag_inverse.cu -- inverses of the 128x128 diagonal blocks of (I + A).
//
// The intra-frame solve of the chunkwise gated delta rule is the unit lower
// triangular system (I + A)[Ub | W] = [beta V | beta e^G K] with
// A_ij = beta_i e^{G_i - G_j} k_i.k_j (j < i) (the UT/WY form of the delta
// rule over one frame; SANA-WM summary, "Memory-Efficient Long-Context
// Modeling (Section 3.2)", frame-wise GDN).  Blocked forward substitution
// over 128-row blocks needs T_ii = (I + A_ii)^{-1} for every diagonal block.
// They depend neither on each other nor on the solve, so this kernel computes
// all of them ahead of it:
//   1. S = K_i K_i^T on the 5th-generation tensor cores (one 128 x 128 tcgen05
//      product into TMEM; K_i arrives by TMA in the 128-byte-swizzled layout)
//      and A = beta_r e^{G_r - G_s} S (s < r) by the epilogue, one row per thread,
//   2. the eight 16x16 diagonal leaves inverted by forward substitution in
//      fp32 (one column per lane),
//   3. three doubling levels 16 -> 32 -> 64 -> 128,
//        X = A21 T11 (written over A21, which no later level reads),
//        T21 = -T22 X,
//      on mma.sync (the blocks are small and triangular; a dense 128-wide
//      tcgen05 product per level would do 4-8x the work).
// Persistent: one CTA per SM walks the (frame-head, block) items.  Warp 0
// loads K_i by TMA into a 2-slot ring, one thread of warp 1 owns TMEM and
// issues the Gram products, and warps 2-9 form two compute groups of four
// warps that take alternate items, so one group's leaves and doubling overlap
// the other's Gram and loads.  T_ii is written row-major bf16
// [n_fh][nblk][128][128] (unit diagonal, zeros above it), the A operand
// layout of the solve's T_ii Y_i product.  Every wait is bounded.
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kThreads = 320;
constexpr int kGroup = 128;                  // threads per compute group
constexpr int TILE = 128 * 128 * 2;          // one 128x128 bf16 tile (256-byte rows, XOR-swizzled chunks)
constexpr int KSLOT = 2 * SLAB_BYTES;        // K_i: two 64-column SW128 slabs of 128 rows

struct Smem {
    static constexpr uint32_t KR = 0;                        // 2 K slots
    static constexpr uint32_t GRP = KR + 2 * KSLOT;          // per group: A, T, leaves, G, beta
    static constexpr uint32_t A = 0, T = TILE, LEAF = 2 * TILE, GB = LEAF + 8 * 256 * 4;
    static constexpr uint32_t GRP_BYTES = GB + 2 * 128 * 4;
    static constexpr uint32_t END = GRP + 2 * GRP_BYTES;
};

enum Bar { KFULL = 0, KEMPTY = 2, SFULL = 4, SFREE = 6, DRAIN = 8, NBAR = 9 };

// byte offset of (row, col) in a 128x128 bf16 tile: 256-byte rows, 16-byte chunks XOR (row & 7),
// so the eight rows an ldmatrix reads at one column hit eight different bank groups
__device__ __forceinline__ uint32_t toff(int r, int c) {
    return (uint32_t)(r * 256 + ((((c >> 3) ^ (r & 7)) & 15) << 4) + (c & 7) * 2);
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A fragment of the 16x16 block at (r0, c0) of a tile.
__device__ __forceinline__ void load_a(uint32_t (&a)[4], uint32_t tile, int r0, int c0, int lane) {
    const int r = r0 + (lane & 15), c = c0 + (lane >> 4) * 8;
    ldsm_x4(a, tile + toff(r, c));
}
// B fragments (two n8 tiles) of B[k][n] = M[k][n] for a row-major M: rows k0..k0+15, cols n0..n0+15.
__device__ __forceinline__ void load_b_trans(uint32_t (&b)[4], uint32_t tile, int k0, int n0, int lane) {
    // matrices: (k 0-7, n 0-7), (k 8-15, n 0-7), (k 0-7, n 8-15), (k 8-15, n 8-15)
    const int k = k0 + (lane & 7) + ((lane >> 3) & 1) * 8;
    const int n = n0 + (lane >> 4) * 8;
    ldsm_x4_t(b, tile + toff(k, n));
}

// a 16x16 fp32 accumulator pair (two n8 halves) -> bf16 at (r0, c0) of a tile, times `scale`
__device__ __forceinline__ void store16(unsigned char *tile, int r0, int c0, const float (&d0)[4],
                                        const float (&d1)[4], float scale, int lane) {
    const int g = lane >> 2, q = lane & 3;
    *reinterpret_cast<uint32_t *>(tile + toff(r0 + g, c0 + 2 * q)) = pack_bf16(scale * d0[0], scale * d0[1]);
    *reinterpret_cast<uint32_t *>(tile + toff(r0 + g + 8, c0 + 2 * q)) = pack_bf16(scale * d0[2], scale * d0[3]);
    *reinterpret_cast<uint32_t *>(tile + toff(r0 + g, c0 + 8 + 2 * q)) = pack_bf16(scale * d1[0], scale * d1[1]);
    *reinterpret_cast<uint32_t *>(tile + toff(r0 + g + 8, c0 + 8 + 2 * q)) = pack_bf16(scale * d1[2], scale * d1[3]);
}

struct InvParams {
    const float *beta;       // [B,T,H]
    const float *G;          // [n_fh][(L+3)&~3]
    __nv_bfloat16 *Tinv;     // [n_fh][nblk][128][128]
    int L, dk, H, nblk;
    long long F, T, nitems;
    int *err;                // bounded-wait error word
    uint64_t wait_ns;        // limit of the bounded waits
    int drop_first_load;     // debug: withhold the first K load, so its consumer's wait gives up
};

__global__ void __launch_bounds__(kThreads, 1)
k_diag_inverse(const __grid_constant__ CUtensorMap tm_k, const InvParams prm) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = (uint64_t *)(smem + Smem::END);
    uint32_t *tmem_slot = (uint32_t *)(bars + NBAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = prm.L, dk = prm.dk, nblk = prm.nblk;
    int *err = prm.err;
    const uint64_t wait_ns = prm.wait_ns;
    // items of this CTA: w = blockIdx.x + t * gridDim.x, t = 0, 1, ...; group t & 1 takes item t
    const long long nmine = prm.nitems > blockIdx.x ? (prm.nitems - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (pass_failed(prm.err)) return;  // an earlier stage of this pass gave up
    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i) sm100::mbar_init(&bars[i], (i == SFREE || i == SFREE + 1) ? kGroup : 1);
        sm100::fence_barrier_init();
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, 256);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const int nslab_k = (dk + SLAB - 1) / SLAB;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            sm100::tma_prefetch_desc(&tm_k);
            long long issued = 0;
            bool ok = true;
            for (long long t = 0; t < nmine && ok; ++t) {
                const int s = (int)(t & 1);
                // the slot's previous Gram (item t - 2) has read it
                if (t >= 2) ok = sm100::mbar_wait(&bars[KEMPTY + s], (uint32_t)(((t >> 1) - 1) & 1), err, wait_ns);
                if (!ok) break;
                const long long w = blockIdx.x + t * gridDim.x;
                const long long fh = w / nblk;
                const int blk = (int)(w % nblk);
                const long long f = fh % prm.F, chain = fh / prm.F;
                const int h = (int)(chain % prm.H), b = (int)(chain / prm.H);
                const int bf = (int)(b * prm.F + f);
                unsigned char *slot = smem + Smem::KR + s * KSLOT;
                if (t == 0 && prm.drop_first_load) continue;  // debug: the Gram issuer's first wait never completes
                sm100::mbar_arrive_expect_tx(&bars[KFULL + s], (uint32_t)(nslab_k * SLAB_BYTES));
                for (int sl = 0; sl < nslab_k; ++sl)
                    sm100::tma_load_4d(slot + sl * SLAB_BYTES, &tm_k, &bars[KFULL + s], sl * SLAB, h, blk * 128, bf);
                issued = t + 1;
            }
            // leave with no copy in flight: wait for the last two items' loads (full limit)
            for (long long t = issued > 2 ? issued - 2 : 0; t < issued; ++t) {
                if (t == 0 && prm.drop_first_load) continue;
                sm100::mbar_wait(&bars[KFULL + (t & 1)], (uint32_t)((t >> 1) & 1), err, sm100::kWaitLimitNs, true);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ Gram issuer
        if (lane == 0) {
            const uint32_t id = sm100::idesc_bf16(128, 128, 0, 0);
            bool ok = true;
            for (long long t = 0; t < nmine && ok; ++t) {
                const int s = (int)(t & 1);
                ok = sm100::mbar_wait(&bars[KFULL + s], (uint32_t)((t >> 1) & 1), err, wait_ns);
                // the group's TMEM buffer has been read out (item t - 2)
                if (ok && t >= 2) ok = sm100::mbar_wait(&bars[SFREE + s], (uint32_t)(((t >> 1) - 1) & 1), err, wait_ns);
                if (!ok) break;
                sm100::tc_fence_after();
                const unsigned char *kt = smem + Smem::KR + s * KSLOT;
                for (int ks = 0; ks < dk / 16; ++ks)
                    sm100::mma_bf16_ss(tbase + s * 128, desc_kmajor(kt, ks, 128), desc_kmajor(kt, ks, 128), id, ks > 0);
                sm100::mma_commit(&bars[SFULL + s]);
                sm100::mma_commit(&bars[KEMPTY + s]);
            }
            sm100::mma_commit(&bars[DRAIN]);  // every product issued completes before TMEM is released
            sm100::mbar_wait(&bars[DRAIN], 0u, err, sm100::kWaitLimitNs, true);
        }
    } else {
        // ------------------------------------------------------------ compute groups
        const int grp = (warp - 2) >> 2;              // 0: warps 2-5, 1: warps 6-9
        const int gw = (warp - 2) & 3;                // warp within the group
        const int q4 = warp & 3;                      // TMEM lane quadrant of this warp
        const int r = q4 * 32 + lane;                 // the block row this thread reads from TMEM
        const int gt = gw * 32 + lane;                // thread index within the group
        const int bar_id = 1 + grp;                   // named barrier of the group
        unsigned char *g = smem + Smem::GRP + grp * Smem::GRP_BYTES;
        unsigned char *sA = g + Smem::A, *sT = g + Smem::T;
        float *sLeaf = (float *)(g + Smem::LEAF);
        float *sG = (float *)(g + Smem::GB), *sB = sG + 128;
        const uint32_t aA = sm100::smem_u32(sA), aT = sm100::smem_u32(sT);
        const uint32_t tmem = tbase + grp * 128;
        bool ok = true;
        for (long long t = grp; t < nmine && ok; t += 2) {
            const long long w = blockIdx.x + t * gridDim.x;
            const long long fh = w / nblk;
            const int blk = (int)(w % nblk);
            const long long f = fh % prm.F, chain = fh / prm.F;
            const int h = (int)(chain % prm.H), b = (int)(chain / prm.H);
            const int r_base = blk * 128;
            // gates of the block's rows; clear T (its upper triangle stays zero)
            {
                const int rr = r_base + gt;
                const float *Gf = prm.G + fh * (long long)((L + 3) & ~3);
                sG[gt] = Gf[rr < L ? rr : L - 1];
                sB[gt] = rr < L ? prm.beta[((long long)b * prm.T + f * L + rr) * prm.H + h] : 0.f;
#pragma unroll
                for (int c = 0; c < 16; ++c) *reinterpret_cast<uint4 *>(sT + gt * 256 + c * 16) = make_uint4(0, 0, 0, 0);
            }
            named_sync(bar_id, kGroup);
            // ---- A = beta_r e^{G_r - G_s} S[r][s], s < r, from the Gram in TMEM
            ok = sm100::mbar_wait(&bars[SFULL + grp], (uint32_t)((t >> 1) & 1), err, wait_ns);
            ok = named_sync_and(bar_id, kGroup, ok);  // one decision for the whole group
            if (!ok) break;
            sm100::tc_fence_after();
            {
                const float br = sB[r], gr = sG[r];
                const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
#pragma unroll
                for (int c0 = 0; c0 < 128; c0 += 32) {
                    float v[32];
                    sm100::tmem_ld32(tmem + lane_off + c0, v);
                    sm100::tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int s2 = c0 + e;
                        v[e] = s2 < r ? br * __expf(gr - sG[s2]) * v[e] : 0.f;
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        *reinterpret_cast<uint4 *>(sA + toff(r, c0 + 8 * u)) =
                            make_uint4(pack_bf16(v[8 * u], v[8 * u + 1]), pack_bf16(v[8 * u + 2], v[8 * u + 3]),
                                       pack_bf16(v[8 * u + 4], v[8 * u + 5]), pack_bf16(v[8 * u + 6], v[8 * u + 7]));
                    // the fp32 16x16 diagonal block of this row, when it lies in these columns
                    const int db = r >> 4;
                    if (db * 16 >= c0 && db * 16 < c0 + 32) {
                        const bool lo = db * 16 == c0;
#pragma unroll
                        for (int e = 0; e < 16; ++e) sLeaf[db * 256 + (r & 15) * 16 + e] = lo ? v[e] : v[16 + e];
                    }
                }
            }
            sm100::tc_fence_before();
            sm100::mbar_arrive(&bars[SFREE + grp]);  // the TMEM buffer may take the next Gram
            named_sync(bar_id, kGroup);
            // ---- leaves: warp gw inverts diagonal blocks 2 gw (lanes 0-15) and 2 gw + 1 (lanes 16-31);
            //      lane owns one column
            {
                const int blk16 = 2 * gw + (lane >> 4), c = lane & 15;
                const float *ad = sLeaf + blk16 * 256;
                float tcol[16];
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) {
                    float x = (rr == c) ? 1.f : 0.f;
#pragma unroll
                    for (int s2 = 0; s2 < rr; ++s2) x -= ad[rr * 16 + s2] * tcol[s2];
                    tcol[rr] = x;
                }
#pragma unroll
                for (int rr = 0; rr < 16; ++rr)
                    *reinterpret_cast<__nv_bfloat16 *>(sT + toff(blk16 * 16 + rr, blk16 * 16 + c)) =
                        __float2bfloat16_rn(tcol[rr]);
            }
            named_sync(bar_id, kGroup);
            // ---- doubling: X = A21 T11 (over A21), then T21 = -T22 X, for block sizes 16, 32, 64
            for (int sz = 16; sz <= 64; sz <<= 1) {
                const int per = (sz / 16) * (sz / 16);          // 16x16 output tiles per merge
                const int total = (128 / (2 * sz)) * per;       // 4, 8, 16
                const int mine = total / 4;                     // tiles per warp: 1, 2, 4
                for (int pass = 0; pass < 2; ++pass) {
                    // pass 0: X = A21 T11 (A operand sA, B operand sT);  pass 1: T21 = -T22 X (sT, sA)
                    const uint32_t Am = pass ? aT : aA, Bm = pass ? aA : aT;
                    // tile u of this warp: merge m = wt / per, 16x16 tile tt = wt % per, wt = gw + 4u;
                    // output rows base + sz + tr (lower half of the merge), columns base + tc
                    auto tile_rc = [&](int u, int &ra, int &nb, int &base) {
                        const int wt = gw + 4 * u;
                        const int m = wt / per, tt = wt % per;
                        base = m * 2 * sz;
                        ra = base + sz + (tt / (sz / 16)) * 16;
                        nb = base + (tt % (sz / 16)) * 16;
                    };
                    float d[4][2][4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) d[u][0][e] = d[u][1][e] = 0.f;
                        if (u < mine) {
                            int ra, nb, base;
                            tile_rc(u, ra, nb, base);
                            const int ca = pass ? base + sz : base;  // A columns: T22 or A21
                            const int kb = pass ? base + sz : base;  // B rows: X (lower half) or T11
                            for (int k = 0; k < sz; k += 16) {
                                uint32_t af[4], bfr[4];
                                load_a(af, Am, ra, ca + k, lane);
                                load_b_trans(bfr, Bm, kb + k, nb, lane);
                                mma16816(d[u][0], af, bfr[0], bfr[1]);
                                mma16816(d[u][1], af, bfr[2], bfr[3]);
                            }
                        }
                    }
                    // every warp has read its operands before any writes over A21 (pass 0)
                    named_sync(bar_id, kGroup);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        if (u < mine) {
                            int ra, nb, base;
                            tile_rc(u, ra, nb, base);
                            store16(pass ? sT : sA, ra, nb, d[u][0], d[u][1], pass ? -1.f : 1.f, lane);
                        }
                    }
                    named_sync(bar_id, kGroup);
                }
            }
            // ---- write T_ii row-major: thread gt writes 16-byte pieces gt, gt + 128, ... (coalesced)
            __nv_bfloat16 *dst = prm.Tinv + (fh * nblk + blk) * (long long)(128 * 128);
#pragma unroll 4
            for (int e = gt; e < 128 * 16; e += kGroup) {
                const int rr = e >> 4, c8 = e & 15;
                *reinterpret_cast<uint4 *>(dst + rr * 128 + c8 * 8) = *reinterpret_cast<const uint4 *>(sT + toff(rr, c8 * 8));
            }
            named_sync(bar_id, kGroup);  // sT, sA, sG are reused by the group's next item
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tbase, 256);
    }
}

}  // namespace

cudaError_t launch_diag_inverse(const CUtensorMap &tm_k, const float *beta, const float *G, __nv_bfloat16 *Tinv,
                                int L, int dk, int H, int nblk, long long F, long long T, long long n_fh,
                                int *err, uint64_t wait_ns, int drop_first_load, int num_sms, cudaStream_t s) {
    InvParams prm{beta, G, Tinv, L, dk, H, nblk, F, T, n_fh * nblk, err, wait_ns, drop_first_load};
    const size_t smem = 1024 + Smem::END + sizeof(uint64_t) * NBAR + 16;
    cudaError_t e = cudaFuncSetAttribute(k_diag_inverse, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long grid = prm.nitems < num_sms ? prm.nitems : num_sms;
    if (grid <= 0) return cudaSuccess;
    k_diag_inverse<<<(unsigned)grid, kThreads, smem, s>>>(tm_k, prm);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace gdn
