// tc_output.cu -- output stage on the 5th-generation tensor cores.
//
// For one frame-head, block by block (128 rows; rows r, columns s of the frame):
//   o_r = q_r . S_r,  S_r = e^{G_r} Sig + sum_{s <= r} e^{G_r - G_s} k_s^T u_s
// (the output of the chunkwise gated delta rule: the state entering the frame
// plus the frame's own pseudo-values; o_r reads S_r, so the causal mask
// includes the diagonal; SANA-WM summary, "Memory-Efficient Long-Context
// Modeling (Section 3.2)", frame-wise GDN).  The columns before block i enter
// it through the state at the block's anchor a_i (the last token before it),
// carried from block to block:
//   Z_0     = Sig,   Z_{i+1} = e^{G_{a_{i+1}} - G_{a_i}} Z_i + Kh_i^T U_i,
//   Kh_i    = diag(e^{G_{a_{i+1}} - G_s}) K_i                 (every factor <= 1)
//   O_i     = Qt_i Z_i + P_i U_i,   Qt_i = diag(e^{G_r - G_{a_i}}) Q_i,
//   P_i     = causal(Q_i K_i^T o e^{G_r - G_s})               (the diagonal block only)
// so each block costs four 128 x 128 x 128 products (Q_i K_i^T, Qt_i Z_i,
// P_i U_i, Kh_i^T U_i) however many blocks come before it.
//
// One CTA per frame-head.  Warp roles (576 threads): warp 0 issues TMA loads,
// warp 1 owns TMEM and issues tcgen05.mma from one thread, and four epilogue
// groups of four warps (each thread one row, TMEM lane quadrant = warp % 4):
//   A (warps 2-5)   carries the state: Z_i to bf16 for Qt_i Z_i, the fp32 Z
//                   rescaled to the next anchor (the only epilogue step on the
//                   block-to-block chain);
//   B (warps 6-9)   turns S = Q_i K_i^T into bf16 P in tensor memory;
//   C (warps 10-13) scales Q_i, K_i into Qt_i, Kh_i in place;
//   D (warps 14-17) writes O out: as a bf16 tile over Q_i's (Qt_i has been read
//                   by then) that the producer stores with the tensor map of o,
//                   or, when o accumulates or goes out token-reversed, row by
//                   row from registers.
// S of block i+1 is issued while block i is still in the epilogue.
//   TMEM: Z (fp32, lane = key dimension), two S/P buffers, O.
//   SMEM: Q_i (then O_i), K_i, U_i (+ G, cf rows) double-buffered; bf16 Z_i.
// Decay in P: e^{G_r - a} cf_s with cf_s = e^{a - G_s} (a = G at the end of
// s's 64-token group); inside the group the row factor is >= 1, bounded by
// e^60, else the exact e^{G_r - G_s} is taken per element.  Every wait is
// bounded (sm100::mbar_wait); the MMA thread drains its products before TMEM
// is released and the producer its copies.
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kThreads = 576;
constexpr int kGrp = 128;                 // threads per epilogue group
constexpr int TILE = 2 * SLAB_BYTES;      // 128 rows x 2 slabs
constexpr int BUF = 3 * TILE;             // Q, K, U of one block
constexpr float kSplitMax = 60.f;         // largest row exponent the in-group split takes

enum Bar {
    FULL = 0, BFREE = FULL + 2, SFULL = BFREE + 2, SPFREE = SFULL + 2, PREADY = SPFREE + 2, QKREADY = PREADY + 2,
    SREADY = QKREADY + 2, OSTAGED = SREADY + 1, ZFULL = OSTAGED + 2, OFULL, OFREE, DRAIN, NBAR
};

// Small objects first, then the swizzled tiles from a 1024-byte boundary (the dynamic shared
// memory base is itself 1024-aligned; the kernel checks it).
struct Smem {
    static constexpr uint32_t BARS = 0;
    static constexpr uint32_t TSLOT = BARS + NBAR * 8;
    static constexpr uint32_t GC = 1024;                  // 2 x (G[128], cf[128])
    static constexpr uint32_t BUFS = 3072;                // 2 x (Q, K, U)
    static constexpr uint32_t ZB = BUFS + 2 * BUF;        // bf16 Z_i (key dimension x value columns)
    static constexpr uint32_t END = ZB + TILE;
};
static_assert(Smem::TSLOT + 4 <= Smem::GC, "barriers overlap the gate rows");
static_assert(Smem::GC + 2 * 2 * BM * 4 <= Smem::BUFS, "gate rows overlap the tiles");
static_assert(Smem::END <= 232448, "over the 227 KB a CTA may use");

// A row of 16-byte bf16 chunks of a swizzled tile scaled in place by f (0 clears it); the
// row's chunks are read before any is written back, so the loads overlap.
__device__ __forceinline__ void scale_row(unsigned char *tile, int r, int ncols, float f) {
#pragma unroll
    for (int c0 = 0; c0 < 128; c0 += 64) {
        if (c0 >= ncols) break;
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (c0 + 8 * u < ncols) v[u] = *reinterpret_cast<const uint4 *>(tile + sw_offset(c0 + 8 * u, r));
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (c0 + 8 * u >= ncols) break;
            __nv_bfloat162 *h2 = reinterpret_cast<__nv_bfloat162 *>(&v[u]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 x = __bfloat1622float2(h2[e]);
                h2[e] = __floats2bfloat162_rn(f * x.x, f * x.y);
            }
            *reinterpret_cast<uint4 *>(tile + sw_offset(c0 + 8 * u, r)) = v[u];
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
k_output_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_g,
            const __grid_constant__ CUtensorMap tm_cf, const __grid_constant__ CUtensorMap tm_o,
            const OutParams prm) {
    extern __shared__ __align__(1024) unsigned char smem[];
    const int L = prm.L, dk = prm.dk, dv = prm.dv, nblk = prm.nblk;
    const long long fh = blockIdx.x;
    const long long F = prm.F;
    const long long f = fh % F, chain = fh / F;
    const int h = (int)(chain % prm.H), b = (int)(chain / prm.H);
    const int bf = (int)(b * F + f);
    const int gs = (L + 3) & ~3;  // G and cf row stride

    uint64_t *bars = (uint64_t *)(smem + Smem::BARS);
    uint32_t *tmem_slot = (uint32_t *)(smem + Smem::TSLOT);
    float *sGC = (float *)(smem + Smem::GC);
    unsigned char *sZ = smem + Smem::ZB;
    auto sQ = [&](int buf) { return smem + Smem::BUFS + buf * BUF; };
    auto sK = [&](int buf) { return smem + Smem::BUFS + buf * BUF + TILE; };
    auto sU = [&](int buf) { return smem + Smem::BUFS + buf * BUF + 2 * TILE; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int *err = prm.err;
    const uint64_t wait_ns = prm.wait_ns;
    const int nslab_k = (dk + SLAB - 1) / SLAB, nslab_v = (dv + SLAB - 1) / SLAB;

    if (pass_failed(prm.err)) return;  // an earlier stage of this pass gave up
    if (sm100::smem_u32(smem) & 1023u) {  // every thread sees the same base: all leave together
        if (threadIdx.x == 0) atomicCAS(err, sm100::kErrNone, sm100::kErrSmemAlign);
        return;
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i)
            sm100::mbar_init(&bars[i], (i >= PREADY && i < OSTAGED + 2) || i == OFREE ? kGrp : 1);
        sm100::fence_barrier_init();
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, 512);
        sm100::tmem_relinquish();
    }
    if (nslab_k == 1) {  // K_i^T as a 128-row operand: key dimensions past the one loaded slab are zero
        for (int o = threadIdx.x * 16; o < SLAB_BYTES; o += kThreads * 16) {
            *reinterpret_cast<uint4 *>(sK(0) + SLAB_BYTES + o) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sK(1) + SLAB_BYTES + o) = make_uint4(0, 0, 0, 0);
        }
        sm100::fence_proxy_async_smem();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t t_z = tbase, t_sp = tbase + 128, t_o = tbase + 384;  // Z; S/P x 2; O

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            sm100::tma_prefetch_desc(&tm_q);
            sm100::tma_prefetch_desc(&tm_k);
            sm100::tma_prefetch_desc(&tm_u);
            sm100::tma_prefetch_desc(&tm_g);
            sm100::tma_prefetch_desc(&tm_cf);
            if (prm.o_tma) sm100::tma_prefetch_desc(&tm_o);
            // O_u, staged over Q_u's tile by group D, stored with the tensor map of o
            auto store_o = [&](int u) {
                for (int sl = 0; sl < nslab_v; ++sl)
                    sm100::tma_store_4d(&tm_o, sQ(u & 1) + sl * SLAB_BYTES, sl * SLAB, h, u * BM, bf);
                sm100::bulk_commit();
            };
            const uint64_t once = sm100::policy_evict_first();
            const uint32_t bytes = (uint32_t)((2 * nslab_k + nslab_v) * SLAB_BYTES + 2 * BM * 4);
            int j = 0;
            bool ok = true;
            for (; j < nblk && ok; ++j) {  // block j into buffer j & 1 once block j - 2 is done with it
                const int buf = j & 1;
                if (j >= 2) {
                    ok = sm100::mbar_wait(&bars[BFREE + buf], (uint32_t)(((j >> 1) - 1) & 1), err, wait_ns);
                    if (ok && prm.o_tma) {  // block j - 2's O out of Q's tile before Q_j lands there
                        ok = sm100::mbar_wait(&bars[OSTAGED + buf], (uint32_t)(((j >> 1) - 1) & 1), err, wait_ns);
                        if (ok) {
                            store_o(j - 2);
                            sm100::bulk_wait_read0();
                        }
                    }
                }
                if (!ok) break;
                uint64_t *bar = &bars[FULL + buf];
                sm100::mbar_arrive_expect_tx(bar, bytes);
                for (int sl = 0; sl < nslab_k; ++sl) {
                    sm100::tma_load_4d_hint(sQ(buf) + sl * SLAB_BYTES, &tm_q, bar, sl * SLAB, h, j * BM, bf, once);
                    sm100::tma_load_4d_hint(sK(buf) + sl * SLAB_BYTES, &tm_k, bar, sl * SLAB, h, j * BM, bf, once);
                }
                for (int sl = 0; sl < nslab_v; ++sl)
                    sm100::tma_load_3d_hint(sU(buf) + sl * SLAB_BYTES, &tm_u, bar, sl * SLAB, j * BM, (int)fh, once);
                sm100::tma_load_2d(sGC + buf * 2 * BM, &tm_g, bar, j * BM, (int)fh);
                sm100::tma_load_2d(sGC + buf * 2 * BM + BM, &tm_cf, bar, j * BM, (int)fh);
            }
            // the last two blocks' O (no later load waited for them)
            for (int u = nblk > 2 ? nblk - 2 : 0; ok && prm.o_tma && u < nblk; ++u) {
                ok = sm100::mbar_wait(&bars[OSTAGED + (u & 1)], (uint32_t)((u >> 1) & 1), err, wait_ns);
                if (ok) store_o(u);
            }
            if (!ok)  // leave with no copy in flight (full-limit drain waits)
                for (int u = j > 2 ? j - 2 : 0; u < j; ++u)
                    sm100::mbar_wait(&bars[FULL + (u & 1)], (uint32_t)((u >> 1) & 1), err, sm100::kWaitLimitNs, true);
            sm100::bulk_wait0();  // and with no store in flight
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Two streams of products, polled so that neither waits on the other's inputs: S_j =
        // Q_j K_j^T as soon as block j has landed and its S/P buffer is free (at most one block
        // ahead of the O product), and, per block i in order, once P_i, Qt_i / Kh_i and bf16 Z_i
        // (with the rescaled fp32 Z) are ready and O has been drained, O_i = Qt_i Z_i + P_i U_i
        // and Z += Kh_i^T U_i.  Each barrier tested is either at the phase tested for or one
        // before it: its next phase needs a product that has not been issued yet.
        if (lane == 0) {
            const uint32_t id_s = sm100::idesc_bf16(BM, BM, 0, 0);  // Q (K-major) x K^T (K-major)
            const uint32_t id_o = sm100::idesc_bf16(BM, dv, 0, 1);  // Qt or P (K-major) x Z or U (MN-major)
            const uint32_t id_z = sm100::idesc_bf16(BM, dv, 1, 1);  // Kh^T (MN-major) x U (MN-major)
            const int nks_d = dk / 16;
            int js = 0, i = 0;  // next S, next O
            bool ok = true;
            sm100::Spin spin(wait_ns);
            while (ok && i < nblk) {
                bool prog = false;
                if (js < nblk && js <= i + 1 && sm100::mbar_test(&bars[FULL + (js & 1)], (uint32_t)((js >> 1) & 1)) &&
                    (js < 2 || sm100::mbar_test(&bars[SPFREE + (js & 1)], (uint32_t)(((js >> 1) - 1) & 1)))) {
                    const int buf = js & 1;
                    sm100::tc_fence_after();
                    for (int ks = 0; ks < nks_d; ++ks)
                        sm100::mma_bf16_ss(t_sp + buf * 128, desc_kmajor(sQ(buf), ks, BM), desc_kmajor(sK(buf), ks, BM),
                                           id_s, ks > 0);
                    sm100::mma_commit(&bars[SFULL + buf]);
                    ++js;
                    prog = true;
                }
                const int buf = i & 1;
                if (js > i && sm100::mbar_test(&bars[PREADY + buf], (uint32_t)((i >> 1) & 1)) &&
                    sm100::mbar_test(&bars[QKREADY + buf], (uint32_t)((i >> 1) & 1)) &&
                    sm100::mbar_test(&bars[SREADY], (uint32_t)(i & 1)) &&
                    (i == 0 || sm100::mbar_test(&bars[OFREE], (uint32_t)((i - 1) & 1)))) {
                    sm100::tc_fence_after();
                    // O_i = Qt_i Z_i + P_i U_i (P of tokens 0..63 in TMEM columns 0..31 of the buffer,
                    // tokens 64..127 in 64..95)
                    for (int ks = 0; ks < nks_d; ++ks)
                        sm100::mma_bf16_ss(t_o, desc_kmajor(sQ(buf), ks, BM), desc_mnmajor(sZ, ks, BM), id_o, ks > 0);
                    for (int ks = 0; ks < BM / 16; ++ks)
                        sm100::mma_bf16_ts(t_o, t_sp + buf * 128 + (ks >> 2) * 64 + (ks & 3) * 8,
                                           desc_mnmajor(sU(buf), ks, BM), id_o, 1u);
                    sm100::mma_commit(&bars[OFULL]);
                    sm100::mma_commit(&bars[SPFREE + buf]);
                    if (i + 1 < nblk) {  // Z_{i+1}: the fp32 Z was rescaled to a_{i+1} with Z_i's bf16 copy
                        for (int ks = 0; ks < BM / 16; ++ks)
                            sm100::mma_bf16_ss(t_z, desc_mnmajor(sK(buf), ks, BM), desc_mnmajor(sU(buf), ks, BM), id_z,
                                               1u);
                        sm100::mma_commit(&bars[ZFULL]);
                    }
                    sm100::mma_commit(&bars[BFREE + buf]);
                    ++i;
                    prog = true;
                }
                if (prog) spin.reset();
                else if (!spin.tick(err)) ok = false;
            }
            sm100::mma_commit(&bars[DRAIN]);  // every product issued completes before TMEM is released
            sm100::mbar_wait(&bars[DRAIN], 0u, err, sm100::kWaitLimitNs, true);
        }
    } else {
        const int grp = (warp - 2) >> 2;  // 0 A, 1 B, 2 C, 3 D
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;  // TMEM lane: block row (token), or key dimension of Z
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const int n16 = dv >> 4;       // d_v is a multiple of 16
        bool ok = true;
        if (grp == 0) {
            // -------------------------------------------------------- A: the state
            const float *Gf = prm.G + fh * (long long)gs;
            auto gend = [&](int j) { return Gf[min((j + 1) * BM, L) - 1]; };  // G at the last token of block j
            float gA = 0.f;  // G at the anchor of block i (block 0: the frame's start, G = 0)
            float gE = gend(0);
            for (int i = 0; i < nblk && ok; ++i) {
                const float gE_next = i + 1 < nblk ? gend(i + 1) : 0.f;  // read a block ahead
                const bool carry = i + 1 < nblk;
                const float gam = __expf(gE - gA);  // Z_i -> anchor a_{i+1}
                if (i == 0) {
                    // Z_0 = Sig: the bf16 copy is the scan's own; fp32 (rescaled) into TMEM
                    const __nv_bfloat16 *sig = prm.SigB + (fh * dk + (r < dk ? r : 0)) * (long long)dv;
                    for (int c16 = 0; c16 < n16; ++c16) {
                        uint4 w[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
                        if (r < dk) {
                            w[0] = reinterpret_cast<const uint4 *>(sig + 16 * c16)[0];
                            w[1] = reinterpret_cast<const uint4 *>(sig + 16 * c16)[1];
                        }
                        *reinterpret_cast<uint4 *>(sZ + sw_offset(16 * c16, r)) = w[0];
                        *reinterpret_cast<uint4 *>(sZ + sw_offset(16 * c16 + 8, r)) = w[1];
                        if (carry) {
                            uint32_t zs[16];
                            const __nv_bfloat162 *z2 = reinterpret_cast<const __nv_bfloat162 *>(w);
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const float2 zf = __bfloat1622float2(z2[e]);
                                zs[2 * e] = __float_as_uint(gam * zf.x);
                                zs[2 * e + 1] = __float_as_uint(gam * zf.y);
                            }
                            sm100::tmem_st16(t_z + lane_off + 16 * c16, zs);
                        }
                    }
                } else {
                    ok = sm100::mbar_wait(&bars[ZFULL], (uint32_t)((i - 1) & 1), err, wait_ns);
                    if (!ok) break;
                    sm100::tc_fence_after();
                    tmem_walk16(t_z + lane_off, n16, [&](int c16, const float (&x)[16]) {
                        *reinterpret_cast<uint4 *>(sZ + sw_offset(16 * c16, r)) = pack8(x);
                        *reinterpret_cast<uint4 *>(sZ + sw_offset(16 * c16 + 8, r)) = pack8(x + 8);
                        if (carry) {
                            uint32_t zs[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) zs[e] = __float_as_uint(gam * x[e]);
                            sm100::tmem_st16(t_z + lane_off + 16 * c16, zs);
                        }
                    });
                }
                sm100::tmem_st_wait();
                sm100::tc_fence_before();
                sm100::fence_proxy_async_smem();
                sm100::mbar_arrive(&bars[SREADY]);
                gA = gE;
                gE = gE_next;
            }
        } else if (grp == 1) {
            // -------------------------------------------------------- B: P
            for (int i = 0; i < nblk && ok; ++i) {
                const int buf = i & 1;
                ok = sm100::mbar_wait(&bars[FULL + buf], (uint32_t)((i >> 1) & 1), err, wait_ns) &&
                     sm100::mbar_wait(&bars[SFULL + buf], (uint32_t)((i >> 1) & 1), err, wait_ns);
                if (!ok) break;
                sm100::tc_fence_after();
                const float *gJ = sGC + buf * 2 * BM, *cfJ = gJ + BM;
                const int nrow = min(BM, L - i * BM);
                const bool valid = r < nrow;
                const float Gr = valid ? gJ[r] : 0.f;
                // P = causal(S o e^{G_r - G_s}) over the two 64-token groups of the block: a row before
                // a group sees none of it, a row after it all of it, a row inside it the columns
                // s <= r.  Decay e^{G_r - a} cf_s (a = G at the group's last token, which cf was
                // made with); inside the group e^{G_r - a} >= 1, so a row whose exponent exceeds
                // kSplitMax takes the exact e^{G_r - G_s} instead.
                float rfh[2];
                bool inh[2], exh[2];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const bool none = r < 64 * hh;
                    inh[hh] = !none && r < 64 * hh + 64;
                    const float dG = Gr - gJ[min(64 * hh + 63, nrow - 1)];
                    exh[hh] = inh[hh] && !(dG <= kSplitMax);
                    rfh[hh] = (valid && !none && !exh[hh]) ? __expf(dG) : 0.f;
                }
                const uint32_t t_s = t_sp + buf * 128 + lane_off;
                uint32_t pk[16];
                // P of each 32 S columns goes, packed, over the first 16 of them (already read)
                tmem_walk16(t_s, 8, [&](int c16, const float (&v)[16]) {
                    const bool g1 = c16 >= 4;
                    const int c0 = 16 * c16;
                    const bool in_g = g1 ? inh[1] : inh[0], ex = g1 ? exh[1] : exh[0];
                    const float rf = g1 ? rfh[1] : rfh[0];
                    uint32_t q[8];
                    if (!ex) {  // rf = 0 where the row sees none of the group
                        float cf[16];  // the chunk's column factors, four 16-byte reads
#pragma unroll
                        for (int q4c = 0; q4c < 4; ++q4c) {
                            const float4 t4 = reinterpret_cast<const float4 *>(cfJ + c0)[q4c];
                            cf[4 * q4c] = t4.x, cf[4 * q4c + 1] = t4.y, cf[4 * q4c + 2] = t4.z, cf[4 * q4c + 3] = t4.w;
                        }
#pragma unroll
                        for (int e = 0; e < 16; e += 2) {
                            float f0 = rf * cf[e], f1 = rf * cf[e + 1];
                            if (in_g) {
                                f0 = c0 + e <= r ? f0 : 0.f;
                                f1 = c0 + e + 1 <= r ? f1 : 0.f;
                            }
                            q[e >> 1] = pack_bf16(v[e] * f0, v[e + 1] * f1);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; e += 2) {
                            const int s0 = c0 + e;
                            const float f0 = (s0 <= r && s0 < nrow) ? __expf(Gr - gJ[s0]) : 0.f;
                            const float f1 = (s0 + 1 <= r && s0 + 1 < nrow) ? __expf(Gr - gJ[s0 + 1]) : 0.f;
                            q[e >> 1] = pack_bf16(v[e] * f0, v[e + 1] * f1);
                        }
                    }
                    if (c16 & 1) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) pk[8 + e] = q[e];
                        sm100::tmem_st16(t_s + 64 * (c16 >> 2) + 16 * ((c16 & 3) >> 1), pk);
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) pk[e] = q[e];
                    }
                });
                sm100::tmem_st_wait();
                sm100::tc_fence_before();
                sm100::mbar_arrive(&bars[PREADY + buf]);
            }
        } else if (grp == 2) {
            // -------------------------------------------------------- C: Qt, Kh
            float gA = 0.f;  // G at the anchor of block i
            for (int i = 0; i < nblk && ok; ++i) {
                const int buf = i & 1;
                ok = sm100::mbar_wait(&bars[FULL + buf], (uint32_t)((i >> 1) & 1), err, wait_ns) &&
                     sm100::mbar_wait(&bars[SFULL + buf], (uint32_t)((i >> 1) & 1), err, wait_ns);
                if (!ok) break;
                const float *gJ = sGC + buf * 2 * BM;
                const int nrow = min(BM, L - i * BM);
                const bool valid = r < nrow;
                const float Gr = valid ? gJ[r] : 0.f, gEnd = gJ[nrow - 1];
                // Qt_i = diag(e^{G_r - G_{a_i}}) Q_i and (for Z_{i+1}) Kh_i = diag(e^{G_{a_{i+1}} - G_r}) K_i,
                // in place now that S_i has read them; rows past the frame become zero
                scale_row(sQ(buf), r, dk, valid ? __expf(Gr - gA) : 0.f);
                if (i + 1 < nblk) scale_row(sK(buf), r, dk, valid ? __expf(gEnd - Gr) : 0.f);
                sm100::fence_proxy_async_smem();
                sm100::mbar_arrive(&bars[QKREADY + buf]);
                gA = gEnd;
            }
        } else {
            // -------------------------------------------------------- D: O out
            // through Q_j's tile and the producer's tiled store; else row by row (rows past the frame
            // are not stored; a reversed scan's rows go back in place)
            for (int j = 0; j < nblk && ok; ++j) {
                ok = sm100::mbar_wait(&bars[OFULL], (uint32_t)(j & 1), err, wait_ns);
                if (!ok) break;
                sm100::tc_fence_after();
                if (prm.o_tma) {  // O_j's product has read Qt_j: its tile takes O_j
                    unsigned char *so = sQ(j & 1);
                    tmem_walk16(t_o + lane_off, n16, [&](int c16, const float (&x)[16]) {
                        *reinterpret_cast<uint4 *>(so + sw_offset(16 * c16, r)) = pack8(x);
                        *reinterpret_cast<uint4 *>(so + sw_offset(16 * c16 + 8, r)) = pack8(x + 8);
                    });
                    sm100::tc_fence_before();
                    sm100::mbar_arrive(&bars[OFREE]);
                    sm100::fence_proxy_async_smem();
                    sm100::mbar_arrive(&bars[OSTAGED + (j & 1)]);
                    continue;
                }
                const int row = j * BM + r;
                const bool valid = row < L;
                const long long tt0 = f * L + row;
                const long long tt = prm.reverse_out ? prm.T - 1 - tt0 : tt0;
                __nv_bfloat16 *o = (__nv_bfloat16 *)prm.o + ((((long long)b * prm.T + tt) * prm.H + h) * dv);
                tmem_walk16(t_o + lane_off, n16, [&](int c16, const float (&x)[16]) {
                    if (!valid) return;
                    float y[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) y[e] = x[e];
                    uint4 *dst = reinterpret_cast<uint4 *>(o + 16 * c16);
                    if (prm.accumulate) {
#pragma unroll
                        for (int w2 = 0; w2 < 2; ++w2) {
                            uint4 old = dst[w2];
                            const __nv_bfloat162 *ob = reinterpret_cast<const __nv_bfloat162 *>(&old);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 fl = __bfloat1622float2(ob[e]);
                                y[8 * w2 + 2 * e] += fl.x;
                                y[8 * w2 + 2 * e + 1] += fl.y;
                            }
                        }
                    }
                    dst[0] = pack8(y);
                    dst[1] = pack8(y + 8);
                });
                sm100::tc_fence_before();
                sm100::mbar_arrive(&bars[OFREE]);
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

cudaError_t launch_output_tc(const CUtensorMap &tm_q, const CUtensorMap &tm_k, const CUtensorMap &tm_u,
                             const CUtensorMap &tm_g, const CUtensorMap &tm_cf, const CUtensorMap &tm_o,
                             const OutParams &prm, cudaStream_t s) {
    const size_t smem = Smem::END;
    cudaError_t e = cudaFuncSetAttribute(k_output_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_output_tc<<<(unsigned)prm.n_fh, kThreads, smem, s>>>(tm_q, tm_k, tm_u, tm_g, tm_cf, tm_o, prm);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace gdn
