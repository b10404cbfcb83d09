// tc_output.cu -- output stage on the 5th-generation tensor cores.
//
// For one 128-row block I of one frame-head (rows r, columns s of the frame):
//   O_I = diag(e^G) Q_I Sig + sum_{s <= r} (q_r . k_s) e^{G_r - G_s} u_s
// (the intra-frame term of the chunkwise gated delta rule; o_r reads S_r, so
// the causal mask includes the diagonal; SANA-WM summary, "Memory-Efficient
// Long-Context Modeling (Section 3.2)", frame-wise GDN).
//
// Persistent kernel: one CTA per SM walks a contiguous range of (frame-head,
// block) items (ranges balanced by tile count), so a frame's K and U tiles
// come from HBM once and are re-read from L2 by the same CTA for the frame's
// other blocks; TMEM and barriers are set up once.  The columns s come in
// 128-token tiles through a 2-deep ring (a tensor-core instruction costs the
// same for every N up to 128, so S = Q K^T is issued with N = 128); the MMA
// thread issues each tile's
// S = Q K^T as soon as its data and an S/P buffer are there and each O += P U
// as soon as the epilogue has written P (polling both in one loop).
// Warp roles (320 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues tcgen05.mma from one thread, warps 2-9 are the epilogue: two
// warpgroups, each thread owning one tile row (TMEM lane quadrant =
// warp % 4) and one 64-column half of each tile.
//   TMEM: two S/P buffers (128 columns each) and two O buffers (128 each).
//         The epilogue turns S (fp32) into P (bf16) in place -- each half
//         into the first 32 TMEM columns of its own range -- and O += P U
//         reads P straight from tensor memory.
//   SMEM: Q_I double buffer; 2 ring slots of (K_j, U_j) + (G_j, cf_j).
// The state term is a pseudo-tile in front of the column tiles: the epilogue
// writes Q~ = diag(e^G) Q_I into an S/P buffer and a ring slot delivers Sig
// (bf16, MN-major), so O starts as Q~ Sig.  Off-diagonal decay factors are
// e^{G_r - a} cf_s with cf_s = e^{a - G_s} (a = G at the end of s's 64-token
// group, both <= 1); in the diagonal group the row factor is >= 1, bounded by
// e^60, else the exact e^{G_r - G_s} is taken per element.  Every wait is
// bounded (sm100::mbar_wait).
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kThreads = 320;
constexpr int kEpi = 256;                 // epilogue threads
constexpr int JT = 128;                   // tokens per column tile (= BM: tile I is block I's diagonal)
constexpr int NSLOT = 3;                  // ring depth
constexpr int NSB = 2;                    // S/P buffers in TMEM
constexpr int JSLAB = JT * 128;           // one 128-row slab
constexpr int SLOT_BYTES = 4 * JSLAB;     // K (2 slabs) + U (2 slabs); or an item's Q (2 slabs) + Sig (<= 32 KB)
constexpr int GC_BYTES = 2 * JT * 4;      // G and cf of one tile
constexpr float kSplitMax = 60.f;         // largest row exponent the in-group split takes

struct Smem {
    static constexpr uint32_t RING = 0;                       // NSLOT x 64 KB
    static constexpr uint32_t GC = RING + NSLOT * SLOT_BYTES; // NSLOT x (G[128], cf[128])
    static constexpr uint32_t END = GC + NSLOT * GC_BYTES;
};

enum Bar {
    RFULL = 0, REMPTY = RFULL + NSLOT, SFULL = REMPTY + NSLOT, SFREE = SFULL + NSB, PFULL = SFREE + NSB,
    OFULL = PFULL + NSB, OEMPTY = OFULL + 1, QFREE = OEMPTY + 1, DRAIN = QFREE + 2, NBAR = DRAIN + 1
};

__global__ void __launch_bounds__(kThreads, 1)
k_output_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_sig,
            const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_cf,
            const OutParams prm) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int L = prm.L, dk = prm.dk, dv = prm.dv, nblk = prm.nblk;
    const long long F = prm.F, nfh = prm.n_fh, nitems = nfh * nblk;
    const int gs = (L + 3) & ~3;           // row stride of G and cf
    const int ntile_frame = (L + JT - 1) / JT;

    unsigned char *sRing = smem + Smem::RING;
    float *sGC = (float *)(smem + Smem::GC);
    uint64_t *bars = (uint64_t *)(smem + Smem::END);
    uint32_t *tmem_slot = (uint32_t *)(bars + NBAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int *err = prm.err;

    if (pass_failed(prm.err)) return;  // an earlier stage of this pass gave up
    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i) {
            const bool epi = (i >= PFULL && i < PFULL + NSB) || i == OEMPTY;
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
    // TMEM: two S/P buffers (128 columns each), the O accumulator (128), and the item's Q in two
    // buffers of 64 columns (two bf16 per column: the A operand of S = Q K^T, read from TMEM)
    const uint32_t t_s0 = tbase, t_o = tbase + 256, t_q0 = tbase + 384;

    const int nks_d = dk / 16;
    const int nslab_k = (dk + SLAB - 1) / SLAB, nslab_v = (dv + SLAB - 1) / SLAB;

    // item w: frame-head w / nblk, block nblk-1 - w % nblk (heaviest block of a frame first);
    // its column tiles are j = 0 .. I, the last one being the diagonal block
    auto item_blk = [&](long long w) { return nblk - 1 - (int)(w % nblk); };
    auto item_fh = [&](long long w) { return w / nblk; };
    auto item_ntiles = [&](int I) { return min(I + 1, ntile_frame); };
    // CTA c takes items [item_start(c), item_start(c + 1)): equal shares of the
    // total weight, an item weighing its tiles plus two (state term, drain)
    auto item_start = [&](long long c) -> long long {
        long long wfh = 0;
        for (int I = 0; I < nblk; ++I) wfh += item_ntiles(I) + 2;
        const long long target = (c * wfh * nfh + gridDim.x - 1) / gridDim.x;
        const long long fh = target / wfh;
        long long rem = target - fh * wfh;
        int k = 0;
        while (k < nblk && rem > 0) rem -= item_ntiles(nblk - 1 - k++) + 2;
        return min(fh * nblk + k, nitems);
    };
    const long long w_begin = item_start(blockIdx.x), w_end = item_start(blockIdx.x + 1);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            sm100::tma_prefetch_desc(&tm_q);
            sm100::tma_prefetch_desc(&tm_k);
            sm100::tma_prefetch_desc(&tm_u);
            sm100::tma_prefetch_desc(&tm_sig);
            sm100::tma_prefetch_desc(&tm_g);
            sm100::tma_prefetch_desc(&tm_cf);
            // L2 policies: a frame's K and U tiles are read again by its other blocks, Q once
            const uint64_t keep = sm100::policy_evict_last(), once = sm100::policy_evict_first();
            bool ok = true;
            int n = 0, t = 0;
            for (long long w = w_begin; w < w_end && ok; ++w, ++t) {
                const int I = item_blk(w);
                const long long fh = item_fh(w);
                const long long f = fh % F, chain = fh / F;
                const int h = (int)(chain % prm.H), b = (int)(chain / prm.H);
                const int bf = (int)(b * F + f);
                const int nt = item_ntiles(I);
                for (int j = -1; j < nt && ok; ++j, ++n) {
                    const int st = n % NSLOT;
                    if (n >= NSLOT) ok = sm100::mbar_wait(&bars[REMPTY + st], ((n / NSLOT) - 1) & 1, err);
                    if (!ok) break;
                    unsigned char *slot = sRing + st * SLOT_BYTES;
                    if (j < 0) {  // the item's Q (2 slabs) and the state term's Sig (after them)
                        sm100::mbar_arrive_expect_tx(&bars[RFULL + st],
                                                     (uint32_t)(nslab_k * JSLAB + nslab_v * dk * 128));
                        for (int sl = 0; sl < nslab_k; ++sl)
                            sm100::tma_load_4d_hint(slot + sl * JSLAB, &tm_q, &bars[RFULL + st], sl * SLAB, h, I * BM,
                                                    bf, once);
                        for (int sl = 0; sl < nslab_v; ++sl)
                            sm100::tma_load_3d(slot + 2 * JSLAB + sl * dk * 128, &tm_sig, &bars[RFULL + st], sl * SLAB,
                                               0, (int)fh);
                    } else {
                        sm100::mbar_arrive_expect_tx(&bars[RFULL + st],
                                                     (uint32_t)((nslab_k + nslab_v) * JSLAB + GC_BYTES));
                        for (int sl = 0; sl < nslab_k; ++sl)
                            sm100::tma_load_4d_hint(slot + sl * JSLAB, &tm_k, &bars[RFULL + st], sl * SLAB, h, j * JT, bf,
                                                    keep);
                        for (int sl = 0; sl < nslab_v; ++sl)
                            sm100::tma_load_3d_hint(slot + (2 + sl) * JSLAB, &tm_u, &bars[RFULL + st], sl * SLAB, j * JT,
                                                    (int)fh, keep);
                        float *gc = sGC + st * 2 * JT;
                        sm100::tma_load_2d(gc, &tm_g, &bars[RFULL + st], j * JT, (int)fh);
                        sm100::tma_load_2d(gc + JT, &tm_cf, &bars[RFULL + st], j * JT, (int)fh);
                    }
                }
            }
            // leave with no copy in flight: the last NSLOT uses of the ring have landed (full limit)
            for (int u = n > NSLOT ? n - NSLOT : 0; u < n; ++u)
                sm100::mbar_wait(&bars[RFULL + (u % NSLOT)], (uint32_t)((u / NSLOT) & 1), err, sm100::kWaitLimitNs,
                                 true);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_s = sm100::idesc_bf16(BM, JT, 0, 0);
            const uint32_t id_o = sm100::idesc_bf16(BM, dv, 0, 1);
            bool ok = true;
            int n = 0, sc = 0, t = 0;
            for (long long w = w_begin; w < w_end && ok; ++w, ++t) {
                const int I = item_blk(w);
                const int nt = item_ntiles(I);
                const int qb = t & 1;
                // ---- state pseudo-tile: hand an S/P buffer to the epilogue, which writes
                //      Q~ = diag(e^G) Q there and Q into TMEM buffer qb
                const int sb0 = sc % NSB, st0 = n % NSLOT, sc0 = sc;
                if (sc >= NSB) ok = sm100::mbar_wait(&bars[SFREE + sb0], ((sc / NSB) - 1) & 1, err);
                if (!ok) break;
                sm100::mma_commit(&bars[SFULL + sb0]);
                ++n;
                ++sc;
                // ---- then, polling: O = Q~ Sig once Q~ is written and the previous item's O has
                //      drained; S = Q K^T (Q from TMEM) as soon as Q, a tile and an S/P buffer are
                //      ready; O += P U (after O = Q~ Sig) as soon as the epilogue has written P
                const int n0 = n, s0 = sc;
                int js = 0, jp = 0;
                bool q_ready = false, o_started = false;
                sm100::Spin spin;
                while (ok && jp < nt) {
                    bool prog = false;
                    if (!q_ready && sm100::mbar_test(&bars[PFULL + sb0], (uint32_t)((sc0 / NSB) & 1))) {
                        q_ready = true;
                        prog = true;
                    }
                    if (q_ready && !o_started && (t == 0 || sm100::mbar_test(&bars[OEMPTY], (uint32_t)((t - 1) & 1)))) {
                        sm100::tc_fence_after();
                        const unsigned char *sig = sRing + st0 * SLOT_BYTES + 2 * JSLAB;
                        for (int ks = 0; ks < nks_d; ++ks)
                            sm100::mma_bf16_ts(t_o, t_s0 + sb0 * JT + ks * 8, desc_mnmajor(sig, ks, dk), id_o, ks > 0);
                        sm100::mma_commit(&bars[SFREE + sb0]);
                        sm100::mma_commit(&bars[REMPTY + st0]);
                        o_started = true;
                        prog = true;
                    }
                    if (q_ready && js < nt && js - jp < NSB) {  // the buffer's previous product has been issued
                        const int cs = s0 + js, nn = n0 + js;
                        const int sb = cs % NSB, st = nn % NSLOT;
                        if (sm100::mbar_test(&bars[RFULL + st], (nn / NSLOT) & 1) &&
                            (cs < NSB || sm100::mbar_test(&bars[SFREE + sb], ((cs / NSB) - 1) & 1))) {
                            sm100::tc_fence_after();
                            const unsigned char *kt = sRing + st * SLOT_BYTES;
                            for (int ks = 0; ks < nks_d; ++ks)
                                sm100::mma_bf16_ts(t_s0 + sb * JT, t_q0 + qb * 64 + ks * 8, desc_kmajor(kt, ks, JT),
                                                   id_s, ks > 0);
                            sm100::mma_commit(&bars[SFULL + sb]);
                            ++js;
                            if (js == nt) sm100::mma_commit(&bars[QFREE + qb]);  // Q buffer qb may be rewritten
                            prog = true;
                        }
                    }
                    if (o_started && jp < js) {
                        const int cs = s0 + jp, nn = n0 + jp;
                        const int pb = cs % NSB, pst = nn % NSLOT;
                        if (sm100::mbar_test(&bars[PFULL + pb], (cs / NSB) & 1)) {
                            sm100::tc_fence_after();
                            const unsigned char *u = sRing + pst * SLOT_BYTES + 2 * JSLAB;
                            // P columns k = 0..63 sit in TMEM columns 0..31, k = 64..127 in columns 64..95
                            for (int ks = 0; ks < JT / 16; ++ks)
                                sm100::mma_bf16_ts(t_o, t_s0 + pb * JT + ks * 8 + (ks >> 2) * 32,
                                                   desc_mnmajor(u, ks, JT), id_o, 1u);
                            sm100::mma_commit(&bars[SFREE + pb]);
                            sm100::mma_commit(&bars[REMPTY + pst]);
                            ++jp;
                            prog = true;
                        }
                    }
                    if (prog) spin.reset();
                    else if (!spin.tick(err)) ok = false;
                }
                n = n0 + nt;
                sc = s0 + nt;
                if (!ok) break;
                sm100::mma_commit(&bars[OFULL]);
            }
            sm100::mma_commit(&bars[DRAIN]);  // every product issued completes before TMEM is released
            sm100::mbar_wait(&bars[DRAIN], 0u, err, sm100::kWaitLimitNs, true);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Order: pseudo(0), tiles(0), pseudo(1), drain(0), tiles(1), pseudo(2), drain(1), ...
        // so one item's O drains while the tensor cores work on the next.
        const int q4 = warp & 3;                  // TMEM lane quadrant
        const int r = q4 * 32 + lane;             // tile row owned by this thread
        const int half = (warp - 2) >> 2;         // which 32-column half of each tile
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        int sc = 0, n = 0;
        struct Item {
            int I, h, b, row, nt;
            long long fh, f;
            bool valid;
            float Gr;
        };
        auto item_of = [&](long long w) {
            Item it;
            it.I = item_blk(w);
            it.nt = item_ntiles(it.I);
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
        // state pseudo-tile: P <- diag(e^G) Q_I, written into the S/P buffer as bf16
        auto pseudo = [&](const Item &it, int t) -> bool {
            const int qb = t & 1, sb = sc % NSB, st = n % NSLOT;
            if (!sm100::mbar_wait(&bars[SFULL + sb], (sc / NSB) & 1, err)) return false;
            if (!sm100::mbar_wait(&bars[RFULL + st], (n / NSLOT) & 1, err)) return false;  // Q and Sig
            // Q buffer qb: the S products of item t - 2 that read it have completed
            if (t >= 2 && !sm100::mbar_wait(&bars[QFREE + qb], (uint32_t)(((t - 2) >> 1) & 1), err)) return false;
            sm100::tc_fence_after();
            const unsigned char *sq = sRing + st * SLOT_BYTES;
            const float eg = it.valid ? __expf(it.Gr) : 0.f;
            for (int c16 = half; c16 * 32 < dk; c16 += 2) {  // 32 bf16 -> 16 TMEM columns per group
                uint32_t pk[16], qk[16];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int lc = c16 * 4 + u;  // logical 8-column chunk
                    if (lc * 8 < dk) {
                        const int sl = lc >> 3, cc = lc & 7;
                        uint4 v = *reinterpret_cast<const uint4 *>(sq + sl * JSLAB + r * 128 + ((cc ^ (r & 7)) << 4));
                        const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
                        const uint32_t *q2 = reinterpret_cast<const uint32_t *>(&v);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 x = __bfloat1622float2(p2[e]);
                            pk[u * 4 + e] = pack_bf16(eg * x.x, eg * x.y);
                            qk[u * 4 + e] = q2[e];
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) pk[u * 4 + e] = qk[u * 4 + e] = 0u;
                    }
                }
                sm100::tmem_st16(t_s0 + sb * JT + lane_off + c16 * 16, pk);
                sm100::tmem_st16(t_q0 + qb * 64 + lane_off + c16 * 16, qk);
            }
            sm100::tmem_st_wait();
            sm100::tc_fence_before();
            sm100::mbar_arrive(&bars[PFULL + sb]);
            ++sc;
            ++n;  // the pseudo-tile's ring slot
            return true;
        };
        auto tiles = [&](const Item &it) -> bool {
            for (int j = 0; j < it.nt; ++j, ++sc, ++n) {
                const int sb = sc % NSB, st = n % NSLOT;
                const bool diag = (j == it.I);
                if (!sm100::mbar_wait(&bars[SFULL + sb], (sc / NSB) & 1, err)) return false;
                if (!sm100::mbar_wait(&bars[RFULL + st], (n / NSLOT) & 1, err)) return false;  // G, cf
                sm100::tc_fence_after();
                const float *gJ = sGC + st * 2 * JT, *cfJ = gJ + JT;
                // In the diagonal tile, a row below the half's 64-token group sees all of it,
                // a row above sees none of it, and a row inside it sees the columns s <= r.
                // Every row takes the split e^{G_r - a} cf_s with a = G at the group's last
                // token (the anchor cf was made with); inside the group e^{G_r - a} >= 1, so a
                // row whose exponent exceeds kSplitMax takes the exact e^{G_r - G_s} instead.
                const bool none = diag && r < 64 * half;
                const bool in_group = diag && !none && r < 64 * half + 64;
                const float dG = it.Gr - gJ[min(64 * half + 63, L - 1 - j * JT)];
                const bool exact = in_group && !(dG <= kSplitMax);
                const float rf = (it.valid && !none && !exact) ? __expf(dG) : 0.f;
#pragma unroll
                // the half's 64 S columns with one wait; P then goes over the first 32 of them
                float vs[2][32];
                sm100::tmem_ld32(t_s0 + sb * JT + lane_off + 64 * half, vs[0]);
                sm100::tmem_ld32(t_s0 + sb * JT + lane_off + 64 * half + 32, vs[1]);
                sm100::tmem_ld_wait();
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int c0 = 64 * half + 32 * rr;
                    const float (&v)[32] = vs[rr];
                    uint32_t pk[16];
                    if (!exact) {  // rf = 0 where the row sees none of the half
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            float f0 = rf * cfJ[c0 + e], f1 = rf * cfJ[c0 + e + 1];
                            if (in_group) {  // the causal mask inside the group
                                f0 = c0 + e <= r ? f0 : 0.f;
                                f1 = c0 + e + 1 <= r ? f1 : 0.f;
                            }
                            pk[e >> 1] = pack_bf16(v[e] * f0, v[e + 1] * f1);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const int s0 = j * JT + c0 + e;
                            const float f0 = (s0 <= it.row && s0 < L) ? __expf(it.Gr - gJ[c0 + e]) : 0.f;
                            const float f1 =
                                (s0 + 1 <= it.row && s0 + 1 < L) ? __expf(it.Gr - gJ[c0 + e + 1]) : 0.f;
                            pk[e >> 1] = pack_bf16(v[e] * f0, v[e + 1] * f1);
                        }
                    }
                    // P of this half goes to TMEM columns [64 half, 64 half + 32): S columns it has read
                    sm100::tmem_st16(t_s0 + sb * JT + lane_off + 64 * half + 16 * rr, pk);
                }
                sm100::tmem_st_wait();
                sm100::tc_fence_before();
                sm100::mbar_arrive(&bars[PFULL + sb]);
            }
            return true;
        };
        auto drain = [&](const Item &it, int t) -> bool {
            if (!sm100::mbar_wait(&bars[OFULL], (uint32_t)(t & 1), err)) return false;
            sm100::tc_fence_after();
            const long long tt0 = it.f * L + it.row;
            const long long tt = prm.reverse_out ? prm.T - 1 - tt0 : tt0;  // a reversed scan's row, back in place
            __nv_bfloat16 *o = (__nv_bfloat16 *)prm.o + ((((long long)it.b * prm.T + tt) * prm.H + it.h) * dv);
            // columns c = 16 half + 32 i (dv <= 128), two 16-column loads per wait (the second
            // may read past dv, inside the O buffer's 128 columns, and is then not stored)
#pragma unroll
            for (int i2 = 0; i2 < 2; ++i2) {
                const int cb = 16 * half + 64 * i2;
                if (cb >= dv) break;
                float acc[2][16];
                sm100::tmem_ld16(t_o + lane_off + cb, acc[0]);
                sm100::tmem_ld16(t_o + lane_off + cb + 32, acc[1]);
                sm100::tmem_ld_wait();
                if (!it.valid) continue;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int c = cb + 32 * i;
                    if (c >= dv) break;
                    if (prm.accumulate) {
                        const uint4 *old = reinterpret_cast<const uint4 *>(o + c);
#pragma unroll
                        for (int w2 = 0; w2 < 2; ++w2) {
                            uint4 x = old[w2];
                            const __nv_bfloat162 *xb = reinterpret_cast<const __nv_bfloat162 *>(&x);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 fl = __bfloat1622float2(xb[e]);
                                acc[i][w2 * 8 + 2 * e] += fl.x;
                                acc[i][w2 * 8 + 2 * e + 1] += fl.y;
                            }
                        }
                    }
                    const float *a16 = acc[i];
                    reinterpret_cast<uint4 *>(o + c)[0] =
                        make_uint4(pack_bf16(a16[0], a16[1]), pack_bf16(a16[2], a16[3]), pack_bf16(a16[4], a16[5]),
                                   pack_bf16(a16[6], a16[7]));
                    reinterpret_cast<uint4 *>(o + c)[1] =
                        make_uint4(pack_bf16(a16[8], a16[9]), pack_bf16(a16[10], a16[11]),
                                   pack_bf16(a16[12], a16[13]), pack_bf16(a16[14], a16[15]));
                }
            }
            sm100::tc_fence_before();
            sm100::mbar_arrive(&bars[OEMPTY]);
            return true;
        };
        long long w = w_begin;
        bool ok = w < w_end;
        Item cur;
        if (ok) {
            cur = item_of(w);
            ok = pseudo(cur, 0);
        }
        for (int t = 0; ok; ++t) {
            // the next item's row (and its G, a global load) is read before this item's tiles
            const long long wn = w + 1;
            Item nxt;
            if (wn < w_end) nxt = item_of(wn);
            ok = tiles(cur);
            if (!ok) break;
            if (wn < w_end) {
                ok = pseudo(nxt, t + 1);
                if (!ok) break;
            }
            ok = drain(cur, t);
            if (!ok || wn >= w_end) break;
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
