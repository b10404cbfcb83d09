// tc_intra.cu -- intra-frame blocked forward substitution on the tensor cores.
//
// Solves, per frame-head, the unit lower triangular system of the chunkwise
// gated delta rule (one chunk per frame; SANA-WM summary,
// "Memory-Efficient Long-Context Modeling (Section 3.2)", frame-wise GDN):
//   (I + A) X = R,   X = [Ub | W],   R = [beta V | beta e^G K],
//   A_rs = beta_r e^{G_r - G_s} k_r.k_s  (s < r)
// over 128-row blocks i, in order:
//   acc_i = sum_{128-token tiles c before block i} P_ic X_c,  P_ic = -A_ic
//   Y_i   = R_i + acc_i
//   X_i   = T_ii Y_i,   T_ii = (I + A_ii)^{-1}  (from tc_diag_inverse.cu)
// X_i is staged in shared memory and stored by TMA to the [n_fh][L][d_v + d_k]
// bf16 workspace, from where later blocks load it again (L2-resident).
//
// A tcgen05.mma costs the same for every N up to 128, so S = K_i K_c^T is
// issued on 128-token tiles (N = 128).  Two rings feed the tensor cores:
//   K ring (2 x 32 KB): the K tile of each S product with its G and cf
//                       (one TMA box), and T_ii as the block's last item;
//   X ring (3 x 32 KB): the 64-token halves of X_c for acc += P X.
// Warp roles (320 threads): warp 0 TMA, warp 1 TMEM owner + MMA issuer (one
// thread), warps 2-9 epilogue: two warpgroups, each thread owning one block
// row (TMEM lane quadrant = warp % 4) and one half of the columns -- 64 of
// the 128 columns of an S tile, and in the diagonal step the Ub columns
// (half 0, which needs v) or the W columns (half 1, which needs k).
//   TMEM: two S/P buffers of 128 columns (the epilogue turns S into bf16 P in
//         place; acc += P X reads P from tensor memory) and acc (256 columns).
//   SMEM: K_i, the two rings; Y_i and then the staged X_i occupy the first
//         two X-ring slots during the diagonal step.
// Decay factors use the gate kernel's 64-token anchors: a = G at the end of
// the 64-token group, e^{G_r - G_s} = e^{G_r - a} cf_s, cf_s = e^{a - G_s}.
// Every wait is bounded (sm100::mbar_wait).
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kThreads = 320;
constexpr int kEpi = 256;                    // epilogue threads
constexpr int CT = 128;                      // tokens per S tile
constexpr int XT = 64;                       // tokens per X tile
constexpr int NK = 2;                        // K ring depth
constexpr int NX = 3;                        // X ring depth
constexpr int NSB = 2;                       // S/P buffers
constexpr int KSLOT = 2 * SLAB_BYTES;        // 128 rows x 2 slabs (a K tile or T_ii)
constexpr int XSLAB = XT * 128;              // one 64-row slab
constexpr int XSLOT = 4 * XSLAB;             // 64 rows x 4 slabs
constexpr int GCT_FLOATS = 2 * CT;           // G[128], cf[128] of a tile

struct Smem {
    static constexpr uint32_t KI = 0;                       // 128 rows x 2 slabs
    static constexpr uint32_t KR = KI + 2 * SLAB_BYTES;     // NK x 32 KB
    static constexpr uint32_t XR = KR + NK * KSLOT;         // NX x 32 KB; Y_i / X_i use the first 64 KB
    static constexpr uint32_t GC = XR + NX * XSLOT;         // NK x (G[128], cf[128])
    static constexpr uint32_t END = GC + NK * GCT_FLOATS * 4;
};
static_assert(2 * XSLOT == 4 * SLAB_BYTES, "Y_i must fill the first two X slots exactly");

enum Bar {
    KIFULL = 0, KIEMPTY, ACCFULL, YFULL, XFULL, XSTAGED,
    KRFULL, KREMPTY = KRFULL + NK, XRFULL = KREMPTY + NK, XREMPTY = XRFULL + NX,
    SFULL = XREMPTY + NX, SFREE = SFULL + NSB, PFULL = SFREE + NSB, NBAR = PFULL + NSB
};

__device__ __forceinline__ uint32_t yx_offset(int c, int r) {  // bf16 column c, row r of Y_i / X_i
    return (uint32_t)((c >> 6) * SLAB_BYTES + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4));
}

__global__ void __launch_bounds__(kThreads, 1)
k_intra_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_x64,
           const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_gct,
           const __grid_constant__ CUtensorMap tm_xs, const IntraParams prm) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int L = prm.L, dk = prm.dk, dv = prm.dv, nc = dk + dv, nblk = prm.nblk;
    const long long fh = blockIdx.x;
    const long long F = prm.F;
    const long long f = fh % F, chain = fh / F;
    const int h = (int)(chain % prm.H), b = (int)(chain / prm.H);
    const int bf = (int)(b * F + f);

    unsigned char *sKi = smem + Smem::KI;
    unsigned char *sKR = smem + Smem::KR;
    unsigned char *sXR = smem + Smem::XR;
    unsigned char *sYX = sXR;  // Y_i, then the staged X_i
    float *sGC = (float *)(smem + Smem::GC);
    uint64_t *bars = (uint64_t *)(smem + Smem::END);
    uint32_t *tmem_slot = (uint32_t *)(bars + NBAR);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int *err = prm.err;

    if (pass_failed(prm.err)) return;  // an earlier stage of this pass gave up
    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i) {
            uint32_t cnt = 1;
            if (i == KIEMPTY || i == YFULL || i == XSTAGED || (i >= PFULL && i < PFULL + NSB)) cnt = kEpi;
            if (i >= KREMPTY && i < KREMPTY + NK) cnt = 1 + kEpi;  // the MMA's commit + the epilogue
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
    const uint32_t t_s0 = tbase, t_acc = tbase + NSB * CT;
    const int nks_d = dk / 16;
    const int nslab_k = (dk + SLAB - 1) / SLAB;
    const int nslab_x = (nc + SLAB - 1) / SLAB;
    const int nt128 = (L + CT - 1) / CT;

    // Item numbering shared by the roles (block b has b S tiles, then T_b in the K ring):
    //   K-ring item of S tile c of block b: b(b+1)/2 + c, of T_b: b(b+1)/2 + b
    //   X-ring item of X tile x (64 tokens) of block b: b(b-1) + x
    //   S tile (and S/P buffer use) of S tile c of block b: b(b-1)/2 + c
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // Polls every kind of load and issues whichever is possible, so the K ring
        // (S products) never waits behind the X ring (P X products) or the stores.
        if (lane == 0) {
            sm100::tma_prefetch_desc(&tm_k);
            sm100::tma_prefetch_desc(&tm_x64);
            sm100::tma_prefetch_desc(&tm_t);
            sm100::tma_prefetch_desc(&tm_gct);
            sm100::tma_prefetch_desc(&tm_xs);
            // L2 policies: K and X tiles are read again by the frame's later blocks, T_ii once
            const uint64_t keep = sm100::policy_evict_last(), once = sm100::policy_evict_first();
            int ki = 0;              // next K_i block
            int kb = 0, kc = 0;      // next K-ring item: block kb, item kc (kc == kb: T_kb)
            int xb = 1, xx = 0;      // next X-ring item: block xb, X tile xx
            int sxb = 0;             // next X block to store; blocks < sxb have been stored and read out
            int kn = 0, xn = 0;
            bool ok = true;
            sm100::Spin spin;
            while (ok && (ki < nblk || kb < nblk || xb < nblk || sxb < nblk)) {
                bool prog = false;
                // K_i once the previous block's Y build has read K_{i-1}
                if (ki < nblk && (ki == 0 || sm100::mbar_test(&bars[KIEMPTY], (ki - 1) & 1))) {
                    sm100::mbar_arrive_expect_tx(&bars[KIFULL], (uint32_t)(nslab_k * SLAB_BYTES));
                    for (int sl = 0; sl < nslab_k; ++sl)
                        sm100::tma_load_4d_hint(sKi + sl * SLAB_BYTES, &tm_k, &bars[KIFULL], sl * SLAB, h, ki * BM, bf,
                                                keep);
                    ++ki;
                    prog = true;
                }
                // the next K-ring item: the K tile (+ G, cf) of an S product, or T_kb
                if (kb < nblk) {
                    const int st = kn % NK;
                    if (kn < NK || sm100::mbar_test(&bars[KREMPTY + st], ((kn / NK) - 1) & 1)) {
                        unsigned char *slot = sKR + st * KSLOT;
                        if (kc < kb) {
                            sm100::mbar_arrive_expect_tx(&bars[KRFULL + st],
                                                         (uint32_t)(nslab_k * SLAB_BYTES + GCT_FLOATS * 4));
                            for (int sl = 0; sl < nslab_k; ++sl)
                                sm100::tma_load_4d_hint(slot + sl * SLAB_BYTES, &tm_k, &bars[KRFULL + st], sl * SLAB, h,
                                                        kc * CT, bf, keep);
                            sm100::tma_load_2d(sGC + st * GCT_FLOATS, &tm_gct, &bars[KRFULL + st], 0,
                                               (int)(fh * nt128 + kc));
                        } else {
                            sm100::mbar_arrive_expect_tx(&bars[KRFULL + st], (uint32_t)(2 * SLAB_BYTES));
                            for (int sl = 0; sl < 2; ++sl)
                                sm100::tma_load_3d_hint(slot + sl * SLAB_BYTES, &tm_t, &bars[KRFULL + st], sl * SLAB, 0,
                                                        (int)(fh * nblk + kb), once);
                        }
                        ++kn;
                        if (++kc > kb) {
                            ++kb;
                            kc = 0;
                        }
                        prog = true;
                    }
                }
                // store the staged X_sxb (rows past the frame, columns past d_v + d_k clipped); the
                // X ring may refill the first two slots (which hold Y / X) once the store has read them
                if (sxb < nblk && sm100::mbar_test(&bars[XSTAGED], sxb & 1)) {
                    for (int sl = 0; sl < nslab_x; ++sl)
                        sm100::tma_store_3d_hint(&tm_xs, sYX + sl * SLAB_BYTES, sl * SLAB, sxb * BM, (int)fh, keep);
                    sm100::bulk_commit();
                    sm100::bulk_wait_read0();
                    ++sxb;
                    prog = true;
                }
                // the next X-ring item: X tile xx of block xb (the tiles of X_{xb-1} come last)
                if (xb < nblk && sxb >= xb) {
                    const int st = xn % NX;
                    if (xn < NX || sm100::mbar_test(&bars[XREMPTY + st], ((xn / NX) - 1) & 1)) {
                        if (xx >= 2 * (xb - 1)) sm100::bulk_wait0();  // X_{xb-1} is in global memory
                        unsigned char *slot = sXR + st * XSLOT;
                        sm100::mbar_arrive_expect_tx(&bars[XRFULL + st], (uint32_t)(nslab_x * XSLAB));
                        for (int sl = 0; sl < nslab_x; ++sl)
                            sm100::tma_load_3d_hint(slot + sl * XSLAB, &tm_x64, &bars[XRFULL + st], sl * SLAB, xx * XT,
                                                    (int)fh, keep);
                        ++xn;
                        if (++xx == 2 * xb) {
                            ++xb;
                            xx = 0;
                        }
                        prog = true;
                    }
                }
                if (prog) spin.reset();
                else if (!spin.tick(err)) ok = false;
            }
            sm100::bulk_wait0();  // leave with no store in flight
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Polls: S = K_b K_c^T as soon as K_b, the K tile and an S/P buffer are there;
        // acc += P X as soon as P and both X halves are there (and acc is free);
        // X_b = T_b Y_b as soon as Y_b and T_b are there.
        if (lane == 0) {
            const uint32_t id_s = sm100::idesc_bf16(BM, CT, 0, 0);
            const uint32_t id_x = sm100::idesc_bf16(BM, nc, 0, 1);
            // A parity test is only unambiguous for the phase right after the last one
            // observed, and the S and T cursors take K-ring items out of order, so the
            // phases of each K slot (and of K_i) are observed one at a time, in order.
            static_assert(NK == 2, "one observed-phase counter per K slot");
            int kobs0 = 0, kobs1 = 0, kiobs = 0;  // scalars: an indexed array would live in local memory
            auto k_ready = [&](int kn) -> bool {
                const int st = kn % NK, u = kn / NK;
                int &obs = st ? kobs1 : kobs0;
                while (obs <= u && sm100::mbar_test(&bars[KRFULL + st], obs & 1)) ++obs;
                return obs > u;
            };
            auto ki_ready = [&](int b) -> bool {
                while (kiobs <= b && sm100::mbar_test(&bars[KIFULL], kiobs & 1)) ++kiobs;
                return kiobs > b;
            };
            // K_1 cannot load before block 0's Y build, which waits for acc_0 = 0 below:
            // observe K_0 first so that KIFULL never runs two phases ahead
            bool ok = sm100::mbar_wait(&bars[KIFULL], 0, err);
            kiobs = 1;
            sm100::mma_commit(&bars[ACCFULL]);  // block 0 has no S tiles: acc_0 = 0
            int sb_ = 1, sc_ = 0, sn = 0;       // next S product: block sb_, tile sc_; S tile count
            int pb_ = 1, pc_ = 0, pn = 0;       // next P X product
            int ty = 0;                         // next T Y
            const int ntile = nblk * (nblk - 1) / 2;
            sm100::Spin spin;
            while (ok && (pn < ntile || ty < nblk)) {
                bool prog = false;
                if (sn < ntile && sn - pn < NSB) {
                    const int kn = sb_ * (sb_ + 1) / 2 + sc_, st = kn % NK, buf = sn % NSB;
                    if (ki_ready(sb_) && k_ready(kn) &&
                        (sn < NSB || sm100::mbar_test(&bars[SFREE + buf], ((sn / NSB) - 1) & 1))) {
                        sm100::tc_fence_after();
                        const unsigned char *kt = sKR + st * KSLOT;
                        for (int ks = 0; ks < nks_d; ++ks)
                            sm100::mma_bf16_ss(t_s0 + buf * CT, desc_kmajor(sKi, ks, BM), desc_kmajor(kt, ks, CT),
                                               id_s, ks > 0);
                        sm100::mma_commit(&bars[SFULL + buf]);
                        sm100::mma_commit(&bars[KREMPTY + st]);
                        ++sn;
                        if (++sc_ == sb_) {
                            ++sb_;
                            sc_ = 0;
                        }
                        prog = true;
                    }
                }
                if (pn < sn) {
                    const int buf = pn % NSB, xn0 = pb_ * (pb_ - 1) + 2 * pc_;
                    const int st0 = xn0 % NX, st1 = (xn0 + 1) % NX;
                    const bool first = pc_ == 0;
                    // the block's first product overwrites acc: X_{pb_-1} must have been read out
                    if (sm100::mbar_test(&bars[PFULL + buf], (pn / NSB) & 1) &&
                        sm100::mbar_test(&bars[XRFULL + st0], (xn0 / NX) & 1) &&
                        sm100::mbar_test(&bars[XRFULL + st1], ((xn0 + 1) / NX) & 1) &&
                        (!first || sm100::mbar_test(&bars[XSTAGED], (pb_ - 1) & 1))) {
                        sm100::tc_fence_after();
                        // P of tokens 0..63 sits in TMEM columns 0..31 of the buffer, tokens 64..127 in 64..95
                        for (int hx = 0; hx < 2; ++hx) {
                            const unsigned char *xt = sXR + (hx ? st1 : st0) * XSLOT;
                            for (int ks = 0; ks < XT / 16; ++ks)
                                sm100::mma_bf16_ts(t_acc, t_s0 + buf * CT + 64 * hx + ks * 8, desc_mnmajor(xt, ks, XT),
                                                   id_x, (first && hx == 0 && ks == 0) ? 0u : 1u);
                            sm100::mma_commit(&bars[XREMPTY + (hx ? st1 : st0)]);
                        }
                        sm100::mma_commit(&bars[SFREE + buf]);
                        if (pc_ == pb_ - 1) sm100::mma_commit(&bars[ACCFULL]);
                        ++pn;
                        if (++pc_ == pb_) {
                            ++pb_;
                            pc_ = 0;
                        }
                        prog = true;
                    }
                }
                if (ty < nblk && pb_ > ty) {  // every P X product of block ty has been issued
                    const int kn = ty * (ty + 1) / 2 + ty, st = kn % NK;
                    if (k_ready(kn) && sm100::mbar_test(&bars[YFULL], ty & 1)) {
                        sm100::tc_fence_after();
                        const unsigned char *tt = sKR + st * KSLOT;
                        for (int ks = 0; ks < BM / 16; ++ks)
                            sm100::mma_bf16_ss(t_acc, desc_kmajor(tt, ks, BM), desc_mnmajor(sYX, ks, BM), id_x,
                                               ks > 0);
                        sm100::mma_commit(&bars[XFULL]);
                        sm100::mma_commit(&bars[KREMPTY + st]);
                        ++ty;
                        prog = true;
                    }
                }
                if (prog) spin.reset();
                else if (!spin.tick(err)) ok = false;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q4 = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r = q4 * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const float *Gf = prm.G + fh * (long long)((L + 3) & ~3);  // G rows are padded to 16 bytes
        bool ok = true;
        int kn = 0, sn = 0;
        // this row's G and beta, read one block ahead so their latency stays off the S -> P steps
        auto row_gates = [&](int i, float &g, float &bb) {
            const int rw = i * BM + r;
            const bool ok_row = i < nblk && rw < L;
            g = ok_row ? Gf[rw] : 0.f;
            bb = ok_row ? prm.beta[((long long)b * prm.T + f * L + rw) * prm.H + h] : 0.f;
        };
        float G_next, be_next;
        row_gates(0, G_next, be_next);
        for (int i = 0; i < nblk && ok; ++i) {
            const int row = i * BM + r;
            const bool valid = row < L;
            const float Gr = G_next, be = be_next;
            row_gates(i + 1, G_next, be_next);
            const long long tok = ((long long)b * prm.T + f * L + row) * prm.H + h;
            // half 0 needs this row's values in the diagonal step: pull them into L2 now
            const __nv_bfloat16 *vp = prm.v + tok * dv;
            if (half == 0 && valid) {
                for (int by = 0; by < dv * 2; by += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"((const char *)vp + by));
                asm volatile("prefetch.global.L2 [%0];" ::"l"((const char *)vp + dv * 2 - 1));
            }
            // ---- S tiles -> P = -beta_r e^{G_r - G_s} S (this half: tile columns 64 half .. 64 half + 63)
            for (int c = 0; c < i && ok; ++c, ++kn, ++sn) {
                const int sb = sn % NSB, st = kn % NK;
                ok = sm100::mbar_wait(&bars[SFULL + sb], (sn / NSB) & 1, err) &&
                     sm100::mbar_wait(&bars[KRFULL + st], (kn / NK) & 1, err);  // G, cf of the tile
                if (!ok) break;
                sm100::tc_fence_after();
                const float *gJ = sGC + st * GCT_FLOATS, *cfJ = gJ + CT;
                // the tile lies before block i, so it is full: the half's anchor is G at its last token
                const float rf = valid ? -be * __expf(Gr - gJ[64 * half + 63]) : 0.f;
                // the half's 64 S columns with one wait; P then goes over the first 32 of them
                float vs[2][32];
                sm100::tmem_ld32(t_s0 + sb * CT + lane_off + 64 * half, vs[0]);
                sm100::tmem_ld32(t_s0 + sb * CT + lane_off + 64 * half + 32, vs[1]);
                sm100::tmem_ld_wait();
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int c0 = 64 * half + 32 * rr;
                    const float (&v)[32] = vs[rr];
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2)
                        pk[e >> 1] = pack_bf16(rf * cfJ[c0 + e] * v[e], rf * cfJ[c0 + e + 1] * v[e + 1]);
                    sm100::tmem_st16(t_s0 + sb * CT + lane_off + 64 * half + 16 * rr, pk);
                }
                sm100::tmem_st_wait();
                sm100::tc_fence_before();
                sm100::mbar_arrive(&bars[PFULL + sb]);
                sm100::mbar_arrive(&bars[KREMPTY + st]);  // done with the slot's G and cf
            }
            if (!ok) break;
            // ---- Y_i = R_i + acc_i  -> sYX (MN-major: row = K index of the T_ii Y_i product)
            // (K_i: the W half reads it; block 0 has no S product that waited for it)
            // half 0: this row's values, read before the accumulator wait so their latency hides
            // behind the block's last products (v is read once: evict first, keep K and X in L2)
            uint4 vrow[16];
            if (half == 0) {
                const uint64_t once = sm100::policy_evict_first();
#pragma unroll
                for (int c8 = 0; c8 < 16; ++c8)
                    vrow[c8] = (valid && c8 < dv / 8) ? sm100::ld_nc_hint(reinterpret_cast<const uint4 *>(vp) + c8, once)
                                                      : make_uint4(0, 0, 0, 0);
            }
            ok = sm100::mbar_wait(&bars[ACCFULL], i & 1, err) && sm100::mbar_wait(&bars[KIFULL], i & 1, err);
            if (!ok) break;
            sm100::tc_fence_after();
            auto store_y = [&](int c, const float (&y)[8]) {
                const uint4 val = valid ? make_uint4(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]),
                                                     pack_bf16(y[4], y[5]), pack_bf16(y[6], y[7]))
                                        : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(sYX + yx_offset(c, r)) = val;
            };
            if (half == 0) {  // Ub columns: beta_r v_r + acc
#pragma unroll
                for (int j2 = 0; j2 < 4; ++j2) {  // two 16-column loads per wait
                    if (32 * j2 >= dv) break;
                    float acc[2][16];
                    if (i > 0) {  // the second load may read past dv, inside the accumulator
                        sm100::tmem_ld16(t_acc + lane_off + 32 * j2, acc[0]);
                        sm100::tmem_ld16(t_acc + lane_off + 32 * j2 + 16, acc[1]);
                        sm100::tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) acc[0][e] = acc[1][e] = 0.f;
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int c = 32 * j2 + 8 * u;
                        if (c >= dv) break;
                        const __nv_bfloat162 *vb = reinterpret_cast<const __nv_bfloat162 *>(&vrow[4 * j2 + u]);
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 fv = __bfloat1622float2(vb[e]);
                            y[2 * e] = be * fv.x + acc[u >> 1][(u & 1) * 8 + 2 * e];
                            y[2 * e + 1] = be * fv.y + acc[u >> 1][(u & 1) * 8 + 2 * e + 1];
                        }
                        store_y(c, y);
                    }
                }
            } else {  // W columns: beta_r e^{G_r} k_r + acc
                const float rk = be * __expf(Gr);
#pragma unroll
                for (int j2 = 0; j2 < 4; ++j2) {  // two 16-column loads per wait
                    if (32 * j2 >= dk) break;
                    float acc[2][16];
                    if (i > 0) {  // the second load may read past dk, inside the accumulator
                        sm100::tmem_ld16(t_acc + lane_off + dv + 32 * j2, acc[0]);
                        sm100::tmem_ld16(t_acc + lane_off + dv + 32 * j2 + 16, acc[1]);
                        sm100::tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) acc[0][e] = acc[1][e] = 0.f;
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int kc = 32 * j2 + 8 * u;
                        if (kc >= dk) break;
                        const uint4 kv = *reinterpret_cast<const uint4 *>(sKi + yx_offset(kc, r));
                        const __nv_bfloat162 *kb = reinterpret_cast<const __nv_bfloat162 *>(&kv);
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 fk = __bfloat1622float2(kb[e]);
                            y[2 * e] = rk * fk.x + acc[u >> 1][(u & 1) * 8 + 2 * e];
                            y[2 * e + 1] = rk * fk.y + acc[u >> 1][(u & 1) * 8 + 2 * e + 1];
                        }
                        store_y(dv + kc, y);
                    }
                }
            }
            sm100::tc_fence_before();
            sm100::fence_proxy_async_smem();
            sm100::mbar_arrive(&bars[YFULL]);
            sm100::mbar_arrive(&bars[KIEMPTY]);
            // the T_ii slot: observe its load (so this thread sees every phase of the slot in
            // order), then release it; the slot refills once T Y has completed as well
            ok = sm100::mbar_wait(&bars[KRFULL + kn % NK], (kn / NK) & 1, err);
            if (!ok) break;
            sm100::mbar_arrive(&bars[KREMPTY + kn % NK]);
            ++kn;
            // ---- X_i = T_ii Y_i -> bf16 staging over Y_i (half 0 the Ub columns, half 1 the W columns)
            ok = sm100::mbar_wait(&bars[XFULL], i & 1, err);
            if (!ok) break;
            sm100::tc_fence_after();
            const int c_lo = half ? dv : 0, c_hi = half ? nc : dv;
            // two 16-column loads per wait (the second may read past c_hi, inside the
            // accumulator's 256 columns, and is then not stored)
            for (int c32 = c_lo; c32 < c_hi; c32 += 32) {
                float x[2][16];
                sm100::tmem_ld16(t_acc + lane_off + c32, x[0]);
                sm100::tmem_ld16(t_acc + lane_off + c32 + 16, x[1]);
                sm100::tmem_ld_wait();
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    if (c32 + 16 * h2 >= c_hi) break;
#pragma unroll
                    for (int u = 0; u < 2; ++u)
                        *reinterpret_cast<uint4 *>(sYX + yx_offset(c32 + 16 * h2 + 8 * u, r)) = make_uint4(
                            pack_bf16(x[h2][8 * u], x[h2][8 * u + 1]), pack_bf16(x[h2][8 * u + 2], x[h2][8 * u + 3]),
                            pack_bf16(x[h2][8 * u + 4], x[h2][8 * u + 5]), pack_bf16(x[h2][8 * u + 6], x[h2][8 * u + 7]));
                }
            }
            sm100::tc_fence_before();
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

cudaError_t launch_intra_tc(const CUtensorMap &tm_k, const CUtensorMap &tm_x64, const CUtensorMap &tm_t,
                            const CUtensorMap &tm_gct, const CUtensorMap &tm_xs, const IntraParams &prm,
                            long long n_fh, cudaStream_t s) {
    const size_t smem = 1024 + Smem::END + sizeof(uint64_t) * NBAR + 16;
    cudaError_t e = cudaFuncSetAttribute(k_intra_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_intra_tc<<<(unsigned)n_fh, kThreads, smem, s>>>(tm_k, tm_x64, tm_t, tm_gct, tm_xs, prm);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace gdn
