// tc_intra.cu -- intra-frame solve and the frame's transition, on the tensor cores.
//
// Solves, per frame-head, the unit lower triangular system of the chunkwise
// gated delta rule (one chunk per frame; SANA-WM summary,
// "Memory-Efficient Long-Context Modeling (Section 3.2)", frame-wise GDN):
//   (I + A) X = R,   X = [Ub | W],   R = [beta V | beta e^G K],
//   A_rs = beta_r e^{G_r - G_s} k_r.k_s  (s < r)
// over 128-row blocks i, in order, and forms the frame's affine state map
//   Sig_next = M Sig + N,   M = e^{G_L} I - Kt^T W,   N = Kt^T Ub,
//   Kt = diag(e^{G_L - G}) K
// (the per-frame transition of the chunk = frame decomposition; cliffmar.tech
// article, "NVIDIA SANA-WM", training section: the maps the sequence composes).
//
// The rows of A left of block i factor through the keys, so the blocks before
// i enter block i through one d_k x (d_v + d_k) matrix, carried from block to
// block like the inter-frame state (anchor a_i = the last token before block i;
// every decay factor below is e^{non-positive}):
//   H_i     = sum_{s < a_i + 1} e^{G_{a_i} - G_s} k_s^T X_s,      H_0 = 0
//   Y_i     = R_i - diag(beta_r e^{G_r - G_{a_i}}) K_i H_i
//   X_i     = T_ii Y_i,   T_ii = (I + A_ii)^{-1}  (from tc_diag_inverse.cu)
//   H_{i+1} = e^{G_{a_{i+1}} - G_{a_i}} H_i + Kh_i^T X_i,   Kh_i = diag(e^{G_{a_{i+1}} - G_s}) K_i
// and after the last block (anchor = the frame's last token) H = Kt^T [Ub | W],
// which gives N and M directly.  Per block: three 128 x (d_v + d_k) x 128
// products and no reread of earlier blocks' X.
//
// Shared memory: K_i double-buffered (the A operand of K_i H_i, then scaled in
// place into Kh_i, the MN-major A operand of Kh_i^T X_i), T_ii, the staging
// tile (Y_i, then X_i: the B operand of T_ii Y_i and of Kh_i^T X_i, and the
// source of X_i's TMA store) and bf16 H_i (the B operand of K_i H_i).
// TMEM: the block's product (K_i H_i, then X_i; 256 columns) and H (fp32,
// 256 columns; lanes = key dimension).
// The Ub columns and the W columns never mix (each column of Y, X and H
// depends on the same column alone), so the two halves run as two chains that
// share K_i, T_ii and Kh_i: each half has its own products (N = d_v or d_k)
// and barriers, and one half's epilogue overlaps the other's products.  In
// shared and tensor memory the W columns start on a 64-column slab (column
// dvp = d_v rounded up to 64), so each half is a whole number of swizzle slabs.
// Warp roles (352 threads): warp 0 TMA loads, warp 1 TMEM owner + MMA issuer
// (one thread), warps 2-9 epilogue: two warpgroups, each thread owning one row
// (TMEM lane quadrant = warp % 4) of one half (warps 2-5 the Ub columns, warps
// 6-9 the W columns; for H, rows are key dimensions); warp 10 stores X (a
// thread of its own, so that waiting for a store's reads holds up no load).
// Every wait is bounded (sm100::mbar_wait); a role that gives up waits for its
// own copies and products in flight before the CTA leaves.
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kThreads = 352;
constexpr int kEpi = 256;                    // epilogue threads
constexpr int TILE = 2 * SLAB_BYTES;         // 128 rows x 2 slabs (K_i or T_ii)
constexpr int WIDE = 4 * SLAB_BYTES;         // 128 rows x 4 slabs (Y_i / X_i, H)

// ACCFULL .. HREADY come per half (index + half); XSTG0 / XSTG1 are the halves' X staged.
enum Bar {
    ACCFULL = 0, YFULL = ACCFULL + 2, XFULL = YFULL + 2, UFULL = XFULL + 2, HREADY = UFULL + 2,
    XSTG0 = HREADY + 2, XSTG1, KHREADY, TFULL, TFREE, VFULL, STAFREE, STBFREE, DRAIN,
    KFULL, KEMPTY = KFULL + 2, NBAR = KEMPTY + 2
};

// Small objects first, then the swizzled tiles from a 1024-byte boundary; the dynamic
// shared memory base is itself 1024-aligned (the kernel declares no static shared memory;
// it checks this and reports it through the error word otherwise).
struct Smem {
    static constexpr uint32_t BARS = 0;
    static constexpr uint32_t TSLOT = BARS + NBAR * 8;
    static constexpr uint32_t KB = 1024;                    // 2 x K_i
    static constexpr uint32_t TB = KB + 2 * TILE;           // T_ii
    static constexpr uint32_t ST = TB + TILE;               // Y_i / X_i
    static constexpr uint32_t HB = ST + WIDE;               // bf16 H_i
    static constexpr uint32_t END = HB + WIDE;
};
static_assert(Smem::TSLOT + 4 <= Smem::KB, "barriers overlap the tiles");
static_assert(Smem::END <= 232448, "over the 227 KB a CTA may use");

// Packed fp32 pairs (lane 0 in the low word).
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
    return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}


// Where a column half stages the frame's transition after its last block: its own slabs of the
// staging tile (stA) and of bf16 H (stB).  N (half 0) as fp32 rows at a pitch of an odd number of
// 16-byte units (one warp's row pieces fall in distinct banks), rows_per rows in each region;
// M's hi / lo images (half 1) in the scan's operand layout, hi over stB, lo over stA.
struct FinalStage {
    unsigned char *stA, *stB, *img;
    int nslab, pitch, rows_per;
    bool stage_n;
    __device__ __forceinline__ FinalStage(unsigned char *sST, unsigned char *sH, int half, int dk, int dv, int dvp,
                                          int nslab_v, __nv_bfloat16 *Mimg, long long fh) {
        const int sl0 = half ? dvp / SLAB : 0;
        stA = sST + sl0 * SLAB_BYTES;
        stB = sH + sl0 * SLAB_BYTES;
        nslab = (dk + SLAB - 1) / SLAB;
        img = Mimg ? reinterpret_cast<unsigned char *>(Mimg) + fh * (long long)(2 * nslab * dk * 128) : nullptr;
        pitch = dv * 4 + 16;
        rows_per = nslab_v * SLAB_BYTES / pitch;
        stage_n = 2 * rows_per >= dk;
    }
    __device__ __forceinline__ unsigned char *nrow(int row) const {
        return (row < rows_per ? stA : stB) + (row % rows_per) * pitch;
    }
};

__global__ void __launch_bounds__(kThreads, 1)
k_intra_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
           const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_xu,
           const __grid_constant__ CUtensorMap tm_xw, const IntraParams prm) {
    extern __shared__ __align__(1024) unsigned char smem[];
    const int L = prm.L, dk = prm.dk, dv = prm.dv, nblk = prm.nblk;
    const int dvp = (dv + SLAB - 1) / SLAB * SLAB;  // first column of the W half in SMEM and TMEM
    const long long fh = blockIdx.x;
    const long long F = prm.F;
    const long long f = fh % F, chain = fh / F;
    const int h = (int)(chain % prm.H), b = (int)(chain / prm.H);
    const int bf = (int)(b * F + f);

    unsigned char *sK = smem + Smem::KB;
    unsigned char *sT = smem + Smem::TB;
    unsigned char *sST = smem + Smem::ST;
    unsigned char *sH = smem + Smem::HB;
    uint64_t *bars = (uint64_t *)(smem + Smem::BARS);
    uint32_t *tmem_slot = (uint32_t *)(smem + Smem::TSLOT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int *err = prm.err;
    const uint64_t wait_ns = prm.wait_ns;
    const int nslab_k = (dk + SLAB - 1) / SLAB;
    const int nslab_v = dvp / SLAB;

    if (pass_failed(prm.err)) return;  // an earlier stage of this pass gave up
    if (sm100::smem_u32(smem) & 1023u) {  // every thread sees the same base: all leave together
        if (threadIdx.x == 0) atomicCAS(err, sm100::kErrNone, sm100::kErrSmemAlign);
        return;
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i)
            sm100::mbar_init(&bars[i], ((i >= YFULL && i < YFULL + 2) || (i >= HREADY && i < HREADY + 2) ||
                                        i == XSTG0 || i == XSTG1 || i == KHREADY) ? kEpi / 2 : 1);
        sm100::fence_barrier_init();
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, 512);
        sm100::tmem_relinquish();
    }
    if (nslab_k == 1) {  // K_i^T as a 128-row operand: key dimensions past the one loaded slab are zero
        for (int o = threadIdx.x * 16; o < SLAB_BYTES; o += kThreads * 16) {
            *reinterpret_cast<uint4 *>(sK + SLAB_BYTES + o) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sK + TILE + SLAB_BYTES + o) = make_uint4(0, 0, 0, 0);
        }
        sm100::fence_proxy_async_smem();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t t_p = tbase, t_h = tbase + 256;  // the block's product; H

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // K_j (double-buffered: once block j-2's Kh^T X has read its buffer), T_j (once T_{j-1}
        // Y_{j-1} has read the tile), V_j into the staging tile's first slabs (once X_{j-1} has
        // been read there by its store and by Kh^T X_{j-1}).
        if (lane == 0) {
            sm100::tma_prefetch_desc(&tm_k);
            sm100::tma_prefetch_desc(&tm_v);
            sm100::tma_prefetch_desc(&tm_t);
            sm100::tma_prefetch_desc(&tm_xu);
            sm100::tma_prefetch_desc(&tm_xw);
            // L2 policies: K and T are read once here; X is read again by the next stages
            const uint64_t once = sm100::policy_evict_first();
            int kj = 0, tj = 0, vj = 0;
            for (int sl = 0; sl < nslab_v; ++sl) sm100::tma_prefetch_l2_4d(&tm_v, sl * SLAB, h, 0, bf);
            bool ok = true;
            sm100::Spin spin(wait_ns);
            while (ok && (kj < nblk || tj < nblk || vj < nblk)) {
                bool prog = false;
                if (kj < nblk && (kj < 2 || sm100::mbar_test(&bars[KEMPTY + (kj & 1)], ((kj >> 1) - 1) & 1))) {
                    uint64_t *bar = &bars[KFULL + (kj & 1)];
                    unsigned char *dst = sK + (kj & 1) * TILE;
                    sm100::mbar_arrive_expect_tx(bar, (uint32_t)(nslab_k * SLAB_BYTES));
                    for (int sl = 0; sl < nslab_k; ++sl)
                        sm100::tma_load_4d_hint(dst + sl * SLAB_BYTES, &tm_k, bar, sl * SLAB, h, kj * BM, bf, once);
                    ++kj;
                    prog = true;
                }
                if (tj < nblk && (tj == 0 || sm100::mbar_test(&bars[TFREE], (tj - 1) & 1))) {
                    sm100::mbar_arrive_expect_tx(&bars[TFULL], (uint32_t)(2 * SLAB_BYTES));
                    for (int sl = 0; sl < 2; ++sl)
                        sm100::tma_load_3d_hint(sT + sl * SLAB_BYTES, &tm_t, &bars[TFULL], sl * SLAB, 0,
                                                (int)(fh * nblk + tj), once);
                    ++tj;
                    prog = true;
                }
                // V_vj into the Ub slabs once X_{vj-1}'s Ub half has been read there by its store and
                // by Kh^T X_{vj-1}
                if (vj < nblk && (vj == 0 || (sm100::mbar_test(&bars[STAFREE], (vj - 1) & 1) &&
                                              sm100::mbar_test(&bars[UFULL + 0], (vj - 1) & 1)))) {
                    sm100::mbar_arrive_expect_tx(&bars[VFULL], (uint32_t)(nslab_v * SLAB_BYTES));
                    for (int sl = 0; sl < nslab_v; ++sl)
                        sm100::tma_load_4d_hint(sST + sl * SLAB_BYTES, &tm_v, &bars[VFULL], sl * SLAB, h, vj * BM, bf,
                                                once);
                    if (vj + 1 < nblk)  // the next block's values into L2 meanwhile
                        for (int sl = 0; sl < nslab_v; ++sl)
                            sm100::tma_prefetch_l2_4d(&tm_v, sl * SLAB, h, (vj + 1) * BM, bf);
                    ++vj;
                    prog = true;
                }
                if (prog) {
                    spin.reset();
                } else if (!spin.tick(err)) {
                    ok = false;
                } else {
                    __nanosleep(64);  // leave the issue slots to the epilogue warps of this sub-partition
                }
            }
            if (!ok) {  // leave with no load in flight (full-limit drain waits)
                for (int j = kj > 2 ? kj - 2 : 0; j < kj; ++j)
                    sm100::mbar_wait(&bars[KFULL + (j & 1)], (uint32_t)((j >> 1) & 1), err, sm100::kWaitLimitNs, true);
                if (tj > 0) sm100::mbar_wait(&bars[TFULL], (uint32_t)((tj - 1) & 1), err, sm100::kWaitLimitNs, true);
                if (vj > 0) sm100::mbar_wait(&bars[VFULL], (uint32_t)((vj - 1) & 1), err, sm100::kWaitLimitNs, true);
            }
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------ X stores
        // X_j's Ub slabs once the Ub half has staged them (the next block's v may then land
        // there), its W slabs once the W half has; each through a map of its own columns of
        // the [Ub | W] rows.  A thread of its own, so that waiting for a store's reads holds up
        // no load.
        if (lane == 0) {
            const uint64_t keep = sm100::policy_evict_last();  // X is read again by the next stages
            unsigned char *sW = sST + nslab_v * SLAB_BYTES;
            bool ok = true;
            for (int j = 0; j < nblk && ok; ++j) {
                ok = sm100::mbar_wait(&bars[XSTG0], (uint32_t)(j & 1), err, wait_ns);
                if (!ok) break;
                for (int sl = 0; sl < nslab_v; ++sl)
                    sm100::tma_store_3d_hint(&tm_xu, sST + sl * SLAB_BYTES, sl * SLAB, j * BM, (int)fh, keep);
                sm100::bulk_commit();
                sm100::bulk_wait_read0();
                sm100::mbar_arrive(&bars[STAFREE]);
                ok = sm100::mbar_wait(&bars[XSTG1], (uint32_t)(j & 1), err, wait_ns);
                if (!ok) break;
                for (int sl = 0; sl < nslab_k; ++sl)
                    sm100::tma_store_3d_hint(&tm_xw, sW + sl * SLAB_BYTES, sl * SLAB, j * BM, (int)fh, keep);
                sm100::bulk_commit();
                sm100::bulk_wait_read0();
                sm100::mbar_arrive(&bars[STBFREE]);
            }
            sm100::bulk_wait0();  // leave with no store in flight
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Two chains, one per half (hf), polled: per block, K_i H_i (from block 1), T_ii Y_i,
        // then H += Kh_i^T X_i, each on the half's columns only.  TFREE / KEMPTY are committed
        // once both halves have issued their T_ii Y_i / Kh_i^T X_i.  T_ii and Kh_i, which both
        // chains read, are observed one phase at a time, in order, through counters.
        if (lane == 0) {
            const int nks_d = dk / 16;
            int op0 = 1, op1 = 1, blk0 = 0, blk1 = 0;  // next product per half: 0 K_i H_i, 1 T_ii Y_i, 2 Kh^T X
            int tobs = 0, khobs = 0;
            int ty_done = 0, u_done = 0;          // blocks whose T Y / Kh^T X both halves have issued
            // K_i is KFULL[i & 1]'s phase i >> 1; the phase after it needs K_{i+2}, which loads
            // only once both halves' Kh_i^T X_i are done, so a direct parity test is unambiguous
            // (a counter would have to observe K_0, which no product here waits for)
            auto k_ready = [&](int i) -> bool {
                return sm100::mbar_test(&bars[KFULL + (i & 1)], (uint32_t)((i >> 1) & 1));
            };
            auto seen = [&](int bar, int &obs, int i) -> bool {
                while (obs <= i && sm100::mbar_test(&bars[bar], obs & 1)) ++obs;
                return obs > i;
            };
            bool ok = true;
            sm100::Spin spin(wait_ns);
            while (ok && (blk0 < nblk || blk1 < nblk)) {
                bool prog = false;
#pragma unroll 1
                for (int hf = 0; hf < 2; ++hf) {
                    int &opr = hf ? op1 : op0, &blkr = hf ? blk1 : blk0;
                    const int i = blkr;
                    if (i >= nblk) continue;
                    const int n = hf ? dk : dv;                              // the half's columns
                    const uint32_t coff = hf ? (uint32_t)dvp : 0u;           // ... in TMEM
                    const uint32_t soff = hf ? (uint32_t)(nslab_v * SLAB_BYTES) : 0u;  // ... in SMEM
                    unsigned char *kt = sK + (i & 1) * TILE;
                    if (opr == 0) {  // acc = K_i H_i, once K_i has landed and H_i is staged in bf16
                        if (k_ready(i) && sm100::mbar_test(&bars[HREADY + hf], (i - 1) & 1)) {
                            sm100::tc_fence_after();
                            const uint32_t id = sm100::idesc_bf16(BM, n, 0, 1);  // K-major A, MN-major B
                            for (int ks = 0; ks < nks_d; ++ks)
                                sm100::mma_bf16_ss(t_p + coff, desc_kmajor(kt, ks, BM), desc_mnmajor(sH + soff, ks, BM),
                                                   id, ks > 0);
                            sm100::mma_commit(&bars[ACCFULL + hf]);
                            opr = 1;
                            prog = true;
                        }
                    } else if (opr == 1) {  // X_i = T_ii Y_i
                        if (seen(TFULL, tobs, i) && sm100::mbar_test(&bars[YFULL + hf], i & 1)) {
                            sm100::tc_fence_after();
                            const uint32_t id = sm100::idesc_bf16(BM, n, 0, 1);
                            for (int ks = 0; ks < BM / 16; ++ks)
                                sm100::mma_bf16_ss(t_p + coff, desc_kmajor(sT, ks, BM), desc_mnmajor(sST + soff, ks, BM),
                                                   id, ks > 0);
                            sm100::mma_commit(&bars[XFULL + hf]);
                            if (++ty_done == 2 * (i + 1)) sm100::mma_commit(&bars[TFREE]);
                            opr = 2;
                            prog = true;
                        }
                    } else {  // H (rescaled to this block's end by the epilogue) += Kh_i^T X_i
                        if (sm100::mbar_test(&bars[hf ? XSTG1 : XSTG0], i & 1) && seen(KHREADY, khobs, i)) {
                            sm100::tc_fence_after();
                            const uint32_t id = sm100::idesc_bf16(BM, n, 1, 1);  // MN-major A (Kh^T), MN-major B
                            for (int ks = 0; ks < BM / 16; ++ks)
                                sm100::mma_bf16_ss(t_h + coff, desc_mnmajor(kt, ks, BM), desc_mnmajor(sST + soff, ks, BM),
                                                   id, (i > 0 || ks > 0) ? 1u : 0u);
                            sm100::mma_commit(&bars[UFULL + hf]);
                            if (++u_done == 2 * (i + 1)) sm100::mma_commit(&bars[KEMPTY + (i & 1)]);
                            blkr = i + 1;
                            opr = 0;
                            prog = true;
                        }
                    }
                }
                if (prog) spin.reset();
                else if (!spin.tick(err)) ok = false;
            }
            sm100::mma_commit(&bars[DRAIN]);  // every product issued completes before TMEM is released
            sm100::mbar_wait(&bars[DRAIN], 0u, err, sm100::kWaitLimitNs, true);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q4 = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r = q4 * 32 + lane;  // block row (token); for H, the key dimension
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const float *Gf = prm.G + fh * (long long)((L + 3) & ~3);  // G rows are padded to 16 bytes
        // G at the anchor of block j >= 1 (the last token before it; the frame's last token for j = nblk)
        auto anchor = [&](int j) -> float { return Gf[min(j * BM, L) - 1]; };
        // this row's G and beta, read one block ahead
        auto row_gates = [&](int i, float &g, float &bb) {
            const int rw = i * BM + r;
            const bool ok_row = i < nblk && rw < L;
            g = ok_row ? Gf[rw] : 0.f;
            bb = ok_row ? prm.beta[((long long)b * prm.T + f * L + rw) * prm.H + h] : 0.f;
        };
        bool ok = true;
        float G_next, be_next;
        row_gates(0, G_next, be_next);
        float an0 = 0.f, an1 = anchor(1), an2 = nblk >= 2 ? anchor(2) : 0.f;
        for (int i = 0; i < nblk && ok; ++i) {
            const int row = i * BM + r;
            const bool valid = row < L;
            const float Gr = G_next, be = be_next;
            row_gates(i + 1, G_next, be_next);
            const float aI = an0, aI1 = an1, aI2 = an2;  // anchors of blocks i, i+1, i+2
            an0 = an1;
            an1 = an2;
            an2 = i + 3 <= nblk ? anchor(i + 3) : 0.f;
            unsigned char *kt = sK + (i & 1) * TILE;

            // ---- Y_i = R_i - diag(beta e^{G_r - G_{a_i}}) K_i H_i -> staging (MN-major: row = K index
            //      of T_ii Y_i)
            if (i > 0) ok = sm100::mbar_wait(&bars[ACCFULL + half], (uint32_t)((i - 1) & 1), err, wait_ns);
            // the Ub half reads its v from (and writes Y over) the staging tile's Ub slabs; the W
            // half reads k from K_i and writes over X_{i-1}'s W slabs, once their store has read them
            if (ok && half == 0) ok = sm100::mbar_wait(&bars[VFULL], (uint32_t)(i & 1), err, wait_ns);
            if (ok && half == 1)
                ok = (i == 0 || sm100::mbar_wait(&bars[STBFREE], (uint32_t)((i - 1) & 1), err, wait_ns)) &&
                     sm100::mbar_wait(&bars[KFULL + (i & 1)], (uint32_t)((i >> 1) & 1), err, wait_ns);
            if (!ok) break;
            sm100::tc_fence_after();
            const float rf = (valid && i > 0) ? be * __expf(Gr - aI) : 0.f;
            const int rlen = half ? dk : dv, c_base = half ? dvp : 0;
            const int n16 = rlen >> 4;  // the half's 16-column chunks (d_v and d_k are multiples of 16)
            const float rs = half ? be * __expf(Gr) : be;
            // y = rs x - rf acc over 8 columns from c, x this row's v (landed in the staging tile,
            // overwritten in place) or k; pairs of columns in packed fp32 x2 arithmetic
            const uint64_t rs2 = f32x2(rs, rs), nrf2 = f32x2(-rf, -rf);
            const unsigned char *xsrc = half ? kt : sST;
            auto build = [&](int c, const float *acc, const uint4 xin) {
                const uint32_t xw[4] = {xin.x, xin.y, xin.z, xin.w};
                float y[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    // bf16 pair -> fp32 pair: the low half shifted up, the high half masked
                    const uint64_t xp = f32x2(__uint_as_float(xw[e] << 16), __uint_as_float(xw[e] & 0xffff0000u));
                    const uint64_t yp = fma_f32x2(nrf2, f32x2(acc[2 * e], acc[2 * e + 1]), mul_f32x2(rs2, xp));
                    y[2 * e] = __uint_as_float((uint32_t)yp);
                    y[2 * e + 1] = __uint_as_float((uint32_t)(yp >> 32));
                }
                *reinterpret_cast<uint4 *>(sST + sw_offset(c_base + c, r)) = valid ? pack8(y) : make_uint4(0, 0, 0, 0);
            };
            // the row's next 16 columns are read from shared memory while these are worked on
            uint4 xn0 = *reinterpret_cast<const uint4 *>(xsrc + sw_offset(0, r));
            uint4 xn1 = *reinterpret_cast<const uint4 *>(xsrc + sw_offset(8, r));
            auto chunk = [&](int j, const float *acc) {
                const uint4 x0 = xn0, x1 = xn1;
                if (j + 1 < n16) {
                    xn0 = *reinterpret_cast<const uint4 *>(xsrc + sw_offset(16 * j + 16, r));
                    xn1 = *reinterpret_cast<const uint4 *>(xsrc + sw_offset(16 * j + 24, r));
                }
                build(16 * j, acc, x0);
                build(16 * j + 8, acc + 8, x1);
            };
            if (i > 0) {
                tmem_walk16(t_p + lane_off + c_base, n16, [&](int j, const float (&acc)[16]) { chunk(j, acc); });
            } else {
                const float zero[16] = {};
                for (int j = 0; j < n16; ++j) chunk(j, zero);
            }
            sm100::tc_fence_before();
            sm100::fence_proxy_async_smem();
            sm100::mbar_arrive(&bars[YFULL + half]);
            if (half == 1) {  // off the chain: K_i becomes Kh_i in place once the Ub half's K_i H_i has read it
                if (i > 0) ok = sm100::mbar_wait(&bars[ACCFULL + 0], (uint32_t)((i - 1) & 1), err, wait_ns);
                if (!ok) break;
                const float ksc = valid ? __expf(aI1 - Gr) : 0.f;
                for (int c = 0; c < dk; c += 8) {
                    uint4 *kp = reinterpret_cast<uint4 *>(kt + sw_offset(c, r));
                    uint4 kv = *kp;
                    __nv_bfloat162 *k2 = reinterpret_cast<__nv_bfloat162 *>(&kv);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 fk = __bfloat1622float2(k2[e]);
                        k2[e] = __floats2bfloat162_rn(ksc * fk.x, ksc * fk.y);
                    }
                    *kp = kv;
                }
                sm100::fence_proxy_async_smem();
                sm100::mbar_arrive(&bars[KHREADY]);
            }

            // ---- X_i = T_ii Y_i -> bf16 staging over Y_i (half 0 the Ub columns, half 1 the W columns)
            ok = sm100::mbar_wait(&bars[XFULL + half], (uint32_t)(i & 1), err, wait_ns);
            if (!ok) break;
            sm100::tc_fence_after();
            const int c_lo = half ? dvp : 0;
            tmem_walk16(t_p + lane_off + c_lo, n16, [&](int j, const float (&x)[16]) {
                *reinterpret_cast<uint4 *>(sST + sw_offset(c_lo + 16 * j, r)) = pack8(x);
                *reinterpret_cast<uint4 *>(sST + sw_offset(c_lo + 16 * j + 8, r)) = pack8(x + 8);
            });
            sm100::tc_fence_before();
            sm100::fence_proxy_async_smem();
            sm100::mbar_arrive(&bars[half ? XSTG1 : XSTG0]);

            // ---- H_{i+1} (TMEM lane = key dimension m = r): bf16 copy for K_{i+1} H_{i+1}, and the
            //      fp32 accumulator rescaled to the next anchor; after the last block, M and N
            ok = sm100::mbar_wait(&bars[UFULL + half], (uint32_t)(i & 1), err, wait_ns);
            if (!ok) break;
            sm100::tc_fence_after();
            if (i + 1 < nblk) {
                const float gam = __expf(aI2 - aI1);
                tmem_walk16(t_h + lane_off + c_lo, n16, [&](int j, const float (&x)[16]) {
                    *reinterpret_cast<uint4 *>(sH + sw_offset(c_lo + 16 * j, r)) = pack8(x);
                    *reinterpret_cast<uint4 *>(sH + sw_offset(c_lo + 16 * j + 8, r)) = pack8(x + 8);
                    uint32_t sc[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) sc[e] = __float_as_uint(gam * x[e]);
                    sm100::tmem_st16(t_h + lane_off + c_lo + 16 * j, sc);
                });
                sm100::tmem_st_wait();
                sm100::tc_fence_before();
                sm100::fence_proxy_async_smem();
                sm100::mbar_arrive(&bars[HREADY + half]);
            } else {
                // H = Kt^T [Ub | W]: N = Kt^T Ub (half 0), M = e^{G_L} I - Kt^T W (half 1); every
                // lane takes part in the (warp-wide) TMEM loads, rows m >= d_k store nothing.
                // N and the scan's images of M are staged in shared memory that nothing reads any
                // more (the half's own slabs of the staging tile, once X's last store has read
                // them, and of bf16 H) and leave as whole lines once every role is done (below);
                // fp32 M, when asked for, goes out row by row.
                const float eGL = __expf(aI1);
                const int m = r;
                const FinalStage fs(sST, sH, half, dk, dv, dvp, nslab_v, prm.Mimg, fh);
                ok = sm100::mbar_wait(&bars[half ? STBFREE : STAFREE], (uint32_t)((nblk - 1) & 1), err, wait_ns);
                if (!ok) break;
                unsigned char *stA = fs.stA, *stB = fs.stB;
                const bool stage_n = fs.stage_n;
                unsigned char *img = fs.img;
                const int c_hi = c_lo + rlen;
                for (int c16 = c_lo; c16 < c_hi; c16 += 16) {  // dv is a multiple of 16
                    float v[16];
                    sm100::tmem_ld16(t_h + lane_off + c16, v);
                    sm100::tmem_ld_wait();
                    if (m >= dk) continue;
                    float *dst;
                    if (half == 0) {
                        if (stage_n) {
                            float4 *sp = reinterpret_cast<float4 *>(fs.nrow(m) + c16 * 4);
#pragma unroll
                            for (int e = 0; e < 4; ++e) sp[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
                            continue;
                        }
                        dst = prm.N + (fh * dk + m) * (long long)dv + c16;
                    } else {
                        const int j0 = c16 - dvp;
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = (m == j0 + e ? eGL : 0.f) - v[e];
                        if (img) {  // hi + lo bf16 images of the scan's A operand: hi over bf16 H's W slabs, lo over the staging tile's
#pragma unroll
                            for (int h8 = 0; h8 < 2; ++h8) {
                                uint32_t hi[4], lo[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float a = v[8 * h8 + 2 * e], bb = v[8 * h8 + 2 * e + 1];
                                    const __nv_bfloat162 h2v = __floats2bfloat162_rn(a, bb);
                                    const float2 hf = __bfloat1622float2(h2v);
                                    hi[e] = *reinterpret_cast<const uint32_t *>(&h2v);
                                    lo[e] = pack_bf16(a - hf.x, bb - hf.y);
                                }
                                const uint32_t off = sm100::sw128_kmajor_offset(m, j0 + 8 * h8, dk);
                                *reinterpret_cast<uint4 *>(stB + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                                *reinterpret_cast<uint4 *>(stA + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                            }
                        }
                        if (!prm.M) continue;
                        dst = prm.M + (fh * dk + m) * (long long)dk + j0;
                    }
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4 *>(dst + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                }
                sm100::fence_proxy_async_smem();  // the images are visible to the bulk copies
            }
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp >= 2 && warp < 10) {  // N and M's images out of shared memory (after a failed wait: whatever is there)
        const int half = (warp - 2) >> 2, r = (warp & 3) * 32 + lane;
        const FinalStage fs(sST, sH, half, dk, dv, dvp, nslab_v, prm.Mimg, fh);
        if (half == 0 && fs.stage_n) {  // N of this frame-head is contiguous: 16-byte pieces in order
            const int n4 = dv / 4;
            float4 *dn = reinterpret_cast<float4 *>(prm.N + fh * (long long)dk * dv);
            for (int c = r; c < dk * n4; c += kEpi / 2) {
                const int row = c / n4;
                dn[c] = *reinterpret_cast<const float4 *>(fs.nrow(row) + (c - row * n4) * 16);
            }
        } else if (half == 1 && fs.img && r == 0) {
            const uint32_t part = (uint32_t)(fs.nslab * dk * 128);
            sm100::bulk_copy_s2g(fs.img, fs.stB, part);
            sm100::bulk_copy_s2g(fs.img + part, fs.stA, part);
            sm100::bulk_commit();
            sm100::bulk_wait0();
        }
    }
    if (warp == 1) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tbase, 512);
    }
}

}  // namespace

cudaError_t launch_intra_tc(const CUtensorMap &tm_k, const CUtensorMap &tm_v, const CUtensorMap &tm_t,
                            const CUtensorMap &tm_xu, const CUtensorMap &tm_xw, const IntraParams &prm,
                            long long n_fh, cudaStream_t s) {
    const size_t smem = Smem::END;
    cudaError_t e = cudaFuncSetAttribute(k_intra_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_intra_tc<<<(unsigned)n_fh, kThreads, smem, s>>>(tm_k, tm_v, tm_t, tm_xu, tm_xw, prm);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace gdn
