// tc_diag_inverse.cu -- inverses of the 128x128 diagonal blocks of (I + A).
//
// The intra-frame solve of the chunkwise gated delta rule is the unit lower
// triangular system (I + A)[Ub | W] = [beta V | beta e^G K] with
// A_ij = beta_i e^{G_i - G_j} k_i.k_j (j < i) (the UT/WY form of the delta
// rule over one frame; SANA-WM summary, "Memory-Efficient Long-Context
// Modeling (Section 3.2)", frame-wise GDN).  Blocked forward substitution
// over 128-row blocks needs T_ii = (I + A_ii)^{-1} for every diagonal block;
// they do not depend on each other or on the solve, so this kernel computes
// all of them in parallel, one CTA per (frame-head, block):
//   1. S = K_i K_i^T on the 5th-generation tensor cores (one 128 x 128 tcgen05
//      product into TMEM; K_i arrives in the 128-byte swizzled layout by two
//      tiled loads through k's tensor map) and A = beta_r e^{G_r - G_s} S
//      (s < r) by the epilogue, one row per thread,
//   2. the eight 16x16 diagonal leaves inverted by forward substitution in
//      fp32 (one column per lane),
//   3. three doubling levels 16 -> 32 -> 64 -> 128:
//      T21 = -(T22 A21) T11  on the tensor cores (mma.sync, fp32 accumulate),
//      one pass per level: each of four warps owns a 16-row panel of T21 and
//      keeps the intermediate T22 A21 in registers, where the accumulator
//      layout is already the A operand layout of the second product, so a
//      level needs no scratch tile and one block barrier; the zero triangles
//      of T11 and T22 are skipped.
// T_ii is written row-major bf16 [n_fh][nblk][128][128] (unit diagonal,
// zeros above it), the A operand layout of the solve's T_ii Y_i product, by
// two tiled stores of the shared-memory tile (held in the tensor map's
// swizzle throughout).
// Shared memory per CTA: A written over K once the Gram has read it, T, and
// the fp32 leaves (74 KB), so three CTAs share an SM and one's loads overlap
// the others' arithmetic.
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kThreads = 256;
constexpr uint32_t TILE = 128 * 256;  // one 128 x 128 bf16 tile (32 KB)
constexpr int AD = 17;         // fp32 row stride of a diagonal leaf (odd: rows hit distinct banks)
constexpr float kSplitMax = 60.f;  // largest row exponent the split decay takes (else the exact one)

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(sm100::smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(sm100::smem_u32(p)));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of element (row, col) of a 128 x 128 bf16 tile in the tensor maps' 128-byte
// swizzle: two 64-column slabs of 128-byte rows whose 16-byte chunks are permuted by the row's
// low three bits, so the eight rows one ldmatrix matrix reads, or one chunk of 32 consecutive
// rows, fall in distinct banks, and T leaves by two tiled stores as it is.
__device__ __forceinline__ uint32_t swz(int row, int col) {
    return (uint32_t)((col >> 6) * SLAB_BYTES + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) +
                      ((col & 7) << 1));
}

// A fragment of the 16x16 block at (r0, c0) of a tile.
__device__ __forceinline__ void load_a(uint32_t (&a)[4], const unsigned char *t, int r0, int c0, int lane) {
    ldsm_x4(a, t + swz(r0 + (lane & 15), c0 + (lane >> 4) * 8));
}
// B fragments (two n8 tiles) of B[k][n] = M[k][n] for the tile M: rows k0..k0+15, cols n0..n0+15.
__device__ __forceinline__ void load_b_trans(uint32_t (&b)[4], const unsigned char *t, int k0, int n0, int lane) {
    // matrices: (k 0-7, n 0-7), (k 8-15, n 0-7), (k 0-7, n 8-15), (k 8-15, n 8-15)
    const int k = k0 + (lane & 7) + ((lane >> 3) & 1) * 8;
    const int n = n0 + (lane >> 4) * 8;
    ldsm_x4_t(b, t + swz(k, n));
}

// Store a 16x16 fp32 accumulator pair as bf16 at (r0, c0), times `scale`.
__device__ __forceinline__ void store16(unsigned char *t, int r0, int c0, const float (&d0)[4], const float (&d1)[4],
                                        float scale, int lane) {
    const int g = lane >> 2, q = lane & 3;
    *reinterpret_cast<uint32_t *>(t + swz(r0 + g, c0 + 2 * q)) = pack_bf16(scale * d0[0], scale * d0[1]);
    *reinterpret_cast<uint32_t *>(t + swz(r0 + g + 8, c0 + 2 * q)) = pack_bf16(scale * d0[2], scale * d0[3]);
    *reinterpret_cast<uint32_t *>(t + swz(r0 + g, c0 + 8 + 2 * q)) = pack_bf16(scale * d1[0], scale * d1[1]);
    *reinterpret_cast<uint32_t *>(t + swz(r0 + g + 8, c0 + 8 + 2 * q)) = pack_bf16(scale * d1[2], scale * d1[3]);
}

// One doubling level: for each pair of SZ x SZ diagonal blocks of T (inverses T11, T22 of the
// diagonal blocks of I + A, already in place), the block below the diagonal
//   T21 = -(T22 A21) T11,
// the off-diagonal block of the inverse of [[I + A11, 0], [A21, I + A22]].  There are always four
// 16-row panels of T21 per level; warp p < 4 takes one: W = T22[panel, :] A21 (16 x SZ, k-steps up
// to the panel's diagonal only, T22 being lower triangular) stays in registers as fp32
// accumulators, is rounded to bf16 A fragments (the accumulator layout of m16n8k16 is the A
// fragment layout), and T21[panel, c] = -W T11[:, c] takes only the k-steps at or below c's
// (T11 is lower triangular).
template <int SZ>
__device__ __forceinline__ void merge_level(unsigned char *sT, const unsigned char *sA, int warp, int lane) {
    constexpr int NP = SZ / 16;  // 16-row panels per merge; 128 / (2 SZ) merges x NP panels = 4
    if (warp >= 4) return;
    const int m = warp / NP, p = warp % NP;
    const int base = m * 2 * SZ;
    const int r0 = base + SZ + 16 * p;  // the panel's rows (of T22, A21 and T21)
    float w[2 * NP][4];
#pragma unroll
    for (int t = 0; t < 2 * NP; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) w[t][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < NP; ++ks) {
        if (ks > p) break;  // T22[panel][k] = 0 past the panel's diagonal block
        uint32_t af[4];
        load_a(af, sT, r0, base + SZ + 16 * ks, lane);
#pragma unroll
        for (int n2 = 0; n2 < NP; ++n2) {
            uint32_t bf[4];
            load_b_trans(bf, sA, base + SZ + 16 * ks, base + 16 * n2, lane);
            mma16816(w[2 * n2], af, bf[0], bf[1]);
            mma16816(w[2 * n2 + 1], af, bf[2], bf[3]);
        }
    }
    uint32_t wa[NP][4];
#pragma unroll
    for (int js = 0; js < NP; ++js) {
        wa[js][0] = pack_bf16(w[2 * js][0], w[2 * js][1]);
        wa[js][1] = pack_bf16(w[2 * js][2], w[2 * js][3]);
        wa[js][2] = pack_bf16(w[2 * js + 1][0], w[2 * js + 1][1]);
        wa[js][3] = pack_bf16(w[2 * js + 1][2], w[2 * js + 1][3]);
    }
#pragma unroll
    for (int cp = 0; cp < NP; ++cp) {
        float d[2][4] = {};
#pragma unroll
        for (int js = cp; js < NP; ++js) {  // T11[j][c] = 0 for j above c's block
            uint32_t bf[4];
            load_b_trans(bf, sT, base + 16 * js, base + 16 * cp, lane);
            mma16816(d[0], wa[js], bf[0], bf[1]);
            mma16816(d[1], wa[js], bf[2], bf[3]);
        }
        store16(sT, r0, base + 16 * cp, d[0], d[1], -1.f, lane);
    }
}

struct InvParams {        // k and T_ii move through tensor maps (tm_k, tm_t)
    const float *beta;       // [B,T,H]
    const float *G;          // [n_fh][(L+3)&~3]
    const float *CF;         // [n_fh][(L+3)&~3] column factors e^{a - G_s} (a = G at the end of s's 64-token group)
    int L, dk, H, nblk;
    long long F, T;
    int *err;                // bounded-wait error word
    uint64_t wait_ns;        // limit of the bounded wait
    int drop_first;          // debug: the first block's Gram is not issued, so its wait gives up
};

__global__ void __launch_bounds__(kThreads, 3)
k_diag_inverse(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_t,
               const InvParams prm) {
    // the K tile's 128-byte swizzle needs a 1024-aligned base: the dynamic shared memory base is
    // (the kernel declares no static shared memory), and it is checked below
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *sKs = smem;             // K_i, SW128 K-major, 2 slabs x 128 rows (32 KB), read by the Gram
    unsigned char *sA = smem;              // A (strictly lower), written over K once the Gram has completed
    unsigned char *sT = smem + TILE;       // T
    float *sAd = (float *)(smem + 2 * TILE);  // [8][16][AD] fp32 diagonal leaves of A
    float *sG = sAd + 8 * 16 * AD;                      // [128]
    float *sCF = sG + 128;                              // [128]
    float *sB = sCF + 128;                              // [128]
    uint64_t *bar = (uint64_t *)(sB + 128);  // the Gram's completion
    uint64_t *lbar = bar + 1;                 // K_i landed
    uint32_t *tslot = (uint32_t *)(bar + 2);
    int *sok = (int *)(tslot + 1);

    if (pass_failed(prm.err)) return;  // an earlier stage of this pass gave up
    if (sm100::smem_u32(smem) & 1023u) {  // every thread sees the same base: all leave together
        if (threadIdx.x == 0) atomicCAS(prm.err, sm100::kErrNone, sm100::kErrSmemAlign);
        return;
    }
    const int L = prm.L, dk = prm.dk, nblk = prm.nblk;
    const long long fh = blockIdx.x / nblk;
    const int blk = (int)(blockIdx.x % nblk);
    const long long f = fh % prm.F, chain = fh / prm.F;
    const int h = (int)(chain % prm.H), b = (int)(chain / prm.H);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r_base = blk * 128;

    // ---- K_i by two tiled loads (rows past the frame and columns past d_k read as zeros), the
    //      gates by asynchronous copies; meanwhile the 16x16 tiles of T above its diagonal are
    //      cleared (T leaves by tiled stores; nothing else writes them)
    if (tid == 0) {
        sm100::mbar_init(bar, 1);
        sm100::mbar_init(lbar, 1);
        sm100::fence_barrier_init();
        const int nslab = (dk + 63) / 64;
        sm100::mbar_arrive_expect_tx(lbar, (uint32_t)(nslab * SLAB_BYTES));
        for (int sl = 0; sl < nslab; ++sl)
            sm100::tma_load_4d(sKs + sl * SLAB_BYTES, &tm_k, lbar, sl * 64, h, r_base, (int)(b * prm.F + f));
    }
    for (int e = tid; e < 128 * 16; e += kThreads) {
        const int r = e >> 4, c8 = e & 15;
        if ((c8 >> 1) > (r >> 4)) *reinterpret_cast<uint4 *>(sT + swz(r, 8 * c8)) = make_uint4(0, 0, 0, 0);
    }
    if (tid < 128) {
        const int r = r_base + tid;
        const float *Gf = prm.G + fh * (long long)((L + 3) & ~3);  // G rows are padded to 16 bytes
        sm100::cp_async4(sG + tid, Gf + (r < L ? r : L - 1));
        sm100::cp_async4(sCF + tid, prm.CF + fh * (long long)((L + 3) & ~3) + (r < L ? r : L - 1));
        if (r < L) sm100::cp_async4(sB + tid, prm.beta + ((long long)b * prm.T + f * L + r) * prm.H + h);
        else sB[tid] = 0.f;
    }
    sm100::cp_async_commit();
    if (warp == 0) {
        sm100::tmem_alloc(tslot, 128);
        sm100::tmem_relinquish();
    }
    sm100::cp_async_wait_all();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tslot;

    // ---- S = K K^T in TMEM (one thread issues once K_i has landed), then the bounded wait by the
    //      same thread
    if (tid == 0) {
        const bool landed = sm100::mbar_wait(lbar, 0, prm.err, prm.wait_ns);
        if (!landed) sm100::mbar_wait(lbar, 0, prm.err, sm100::kWaitLimitNs, true);  // no copy left in flight
        // debug switch: the first block's product is never issued, so this wait gives up (no fault)
        const bool issue = landed && !(prm.drop_first && blockIdx.x == 0);
        if (issue) {
            const uint32_t id = sm100::idesc_bf16(128, 128, 0, 0);
            for (int ks = 0; ks < dk / 16; ++ks)
                sm100::mma_bf16_ss(tmem, desc_kmajor(sKs, ks, 128), desc_kmajor(sKs, ks, 128), id, ks > 0);
            sm100::mma_commit(bar);
        }
        *sok = sm100::mbar_wait(bar, 0, prm.err, prm.wait_ns) ? 1 : 0;
        // a product issued but not seen complete finishes before TMEM is released (full limit)
        if (!*sok && issue) sm100::mbar_wait(bar, 0, prm.err, sm100::kWaitLimitNs, true);
    }
    __syncthreads();
    if (*sok) {
        sm100::tc_fence_after();
        // ---- A = beta_r e^{G_r - G_s} S[r][s], s < r: thread (warp, lane) owns row r = 32 (warp % 4) + lane
        //      and columns 64 (warp / 4) .. + 63, read from TMEM 32 at a time (warp-uniform skips)
        const int q4 = warp & 3, hw = warp >> 2, r = q4 * 32 + lane;
        const float br = sB[r], gr = sG[r];
        // Decay e^{G_r - G_s} = e^{G_r - a} cf_s, a = G at the end of the 64-token group of
        // columns 64 hw .. 64 hw + 63 (the anchor cf was made with; the block starts on a group
        // boundary).  A row after the group: e^{G_r - a} <= 1.  A row inside it: >= 1, bounded by
        // e^{kSplitMax}, else the exact per-element exponential.  A row before it sees none of it.
        const int nrow = min(128, L - r_base);
        const float dG = gr - sG[min(64 * hw + 63, nrow - 1)];
        const bool before = r < 64 * hw, inside = !before && r < 64 * hw + 64;
        const bool exact = inside && !(dG <= kSplitMax);
        const float rf = (before || exact) ? 0.f : br * __expf(dG);
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int c0 = 64 * hw + 32 * rr;
            if (c0 >= q4 * 32 + 32) continue;  // no row of this warp has s < r in these columns
            float v[32];
            sm100::tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + c0, v);
            sm100::tmem_ld_wait();
            float a[32];
            if (!exact) {
#pragma unroll
                for (int e = 0; e < 32; ++e) a[e] = c0 + e < r ? rf * sCF[c0 + e] * v[e] : 0.f;
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) a[e] = c0 + e < r ? br * __expf(gr - sG[c0 + e]) * v[e] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
                *reinterpret_cast<uint4 *>(sA + swz(r, c0 + 8 * u)) =
                    make_uint4(pack_bf16(a[8 * u], a[8 * u + 1]), pack_bf16(a[8 * u + 2], a[8 * u + 3]),
                               pack_bf16(a[8 * u + 4], a[8 * u + 5]), pack_bf16(a[8 * u + 6], a[8 * u + 7]));
            // the fp32 diagonal 16 x 16 block of this row, when it lies in these columns
            const int db = r >> 4;
            if ((db * 16) >= c0 && (db * 16) < c0 + 32) {
                const bool lo = db * 16 == c0;
#pragma unroll
                for (int e = 0; e < 16; ++e) sAd[(db * 16 + (r & 15)) * AD + e] = lo ? a[e] : a[16 + e];
            }
        }
    }
    sm100::tc_fence_before();
    __syncthreads();

    // ---- leaves: warp w inverts diagonal block w; lane c < 16 owns column c.  Right-looking:
    //      once t_s is final it is taken out of every later row at once, so each step's
    //      updates are independent (the chain is 16 steps deep, not 120)
    if (lane < 16) {
        const float *ad = sAd + warp * 16 * AD;
        const int c = lane;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == c) ? 1.f : 0.f;
#pragma unroll
        for (int s = 0; s < 15; ++s) {
#pragma unroll
            for (int r = s + 1; r < 16; ++r) x[r] = fmaf(-ad[r * AD + s], x[s], x[r]);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r)
            *reinterpret_cast<__nv_bfloat16 *>(sT + swz(warp * 16 + r, warp * 16 + c)) = __float2bfloat16_rn(x[r]);
    }
    __syncthreads();

    // ---- doubling: T21 = -(T22 A21) T11 for block sizes 16, 32, 64 (one merge level per pass)
    merge_level<16>(sT, sA, warp, lane);
    __syncthreads();
    merge_level<32>(sT, sA, warp, lane);
    __syncthreads();
    merge_level<64>(sT, sA, warp, lane);
    sm100::fence_proxy_async_smem();  // T's writes are visible to the tiled stores
    __syncthreads();

    // ---- T_ii out: two tiled stores (its layout is the tensor map's), complete before the CTA leaves
    if (tid == 0) {
        for (int sl = 0; sl < 2; ++sl)
            sm100::tma_store_3d(&tm_t, sT + sl * SLAB_BYTES, sl * 64, 0, (int)(fh * nblk + blk));
        sm100::bulk_commit();
        sm100::bulk_wait0();
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, 128);
    }
}

}  // namespace

size_t diag_inverse_smem_bytes() {
    return 2 * TILE + sizeof(float) * (8 * 16 * AD + 3 * 128) + 24;
}

cudaError_t launch_diag_inverse(const CUtensorMap &tm_k, const CUtensorMap &tm_t, const float *beta, const float *G,
                                const float *CF, int L, int dk, int H, int nblk, long long F, long long T,
                                long long n_fh, int *err, uint64_t wait_ns, int drop_first, cudaStream_t s) {
    InvParams prm{beta, G, CF, L, dk, H, nblk, F, T, err, wait_ns, drop_first};
    const size_t smem = diag_inverse_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(k_diag_inverse, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // three CTAs per SM (their shared memory, registers and TMEM columns all fit three times)
    e = cudaFuncSetAttribute(k_diag_inverse, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    k_diag_inverse<<<(unsigned)(n_fh * nblk), kThreads, smem, s>>>(tm_k, tm_t, prm);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace gdn
