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
//   1. S = K_i K_i^T on 16x16 lower blocks (mma.sync bf16 -> fp32) and
//      A = beta_r e^{G_r - G_s} S (s < r),
//   2. the eight 16x16 diagonal leaves inverted by forward substitution in
//      fp32 (one column per lane),
//   3. three doubling levels 16 -> 32 -> 64 -> 128:
//      T21 = -T22 (A21 T11)  on the tensor cores (mma.sync, fp32 accumulate).
// T_ii is written row-major bf16 [n_fh][nblk][128][128] (unit diagonal,
// zeros above it), the A operand layout of the solve's T_ii Y_i product.
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kThreads = 256;
constexpr int LDK = 128 + 8;   // bf16 row stride of the K tile (conflict-free ldmatrix)
constexpr int LDT = 128 + 8;   // bf16 row stride of the A / T / scratch tiles
static_assert(LDK == LDT, "the scratch tile reuses the K tile");

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

// A fragment of the 16x16 row-major bf16 block at (r0, c0) of a tile with row stride ld.
__device__ __forceinline__ void load_a(uint32_t (&a)[4], const __nv_bfloat16 *t, int ld, int r0, int c0, int lane) {
    ldsm_x4(a, t + (r0 + (lane & 15)) * ld + c0 + (lane >> 4) * 8);
}
// B fragments (two n8 tiles) of B[k][n] = M[n][k] for a row-major M: rows n0..n0+15, cols k0..k0+15.
__device__ __forceinline__ void load_b_rows(uint32_t (&b)[4], const __nv_bfloat16 *t, int ld, int n0, int k0,
                                            int lane) {
    // matrices: (n 0-7, k 0-7), (n 0-7, k 8-15), (n 8-15, k 0-7), (n 8-15, k 8-15)
    const int n = n0 + (lane & 7) + ((lane >> 4) << 3);
    const int k = k0 + ((lane >> 3) & 1) * 8;
    ldsm_x4(b, t + n * ld + k);
}
// B fragments (two n8 tiles) of B[k][n] = M[k][n] for a row-major M: rows k0..k0+15, cols n0..n0+15.
__device__ __forceinline__ void load_b_trans(uint32_t (&b)[4], const __nv_bfloat16 *t, int ld, int k0, int n0,
                                             int lane) {
    // matrices: (k 0-7, n 0-7), (k 8-15, n 0-7), (k 0-7, n 8-15), (k 8-15, n 8-15)
    const int k = k0 + (lane & 7) + ((lane >> 3) & 1) * 8;
    const int n = n0 + (lane >> 4) * 8;
    ldsm_x4_t(b, t + k * ld + n);
}

// D(16x16) = sum over K of A(16xK) B(Kx16); A row-major at (ra, ca), B = M[k][n] row-major at (kb, nb).
__device__ __forceinline__ void mm16_trans(float (&d0)[4], float (&d1)[4], const __nv_bfloat16 *A, int ra, int ca,
                                           const __nv_bfloat16 *M, int kb, int nb, int K, int lane) {
    for (int k = 0; k < K; k += 16) {
        uint32_t a[4], b[4];
        load_a(a, A, LDT, ra, ca + k, lane);
        load_b_trans(b, M, LDT, kb + k, nb, lane);
        mma16816(d0, a, b[0], b[1]);
        mma16816(d1, a, b[2], b[3]);
    }
}

// Store a 16x16 fp32 accumulator pair as bf16 at (r0, c0), times `scale`.
__device__ __forceinline__ void store16(__nv_bfloat16 *t, int r0, int c0, const float (&d0)[4],
                                        const float (&d1)[4], float scale, int lane) {
    const int g = lane >> 2, q = lane & 3;
    __nv_bfloat162 *p;
    p = reinterpret_cast<__nv_bfloat162 *>(t + (r0 + g) * LDT + c0 + 2 * q);
    *p = __floats2bfloat162_rn(scale * d0[0], scale * d0[1]);
    p = reinterpret_cast<__nv_bfloat162 *>(t + (r0 + g + 8) * LDT + c0 + 2 * q);
    *p = __floats2bfloat162_rn(scale * d0[2], scale * d0[3]);
    p = reinterpret_cast<__nv_bfloat162 *>(t + (r0 + g) * LDT + c0 + 8 + 2 * q);
    *p = __floats2bfloat162_rn(scale * d1[0], scale * d1[1]);
    p = reinterpret_cast<__nv_bfloat162 *>(t + (r0 + g + 8) * LDT + c0 + 8 + 2 * q);
    *p = __floats2bfloat162_rn(scale * d1[2], scale * d1[3]);
}

struct InvParams {
    const __nv_bfloat16 *k;  // [B,T,H,dk]
    const float *beta;       // [B,T,H]
    const float *G;          // [n_fh][L]
    __nv_bfloat16 *Tinv;     // [n_fh][nblk][128][128]
    int L, dk, H, nblk;
    long long F, T;
};

__global__ void __launch_bounds__(kThreads, 2) k_diag_inverse(const InvParams prm) {
    extern __shared__ __align__(16) unsigned char smem[];
    __nv_bfloat16 *sK = (__nv_bfloat16 *)smem;          // [128][LDK]
    __nv_bfloat16 *sA = sK + 128 * LDK;                 // [128][LDT]  A (strictly lower)
    __nv_bfloat16 *sT = sA + 128 * LDT;                 // [128][LDT]  T
    __nv_bfloat16 *sX = sK;                             // scratch products reuse the K tile (LDK == LDT)
    float *sAd = (float *)(sT + 128 * LDT);             // [8][16][16] fp32 diagonal leaves of A
    float *sG = sAd + 8 * 256;                          // [128]
    float *sB = sG + 128;                               // [128]

    const int L = prm.L, dk = prm.dk, nblk = prm.nblk;
    const long long fh = blockIdx.x / nblk;
    const int blk = (int)(blockIdx.x % nblk);
    const long long f = fh % prm.F, chain = fh / prm.F;
    const int h = (int)(chain % prm.H), b = (int)(chain / prm.H);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r_base = blk * 128;

    // ---- load K_i (rows past the frame are zero), gates, clear T
    for (int e = tid; e < 128 * (dk / 8); e += kThreads) {
        const int r = e / (dk / 8), c8 = e % (dk / 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r_base + r < L) {
            const long long t = f * L + r_base + r;
            v = *reinterpret_cast<const uint4 *>(prm.k + (((long long)b * prm.T + t) * prm.H + h) * dk + c8 * 8);
        }
        *reinterpret_cast<uint4 *>(sK + r * LDK + c8 * 8) = v;
    }
    for (int e = tid; e < 128 * ((128 - dk) / 8); e += kThreads) {  // zero the padding columns up to 128
        const int r = e / ((128 - dk) / 8), c8 = e % ((128 - dk) / 8);
        *reinterpret_cast<uint4 *>(sK + r * LDK + dk + c8 * 8) = make_uint4(0, 0, 0, 0);
    }
    for (int e = tid; e < 128 * 16; e += kThreads) {
        const int r = e >> 4, c8 = e & 15;
        *reinterpret_cast<uint4 *>(sT + r * LDT + c8 * 8) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>(sA + r * LDT + c8 * 8) = make_uint4(0, 0, 0, 0);
    }
    if (tid < 128) {
        const int r = r_base + tid;
        const float *Gf = prm.G + fh * (long long)((L + 3) & ~3);  // G rows are padded to 16 bytes
        sG[tid] = Gf[r < L ? r : L - 1];
        sB[tid] = (r < L) ? prm.beta[((long long)b * prm.T + f * L + r) * prm.H + h] : 0.f;
    }
    __syncthreads();

    // ---- A = beta_r e^{G_r - G_s} (K K^T)[r][s], s < r, on the 36 lower 16x16 blocks
    const int g = lane >> 2, q = lane & 3;
    for (int blkid = warp; blkid < 36; blkid += 8) {
        int ab = 0, rem = blkid;  // block row ab, block column cb <= ab
        while (rem > ab) { rem -= ab + 1; ++ab; }
        const int cb = rem;
        float d0[4] = {0, 0, 0, 0}, d1[4] = {0, 0, 0, 0};
        for (int kk = 0; kk < dk; kk += 16) {
            uint32_t a[4], bb[4];
            load_a(a, sK, LDK, ab * 16, kk, lane);
            load_b_rows(bb, sK, LDK, cb * 16, kk, lane);
            mma16816(d0, a, bb[0], bb[1]);
            mma16816(d1, a, bb[2], bb[3]);
        }
        // element (r, s) of this thread's fragments
        const float *dd[2] = {d0, d1};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = ab * 16 + g + (e >> 1) * 8;
                const int s = cb * 16 + nt * 8 + 2 * q + (e & 1);
                const float val = (s < r) ? sB[r] * __expf(sG[r] - sG[s]) * dd[nt][e] : 0.f;
                sA[r * LDT + s] = __float2bfloat16_rn(val);
                if (ab == cb) sAd[ab * 256 + (r - ab * 16) * 16 + (s - cb * 16)] = val;
            }
        }
    }
    __syncthreads();

    // ---- leaves: warp w inverts diagonal block w; lane c < 16 owns column c
    if (lane < 16) {
        const float *ad = sAd + warp * 256;
        const int c = lane;
        float t[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float x = (r == c) ? 1.f : 0.f;
#pragma unroll
            for (int s = 0; s < r; ++s) x -= ad[r * 16 + s] * t[s];
            t[r] = x;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) sT[(warp * 16 + r) * LDT + warp * 16 + c] = __float2bfloat16_rn(t[r]);
    }
    __syncthreads();

    // ---- doubling: T21 = -T22 (A21 T11) for block sizes 16, 32, 64
    for (int sz = 16; sz <= 64; sz <<= 1) {
        const int nmerge = 128 / (2 * sz);
        const int tiles = (sz / 16) * (sz / 16);   // 16x16 output tiles per merge
        // X = A21 T11 into sX (rows of the lower half, cols of the upper half)
        for (int w = warp; w < nmerge * tiles; w += 8) {
            const int m = w / tiles, tt = w % tiles;
            const int base = m * 2 * sz;
            const int tr = (tt / (sz / 16)) * 16, tc = (tt % (sz / 16)) * 16;
            float d0[4] = {0, 0, 0, 0}, d1[4] = {0, 0, 0, 0};
            mm16_trans(d0, d1, sA, base + sz + tr, base, sT, base, base + tc, sz, lane);
            store16(sX, base + sz + tr, base + tc, d0, d1, 1.f, lane);
        }
        __syncthreads();
        // T21 = -T22 X
        for (int w = warp; w < nmerge * tiles; w += 8) {
            const int m = w / tiles, tt = w % tiles;
            const int base = m * 2 * sz;
            const int tr = (tt / (sz / 16)) * 16, tc = (tt % (sz / 16)) * 16;
            float d0[4] = {0, 0, 0, 0}, d1[4] = {0, 0, 0, 0};
            mm16_trans(d0, d1, sT, base + sz + tr, base + sz, sX, base + sz, base + tc, sz, lane);
            store16(sT, base + sz + tr, base + tc, d0, d1, -1.f, lane);
        }
        __syncthreads();
    }

    // ---- write T_ii row-major
    __nv_bfloat16 *dst = prm.Tinv + (fh * nblk + blk) * (long long)(128 * 128);
    for (int e = tid; e < 128 * 16; e += kThreads) {
        const int r = e >> 4, c8 = e & 15;
        *reinterpret_cast<uint4 *>(dst + r * 128 + c8 * 8) = *reinterpret_cast<const uint4 *>(sT + r * LDT + c8 * 8);
    }
}

}  // namespace

size_t diag_inverse_smem_bytes() {
    return sizeof(__nv_bfloat16) * (128 * LDK + 2 * 128 * LDT) + sizeof(float) * (8 * 256 + 256);
}

cudaError_t launch_diag_inverse(const __nv_bfloat16 *k, const float *beta, const float *G, __nv_bfloat16 *Tinv,
                                int L, int dk, int H, int nblk, long long F, long long T, long long n_fh,
                                cudaStream_t s) {
    InvParams prm{k, beta, G, Tinv, L, dk, H, nblk, F, T};
    const size_t smem = diag_inverse_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(k_diag_inverse, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_diag_inverse<<<(unsigned)(n_fh * nblk), kThreads, smem, s>>>(prm);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace gdn
