// tc_common.cuh -- shared pieces of the tensor-core (tcgen05) kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "gdn_internal.h"
#include "sm100.cuh"

namespace gdn {
namespace tc {

constexpr int BM = 128;          // token rows per tile (UMMA M)
constexpr int SLAB = 64;         // bf16 columns per 128-byte swizzle slab
constexpr int SLAB_BYTES = BM * 128;  // one 128-row slab

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Barrier among `nthreads` threads (a multiple of 32) on hardware barrier `id` (1..15).
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// The same barrier, returning the AND of every participant's `ok`: threads that each
// made a bounded wait take one common decision to go on or to leave, so no thread is
// left waiting at a later barrier for one that left.
__device__ __forceinline__ bool named_sync_and(int id, int nthreads, bool ok) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)ok), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// A kernel of a pass whose earlier stage recorded a failure in the error word does
// nothing: every thread reads the word before any barrier is armed or TMEM allocated, so a
// pass that gave up leaves no copy or product in flight behind it.  Only earlier kernels of
// the same stream write the word, so every thread of this kernel reads the same value (and
// no shared memory is spent on it: occupancy stays as the kernel's own budget sets it).
__device__ __forceinline__ bool pass_failed(const int *err) { return *(volatile const int *)err != 0; }

// K-major SW128 operand: tile of `rows` rows, 64-column slabs; K step ks (16 columns).
__device__ __forceinline__ uint64_t desc_kmajor(const void *tile, int ks, int rows) {
    const uint32_t a = sm100::smem_u32(tile) + (uint32_t)((ks >> 2) * rows * 128 + (ks & 3) * 32);
    return sm100::smem_desc(a, 16, 1024, sm100::kSwizzle128B);
}

// MN-major SW128 operand: `krows` rows along K, 64-column slabs along MN
// (slab stride krows*128 bytes); K step ks covers rows 16ks..16ks+15.
__device__ __forceinline__ uint64_t desc_mnmajor(const void *tile, int ks, int krows) {
    const uint32_t a = sm100::smem_u32(tile) + (uint32_t)(ks * 16 * 128);
    return sm100::smem_desc(a, (uint32_t)krows * 128, 1024, sm100::kSwizzle128B);
}

// bf16 column c, row r of a 128-row tile of 64-column SW128 slabs (K-major rows)
__device__ __forceinline__ uint32_t sw_offset(int c, int r) {
    return (uint32_t)((c >> 6) * SLAB_BYTES + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4));
}

// Walks n16 16-column chunks of this warp's TMEM lanes from taddr, loading each chunk while
// fn(j, chunk) works on the one before it (tcgen05.wait::ld waits for every load in flight,
// so one load is ahead at a time).  Two chunks per loop turn: a small body, because a
// kernel's warp roles share the instruction cache.  Warp-uniform: every lane takes part.
template <typename F>
__device__ __forceinline__ void tmem_walk16(uint32_t taddr, int n16, F &&fn) {
    if (n16 <= 0) return;
    float b0[16], b1[16];
    sm100::tmem_ld16(taddr, b0);
#pragma unroll 1
    for (int j = 0; j < n16; j += 2) {
        sm100::tmem_ld_wait();
        if (j + 1 < n16) sm100::tmem_ld16(taddr + 16 * (j + 1), b1);
        fn(j, b0);
        if (j + 1 >= n16) break;
        sm100::tmem_ld_wait();
        if (j + 2 < n16) sm100::tmem_ld16(taddr + 16 * (j + 2), b0);
        fn(j + 1, b1);
    }
}

__device__ __forceinline__ uint4 pack8(const float *x) {
    return make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
}

struct OutParams {
    const float *G;          // [n_fh][(L+3)&~3] inclusive prefix of clamped log alpha per frame
    const float *CF;         // [n_fh][(L+3)&~3] column decay factors e^{a(s) - G_s}, a = G at the end of s's
                             // 64-token tile (G and cf rows are padded to a multiple of 4 floats)
    void *o;                 // [B,T,H,dv] bf16
    int L, dk, dv, H, nblk;
    long long F, T, n_fh;
    int accumulate;          // o += result (formed in fp32, rounded once)
    int reverse_out;         // the pass ran on token-reversed inputs: row t goes to token T - 1 - t
    const __nv_bfloat16 *SigB;  // [n_fh][dk][dv] bf16 state entering each frame (from the scan)
    int *err;
    uint64_t wait_ns;
    int o_tma;               // o is written by tiled stores through tm_o (neither accumulate nor reverse_out)
};

struct IntraParams {
    const float *G;            // [n_fh][(L+3)&~3]
    const float *beta;         // [B,T,H]
    __nv_bfloat16 *X;          // [n_fh][L][dk + dv]: Ub (first dv columns) then W
    float *M;                  // [n_fh][dk][dk] fp32, or null
    __nv_bfloat16 *Mimg;       // or null: M as the scan's bf16 hi + lo operand images (see TransParams)
    float *N;                  // [n_fh][dk][dv]
    int L, dk, dv, H, nblk;
    long long F, T;
    int *err;
    uint64_t wait_ns;
};

struct TransParams {
    float *M;                  // [n_fh][dk][dk] fp32, or null
    __nv_bfloat16 *Mimg;       // or null: M split into bf16 hi + lo, each in the 128-byte-swizzled
                               // K-major image of 64-column slabs of dk rows (the scan's A operand)
    float *N;                  // [n_fh][dk][dv]
    int L, dk, dv, H;
    long long F;
    int *err;
    // the frame-wise operator's map: M = gamma (I - K^T diag(beta) K), N = K^T diag(beta) V
    const float *beta;         // [B,T,H]
    const float *gamma;        // [B,F,H]
    long long T;
    uint64_t wait_ns;          // limit of the bounded waits
    // the key feature map applied to the staged K rows (both copies) before the products,
    // K <- max(RMSNorm(K) * w, 0) * k_post; 0: keys used as given
    int norm_k;
    const float *k_w;          // [dk] RMSNorm weight or null (ones)
    float k_post;              // 1 / sqrt(dk * L)
};

struct UParams {
    const __nv_bfloat16 *X;    // [n_fh][L][dv + dk]
    __nv_bfloat16 *U;          // [n_fh][L][dv]
    int L, dk, dv, nblk;
    int *err;
    // frame-wise operator: A = the frame's queries (tm_q), o = Q Sig written (or added) to o
    int frame;
    __nv_bfloat16 *o;          // [B,T,H,dv]
    long long T, F;
    int H, accumulate;
    uint64_t wait_ns;          // limit of the bounded waits
    // frame-wise operator: the query feature map applied to the staged Q rows before the
    // product, Q <- max(RMSNorm(Q) * w, 0); 0: queries used as given
    int norm_q;
    const float *q_w;          // [dk] RMSNorm weight or null (ones)
};

// RMSNorm epsilon of the q/k feature maps (the pages give none; 1e-6).
constexpr float kRmsEps = 1e-6f;

// tm_k / tm_v deliver 64-token boxes of k / v.  The frame-wise operator's per-frame map.
cudaError_t launch_transition_tc(const CUtensorMap &tm_k, const CUtensorMap &tm_v, const TransParams &prm,
                                 long long n_fh, cudaStream_t s);
// tm_x delivers 128-row boxes of X, tm_q 128-token boxes of q (frame-wise
// operator), tm_sig the bf16 state of a frame-head.
// tm_u stores 128-row boxes of U (chunkwise; unused by the frame-wise operator).
cudaError_t launch_u_tc(const CUtensorMap &tm_x, const CUtensorMap &tm_q, const CUtensorMap &tm_sig,
                        const CUtensorMap &tm_u, const UParams &prm, long long n_fh, int num_sms, cudaStream_t s);

// tm_k / tm_v deliver 128-token boxes of k / v, tm_t one 128 x 128 block of T; tm_xu / tm_xw
// store 128-row boxes of X's Ub columns / W columns (maps over those columns of the
// [Ub | W] rows).  Also writes the frame's transition (N, and M and/or its images).
cudaError_t launch_intra_tc(const CUtensorMap &tm_k, const CUtensorMap &tm_v, const CUtensorMap &tm_t,
                            const CUtensorMap &tm_xu, const CUtensorMap &tm_xw, const IntraParams &prm,
                            long long n_fh, cudaStream_t s);

// One CTA per (frame-head, 128-row block).  drop_first (debug): the first block's Gram is not
// issued, so its bounded wait gives up and the pass reports a timeout without any fault.
// tm_k delivers 128-token boxes of k (as for intra); tm_t is T's map (the one intra loads with),
// through which the kernel stores each T_ii.
cudaError_t launch_diag_inverse(const CUtensorMap &tm_k, const CUtensorMap &tm_t, const float *beta, const float *G,
                                const float *CF, int L, int dk, int H, int nblk, long long F, long long T,
                                long long n_fh, int *err, uint64_t wait_ns, int drop_first, cudaStream_t s);

// tm_q / tm_k / tm_u / tm_g / tm_cf deliver 128-token boxes.
// The scan over frames on the tensor cores (tc_scan.cu): M from the transition
// kernel's images, N fp32; writes the bf16 (and optionally fp32) state of every
// frame and S_out.  scan_tc_supported: whether its shared memory fits these dims.
bool scan_tc_supported(int dk, int dv);
size_t scan_mimg_bytes(int dk);
cudaError_t launch_scan_tc(const Problem &p, const __nv_bfloat16 *Mimg, const float *Nb, __nv_bfloat16 *SigB,
                           float *SigF, int *err, uint64_t wait_ns, cudaStream_t s);

// tm_o: o [B,T,H,dv] seen like q (used when prm.o_tma is set).
cudaError_t launch_output_tc(const CUtensorMap &tm_q, const CUtensorMap &tm_k, const CUtensorMap &tm_u,
                             const CUtensorMap &tm_g, const CUtensorMap &tm_cf, const CUtensorMap &tm_o,
                             const OutParams &prm, cudaStream_t s);

}  // namespace tc
}  // namespace gdn
