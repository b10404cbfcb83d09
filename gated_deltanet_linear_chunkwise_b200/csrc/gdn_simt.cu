// gdn_simt.cu -- CUDA-core (fp32 FMA) kernels of the chunkwise gated delta rule.
//
// This is the full-precision path: it serves gdn_fwd_f32 / gdn_step_f32
// (fp32 q/k/v/o, fp32 arithmetic, fp64 gate prefix sums) and any shape the
// tensor-core path does not take.  The four kernels follow the chunk = frame
// decomposition written out in gdn_internal.h:
//   k1  intra-frame: A = strict_lower(diag(beta) K K^T o Gamma) and the
//       blocked forward substitution (I + A)[Ub | W] = [beta V | beta e^G K]
//   k2  per-frame affine map of the state: M = e^{G_L} I - Kt^T W, N = Kt^T Ub
//   k3  scan over frames: Sig_f+1 = M_f Sig_f + N_f (state kept on chip)
//   k4  U = Ub - W Sig_f and O = diag(e^G) Q Sig_f + tril_incl(Q K^T o Gamma) U
// Row blocks are 32 tokens; every thread owns one output column and keeps
// the block's 32 (or 16) rows of that column in registers.
#include "gates.cuh"
#include "gdn_internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

constexpr int RB = 32;        // token rows per block
constexpr int NT = 256;       // threads per CTA
constexpr int SCAN_COLS = 16; // state columns per scan CTA

__host__ __device__ constexpr size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

template <typename T> __device__ __forceinline__ float ld_in(const T *p, long long i);
template <> __device__ __forceinline__ float ld_in<float>(const float *p, long long i) { return p[i]; }
template <> __device__ __forceinline__ float ld_in<__nv_bfloat16>(const __nv_bfloat16 *p, long long i) {
    return __bfloat162float(p[i]);
}
template <typename T> __device__ __forceinline__ void st_out(T *p, long long i, float x);
template <> __device__ __forceinline__ void st_out<float>(float *p, long long i, float x) { p[i] = x; }
template <> __device__ __forceinline__ void st_out<__nv_bfloat16>(__nv_bfloat16 *p, long long i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

// Shared-memory carve-up shared by the kernels that scan a frame's gates.
template <typename TG> struct GateSmem {
    static __host__ __device__ size_t bytes(int L) {
        return align16(sizeof(TG) * (size_t)L) + align16(sizeof(TG) * 32) + align16(sizeof(float) * (size_t)L);
    }
};

// ---------------------------------------------------------------- k1 intra-frame
template <typename TIn, typename TG, typename TX>
__global__ void __launch_bounds__(NT) k1_intra_simt(Problem p, TX *__restrict__ X) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int L = p.L, dk = p.dk, dv = p.dv, nc = dk + dv;
    const long long fh = blockIdx.x;
    const long long f = fh % p.F, chain = fh / p.F;
    const int h = (int)(chain % p.H), b = (int)(chain / p.H);

    unsigned char *ptr = smem;
    TG *sG = (TG *)ptr;            ptr += align16(sizeof(TG) * L);
    TG *sScr = (TG *)ptr;          ptr += align16(sizeof(TG) * 32);
    float *sB = (float *)ptr;      ptr += align16(sizeof(float) * L);
    float *sKiT = (float *)ptr;    ptr += sizeof(float) * dk * RB;   // [dk][32]
    float *sKjT = (float *)ptr;    ptr += sizeof(float) * dk * RB;   // [dk][32]
    float *sAT = (float *)ptr;     ptr += sizeof(float) * RB * RB;   // A^T [s][r]
    float *sX = (float *)ptr;                                        // [32][nc]

    frame_gates<TG>(p, b, h, f, sG, sB, sScr);
    const TIn *k = (const TIn *)p.k, *v = (const TIn *)p.v;
    TX *Xf = X + fh * (long long)L * nc;
    const int tid = threadIdx.x;
    const int nblk = (L + RB - 1) / RB;

    for (int ib = 0; ib < nblk; ++ib) {
        const int r0 = ib * RB, nr = min(RB, L - r0);
        for (int e = tid; e < RB * dk; e += NT) {
            const int r = e / dk, c = e - r * dk;
            float val = 0.f;
            if (r < nr) val = ld_in(k, tok_row(p, b, h, phys_token(p, f, r0 + r)) * dk + c);
            sKiT[c * RB + r] = val;
        }
        float acc[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) acc[r] = 0.f;
        if (tid < nc) {
#pragma unroll
            for (int r = 0; r < RB; ++r) {
                if (r < nr) {
                    const long long row = tok_row(p, b, h, phys_token(p, f, r0 + r));
                    const float be = sB[r0 + r];
                    acc[r] = (tid < dv) ? be * ld_in(v, row * dv + tid)
                                        : be * expf((float)sG[r0 + r]) * ld_in(k, row * dk + (tid - dv));
                }
            }
        }
        __syncthreads();
        for (int jb = 0; jb <= ib; ++jb) {
            const int s0 = jb * RB, ns = min(RB, L - s0);
            const bool diag = (jb == ib);
            if (!diag) {
                for (int e = tid; e < RB * dk; e += NT) {
                    const int s = e / dk, c = e - s * dk;
                    sKjT[c * RB + s] = ld_in(k, tok_row(p, b, h, phys_token(p, f, s0 + s)) * dk + c);
                }
                for (int e = tid; e < RB * nc; e += NT) sX[e] = ld_in(Xf, (long long)s0 * nc + e);
            }
            __syncthreads();
            const float *KjT = diag ? sKiT : sKjT;
            {
                const int r = tid & 31, sg = tid >> 5;
                float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
                for (int c = 0; c < dk; ++c) {
                    const float a = sKiT[c * RB + r];
                    const float4 kb = *reinterpret_cast<const float4 *>(&KjT[c * RB + sg * 4]);
                    d0 += a * kb.x; d1 += a * kb.y; d2 += a * kb.z; d3 += a * kb.w;
                }
                const float dd[4] = {d0, d1, d2, d3};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int s = sg * 4 + u;
                    float val = 0.f;
                    if (r < nr && s < ns && (!diag || s < r))
                        val = sB[r0 + r] * expf((float)(sG[r0 + r] - sG[s0 + s])) * dd[u];
                    sAT[s * RB + r] = val;
                }
            }
            __syncthreads();
            if (tid < nc) {
                if (!diag) {
                    for (int s = 0; s < RB; ++s) {
                        const float x = sX[s * nc + tid];
#pragma unroll
                        for (int r4 = 0; r4 < RB / 4; ++r4) {
                            const float4 a = *reinterpret_cast<const float4 *>(&sAT[s * RB + r4 * 4]);
                            acc[r4 * 4 + 0] -= a.x * x;
                            acc[r4 * 4 + 1] -= a.y * x;
                            acc[r4 * 4 + 2] -= a.z * x;
                            acc[r4 * 4 + 3] -= a.w * x;
                        }
                    }
                } else {
#pragma unroll
                    for (int r = 1; r < RB; ++r) {
                        float x = acc[r];
#pragma unroll
                        for (int s = 0; s < r; ++s) x -= sAT[s * RB + r] * acc[s];
                        acc[r] = x;
                    }
                }
            }
            __syncthreads();
        }
        if (tid < nc) {
#pragma unroll
            for (int r = 0; r < RB; ++r)
                if (r < nr) st_out(Xf, (long long)(r0 + r) * nc + tid, acc[r]);
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------- k2 frame transition
// grid (frame-heads, ceil(dk/32)); the block owns rows m0..m0+31 of [N | M].
template <typename TIn, typename TG, typename TX>
__global__ void __launch_bounds__(NT) k2_transition_simt(Problem p, const TX *__restrict__ X,
                                                         float *__restrict__ Mb, float *__restrict__ Nb) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int L = p.L, dk = p.dk, dv = p.dv, nc = dk + dv;
    const long long fh = blockIdx.x;
    const long long f = fh % p.F, chain = fh / p.F;
    const int h = (int)(chain % p.H), b = (int)(chain / p.H);
    const int m0 = blockIdx.y * 32, nm = min(32, dk - m0);

    unsigned char *ptr = smem;
    TG *sG = (TG *)ptr;            ptr += align16(sizeof(TG) * L);
    TG *sScr = (TG *)ptr;          ptr += align16(sizeof(TG) * 32);
    float *sB = (float *)ptr;      ptr += align16(sizeof(float) * L);
    float *sKt = (float *)ptr;     ptr += sizeof(float) * RB * 32;   // [s][m]
    float *sX = (float *)ptr;                                        // [32][nc]

    frame_gates<TG>(p, b, h, f, sG, sB, sScr);
    const TIn *k = (const TIn *)p.k;
    const TX *Xf = X + fh * (long long)L * nc;
    const int tid = threadIdx.x;
    const TG GL = sG[L - 1];

    float acc[32];
#pragma unroll
    for (int m = 0; m < 32; ++m) acc[m] = 0.f;
    for (int s0 = 0; s0 < L; s0 += RB) {
        const int ns = min(RB, L - s0);
        for (int e = tid; e < RB * 32; e += NT) {
            const int s = e >> 5, m = e & 31;
            float val = 0.f;
            if (s < ns && m < nm)
                val = expf((float)(GL - sG[s0 + s])) *
                      ld_in(k, tok_row(p, b, h, phys_token(p, f, s0 + s)) * dk + m0 + m);
            sKt[e] = val;
        }
        for (int e = tid; e < RB * nc; e += NT) {
            const int s = e / nc;
            sX[e] = (s < ns) ? ld_in(Xf, (long long)s0 * nc + e) : 0.f;
        }
        __syncthreads();
        if (tid < nc) {
            for (int s = 0; s < RB; ++s) {
                const float x = sX[s * nc + tid];
#pragma unroll
                for (int m4 = 0; m4 < 8; ++m4) {
                    const float4 kk = *reinterpret_cast<const float4 *>(&sKt[s * 32 + m4 * 4]);
                    acc[m4 * 4 + 0] += kk.x * x;
                    acc[m4 * 4 + 1] += kk.y * x;
                    acc[m4 * 4 + 2] += kk.z * x;
                    acc[m4 * 4 + 3] += kk.w * x;
                }
            }
        }
        __syncthreads();
    }
    if (tid < nc) {
        const float eGL = expf((float)GL);
#pragma unroll
        for (int m = 0; m < 32; ++m) {
            if (m < nm) {
                const int row = m0 + m;
                if (tid < dv) {
                    Nb[(fh * dk + row) * (long long)dv + tid] = acc[m];
                } else {
                    const int j = tid - dv;
                    Mb[(fh * dk + row) * (long long)dk + j] = (row == j ? eGL : 0.f) - acc[m];
                }
            }
        }
    }
}

// ---------------------------------------------------------------- k3 scan over frames
// grid (B*H, ceil(dv/16)); the block carries 16 columns of Sig = S^T through
// all frames of its chain (Sig_next = M Sig + N), writing the state entering
// each frame (token-wise operator) or the state after each frame's update
// (frame-wise operator, whose tokens read the post-update state) to SigIn
// (fp32) and/or SigB (bf16).  The next frame's M is
// brought in by cp.async into the other half of a double buffer while the
// current step computes.
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Thread layout: 256 threads = 2 halves of the contraction index l x 8
// column pairs x 16 row groups; each thread accumulates rows m = g + 16i of
// two columns over its half of l (2 DK/16 independent sums), and the halves
// are added through shared memory.  N for the next frame is loaded one step
// ahead.  DK is a template parameter so every loop has a fixed trip count.
template <int DK>
__global__ void __launch_bounds__(NT) k3_scan_simt(Problem p, const float *__restrict__ Mb,
                                                   const float *__restrict__ Nb, float *__restrict__ SigIn,
                                                   __nv_bfloat16 *__restrict__ SigB) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int R = DK / 16;                       // rows per thread
    constexpr int HALF = DK / 2;                     // contraction length per thread half
    const int dv = p.dv;
    const long long chain = blockIdx.x;
    // segment-map mode: the state is [Sig | P] (d_v + d_k columns) starting from [0 | I]; N is
    // added to the Sig columns only (d_v is a multiple of 16, so a group lies in one part)
    const bool map = p.map_out != nullptr;
    const int ncols_all = map ? dv + DK : dv;
    const int c0 = blockIdx.y * SCAN_COLS, ncol = min(SCAN_COLS, ncols_all - c0);
    const bool add_n = c0 < dv;
    float *sM = (float *)smem;                       // 2 x [DK][DK]
    float *sS = sM + 2 * DK * DK;                    // [DK][16]
    float2 *sRed = reinterpret_cast<float2 *>(sS + DK * SCAN_COLS);  // [R][128] partial sums of the upper half
    const int tid = threadIdx.x;
    const int kh = tid >> 7, t7 = tid & 127, cp = t7 & 7, g = t7 >> 3;
    const int ca = 2 * cp, cb = 2 * cp + 1;          // this thread's two columns
    const int l0 = kh * HALF;

    for (int e = tid; e < DK * SCAN_COLS; e += NT) {
        const int m = e >> 4, cc = e & 15;
        float val = 0.f;
        if (map) val = (cc < ncol && c0 + cc >= dv && m == c0 + cc - dv) ? 1.f : 0.f;
        else if (p.S_in && cc < ncol) val = p.S_in[(chain * dv + c0 + cc) * (long long)DK + m];
        sS[e] = val;
    }
    constexpr int NVEC = DK * DK / 4;  // 16-byte pieces of one M
    const bool post = p.mode == GDN_MODE_FRAME;
    if (p.F > 0) {
        const float4 *src = reinterpret_cast<const float4 *>(Mb + (chain * p.F + scan_frame(p, 0)) * (long long)DK * DK);
        for (int e = tid; e < NVEC; e += NT) cp_async16(sM + 4 * e, src + e);
    }
    cp_async_commit();
    // N of the first frame (the lower l half adds N; the upper half does not)
    float2 nxt[R];
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int m = g + 16 * i;
        nxt[i] = make_float2(0.f, 0.f);
        if (kh == 0 && p.F > 0 && add_n) {
            const long long idx = ((chain * p.F + scan_frame(p, 0)) * DK + m) * (long long)dv + c0;
            nxt[i].x = ca < ncol ? Nb[idx + ca] : 0.f;
            nxt[i].y = cb < ncol ? Nb[idx + cb] : 0.f;
        }
    }
    __syncthreads();
    for (long long f = 0; f < p.F; ++f) {
        const long long fh = chain * p.F + scan_frame(p, f);
        const long long fhn = f + 1 < p.F ? chain * p.F + scan_frame(p, f + 1) : fh;
        const int buf = (int)(f & 1);
        if (f + 1 < p.F) {  // prefetch the next frame's M into the other buffer
            const float4 *src = reinterpret_cast<const float4 *>(Mb + fhn * (long long)DK * DK);
            float *dst = sM + (buf ^ 1) * DK * DK;
            for (int e = tid; e < NVEC; e += NT) cp_async16(dst + 4 * e, src + e);
        }
        cp_async_commit();
        if (frame_resets(p, f)) {
            for (int e = tid; e < DK * SCAN_COLS; e += NT) sS[e] = 0.f;
            __syncthreads();
        }
        float2 acc[R];
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int m = g + 16 * i;
            acc[i] = nxt[i];
            nxt[i] = make_float2(0.f, 0.f);
            if (kh == 0) {
                const long long idx = (fh * DK + m) * (long long)dv + c0;
                const float2 cur = *reinterpret_cast<const float2 *>(&sS[m * SCAN_COLS + ca]);
                if (!post && SigIn) *reinterpret_cast<float2 *>(SigIn + idx + ca) = cur;
                if (!post && SigB) *reinterpret_cast<__nv_bfloat162 *>(SigB + idx + ca) = __floats2bfloat162_rn(cur.x, cur.y);
                if (f + 1 < p.F && add_n)
                    nxt[i] = *reinterpret_cast<const float2 *>(Nb + (fhn * DK + m) * (long long)dv + c0 + ca);
            }
        }
        cp_async_wait_one();  // this frame's M (committed one step earlier) has landed
        __syncthreads();
        const float *Mf = sM + buf * DK * DK + l0;
        const float *Sf = sS + l0 * SCAN_COLS + ca;
#pragma unroll 2
        for (int l = 0; l < HALF; l += 4) {
            const float2 s0 = *reinterpret_cast<const float2 *>(&Sf[(l + 0) * SCAN_COLS]);
            const float2 s1 = *reinterpret_cast<const float2 *>(&Sf[(l + 1) * SCAN_COLS]);
            const float2 s2 = *reinterpret_cast<const float2 *>(&Sf[(l + 2) * SCAN_COLS]);
            const float2 s3 = *reinterpret_cast<const float2 *>(&Sf[(l + 3) * SCAN_COLS]);
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const float4 mm = *reinterpret_cast<const float4 *>(&Mf[(g + 16 * i) * DK + l]);
                acc[i].x = fmaf(mm.x, s0.x, acc[i].x);
                acc[i].y = fmaf(mm.x, s0.y, acc[i].y);
                acc[i].x = fmaf(mm.y, s1.x, acc[i].x);
                acc[i].y = fmaf(mm.y, s1.y, acc[i].y);
                acc[i].x = fmaf(mm.z, s2.x, acc[i].x);
                acc[i].y = fmaf(mm.z, s2.y, acc[i].y);
                acc[i].x = fmaf(mm.w, s3.x, acc[i].x);
                acc[i].y = fmaf(mm.w, s3.y, acc[i].y);
            }
        }
        if (kh == 1) {
#pragma unroll
            for (int i = 0; i < R; ++i) sRed[i * 128 + t7] = acc[i];
        }
        __syncthreads();  // every read of sS and of this M buffer is done; partial sums are in sRed
        if (kh == 0) {
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const int m = g + 16 * i;
                const float2 o = sRed[i * 128 + t7];
                const float2 nw = make_float2(acc[i].x + o.x, acc[i].y + o.y);
                *reinterpret_cast<float2 *>(&sS[m * SCAN_COLS + ca]) = nw;
                if (post) {  // the state after this frame's update
                    const long long idx = (fh * DK + m) * (long long)dv + c0;
                    if (SigIn) *reinterpret_cast<float2 *>(SigIn + idx + ca) = nw;
                    if (SigB) *reinterpret_cast<__nv_bfloat162 *>(SigB + idx + ca) = __floats2bfloat162_rn(nw.x, nw.y);
                }
            }
        }
        __syncthreads();
    }
    if (map) {  // Phi[l][m] = P[m][l] (rows 0 .. d_k - 1), Psi[c][m] = Sig[m][c] (rows d_k ..)
        for (int e = tid; e < DK * SCAN_COLS; e += NT) {
            const int m = e >> 4, cc = e & 15;
            if (cc >= ncol) continue;
            const int col = c0 + cc, row = col >= dv ? col - dv : DK + col;
            p.map_out[(chain * (DK + dv) + row) * (long long)DK + m] = sS[e];
        }
    } else if (p.S_out) {
        for (int e = tid; e < DK * SCAN_COLS; e += NT) {
            const int m = e >> 4, cc = e & 15;
            if (cc < ncol) p.S_out[(chain * dv + c0 + cc) * (long long)DK + m] = sS[e];
        }
    }
    cp_async_wait_all();  // leave with no copy in flight
}

template <int DK>
cudaError_t launch_scan_dk(const Problem &p, const float *Mb, const float *Nb, float *Sig, __nv_bfloat16 *SigB,
                           cudaStream_t s) {
    const size_t sm = sizeof(float) * (2 * DK * DK + DK * SCAN_COLS) + sizeof(float2) * (DK / 16) * 128;
    cudaError_t e = cudaFuncSetAttribute(k3_scan_simt<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e) return e;
    const int ncols_all = p.map_out ? p.dv + DK : p.dv;
    k3_scan_simt<DK><<<dim3((unsigned)(p.B * p.H), (ncols_all + SCAN_COLS - 1) / SCAN_COLS), NT, sm, s>>>(p, Mb, Nb,
                                                                                                          Sig, SigB);
    return cudaGetLastError();
}

cudaError_t launch_scan(const Problem &p, const float *Mb, const float *Nb, float *Sig, __nv_bfloat16 *SigB,
                        cudaStream_t s) {
    switch (p.dk) {
        case 16: return launch_scan_dk<16>(p, Mb, Nb, Sig, SigB, s);
        case 32: return launch_scan_dk<32>(p, Mb, Nb, Sig, SigB, s);
        case 48: return launch_scan_dk<48>(p, Mb, Nb, Sig, SigB, s);
        case 64: return launch_scan_dk<64>(p, Mb, Nb, Sig, SigB, s);
        case 80: return launch_scan_dk<80>(p, Mb, Nb, Sig, SigB, s);
        case 96: return launch_scan_dk<96>(p, Mb, Nb, Sig, SigB, s);
        case 112: return launch_scan_dk<112>(p, Mb, Nb, Sig, SigB, s);
        case 128: return launch_scan_dk<128>(p, Mb, Nb, Sig, SigB, s);
        default: return cudaErrorInvalidValue;
    }
}

// ---------------------------------------------------------------- k4 output
// grid (frame-heads); for each 32-row block I in order: U_I = Ub_I - W_I Sig
// (kept in the U workspace for later blocks), then
// O_I = diag(e^G) Q_I Sig + sum_{J <= I} mask(Q_I K_J^T o Gamma) U_J.
template <typename TIn, typename TG>
__global__ void __launch_bounds__(NT) k4_output_simt(Problem p, const float *__restrict__ X,
                                                     const float *__restrict__ SigIn, float *__restrict__ U) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int L = p.L, dk = p.dk, dv = p.dv, nc = dk + dv;
    const long long fh = blockIdx.x;
    const long long f = fh % p.F, chain = fh / p.F;
    const int h = (int)(chain % p.H), b = (int)(chain / p.H);

    unsigned char *ptr = smem;
    TG *sG = (TG *)ptr;            ptr += align16(sizeof(TG) * L);
    TG *sScr = (TG *)ptr;          ptr += align16(sizeof(TG) * 32);
    float *sB = (float *)ptr;      ptr += align16(sizeof(float) * L);
    float *sSig = (float *)ptr;    ptr += sizeof(float) * dk * dv;   // [dk][dv]
    float *sQT = (float *)ptr;     ptr += sizeof(float) * dk * RB;   // [dk][32]
    float *sWT = (float *)ptr;     ptr += sizeof(float) * dk * RB;   // [dk][32]
    float *sKT = (float *)ptr;     ptr += sizeof(float) * dk * RB;   // [dk][32]
    float *sPT = (float *)ptr;     ptr += sizeof(float) * RB * RB;   // [s][r]
    float *sU = (float *)ptr;                                        // [32][dv]

    frame_gates<TG>(p, b, h, f, sG, sB, sScr);
    const TIn *q = (const TIn *)p.q, *k = (const TIn *)p.k;
    TIn *o = (TIn *)p.o;
    const float *Xf = X + fh * (long long)L * nc;
    float *Uf = U + fh * (long long)L * dv;
    const float *Sf = SigIn + fh * (long long)dk * dv;
    const int tid = threadIdx.x;
    for (int e = tid; e < dk * dv; e += NT) sSig[e] = Sf[e];

    const int c = tid & 127, rh = tid >> 7;  // column, half of the row block
    const bool active = c < dv;
    const int nblk = (L + RB - 1) / RB;
    for (int ib = 0; ib < nblk; ++ib) {
        const int r0 = ib * RB, nr = min(RB, L - r0);
        for (int e = tid; e < RB * dk; e += NT) {
            const int r = e / dk, cc = e - r * dk;
            float qv = 0.f, wv = 0.f;
            if (r < nr) {
                qv = ld_in(q, tok_row(p, b, h, phys_token(p, f, r0 + r)) * dk + cc);
                wv = Xf[(long long)(r0 + r) * nc + dv + cc];
            }
            sQT[cc * RB + r] = qv;
            sWT[cc * RB + r] = wv;
        }
        __syncthreads();
        float acc[16];
        if (active) {
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const int rr = rh * 16 + r;
                acc[r] = (rr < nr) ? Xf[(long long)(r0 + rr) * nc + c] : 0.f;
            }
            for (int l = 0; l < dk; ++l) {
                const float sg = sSig[l * dv + c];
#pragma unroll
                for (int r4 = 0; r4 < 4; ++r4) {
                    const float4 w = *reinterpret_cast<const float4 *>(&sWT[l * RB + rh * 16 + r4 * 4]);
                    acc[r4 * 4 + 0] -= w.x * sg;
                    acc[r4 * 4 + 1] -= w.y * sg;
                    acc[r4 * 4 + 2] -= w.z * sg;
                    acc[r4 * 4 + 3] -= w.w * sg;
                }
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const int rr = rh * 16 + r;
                if (rr < nr) Uf[(long long)(r0 + rr) * dv + c] = acc[r];
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) acc[r] = 0.f;
            for (int l = 0; l < dk; ++l) {
                const float sg = sSig[l * dv + c];
#pragma unroll
                for (int r4 = 0; r4 < 4; ++r4) {
                    const float4 qq = *reinterpret_cast<const float4 *>(&sQT[l * RB + rh * 16 + r4 * 4]);
                    acc[r4 * 4 + 0] += qq.x * sg;
                    acc[r4 * 4 + 1] += qq.y * sg;
                    acc[r4 * 4 + 2] += qq.z * sg;
                    acc[r4 * 4 + 3] += qq.w * sg;
                }
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const int rr = rh * 16 + r;
                acc[r] *= (rr < nr) ? expf((float)sG[r0 + rr]) : 0.f;
            }
        }
        __syncthreads();  // this block's U rows are visible to the whole CTA
        for (int jb = 0; jb <= ib; ++jb) {
            const int s0 = jb * RB, ns = min(RB, L - s0);
            const bool diag = (jb == ib);
            for (int e = tid; e < RB * dk; e += NT) {
                const int s = e / dk, cc = e - s * dk;
                sKT[cc * RB + s] = (s < ns) ? ld_in(k, tok_row(p, b, h, phys_token(p, f, s0 + s)) * dk + cc) : 0.f;
            }
            for (int e = tid; e < RB * dv; e += NT) {
                const int s = e / dv;
                sU[e] = (s < ns) ? Uf[(long long)s0 * dv + e] : 0.f;
            }
            __syncthreads();
            {
                const int r = tid & 31, sg = tid >> 5;
                float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
                for (int cc = 0; cc < dk; ++cc) {
                    const float a = sQT[cc * RB + r];
                    const float4 kb = *reinterpret_cast<const float4 *>(&sKT[cc * RB + sg * 4]);
                    d0 += a * kb.x; d1 += a * kb.y; d2 += a * kb.z; d3 += a * kb.w;
                }
                const float dd[4] = {d0, d1, d2, d3};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int s = sg * 4 + u;
                    float val = 0.f;
                    if (r < nr && s < ns && (!diag || s <= r))
                        val = expf((float)(sG[r0 + r] - sG[s0 + s])) * dd[u];
                    sPT[s * RB + r] = val;
                }
            }
            __syncthreads();
            if (active) {
                for (int s = 0; s < RB; ++s) {
                    const float u = sU[s * dv + c];
#pragma unroll
                    for (int r4 = 0; r4 < 4; ++r4) {
                        const float4 pp = *reinterpret_cast<const float4 *>(&sPT[s * RB + rh * 16 + r4 * 4]);
                        acc[r4 * 4 + 0] += pp.x * u;
                        acc[r4 * 4 + 1] += pp.y * u;
                        acc[r4 * 4 + 2] += pp.z * u;
                        acc[r4 * 4 + 3] += pp.w * u;
                    }
                }
            }
            __syncthreads();
        }
        if (active) {
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const int rr = rh * 16 + r;
                if (rr < nr) {
                    const long long idx = tok_row(p, b, h, phys_token(p, f, r0 + rr)) * dv + c;
                    float val = acc[r];
                    if (p.accumulate) val += ld_in(o, idx);
                    st_out(o, idx, val);
                }
            }
        }
    }
}


// ---------------------------------------------------------------- U = Ub - W Sig
// grid (frame-heads, ceil(L/128)); 128 rows per block in four 32-row passes.
// Reads [Ub | W] (TX) and the entering state Sig (fp32), writes U in bf16.
template <typename TX>
__global__ void __launch_bounds__(NT) ku_simt(Problem p, const TX *__restrict__ X, const float *__restrict__ SigIn,
                                              __nv_bfloat16 *__restrict__ U) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int L = p.L, dk = p.dk, dv = p.dv, nc = dk + dv;
    const long long fh = blockIdx.x;
    float *sSig = (float *)smem;          // [dk][dv]
    float *sWT = sSig + dk * dv;          // [dk][32]
    const TX *Xf = X + fh * (long long)L * nc;
    const float *Sf = SigIn + fh * (long long)dk * dv;
    __nv_bfloat16 *Uf = U + fh * (long long)L * dv;
    const int tid = threadIdx.x;
    for (int e = tid; e < dk * dv; e += NT) sSig[e] = Sf[e];
    const int c = tid & 127, rh = tid >> 7;
    const bool active = c < dv;
    for (int pass = 0; pass < 4; ++pass) {
        const int r0 = blockIdx.y * 128 + pass * RB;
        if (r0 >= L) break;
        const int nr = min(RB, L - r0);
        __syncthreads();
        for (int e = tid; e < RB * dk; e += NT) {
            const int r = e / dk, cc = e - r * dk;
            sWT[cc * RB + r] = (r < nr) ? ld_in(Xf, (long long)(r0 + r) * nc + dv + cc) : 0.f;
        }
        __syncthreads();
        if (active) {
            float acc[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const int rr = rh * 16 + r;
                acc[r] = (rr < nr) ? ld_in(Xf, (long long)(r0 + rr) * nc + c) : 0.f;
            }
            for (int l = 0; l < dk; ++l) {
                const float sg = sSig[l * dv + c];
#pragma unroll
                for (int r4 = 0; r4 < 4; ++r4) {
                    const float4 w = *reinterpret_cast<const float4 *>(&sWT[l * RB + rh * 16 + r4 * 4]);
                    acc[r4 * 4 + 0] -= w.x * sg;
                    acc[r4 * 4 + 1] -= w.y * sg;
                    acc[r4 * 4 + 2] -= w.z * sg;
                    acc[r4 * 4 + 3] -= w.w * sg;
                }
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const int rr = rh * 16 + r;
                if (rr < nr) Uf[(long long)(r0 + rr) * dv + c] = __float2bfloat16_rn(acc[r]);
            }
        }
    }
}

template <typename TIn, typename TG>
cudaError_t launch_typed(const Problem &p, void *ws, cudaStream_t s, cudaEvent_t *ev) {
    const SimtLayout lay = simt_layout(p);
    char *base = (char *)ws;
    float *X = (float *)(base + lay.X), *U = (float *)(base + lay.U);
    float *Mb = (float *)(base + lay.M), *Nb = (float *)(base + lay.N), *Sig = (float *)(base + lay.Sig);
    const long long nfh = (long long)p.B * p.H * p.F;
    const int dk = p.dk, dv = p.dv, nc = dk + dv;
    const size_t gsm = GateSmem<TG>::bytes(p.L);

    const size_t sm1 = gsm + sizeof(float) * (2 * dk * RB + RB * RB + RB * nc);
    const size_t sm2 = gsm + sizeof(float) * (RB * 32 + RB * nc);
    const size_t sm4 = gsm + sizeof(float) * (dk * dv + 3 * dk * RB + RB * RB + RB * dv);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k1_intra_simt<TIn, TG, float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1))) return e;
    if ((e = cudaFuncSetAttribute(k2_transition_simt<TIn, TG, float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2))) return e;
    if ((e = cudaFuncSetAttribute(k4_output_simt<TIn, TG>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm4))) return e;

    // stages 0, 1 (gates, diagonal inverses) are folded into the intra kernel, 5 (U) into the output
    for (int i = 0; i <= 2; ++i)
        if ((e = mark(ev, i, s))) return e;
    if (p.phase != GDN_PHASE_FINISH) {  // the state-independent stages
        k1_intra_simt<TIn, TG, float><<<(unsigned)nfh, NT, sm1, s>>>(p, X);
        if ((e = cudaGetLastError())) return e;
        if ((e = mark(ev, 3, s))) return e;
        k2_transition_simt<TIn, TG, float><<<dim3((unsigned)nfh, (dk + 31) / 32), NT, sm2, s>>>(p, X, Mb, Nb);
        if ((e = cudaGetLastError())) return e;
        if (p.map_out && (e = simt_segment_map(p, Mb, Nb, s))) return e;
        if (p.phase == GDN_PHASE_PREPARE) {
            for (int i = 4; i <= GDN_NUM_STAGES; ++i)
                if ((e = mark(ev, i, s))) return e;
            return cudaSuccess;
        }
    } else if ((e = mark(ev, 3, s))) {
        return e;
    }
    if ((e = mark(ev, 4, s))) return e;
    if ((e = launch_scan(p, Mb, Nb, Sig, nullptr, s))) return e;
    if ((e = cudaGetLastError())) return e;
    if ((e = mark(ev, 5, s)) || (e = mark(ev, 6, s))) return e;
    k4_output_simt<TIn, TG><<<(unsigned)nfh, NT, sm4, s>>>(p, X, Sig, U);
    if ((e = cudaGetLastError())) return e;
    return mark(ev, 7, s);
}

}  // namespace

SimtLayout simt_layout(const Problem &p) {
    const size_t nfh = (size_t)p.B * p.H * p.F;
    SimtLayout lay;
    size_t off = 0;
    lay.X = off;   off += align256(sizeof(float) * nfh * p.L * (p.dk + p.dv));
    lay.U = off;   off += align256(sizeof(float) * nfh * p.L * p.dv);
    lay.M = off;   off += align256(sizeof(float) * nfh * p.dk * p.dk);
    lay.N = off;   off += align256(sizeof(float) * nfh * p.dk * p.dv);
    lay.Sig = off; off += align256(sizeof(float) * nfh * p.dk * p.dv);
    lay.total = off;
    return lay;
}

size_t simt_workspace_bytes(const Problem &p) { return simt_layout(p).total; }

cudaError_t launch_simt(const Problem &p, void *ws, cudaStream_t s, cudaEvent_t *ev) {
    if (p.mode == GDN_MODE_FRAME) return launch_simt_frame(p, ws, s, ev);
    if (p.dtype == GDN_DTYPE_F32) return launch_typed<float, double>(p, ws, s, ev);
    return launch_typed<__nv_bfloat16, float>(p, ws, s, ev);
}

cudaError_t simt_intra_bf16x(const Problem &p, __nv_bfloat16 *X, cudaStream_t s) {
    const int dk = p.dk, nc = p.dk + p.dv;
    const size_t sm = GateSmem<float>::bytes(p.L) + sizeof(float) * (2 * dk * RB + RB * RB + RB * nc);
    auto k = k1_intra_simt<__nv_bfloat16, float, __nv_bfloat16>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e) return e;
    k<<<(unsigned)((long long)p.B * p.H * p.F), NT, sm, s>>>(p, X);
    return cudaGetLastError();
}

cudaError_t simt_transition_bf16x(const Problem &p, const __nv_bfloat16 *X, float *Mb, float *Nb, cudaStream_t s) {
    const int nc = p.dk + p.dv;
    const size_t sm = GateSmem<float>::bytes(p.L) + sizeof(float) * (RB * 32 + RB * nc);
    auto k = k2_transition_simt<__nv_bfloat16, float, __nv_bfloat16>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e) return e;
    k<<<dim3((unsigned)((long long)p.B * p.H * p.F), (p.dk + 31) / 32), NT, sm, s>>>(p, X, Mb, Nb);
    return cudaGetLastError();
}

cudaError_t simt_scan(const Problem &p, const float *Mb, const float *Nb, float *Sig, __nv_bfloat16 *SigB,
                      cudaStream_t s) {
    return launch_scan(p, Mb, Nb, Sig, SigB, s);
}

cudaError_t simt_segment_map(const Problem &p, const float *Mb, const float *Nb, cudaStream_t s) {
    Problem q = p;
    q.S_in = nullptr;
    q.S_out = nullptr;
    return launch_scan(q, Mb, Nb, nullptr, nullptr, s);
}

namespace {

// S <- S Phi + Psi per (b, h) chain, for each map in turn: S [d_v][d_k] and Phi [d_k][d_k] in
// shared memory, each thread owning output columns m of a few rows c.
__global__ void __launch_bounds__(NT) apply_maps_kernel(float *S, const float *maps, int n, int dk, int dv) {
    extern __shared__ __align__(16) float sm[];
    float *sS = sm, *sP = sm + dv * dk, *sNew = sP + dk * dk;
    const long long chain = blockIdx.x;
    float *Sc = S + chain * (long long)dv * dk;
    for (int e = threadIdx.x; e < dv * dk; e += NT) sS[e] = Sc[e];
    for (int j = 0; j < n; ++j) {
        const float *mp = maps + ((long long)j * gridDim.x + chain) * (long long)(dk + dv) * dk;
        __syncthreads();
        for (int e = threadIdx.x; e < dk * dk; e += NT) sP[e] = mp[e];
        __syncthreads();
        for (int e = threadIdx.x; e < dv * dk; e += NT) {
            const int c = e / dk, m = e - c * dk;
            float acc = mp[(long long)(dk + c) * dk + m];  // Psi[c][m]
            for (int l = 0; l < dk; ++l) acc = fmaf(sS[c * dk + l], sP[l * dk + m], acc);
            sNew[e] = acc;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < dv * dk; e += NT) sS[e] = sNew[e];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < dv * dk; e += NT) Sc[e] = sS[e];
}

}  // namespace

namespace {
__global__ void identity_map_kernel(float *map, long long n, int dk, int rows) {
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(e % dk), r = (int)((e / dk) % rows);
        map[e] = (r == m) ? 1.f : 0.f;  // rows r < dk: Phi = I; rows dk ..: Psi = 0
    }
}
}  // namespace

cudaError_t launch_identity_map(float *map, int B, int H, int dk, int dv, cudaStream_t s) {
    const long long n = (long long)B * H * (dk + dv) * dk;
    if (n == 0) return cudaSuccess;
    identity_map_kernel<<<148, 256, 0, s>>>(map, n, dk, dk + dv);
    return cudaGetLastError();
}

cudaError_t launch_apply_maps(float *S, const float *maps, int n, int B, int H, int dk, int dv, cudaStream_t s) {
    const size_t sm = sizeof(float) * (2 * (size_t)dv * dk + (size_t)dk * dk);
    cudaError_t e = cudaFuncSetAttribute(apply_maps_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e) return e;
    if ((long long)B * H == 0 || n == 0) return cudaSuccess;
    apply_maps_kernel<<<(unsigned)((long long)B * H), NT, sm, s>>>(S, maps, n, dk, dv);
    return cudaGetLastError();
}

cudaError_t simt_u_bf16x(const Problem &p, const __nv_bfloat16 *X, const float *Sig, __nv_bfloat16 *U,
                         cudaStream_t s) {
    const size_t sm = sizeof(float) * (p.dk * p.dv + p.dk * RB);
    auto k = ku_simt<__nv_bfloat16>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e) return e;
    k<<<dim3((unsigned)((long long)p.B * p.H * p.F), (p.L + 127) / 128), NT, sm, s>>>(p, X, Sig, U);
    return cudaGetLastError();
}

}  // namespace gdn
