// frame_simt.cu -- the frame-wise operator on the CUDA cores (the fp32 path,
// and bf16 when the tensor-core path is switched off).
//
// SANA-WM summary, "Memory-Efficient Long-Context Modeling (Section 3.2)",
// paragraph "Adaptation to video: frame-wise recurrence": per frame t of L
// tokens (keys and values as the columns of K_t, V_t, B_t = diag(beta)),
//   S_t = S_{t-1} M_t + U_t,  M_t = gamma_t (I - K_t B_t K_t^T),
//   U_t = V_t B_t K_t^T,      o = S_t q for every token of frame t.
// With Sig = S^T (d_k x d_v) this is the scan's affine map
//   Sig_t = M_t Sig_{t-1} + N_t,  N_t = U_t^T = sum_r beta_r k_r v_r^T
// (M_t is symmetric), so the pass is: the per-frame maps (this file), the
// scan over frames shared with the token-wise path (which emits the state
// after each frame's update in this mode), and o_r = Sig_t^T q_r (this file).
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int NTF = 256;   // threads per block
constexpr int RCH = 32;    // tokens per staged chunk

template <typename T> __device__ __forceinline__ float ldf(const T *p, long long i);
template <> __device__ __forceinline__ float ldf<float>(const float *p, long long i) { return p[i]; }
template <> __device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16 *p, long long i) {
    return __bfloat162float(p[i]);
}
template <typename T> __device__ __forceinline__ void stf(T *p, long long i, float x);
template <> __device__ __forceinline__ void stf<float>(float *p, long long i, float x) { p[i] = x; }
template <> __device__ __forceinline__ void stf<__nv_bfloat16>(__nv_bfloat16 *p, long long i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

// grid (n_fh, ceil(d_k / 32)): rows m0 .. m0+31 of P = sum_r beta_r k_r [k_r | v_r]^T over the
// frame's tokens; thread n owns column n of [k | v] (n < d_k + d_v) and 32 row sums.
// M = gamma (I - P[:, :d_k]), N = P[:, d_k:].  The frame's sum does not depend on token order.
template <typename TIn, typename TA>
__global__ void __launch_bounds__(NTF) k_frame_maps_simt(Problem p, float *__restrict__ Mb,
                                                         float *__restrict__ Nb) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int dk = p.dk, dv = p.dv, nc = dk + dv, L = p.L;
    const long long fh = blockIdx.x;
    const long long f = fh % p.F, chain = fh / p.F;
    const int h = (int)(chain % p.H), b = (int)(chain / p.H);
    const int m0 = blockIdx.y * 32;
    float *sKb = (float *)smem;           // [RCH][32]: beta_r k_r[m0 + i]
    float *sX = sKb + RCH * 32;           // [RCH][nc]: [k_r | v_r]
    const TIn *k = (const TIn *)p.k, *v = (const TIn *)p.v;
    const int n = threadIdx.x;
    TA acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = (TA)0;
    for (int r0 = 0; r0 < L; r0 += RCH) {
        const int nr = min(RCH, L - r0);
        __syncthreads();  // the previous chunk has been read
        for (int e = threadIdx.x; e < RCH * nc; e += NTF) {
            const int r = e / nc, c = e % nc;
            float x = 0.f;
            if (r < nr) {
                const long long row = tok_row(p, b, h, f * L + r0 + r);
                x = c < dk ? ldf(k, row * dk + c) : ldf(v, row * dv + (c - dk));
            }
            sX[e] = x;
        }
        for (int e = threadIdx.x; e < RCH * 32; e += NTF) {
            const int r = e >> 5, i = e & 31;
            float x = 0.f;
            if (r < nr && m0 + i < dk) {
                const long long row = tok_row(p, b, h, f * L + r0 + r);
                x = p.beta[row] * ldf(k, row * dk + m0 + i);
            }
            sKb[e] = x;
        }
        __syncthreads();
        if (n < nc) {
            for (int r = 0; r < nr; ++r) {
                const TA x = (TA)sX[r * nc + n];
#pragma unroll
                for (int i = 0; i < 32; ++i) acc[i] += (TA)sKb[r * 32 + i] * x;
            }
        }
    }
    if (n >= nc) return;
    const float g = p.gamma[((long long)b * p.F + f) * p.H + h];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int m = m0 + i;
        if (m >= dk) break;
        if (n < dk) Mb[(fh * dk + m) * (long long)dk + n] = (float)((TA)g * ((m == n ? (TA)1 : (TA)0) - acc[i]));
        else Nb[(fh * dk + m) * (long long)dv + (n - dk)] = (float)acc[i];
    }
}

// grid (n_fh, ceil(L / 32)): o_r = Sig_t^T q_r for 32 tokens of the frame, Sig_t the state
// after the frame's update; thread (c, lane group) owns column c and every second token.
template <typename TIn>
__global__ void __launch_bounds__(NTF) k_frame_out_simt(Problem p, const float *__restrict__ Sig) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int dk = p.dk, dv = p.dv, L = p.L;
    const long long fh = blockIdx.x;
    const long long f = fh % p.F, chain = fh / p.F;
    const int h = (int)(chain % p.H), b = (int)(chain / p.H);
    const int r0 = blockIdx.y * RCH, nr = min(RCH, L - r0);
    float *sS = (float *)smem;     // [dk][dv]
    float *sQ = sS + dk * dv;      // [RCH][dk]
    const TIn *q = (const TIn *)p.q;
    TIn *o = (TIn *)p.o;
    for (int e = threadIdx.x; e < dk * dv; e += NTF) sS[e] = Sig[fh * (long long)dk * dv + e];
    for (int e = threadIdx.x; e < RCH * dk; e += NTF) {
        const int r = e / dk, m = e % dk;
        sQ[e] = r < nr ? ldf(q, tok_row(p, b, h, f * L + r0 + r) * dk + m) : 0.f;
    }
    __syncthreads();
    const int c = threadIdx.x & 127, rg = threadIdx.x >> 7;
    if (c >= dv) return;
    for (int r = rg; r < nr; r += 2) {
        float acc = 0.f;
        for (int m = 0; m < dk; ++m) acc = fmaf(sQ[r * dk + m], sS[m * dv + c], acc);
        const long long idx = tok_row(p, b, h, f * L + r0 + r) * dv + c;
        if (p.accumulate) acc += ldf(o, idx);
        stf(o, idx, acc);
    }
}

template <typename TIn, typename TA>
cudaError_t launch_frame_typed(const Problem &p, void *ws, cudaStream_t s, cudaEvent_t *ev) {
    const SimtLayout lay = simt_layout(p);
    char *base = (char *)ws;
    float *Mb = (float *)(base + lay.M), *Nb = (float *)(base + lay.N), *Sig = (float *)(base + lay.Sig);
    const long long nfh = (long long)p.B * p.H * p.F;
    const size_t sm1 = sizeof(float) * RCH * (32 + p.dk + p.dv);
    const size_t sm3 = sizeof(float) * (p.dk * p.dv + RCH * p.dk);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k_frame_maps_simt<TIn, TA>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1)))
        return e;
    if ((e = cudaFuncSetAttribute(k_frame_out_simt<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm3)))
        return e;
    // stages 0-2 (gates, inverses, intra solve) and 5 (U) do not exist in this operator
    for (int i = 0; i <= 3; ++i)
        if ((e = mark(ev, i, s))) return e;
    k_frame_maps_simt<TIn, TA><<<dim3((unsigned)nfh, (p.dk + 31) / 32), NTF, sm1, s>>>(p, Mb, Nb);
    if ((e = cudaGetLastError())) return e;
    if ((e = mark(ev, 4, s))) return e;
    if ((e = simt_scan(p, Mb, Nb, Sig, nullptr, s))) return e;
    if ((e = mark(ev, 5, s)) || (e = mark(ev, 6, s))) return e;
    k_frame_out_simt<TIn><<<dim3((unsigned)nfh, (p.L + RCH - 1) / RCH), NTF, sm3, s>>>(p, Sig);
    if ((e = cudaGetLastError())) return e;
    return mark(ev, 7, s);
}

}  // namespace

cudaError_t launch_simt_frame(const Problem &p, void *ws, cudaStream_t s, cudaEvent_t *ev) {
    if (p.dtype == GDN_DTYPE_F32) return launch_frame_typed<float, double>(p, ws, s, ev);
    return launch_frame_typed<__nv_bfloat16, float>(p, ws, s, ev);
}

}  // namespace gdn
