// qk_prologue.cu -- the q/k feature maps applied before the operator.
//
// SANA-WM summary, "Memory-Efficient Long-Context Modeling (Section 3.2)",
// paragraph "Algebraic Stabilization for Spatial Token Explosion": keys pass
// through k_bar = ReLU(RMSNorm(k)) and are scaled by 1/sqrt(D * S) (D the
// head dimension, S the tokens of a frame), which bounds the key energy of a
// frame, tr(K_hat^T B K_hat) <= 1, and keeps every frame transition
// non-expansive; queries take ReLU(RMSNorm(q)) without the scale.
// RMSNorm(x) = x / sqrt(mean(x^2) + 1e-6) * weight over the D entries of a
// token-head row.  One warp per row: each lane holds up to four entries, the
// mean square is a warp reduction in fp32, and the result is written in the
// input's dtype to a copy in the workspace.
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr float kEps = 1e-6f;

template <typename T> __device__ __forceinline__ float ldv(const T *p, long long i);
template <> __device__ __forceinline__ float ldv<float>(const float *p, long long i) { return p[i]; }
template <> __device__ __forceinline__ float ldv<__nv_bfloat16>(const __nv_bfloat16 *p, long long i) {
    return __bfloat162float(p[i]);
}
template <typename T> __device__ __forceinline__ void stv(T *p, long long i, float x);
template <> __device__ __forceinline__ void stv<float>(float *p, long long i, float x) { p[i] = x; }
template <> __device__ __forceinline__ void stv<__nv_bfloat16>(__nv_bfloat16 *p, long long i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

// rows of d entries (d <= 128): y = max(x / sqrt(mean(x^2) + eps) * w, 0) * post
template <typename T>
__global__ void __launch_bounds__(256) qk_feature_map_kernel(const T *__restrict__ x, T *__restrict__ y,
                                                             const float *__restrict__ w, long long rows, int d,
                                                             float post) {
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const T *xr = x + r * d;
        float v[4];
        float ss = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c = lane + 32 * u;
            v[u] = c < d ? ldv(xr, c) : 0.f;
            ss = fmaf(v[u], v[u], ss);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float inv = 1.f / sqrtf(ss / (float)d + kEps);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c = lane + 32 * u;
            if (c < d) {
                float o = v[u] * inv;
                if (w) o *= w[c];
                stv(y + r * d, c, fmaxf(o, 0.f) * post);
            }
        }
    }
}

template <typename T>
cudaError_t launch_map(const void *x, void *y, const float *w, long long rows, int d, float post, cudaStream_t s) {
    const long long blocks_needed = (rows + 7) / 8;
    const unsigned grid = (unsigned)(blocks_needed < 148 * 16 ? blocks_needed : 148 * 16);
    qk_feature_map_kernel<T><<<grid, 256, 0, s>>>((const T *)x, (T *)y, w, rows, d, post);
    return cudaGetLastError();
}

}  // namespace

size_t qk_prologue_bytes(const Problem &p) {
    const size_t es = p.dtype == GDN_DTYPE_BF16 ? 2 : 4;
    const size_t n = (size_t)p.B * p.T * p.H * p.dk * es;
    size_t bytes = 0;
    if (p.qk_norm & GDN_QK_NORM_KEYS) bytes += align256(n);
    if (p.qk_norm & GDN_QK_NORM_QUERIES) bytes += align256(n);
    return bytes;
}

cudaError_t launch_qk_prologue(Problem &p, void *scratch, cudaStream_t s) {
    const size_t es = p.dtype == GDN_DTYPE_BF16 ? 2 : 4;
    const long long rows = (long long)p.B * p.T * p.H;
    char *dst = (char *)scratch;
    cudaError_t e;
    if (rows == 0) return cudaSuccess;
    if (p.qk_norm & GDN_QK_NORM_KEYS) {
        const float post = 1.f / sqrtf((float)p.dk * (float)p.L);
        e = p.dtype == GDN_DTYPE_BF16 ? launch_map<__nv_bfloat16>(p.k, dst, p.k_norm_weight, rows, p.dk, post, s)
                                      : launch_map<float>(p.k, dst, p.k_norm_weight, rows, p.dk, post, s);
        if (e) return e;
        p.k = dst;
        dst += align256((size_t)rows * p.dk * es);
    }
    if (p.qk_norm & GDN_QK_NORM_QUERIES) {
        e = p.dtype == GDN_DTYPE_BF16 ? launch_map<__nv_bfloat16>(p.q, dst, p.q_norm_weight, rows, p.dk, 1.f, s)
                                      : launch_map<float>(p.q, dst, p.q_norm_weight, rows, p.dk, 1.f, s);
        if (e) return e;
        p.q = dst;
    }
    p.qk_norm = 0;
    return cudaSuccess;
}

}  // namespace gdn
