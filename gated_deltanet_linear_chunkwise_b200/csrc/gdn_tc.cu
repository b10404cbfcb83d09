// gdn_tc.cu -- the tensor-core path for bf16 inputs: workspace layout, TMA
// tensor maps, the gate prologue and the stage sequence.
//
// Stage sequence (forward scans, bf16 q/k/v/o):
//   gates       G = per-frame prefix of log alpha and the column factors (fp32)
//   inverse     T_ii = (I + A_ii)^{-1} per 128-row diagonal block (Gram on tcgen05,
//               doubling on mma.sync)
//   intra       [Ub | W] per frame-head (bf16) by the block recurrence, and the frame's
//               map M, N from its carried matrix (tcgen05)
//   scan        entering state per frame, bf16             (tcgen05; CUDA cores where its
//                                                          shared memory does not fit)
//   U, output   U = Ub - W Sig (tcgen05), then the output by the block recurrence over
//               the frame's state (tcgen05)
// The frame-wise operator: its per-frame maps (the transition kernel), the scan, and the
// U kernel in its output mode.
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "gates.cuh"
#include "gdn_tc.h"
#include "tc_common.cuh"

namespace gdn {
namespace {

// Row stride of the column-factor rows: a multiple of 4 floats so that
// every row starts on a 16-byte boundary (they are read as float4).
inline int cf_stride(int L) { return (L + 3) & ~3; }

struct TcLayout {
    size_t G, CF, Tinv, X, M, Mimg, N, Sig, SigB, U, err;
    size_t Qr, Kr, Vr, Ar, Br;  // token-reversed input copies: reversed calls only (0 bytes otherwise)
    size_t total;
};

TcLayout tc_layout(const Problem &p) {
    const size_t nfh = (size_t)p.B * p.H * p.F;
    const size_t nc = (size_t)p.dk + p.dv;
    TcLayout lay;
    size_t off = 0;
    lay.G = off;    off += align256(sizeof(float) * nfh * (size_t)cf_stride(p.L));
    lay.CF = off;   off += align256(sizeof(float) * nfh * (size_t)cf_stride(p.L));
    lay.Tinv = off; off += align256(2 * nfh * (size_t)((p.L + 127) / 128) * 128 * 128);
    lay.X = off;    off += align256(2 * nfh * p.L * nc);
    // the scan takes M as the tensor-core scan's operand images (or fp32 for the CUDA-core one)
    const bool scan_tc = tc::scan_tc_supported(p.dk, p.dv);
    lay.M = off;    off += align256(sizeof(float) * nfh * p.dk * p.dk);  // CUDA-core scan, segment maps
    lay.Mimg = off; off += scan_tc ? align256(nfh * tc::scan_mimg_bytes(p.dk)) : 0;
    lay.N = off;    off += align256(sizeof(float) * nfh * p.dk * p.dv);
    lay.Sig = off;  off += scan_tc ? 0 : align256(sizeof(float) * nfh * p.dk * p.dv);
    lay.SigB = off; off += align256(2 * nfh * p.dk * p.dv);
    lay.U = off;    off += align256(2 * nfh * p.L * p.dv);
    lay.err = off;  off += 256;
    // A reversed scan runs the forward kernels on token-reversed copies of the inputs.
    const size_t ntok = (size_t)p.B * p.T * p.H;
    const bool rev = p.reverse;
    lay.Qr = off;   off += rev ? align256(2 * ntok * p.dk) : 0;
    lay.Kr = off;   off += rev ? align256(2 * ntok * p.dk) : 0;
    lay.Vr = off;   off += rev ? align256(2 * ntok * p.dv) : 0;
    lay.Ar = off;   off += rev ? align256(4 * ntok) : 0;
    lay.Br = off;   off += rev ? align256(4 * ntok) : 0;
    lay.total = off;
    return lay;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// bf16 tensor map with 128-byte swizzle; dims/strides innermost first
// (strides in bytes for dims 1..rank-1).
bool make_map(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims, const cuuint64_t *strides,
              const cuuint32_t *box) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q/k [B,T,H,d] seen as 4-D (d, H, L, B*F): a frame-head's 128-token tile is
// one box (64 columns, 1 head, 128 tokens, 1 frame); rows past the frame are
// out of bounds and read as zeros.
bool map_tokens(CUtensorMap *m, const void *x, const Problem &p, int d, int box_rows = 128) {
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)p.H, (cuuint64_t)p.L, (cuuint64_t)(p.B * p.F)};
    const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)p.H * d * 2, (cuuint64_t)p.L * p.H * d * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
    return make_map(m, x, 4, dims, strides, box);
}

// fp32 rows [n_fh][stride] seen as 2-D (len, n_fh), boxes of `box` elements, no swizzle;
// elements past `len` read as zeros.
bool map_f32_rows(CUtensorMap *m, const float *x, long long nfh, int len, int stride, int box_len) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)len, (cuuint64_t)nfh};
    const cuuint64_t strides[1] = {(cuuint64_t)stride * 4};
    const cuuint32_t box[2] = {(cuuint32_t)box_len, 1};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(x), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Workspace [n_fh][rows][cols] bf16 seen as 3-D (cols, rows, n_fh).
// Columns [col0, col0 + ncols) of rows of `cols` bf16 ([n_fh][rows][cols]) seen as 3-D
// (ncols, rows, n_fh): stores clip at the part's last column.  col0 * 2 bytes must be a
// multiple of 16 (the map's base).
bool map_row_part(CUtensorMap *m, const void *x, long long nfh, int rows, int cols, int col0, int ncols,
                  int box_rows) {
    const cuuint64_t dims[3] = {(cuuint64_t)ncols, (cuuint64_t)rows, (cuuint64_t)nfh};
    const cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)rows * cols * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    return make_map(m, (const __nv_bfloat16 *)x + col0, 3, dims, strides, box);
}

bool map_rows(CUtensorMap *m, const void *x, long long nfh, int rows, int cols, int box_rows) {
    const cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)nfh};
    const cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)rows * cols * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    return make_map(m, x, 3, dims, strides, box);
}

// G = per-frame inclusive prefix of log alpha; CF = e^{a(s) - G_s} with a(s)
// = G at the last token of s's 64-token tile (<= 1): the column half of the
// split decay factor e^{G_r - G_s} = e^{G_r - a} e^{a - G_s}.
__global__ void __launch_bounds__(256)
gate_prefix_kernel(Problem p, float *__restrict__ G, float *__restrict__ CF) {
    extern __shared__ __align__(16) unsigned char smem[];
    const long long fh = blockIdx.x;
    const long long f = fh % p.F, chain = fh / p.F;
    const int h = (int)(chain % p.H), b = (int)(chain / p.H);
    float *sG = (float *)smem;
    float *sB = sG + p.L;
    float *sScr = sB + p.L;
    frame_gates<float>(p, b, h, f, sG, sB, sScr);
    const int cfs = (p.L + 3) & ~3;  // cf_stride(L): G and CF rows start on 16-byte boundaries
    for (int i = threadIdx.x; i < p.L; i += blockDim.x) {
        const int end = min((i / 64) * 64 + 63, p.L - 1);
        G[fh * cfs + i] = sG[i];
        CF[fh * cfs + i] = __expf(sG[end] - sG[i]);
    }
}

bool tc_disabled_by_env() {
    const char *e = getenv("GDN_DISABLE_TC");
    return e && e[0] == '1';
}

}  // namespace

bool tc_fuses_qk_prologue(const Problem &p) { return tc_supports(p) && p.mode == GDN_MODE_FRAME; }

bool tc_supports(const Problem &p) {
    static const bool disabled = tc_disabled_by_env();
    return !disabled && p.dtype == GDN_DTYPE_BF16;
}

size_t tc_workspace_bytes(const Problem &p) { return tc_layout(p).total; }

// The forward pass.  `scan_reverse` is the caller's reverse flag: on token-reversed copies the
// kernels run forward, and only the chunk-reset rule of the scan still follows the original
// token positions.
cudaError_t launch_tc_forward(const Problem &p, void *ws, int scan_reverse, cudaStream_t s, cudaEvent_t *ev) {
    const TcLayout lay = tc_layout(p);
    char *base = (char *)ws;
    const long long nfh = (long long)p.B * p.H * p.F;
    const int nblk = (p.L + tc::BM - 1) / tc::BM;
    float *G = (float *)(base + lay.G);
    float *CF = (float *)(base + lay.CF);
    __nv_bfloat16 *X = (__nv_bfloat16 *)(base + lay.X);
    float *Mb = (float *)(base + lay.M), *Nb = (float *)(base + lay.N), *Sig = (float *)(base + lay.Sig);
    __nv_bfloat16 *SigB = (__nv_bfloat16 *)(base + lay.SigB);
    __nv_bfloat16 *U = (__nv_bfloat16 *)(base + lay.U);
    int *err = (int *)(base + lay.err);
    cudaError_t e;

    __nv_bfloat16 *Tinv = (__nv_bfloat16 *)(base + lay.Tinv);
    const int nc = p.dk + p.dv;
    CUtensorMap tm_q, tm_k, tm_v, tm_u128, tm_sig, tm_t, tm_x128, tm_xu, tm_xw, tm_g128, tm_cf128;
    if (!map_tokens(&tm_q, p.q, p, p.dk) || !map_tokens(&tm_k, p.k, p, p.dk) || !map_tokens(&tm_v, p.v, p, p.dv) ||
        !map_rows(&tm_u128, U, nfh, p.L, p.dv, 128) || !map_rows(&tm_sig, SigB, nfh, p.dk, p.dv, p.dk) ||
        !map_rows(&tm_t, Tinv, nfh * nblk, 128, 128, 128) || !map_rows(&tm_x128, X, nfh, p.L, nc, 128) ||
        !map_row_part(&tm_xu, X, nfh, p.L, nc, 0, p.dv, 128) || !map_row_part(&tm_xw, X, nfh, p.L, nc, p.dv, p.dk, 128) ||
        !map_f32_rows(&tm_g128, G, nfh, p.L, cf_stride(p.L), 128) ||
        !map_f32_rows(&tm_cf128, CF, nfh, p.L, cf_stride(p.L), 128))
        return cudaErrorInvalidValue;

    int dev = 0, num_sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    const uint64_t wait_ns = wait_limit_ns();
    const bool scan_tc = tc::scan_tc_supported(p.dk, p.dv);
    __nv_bfloat16 *Mimg = (__nv_bfloat16 *)(base + lay.Mimg);
    if (p.phase == GDN_PHASE_FINISH) {  // the state-independent stages ran in a PREPARE call
        for (int i = 0; i <= 4; ++i)
            if ((e = mark(ev, i, s))) return e;
        goto finish;
    }
    {
    if ((e = cudaMemsetAsync(err, 0, sizeof(int), s))) return e;
    const size_t gsm = sizeof(float) * (2 * p.L + 32);
    if (gsm > 48 * 1024 &&
        (e = cudaFuncSetAttribute(gate_prefix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gsm)))
        return e;
    if ((e = mark(ev, 0, s))) return e;
    gate_prefix_kernel<<<(unsigned)nfh, 256, gsm, s>>>(p, G, CF);
    if ((e = cudaGetLastError())) return e;
    if ((e = mark(ev, 1, s))) return e;
    if ((e = tc::launch_diag_inverse(tm_k, tm_t, p.beta, G, CF, p.L, p.dk, p.H, nblk, p.F, p.T, nfh, err, wait_ns,
                                     debug_drop_signal(), s)))
        return e;
    if ((e = mark(ev, 2, s))) return e;
    // the intra-frame solve also forms the frame's transition: fp32 M for the CUDA-core scan (and the
    // segment-map scan), the operand images for the tensor-core one
    tc::IntraParams ip;
    ip.G = G; ip.beta = p.beta; ip.X = X;
    ip.M = (!scan_tc || p.map_out) ? Mb : nullptr; ip.Mimg = scan_tc ? Mimg : nullptr; ip.N = Nb;
    ip.L = p.L; ip.dk = p.dk; ip.dv = p.dv; ip.H = p.H; ip.nblk = nblk;
    ip.F = p.F; ip.T = p.T; ip.err = err; ip.wait_ns = wait_ns;
    if ((e = tc::launch_intra_tc(tm_k, tm_v, tm_t, tm_xu, tm_xw, ip, nfh, s))) return e;
    if ((e = mark(ev, 3, s))) return e;
    if (p.map_out && (e = simt_segment_map(p, Mb, Nb, s))) return e;
    if ((e = mark(ev, 4, s))) return e;
    if (p.phase == GDN_PHASE_PREPARE) {
        for (int i = 5; i <= GDN_NUM_STAGES; ++i)
            if ((e = mark(ev, i, s))) return e;
        return cudaSuccess;
    }
    }
finish:
    Problem ps = p;
    ps.reverse = scan_reverse;
    if (scan_tc) {
        if ((e = tc::launch_scan_tc(ps, Mimg, Nb, SigB, nullptr, err, wait_limit_ns(), s))) return e;
    } else if ((e = simt_scan(ps, Mb, Nb, Sig, SigB, s))) {
        return e;
    }
    if ((e = mark(ev, 5, s))) return e;
    tc::UParams up;
    up.X = X; up.U = U;
    up.L = p.L; up.dk = p.dk; up.dv = p.dv; up.nblk = nblk; up.err = err;
    up.frame = 0; up.o = nullptr; up.T = p.T; up.F = p.F; up.H = p.H; up.accumulate = 0;
    up.norm_q = 0; up.q_w = nullptr; up.wait_ns = wait_ns;
    if ((e = tc::launch_u_tc(tm_x128, tm_q, tm_sig, tm_u128, up, nfh, num_sms, s))) return e;
    if ((e = mark(ev, 6, s))) return e;

    tc::OutParams op;
    op.G = G;
    op.CF = CF;
    op.o = p.o;
    op.L = p.L; op.dk = p.dk; op.dv = p.dv; op.H = p.H; op.nblk = nblk;
    op.F = p.F; op.T = p.T; op.n_fh = nfh;
    op.accumulate = p.accumulate;
    op.reverse_out = scan_reverse;
    op.SigB = SigB;
    op.err = err;
    op.wait_ns = wait_ns;
    // o by tiled stores when it is written plainly and its map can be made (16-byte aligned base)
    CUtensorMap tm_o;
    memset(&tm_o, 0, sizeof(tm_o));
    op.o_tma = !p.accumulate && !scan_reverse && map_tokens(&tm_o, p.o, p, p.dv);
    if ((e = tc::launch_output_tc(tm_q, tm_k, tm_u128, tm_g128, tm_cf128, tm_o, op, s))) return e;
    return mark(ev, 7, s);
}

namespace {

// dst row (b, T-1-t) = src row (b, t) of a [B, T, ...] tensor, one warp per row, 16-byte
// pieces when the row length allows (else 4-byte words); bandwidth bound.
template <typename V>
__global__ void __launch_bounds__(256) reverse_rows_kernel(const V *__restrict__ src, V *__restrict__ dst,
                                                           long long rows, long long T, int row_vecs) {
    const long long row = blockIdx.x * 8ll + (threadIdx.x >> 5);
    if (row >= rows) return;
    const long long t = row % T, b = row / T;
    const V *s = src + row * row_vecs;
    V *d = dst + (b * T + (T - 1 - t)) * row_vecs;
    for (int i = threadIdx.x & 31; i < row_vecs; i += 32) d[i] = s[i];
}

cudaError_t reverse_rows(const void *src, void *dst, int B, long long T, size_t row_bytes, cudaStream_t s) {
    const long long rows = (long long)B * T;
    const unsigned grid = (unsigned)((rows + 7) / 8);
    if (rows == 0) return cudaSuccess;
    if (row_bytes % 16 == 0 && ((uintptr_t)src | (uintptr_t)dst) % 16 == 0)
        reverse_rows_kernel<uint4><<<grid, 256, 0, s>>>((const uint4 *)src, (uint4 *)dst, rows, T, (int)(row_bytes / 16));
    else
        reverse_rows_kernel<uint32_t><<<grid, 256, 0, s>>>((const uint32_t *)src, (uint32_t *)dst, rows, T,
                                                           (int)(row_bytes / 4));
    return cudaGetLastError();
}

}  // namespace

// The frame-wise operator (SANA-WM summary, "Memory-Efficient Long-Context Modeling
// (Section 3.2)", paragraph "Adaptation to video: frame-wise recurrence"): the per-frame
// maps M = gamma (I - K^T B K), N = K^T B V (transition kernel, frame mode), the scan
// (states after each frame's update; frames walked backwards when reversed), and
// o (+)= Q Sig_t (U kernel, frame mode).  Per-frame sums do not depend on token order, so
// a reversed call needs no reversed copies.
cudaError_t launch_tc_frame(const Problem &p, void *ws, cudaStream_t s, cudaEvent_t *ev) {
    const TcLayout lay = tc_layout(p);
    char *base = (char *)ws;
    const long long nfh = (long long)p.B * p.H * p.F;
    const int nblk = (p.L + tc::BM - 1) / tc::BM;
    float *Mb = (float *)(base + lay.M), *Nb = (float *)(base + lay.N);
    __nv_bfloat16 *Mimg = (__nv_bfloat16 *)(base + lay.Mimg);
    const bool scan_tc = tc::scan_tc_supported(p.dk, p.dv);
    __nv_bfloat16 *SigB = (__nv_bfloat16 *)(base + lay.SigB);
    int *err = (int *)(base + lay.err);
    cudaError_t e;
    CUtensorMap tm_q, tm_k64, tm_v64, tm_sig;
    if (!map_tokens(&tm_q, p.q, p, p.dk) || !map_tokens(&tm_k64, p.k, p, p.dk, 64) ||
        !map_tokens(&tm_v64, p.v, p, p.dv, 64) || !map_rows(&tm_sig, SigB, nfh, p.dk, p.dv, p.dk))
        return cudaErrorInvalidValue;
    if ((e = cudaMemsetAsync(err, 0, sizeof(int), s))) return e;
    // stages 0-2 (gates, inverses, intra solve) and 5 (U) do not exist in this operator
    for (int i = 0; i <= 3; ++i)
        if ((e = mark(ev, i, s))) return e;
    tc::TransParams tp;
    tp.M = scan_tc ? nullptr : Mb; tp.Mimg = scan_tc ? Mimg : nullptr; tp.N = Nb;
    tp.L = p.L; tp.dk = p.dk; tp.dv = p.dv; tp.H = p.H; tp.F = p.F; tp.err = err;
    tp.beta = p.beta; tp.gamma = p.gamma; tp.T = p.T;
    // the q/k feature maps, when requested, are applied to the staged tiles (no copy pass)
    tp.norm_k = (p.qk_norm & GDN_QK_NORM_KEYS) ? 1 : 0;
    tp.k_w = p.k_norm_weight;
    tp.k_post = 1.f / sqrtf((float)p.dk * (float)p.L);
    tp.wait_ns = wait_limit_ns();
    int dev = 0, num_sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if ((e = tc::launch_transition_tc(tm_k64, tm_v64, tp, nfh, s))) return e;
    if ((e = mark(ev, 4, s))) return e;
    if (scan_tc) {
        if ((e = tc::launch_scan_tc(p, Mimg, Nb, SigB, nullptr, err, wait_limit_ns(), s))) return e;
    } else if ((e = simt_scan(p, Mb, Nb, nullptr, SigB, s))) {
        return e;
    }
    if ((e = mark(ev, 5, s)) || (e = mark(ev, 6, s))) return e;
    tc::UParams up;
    up.X = nullptr; up.U = nullptr;
    up.L = p.L; up.dk = p.dk; up.dv = p.dv; up.nblk = nblk; up.err = err;
    up.frame = 1; up.o = (__nv_bfloat16 *)p.o; up.T = p.T; up.F = p.F; up.H = p.H; up.accumulate = p.accumulate;
    up.norm_q = (p.qk_norm & GDN_QK_NORM_QUERIES) ? 1 : 0;
    up.q_w = p.q_norm_weight;
    up.wait_ns = tp.wait_ns;
    if ((e = tc::launch_u_tc(tm_q, tm_q, tm_sig, tm_q, up, nfh, num_sms, s))) return e;
    return mark(ev, 7, s);
}

cudaError_t launch_tc(const Problem &p, void *ws, cudaStream_t s, cudaEvent_t *ev) {
    if (p.mode == GDN_MODE_FRAME) return launch_tc_frame(p, ws, s, ev);
    if (!p.reverse) return launch_tc_forward(p, ws, 0, s, ev);  // accumulate_o is the output kernel's
    // A reversed scan runs the forward kernels on token-reversed copies of the inputs (the
    // reversed recurrence is the forward one on them); the output kernel writes each row back
    // to its own token (adding to o when accumulating), and the chunk-reset rule of the scan
    // follows the original token positions.
    const TcLayout lay = tc_layout(p);
    char *base = (char *)ws;
    Problem q = p;
    q.reverse = 0;
    cudaError_t e;
    const size_t rq = (size_t)p.H * p.dk * 2, rv = (size_t)p.H * p.dv * 2, rg = (size_t)p.H * 4;
    if ((e = reverse_rows(p.q, base + lay.Qr, p.B, p.T, rq, s))) return e;
    if ((e = reverse_rows(p.k, base + lay.Kr, p.B, p.T, rq, s))) return e;
    if ((e = reverse_rows(p.v, base + lay.Vr, p.B, p.T, rv, s))) return e;
    if ((e = reverse_rows(p.alpha, base + lay.Ar, p.B, p.T, rg, s))) return e;
    if ((e = reverse_rows(p.beta, base + lay.Br, p.B, p.T, rg, s))) return e;
    q.q = base + lay.Qr;
    q.k = base + lay.Kr;
    q.v = base + lay.Vr;
    q.alpha = (const float *)(base + lay.Ar);
    q.beta = (const float *)(base + lay.Br);
    return launch_tc_forward(q, ws, p.reverse, s, ev);
}

int *tc_error_word(const Problem &p, void *ws) { return (int *)((char *)ws + tc_layout(p).err); }

}  // namespace gdn
