// gdn_internal.h -- shared host/device definitions of the CUDA library.
//
// Chunkwise evaluation of the token-wise gated delta rule with one chunk per
// frame (SANA-WM summary, paper-graph-ui, "Memory-Efficient Long-Context
// Modeling (Section 3.2)", paragraph "Frame-wise Gated DeltaNet (GDN)": one
// latent frame per recurrence step, all of the frame's tokens in parallel).
//
// Per (b, h) chain and frame f, with L = frame_len tokens i, j in [0, L) and
//   G_i   = sum_{m <= i} log alpha_m           (inclusive, within the frame)
//   Sig   = S^T  (d_k x d_v), Sig_0 = the state entering the frame,
// the substitution u_i = beta_i (v_i - alpha_i S_{i-1} k_i) turns the update
// into S_i = alpha_i S_{i-1} + u_i k_i^T, hence
//   (I + A) [Ub | W] = [diag(beta) V | diag(beta e^G) K],
//   A_ij = beta_i e^{G_i - G_j} k_i.k_j  (j < i),           -- kernel 1
//   U = Ub - W Sig_0,
//   M = e^{G_L} I - Kt^T W,  N = Kt^T Ub,  Kt = diag(e^{G_L - G}) K   -- kernel 2
//   Sig_next = M Sig_0 + N                                  -- kernel 3 (scan over frames)
//   O = diag(e^G) Q Sig_0 + tril_incl(Q K^T o e^{G_i - G_j}) U  -- kernel 4
// Every decay factor used is e^{G_i - G_j} with j <= i (<= 1), so no factor
// overflows; log alpha is clamped at -200 so alpha = 0 (a full reset) stays
// finite (e^{-200} is 0 in fp32).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <nvtx3/nvToolsExt.h>

#include "../../include/gdn.h"

namespace gdn {

constexpr float kLogAlphaFloor = -200.0f;

struct Problem {
    int dtype;  // GDN_DTYPE_BF16 / GDN_DTYPE_F32
    const void *q, *k, *v;
    const float *alpha, *beta;
    const float *S_in;
    float *S_out;
    void *o;
    int B, H;
    long long T;
    int L;       // frame_len
    int dk, dv;
    long long F;  // frames per chain, T / L
    int reverse;
    int accumulate;
    long long reset_every;  // tokens; 0 = never
    int mode;               // GDN_MODE_TOKEN / GDN_MODE_FRAME
    const float *gamma;     // GDN_MODE_FRAME: [B, F, H] per-frame decay
    int qk_norm;            // GDN_QK_NORM_* bits still to apply (the prologue clears them)
    const float *k_norm_weight, *q_norm_weight;  // [d_k] or NULL
    int phase;              // GDN_PHASE_ALL / _PREPARE (state-independent stages) / _FINISH (scan on)
    float *map_out;         // PREPARE: the segment's map [B, H, d_k + d_v, d_k] (Phi rows, then Psi), or NULL
};

// Memory index of the frame the scan visits at logical step f.  The
// token-wise paths store per-frame data in visiting order; the frame-wise
// operator stores it by time and the scan walks it backwards when reversed.
__host__ __device__ __forceinline__ long long scan_frame(const Problem &p, long long f) {
    return (p.mode == GDN_MODE_FRAME && p.reverse) ? p.F - 1 - f : f;
}

// Physical token index of logical position i of logical frame f.  The
// reversed-time scan visits frames and the tokens inside them backwards.
__host__ __device__ __forceinline__ long long phys_token(const Problem &p, long long f, int i) {
    return p.reverse ? ((p.F - 1 - f) * p.L + (p.L - 1 - i)) : (f * p.L + i);
}

// Row of token t of chain (b, h) in a [B, T, H, *] tensor.
__host__ __device__ __forceinline__ long long tok_row(const Problem &p, int b, int h, long long t) {
    return ((long long)b * p.T + t) * p.H + h;
}

// Does the state restart from zero before logical frame f (f > 0)?
__host__ __device__ __forceinline__ bool frame_resets(const Problem &p, long long f) {
    if (p.reset_every <= 0 || f == 0) return false;
    if (!p.reverse) return (f * p.L) % p.reset_every == 0;
    const long long pf = p.F - 1 - f;  // physical frame visited at logical f
    return ((pf + 1) * p.L) % p.reset_every == 0;
}

// Workspace carved out of one allocation.
struct Workspace {
    void *base = nullptr;
    size_t bytes = 0;
};

// Optional stage timing: when `ev` is non-null it holds GDN_NUM_STAGES + 1
// events; ev[i] is recorded before stage i and ev[GDN_NUM_STAGES] after the last.
// Every call also leaves an NVTX marker at each stage boundary (host side; free when no
// profiler is attached), inside the NVTX range the entry point opens for the call.
inline cudaError_t mark(cudaEvent_t *ev, int i, cudaStream_t s) {
    static const char *const names[GDN_NUM_STAGES + 1] = {"gdn: gates",      "gdn: diagonal inverses",
                                                          "gdn: intra-frame solve", "gdn: frame transition",
                                                          "gdn: scan",       "gdn: pseudo-values",
                                                          "gdn: output",     "gdn: end"};
    nvtxMarkA(names[i]);
    return ev ? cudaEventRecord(ev[i], s) : cudaSuccess;
}

// NVTX range around one call of the library (RAII).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

// Limit of the kernels' bounded device-side waits for this call, in ns: 2 s, unless the
// debug variable GDN_DEBUG_WAIT_LIMIT_US (read at every call) sets a shorter one so a
// test can make the waits give up (gdn_api.cu).
uint64_t wait_limit_ns();
// Debug: GDN_DEBUG_DROP_SIGNAL=1 (read at every call) makes the diagonal-inverse kernel
// withhold its first block's product, so the wait on it gives up at the limit above and the
// pass reports GDN_ERR_TIMEOUT without any fault (the bounded-wait test).  0 otherwise.
int debug_drop_signal();

// Argument validation of the C ABI (gdn_api.cu): fills p or returns a gdn_status.
int validate_args(const gdn_args &a, Problem &p);
// Sets the thread-local text gdn_last_error() returns.
void set_error_text(const char *msg);

// Scratch layout of the CUDA-core path (byte offsets into the workspace).
struct SimtLayout {
    size_t X, U, M, N, Sig, total;
};
__host__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
SimtLayout simt_layout(const Problem &p);

size_t simt_workspace_bytes(const Problem &p);

// Single CUDA-core stages over bf16 [Ub | W] rows, used as interim stages of
// the tensor-core path (bf16 inputs).
cudaError_t simt_intra_bf16x(const Problem &p, __nv_bfloat16 *X, cudaStream_t s);
cudaError_t simt_transition_bf16x(const Problem &p, const __nv_bfloat16 *X, float *Mb, float *Nb, cudaStream_t s);
cudaError_t simt_scan(const Problem &p, const float *Mb, const float *Nb, float *Sig, __nv_bfloat16 *SigB,
                      cudaStream_t s);
// The segment's composed map (p.map_out): the same scan over the augmented state
// [Sig | P] from [0 | I], N added to the Sig part only, written as Phi = P^T, Psi = Sig^T so
// that S_end = S_begin Phi + Psi over the call's frames.
cudaError_t simt_segment_map(const Problem &p, const float *Mb, const float *Nb, cudaStream_t s);
// S <- S Phi_j + Psi_j for the n maps in order (maps [n][B, H, d_k + d_v, d_k]).
cudaError_t launch_apply_maps(float *S, const float *maps, int n, int B, int H, int dk, int dv, cudaStream_t s);
// Phi = I, Psi = 0: the map of an empty segment.
cudaError_t launch_identity_map(float *map, int B, int H, int dk, int dv, cudaStream_t s);
cudaError_t simt_u_bf16x(const Problem &p, const __nv_bfloat16 *X, const float *Sig, __nv_bfloat16 *U,
                         cudaStream_t s);
cudaError_t launch_simt(const Problem &p, void *ws, cudaStream_t s, cudaEvent_t *ev);
// The frame-wise operator on the CUDA cores (launch_simt dispatches to it).
cudaError_t launch_simt_frame(const Problem &p, void *ws, cudaStream_t s, cudaEvent_t *ev);

// The q/k prologue (qk_prologue.cu): scratch bytes it needs, and the launch that writes the
// normalised copies into `scratch` and points p's q / k at them (clearing p.qk_norm).
size_t qk_prologue_bytes(const Problem &p);
cudaError_t launch_qk_prologue(Problem &p, void *scratch, cudaStream_t s);

}  // namespace gdn
