// gdn_api.cu -- the C ABI: argument validation, workspace, dispatch.
//
// Validation happens before anything is enqueued; on a validation error the
// call returns its status with no launch and no output touched.  No C++
// exception crosses the ABI (every entry point is noexcept and catches).
#include <cstdarg>
#include <cstdlib>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "gdn_internal.h"
#include "gdn_tc.h"

namespace {

thread_local char g_err[512] = "";

void set_err(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
}

// The library's own scratch (the workspace when the caller passes none, and
// gdn_fwd_host's device copies) comes from one stream-ordered pool per
// device whose release threshold is unlimited: memory freed at the end of a
// call stays reserved for the next one instead of being unmapped, so a
// repeated call does not pay for mapping gigabytes again.
cudaError_t scratch_alloc(void **ptr, size_t bytes, cudaStream_t s) {
    static std::mutex mu;
    static cudaMemPool_t pools[128] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 128) return cudaMallocAsync(ptr, bytes, s);
    cudaMemPool_t pool;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!pools[dev]) {
            cudaMemPoolProps props;
            memset(&props, 0, sizeof(props));
            props.allocType = cudaMemAllocationTypePinned;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            if ((e = cudaMemPoolCreate(&pools[dev], &props)) != cudaSuccess) {
                pools[dev] = nullptr;
                return e;
            }
            uint64_t keep = UINT64_MAX;
            cudaMemPoolSetAttribute(pools[dev], cudaMemPoolAttrReleaseThreshold, &keep);
        }
        pool = pools[dev];
    }
    return cudaMallocFromPoolAsync(ptr, bytes, pool, s);
}

bool misaligned(const void *ptr) { return ptr && (reinterpret_cast<uintptr_t>(ptr) & 15u); }

bool head_dim_ok(int d) { return d >= 16 && d <= 128 && d % 16 == 0; }

// Range [p, p+n) of two buffers overlap?
bool overlap(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || !na || !nb) return false;
    const char *x = (const char *)a, *y = (const char *)b;
    return x < y + nb && y < x + na;
}

int validate_sizes(const gdn_args &a) {
    if (a.dtype != GDN_DTYPE_BF16 && a.dtype != GDN_DTYPE_F32) {
        set_err("dtype %d is neither GDN_DTYPE_BF16 nor GDN_DTYPE_F32", a.dtype);
        return GDN_ERR_INVALID_ARG;
    }
    if (a.B < 0 || a.H < 0 || a.T < 0) {
        set_err("negative size: B=%d H=%d T=%lld", a.B, a.H, a.T);
        return GDN_ERR_INVALID_ARG;
    }
    if (a.frame_len <= 0) {
        set_err("frame_len must be positive (got %d)", a.frame_len);
        return GDN_ERR_INVALID_ARG;
    }
    if (a.reverse != 0 && a.reverse != 1) { set_err("reverse must be 0 or 1"); return GDN_ERR_INVALID_ARG; }
    if (a.accumulate_o != 0 && a.accumulate_o != 1) { set_err("accumulate_o must be 0 or 1"); return GDN_ERR_INVALID_ARG; }
    if (a.check_finite != 0 && a.check_finite != 1) { set_err("check_finite must be 0 or 1"); return GDN_ERR_INVALID_ARG; }
    if (a.mode != GDN_MODE_TOKEN && a.mode != GDN_MODE_FRAME) {
        set_err("mode must be GDN_MODE_TOKEN or GDN_MODE_FRAME (got %d)", a.mode);
        return GDN_ERR_INVALID_ARG;
    }
    if (a.qk_norm < 0 || a.qk_norm > (GDN_QK_NORM_KEYS | GDN_QK_NORM_QUERIES)) {
        set_err("qk_norm must be a mask of GDN_QK_NORM_KEYS and GDN_QK_NORM_QUERIES (got %d)", a.qk_norm);
        return GDN_ERR_INVALID_ARG;
    }
    if (a.reset_every < 0 || (a.reset_every > 0 && a.reset_every % a.frame_len != 0)) {
        set_err("reset_every (%lld) must be 0 or a positive multiple of frame_len (%d)", a.reset_every, a.frame_len);
        return GDN_ERR_INVALID_ARG;
    }
    if (a.T % a.frame_len != 0) {
        set_err("T (%lld) is not a multiple of frame_len (%d)", a.T, a.frame_len);
        return GDN_ERR_SHAPE;
    }
    if (!head_dim_ok(a.d_k) || !head_dim_ok(a.d_v)) {
        set_err("head dims d_k=%d d_v=%d: each must be a multiple of 16 in [16, 128]", a.d_k, a.d_v);
        return GDN_ERR_UNSUPPORTED;
    }
    if (a.frame_len > 4096) {
        set_err("frame_len %d exceeds the supported maximum 4096", a.frame_len);
        return GDN_ERR_UNSUPPORTED;
    }
    const long long dmax = a.d_k > a.d_v ? a.d_k : a.d_v;
    // B*T*H*dmax < 2^62 and B*H*F < 2^31, checked without overflow
    const long double elems = (long double)a.B * (long double)a.T * (long double)a.H * (long double)dmax;
    if (elems >= 4.611686018427387904e18L) {
        set_err("B*T*H*d = %.3Le elements overflows the 2^62 index range", elems);
        return GDN_ERR_SHAPE;
    }
    const long long F = a.T / a.frame_len;
    if ((long double)a.B * a.H * F >= 2147483648.0L) {
        set_err("B*H*frames = %.3Le exceeds 2^31", (long double)a.B * a.H * F);
        return GDN_ERR_SHAPE;
    }
    return GDN_OK;
}

int validate(const gdn_args &a, gdn::Problem &p) {
    int st = validate_sizes(a);
    if (st != GDN_OK) return st;
    const long long F = a.T / a.frame_len;
    const bool empty = (a.B == 0 || a.H == 0 || a.T == 0);
    const bool frame = a.mode == GDN_MODE_FRAME;
    if (a.phase != GDN_PHASE_ALL && a.phase != GDN_PHASE_PREPARE && a.phase != GDN_PHASE_FINISH) {
        set_err("phase must be GDN_PHASE_ALL, GDN_PHASE_PREPARE or GDN_PHASE_FINISH (got %d)", a.phase);
        return GDN_ERR_INVALID_ARG;
    }
    if (a.phase != GDN_PHASE_ALL) {
        if (!a.workspace) {
            set_err("a PREPARE / FINISH call keeps its state in a caller workspace (workspace is NULL)");
            return GDN_ERR_INVALID_ARG;
        }
        if (frame || a.reverse || a.accumulate_o || a.qk_norm) {
            set_err("PREPARE / FINISH calls take the token-wise forward scan without reverse, accumulate_o or qk_norm");
            return GDN_ERR_NOT_IMPLEMENTED;
        }
    }
    if (a.segment_map && a.phase != GDN_PHASE_PREPARE) {
        set_err("segment_map is written by GDN_PHASE_PREPARE calls only");
        return GDN_ERR_INVALID_ARG;
    }
    if (misaligned(a.segment_map)) {
        set_err("segment_map = %p is not 16-byte aligned", (const void *)a.segment_map);
        return GDN_ERR_ALIGNMENT;
    }
    const bool need_o = a.phase != GDN_PHASE_PREPARE;
    if (!empty && (!a.q || !a.k || !a.v || !a.beta || (need_o && !a.o))) {
        set_err("q, k, v, beta and o are required (one is NULL)");
        return GDN_ERR_INVALID_ARG;
    }
    if (!empty && !frame && !a.alpha) {
        set_err("alpha is required (NULL)");
        return GDN_ERR_INVALID_ARG;
    }
    if (!empty && frame && !a.gamma) {
        set_err("gamma is required in GDN_MODE_FRAME (NULL)");
        return GDN_ERR_INVALID_ARG;
    }
    const void *ptrs[] = {a.q, a.k, a.v, a.alpha, a.beta, a.S_in, a.S_out, a.o};
    const char *names[] = {"q", "k", "v", "alpha", "beta", "S_in", "S_out", "o"};
    for (int i = 0; i < 8; ++i)
        if (misaligned(ptrs[i])) {
            set_err("%s = %p is not 16-byte aligned", names[i], ptrs[i]);
            return GDN_ERR_ALIGNMENT;
        }
    if (a.status_dev && (reinterpret_cast<uintptr_t>(a.status_dev) & 3u)) {
        set_err("status_dev = %p is not 4-byte aligned", (const void *)a.status_dev);
        return GDN_ERR_ALIGNMENT;
    }
    if (a.workspace && (reinterpret_cast<uintptr_t>(a.workspace) & 255u)) {
        set_err("workspace = %p is not 256-byte aligned", a.workspace);
        return GDN_ERR_ALIGNMENT;
    }
    // outputs may not overlap inputs (S_in == S_out exactly is allowed)
    const size_t es = a.dtype == GDN_DTYPE_BF16 ? 2 : 4;
    const size_t nqk = (size_t)a.B * a.T * a.H * a.d_k * es, nv = (size_t)a.B * a.T * a.H * a.d_v * es;
    const size_t ng = (size_t)a.B * a.T * a.H * 4, ns = (size_t)a.B * a.H * a.d_v * a.d_k * 4;
    const size_t ngam = frame ? (size_t)a.B * F * a.H * 4 : 0;
    const void *ins[] = {a.q, a.k, a.v, frame ? nullptr : a.alpha, a.beta, a.S_in, frame ? a.gamma : nullptr};
    const size_t insz[] = {nqk, nqk, nv, ng, ng, ns, ngam};
    const char *in_names[] = {"q", "k", "v", "alpha", "beta", "S_in", "gamma"};
    for (int i = 0; i < 7; ++i) {
        if (overlap(a.o, nv, ins[i], insz[i])) {
            set_err("o overlaps input %s", in_names[i]);
            return GDN_ERR_INVALID_ARG;
        }
        if (a.S_out && !(i == 5 && a.S_out == a.S_in) && overlap(a.S_out, ns, ins[i], insz[i])) {
            set_err("S_out overlaps input %s", in_names[i]);
            return GDN_ERR_INVALID_ARG;
        }
    }
    if (overlap(a.o, nv, a.S_out, ns)) { set_err("o overlaps S_out"); return GDN_ERR_INVALID_ARG; }
    if (a.segment_map) {
        const size_t nm = (size_t)a.B * a.H * (a.d_k + a.d_v) * a.d_k * 4;
        for (int i = 0; i < 7; ++i)
            if (overlap(a.segment_map, nm, ins[i], insz[i])) {
                set_err("segment_map overlaps input %s", in_names[i]);
                return GDN_ERR_INVALID_ARG;
            }
    }

    p.dtype = a.dtype;
    p.q = a.q; p.k = a.k; p.v = a.v;
    p.alpha = a.alpha; p.beta = a.beta;
    p.S_in = a.S_in; p.S_out = a.S_out; p.o = a.o;
    p.B = a.B; p.H = a.H; p.T = a.T; p.L = a.frame_len;
    p.dk = a.d_k; p.dv = a.d_v; p.F = F;
    p.reverse = a.reverse; p.accumulate = a.accumulate_o; p.reset_every = a.reset_every;
    p.mode = a.mode; p.gamma = frame ? a.gamma : nullptr;
    p.qk_norm = a.qk_norm;
    p.k_norm_weight = (a.qk_norm & GDN_QK_NORM_KEYS) ? a.k_norm_weight : nullptr;
    p.q_norm_weight = (a.qk_norm & GDN_QK_NORM_QUERIES) ? a.q_norm_weight : nullptr;
    if (frame) p.alpha = nullptr;
    p.phase = a.phase;
    p.map_out = a.segment_map;
    if (p.phase == GDN_PHASE_PREPARE) {  // nothing of the state or the output is touched
        p.S_in = nullptr;
        p.S_out = nullptr;
        p.o = nullptr;
    }
    return GDN_OK;
}

// Which implementation serves this problem, and how much scratch it needs.
bool use_tc(const gdn::Problem &p) { return gdn::tc_supports(p); }

// The operator's scratch (the q/k prologue's copies follow it).
size_t operator_workspace(const gdn::Problem &p) {
    return use_tc(p) ? gdn::tc_workspace_bytes(p) : gdn::simt_workspace_bytes(p);
}

// The q/k prologue runs as its own pass (normalised copies after the operator's scratch)
// except where the kernels apply it to their staged tiles.
bool separate_prologue(const gdn::Problem &p) { return p.qk_norm && !gdn::tc_fuses_qk_prologue(p); }

size_t workspace_for(const gdn::Problem &p) {
    return operator_workspace(p) + (separate_prologue(p) ? gdn::qk_prologue_bytes(p) : 0);
}

__global__ void nonfinite_scan_f32(const float *x, long long n, int *flag) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        if (!isfinite(x[i])) { atomicOr(flag, 1); return; }
}
__global__ void nonfinite_scan_bf16(const __nv_bfloat16 *x, long long n, int *flag) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        if (!isfinite(__bfloat162float(x[i]))) { atomicOr(flag, 1); return; }
}

int cuda_fail(cudaError_t e, const char *what) {
    set_err("%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
    return GDN_ERR_CUDA;
}

int run(const gdn_args &a) noexcept {
    try {
        gdn::NvtxRange range(a.phase == GDN_PHASE_PREPARE  ? "gdn_fwd_ex (prepare)"
                             : a.phase == GDN_PHASE_FINISH ? "gdn_fwd_ex (finish)"
                                                           : "gdn_fwd_ex");
        g_err[0] = '\0';
        if (a.struct_size != (int)sizeof(gdn_args)) {
            set_err("gdn_args.struct_size = %d, this library expects %d", a.struct_size, (int)sizeof(gdn_args));
            return GDN_ERR_INVALID_ARG;
        }
        gdn::Problem p;
        int st = validate(a, p);
        if (st != GDN_OK) return st;
        cudaStream_t s = reinterpret_cast<cudaStream_t>(a.stream);
        const size_t sbytes = (size_t)a.B * a.H * a.d_v * a.d_k * sizeof(float);

        if (a.B == 0 || a.H == 0 || a.T == 0) {  // nothing to compute
            if (a.status_dev) {
                cudaError_t e = cudaMemsetAsync(a.status_dev, 0, sizeof(int), s);
                if (e) return cuda_fail(e, "status word");
            }
        }
        if (a.B == 0 || a.H == 0) return GDN_OK;
        if (a.T == 0 && a.phase == GDN_PHASE_PREPARE) {  // an empty segment maps every state to itself
            if (a.segment_map) {
                cudaError_t e = gdn::launch_identity_map(a.segment_map, a.B, a.H, a.d_k, a.d_v, s);
                if (e) return cuda_fail(e, "segment map");
            }
            return GDN_OK;
        }
        if (a.T == 0) {  // nothing to scan: the final state is the initial state
            if (a.S_out && a.S_out != a.S_in) {
                cudaError_t e = a.S_in ? cudaMemcpyAsync(a.S_out, a.S_in, sbytes, cudaMemcpyDeviceToDevice, s)
                                       : cudaMemsetAsync(a.S_out, 0, sbytes, s);
                if (e) return cuda_fail(e, "state copy");
            }
            return GDN_OK;
        }
        const size_t need = workspace_for(p);
        void *ws = a.workspace;
        bool owned = false;
        if (ws) {
            if (a.workspace_bytes < need) {
                set_err("workspace_bytes = %zu < %zu required", a.workspace_bytes, need);
                return GDN_ERR_NO_MEMORY;
            }
        } else {
            cudaError_t e = scratch_alloc(&ws, need, s);
            if (e != cudaSuccess || !ws) {
                cudaGetLastError();
                set_err("device scratch allocation (%zu bytes) failed: %s", need, cudaGetErrorString(e));
                return GDN_ERR_NO_MEMORY;
            }
            owned = true;
        }
        cudaEvent_t ev[GDN_NUM_STAGES + 1] = {};
        cudaEvent_t *evp = nullptr;
        if (a.stage_ms) {
            for (int i = 0; i <= GDN_NUM_STAGES; ++i) {
                cudaError_t ee = cudaEventCreate(&ev[i]);
                if (ee) {
                    for (int j = 0; j < i; ++j) cudaEventDestroy(ev[j]);
                    if (owned) cudaFreeAsync(ws, s);
                    return cuda_fail(ee, "stage timing events");
                }
            }
            evp = ev;
        }
        const bool tc = use_tc(p);
        cudaError_t e = cudaSuccess;
        if (separate_prologue(p))  // normalised q / k copies after the operator's scratch; p now points at them
            e = gdn::launch_qk_prologue(p, (char *)ws + operator_workspace(p), s);
        if (e == cudaSuccess) e = tc ? gdn::launch_tc(p, ws, s, evp) : gdn::launch_simt(p, ws, s, evp);
        // the device-side wait status, in stream order, for callers that check it later
        if (e == cudaSuccess && a.status_dev)
            e = tc ? cudaMemcpyAsync(a.status_dev, gdn::tc_error_word(p, ws), sizeof(int), cudaMemcpyDeviceToDevice, s)
                   : cudaMemsetAsync(a.status_dev, 0, sizeof(int), s);
        // synchronous modes also report a device-side wait that gave up
        int timed_out = 0;
        if (e == cudaSuccess && tc && (a.stage_ms || a.check_finite)) {
            e = cudaMemcpyAsync(&timed_out, gdn::tc_error_word(p, ws), sizeof(int), cudaMemcpyDeviceToHost, s);
            if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        }
        if (owned) {
            cudaError_t e2 = cudaFreeAsync(ws, s);
            if (e == cudaSuccess) e = e2;
        }
        if (evp) {
            if (e == cudaSuccess) e = cudaStreamSynchronize(s);
            for (int i = 0; i < GDN_NUM_STAGES; ++i) {
                float ms = -1.f;
                if (e == cudaSuccess && cudaEventElapsedTime(&ms, ev[i], ev[i + 1]) != cudaSuccess) ms = -1.f;
                a.stage_ms[i] = ms;
            }
            for (int i = 0; i <= GDN_NUM_STAGES; ++i) cudaEventDestroy(ev[i]);
        }
        if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
        if (timed_out == 2) {  // sm100::kErrSmemAlign
            set_err("a kernel's dynamic shared memory did not start on a 1024-byte boundary; it did no work");
            return GDN_ERR_CUDA;
        }
        if (timed_out) {
            set_err("a bounded device-side wait gave up (error word %d)", timed_out);
            return GDN_ERR_TIMEOUT;
        }

        if (a.check_finite) {
            int *flag = nullptr;
            int host = 0;
            if ((e = cudaMallocAsync((void **)&flag, sizeof(int), s))) return cuda_fail(e, "finite-check flag");
            cudaMemsetAsync(flag, 0, sizeof(int), s);
            const long long no = (long long)a.B * a.T * a.H * a.d_v;
            if (a.dtype == GDN_DTYPE_F32) nonfinite_scan_f32<<<1184, 256, 0, s>>>((const float *)a.o, no, flag);
            else nonfinite_scan_bf16<<<1184, 256, 0, s>>>((const __nv_bfloat16 *)a.o, no, flag);
            if (a.S_out) nonfinite_scan_f32<<<148, 256, 0, s>>>(a.S_out, (long long)(sbytes / 4), flag);
            cudaMemcpyAsync(&host, flag, sizeof(int), cudaMemcpyDeviceToHost, s);
            cudaFreeAsync(flag, s);
            if ((e = cudaStreamSynchronize(s))) return cuda_fail(e, "finite check");
            if (host) {
                set_err("o or S_out holds a NaN or Inf");
                return GDN_ERR_NONFINITE;
            }
        }
        return GDN_OK;
    } catch (...) {
        set_err("internal error (exception caught at the ABI boundary)");
        return GDN_ERR_CUDA;
    }
}

gdn_args make_args(int dtype, const void *q, const void *k, const void *v, const float *alpha,
                   const float *beta, const float *S_in, float *S_out, void *o, int B, int H,
                   long long T, int frame_len, int d_k, int d_v, gdn_stream_t stream) {
    gdn_args a;
    memset(&a, 0, sizeof(a));
    a.struct_size = (int)sizeof(gdn_args);
    a.dtype = dtype;
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta;
    a.S_in = S_in; a.S_out = S_out; a.o = o;
    a.B = B; a.H = H; a.T = T; a.frame_len = frame_len; a.d_k = d_k; a.d_v = d_v;
    a.stream = stream;
    return a;
}

}  // namespace

namespace gdn {
// Validation and error text shared with the other entry-point files.
int validate_args(const gdn_args &a, Problem &p) { return validate(a, p); }
void set_error_text(const char *msg) { set_err("%s", msg); }

int debug_drop_signal() {
    const char *e = getenv("GDN_DEBUG_DROP_SIGNAL");
    return (e && e[0] == '1') ? 1 : 0;
}

uint64_t wait_limit_ns() {
    const char *e = getenv("GDN_DEBUG_WAIT_LIMIT_US");
    if (!e || !*e) return 2000000000ull;
    char *end = nullptr;
    const unsigned long long us = strtoull(e, &end, 10);
    if (end == e || us >= 2000000ull) return 2000000000ull;
    return (uint64_t)us * 1000ull;
}
}  // namespace gdn

extern "C" {

int gdn_fwd(const void *q, const void *k, const void *v, const float *alpha, const float *beta,
            const float *S_in, float *S_out, void *o, int B, int H, long long T, int frame_len,
            int d_k, int d_v, gdn_stream_t stream) {
    return run(make_args(GDN_DTYPE_BF16, q, k, v, alpha, beta, S_in, S_out, o, B, H, T, frame_len, d_k, d_v, stream));
}

int gdn_fwd_f32(const float *q, const float *k, const float *v, const float *alpha, const float *beta,
                const float *S_in, float *S_out, float *o, int B, int H, long long T, int frame_len,
                int d_k, int d_v, gdn_stream_t stream) {
    return run(make_args(GDN_DTYPE_F32, q, k, v, alpha, beta, S_in, S_out, o, B, H, T, frame_len, d_k, d_v, stream));
}

int gdn_step(const void *q, const void *k, const void *v, const float *alpha, const float *beta,
             const float *S_in, float *S_out, void *o, int B, int H, long long T, int frame_len,
             int d_k, int d_v, gdn_stream_t stream) {
    if (!S_in) {
        set_err("gdn_step requires S_in (the carried state)");
        return GDN_ERR_INVALID_ARG;
    }
    return gdn_fwd(q, k, v, alpha, beta, S_in, S_out, o, B, H, T, frame_len, d_k, d_v, stream);
}

int gdn_step_f32(const float *q, const float *k, const float *v, const float *alpha, const float *beta,
                 const float *S_in, float *S_out, float *o, int B, int H, long long T, int frame_len,
                 int d_k, int d_v, gdn_stream_t stream) {
    if (!S_in) {
        set_err("gdn_step_f32 requires S_in (the carried state)");
        return GDN_ERR_INVALID_ARG;
    }
    return gdn_fwd_f32(q, k, v, alpha, beta, S_in, S_out, o, B, H, T, frame_len, d_k, d_v, stream);
}

int gdn_apply_maps(float *S, const float *maps, int n_maps, int B, int H, int d_k, int d_v, gdn_stream_t stream) {
    try {
        g_err[0] = '\0';
        if (B < 0 || H < 0 || n_maps < 0) {
            set_err("negative size: B=%d H=%d n_maps=%d", B, H, n_maps);
            return GDN_ERR_INVALID_ARG;
        }
        if (!head_dim_ok(d_k) || !head_dim_ok(d_v)) {
            set_err("head dims d_k=%d d_v=%d: each must be a multiple of 16 in [16, 128]", d_k, d_v);
            return GDN_ERR_UNSUPPORTED;
        }
        if ((long long)B * H >= 2147483648ll) {
            set_err("B*H exceeds 2^31");
            return GDN_ERR_SHAPE;
        }
        if ((long long)B * H == 0 || n_maps == 0) return GDN_OK;
        if (!S || !maps) {
            set_err("S and maps are required (one is NULL)");
            return GDN_ERR_INVALID_ARG;
        }
        if (misaligned(S) || misaligned(maps)) {
            set_err("S = %p or maps = %p is not 16-byte aligned", (void *)S, (const void *)maps);
            return GDN_ERR_ALIGNMENT;
        }
        const size_t ns = (size_t)B * H * d_v * d_k * 4, nm = (size_t)n_maps * B * H * (d_k + d_v) * d_k * 4;
        if (overlap(S, ns, maps, nm)) {
            set_err("S overlaps maps");
            return GDN_ERR_INVALID_ARG;
        }
        cudaError_t e = gdn::launch_apply_maps(S, maps, n_maps, B, H, d_k, d_v, reinterpret_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e, "apply maps");
        return GDN_OK;
    } catch (...) {
        set_err("internal error (exception caught at the ABI boundary)");
        return GDN_ERR_CUDA;
    }
}

int gdn_fwd_ex(const gdn_args *a) {
    if (!a) {
        set_err("gdn_fwd_ex: args is NULL");
        return GDN_ERR_INVALID_ARG;
    }
    return run(*a);
}

int gdn_fwd_host(int dtype, const void *q, const void *k, const void *v, const float *alpha, const float *beta,
                 const float *S_in, float *S_out, void *o, int B, int H, long long T, int frame_len, int d_k,
                 int d_v, gdn_stream_t stream) {
    try {
        g_err[0] = '\0';
        gdn_args a = make_args(dtype, q, k, v, alpha, beta, S_in, S_out, o, B, H, T, frame_len, d_k, d_v, stream);
        int st = validate_sizes(a);
        if (st != GDN_OK) return st;
        if (B == 0 || H == 0) return GDN_OK;
        if (T > 0 && (!q || !k || !v || !alpha || !beta || !o)) {
            set_err("q, k, v, alpha, beta and o are required (one is NULL)");
            return GDN_ERR_INVALID_ARG;
        }
        cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
        const size_t es = dtype == GDN_DTYPE_BF16 ? 2 : 4;
        const size_t ntok = (size_t)B * T * H;
        const size_t nq = ntok * d_k * es, nv = ntok * d_v * es, ng = ntok * 4;
        const size_t ns = (size_t)B * H * d_v * d_k * 4;
        // one device block: q | k | v | alpha | beta | S_in | S_out | o | workspace
        const size_t sz[8] = {nq, nq, nv, ng, ng, S_in ? ns : 0, S_out ? ns : 0, nv};
        size_t off[9];
        off[0] = 0;
        for (int i = 0; i < 8; ++i) off[i + 1] = off[i] + ((sz[i] + 255) & ~(size_t)255);
        const size_t wsb = gdn_workspace_bytes(B, H, T, frame_len, d_k, d_v, dtype);
        char *dev = nullptr;
        cudaError_t e = scratch_alloc((void **)&dev, off[8] + wsb, s);
        if (e != cudaSuccess || !dev) {
            cudaGetLastError();
            set_err("device buffer allocation (%zu bytes) failed: %s", off[8] + wsb, cudaGetErrorString(e));
            return GDN_ERR_NO_MEMORY;
        }
        const void *hin[6] = {q, k, v, alpha, beta, S_in};
        for (int i = 0; i < 6 && e == cudaSuccess; ++i)
            if (sz[i]) e = cudaMemcpyAsync(dev + off[i], hin[i], sz[i], cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) {
            cudaFreeAsync(dev, s);
            return cuda_fail(e, "host-to-device copy");
        }
        gdn_args d = make_args(dtype, dev + off[0], dev + off[1], dev + off[2], (const float *)(dev + off[3]),
                               (const float *)(dev + off[4]), S_in ? (const float *)(dev + off[5]) : nullptr,
                               S_out ? (float *)(dev + off[6]) : nullptr, dev + off[7], B, H, T, frame_len, d_k,
                               d_v, stream);
        d.workspace = wsb ? dev + off[8] : nullptr;
        d.workspace_bytes = wsb;
        st = run(d);
        if (st == GDN_OK) {
            e = cudaMemcpyAsync(o, dev + off[7], sz[7], cudaMemcpyDeviceToHost, s);
            if (e == cudaSuccess && S_out) e = cudaMemcpyAsync(S_out, dev + off[6], ns, cudaMemcpyDeviceToHost, s);
        }
        cudaError_t e2 = cudaFreeAsync(dev, s);
        cudaError_t e3 = cudaStreamSynchronize(s);
        if (st != GDN_OK) return st;
        if (e == cudaSuccess) e = e2 ? e2 : e3;
        if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
        return GDN_OK;
    } catch (...) {
        set_err("internal error (exception caught at the ABI boundary)");
        return GDN_ERR_CUDA;
    }
}

size_t gdn_workspace_bytes(int B, int H, long long T, int frame_len, int d_k, int d_v, int dtype) {
    gdn_args a = make_args(dtype, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                           B, H, T, frame_len, d_k, d_v, nullptr);
    if (validate_sizes(a) != GDN_OK) return 0;
    if (B == 0 || H == 0 || T == 0) return 0;
    gdn::Problem p;
    memset(&p, 0, sizeof(p));
    p.dtype = dtype; p.B = B; p.H = H; p.T = T; p.L = frame_len; p.dk = d_k; p.dv = d_v;
    p.F = T / frame_len;
    // the largest case: a reversed, accumulating call (token-reversed input copies and a
    // staged o) with both prologue copies, so a workspace of this size serves every flag
    // combination
    p.reverse = 1;
    p.accumulate = 1;
    p.qk_norm = GDN_QK_NORM_KEYS | GDN_QK_NORM_QUERIES;
    return workspace_for(p);
}

const char *gdn_status_string(int s) {
    switch (s) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
        case GDN_ERR_SHAPE: return "GDN_ERR_SHAPE";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_ALIGNMENT: return "GDN_ERR_ALIGNMENT";
        case GDN_ERR_NO_MEMORY: return "GDN_ERR_NO_MEMORY";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
        case GDN_ERR_NONFINITE: return "GDN_ERR_NONFINITE";
        case GDN_ERR_NOT_IMPLEMENTED: return "GDN_ERR_NOT_IMPLEMENTED";
        default: return "GDN_ERR_UNKNOWN";
    }
}

const char *gdn_last_error(void) { return g_err; }

int gdn_version(void) { return GDN_VERSION; }

}  // extern "C"
