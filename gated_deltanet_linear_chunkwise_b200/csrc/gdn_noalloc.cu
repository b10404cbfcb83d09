// gdn_noalloc.cu -- gdn_fwd_noalloc: the bf16 forward pass with its scratch
// in a fixed device array, for callers that cannot allocate device memory.
//
// Who needs this: code that must not call cudaMalloc / cudaMallocAsync or a
// framework allocator on the path of a pass -- a streaming decode loop whose
// latency budget cannot absorb an allocation (a cudaMalloc may synchronise
// the device), a host that owns all device memory through its own pool and
// forbids allocations behind its back, or code running where allocation is
// not allowed at all.  Such a caller still passes q/k/v/alpha/beta/S/o.
//
// How: the scratch is one file-scope __device__ array of
// GDN_NOALLOC_SCRATCH_BYTES bytes.  Every GPU that loads this library holds
// that array until the process exits.  Host code cannot pass the array's
// name to a kernel (on the host it is only a stand-in symbol), so the first
// call on each device looks up its device address with
// cudaGetSymbolAddress while that device is current, and caches it.  Make
// that first call on a device before any stream capture.
//
// Every call shares the one array and it keeps the previous call's
// contents.  Nothing in it has to start at zero: each kernel writes every
// scratch element before any kernel reads it.  Calls whose executions
// overlap on the GPU (different streams, or several host threads without
// ordering) race on the array; issue them on one stream or order them with
// events.
#include <cstdio>
#include <mutex>

#include "gdn_internal.h"

namespace {

constexpr size_t kScratchBytes = (size_t)GDN_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_dev_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
int scratch_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        gdn::set_error_text("gdn_fwd_noalloc: cudaGetDevice failed");
        return GDN_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        gdn::set_error_text("gdn_fwd_noalloc: device ordinal out of range");
        return GDN_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_dev_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            gdn::set_error_text("gdn_fwd_noalloc: cudaGetSymbolAddress of the scratch array failed");
            return GDN_ERR_CUDA;
        }
        g_dev_ptr[dev] = p;
    }
    *out = g_dev_ptr[dev];
    return GDN_OK;
}

}  // namespace

extern "C" int gdn_fwd_noalloc(const void *q, const void *k, const void *v, const float *alpha,
                               const float *beta, const float *S_in, float *S_out, void *o, int B,
                               int H, long long T, int frame_len, int d_k, int d_v,
                               gdn_stream_t stream) {
    try {
        gdn::set_error_text("");  // like every entry point: no stale text after a successful call
        gdn_args a = {};
        a.struct_size = (int)sizeof(gdn_args);
        a.dtype = GDN_DTYPE_BF16;
        a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta;
        a.S_in = S_in; a.S_out = S_out; a.o = o;
        a.B = B; a.H = H; a.T = T; a.frame_len = frame_len; a.d_k = d_k; a.d_v = d_v;
        a.stream = stream;
        gdn::Problem p;
        const int st = gdn::validate_args(a, p);
        if (st != GDN_OK) return st;
        if (B == 0 || H == 0) return GDN_OK;
        cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
        if (T == 0) {  // nothing to scan: the final state is the initial state
            if (S_out && S_out != S_in) {
                const size_t sbytes = (size_t)B * H * d_v * d_k * sizeof(float);
                cudaError_t e = S_in ? cudaMemcpyAsync(S_out, S_in, sbytes, cudaMemcpyDeviceToDevice, s)
                                     : cudaMemsetAsync(S_out, 0, sbytes, s);
                if (e != cudaSuccess) {
                    gdn::set_error_text("gdn_fwd_noalloc: state copy failed");
                    return GDN_ERR_CUDA;
                }
            }
            return GDN_OK;
        }
        const size_t need = gdn::simt_workspace_bytes(p);
        if (need > kScratchBytes) {
            char msg[256];
            snprintf(msg, sizeof(msg),
                     "gdn_fwd_noalloc: this problem needs %zu bytes of scratch; the fixed array holds %zu "
                     "(GDN_NOALLOC_SCRATCH_BYTES); use gdn_fwd or gdn_fwd_ex with a caller workspace",
                     need, kScratchBytes);
            gdn::set_error_text(msg);
            return GDN_ERR_UNSUPPORTED;
        }
        void *ws = nullptr;
        const int st2 = scratch_address(&ws);
        if (st2 != GDN_OK) return st2;
        const cudaError_t e = gdn::launch_simt(p, ws, s, nullptr);
        if (e != cudaSuccess) {
            gdn::set_error_text(cudaGetErrorString(e));
            return GDN_ERR_CUDA;
        }
        return GDN_OK;
    } catch (...) {
        gdn::set_error_text("gdn_fwd_noalloc: internal error");
        return GDN_ERR_CUDA;
    }
}
