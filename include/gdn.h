/*
 * gdn.h -- C ABI of the B200 (sm_100a) chunkwise gated delta rule.
 *
 * The operation (SANA-WM summary, paper-graph-ui, section 3.2
 * "Memory-Efficient Long-Context Modeling", paragraph "Frame-wise Gated
 * DeltaNet (GDN)", the token-wise update; SANA-WM teardown, thesatyajit,
 * section "The linear part: a gated delta rule, one frame per step"), per
 * batch b and head h, over tokens t = 0..T-1:
 *
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = S_t q_t                      (the state AFTER token t's update)
 *
 * S is d_v x d_k and S_0 = S_in (or 0).  The library evaluates it in
 * chunkwise form with one chunk per frame of frame_len tokens (one latent
 * video frame per recurrence step, same paragraph); the result equals the
 * token loop up to rounding.
 *
 * Layouts (all contiguous, row-major; the pages' D x S frame matrices are
 * notation only):
 *   q, k        [B, T, H, d_k]      token-major, as a fused QKV projection emits them
 *   v, o        [B, T, H, d_v]
 *   alpha, beta [B, T, H]  fp32     alpha in [0,1] (linear, not log), beta in [0,1]
 *   S_in, S_out [B, H, d_v, d_k] fp32  (S as the page writes it: o = S q)
 *   frame f covers tokens [f*frame_len, (f+1)*frame_len)
 *
 * Pointers: every tensor pointer is a DEVICE pointer owned by the caller
 * (except gdn_fwd_host, whose tensors are host pointers).  The library keeps
 * no pointer after the call returns.
 *
 * Supported: T % frame_len == 0; 1 <= frame_len <= 4096; d_k, d_v in
 * {16, 32, ..., 128}; every base pointer 16-byte aligned; B*T*H*max(d_k,d_v)
 * < 2^62 and B*H*(T/frame_len) < 2^31.
 *
 * Errors: arguments are validated before anything is enqueued; on a
 * validation error nothing is launched and no output is touched.  A failed
 * launch returns GDN_ERR_CUDA.  Execution is asynchronous on `stream`, so a
 * device-side fault surfaces at the caller's next synchronisation.  No C++
 * exception crosses this ABI.  gdn_last_error() gives a thread-local text
 * for the most recent failure on the calling thread.
 *
 * S_in == NULL means a zero initial state; S_out == NULL means the final
 * state is not stored (repeated denoising passes over one chunk read the
 * same S_in); S_in == S_out is allowed (the state is updated in place).
 * S_in and S_out may not partially overlap, and no output may overlap an
 * input other than that S_in == S_out case.
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ABI-compatible with cudaStream_t / CUstream; NULL = the legacy default stream. */
typedef struct CUstream_st *gdn_stream_t;

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,     /* null required pointer, negative size, bad flag */
    GDN_ERR_SHAPE = 2,           /* T not a multiple of frame_len, size overflow */
    GDN_ERR_UNSUPPORTED = 3,     /* head dim or frame length outside the supported set */
    GDN_ERR_ALIGNMENT = 4,       /* a base pointer is not 16-byte aligned */
    GDN_ERR_NO_MEMORY = 5,       /* workspace allocation failed or caller workspace too small */
    GDN_ERR_CUDA = 6,            /* a CUDA runtime/driver call or a launch failed */
    GDN_ERR_TIMEOUT = 7,         /* a bounded device-side wait gave up */
    GDN_ERR_NONFINITE = 8,       /* finite-check requested and o / S_out holds NaN or Inf */
    GDN_ERR_NOT_IMPLEMENTED = 9  /* a flag combination this build does not provide */
} gdn_status;

enum { GDN_DTYPE_BF16 = 0, GDN_DTYPE_F32 = 1 };

/*
 * gdn_fwd -- forward scan, bf16 q/k/v/o (fp32 alpha, beta and state).
 * Tensor-core path: bf16 products with fp32 accumulation, fp32 gate math and
 * fp32 state.  Returns a gdn_status.
 */
int gdn_fwd(const void *q, const void *k, const void *v,
            const float *alpha, const float *beta,
            const float *S_in, float *S_out, void *o,
            int B, int H, long long T, int frame_len, int d_k, int d_v,
            gdn_stream_t stream);

/* gdn_fwd_f32 -- same operation with fp32 q/k/v/o; fp32 arithmetic
 * throughout with fp64 gate prefix sums (for the tight-tolerance path). */
int gdn_fwd_f32(const float *q, const float *k, const float *v,
                const float *alpha, const float *beta,
                const float *S_in, float *S_out, float *o,
                int B, int H, long long T, int frame_len, int d_k, int d_v,
                gdn_stream_t stream);

/*
 * gdn_step -- one call of a chunk-causal rollout: identical to gdn_fwd but
 * S_in is required (the state carried from the previous call).  Chaining
 * gdn_step calls S_out -> S_in over consecutive token ranges equals one
 * gdn_fwd over their concatenation (SANA-WM summary, section 3.1 "Stage 4:
 * Chunk-Causal Fine-Tuning", the global forward scan that carries past
 * context across chunks).
 */
int gdn_step(const void *q, const void *k, const void *v,
             const float *alpha, const float *beta,
             const float *S_in, float *S_out, void *o,
             int B, int H, long long T, int frame_len, int d_k, int d_v,
             gdn_stream_t stream);

int gdn_step_f32(const float *q, const float *k, const float *v,
                 const float *alpha, const float *beta,
                 const float *S_in, float *S_out, float *o,
                 int B, int H, long long T, int frame_len, int d_k, int d_v,
                 gdn_stream_t stream);

/*
 * gdn_fwd_host -- the whole pass from HOST buffers: the same operation,
 * arguments and layouts as gdn_fwd (dtype = GDN_DTYPE_BF16) or gdn_fwd_f32
 * (GDN_DTYPE_F32), except that q, k, v, alpha, beta, S_in, S_out and o are
 * host pointers (pinned memory gives the fastest copies; pageable works).
 * The call allocates device buffers (stream-ordered, from the library's
 * scratch pool; see gdn_fwd_ex's workspace) on `stream`, copies
 * the inputs in, runs the pass, copies o (and S_out) out, frees the buffers
 * and synchronises `stream` before it returns, so the host outputs are
 * ready.  Host pointers need no alignment.  Errors as gdn_fwd, plus
 * GDN_ERR_NO_MEMORY when the device buffers cannot be allocated; on any
 * error after the copies began, o and S_out may be partly written.
 */
int gdn_fwd_host(int dtype, const void *q, const void *k, const void *v,
                 const float *alpha, const float *beta,
                 const float *S_in, float *S_out, void *o,
                 int B, int H, long long T, int frame_len, int d_k, int d_v,
                 gdn_stream_t stream);

/*
 * gdn_fwd_noalloc -- gdn_fwd for callers that cannot allocate device memory.
 * (The SANA-WM pages have no counterpart: this is a deployment variant.)
 *
 * Some callers may not allocate on the path of a pass: a streaming decode
 * loop whose latency budget cannot take an allocation (cudaMalloc can
 * synchronise the device), a host whose own pool owns all device memory, or
 * code running where allocating is not allowed.  This entry point computes
 * exactly what gdn_fwd computes (bf16 q/k/v/o, fp32 gates and state; same
 * arguments, layouts and errors) on the CUDA-core kernels, with its scratch
 * in one fixed device array of GDN_NOALLOC_SCRATCH_BYTES that every GPU
 * loading the library holds until the process exits.  It calls no
 * allocator.  A problem whose scratch would exceed that size is rejected
 * with GDN_ERR_UNSUPPORTED before anything is launched (at 880-token frames
 * and d_k = d_v = 112 each frame-head needs about 1.33 MB, so up to 50
 * frame-heads fit, e.g. one frame of B = 2, H = 20).
 *
 * The first call on each device looks up the array's device address (with
 * that device current) and caches it: make that first call before any
 * stream capture.  All calls share the array and it keeps the last call's
 * contents (no part needs to start at zero); calls whose executions overlap
 * on the GPU (other streams, or unordered host threads) race on it, so
 * issue them on one stream or order them with events.
 */
#define GDN_NOALLOC_SCRATCH_BYTES (64u << 20)

int gdn_fwd_noalloc(const void *q, const void *k, const void *v,
                    const float *alpha, const float *beta,
                    const float *S_in, float *S_out, void *o,
                    int B, int H, long long T, int frame_len, int d_k, int d_v,
                    gdn_stream_t stream);

/*
 * Extended call.  Fields not listed for a flag are as in gdn_fwd.
 *   struct_size     sizeof(gdn_args) as compiled by the caller (ABI guard).
 *   dtype           GDN_DTYPE_BF16 or GDN_DTYPE_F32 (q/k/v/o element type).
 *   workspace       optional device scratch of workspace_bytes bytes, at
 *                   least gdn_workspace_bytes(...) and 256-byte aligned; NULL
 *                   lets the call take stream-ordered scratch and return it
 *                   before the call returns.  That scratch comes from one
 *                   pool per device owned by the library, which keeps the
 *                   freed memory reserved for later calls (up to the largest
 *                   scratch any call has needed) until the process exits.
 *   reverse         1: reversed-time scan (tokens visited T-1..0, each gate
 *                   applied at its own token; SANA-WM summary, section 3.2,
 *                   paragraph "Bidirectional and Chunk-Causal GDN Variants").
 *   accumulate_o    1: o += result instead of o = result (sums the forward
 *                   and reversed scans of the bidirectional variant).
 *   reset_every     > 0: the state restarts from zero at each boundary of
 *                   reset_every tokens, counted from token 0 (with reverse:
 *                   the chunk-causal reversed scan); a multiple of
 *                   frame_len.  0: no reset.
 *   check_finite    1: after the pass, scan o (and S_out) and return
 *                   GDN_ERR_NONFINITE if any NaN/Inf is found (synchronises
 *                   the stream).
 *   stage_ms        optional HOST array of GDN_NUM_STAGES floats: when set,
 *                   CUDA events bracket each kernel stage on `stream` and the
 *                   call synchronises the stream and writes each stage's
 *                   device time in ms (tracing; off in production calls).
 *   mode            GDN_MODE_TOKEN (0): the token-wise gated delta rule
 *                   above.  GDN_MODE_FRAME (1): the frame-wise operator
 *                   (SANA-WM summary, "Memory-Efficient Long-Context Modeling
 *                   (Section 3.2)", paragraph "Adaptation to video: frame-wise
 *                   recurrence"): one state update per frame t of frame_len
 *                   tokens,
 *                     S_t = S_{t-1} M_t + U_t,  M_t = gamma_t (I - K_t B_t K_t^T),
 *                     U_t = V_t B_t K_t^T,      o = S_t q for every token of t,
 *                   with K_t, V_t the frame's keys and values as columns and
 *                   B_t = diag(beta) over its tokens; alpha is not read (may
 *                   be NULL).  reverse visits the frames backwards; reset_every
 *                   and accumulate_o as above.
 *   gamma           GDN_MODE_FRAME only: device fp32 [B, T / frame_len, H],
 *                   the per-frame decay gamma_t of each head (required there,
 *                   ignored otherwise).
 *   qk_norm         bit mask of the q/k prologue (SANA-WM summary, section
 *                   3.2, paragraph "Algebraic Stabilization for Spatial Token
 *                   Explosion"), applied to the inputs before the operator:
 *                   GDN_QK_NORM_KEYS    k <- ReLU(RMSNorm(k)) / sqrt(d_k * frame_len),
 *                   GDN_QK_NORM_QUERIES q <- ReLU(RMSNorm(q)),
 *                   RMSNorm(x) = x / sqrt(mean over d_k of x^2 + 1e-6) * weight.
 *                   The normalised copies live in the workspace; q and k are
 *                   not modified.  0: the inputs are used as given.
 *   k_norm_weight,  optional device fp32 [d_k] RMSNorm weights of the keys and
 *   q_norm_weight   queries (NULL: ones); read only when their bit is set.
 *   status_dev      optional device int: at the end of the pass (in stream
 *                   order, without synchronising) the library writes 0 there,
 *                   or nonzero when a bounded device-side wait gave up and the
 *                   outputs are not valid (what the synchronous modes report
 *                   as GDN_ERR_TIMEOUT).  4-byte aligned.
 *   phase           GDN_PHASE_ALL (0): the whole pass.  The two halves of a
 *                   pass, for context parallelism over time (SANA-WM summary,
 *                   section 3.1, Stage 3: the sequence split over GPUs; the
 *                   cliffmar.tech article, "NVIDIA SANA-WM", training section:
 *                   "prefix-sum composition of GDN transition matrices"):
 *                   GDN_PHASE_PREPARE (1) runs only the stages that do not
 *                   depend on the entering state (gates, diagonal inverses,
 *                   intra-frame solve, per-frame maps) into `workspace`;
 *                   o, S_in and S_out are not touched.  GDN_PHASE_FINISH (2)
 *                   runs the rest (scan from S_in, pseudo-values, output) from
 *                   the workspace a PREPARE call with the same inputs and
 *                   sizes filled on the same stream.  Both require a caller
 *                   workspace, mode = GDN_MODE_TOKEN and no reverse,
 *                   accumulate_o or qk_norm (else GDN_ERR_NOT_IMPLEMENTED).
 *   segment_map     PREPARE only, optional: device fp32 [B, H, d_k + d_v, d_k]
 *                   (16-byte aligned) that receives the affine map of this
 *                   call's tokens on the state, S_end = S_begin Phi + Psi:
 *                   rows 0 .. d_k-1 hold Phi (d_k x d_k), rows d_k .. hold Psi
 *                   (d_v x d_k), per (b, h).  gdn_apply_maps composes maps.
 */
typedef struct gdn_args {
    int struct_size;
    int dtype;
    const void *q, *k, *v;
    const float *alpha, *beta;
    const float *S_in;
    float *S_out;
    void *o;
    int B, H;
    long long T;
    int frame_len, d_k, d_v;
    void *workspace;
    size_t workspace_bytes;
    int reverse;
    int accumulate_o;
    long long reset_every;
    int check_finite;
    gdn_stream_t stream;
    float *stage_ms;
    int mode;
    const float *gamma;
    int qk_norm;
    const float *k_norm_weight;
    const float *q_norm_weight;
    int *status_dev;
    int phase;
    float *segment_map;
} gdn_args;

enum { GDN_MODE_TOKEN = 0, GDN_MODE_FRAME = 1 };
enum { GDN_PHASE_ALL = 0, GDN_PHASE_PREPARE = 1, GDN_PHASE_FINISH = 2 };
enum { GDN_QK_NORM_KEYS = 1, GDN_QK_NORM_QUERIES = 2 };

/* Kernel stages reported through gdn_args.stage_ms, in launch order:
 * 0 per-frame gate prefix sums, 1 inverses of the 128 x 128 diagonal blocks
 * of the intra-frame system, 2 intra-frame solve, 3 frame transition,
 * 4 scan over frames, 5 pseudo-values U, 6 output.  A path without a stage
 * reports 0 for it: the fp32 path folds 0, 1 into 2 and 5 into 6; the
 * frame-wise operator has only 3 (its per-frame maps), 4 and 6.  Work
 * outside the seven stages is not counted: the q/k prologue pass (where the
 * kernels do not apply it themselves) and a reversed bf16 call's copies of
 * its inputs in reversed token order. */
enum { GDN_NUM_STAGES = 7 };

int gdn_fwd_ex(const gdn_args *a);

/*
 * gdn_apply_maps -- S <- S Phi_j + Psi_j for j = 0 .. n_maps-1 in order, in
 * place: the state entering a segment of a sequence split over ranks, from
 * the state entering the sequence and the segment maps of the segments before
 * it (the exclusive prefix of the maps; same passages as gdn_args.phase).
 *   S     device fp32 [B, H, d_v, d_k], read and written (16-byte aligned)
 *   maps  device fp32 [n_maps][B, H, d_k + d_v, d_k], each as gdn_fwd_ex's
 *         segment_map writes it (16-byte aligned; may not overlap S)
 * Sizes as gdn_fwd (d_k, d_v in {16, ..., 128}); n_maps >= 0.  Asynchronous
 * on `stream`; argument errors return before anything is enqueued.
 */
int gdn_apply_maps(float *S, const float *maps, int n_maps, int B, int H, int d_k, int d_v,
                   gdn_stream_t stream);

/* Device scratch a call with these sizes needs with any flags of gdn_fwd_ex
 * (the size of the largest case, a reversed accumulating call; 0 if the
 * sizes are invalid). */
size_t gdn_workspace_bytes(int B, int H, long long T, int frame_len, int d_k, int d_v, int dtype);

/* Static text for a status code; never NULL. */
const char *gdn_status_string(int status);

/* Thread-local detail of the last failure on this thread ("" if none). */
const char *gdn_last_error(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH.  The gdn_args layout
 * belongs to the version: 0.2.0 added mode, gamma, qk_norm, the RMSNorm
 * weights and status_dev; 0.3.0 added phase and segment_map (struct_size
 * guards a caller built against another layout). */
#define GDN_VERSION 300
int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
