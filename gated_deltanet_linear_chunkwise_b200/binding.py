"""Thin ctypes binding of ``libgdn_b200.so`` (argument marshalling only).

Every step of the computation runs in the library's CUDA kernels; torch is
used here only to allocate device tensors and to name the current stream.
There is no CPU fallback: if the library is missing the call raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgdn_b200.so")

GDN_DTYPE_BF16 = 0
GDN_DTYPE_F32 = 1

STATUS = {
    0: "GDN_OK", 1: "GDN_ERR_INVALID_ARG", 2: "GDN_ERR_SHAPE", 3: "GDN_ERR_UNSUPPORTED",
    4: "GDN_ERR_ALIGNMENT", 5: "GDN_ERR_NO_MEMORY", 6: "GDN_ERR_CUDA", 7: "GDN_ERR_TIMEOUT",
    8: "GDN_ERR_NONFINITE", 9: "GDN_ERR_NOT_IMPLEMENTED",
}

# every symbol include/gdn.h declares
EXPORTS = ("gdn_fwd", "gdn_fwd_f32", "gdn_step", "gdn_step_f32", "gdn_fwd_ex", "gdn_fwd_host",
           "gdn_apply_maps", "gdn_workspace_bytes", "gdn_status_string", "gdn_last_error", "gdn_version")


class GdnError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        self.name = STATUS.get(status, "GDN_ERR_UNKNOWN")
        super().__init__("%s: %s" % (self.name, detail))


class GdnArgs(ctypes.Structure):
    """Mirror of ``gdn_args`` in include/gdn.h (same field order and types)."""
    _fields_ = [
        ("struct_size", ctypes.c_int), ("dtype", ctypes.c_int),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("alpha", ctypes.c_void_p), ("beta", ctypes.c_void_p),
        ("S_in", ctypes.c_void_p), ("S_out", ctypes.c_void_p), ("o", ctypes.c_void_p),
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_longlong),
        ("frame_len", ctypes.c_int), ("d_k", ctypes.c_int), ("d_v", ctypes.c_int),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("reverse", ctypes.c_int), ("accumulate_o", ctypes.c_int),
        ("reset_every", ctypes.c_longlong), ("check_finite", ctypes.c_int),
        ("stream", ctypes.c_void_p), ("stage_ms", ctypes.c_void_p),
        ("mode", ctypes.c_int), ("gamma", ctypes.c_void_p),
        ("qk_norm", ctypes.c_int), ("k_norm_weight", ctypes.c_void_p), ("q_norm_weight", ctypes.c_void_p),
        ("status_dev", ctypes.c_void_p),
        ("phase", ctypes.c_int), ("segment_map", ctypes.c_void_p),
    ]

GDN_MODE_TOKEN = 0
GDN_MODE_FRAME = 1
GDN_QK_NORM_KEYS = 1
GDN_QK_NORM_QUERIES = 2
PHASES = {"all": 0, "prepare": 1, "finish": 2}

NUM_STAGES = 7
STAGES = ("gates", "diag_inverse", "intra", "transition", "scan", "u", "output")


_lib = None


def load_library(path: str = LIB_PATH):
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("CUDA library %s is missing; build it with "
                           "`python -m gated_deltanet_linear_chunkwise_b200.build`" % path)
    lib = ctypes.CDLL(path)
    V, I, LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong
    fwd_sig = [V, V, V, V, V, V, V, V, I, I, LL, I, I, I, V]
    for name in ("gdn_fwd", "gdn_fwd_f32", "gdn_step", "gdn_step_f32"):
        fn = getattr(lib, name)
        fn.argtypes = fwd_sig
        fn.restype = I
    lib.gdn_fwd_host.argtypes = [I] + fwd_sig
    lib.gdn_fwd_host.restype = I
    lib.gdn_fwd_ex.argtypes = [ctypes.POINTER(GdnArgs)]
    lib.gdn_fwd_ex.restype = I
    lib.gdn_apply_maps.argtypes = [V, V, I, I, I, I, I, V]
    lib.gdn_apply_maps.restype = I
    lib.gdn_workspace_bytes.argtypes = [I, I, LL, I, I, I, I]
    lib.gdn_workspace_bytes.restype = ctypes.c_size_t
    lib.gdn_status_string.argtypes = [I]
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_last_error.argtypes = []
    lib.gdn_last_error.restype = ctypes.c_char_p
    lib.gdn_version.argtypes = []
    lib.gdn_version.restype = I
    _lib = lib
    return lib


def last_error() -> str:
    return load_library().gdn_last_error().decode()


def check(status: int):
    if status != 0:
        raise GdnError(status, last_error())


def workspace_bytes(B, H, T, frame_len, d_k, d_v, dtype="bf16") -> int:
    dt = GDN_DTYPE_BF16 if dtype in ("bf16", GDN_DTYPE_BF16) else GDN_DTYPE_F32
    return int(load_library().gdn_workspace_bytes(B, H, T, frame_len, d_k, d_v, dt))


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream_handle(stream, device):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def gdn_fwd(q, k, v, alpha, beta, frame_len, S_in=None, *, S_out=None, o=None,
            return_state=False, reverse=False, accumulate=False, reset_every=0,
            check_finite=False, workspace=None, stream=None, stage_ms=None, mode="token", gamma=None,
            norm_keys=False, norm_queries=False, k_norm_weight=None, q_norm_weight=None, status=None,
            phase="all", segment_map=None):
    """Chunkwise gated delta rule forward on CUDA tensors.

    q,k [B,T,H,d_k], v [B,T,H,d_v] (bf16 or fp32, all the same), alpha/beta
    [B,T,H] fp32, S_in [B,H,d_v,d_k] fp32 or None.  ``o`` and ``S_out`` may be
    given (written in place; ``o`` is accumulated into when ``accumulate``);
    with ``return_state`` and no ``S_out`` a state tensor is allocated.
    ``stage_ms`` (a ``(ctypes.c_float * NUM_STAGES)()``) receives each kernel
    stage's device time; that call synchronises the stream.
    ``mode="frame"`` runs the frame-wise operator instead (one state update
    per frame of ``frame_len`` tokens); it reads ``gamma`` [B, T/frame_len, H]
    fp32, the per-frame decay, and not ``alpha`` (which may be None).
    ``norm_keys`` / ``norm_queries`` apply the q/k prologue first: keys
    ReLU(RMSNorm(k)) / sqrt(d_k * frame_len), queries ReLU(RMSNorm(q)), with
    optional fp32 [d_k] RMSNorm weights.
    ``status`` (a CUDA int32 tensor of one element) receives, in stream order,
    0 or a nonzero code when a bounded device-side wait gave up.
    ``phase="prepare"`` runs only the stages that do not depend on the entering
    state into ``workspace`` (required), and with ``segment_map`` (fp32
    [B, H, d_k + d_v, d_k]) also writes the call's map S_end = S_begin Phi + Psi;
    ``phase="finish"`` then runs the rest from ``S_in`` on the same workspace.
    Returns (o, S_out or None) (o is None for a prepare call).
    """
    import torch
    B, T, H, d_k = q.shape
    d_v = v.shape[-1]
    if mode not in ("token", "frame"):
        raise GdnError(1, "mode must be 'token' or 'frame'")
    frame = mode == "frame"
    gates = (("beta", beta), ("gamma", gamma)) if frame else (("alpha", alpha), ("beta", beta))
    for name, t in (("q", q), ("k", k), ("v", v)) + gates:
        if t is None:
            raise GdnError(1, "%s is required" % name)
    for name, t in (("q", q), ("k", k), ("v", v)) + gates:
        if not t.is_cuda:
            raise GdnError(1, "%s is not a CUDA tensor" % name)
        if not t.is_contiguous():
            raise GdnError(1, "%s is not contiguous" % name)
    if q.dtype != k.dtype or q.dtype != v.dtype or q.dtype not in (torch.bfloat16, torch.float32):
        raise GdnError(1, "q/k/v must share one dtype, bf16 or fp32")
    if any(t.dtype != torch.float32 for _, t in gates):
        raise GdnError(1, "%s must be fp32" % " and ".join(n for n, _ in gates))
    if frame and tuple(gamma.shape) != (B, T // max(int(frame_len), 1), H):
        raise GdnError(2, "gamma must have shape [B, T / frame_len, H]")
    for name, wt, on in (("k_norm_weight", k_norm_weight, norm_keys), ("q_norm_weight", q_norm_weight, norm_queries)):
        if wt is not None and on and (not wt.is_cuda or not wt.is_contiguous() or wt.dtype != torch.float32
                                      or wt.numel() != d_k):
            raise GdnError(1, "%s must be a contiguous fp32 CUDA tensor of d_k entries" % name)
    for name, t in (("S_in", S_in), ("S_out", S_out), ("o", o)):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise GdnError(1, "%s must be a contiguous CUDA tensor" % name)
    if phase not in PHASES:
        raise GdnError(1, "phase must be 'all', 'prepare' or 'finish'")
    prepare = phase == "prepare"
    if segment_map is not None and (not segment_map.is_cuda or not segment_map.is_contiguous()
                                    or segment_map.dtype != torch.float32
                                    or tuple(segment_map.shape) != (B, H, d_k + d_v, d_k)):
        raise GdnError(1, "segment_map must be a contiguous fp32 CUDA tensor [B, H, d_k + d_v, d_k]")
    if o is None and not prepare:
        o = (torch.zeros if accumulate else torch.empty)((B, T, H, d_v), dtype=q.dtype, device=q.device)
    if S_out is None and return_state and not prepare:
        S_out = torch.empty((B, H, d_v, d_k), dtype=torch.float32, device=q.device)
    a = GdnArgs()
    a.phase = PHASES[phase]
    a.segment_map = _ptr(segment_map)
    a.struct_size = ctypes.sizeof(GdnArgs)
    a.dtype = GDN_DTYPE_BF16 if q.dtype == torch.bfloat16 else GDN_DTYPE_F32
    a.q, a.k, a.v = _ptr(q), _ptr(k), _ptr(v)
    a.alpha, a.beta = (None if frame else _ptr(alpha)), _ptr(beta)
    a.S_in, a.S_out, a.o = _ptr(S_in), _ptr(S_out), _ptr(o)
    a.mode = GDN_MODE_FRAME if frame else GDN_MODE_TOKEN
    a.gamma = _ptr(gamma) if frame else None
    if status is not None and (not status.is_cuda or status.dtype != torch.int32 or status.numel() < 1):
        raise GdnError(1, "status must be a CUDA int32 tensor")
    a.status_dev = _ptr(status)
    a.qk_norm = (GDN_QK_NORM_KEYS if norm_keys else 0) | (GDN_QK_NORM_QUERIES if norm_queries else 0)
    a.k_norm_weight = _ptr(k_norm_weight) if norm_keys else None
    a.q_norm_weight = _ptr(q_norm_weight) if norm_queries else None
    a.B, a.H, a.T = B, H, T
    a.frame_len, a.d_k, a.d_v = int(frame_len), d_k, d_v
    if workspace is not None:
        a.workspace = workspace.data_ptr()
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    a.reverse, a.accumulate_o = int(bool(reverse)), int(bool(accumulate))
    a.reset_every, a.check_finite = int(reset_every), int(bool(check_finite))
    a.stream = _stream_handle(stream, q.device)
    if stage_ms is not None:  # a ctypes float array of NUM_STAGES; the call synchronises
        a.stage_ms = ctypes.cast(stage_ms, ctypes.c_void_p)
    check(load_library().gdn_fwd_ex(ctypes.byref(a)))
    return o, S_out


def apply_maps(S, maps, *, stream=None):
    """S <- S Phi_j + Psi_j for each segment map in order, in place (``gdn_apply_maps``):
    S fp32 [B, H, d_v, d_k], maps fp32 [n, B, H, d_k + d_v, d_k] (CUDA, contiguous).
    Returns S."""
    import torch
    B, H, d_v, d_k = S.shape
    for name, t in (("S", S), ("maps", maps)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != torch.float32:
            raise GdnError(1, "%s must be a contiguous fp32 CUDA tensor" % name)
    if maps.dim() != 5 or tuple(maps.shape[1:]) != (B, H, d_k + d_v, d_k):
        raise GdnError(2, "maps must have shape [n, B, H, d_k + d_v, d_k]")
    check(load_library().gdn_apply_maps(_ptr(S), _ptr(maps), maps.shape[0], B, H, d_k, d_v,
                                        _stream_handle(stream, S.device)))
    return S


def gdn_fwd_host(q, k, v, alpha, beta, frame_len, S_in=None, *, S_out=None, o=None,
                 return_state=False, stream=None, device=None):
    """The whole pass from HOST (CPU) tensors through ``gdn_fwd_host``: the
    library copies the inputs to the GPU, runs the pass, copies o (and the
    state) back and synchronises.  Pinned tensors copy fastest.  Same shapes
    and dtypes as ``gdn_fwd``; returns (o, S_out or None) on the host."""
    import torch
    B, T, H, d_k = q.shape
    d_v = v.shape[-1]
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta), ("S_in", S_in),
                    ("S_out", S_out), ("o", o)):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise GdnError(1, "%s must be a contiguous host tensor" % name)
    if q.dtype != k.dtype or q.dtype != v.dtype or q.dtype not in (torch.bfloat16, torch.float32):
        raise GdnError(1, "q/k/v must share one dtype, bf16 or fp32")
    if alpha.dtype != torch.float32 or beta.dtype != torch.float32:
        raise GdnError(1, "alpha and beta must be fp32")
    if o is None:
        o = torch.empty((B, T, H, d_v), dtype=q.dtype)
    if S_out is None and return_state:
        S_out = torch.empty((B, H, d_v, d_k), dtype=torch.float32)
    dt = GDN_DTYPE_BF16 if q.dtype == torch.bfloat16 else GDN_DTYPE_F32
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    check(load_library().gdn_fwd_host(dt, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S_in),
                                      _ptr(S_out), _ptr(o), B, H, T, int(frame_len), d_k, d_v,
                                      _stream_handle(stream, device)))
    return o, S_out


def gdn_step(q, k, v, alpha, beta, frame_len, S_in, *, S_out=None, o=None, workspace=None,
             stream=None):
    """One chunk-causal rollout call: S_in is required; returns (o, S_out).
    ``S_out`` may be ``S_in`` itself (in-place state update)."""
    if S_in is None:
        raise GdnError(1, "gdn_step requires S_in")
    return gdn_fwd(q, k, v, alpha, beta, frame_len, S_in, S_out=S_out, o=o, return_state=True,
                   workspace=workspace, stream=stream)


def bidirectional(q, k, v, alpha, beta, frame_len, *, chunk_len=0, S_in=None, stream=None):
    """Forward scan plus reversed-time scan, outputs summed; ``chunk_len`` > 0
    restarts the reversed scan at every chunk boundary (chunk-causal form).
    Returns (o, S_out of the forward scan)."""
    o, S = gdn_fwd(q, k, v, alpha, beta, frame_len, S_in, return_state=True, stream=stream)
    gdn_fwd(q, k, v, alpha, beta, frame_len, None, o=o, reverse=True, accumulate=True,
            reset_every=chunk_len, stream=stream)
    return o, S
