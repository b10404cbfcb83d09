"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, its argument struct matches the header, and argument validation
returns the documented status before anything is enqueued.  The pointers
below are never dereferenced: every call is rejected by validation first.
"""
import ctypes
import os
import re

import pytest

import gated_deltanet_linear_chunkwise_b200 as g
from gated_deltanet_linear_chunkwise_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")

FAKE = 1 << 40  # aligned, never dereferenced (validation rejects first)


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_\w+)\s*\(", src)))


def test_header_declarations_all_exported():
    lib = g.load_library()
    declared = _declared()
    assert set(binding.EXPORTS) <= set(declared)
    for name in declared:
        assert hasattr(lib, name), name


def test_exports_via_nm():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    syms = {l.split()[-1] for l in out.splitlines() if " T " in l}
    for name in _declared():
        assert name in syms, name


def test_struct_size_matches_header():
    # the library rejects a struct whose size differs from its own
    a = binding.GdnArgs()
    a.struct_size = ctypes.sizeof(binding.GdnArgs) + 8
    rc = g.load_library().gdn_fwd_ex(ctypes.byref(a))
    assert rc == 1 and "struct_size" in g.last_error()
    assert ctypes.sizeof(binding.GdnArgs) == 224  # LP64 layout of gdn_args


def _ex_args(**kw):
    a = binding.GdnArgs()
    a.struct_size = ctypes.sizeof(binding.GdnArgs)
    a.q, a.k, a.v, a.alpha, a.beta, a.o = FAKE, FAKE + 1024, FAKE + 2048, FAKE + 4096, FAKE + 8192, FAKE + 16384
    a.B, a.H, a.T, a.frame_len, a.d_k, a.d_v = 1, 2, 128, 64, 64, 64
    for key, val in kw.items():
        setattr(a, key, val)
    return a


@pytest.mark.parametrize("kw,status,text", [
    (dict(mode=2), 1, "mode"),                        # neither operator
    (dict(mode=1), 1, "gamma"),                       # frame-wise operator without its decay
    (dict(alpha=None), 1, "alpha"),                   # token-wise operator without alpha
    (dict(mode=1, alpha=None, gamma=FAKE + 16384 + 8), 1, "overlaps"),  # o over gamma
    (dict(qk_norm=4), 1, "qk_norm"),                  # not a mask of the two prologue bits
    (dict(qk_norm=-1), 1, "qk_norm"),
    (dict(status_dev=FAKE + 2), 4, "status_dev"),     # not 4-byte aligned
    (dict(phase=3), 1, "phase"),                      # no such phase
    (dict(phase=1), 1, "workspace"),                  # the phases keep their state in a caller workspace
    (dict(phase=2, workspace=FAKE + (1 << 30), workspace_bytes=1 << 30, reverse=1), 9, "reverse"),
    (dict(phase=1, workspace=FAKE + (1 << 30), workspace_bytes=1 << 30, mode=1, alpha=None,
          gamma=FAKE + (1 << 29)), 9, "token-wise"),
    (dict(segment_map=FAKE + (1 << 29)), 1, "segment_map"),                  # only a PREPARE call writes it
    (dict(phase=1, workspace=FAKE + (1 << 30), workspace_bytes=1 << 30,
          segment_map=FAKE + (1 << 29) + 4), 4, "segment_map"),              # misaligned
    (dict(phase=1, workspace=FAKE + (1 << 30), workspace_bytes=1 << 30, segment_map=FAKE), 1, "overlaps"),
])
def test_mode_validation(kw, status, text):
    # rejected before any device work (no GPU needed)
    rc = g.load_library().gdn_fwd_ex(ctypes.byref(_ex_args(**kw)))
    assert rc == status and text in g.last_error()


def test_stage_count_matches_header():
    src = open(HEADER).read()
    m = re.search(r"GDN_NUM_STAGES\s*=\s*(\d+)", src)
    assert m and int(m.group(1)) == binding.NUM_STAGES == len(binding.STAGES)


def _call(fn="gdn_fwd", q=FAKE, k=FAKE + 1024, v=FAKE + 2048, alpha=FAKE + 4096, beta=FAKE + 8192,
          S_in=None, S_out=None, o=FAKE + 16384, B=1, H=2, T=128, L=64, dk=64, dv=64):
    lib = g.load_library()
    return getattr(lib, fn)(q, k, v, alpha, beta, S_in, S_out, o, B, H, T, L, dk, dv, None)


@pytest.mark.parametrize("kw,status", [
    (dict(T=100, L=64), 2),                # T not a multiple of frame_len
    (dict(L=0), 1),                        # frame_len must be positive
    (dict(B=-1), 1),
    (dict(dk=120), 3), (dict(dv=136), 3), (dict(dk=8), 3),
    (dict(L=8192, T=8192), 3),             # frame_len above 4096
    (dict(q=None), 1), (dict(o=None), 1), (dict(alpha=None), 1),
    (dict(k=FAKE + 8), 4), (dict(S_in=FAKE + 3), 4),
    (dict(B=1 << 20, H=1 << 10, T=1 << 30, L=1 << 10), 2),   # index overflow
])
def test_validation_errors(kw, status):
    assert _call(**kw) == status
    assert g.last_error() != ""


def test_apply_maps_validation():
    lib = g.load_library()
    assert lib.gdn_apply_maps(FAKE, FAKE + (1 << 30), 1, 1, 2, 120, 64, None) == 3   # head dim
    assert lib.gdn_apply_maps(FAKE + 4, FAKE + (1 << 30), 1, 1, 2, 64, 64, None) == 4  # alignment
    assert lib.gdn_apply_maps(None, FAKE, 1, 1, 2, 64, 64, None) == 1                 # NULL state
    assert lib.gdn_apply_maps(FAKE, FAKE + 1024, 1, 1, 2, 64, 64, None) == 1          # overlap
    assert "overlaps" in g.last_error()
    assert lib.gdn_apply_maps(FAKE, FAKE + (1 << 30), -1, 1, 2, 64, 64, None) == 1    # negative count
    assert lib.gdn_apply_maps(None, None, 0, 1, 2, 64, 64, None) == 0                 # nothing to apply
    assert g.last_error() == ""


def test_overlap_rejected():
    # o aliasing q
    assert _call(o=FAKE) == 1 and "overlaps" in g.last_error()


def test_step_requires_state():
    assert _call(fn="gdn_step") == 1
    assert _call(fn="gdn_step_f32") == 1


def test_status_strings():
    lib = g.load_library()
    for code, name in binding.STATUS.items():
        assert lib.gdn_status_string(code).decode() == name
    assert lib.gdn_status_string(99).decode() == "GDN_ERR_UNKNOWN"


def test_workspace_bytes():
    assert g.workspace_bytes(1, 20, 106480, 880, 112, 112) > 0
    assert g.workspace_bytes(1, 20, 100, 880, 112, 112) == 0      # invalid shape
    assert g.workspace_bytes(0, 20, 880, 880, 112, 112) == 0      # empty
    # grows with the batch
    assert g.workspace_bytes(2, 4, 880, 880, 64, 64) > g.workspace_bytes(1, 4, 880, 880, 64, 64)


def test_python_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 64, 1, 16)
    with pytest.raises(g.GdnError):
        g.gdn_fwd(x, x, x, torch.zeros(1, 64, 1), torch.zeros(1, 64, 1), 64)


@pytest.mark.parametrize("kw,status", [
    (dict(T=100, L=64), 2), (dict(L=0), 1), (dict(dk=120), 3), (dict(q=None), 1), (dict(o=None), 1),
])
def test_host_entry_validates_before_touching_the_gpu(kw, status):
    # gdn_fwd_host takes host pointers: its size checks run before any CUDA call
    args = dict(q=FAKE, k=FAKE + 1024, v=FAKE + 2048, alpha=FAKE + 4096, beta=FAKE + 8192, S_in=None,
                S_out=None, o=FAKE + 16384, B=1, H=2, T=128, L=64, dk=64, dv=64)
    args.update(kw)
    lib = g.load_library()
    rc = lib.gdn_fwd_host(binding.GDN_DTYPE_BF16, args["q"], args["k"], args["v"], args["alpha"], args["beta"],
                          args["S_in"], args["S_out"], args["o"], args["B"], args["H"], args["T"], args["L"],
                          args["dk"], args["dv"], None)
    assert rc == status, g.last_error()
    assert g.last_error()


def test_host_binding_rejects_device_tensors_by_type():
    import torch
    x = torch.zeros(1, 64, 1, 16, dtype=torch.float16)
    with pytest.raises(g.GdnError):
        g.gdn_fwd_host(x, x, x, torch.zeros(1, 64, 1), torch.zeros(1, 64, 1), 64)


def test_python_binding_frame_mode_checks():
    import torch
    x = torch.zeros(1, 64, 1, 16)
    a = torch.zeros(1, 64, 1)
    with pytest.raises(g.GdnError, match="mode"):
        g.gdn_fwd(x, x, x, a, a, 64, mode="frames")
    with pytest.raises(g.GdnError, match="gamma is required"):
        g.gdn_fwd(x, x, x, None, a, 64, mode="frame")
    with pytest.raises(g.GdnError, match="alpha is required"):
        g.gdn_fwd(x, x, x, None, a, 64)


def test_workspace_bytes_covers_every_flag():
    # the public size is the largest case: it grows with neither flag, and a forward-only
    # problem of the same sizes needs no more
    from gated_deltanet_linear_chunkwise_b200 import binding as b
    lib = g.load_library()
    full = lib.gdn_workspace_bytes(1, 20, 880 * 4, 880, 112, 112, b.GDN_DTYPE_BF16)
    smaller = lib.gdn_workspace_bytes(1, 20, 880 * 3, 880, 112, 112, b.GDN_DTYPE_BF16)
    assert full > smaller > 0
    # bf16 q, k, v, o and the two prologue copies all fit: at least 5 token-major bf16 tensors
    assert full >= 5 * 2 * 880 * 4 * 20 * 112


def test_version_matches_header():
    m = re.search(r"#define\s+GDN_VERSION\s+(\d+)", open(HEADER).read())
    assert m and g.load_library().gdn_version() == int(m.group(1))
