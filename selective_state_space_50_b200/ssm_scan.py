"""Python binding of libssmscan.so (the C ABI in include/ssm_scan.h).

Argument marshalling only: torch provides device memory and the current CUDA
stream; every step of the scan runs in the library's kernels.  There is no
fallback implementation: if the shared library is missing or cannot be
loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# SSM_LIB_PATH selects another build of the library (e.g. one compiled with
# different tuning macros); the default is the in-tree build.
LIB_PATH = os.environ.get("SSM_LIB_PATH") or os.path.join(_HERE, "libssmscan.so")

SSM_OK, SSM_ERR_INVALID_ARG, SSM_ERR_UNSUPPORTED, SSM_ERR_CUDA, SSM_ERR_TIMEOUT = range(5)
SSM_F32, SSM_BF16 = 0, 1
CKPT_CHUNK = 8  # SSM_CKPT_CHUNK in include/ssm_scan.h

EXPORTS = ("ssm_version", "ssm_last_error_string", "ssm_last_kernel_path",
           "ssm_selective_scan_ckpt_bytes",
           "ssm_selective_scan_fwd", "ssm_selective_scan_bwd_scratch_bytes",
           "ssm_selective_scan_bwd", "ssm_device_error_status",
           "ssm_selective_scan_bwd_noalloc", "ssm_selective_state_update",
           "ssm_selective_scan_fwd_ex", "ssm_selective_scan_bwd_ex",
           "ssm_selective_state_update_ex", "ssm_selftest_wait_timeout",
           "ssm_selection_projections", "ssm_selective_scan_fwd_segment",
           "ssm_scan_combine_carries", "ssm_selective_scan_fwd_workspace_bytes",
           "ssm_selective_scan_fwd_ws", "ssm_selective_scan_workspace_size",
           "ssm_check_device_errors")
SSM_DISC_DELTA_B, SSM_DISC_ZOH = 0, 1
NOALLOC_SCRATCH_BYTES = 32 << 20  # SSM_NOALLOC_SCRATCH_BYTES in include/ssm_scan.h


class SSMError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"ssm status {status}: {msg}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("dim", ctypes.c_int), ("seqlen", ctypes.c_int),
                ("dstate", ctypes.c_int), ("io_dtype", ctypes.c_int)]


class Options(ctypes.Structure):
    _fields_ = [("delta_softplus", ctypes.c_int), ("discretization", ctypes.c_int)]


def _opts(delta_softplus: bool, zoh: bool) -> Options:
    return Options(int(bool(delta_softplus)), SSM_DISC_ZOH if zoh else SSM_DISC_DELTA_B)


_lib = None


def load_library(path: str = LIB_PATH):
    """Loads the library (once) and declares the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m selective_state_space_50_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sp = ctypes.POINTER(Shape)
    lib.ssm_version.restype = i
    lib.ssm_last_error_string.restype = ctypes.c_char_p
    lib.ssm_last_kernel_path.restype = ctypes.c_char_p
    lib.ssm_selective_scan_ckpt_bytes.argtypes = [sp, ctypes.POINTER(sz)]
    lib.ssm_selective_scan_ckpt_bytes.restype = i
    lib.ssm_selective_scan_bwd_scratch_bytes.argtypes = [sp, i, ctypes.POINTER(sz)]
    lib.ssm_selective_scan_bwd_scratch_bytes.restype = i
    lib.ssm_selective_scan_fwd.argtypes = [sp] + [vp] * 8 + [i] + [vp] * 4
    lib.ssm_selective_scan_fwd.restype = i
    lib.ssm_selective_scan_bwd.argtypes = [sp] + [vp] * 8 + [i] + [vp] * 11 + [sz, vp]
    lib.ssm_selective_scan_bwd.restype = i
    lib.ssm_device_error_status.argtypes = [vp]
    lib.ssm_device_error_status.restype = i
    lib.ssm_selective_scan_workspace_size.argtypes = [sp, ctypes.POINTER(sz)]
    lib.ssm_selective_scan_workspace_size.restype = i
    lib.ssm_check_device_errors.argtypes = [vp]
    lib.ssm_check_device_errors.restype = i
    lib.ssm_selective_scan_bwd_noalloc.argtypes = [sp] + [vp] * 8 + [i] + [vp] * 10
    lib.ssm_selective_scan_bwd_noalloc.restype = i
    lib.ssm_selective_state_update.argtypes = [sp] + [vp] * 9 + [i] + [vp] * 2
    lib.ssm_selective_state_update.restype = i
    op = ctypes.POINTER(Options)
    lib.ssm_selective_scan_fwd_ex.argtypes = [sp, op] + [vp] * 12
    lib.ssm_selective_scan_fwd_ex.restype = i
    lib.ssm_selective_scan_fwd_workspace_bytes.argtypes = [sp, op, ctypes.POINTER(sz)]
    lib.ssm_selective_scan_fwd_workspace_bytes.restype = i
    lib.ssm_selective_scan_fwd_ws.argtypes = [sp, op] + [vp] * 12 + [sz, vp]
    lib.ssm_selective_scan_fwd_ws.restype = i
    lib.ssm_selective_scan_bwd_ex.argtypes = [sp, op] + [vp] * 19 + [sz, vp]
    lib.ssm_selective_scan_bwd_ex.restype = i
    lib.ssm_selective_state_update_ex.argtypes = [sp, op] + [vp] * 11
    lib.ssm_selective_state_update_ex.restype = i
    lib.ssm_selftest_wait_timeout.argtypes = [vp]
    lib.ssm_selftest_wait_timeout.restype = i
    lib.ssm_selection_projections.argtypes = [sp, i] + [vp] * 8
    lib.ssm_selection_projections.restype = i
    lib.ssm_selective_scan_fwd_segment.argtypes = [sp, op] + [vp] * 14
    lib.ssm_selective_scan_fwd_segment.restype = i
    lib.ssm_scan_combine_carries.argtypes = [i, i, i, i] + [vp] * 5 + [vp]
    lib.ssm_scan_combine_carries.restype = i
    _lib = lib
    return lib


def last_error() -> str:
    return load_library().ssm_last_error_string().decode()


def last_kernel_path() -> str:
    """Which kernels the last forward or backward call on this thread used
    ("fwd:tma", "fwd:general", "fwd:chunked", "bwd:tma", "bwd:general")."""
    return load_library().ssm_last_kernel_path().decode()


def device_error_status(stream=None):
    """Synchronises the stream and raises SSMError if a kernel's bounded wait gave up."""
    _check(load_library().ssm_device_error_status(_stream_ptr(stream)))


def _check(status: int):
    if status != SSM_OK:
        raise SSMError(status, last_error())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def make_shape(batch, dim, seqlen, dstate, io_dtype) -> Shape:
    if isinstance(io_dtype, torch.dtype):
        io_dtype = {torch.float32: SSM_F32, torch.bfloat16: SSM_BF16}[io_dtype]
    return Shape(batch, dim, seqlen, dstate, io_dtype)


def ckpt_numel(shape: Shape) -> int:
    n = ctypes.c_size_t()
    _check(load_library().ssm_selective_scan_ckpt_bytes(ctypes.byref(shape), ctypes.byref(n)))
    return n.value // 4


def bwd_scratch_bytes(shape: Shape, have_ckpt: bool) -> int:
    n = ctypes.c_size_t()
    _check(load_library().ssm_selective_scan_bwd_scratch_bytes(ctypes.byref(shape),
                                                               int(bool(have_ckpt)),
                                                               ctypes.byref(n)))
    return n.value


def _shape_of(u: torch.Tensor, A: torch.Tensor) -> Shape:
    if u.dim() != 3 or A.dim() != 2:
        raise ValueError("u must be [batch, dim, seqlen] and A [dim, dstate]")
    return make_shape(u.shape[0], u.shape[1], u.shape[2], A.shape[1], u.dtype)


def fwd_workspace_bytes(shape: Shape, delta_softplus: bool = True, zoh: bool = False) -> int:
    """Workspace bytes of ssm_selective_scan_fwd_ws for this shape on the
    current device (0: the one-pass forward, no workspace needed)."""
    n = ctypes.c_size_t()
    o = _opts(delta_softplus, zoh)
    _check(load_library().ssm_selective_scan_fwd_workspace_bytes(ctypes.byref(shape), ctypes.byref(o),
                                                                 ctypes.byref(n)))
    return int(n.value)


def fwd_raw(shape: Shape, u, delta, A, B, C, D, z, delta_bias, delta_softplus: bool,
            out, last_state, ckpt, stream=None, zoh: bool = False, workspace=None):
    """Direct C-ABI call on raw tensors (no checks beyond the library's own).
    zoh selects the zero-order-hold B̄ (ssm_selective_scan_fwd_ex); a
    workspace tensor selects ssm_selective_scan_fwd_ws (the two-level scan
    along the sequence where the shape calls for it)."""
    if workspace is not None:
        o = _opts(delta_softplus, zoh)
        _check(load_library().ssm_selective_scan_fwd_ws(
            ctypes.byref(shape), ctypes.byref(o), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
            _ptr(D), _ptr(z), _ptr(delta_bias), _ptr(out), _ptr(last_state), _ptr(ckpt),
            _ptr(workspace), workspace.numel() * workspace.element_size(), _stream_ptr(stream)))
        return
    if zoh:
        o = _opts(delta_softplus, True)
        _check(load_library().ssm_selective_scan_fwd_ex(
            ctypes.byref(shape), ctypes.byref(o), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
            _ptr(D), _ptr(z), _ptr(delta_bias), _ptr(out), _ptr(last_state), _ptr(ckpt),
            _stream_ptr(stream)))
        return
    _check(load_library().ssm_selective_scan_fwd(
        ctypes.byref(shape), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(delta_bias), int(bool(delta_softplus)), _ptr(out), _ptr(last_state), _ptr(ckpt),
        _stream_ptr(stream)))


def bwd_raw(shape: Shape, u, delta, A, B, C, D, z, delta_bias, delta_softplus: bool, dout,
            ckpt, du, ddelta, dA, dB, dC, dD, dz, ddelta_bias, scratch, stream=None,
            zoh: bool = False):
    nbytes = 0 if scratch is None else scratch.numel() * scratch.element_size()
    if zoh:
        o = _opts(delta_softplus, True)
        _check(load_library().ssm_selective_scan_bwd_ex(
            ctypes.byref(shape), ctypes.byref(o), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
            _ptr(D), _ptr(z), _ptr(delta_bias), _ptr(dout), _ptr(ckpt), _ptr(du), _ptr(ddelta),
            _ptr(dA), _ptr(dB), _ptr(dC), _ptr(dD), _ptr(dz), _ptr(ddelta_bias), _ptr(scratch),
            ctypes.c_size_t(nbytes), _stream_ptr(stream)))
        return
    _check(load_library().ssm_selective_scan_bwd(
        ctypes.byref(shape), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(delta_bias), int(bool(delta_softplus)), _ptr(dout), _ptr(ckpt), _ptr(du),
        _ptr(ddelta), _ptr(dA), _ptr(dB), _ptr(dC), _ptr(dD), _ptr(dz), _ptr(ddelta_bias),
        _ptr(scratch), ctypes.c_size_t(nbytes), _stream_ptr(stream)))


def bwd_noalloc_raw(shape: Shape, u, delta, A, B, C, D, z, delta_bias, delta_softplus: bool,
                    dout, du, ddelta, dA, dB, dC, dD, dz, ddelta_bias, stream=None):
    """Direct call of ssm_selective_scan_bwd_noalloc: the backward for callers
    that can neither allocate device memory nor pass scratch; its checkpoint
    scratch is a static array inside the library (see include/ssm_scan.h)."""
    _check(load_library().ssm_selective_scan_bwd_noalloc(
        ctypes.byref(shape), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(delta_bias), int(bool(delta_softplus)), _ptr(dout), _ptr(du), _ptr(ddelta), _ptr(dA),
        _ptr(dB), _ptr(dC), _ptr(dD), _ptr(dz), _ptr(ddelta_bias), _stream_ptr(stream)))


def state_update_raw(shape: Shape, state, u, delta, A, B, C, D, z, delta_bias,
                     delta_softplus: bool, out, stream=None, zoh: bool = False):
    """Direct call of ssm_selective_state_update(_ex) (one decoding step, state
    updated in place)."""
    if zoh:
        o = _opts(delta_softplus, True)
        _check(load_library().ssm_selective_state_update_ex(
            ctypes.byref(shape), ctypes.byref(o), _ptr(state), _ptr(u), _ptr(delta), _ptr(A),
            _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias), _ptr(out), _stream_ptr(stream)))
        return
    _check(load_library().ssm_selective_state_update(
        ctypes.byref(shape), _ptr(state), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
        _ptr(z), _ptr(delta_bias), int(bool(delta_softplus)), _ptr(out), _stream_ptr(stream)))


def projections_raw(shape: Shape, dt_rank: int, x, W_x, W_dt, dt_low, delta, B, C, stream=None):
    """Direct call of ssm_selection_projections (x_proj then dt_proj)."""
    _check(load_library().ssm_selection_projections(
        ctypes.byref(shape), int(dt_rank), _ptr(x), _ptr(W_x), _ptr(W_dt), _ptr(dt_low),
        _ptr(delta), _ptr(B), _ptr(C), _stream_ptr(stream)))


def _need(t, name, dtype=None, cuda=True):
    if t is None:
        return
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def selective_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                       delta_softplus: bool = True, return_last_state: bool = False,
                       return_ckpt: bool = False, out=None, stream=None, zoh: bool = False):
    """Forward selective scan.  u, delta, z, B, C share one io dtype (float32 or
    bfloat16); A, D, delta_bias are float32.  Returns (out, last_state, ckpt)
    with the last two None unless requested."""
    io = u.dtype
    for t, n in ((u, "u"), (delta, "delta"), (B, "B"), (C, "C"), (z, "z")):
        _need(t, n, io)
    for t, n in ((A, "A"), (D, "D"), (delta_bias, "delta_bias")):
        _need(t, n, torch.float32)
    shape = _shape_of(u, A)
    if out is None:
        out = torch.empty_like(u)
    last = (torch.empty(shape.batch, shape.dim, shape.dstate, device=u.device,
                        dtype=torch.float32) if return_last_state else None)
    ck = (torch.empty(ckpt_numel(shape), device=u.device, dtype=torch.float32)
          if return_ckpt else None)
    nws = fwd_workspace_bytes(shape, delta_softplus, zoh)
    ws = torch.empty(nws // 4, device=u.device, dtype=torch.float32) if nws else None
    fwd_raw(shape, u, delta, A, B, C, D, z, delta_bias, delta_softplus, out, last, ck, stream, zoh,
            workspace=ws)
    return out, last, ck


def selective_state_update(state, u, delta, A, B, C, D=None, z=None, delta_bias=None,
                           delta_softplus: bool = True, out=None, stream=None, zoh: bool = False):
    """One decoding step: advances `state` ([batch, dim, dstate] float32) in
    place by one token and returns out [batch, dim].  u, delta, z are
    [batch, dim] and B, C [batch, dstate] in one io dtype; A, D, delta_bias
    are float32."""
    io = u.dtype
    for t, n in ((u, "u"), (delta, "delta"), (B, "B"), (C, "C"), (z, "z")):
        _need(t, n, io)
    for t, n in ((state, "state"), (A, "A"), (D, "D"), (delta_bias, "delta_bias")):
        _need(t, n, torch.float32)
    if u.dim() != 2 or state.dim() != 3 or tuple(state.shape) != (u.shape[0], u.shape[1], A.shape[1]):
        raise ValueError("u must be [batch, dim], A [dim, dstate] and state [batch, dim, dstate]")
    shape = make_shape(u.shape[0], u.shape[1], 1, A.shape[1], io)
    if out is None:
        out = torch.empty_like(u)
    state_update_raw(shape, state, u, delta, A, B, C, D, z, delta_bias, delta_softplus, out, stream,
                     zoh)
    return out


def selective_scan_bwd(u, delta, A, B, C, D, z, delta_bias, delta_softplus: bool, dout,
                       ckpt=None, stream=None, zoh: bool = False):
    """Backward selective scan; returns a dict of float32 gradients (du, ddelta,
    dA, dB, dC and, for the optional inputs that were given, dD, dz,
    ddelta_bias).  zoh must match the forward that wrote `ckpt`."""
    io = u.dtype
    for t, n in ((u, "u"), (delta, "delta"), (B, "B"), (C, "C"), (z, "z"), (dout, "dout")):
        _need(t, n, io)
    for t, n in ((A, "A"), (D, "D"), (delta_bias, "delta_bias"), (ckpt, "ckpt")):
        _need(t, n, torch.float32)
    shape = _shape_of(u, A)
    f32 = dict(device=u.device, dtype=torch.float32)
    g = {"du": torch.empty(u.shape, **f32), "ddelta": torch.empty(u.shape, **f32),
         "dA": torch.empty(A.shape, **f32), "dB": torch.empty(B.shape, **f32),
         "dC": torch.empty(C.shape, **f32),
         "dD": torch.empty(D.shape, **f32) if D is not None else None,
         "dz": torch.empty(u.shape, **f32) if z is not None else None,
         "ddelta_bias": torch.empty(delta_bias.shape, **f32) if delta_bias is not None else None}
    nscratch = bwd_scratch_bytes(shape, ckpt is not None)
    scratch = torch.empty(max(1, nscratch // 4), **f32) if nscratch else None
    bwd_raw(shape, u, delta, A, B, C, D, z, delta_bias, delta_softplus, dout, ckpt,
            g["du"], g["ddelta"], g["dA"], g["dB"], g["dC"], g["dD"], g["dz"],
            g["ddelta_bias"], scratch, stream, zoh)
    return {k: v for k, v in g.items() if v is not None}


def selection_projections(x, W_x, W_dt, dstate: int, stream=None):
    """The selection projections in front of the scan: x [batch, dim, L],
    W_x [dt_rank + 2 dstate, dim], W_dt [dim, dt_rank], all bfloat16.
    Returns (delta [batch, dim, L], B [batch, dstate, L], C [batch, dstate, L],
    dt_low [batch, dt_rank, L]); delta, B and C are the scan's inputs."""
    for t, n in ((x, "x"), (W_x, "W_x"), (W_dt, "W_dt")):
        _need(t, n, torch.bfloat16)
    if x.dim() != 3 or W_x.dim() != 2 or W_dt.dim() != 2:
        raise ValueError("x must be [batch, dim, L], W_x [M, dim] and W_dt [dim, dt_rank]")
    batch, dim, L = x.shape
    dt_rank = W_dt.shape[1]
    if W_dt.shape[0] != dim or tuple(W_x.shape) != (dt_rank + 2 * dstate, dim):
        raise ValueError("W_x must be [dt_rank + 2 dstate, dim] and W_dt [dim, dt_rank]")
    shape = make_shape(batch, dim, L, dstate, SSM_BF16)
    kw = dict(device=x.device, dtype=torch.bfloat16)
    dt_low = torch.empty(batch, dt_rank, L, **kw)
    delta = torch.empty(batch, dim, L, **kw)
    B = torch.empty(batch, dstate, L, **kw)
    C = torch.empty(batch, dstate, L, **kw)
    projections_raw(shape, dt_rank, x, W_x, W_dt, dt_low, delta, B, C, stream)
    return delta, B, C, dt_low


def fwd_segment_raw(shape: Shape, u, delta, A, B, C, D, z, delta_bias, delta_softplus: bool, h0,
                    out, last_state, ckpt=None, delta_sum=None, stream=None, zoh: bool = False):
    """Direct call of ssm_selective_scan_fwd_segment."""
    o = _opts(delta_softplus, zoh)
    _check(load_library().ssm_selective_scan_fwd_segment(
        ctypes.byref(shape), ctypes.byref(o), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
        _ptr(D), _ptr(z), _ptr(delta_bias), _ptr(h0), _ptr(out), _ptr(last_state), _ptr(ckpt),
        _ptr(delta_sum), _stream_ptr(stream)))


def combine_carries_raw(nseg, batch, dim, dstate, A, delta_sums, h_ends, h0, h_in, stream=None):
    """Direct call of ssm_scan_combine_carries."""
    _check(load_library().ssm_scan_combine_carries(
        int(nseg), int(batch), int(dim), int(dstate), _ptr(A), _ptr(delta_sums), _ptr(h_ends),
        _ptr(h0), _ptr(h_in), _stream_ptr(stream)))


def selective_scan_fwd_segment(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                               delta_softplus: bool = True, h0=None, out=None, stream=None,
                               zoh: bool = False):
    """Forward over one segment of a sequence from state h0 ([batch, dim,
    dstate] float32, None = zeros).  Returns (out, last_state, delta_sum)
    with delta_sum [batch, dim] = Σ_t Δ_t over the segment."""
    io = u.dtype
    for t, n in ((u, "u"), (delta, "delta"), (B, "B"), (C, "C"), (z, "z")):
        _need(t, n, io)
    for t, n in ((A, "A"), (D, "D"), (delta_bias, "delta_bias"), (h0, "h0")):
        _need(t, n, torch.float32)
    shape = _shape_of(u, A)
    if out is None:
        out = torch.empty_like(u)
    f32 = dict(device=u.device, dtype=torch.float32)
    last = torch.empty(shape.batch, shape.dim, shape.dstate, **f32)
    dsum = torch.empty(shape.batch, shape.dim, **f32)
    fwd_segment_raw(shape, u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, out, last,
                    None, dsum, stream, zoh)
    return out, last, dsum


def combine_carries(A, delta_sums, h_ends, h0=None, stream=None):
    """States entering each of S segments from their summaries: delta_sums
    [S, batch, dim], h_ends [S, batch, dim, dstate] (float32, device).
    Returns h_in [S, batch, dim, dstate]."""
    for t, n in ((A, "A"), (delta_sums, "delta_sums"), (h_ends, "h_ends"), (h0, "h0")):
        _need(t, n, torch.float32)
    S, batch, dim, dstate = h_ends.shape
    h_in = torch.empty_like(h_ends)
    combine_carries_raw(S, batch, dim, dstate, A, delta_sums, h_ends, h0, h_in, stream)
    return h_in
