"""Thin Python binding of libmamba2ssd.so, the B200 Mamba-2 mixer-core library.

Argument marshalling only: every step of the mixer runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  There is no
CPU path: if the library is missing, importing the entry points raises.

Entry points (same names as the C ABI in include/mamba2ssd.h):
    mamba2_prefill_workspace_size(dims) -> int
    mamba2_conv_ssd_prefill(dims, params, xBC, z, dt_raw, y, conv_state, ssm_state,
                            states_in, workspace, stream=None)
    mamba2_ssd_step(dims, params, xBC, z, dt_raw, y, conv_state, ssm_state, stream=None)
Conveniences that allocate outputs and workspace with torch and call the above:
    prefill(...), step(...)
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "Mamba2Dims", "Mamba2Params", "Mamba2Error", "MAMBA2_F32", "MAMBA2_BF16", "lib",
    "library_path", "make_dims", "make_params", "mamba2_prefill_workspace_size",
    "mamba2_conv_ssd_prefill", "mamba2_conv_ssd_prefill_noalloc", "mamba2_ssd_step", "prefill",
    "step", "status_string", "mamba2_prefill_backward_workspace_size",
    "mamba2_conv_ssd_prefill_backward", "prefill_backward",
    "mamba2_prefill_host_workspace_size", "mamba2_conv_ssd_prefill_host", "prefill_host",
]

MAMBA2_F32, MAMBA2_BF16 = 0, 1
_PKG = os.path.dirname(os.path.abspath(__file__))
# MAMBA2SSD_LIBRARY selects another build of the library, e.g. the bounds-checked
# libmamba2ssd_checked.so (see build.py)
library_path = os.environ.get("MAMBA2SSD_LIBRARY") or os.path.join(_PKG, "libmamba2ssd.so")


class Mamba2Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("nheads", ctypes.c_int32), ("headdim", ctypes.c_int32),
                ("dstate", ctypes.c_int32), ("ngroups", ctypes.c_int32),
                ("d_conv", ctypes.c_int32), ("chunk_size", ctypes.c_int32),
                ("io_dtype", ctypes.c_int32), ("norm_before_gate", ctypes.c_int32),
                ("norm_eps", ctypes.c_float)]


class Mamba2Params(ctypes.Structure):
    _fields_ = [("conv_w", ctypes.c_void_p), ("conv_b", ctypes.c_void_p),
                ("dt_bias", ctypes.c_void_p), ("A", ctypes.c_void_p), ("D", ctypes.c_void_p),
                ("norm_w", ctypes.c_void_p)]


class Mamba2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built (no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise RuntimeError(
                f"{library_path} is missing: build it with "
                "`python -m mamba_ssd_scan_mixer_b200.build` (there is no CPU fallback)")
        L = ctypes.CDLL(library_path)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        pd, pp = ctypes.POINTER(Mamba2Dims), ctypes.POINTER(Mamba2Params)
        L.mamba2_status_string.restype = ctypes.c_char_p
        L.mamba2_status_string.argtypes = [ctypes.c_int]
        L.mamba2_version.restype = ctypes.c_int
        L.mamba2_version.argtypes = []
        L.mamba2_prefill_workspace_size.restype = sz
        L.mamba2_prefill_workspace_size.argtypes = [pd]
        L.mamba2_conv_ssd_prefill.restype = ctypes.c_int
        L.mamba2_conv_ssd_prefill.argtypes = [pd, pp, vp, i64, vp, i64, vp, i64, vp, vp, vp, i32,
                                              vp, sz, vp]
        L.mamba2_prefill_host_workspace_size.restype = sz
        L.mamba2_prefill_host_workspace_size.argtypes = [pd]
        L.mamba2_conv_ssd_prefill_host.restype = ctypes.c_int
        L.mamba2_conv_ssd_prefill_host.argtypes = [pd, pp, vp, i64, vp, i64, vp, i64, vp, vp, vp,
                                                   i32, vp, sz, vp]
        L.mamba2_prefill_varlen_workspace_size.restype = sz
        L.mamba2_prefill_varlen_workspace_size.argtypes = [pd]
        L.mamba2_conv_ssd_prefill_varlen.restype = ctypes.c_int
        L.mamba2_conv_ssd_prefill_varlen.argtypes = [pd, pp, vp, i64, vp, i64, vp, i64, vp, vp,
                                                     vp, vp, i32, vp, sz, vp]
        L.mamba2_conv_ssd_prefill_noalloc.restype = ctypes.c_int
        L.mamba2_conv_ssd_prefill_noalloc.argtypes = [pd, pp, vp, i64, vp, i64, vp, i64, vp, vp,
                                                      vp, i32, vp]
        L.mamba2_device_errors.restype = ctypes.c_int
        L.mamba2_device_errors.argtypes = [ctypes.POINTER(ctypes.c_uint)]
        L.mamba2_debug_stall_waits.restype = ctypes.c_int
        L.mamba2_debug_stall_waits.argtypes = [ctypes.c_int]
        L.mamba2_prefill_backward_workspace_size.restype = sz
        L.mamba2_prefill_backward_workspace_size.argtypes = [pd]
        L.mamba2_conv_ssd_prefill_backward.restype = ctypes.c_int
        L.mamba2_conv_ssd_prefill_backward.argtypes = ([pd, pp, vp, i64, vp, i64, vp, i64]
                                                       + [vp] * 15 + [vp, sz, vp])
        L.mamba2_ssd_step.restype = ctypes.c_int
        L.mamba2_ssd_step.argtypes = [pd, pp, vp, i64, vp, i64, vp, i64, vp, vp, vp, vp]
        _lib = L
    return _lib


def device_errors() -> int:
    """Synchronise the current device and return (and clear) the flags raised by
    kernels whose bounded waits ran out (0 = none)."""
    f = ctypes.c_uint(0)
    st = lib().mamba2_device_errors(ctypes.byref(f))
    if st != 0:
        raise Mamba2Error(st, "mamba2_device_errors")
    return int(f.value)


def debug_stall_waits(enable: bool) -> None:
    """Test aid: while enabled, every waiting kernel's first wait runs out (20 ms)
    and the kernel returns without doing its work, raising the flag that
    device_errors() reports (bit 0).  Synchronises the current device."""
    st = lib().mamba2_debug_stall_waits(int(bool(enable)))
    if st != 0:
        raise Mamba2Error(st, "mamba2_debug_stall_waits")


def status_string(status: int) -> str:
    return lib().mamba2_status_string(int(status)).decode()


def make_dims(batch, seqlen, nheads, headdim, dstate, ngroups, *, d_conv=4, chunk_size=256,
              io_dtype="bf16", norm_before_gate=False, norm_eps=1e-5) -> Mamba2Dims:
    io = {"f32": MAMBA2_F32, "bf16": MAMBA2_BF16}.get(io_dtype, io_dtype)
    return Mamba2Dims(int(batch), int(seqlen), int(nheads), int(headdim), int(dstate),
                      int(ngroups), int(d_conv), int(chunk_size), int(io),
                      int(bool(norm_before_gate)), float(norm_eps))


def dims_from_config(cfg, batch=None, seqlen=None) -> Mamba2Dims:
    return make_dims(cfg.batch if batch is None else batch,
                     cfg.seqlen if seqlen is None else seqlen, cfg.nheads, cfg.headdim,
                     cfg.dstate, cfg.ngroups, d_conv=cfg.d_conv, chunk_size=cfg.chunk_size,
                     io_dtype=cfg.io_dtype, norm_before_gate=cfg.norm_before_gate,
                     norm_eps=cfg.norm_eps)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def make_params(conv_w, conv_b, dt_bias, A, D, norm_w) -> Mamba2Params:
    """Pointers of fp32 device tensors; the caller keeps the tensors alive."""
    ts = (conv_w, conv_b, dt_bias, A, D, norm_w)
    for t in ts:
        import torch
        if not (t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()):
            raise ValueError("parameters must be contiguous fp32 CUDA tensors")
    return Mamba2Params(*[t.data_ptr() for t in ts])


def _stream(stream):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if hasattr(stream, "cuda_stream"):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _rows(t, name, width, batch, rows_per_batch):
    """Row stride (elements) of a [batch, rows, width]-shaped view with unit last stride."""
    if t.stride(-1) != 1:
        raise ValueError(f"{name}: last dimension must be contiguous")
    rs = t.stride(-2) if t.dim() >= 2 else width
    if (t.dim() == 3 and t.shape[0] > 1 and rows_per_batch > 0
            and t.stride(0) != rows_per_batch * rs):
        raise ValueError(f"{name}: batch stride must be rows * row stride")
    return rs


def mamba2_prefill_workspace_size(dims: Mamba2Dims) -> int:
    return int(lib().mamba2_prefill_workspace_size(ctypes.byref(dims)))


def mamba2_conv_ssd_prefill(dims, params, xBC, z, dt_raw, y, conv_state=None, ssm_state=None,
                            states_in=False, workspace=None, stream=None) -> None:
    """Enqueue one prefill on `stream` (default: torch's current stream).

    xBC [b, L, conv_dim], z [b, L, d_inner], dt_raw [b, L, H] (views with unit last
    stride; row strides are passed through); y [b, L, d_inner] contiguous;
    conv_state [b, conv_dim, 4] / ssm_state [b, H, P, N] fp32 or None;
    workspace: a CUDA byte tensor of mamba2_prefill_workspace_size(dims) bytes."""
    L = dims.seqlen
    lx = _rows(xBC, "xBC", None, dims.batch, L)
    lz = _rows(z, "z", None, dims.batch, L)
    ld = _rows(dt_raw, "dt_raw", None, dims.batch, L)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().mamba2_conv_ssd_prefill(
        ctypes.byref(dims), ctypes.byref(params), _ptr(xBC), lx, _ptr(z), lz, _ptr(dt_raw), ld,
        _ptr(y), _ptr(conv_state), _ptr(ssm_state), int(bool(states_in)), _ptr(workspace),
        ws_bytes, _stream(stream))
    if st != 0:
        raise Mamba2Error(st, "mamba2_conv_ssd_prefill")


def mamba2_prefill_host_workspace_size(dims: Mamba2Dims) -> int:
    return int(lib().mamba2_prefill_host_workspace_size(ctypes.byref(dims)))


def mamba2_conv_ssd_prefill_host(dims, params, xBC, z, dt_raw, y, conv_state=None,
                                 ssm_state=None, states_in=False, workspace=None,
                                 stream=None) -> None:
    """Enqueue one prefill whose inputs, y and states are CPU tensors (page-locked
    for overlapped copies); layouts as mamba2_conv_ssd_prefill; workspace: a CUDA
    byte tensor of mamba2_prefill_host_workspace_size(dims) bytes.  Synchronise
    the stream before reading y or the states."""
    for name, t in (("xBC", xBC), ("z", z), ("dt_raw", dt_raw), ("y", y),
                    ("conv_state", conv_state), ("ssm_state", ssm_state)):
        if t is not None and t.is_cuda:
            raise ValueError(f"{name}: the host entry takes CPU tensors")
    L = dims.seqlen
    lx = _rows(xBC, "xBC", None, dims.batch, L)
    lz = _rows(z, "z", None, dims.batch, L)
    ld = _rows(dt_raw, "dt_raw", None, dims.batch, L)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().mamba2_conv_ssd_prefill_host(
        ctypes.byref(dims), ctypes.byref(params), _ptr(xBC), lx, _ptr(z), lz, _ptr(dt_raw), ld,
        _ptr(y), _ptr(conv_state), _ptr(ssm_state), int(bool(states_in)), _ptr(workspace),
        ws_bytes, _stream(stream))
    if st != 0:
        raise Mamba2Error(st, "mamba2_conv_ssd_prefill_host")


def prefill_host(dims, params, xBC, z, dt_raw, conv_state=None, ssm_state=None,
                 states_in=False, workspace=None, y=None, stream=None, device=None):
    """Allocate y (page-locked) and the device workspace if not given, run a
    host-buffer prefill and wait for it.  Returns y [b, L, d_inner] on the CPU;
    the states, if given, are updated in place."""
    import torch
    dev = torch.device("cuda") if device is None else torch.device(device)
    if y is None:
        y = torch.empty(dims.batch, dims.seqlen, dims.nheads * dims.headdim, dtype=xBC.dtype,
                        pin_memory=True)
    if workspace is None:
        workspace = torch.empty(max(1, mamba2_prefill_host_workspace_size(dims)),
                                dtype=torch.uint8, device=dev)
    mamba2_conv_ssd_prefill_host(dims, params, xBC, z, dt_raw, y, conv_state, ssm_state,
                                 states_in, workspace, stream)
    torch.cuda.synchronize(dev)
    return y


def mamba2_prefill_varlen_workspace_size(dims: Mamba2Dims) -> int:
    return int(lib().mamba2_prefill_varlen_workspace_size(ctypes.byref(dims)))


def mamba2_conv_ssd_prefill_varlen(dims, params, xBC, z, dt_raw, cu_seqlens, y, conv_state=None,
                                   ssm_state=None, states_in=False, workspace=None,
                                   stream=None) -> None:
    """Enqueue one prefill of dims.batch sequences packed along the token axis
    (dims.seqlen = total tokens): xBC [T, conv_dim], z [T, d_inner], dt_raw [T, H]
    (unit last stride, row strides passed through), y [T, d_inner] contiguous;
    cu_seqlens: CUDA int32 [batch + 1] (0, running token counts, T); states per
    sequence; workspace of mamba2_prefill_varlen_workspace_size(dims) bytes."""
    lx = _rows(xBC, "xBC", None, 1, 0)
    lz = _rows(z, "z", None, 1, 0)
    ld = _rows(dt_raw, "dt_raw", None, 1, 0)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().mamba2_conv_ssd_prefill_varlen(
        ctypes.byref(dims), ctypes.byref(params), _ptr(xBC), lx, _ptr(z), lz, _ptr(dt_raw), ld,
        _ptr(cu_seqlens), _ptr(y), _ptr(conv_state), _ptr(ssm_state), int(bool(states_in)),
        _ptr(workspace), ws_bytes, _stream(stream))
    if st != 0:
        raise Mamba2Error(st, "mamba2_conv_ssd_prefill_varlen")


def prefill_varlen(dims, params, xBC, z, dt_raw, cu_seqlens, conv_state=None, ssm_state=None,
                   states_in=False, workspace=None, y=None, stream=None):
    """Allocate y (and the workspace if not given) and run a packed-sequence prefill.
    Returns y [T, d_inner]; the states, if given, are updated in place."""
    import torch
    if y is None:
        y = torch.empty(dims.seqlen, dims.nheads * dims.headdim, dtype=xBC.dtype,
                        device=xBC.device)
    if workspace is None:
        workspace = torch.empty(max(1, mamba2_prefill_varlen_workspace_size(dims)),
                                dtype=torch.uint8, device=xBC.device)
    mamba2_conv_ssd_prefill_varlen(dims, params, xBC, z, dt_raw, cu_seqlens, y, conv_state,
                                   ssm_state, states_in, workspace, stream)
    return y


def mamba2_conv_ssd_prefill_noalloc(dims, params, xBC, z, dt_raw, y, conv_state=None,
                                    ssm_state=None, states_in=False, stream=None) -> None:
    """Prefill without a workspace, for callers that may not allocate device memory:
    the library's fixed device scratch array (MAMBA2_STATIC_SCRATCH_BYTES, 64 MiB)
    is used instead.  Larger problems raise Mamba2Error (workspace status).  Calls
    that overlap on the GPU share that array and race; serialise them."""
    L = dims.seqlen
    lx = _rows(xBC, "xBC", None, dims.batch, L)
    lz = _rows(z, "z", None, dims.batch, L)
    ld = _rows(dt_raw, "dt_raw", None, dims.batch, L)
    st = lib().mamba2_conv_ssd_prefill_noalloc(
        ctypes.byref(dims), ctypes.byref(params), _ptr(xBC), lx, _ptr(z), lz, _ptr(dt_raw), ld,
        _ptr(y), _ptr(conv_state), _ptr(ssm_state), int(bool(states_in)), _stream(stream))
    if st != 0:
        raise Mamba2Error(st, "mamba2_conv_ssd_prefill_noalloc")


def mamba2_ssd_step(dims, params, xBC, z, dt_raw, y, conv_state, ssm_state, stream=None) -> None:
    """Enqueue one decode step.  xBC [b, conv_dim], z [b, d_inner], dt_raw [b, H]
    (unit last stride); y [b, d_inner]; states updated in place."""
    st = lib().mamba2_ssd_step(
        ctypes.byref(dims), ctypes.byref(params), _ptr(xBC), xBC.stride(0), _ptr(z), z.stride(0),
        _ptr(dt_raw), dt_raw.stride(0), _ptr(y), _ptr(conv_state), _ptr(ssm_state),
        _stream(stream))
    if st != 0:
        raise Mamba2Error(st, "mamba2_ssd_step")


def prefill(dims, params, xBC, z, dt_raw, conv_state=None, ssm_state=None, states_in=False,
            workspace=None, y=None, stream=None):
    """Allocate y (and the workspace if not given) on xBC's device and run a prefill.
    Returns y; the states, if given, are updated in place."""
    import torch
    if y is None:
        y = torch.empty(dims.batch, dims.seqlen, dims.nheads * dims.headdim, dtype=xBC.dtype,
                        device=xBC.device)
    if workspace is None:
        workspace = torch.empty(max(1, mamba2_prefill_workspace_size(dims)), dtype=torch.uint8,
                                device=xBC.device)
    mamba2_conv_ssd_prefill(dims, params, xBC, z, dt_raw, y, conv_state, ssm_state, states_in,
                            workspace, stream)
    return y


def step(dims, params, xBC, z, dt_raw, conv_state, ssm_state, y=None, stream=None):
    """Allocate y and run one decode step; returns y."""
    import torch
    if y is None:
        y = torch.empty(dims.batch, dims.nheads * dims.headdim, dtype=xBC.dtype,
                        device=xBC.device)
    mamba2_ssd_step(dims, params, xBC, z, dt_raw, y, conv_state, ssm_state, stream)
    return y


def mamba2_prefill_backward_workspace_size(dims: Mamba2Dims) -> int:
    return int(lib().mamba2_prefill_backward_workspace_size(ctypes.byref(dims)))


def mamba2_conv_ssd_prefill_backward(dims, params, xBC, z, dt_raw, dy, grads, conv_state_in=None,
                                     ssm_state_in=None, d_ssm_state_out=None, workspace=None,
                                     stream=None) -> None:
    """Enqueue the prefill's backward pass on `stream`.

    xBC, z, dt_raw as for the prefill; dy [b, L, d_inner] contiguous; grads: a dict of
    output tensors "xBC", "z", "dt_raw" (io dtype, contiguous), "conv_w", "conv_b",
    "dt_bias", "A", "D", "norm_w" (fp32) and optionally "conv_state", "ssm_state" (the
    initial states' gradients); workspace: a CUDA byte tensor of
    mamba2_prefill_backward_workspace_size(dims) bytes."""
    L = dims.seqlen
    lx = _rows(xBC, "xBC", None, dims.batch, L)
    lz = _rows(z, "z", None, dims.batch, L)
    ld = _rows(dt_raw, "dt_raw", None, dims.batch, L)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    g = lambda k: _ptr(grads.get(k))
    st = lib().mamba2_conv_ssd_prefill_backward(
        ctypes.byref(dims), ctypes.byref(params), _ptr(xBC), lx, _ptr(z), lz, _ptr(dt_raw), ld,
        _ptr(conv_state_in), _ptr(ssm_state_in), _ptr(dy), _ptr(d_ssm_state_out), g("xBC"),
        g("z"), g("dt_raw"), g("conv_w"), g("conv_b"), g("dt_bias"), g("A"), g("D"), g("norm_w"),
        g("conv_state"), g("ssm_state"), _ptr(workspace), ws_bytes, _stream(stream))
    if st != 0:
        raise Mamba2Error(st, "mamba2_conv_ssd_prefill_backward")


def prefill_backward(dims, params, xBC, z, dt_raw, dy, conv_state_in=None, ssm_state_in=None,
                     d_ssm_state_out=None, workspace=None, stream=None):
    """Allocate the gradients (and the workspace if not given) and run the backward pass.
    Returns the dict of gradients (initial-state gradients when those states are given)."""
    import torch
    dev, dt = xBC.device, xBC.dtype
    b, L, H, P, N, G = (dims.batch, dims.seqlen, dims.nheads, dims.headdim, dims.dstate,
                        dims.ngroups)
    d_inner, conv_dim = H * P, H * P + 2 * G * N
    f32 = dict(dtype=torch.float32, device=dev)
    grads = {"xBC": torch.empty(b, L, conv_dim, dtype=dt, device=dev),
             "z": torch.empty(b, L, d_inner, dtype=dt, device=dev),
             "dt_raw": torch.empty(b, L, H, dtype=dt, device=dev),
             "conv_w": torch.empty(conv_dim, dims.d_conv, **f32),
             "conv_b": torch.empty(conv_dim, **f32), "dt_bias": torch.empty(H, **f32),
             "A": torch.empty(H, **f32), "D": torch.empty(H, **f32),
             "norm_w": torch.empty(d_inner, **f32)}
    if conv_state_in is not None:
        grads["conv_state"] = torch.empty_like(conv_state_in)
    if ssm_state_in is not None:
        grads["ssm_state"] = torch.empty_like(ssm_state_in)
    if workspace is None:
        workspace = torch.empty(max(1, mamba2_prefill_backward_workspace_size(dims)),
                                dtype=torch.uint8, device=dev)
    mamba2_conv_ssd_prefill_backward(dims, params, xBC, z, dt_raw, dy, grads, conv_state_in,
                                     ssm_state_in, d_ssm_state_out, workspace, stream)
    return grads
