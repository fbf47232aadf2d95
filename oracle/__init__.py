"""fp64 CPU oracle for the Mamba-2 mixer core -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of bench.py
may import this package.  The product library (mamba_ssd_scan_mixer_b200) never
imports it and it never imports the product library: the two share no code.

Every function takes array-likes (numpy arrays or CPU torch tensors of any
float dtype), upcasts them to float64 exactly, calls the plain C routines in
mamba2_oracle.c and returns float64 numpy arrays.  The C source documents the
formulas and the passages they follow:

* conv1d + SiLU with carried conv state -- "Zamba2 hybrid architecture in
  Transformers" (qwbw.cn), section 三 step 2, section 五 (use_conv_bias).
* softplus dt and the selective SSM recurrence -- the Mamba-2 SSD layer named
  on the state-spaces/mamba repository page (opendeer.net), "About the
  project"; chunked scan vs single-step update per qwbw.cn section 三 step 3.
* gated group RMSNorm with norm_before_gate -- qwbw.cn section 三 step 4 and
  section 五 (rms_norm_eps = 1e-5).

Scan forms: "sequential" (token-by-token definition), "quadratic" (materialised
semiseparable matrix, tiny inputs only), "chunked" (state-space-duality
block form, any chunk length >= 1).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None
_FORMS = {"sequential": 0, "quadratic": 1, "chunked": 2}


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        d, i64, i32, vp = ctypes.c_double, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        lib.m2o_silu.restype = d
        lib.m2o_silu.argtypes = [d]
        lib.m2o_softplus.restype = d
        lib.m2o_softplus.argtypes = [d]
        lib.m2o_conv_silu.restype = None
        lib.m2o_conv_silu.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp]
        lib.m2o_scan.restype = i32
        lib.m2o_scan.argtypes = [i32, i64, i64, i64, i64, i64, vp, i64, vp, vp, i64, vp, vp, vp,
                                 vp, vp, i64, vp, i64, i32]
        lib.m2o_gated_rmsnorm.restype = None
        lib.m2o_gated_rmsnorm.argtypes = [i64, i64, i64, vp, i64, vp, i64, vp, d, i32, vp, i64]
        lib.m2o_mixer_prefill.restype = i32
        lib.m2o_mixer_prefill.argtypes = [i64] * 7 + [vp] * 14 + [d, i32, i32, i64, i32]
        lib.m2o_mixer_step.restype = i32
        lib.m2o_mixer_step.argtypes = [i64] * 6 + [vp] * 12 + [d, i32, i32]
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _f64(a):
    """Exact upcast to a C-contiguous float64 numpy array (None passes through)."""
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu")
        import torch
        a = a.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def silu(s: float) -> float:
    return _load().m2o_silu(float(s))


def softplus(s: float) -> float:
    return _load().m2o_softplus(float(s))


def conv_silu(xBC, conv_w, conv_b, conv_state=None):
    """Causal depthwise conv1d + SiLU of one sequence.

    xBC [L, conv_dim]; conv_w [conv_dim, K]; conv_b [conv_dim];
    conv_state [conv_dim, K] (oldest first) or None for zeros.
    Returns (u [L, conv_dim], conv_state_out [conv_dim, K])."""
    xBC, conv_w, conv_b, cs = _f64(xBC), _f64(conv_w), _f64(conv_b), _f64(conv_state)
    L, conv_dim = xBC.shape
    K = conv_w.shape[1]
    u = np.empty((L, conv_dim))
    cs_out = np.empty((conv_dim, K))
    _load().m2o_conv_silu(L, conv_dim, K, _p(xBC), _p(cs), _p(conv_w), _p(conv_b), _p(u),
                          _p(cs_out))
    return u, cs_out


def scan(x, B, C, dt, A, D, h0=None, form="sequential", chunk=0, nthreads=1):
    """The selective scan of one sequence (D skip included, no gate/norm).

    x [L, H, P]; B, C [L, G, N]; dt [L, H] (already softplus'd); A, D [H];
    h0 [H, P, N] or None.  Returns (y [L, H, P], hL [H, P, N])."""
    x, B, C, dt, A, D, h0 = map(_f64, (x, B, C, dt, A, D, h0))
    L, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    y = np.empty((L, H, P))
    hL = np.empty((H, P, N))
    rc = _load().m2o_scan(_FORMS[form], L, H, P, N, G, _p(x), H * P, _p(B), _p(C), G * N,
                          _p(dt), _p(A), _p(D), _p(h0), _p(y), H * P, _p(hL), int(chunk),
                          int(nthreads))
    if rc != 0:
        raise ValueError("oracle scan rejected its arguments")
    return y, hL


def gated_rmsnorm(y, z, norm_w, ngroups, eps=1e-5, norm_before_gate=False):
    """y, z [L, d_inner]; norm_w [d_inner]; returns out [L, d_inner]."""
    y, z, w = _f64(y), _f64(z), _f64(norm_w)
    L, d_inner = y.shape
    out = np.empty((L, d_inner))
    _load().m2o_gated_rmsnorm(L, d_inner, int(ngroups), _p(y), d_inner, _p(z), d_inner, _p(w),
                              float(eps), int(bool(norm_before_gate)), _p(out), d_inner)
    return out


def mixer_prefill(xBC, z, dt_raw, params, *, nheads, headdim, dstate, ngroups,
                  conv_state=None, ssm_state=None, eps=1e-5, norm_before_gate=False,
                  form="sequential", chunk=0, nthreads=None):
    """Whole mixer core over a batch: conv+SiLU -> dt -> scan (+D) -> gated norm.

    xBC [b, L, conv_dim]; z [b, L, H*P]; dt_raw [b, L, H]; params: dict with
    conv_w [conv_dim, K], conv_b, dt_bias [H], A [H], D [H], norm_w [H*P];
    conv_state [b, conv_dim, K] / ssm_state [b, H, P, N] or None (zeros).
    Returns dict(y [b, L, H*P], conv_state [b, conv_dim, K], ssm_state [b, H, P, N])."""
    xBC, z, dt_raw = _f64(xBC), _f64(z), _f64(dt_raw)
    pw = {k: _f64(params[k]) for k in ("conv_w", "conv_b", "dt_bias", "A", "D", "norm_w")}
    cs_in, hs_in = _f64(conv_state), _f64(ssm_state)
    b, L, conv_dim = xBC.shape
    H, P, N, G = nheads, headdim, dstate, ngroups
    K = pw["conv_w"].shape[1]
    assert conv_dim == H * P + 2 * G * N
    y = np.empty((b, L, H * P))
    cs_out = np.empty((b, conv_dim, K))
    hs_out = np.empty((b, H, P, N))
    rc = _load().m2o_mixer_prefill(
        b, L, H, P, N, G, K, _p(xBC), _p(z), _p(dt_raw), _p(pw["conv_w"]), _p(pw["conv_b"]),
        _p(pw["dt_bias"]), _p(pw["A"]), _p(pw["D"]), _p(pw["norm_w"]), _p(cs_in), _p(hs_in),
        _p(y), _p(cs_out), _p(hs_out), float(eps), int(bool(norm_before_gate)), _FORMS[form],
        int(chunk), int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError("oracle prefill rejected its arguments")
    return {"y": y, "conv_state": cs_out, "ssm_state": hs_out}


def mixer_step(xBC, z, dt_raw, params, conv_state, ssm_state, *, nheads, headdim, dstate,
               ngroups, eps=1e-5, norm_before_gate=False, nthreads=None):
    """One decode step over a batch.  xBC [b, conv_dim]; z [b, H*P]; dt_raw [b, H];
    conv_state [b, conv_dim, K], ssm_state [b, H, P, N] (copied, not modified).
    Returns dict(y [b, H*P], conv_state, ssm_state) with the updated states."""
    xBC, z, dt_raw = _f64(xBC), _f64(z), _f64(dt_raw)
    pw = {k: _f64(params[k]) for k in ("conv_w", "conv_b", "dt_bias", "A", "D", "norm_w")}
    cs = _f64(conv_state).copy()
    hs = _f64(ssm_state).copy()
    b, conv_dim = xBC.shape
    H, P, N, G = nheads, headdim, dstate, ngroups
    K = pw["conv_w"].shape[1]
    y = np.empty((b, H * P))
    rc = _load().m2o_mixer_step(
        b, H, P, N, G, K, _p(xBC), _p(z), _p(dt_raw), _p(pw["conv_w"]), _p(pw["conv_b"]),
        _p(pw["dt_bias"]), _p(pw["A"]), _p(pw["D"]), _p(pw["norm_w"]), _p(cs), _p(hs), _p(y),
        float(eps), int(bool(norm_before_gate)), int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError("oracle step rejected its arguments")
    return {"y": y, "conv_state": cs, "ssm_state": hs}
