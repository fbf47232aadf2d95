"""Helpers shared by the GPU parity tests: run the library and the oracle on the
same seeded inputs and compare them under the stated tolerances.

Tolerances (written here once, used by every parity test):
* fp32 I/O: per element |g - o| <= 1e-3 * max(|o|, rms(o)) for y and both
  states (max relative error 1e-3, with elements near zero measured against
  the tensor's RMS).
* bf16 I/O (fp32 accumulation, fp32 state): the final SSM state (fp32) must
  satisfy max |g - o| <= 2e-2 * rms(o).  For y, which the library returns in
  bf16, the exact result is first subject to its own rounding to bf16: half
  the spacing of bf16 values in the binade of the element (2^(e-8) for a
  value in [2^e, 2^(e+1)); the binade of max(|o|, |g|), so that a result
  that rounded across a power of two is judged by the spacing it was rounded
  in).  The bound applies to what is left:
  max (|g - o| - halfulp) <= 2e-2 * rms(o).  The raw max |g - o| / rms(o) is
  reported alongside.
* the final conv state is a copy of inputs: bit-exact.
"""
from __future__ import annotations

import numpy as np
import torch

import mamba_ssd_scan_mixer_b200 as m2
import oracle
from mamba_ssd_scan_mixer_b200 import workloads as W

F32_REL = 1e-3
BF16_RMS = 2e-2


def dev_params(params, device="cuda"):
    t = {k: v.to(device).contiguous() for k, v in params.items()}
    return t, m2.make_params(t["conv_w"], t["conv_b"], t["dt_bias"], t["A"], t["D"], t["norm_w"])


def gpu_prefill(cfg, inp, params, states=None, states_in=False, want_states=True):
    """Run the library's prefill on cfg-shaped inputs (CPU tensors); returns CPU tensors."""
    dims = m2.dims_from_config(cfg)
    v = W.split_packed(cfg, inp["zxbcdt"].cuda())
    z, xBC, dt = v["z"], v["xBC"], v["dt_raw"]
    cd = cfg.conv_dim
    pt, pp = dev_params(params)
    if states is not None:
        cs = states["conv_state"].cuda().contiguous()
        hs = states["ssm_state"].cuda().contiguous()
    elif want_states:
        cs = torch.full((cfg.batch, cd, cfg.d_conv), 7.0, dtype=cfg.torch_dtype, device="cuda")
        hs = torch.full((cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate), 7.0, device="cuda")
    else:
        cs = hs = None
    y = m2.prefill(dims, pp, xBC, z, dt, cs, hs, states_in=states_in)
    torch.cuda.synchronize()
    out = {"y": y.cpu()}
    if cs is not None:
        out["conv_state"] = cs.cpu()
        out["ssm_state"] = hs.cpu()
    return out


def oracle_prefill(cfg, inp, params, states=None, nthreads=None):
    return oracle.mixer_prefill(
        inp["xBC"], inp["z"], inp["dt_raw"], params, nheads=cfg.nheads, headdim=cfg.headdim,
        dstate=cfg.dstate, ngroups=cfg.ngroups,
        conv_state=None if states is None else states["conv_state"],
        ssm_state=None if states is None else states["ssm_state"], eps=cfg.norm_eps,
        norm_before_gate=cfg.norm_before_gate, nthreads=nthreads)


def _np(t):
    return t.to(torch.float64).numpy() if isinstance(t, torch.Tensor) else np.asarray(t, np.float64)


def rms(o):
    return float(np.sqrt(np.mean(np.square(o)))) if o.size else 0.0


def check_f32(g, o, what):
    g, o = _np(g), _np(o)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    if o.size == 0:
        return 0.0
    denom = np.maximum(np.abs(o), rms(o))
    err = float(np.max(np.abs(g - o) / np.where(denom > 0, denom, 1.0)))
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    assert err <= F32_REL, f"{what}: max relative error {err:.3e} > {F32_REL}"
    return err


def bf16_half_ulp(a):
    """Half the spacing of bf16 values around each |a| (0 where a == 0): for a
    value in [2^e, 2^(e+1)) the spacing is 2^(e-7)."""
    a = np.abs(np.asarray(a, np.float64))
    _, ex = np.frexp(a)  # a = m * 2^ex, m in [0.5, 1): the binade is [2^(ex-1), 2^ex)
    return np.where(a > 0, np.ldexp(1.0, ex - 9), 0.0)


def check_bf16_out(g, o, what):
    """y in bf16 against the fp64 oracle: 2e-2 of RMS beyond the output's own rounding."""
    g, o = _np(g), _np(o)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    if o.size == 0:
        return 0.0, 0.0
    r = rms(o)
    d = np.abs(g - o)
    allow = bf16_half_ulp(np.maximum(np.abs(o), np.abs(g)))
    beyond = float(np.max(np.maximum(d - allow, 0.0))) / r
    raw = float(np.max(d)) / r
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    assert beyond <= BF16_RMS, (f"{what}: error beyond bf16 rounding {beyond:.3e} of RMS "
                                f"> {BF16_RMS} (raw max {raw:.3e})")
    return beyond, raw


def check_rms(g, o, what, tol=BF16_RMS):
    g, o = _np(g), _np(o)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    if o.size == 0:
        return 0.0
    r = rms(o)
    err = float(np.max(np.abs(g - o))) / (r if r > 0 else 1.0)
    assert err <= tol, f"{what}: max abs error {err:.3e} of RMS > {tol}"
    return err


def check_exact(g, o, what):
    g, o = _np(g), _np(o)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    bad = np.flatnonzero(g != o)
    assert bad.size == 0, f"{what}: {bad.size} elements differ (first at flat index {bad[0]})"


def compare_prefill(cfg, got, ref, with_states=True):
    """Apply the tolerances above; returns a dict of the measured errors."""
    rep = {}
    if cfg.io_dtype == "f32":
        rep["y"] = check_f32(got["y"], ref["y"], "y")
        if with_states:
            rep["ssm_state"] = check_f32(got["ssm_state"], ref["ssm_state"], "ssm_state")
    else:
        rep["y"], rep["y_raw"] = check_bf16_out(got["y"], ref["y"], "y")
        if with_states:
            rep["ssm_state"] = check_rms(got["ssm_state"], ref["ssm_state"], "ssm_state")
    if with_states:
        # the oracle's conv state is the exact double of the io-dtype inputs
        check_exact(got["conv_state"], ref["conv_state"], "conv_state")
    return rep


def case(base: str, **kw) -> W.MixerConfig:
    return W.CONFIGS[base].with_(name=f"{base}+" + ",".join(f"{k}={v}" for k, v in kw.items()),
                                 **kw)
