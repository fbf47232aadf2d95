"""Host-side tests of the C ABI (no GPU needed).

The library must load, export every function that include/*.h declares, size
its workspace, and reject bad arguments with the documented status codes
before it touches CUDA (validation runs on the host; fake device addresses are
never dereferenced).
"""
import ctypes
import glob
import os
import re

import pytest

import mamba_ssd_scan_mixer_b200 as m2
from mamba_ssd_scan_mixer_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, UNSUPPORTED, WORKSPACE = 0, -1, -2, -3


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names.update(re.findall(r"MAMBA2_API[^;(]*?\b(mamba2_\w+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert "mamba2_conv_ssd_prefill" in names and "mamba2_ssd_step" in names
    lib = m2.lib()
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_library_exports_nothing_undeclared():
    # -fvisibility=hidden: the only dynamic symbols with our prefix are the API
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", m2.library_path], capture_output=True,
                         text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    ours = {s for s in exported if s.startswith("mamba2_")}
    assert ours == set(_declared_functions())


def test_status_strings_and_version():
    assert m2.status_string(0) == "ok"
    assert "workspace" in m2.status_string(WORKSPACE)
    assert m2.lib().mamba2_version() >= 100


def _dims(**kw):
    cfg = W.CONFIGS["zamba2_2p7b_prefill"]
    d = m2.dims_from_config(cfg)
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_workspace_size_scales_and_rejects_bad_dims():
    lib = m2.lib()
    d = _dims()
    ws = lib.mamba2_prefill_workspace_size(ctypes.byref(d))
    assert ws > 0
    d2 = _dims(seqlen=8192)
    assert lib.mamba2_prefill_workspace_size(ctypes.byref(d2)) >= 2 * ws - 4096
    for bad in (dict(ngroups=3), dict(d_conv=3), dict(headdim=48), dict(chunk_size=100),
                dict(norm_eps=0.0), dict(io_dtype=7)):
        assert lib.mamba2_prefill_workspace_size(ctypes.byref(_dims(**bad))) == 0, bad


# fake, suitably aligned device addresses: validation never dereferences them
A0 = 1 << 20


def _fake_params():
    return m2.Mamba2Params(A0, A0 + 0x1000, A0 + 0x2000, A0 + 0x3000, A0 + 0x4000, A0 + 0x5000)


def _call_prefill(d, **kw):
    lib = m2.lib()
    cd, di = d.nheads * d.headdim + 2 * d.ngroups * d.dstate, d.nheads * d.headdim
    args = dict(params=_fake_params(), xBC=A0 + 0x10000, ld_x=cd, z=A0 + 0x20000, ld_z=di,
                dt=A0 + 0x30000, ld_dt=d.nheads, y=A0 + 0x40000, cs=A0 + 0x50000,
                hs=A0 + 0x60000, states_in=0, ws=A0 + 0x100000,
                ws_bytes=lib.mamba2_prefill_workspace_size(ctypes.byref(d)) or 1)
    args.update(kw)
    p = args["params"]
    return lib.mamba2_conv_ssd_prefill(
        ctypes.byref(d), ctypes.byref(p) if p is not None else None, args["xBC"], args["ld_x"],
        args["z"], args["ld_z"], args["dt"], args["ld_dt"], args["y"], args["cs"], args["hs"],
        args["states_in"], args["ws"], args["ws_bytes"], None)


@pytest.mark.parametrize("kw,expect", [
    (dict(params=None), INVALID),
    (dict(xBC=None), INVALID),
    (dict(z=None), INVALID),
    (dict(y=None), INVALID),
    (dict(ld_x=100), INVALID),                 # row stride < conv_dim
    (dict(ld_z=5120 + 4), INVALID),            # not a multiple of 8
    (dict(xBC=A0 + 0x10008), INVALID),         # not 16-byte aligned
    (dict(y=A0 + 0x40002), INVALID),
    (dict(hs=A0 + 0x60004), INVALID),
    (dict(states_in=1, cs=None), INVALID),     # states_in needs both states
    (dict(states_in=2), INVALID),
    (dict(ws=None), WORKSPACE),
    (dict(ws_bytes=1024), WORKSPACE),
    (dict(ws=A0 + 0x100010), WORKSPACE),       # workspace not 256-byte aligned
])
def test_prefill_rejects_bad_arguments(kw, expect):
    assert _call_prefill(_dims(), **kw) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(nheads=80, ngroups=3), INVALID),
    (dict(batch=-1), INVALID),
    (dict(seqlen=-5), INVALID),
    (dict(norm_before_gate=2), INVALID),
    (dict(d_conv=2), UNSUPPORTED),
    (dict(dstate=256), UNSUPPORTED),
    (dict(headdim=128), UNSUPPORTED),
    (dict(chunk_size=32), UNSUPPORTED),
])
def test_prefill_rejects_bad_dims(kw, expect):
    assert _call_prefill(_dims(**kw)) == expect


def test_empty_batch_is_a_no_op():
    assert _call_prefill(_dims(batch=0), xBC=None, z=None, y=None, ws=None) == OK


def test_step_rejects_bad_arguments():
    lib = m2.lib()
    cfg = W.CONFIGS["zamba2_2p7b_decode"]
    d = m2.dims_from_config(cfg)
    p = _fake_params()

    def call(**kw):
        a = dict(x=A0 + 0x10000, lx=cfg.conv_dim, z=A0 + 0x20000, lz=cfg.d_inner,
                 dt=A0 + 0x30000, ld=cfg.nheads, y=A0 + 0x40000, cs=A0 + 0x50000,
                 hs=A0 + 0x60000)
        a.update(kw)
        return lib.mamba2_ssd_step(ctypes.byref(d), ctypes.byref(p), a["x"], a["lx"], a["z"],
                                   a["lz"], a["dt"], a["ld"], a["y"], a["cs"], a["hs"], None)

    assert call(cs=None) == INVALID
    assert call(hs=None) == INVALID
    assert call(hs=A0 + 0x60008) == INVALID
    assert call(lx=cfg.conv_dim - 8) == INVALID
    assert call(lz=cfg.d_inner + 1) == INVALID


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(m2, "_lib", None)
    monkeypatch.setattr(m2, "library_path", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        m2.lib()


def test_debug_stall_rejects_bad_values():
    # validated before any CUDA call, so this runs without a GPU
    assert m2.lib().mamba2_debug_stall_waits(2) == INVALID
    assert m2.lib().mamba2_debug_stall_waits(-1) == INVALID


def test_noalloc_rejects_bad_dims_before_touching_the_device():
    lib = m2.lib()
    p = _fake_params()
    for kw, expect in [(dict(nheads=6, ngroups=4), INVALID), (dict(d_conv=2), UNSUPPORTED),
                       (dict(seqlen=-1), INVALID)]:
        d = _dims(**kw)
        st = lib.mamba2_conv_ssd_prefill_noalloc(ctypes.byref(d), ctypes.byref(p), A0, 5248,
                                                 A0, 5120, A0, 80, A0, None, None, 0, None)
        assert st == expect, kw


# ---- packed-sequence prefill: validated on the host before any CUDA call

def _call_varlen(d, **kw):
    lib = m2.lib()
    cd, di = d.nheads * d.headdim + 2 * d.ngroups * d.dstate, d.nheads * d.headdim
    args = dict(params=_fake_params(), xBC=A0 + 0x10000, ld_x=cd, z=A0 + 0x20000, ld_z=di,
                dt=A0 + 0x30000, ld_dt=d.nheads, cu=A0 + 0x70000, y=A0 + 0x40000,
                cs=A0 + 0x50000, hs=A0 + 0x60000, states_in=0, ws=A0 + 0x100000,
                ws_bytes=lib.mamba2_prefill_varlen_workspace_size(ctypes.byref(d)) or 1)
    args.update(kw)
    p = args["params"]
    return lib.mamba2_conv_ssd_prefill_varlen(
        ctypes.byref(d), ctypes.byref(p) if p is not None else None, args["xBC"], args["ld_x"],
        args["z"], args["ld_z"], args["dt"], args["ld_dt"], args["cu"], args["y"], args["cs"],
        args["hs"], args["states_in"], args["ws"], args["ws_bytes"], None)


def test_varlen_workspace_size():
    lib = m2.lib()
    d = _dims(batch=7, seqlen=4096)  # 7 sequences, 4096 tokens in all
    ws = lib.mamba2_prefill_varlen_workspace_size(ctypes.byref(d))
    fixed = lib.mamba2_prefill_workspace_size(ctypes.byref(_dims(batch=1, seqlen=4096)))
    # room for up to ceil(4096 / 128) + 7 chunks instead of 32
    assert fixed < ws < fixed * (32 + 7 + 1) / 32
    # the CUDA-core configurations have no packed-sequence path
    assert lib.mamba2_prefill_varlen_workspace_size(ctypes.byref(_dims(io_dtype=0))) == 0
    assert lib.mamba2_prefill_varlen_workspace_size(ctypes.byref(_dims(headdim=32))) == 0


@pytest.mark.parametrize("kw,expect", [
    (dict(cu=None), INVALID),                  # no offsets
    (dict(cu=A0 + 0x70002), INVALID),          # offsets not 4-byte aligned
    (dict(params=None), INVALID),
    (dict(xBC=A0 + 0x10008), INVALID),
    (dict(states_in=1, hs=None), INVALID),
    (dict(ws=None), WORKSPACE),
    (dict(ws_bytes=4096), WORKSPACE),
])
def test_varlen_rejects_bad_arguments(kw, expect):
    assert _call_varlen(_dims(batch=3, seqlen=1000), **kw) == expect


def test_varlen_unsupported_configurations():
    for bad in (dict(io_dtype=0), dict(headdim=32), dict(dstate=128)):
        d = _dims(batch=3, seqlen=1000, **bad)
        assert _call_varlen(d, ld_x=d.nheads * d.headdim + 2 * d.ngroups * d.dstate,
                            ld_z=d.nheads * d.headdim) == UNSUPPORTED, bad


# ---- prefill backward: validated on the host before any CUDA call

def _call_backward(d, **kw):
    lib = m2.lib()
    cd, di = d.nheads * d.headdim + 2 * d.ngroups * d.dstate, d.nheads * d.headdim
    a = dict(params=_fake_params(), xBC=A0 + 0x10000, ld_x=cd, z=A0 + 0x20000, ld_z=di,
             dt=A0 + 0x30000, ld_dt=d.nheads, cs=None, hs=None, dy=A0 + 0x40000, dhl=None,
             dxbc=A0 + 0x50000, dz=A0 + 0x60000, ddt=A0 + 0x70000, dw=A0 + 0x80000,
             db=A0 + 0x90000, ddtb=A0 + 0xa0000, dA=A0 + 0xb0000, dD=A0 + 0xc0000,
             dnw=A0 + 0xd0000, dcs=None, dhs=None, ws=A0 + 0x100000,
             ws_bytes=lib.mamba2_prefill_backward_workspace_size(ctypes.byref(d)) or 1)
    a.update(kw)
    p = a["params"]
    return lib.mamba2_conv_ssd_prefill_backward(
        ctypes.byref(d), ctypes.byref(p) if p is not None else None, a["xBC"], a["ld_x"], a["z"],
        a["ld_z"], a["dt"], a["ld_dt"], a["cs"], a["hs"], a["dy"], a["dhl"], a["dxbc"], a["dz"],
        a["ddt"], a["dw"], a["db"], a["ddtb"], a["dA"], a["dD"], a["dnw"], a["dcs"], a["dhs"],
        a["ws"], a["ws_bytes"], None)


def test_backward_workspace_size():
    lib = m2.lib()
    d = _dims(batch=1, seqlen=4096)
    ws = lib.mamba2_prefill_backward_workspace_size(ctypes.byref(d))
    states = 4096 * 80 * 64 * 64 * 4  # the state after every token
    assert states < ws < 2 * states
    assert lib.mamba2_prefill_backward_workspace_size(ctypes.byref(_dims(d_conv=2))) == 0


@pytest.mark.parametrize("kw,expect", [
    (dict(params=None), INVALID),
    (dict(dy=None), INVALID),
    (dict(dw=None), INVALID),
    (dict(dxbc=A0 + 0x50001), INVALID),       # misaligned bf16 gradient
    (dict(dhs=A0 + 0xe0002), INVALID),        # misaligned fp32 gradient
    (dict(ld_x=8), INVALID),                  # row stride below conv_dim
    (dict(ws=None), WORKSPACE),
    (dict(ws_bytes=4096), WORKSPACE),
])
def test_backward_rejects_bad_arguments(kw, expect):
    assert _call_backward(_dims(batch=2, seqlen=300), **kw) == expect


def test_backward_unsupported_configurations():
    for bad in (dict(d_conv=2), dict(dstate=256), dict(headdim=128)):
        assert _call_backward(_dims(batch=2, seqlen=300, **bad)) == UNSUPPORTED, bad


def test_host_workspace_size():
    lib = m2.lib()
    d = _dims()  # b1 L4096: eight pieces of 512 tokens
    ws = lib.mamba2_prefill_host_workspace_size(ctypes.byref(d))
    piece = lib.mamba2_prefill_workspace_size(ctypes.byref(_dims(seqlen=512)))
    whole = lib.mamba2_prefill_workspace_size(ctypes.byref(d))
    # one piece's workspace plus two staged pieces each way and the states
    assert piece < ws < whole
    assert lib.mamba2_prefill_host_workspace_size(ctypes.byref(_dims(ngroups=3))) == 0


def _call_host(d, **kw):
    lib = m2.lib()
    cd, di = d.nheads * d.headdim + 2 * d.ngroups * d.dstate, d.nheads * d.headdim
    args = dict(params=_fake_params(), xBC=A0 + 0x10000, ld_x=cd, z=A0 + 0x20000, ld_z=di,
                dt=A0 + 0x30000, ld_dt=d.nheads, y=A0 + 0x40000, cs=A0 + 0x50000,
                hs=A0 + 0x60000, states_in=0, ws=A0 + 0x100000,
                ws_bytes=lib.mamba2_prefill_host_workspace_size(ctypes.byref(d)) or 1)
    args.update(kw)
    p = args["params"]
    return lib.mamba2_conv_ssd_prefill_host(
        ctypes.byref(d), ctypes.byref(p) if p is not None else None, args["xBC"], args["ld_x"],
        args["z"], args["ld_z"], args["dt"], args["ld_dt"], args["y"], args["cs"], args["hs"],
        args["states_in"], args["ws"], args["ws_bytes"], None)


@pytest.mark.parametrize("kw,expect", [
    (dict(params=None), INVALID),
    (dict(xBC=None), INVALID),
    (dict(y=None), INVALID),
    (dict(ld_z=5), INVALID),                   # row stride below the width
    (dict(states_in=1, cs=None), INVALID),
    (dict(states_in=2), INVALID),
    (dict(ws=None), WORKSPACE),
    (dict(ws=A0 + 0x100010), WORKSPACE),       # device workspace not 256-byte aligned
    (dict(ws_bytes=4096), WORKSPACE),
])
def test_host_entry_rejects_bad_arguments(kw, expect):
    # host pointers need no alignment; everything here is rejected before CUDA
    assert _call_host(_dims(batch=2, seqlen=1000), **kw) == expect


def test_host_entry_empty_batch_and_bad_dims():
    assert _call_host(_dims(batch=0)) == OK
    assert _call_host(_dims(ngroups=3)) == INVALID
    assert _call_host(_dims(d_conv=3)) == UNSUPPORTED
