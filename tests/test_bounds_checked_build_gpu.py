"""The bounds-checked build of the library (libmamba2ssd_checked.so), the
debugging aid that stands in for a memory checker: every plain global load and
store of the tensor-core prefill kernels and of the decode kernel is checked
against the extent and alignment of the buffer it addresses, and a failing
access is skipped and reported by mamba2_device_errors (bit 1).

Odd and ragged shapes run through the checked library in a child process (so
that it is the only build loaded there); the results must match the oracle and
no access may have been flagged.
"""
import os
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu

CHILD = textwrap.dedent("""
    import sys
    sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
    import torch
    import mamba_ssd_scan_mixer_b200 as m2
    import oracle
    from mamba_ssd_scan_mixer_b200 import workloads as W
    from harness import case, compare_prefill, gpu_prefill, oracle_prefill, check_bf16_out, dev_params
    assert m2.library_path.endswith("libmamba2ssd_checked.so"), m2.library_path
    cases = [
        (case("zamba2_2p7b_prefill", batch=2, seqlen=333, nheads=6, ngroups=2), True),
        (case("zamba2_2p7b_prefill", batch=1, seqlen=1100, nheads=80), False),
        (case("zamba2_2p7b_prefill", batch=3, seqlen=129, nheads=13), True),
        (case("zamba2_2p7b_prefill", batch=2, seqlen=5, nheads=4), True),
        (case("zamba2_2p7b_prefill", batch=2, seqlen=300, nheads=4, norm_before_gate=True), True),
    ]
    for cfg, states_in in cases:
        params = W.make_params(cfg, 5); inp = W.make_prefill_inputs(cfg, 5)
        st = W.make_states(cfg, 5) if states_in else None
        got = gpu_prefill(cfg, inp, params, states=st, states_in=states_in)
        compare_prefill(cfg, got, oracle_prefill(cfg, inp, params, states=st))
        flags = m2.device_errors()
        assert flags == 0, (cfg.name, flags)
    for cfg in [case("zamba2_2p7b_decode", batch=37, nheads=8),
                case("zamba2_2p7b_decode", batch=3, nheads=6, ngroups=2)]:
        params = W.make_params(cfg, 6); st = W.make_states(cfg, 6)
        dims = m2.dims_from_config(cfg); _, pp = dev_params(params)
        cs = st["conv_state"].cuda().contiguous(); hs = st["ssm_state"].cuda().contiguous()
        ocs, ohs = st["conv_state"], st["ssm_state"]
        for s in range(3):
            si = W.make_step_inputs(cfg, 6, s)
            v = W.split_packed(cfg, si["zxbcdt"].cuda())
            y = m2.step(dims, pp, v["xBC"], v["z"], v["dt_raw"], cs, hs).cpu()
            o = oracle.mixer_step(si["xBC"], si["z"], si["dt_raw"], params, ocs, ohs,
                                  nheads=cfg.nheads, headdim=64, dstate=64, ngroups=cfg.ngroups)
            ocs, ohs = o["conv_state"], o["ssm_state"]
            check_bf16_out(y, o["y"], "decode y")
        flags = m2.device_errors()
        assert flags == 0, (cfg.name, flags)
    print("CHECKED-OK")
""")


def test_checked_build_flags_no_access_on_odd_shapes():
    from mamba_ssd_scan_mixer_b200 import build
    lib = build.LIB_CHECKED
    if not os.path.exists(lib):
        build.build(checked=True)
    env = dict(os.environ, MAMBA2SSD_LIBRARY=lib)
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))],
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "CHECKED-OK" in r.stdout, (r.stdout[-3000:], r.stderr[-3000:])
