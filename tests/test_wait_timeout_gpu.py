"""A bounded wait that runs out on the GPU, without a fault.

Every wait of a kernel on an asynchronous copy, an MMA or another CTA has a
time limit; when it runs out the kernel raises a flag, lets nothing stay in
flight and returns, so the context stays usable.  mamba2_debug_stall_waits
makes the first wait of every waiting kernel run out on purpose (a barrier that
nothing completes, 20 ms limit).  This checks that the host reads the flag
through mamba2_device_errors, and that the next ordinary calls on the same
context are correct again.
"""
import pytest
import torch

import mamba_ssd_scan_mixer_b200 as m2
import oracle
from mamba_ssd_scan_mixer_b200 import workloads as W

from harness import case, check_bf16_out, compare_prefill, dev_params, gpu_prefill, oracle_prefill

pytestmark = pytest.mark.gpu


def _step(cfg, params, st, si):
    dims = m2.dims_from_config(cfg)
    _, pp = dev_params(params)
    cs = st["conv_state"].cuda().contiguous()
    hs = st["ssm_state"].cuda().contiguous()
    v = W.split_packed(cfg, si["zxbcdt"].cuda())
    y = m2.step(dims, pp, v["xBC"], v["z"], v["dt_raw"], cs, hs)
    torch.cuda.synchronize()
    return y.cpu()


def test_wait_limit_runs_out_and_the_context_stays_usable():
    pcfg = case("zamba2_2p7b_prefill", batch=2, seqlen=700, nheads=8)   # tensor-core path
    dcfg = case("zamba2_2p7b_decode", batch=5, nheads=8)
    params = W.make_params(pcfg, 31)
    inp = W.make_prefill_inputs(pcfg, 31)
    dparams = W.make_params(dcfg, 31)
    dst = W.make_states(dcfg, 31)
    si = W.make_step_inputs(dcfg, 31, 0)
    assert m2.device_errors() == 0
    m2.debug_stall_waits(True)
    try:
        gpu_prefill(pcfg, inp, params)
        assert m2.device_errors() & 1, "prefill: no wait ran out"
        _step(dcfg, dparams, dst, si)
        assert m2.device_errors() & 1, "decode: no wait ran out"
    finally:
        m2.debug_stall_waits(False)
    assert m2.device_errors() == 0
    # the same context, ordinary calls: correct results and no flag
    got = gpu_prefill(pcfg, inp, params)
    compare_prefill(pcfg, got, oracle_prefill(pcfg, inp, params))
    y = _step(dcfg, dparams, dst, si)
    o = oracle.mixer_step(si["xBC"], si["z"], si["dt_raw"], dparams, dst["conv_state"],
                          dst["ssm_state"], nheads=dcfg.nheads, headdim=dcfg.headdim,
                          dstate=dcfg.dstate, ngroups=dcfg.ngroups)
    check_bf16_out(y, o["y"], "decode y")
    assert m2.device_errors() == 0
