"""The allocation-free prefill entry point against the ordinary one.

mamba2_conv_ssd_prefill_noalloc exists for callers that may not allocate
device memory themselves (a plugin inside a runtime whose pool owns every
device allocation, or a latency-critical path that cannot take cudaMalloc's
synchronisation).  It must give the results of mamba2_conv_ssd_prefill with a
caller-allocated workspace.  Two calls in a row on different inputs check
that the scratch left over from one call does not leak into the next.

This file is collected last, and passes run alone or after the other tests.
"""
import pytest
import torch

import mamba_ssd_scan_mixer_b200 as m2
from mamba_ssd_scan_mixer_b200 import workloads as W

from harness import case, dev_params

pytestmark = pytest.mark.gpu


def _inputs(cfg, seed):
    params = W.make_params(cfg, seed)
    views = W.split_packed(cfg, W.make_prefill_inputs(cfg, seed)["zxbcdt"].cuda())
    st = W.make_states(cfg, seed)
    return params, views, st


def _outputs(cfg, seed, noalloc):
    params, v, st = _inputs(cfg, seed)
    _, pp = dev_params(params)
    dims = m2.dims_from_config(cfg)
    cs = st["conv_state"].cuda()
    hs = st["ssm_state"].cuda()
    y = torch.empty(cfg.batch, cfg.seqlen, cfg.d_inner, dtype=cfg.torch_dtype, device="cuda")
    if noalloc:
        m2.mamba2_conv_ssd_prefill_noalloc(dims, pp, v["xBC"], v["z"], v["dt_raw"], y, cs, hs,
                                           states_in=True)
    else:
        m2.prefill(dims, pp, v["xBC"], v["z"], v["dt_raw"], cs, hs, states_in=True, y=y)
    torch.cuda.synchronize()
    return {"y": y.cpu(), "conv_state": cs.cpu(), "ssm_state": hs.cpu()}


@pytest.mark.parametrize("cfg", [
    case("zamba2_2p7b_prefill", batch=2, seqlen=700, nheads=8, ngroups=2),
    case("tiny_f32", batch=2, seqlen=300, nheads=4),
], ids=lambda c: c.name)
def test_noalloc_prefill_matches_workspace_prefill_twice(cfg):
    assert m2.mamba2_prefill_workspace_size(m2.dims_from_config(cfg)) <= 64 * 1024 * 1024
    # a larger call of another shape first, so that the scratch holds differently
    # laid-out leftovers when the checked calls run
    other = cfg.with_(batch=3, seqlen=1500, nheads=cfg.nheads * 2, ngroups=1)
    assert m2.mamba2_prefill_workspace_size(m2.dims_from_config(other)) <= 64 * 1024 * 1024
    _outputs(other, 10, noalloc=True)
    for seed in (11, 12):  # two calls in a row, different inputs
        ref = _outputs(cfg, seed, noalloc=False)
        got = _outputs(cfg, seed, noalloc=True)
        # same kernels, same launch configuration, no atomics: bitwise identical
        for k in ("y", "conv_state", "ssm_state"):
            assert torch.equal(got[k], ref[k]), k


def test_noalloc_prefill_rejects_problems_beyond_the_static_scratch():
    cfg = W.CONFIGS["zamba2_7b_long_prefill"]
    dims = m2.dims_from_config(cfg)
    assert m2.mamba2_prefill_workspace_size(dims) > 64 * 1024 * 1024
    # full-size (uninitialised) buffers, so that even a wrongly accepted call stays in bounds
    params = W.make_params(cfg, 0)
    _, pp = dev_params(params)
    packed = torch.empty(cfg.batch, cfg.seqlen, cfg.packed_width, dtype=cfg.torch_dtype,
                         device="cuda")
    v = W.split_packed(cfg, packed)
    y = torch.empty(cfg.batch, cfg.seqlen, cfg.d_inner, dtype=cfg.torch_dtype, device="cuda")
    with pytest.raises(m2.Mamba2Error) as ei:
        m2.mamba2_conv_ssd_prefill_noalloc(dims, pp, v["xBC"], v["z"], v["dt_raw"], y)
    assert ei.value.status == -3  # MAMBA2_ERR_WORKSPACE
