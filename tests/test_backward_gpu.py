"""GPU parity of the prefill backward (mamba2_conv_ssd_prefill_backward) against the
fp64 autograd oracle (oracle/backward.py) on the same seeded inputs.

Tolerances: fp32 gradients (and every gradient of an fp32-I/O call) within
1e-3 * max(|o|, rms(o)) per element, as for the fp32 forward; the gradients the
library returns in bf16 (d_xBC, d_z, d_dt_raw, d_conv_state of a bf16 call)
within bf16's half-ulp plus 2e-2 * rms(o), as for the bf16 forward's y.
"""
import numpy as np
import pytest
import torch

import mamba_ssd_scan_mixer_b200 as m2
from mamba_ssd_scan_mixer_b200 import workloads as W
from oracle import backward as OB
from harness import case, check_bf16_out, check_f32, dev_params

pytestmark = pytest.mark.gpu

IO_GRADS = ("xBC", "z", "dt_raw", "conv_state")


def _run(cfg, seed, states, d_state_out):
    params = W.make_params(cfg, seed)
    inp = W.make_prefill_inputs(cfg, seed)
    st = W.make_states(cfg, seed) if states else None
    g = torch.Generator().manual_seed(1000 + seed)
    dy = torch.randn(cfg.batch, cfg.seqlen, cfg.d_inner, generator=g).to(cfg.torch_dtype)
    dhL = (0.1 * torch.randn(cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate, generator=g)
           if d_state_out else None)
    dims = m2.dims_from_config(cfg)
    v = W.split_packed(cfg, inp["zxbcdt"].cuda())
    _, pp = dev_params(params)
    cs = st["conv_state"].cuda().contiguous() if states else None
    hs = st["ssm_state"].cuda().contiguous() if states else None
    got = m2.prefill_backward(dims, pp, v["xBC"], v["z"], v["dt_raw"], dy.cuda().contiguous(),
                              conv_state_in=cs, ssm_state_in=hs,
                              d_ssm_state_out=None if dhL is None else dhL.cuda().contiguous())
    torch.cuda.synchronize()
    assert m2.device_errors() == 0
    got = {k: t.float().cpu().numpy() for k, t in got.items()}
    ref = OB.mixer_prefill_grads(
        inp["xBC"], inp["z"], inp["dt_raw"], params, dy, nheads=cfg.nheads,
        headdim=cfg.headdim, dstate=cfg.dstate, ngroups=cfg.ngroups,
        conv_state=st["conv_state"] if states else None,
        ssm_state=st["ssm_state"] if states else None, d_ssm_state=dhL,
        eps=cfg.norm_eps, norm_before_gate=cfg.norm_before_gate)
    keys = ["xBC", "z", "dt_raw", "conv_w", "conv_b", "dt_bias", "A", "D", "norm_w"]
    if states:
        keys += ["conv_state", "ssm_state"]
    for k in keys:
        if cfg.io_dtype == "bf16" and k in IO_GRADS:
            check_bf16_out(got[k], ref[k], f"d{k}")
        else:
            check_f32(got[k], ref[k], f"d{k}")


@pytest.mark.parametrize("cfg,states,dhl", [
    (case("tiny_f32", batch=2, seqlen=37, nheads=4, headdim=16, dstate=16), False, False),
    (case("tiny_f32", batch=1, seqlen=70, nheads=4, ngroups=2, headdim=32, dstate=64), True, True),
    (case("tiny_f32", batch=2, seqlen=50, nheads=2, headdim=16, dstate=128,
          norm_before_gate=True), True, False),
    (case("zamba2_2p7b_prefill", batch=1, seqlen=65, nheads=4, headdim=64, dstate=64), True, True),
    (case("zamba2_2p7b_prefill", batch=2, seqlen=40, nheads=6, ngroups=3, headdim=64,
          dstate=64), False, False),
], ids=lambda c: getattr(c, "name", str(c)))
def test_backward_matches_oracle(cfg, states, dhl):
    _run(cfg, 11, states, dhl)


@pytest.mark.parametrize("L", [1, 2, 3])
def test_backward_short_sequences_reach_the_conv_state(L):
    # fewer tokens than the conv window: the carried conv state's gradient comes
    # from several taps of the first tokens
    _run(case("tiny_f32", batch=1, seqlen=L, nheads=2, headdim=16, dstate=16), 12, True, True)


def test_backward_without_tokens_passes_the_state_gradient_through():
    cfg = case("tiny_f32", batch=2, seqlen=0, nheads=2, headdim=16, dstate=16)
    dims = m2.dims_from_config(cfg)
    params = W.make_params(cfg, 0)
    _, pp = dev_params(params)
    e = torch.empty(2, 0, cfg.packed_width, device="cuda")
    v = W.split_packed(cfg, e)
    cs = torch.randn(2, cfg.conv_dim, 4, device="cuda")
    hs = torch.randn(2, cfg.nheads, cfg.headdim, cfg.dstate, device="cuda")
    dhl = torch.randn_like(hs)
    g = m2.prefill_backward(dims, pp, v["xBC"], v["z"], v["dt_raw"],
                            torch.empty(2, 0, cfg.d_inner, device="cuda"), conv_state_in=cs,
                            ssm_state_in=hs, d_ssm_state_out=dhl)
    torch.cuda.synchronize()
    assert torch.equal(g["ssm_state"], dhl)
    assert torch.count_nonzero(g["conv_state"]) == 0
    for k in ("conv_w", "conv_b", "dt_bias", "A", "D", "norm_w"):
        assert torch.count_nonzero(g[k]) == 0, k
