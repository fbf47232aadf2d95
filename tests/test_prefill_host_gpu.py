"""GPU parity of the host-buffer prefill (mamba2_conv_ssd_prefill_host): inputs, y
and states in page-locked host memory, the sequence cut into pieces of whole
chunks that continue from one another's states (the chunked prefill of
"Zamba2 hybrid architecture in Transformers", qwbw.cn, section 三 step 3), with
the copies overlapped.  Checked against the fp64 oracle with the prefill's own
tolerances, and against the one-call device prefill."""
import pytest
import torch

import mamba_ssd_scan_mixer_b200 as m2
from mamba_ssd_scan_mixer_b200 import workloads as W
from harness import case, compare_prefill, dev_params, gpu_prefill, oracle_prefill

pytestmark = pytest.mark.gpu


def _host(cfg, inp, params, states=None, states_in=False):
    dims = m2.dims_from_config(cfg)
    _, pp = dev_params(params)
    packed = inp["zxbcdt"].contiguous().pin_memory()
    v = W.split_packed(cfg, packed)
    out = {}
    cs = hs = None
    if states is not None:
        cs = states["conv_state"].clone().pin_memory()
        hs = states["ssm_state"].clone().pin_memory()
    y = m2.prefill_host(dims, pp, v["xBC"], v["z"], v["dt_raw"], cs, hs, states_in=states_in)
    assert m2.device_errors() == 0
    out["y"] = y
    if cs is not None:
        out["conv_state"], out["ssm_state"] = cs, hs
    return out


@pytest.mark.parametrize("cfg,states_in", [
    # 4 pieces of 256 tokens, the last (232) shorter with two batch rows
    (case("zamba2_2p7b_prefill", batch=2, seqlen=1000, nheads=8, ngroups=2), True),
    (case("zamba2_2p7b_prefill", batch=2, seqlen=1000, nheads=8, ngroups=2), False),
    # one piece shorter than a chunk; fp32 I/O (CUDA-core path)
    (case("tiny_f32", batch=2, seqlen=37, nheads=4, headdim=16, dstate=16), True),
    # 6 pieces of 256 over three rows (the last 20 tokens), norm before the gate
    (case("zamba2_2p7b_prefill", batch=3, seqlen=1300, nheads=4, norm_before_gate=True), True),
], ids=lambda c: getattr(c, "name", str(c)))
def test_host_entry_matches_oracle(cfg, states_in):
    params = W.make_params(cfg, 5)
    inp = W.make_prefill_inputs(cfg, 5)
    st = W.make_states(cfg, 5)
    got = _host(cfg, inp, params, states=st, states_in=states_in)
    ref = oracle_prefill(cfg, inp, params, states=st if states_in else None)
    print(cfg.name, states_in, compare_prefill(cfg, got, ref))


def test_host_entry_full_size_matches_device_entry():
    # the 2.7B workload (8 pieces of 512 tokens) against the one-call device prefill:
    # both within the prefill's tolerance of each other
    cfg = W.CONFIGS["zamba2_2p7b_prefill"]
    params = W.make_params(cfg, 2)
    inp = W.make_prefill_inputs(cfg, 2)
    st = W.make_states(cfg, 2)
    got = _host(cfg, inp, params, states=st, states_in=True)
    dev = gpu_prefill(cfg, inp, params, states={k: v.clone() for k, v in st.items()},
                      states_in=True)
    rep = compare_prefill(cfg, got, {k: v.double().numpy() for k, v in dev.items()})
    print(rep)


@pytest.mark.parametrize("states_in", [True, False])
def test_host_entry_without_tokens(states_in):
    cfg = case("zamba2_2p7b_prefill", batch=2, seqlen=0, nheads=4)
    dims = m2.dims_from_config(cfg)
    _, pp = dev_params(W.make_params(cfg, 0))
    st = W.make_states(cfg, 0)
    cs = st["conv_state"].clone().pin_memory()
    hs = st["ssm_state"].clone().pin_memory()
    e = torch.empty(2, 0, cfg.packed_width, dtype=cfg.torch_dtype).pin_memory()
    v = W.split_packed(cfg, e)
    m2.prefill_host(dims, pp, v["xBC"], v["z"], v["dt_raw"], cs, hs, states_in=states_in)
    if states_in:  # the states pass through
        assert torch.equal(cs, st["conv_state"]) and torch.equal(hs, st["ssm_state"])
    else:  # they start (and stay) at zero
        assert torch.count_nonzero(cs) == 0 and torch.count_nonzero(hs) == 0


def test_host_entry_separate_views_equal_packed_rows():
    # xBC, z and dt_raw as three separate host tensors (per-view copies) against the
    # same values in one packed buffer (whole-row copies): the same result
    cfg = case("zamba2_2p7b_prefill", batch=2, seqlen=900, nheads=8)
    params = W.make_params(cfg, 6)
    inp = W.make_prefill_inputs(cfg, 6)
    st = W.make_states(cfg, 6)
    packed = _host(cfg, inp, params, states=st, states_in=True)
    dims = m2.dims_from_config(cfg)
    _, pp = dev_params(params)
    sep = {k: inp[k].contiguous().pin_memory() for k in ("xBC", "z", "dt_raw")}
    cs = st["conv_state"].clone().pin_memory()
    hs = st["ssm_state"].clone().pin_memory()
    y = m2.prefill_host(dims, pp, sep["xBC"], sep["z"], sep["dt_raw"], cs, hs, states_in=True)
    assert torch.equal(y, packed["y"])
    assert torch.equal(cs, packed["conv_state"]) and torch.equal(hs, packed["ssm_state"])
