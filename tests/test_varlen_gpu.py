"""Packed-sequence prefill (mamba2_conv_ssd_prefill_varlen) on the GPU.

Sequences of different lengths are packed along the token axis and described
by cu_seqlens; each is a separate request with its own conv and SSM state (the
chunked prefill with a cache of "Zamba2 hybrid architecture in Transformers",
qwbw.cn, section 三 step 3).  Checks:
* against the oracle run on each sequence alone (its own batch-1 prefill), with
  the harness's tolerances, for ragged lengths that cover the empty sequence,
  fewer tokens than the conv width, exact chunk multiples and chunk tails;
* bitwise equality with the fixed-length path where both apply (one sequence;
  equal lengths), which pins the packed layout to the tested batched one;
* offsets that break the contract are reported by mamba2_device_errors (bit 2)
  and leave every output untouched.
"""
import numpy as np
import pytest
import torch

import mamba_ssd_scan_mixer_b200 as m2
from mamba_ssd_scan_mixer_b200 import workloads as W

from harness import case, check_exact, compare_prefill, dev_params, gpu_prefill, oracle_prefill

pytestmark = pytest.mark.gpu


def _packed(lengths, nheads=8, ngroups=1, seed=0):
    T = int(sum(lengths))
    cfg = case("zamba2_2p7b_prefill", batch=1, seqlen=T, nheads=nheads, ngroups=ngroups)
    return cfg, W.make_params(cfg, seed), W.make_prefill_inputs(cfg, seed)


def _gpu_varlen(cfg, params, inp, lengths, states=None, states_in=False, cu=None):
    n, T = len(lengths), cfg.seqlen
    dims = m2.dims_from_config(cfg.with_(batch=n))
    v = W.split_packed(cfg, inp["zxbcdt"][0].cuda())
    if cu is None:
        cu = [0] + [int(x) for x in np.cumsum(lengths)]
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    _, pp = dev_params(params)
    if states is not None:
        cs = states["conv_state"].cuda().contiguous().clone()
        hs = states["ssm_state"].cuda().contiguous().clone()
    else:
        cs = torch.full((n, cfg.conv_dim, cfg.d_conv), 7.0, dtype=cfg.torch_dtype, device="cuda")
        hs = torch.full((n, cfg.nheads, cfg.headdim, cfg.dstate), 7.0, device="cuda")
    y = torch.full((T, cfg.d_inner), 7.0, dtype=cfg.torch_dtype, device="cuda")
    m2.prefill_varlen(dims, pp, v["xBC"], v["z"], v["dt_raw"], cu_d, cs, hs,
                      states_in=states_in, y=y)
    torch.cuda.synchronize()
    return {"y": y.cpu(), "conv_state": cs.cpu(), "ssm_state": hs.cpu()}


def _check_against_oracle(cfg, params, inp, lengths, got, states=None):
    t0 = 0
    for s, Ls in enumerate(lengths):
        c1 = cfg.with_(batch=1, seqlen=int(Ls))
        sub = {k: inp[k][:, t0:t0 + Ls] for k in ("xBC", "z", "dt_raw")}
        st = None if states is None else {k: v[s:s + 1] for k, v in states.items()}
        ref = oracle_prefill(c1, sub, params, states=st)
        g = {"y": got["y"][t0:t0 + Ls][None], "conv_state": got["conv_state"][s:s + 1],
             "ssm_state": got["ssm_state"][s:s + 1]}
        compare_prefill(c1, g, ref)
        t0 += Ls


@pytest.mark.parametrize("states_in", [True, False])
def test_varlen_ragged_matches_per_sequence_oracle(states_in):
    lengths = [1, 130, 256, 0, 700, 3, 128]
    cfg, params, inp = _packed(lengths, seed=31)
    st = W.make_states(cfg.with_(batch=len(lengths)), 31) if states_in else None
    got = _gpu_varlen(cfg, params, inp, lengths, states=st, states_in=states_in)
    assert m2.device_errors() == 0
    _check_against_oracle(cfg, params, inp, lengths, got, states=st)


def test_varlen_two_groups():
    lengths = [200, 77, 513]
    cfg, params, inp = _packed(lengths, nheads=16, ngroups=2, seed=32)
    st = W.make_states(cfg.with_(batch=len(lengths)), 32)
    got = _gpu_varlen(cfg, params, inp, lengths, states=st, states_in=True)
    assert m2.device_errors() == 0
    _check_against_oracle(cfg, params, inp, lengths, got, states=st)


def test_varlen_long_and_short_chains():
    # one sequence of 19 chunks (a full 16-chunk batch of state-pass loads and a
    # ragged 3-chunk remainder) beside sequences of one and two chunks
    lengths = [5, 2400, 129]
    cfg, params, inp = _packed(lengths, seed=34)
    st = W.make_states(cfg.with_(batch=len(lengths)), 34)
    got = _gpu_varlen(cfg, params, inp, lengths, states=st, states_in=True)
    assert m2.device_errors() == 0
    _check_against_oracle(cfg, params, inp, lengths, got, states=st)


@pytest.mark.parametrize("lengths", [[700], [384, 384]])
def test_varlen_equals_fixed_length_path_bitwise(lengths):
    # equal lengths: the packed call must reproduce the batched call exactly
    cfg, params, inp = _packed(lengths, seed=33)
    n, L = len(lengths), lengths[0]
    st = W.make_states(cfg.with_(batch=n), 33)
    got = _gpu_varlen(cfg, params, inp, lengths, states=st, states_in=True)
    fcfg = cfg.with_(batch=n, seqlen=L)
    finp = W.split_packed(fcfg, inp["zxbcdt"].reshape(n, L, -1))
    ref = gpu_prefill(fcfg, finp, params, states={k: v.clone() for k, v in st.items()},
                      states_in=True)
    check_exact(got["y"].reshape(n, L, -1), ref["y"], "y")
    check_exact(got["conv_state"], ref["conv_state"], "conv_state")
    check_exact(got["ssm_state"], ref["ssm_state"], "ssm_state")
    assert m2.device_errors() == 0


def test_varlen_invalid_offsets_are_reported_and_write_nothing():
    lengths = [100, 200]
    cfg, params, inp = _packed(lengths, seed=34)
    got = _gpu_varlen(cfg, params, inp, lengths, cu=[0, 250, 200])  # decreasing offsets
    assert m2.device_errors() & 4
    assert torch.all(got["y"] == 7.0)
    assert torch.all(got["conv_state"] == 7.0) and torch.all(got["ssm_state"] == 7.0)
    assert m2.device_errors() == 0


def test_varlen_fullsize_request_mix():
    # the benchmark's mix: eight requests of 1 .. 1600 tokens (4096 in all) on the
    # 2.7B-shaped mixer (80 heads), each continuing from its own carried state
    lengths = [1, 3, 127, 129, 512, 700, 1024, 1600]
    cfg, params, inp = _packed(lengths, nheads=80, seed=35)
    st = W.make_states(cfg.with_(batch=len(lengths)), 35)
    got = _gpu_varlen(cfg, params, inp, lengths, states=st, states_in=True)
    assert m2.device_errors() == 0
    _check_against_oracle(cfg, params, inp, lengths, got, states=st)
