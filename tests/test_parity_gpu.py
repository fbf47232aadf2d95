"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle on
the same seeded inputs, at small sizes that span several tiles and a ragged
tail, at the full benchmark sizes, and on the edge cases of the method."""
import numpy as np
import pytest
import torch

import mamba_ssd_scan_mixer_b200 as m2
import oracle
from mamba_ssd_scan_mixer_b200 import workloads as W

from harness import (case, check_bf16_out, check_exact, check_f32, check_rms, compare_prefill,
                     dev_params, gpu_prefill, oracle_prefill)

pytestmark = pytest.mark.gpu


def _run_case(cfg, seed=0, states_in=False):
    params = W.make_params(cfg, seed)
    inp = W.make_prefill_inputs(cfg, seed)
    states = W.make_states(cfg, seed) if states_in else None
    got = gpu_prefill(cfg, inp, params, states=states, states_in=states_in)
    ref = oracle_prefill(cfg, inp, params, states=states)
    return compare_prefill(cfg, got, ref)


# ---------------------------------------------------------------- small cases

def test_tiny_f32_config():
    rep = _run_case(W.CONFIGS["tiny_f32"])
    print("tiny_f32", rep)


@pytest.mark.parametrize("cfg", [
    # several chunks and token tiles, ragged tail, two groups
    case("zamba2_2p7b_prefill", batch=2, seqlen=700, nheads=8, ngroups=2),
    case("zamba2_2p7b_prefill", batch=1, seqlen=333, nheads=4, chunk_size=64),
    case("zamba2_2p7b_prefill", batch=3, seqlen=129, nheads=6, ngroups=3, chunk_size=128),
    case("zamba2_2p7b_prefill", batch=2, seqlen=300, nheads=4, norm_before_gate=True),
    # head blocks of the tensor-core output kernel: odd heads per group (a lone head in
    # the last pair of the chunk-state kernel), 13 and 17 heads (blocks of unequal
    # size), two groups of 16 heads, and 20 heads over 24 (row, chunk) pairs
    case("zamba2_2p7b_prefill", batch=1, seqlen=300, nheads=6, ngroups=2),
    case("zamba2_2p7b_prefill", batch=1, seqlen=260, nheads=13),
    case("zamba2_2p7b_prefill", batch=1, seqlen=200, nheads=17),
    case("zamba2_2p7b_prefill", batch=2, seqlen=256, nheads=32, ngroups=2),
    case("zamba2_2p7b_prefill", batch=3, seqlen=1000, nheads=20),
    # 80 heads (16 blocks of 5 per (chunk, group); several chunk-state items per CTA,
    # crossing (row, chunk) keys), 64 heads (13 blocks of 4 or 5), 80 heads over 24
    # (row, chunk) pairs (384 units: three rounds of the 144-CTA grid, blocks that
    # change heads from unit to unit) and 96 heads in one group (20 blocks)
    case("zamba2_2p7b_prefill", batch=1, seqlen=1100, nheads=80),
    case("zamba2_2p7b_prefill", batch=2, seqlen=640, nheads=64),
    case("zamba2_2p7b_prefill", batch=2, seqlen=1500, nheads=80),
    case("zamba2_2p7b_prefill", batch=1, seqlen=400, nheads=96),
    # state-pass chains longer than one 16-chunk batch of loads, with a shorter
    # last batch (21 and 17 chunks, the last one ragged)
    case("zamba2_2p7b_prefill", batch=2, seqlen=2600, nheads=16),
    case("zamba2_2p7b_prefill", batch=1, seqlen=2100, nheads=8, ngroups=2),
    case("zamba2_2p7b_prefill", batch=1, seqlen=257, nheads=4, headdim=32, dstate=128),
    case("zamba2_2p7b_prefill", batch=1, seqlen=200, nheads=4, headdim=16, dstate=32),
    case("tiny_f32", batch=2, seqlen=517, nheads=6, ngroups=2, headdim=64, dstate=64,
         chunk_size=256),
    case("tiny_f32", batch=1, seqlen=130, headdim=32, dstate=128, chunk_size=128),
], ids=lambda c: c.name)
@pytest.mark.parametrize("states_in", [False, True])
def test_small_cases(cfg, states_in):
    rep = _run_case(cfg, seed=3, states_in=states_in)
    print(cfg.name, states_in, rep)


@pytest.mark.parametrize("L", [1, 2, 3, 4, 5, 63, 64, 65])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_short_sequences_take_conv_context_from_the_state(L, io):
    cfg = case("zamba2_2p7b_prefill", batch=2, seqlen=L, nheads=4, io_dtype=io, chunk_size=64)
    _run_case(cfg, seed=5, states_in=True)


@pytest.mark.parametrize("states_in", [False, True])
def test_empty_sequence(states_in):
    cfg = case("zamba2_2p7b_prefill", batch=2, seqlen=0, nheads=4)
    params = W.make_params(cfg, 0)
    inp = W.make_prefill_inputs(cfg, 0)
    st = W.make_states(cfg, 0)
    got = gpu_prefill(cfg, inp, params, states={k: v.clone() for k, v in st.items()},
                      states_in=states_in)
    assert got["y"].numel() == 0
    if states_in:
        check_exact(got["conv_state"], st["conv_state"], "conv_state")
        check_exact(got["ssm_state"], st["ssm_state"], "ssm_state")
    else:
        assert torch.count_nonzero(got["conv_state"]) == 0
        assert torch.count_nonzero(got["ssm_state"]) == 0


def test_dt_zero_gives_D_skip_on_gpu():
    # dt_raw = -inf: softplus gives 0 exactly, the state is frozen and y_pre = C h0 + D x
    cfg = case("zamba2_2p7b_prefill", batch=1, seqlen=300, nheads=4, io_dtype="f32")
    params = W.make_params(cfg, 1)
    inp = W.make_prefill_inputs(cfg, 1)
    inp["dt_raw"][...] = float("-inf")
    st = W.make_states(cfg, 1)
    got = gpu_prefill(cfg, inp, params, states={k: v.clone() for k, v in st.items()},
                      states_in=True)
    ref = oracle_prefill(cfg, inp, params, states=st)
    compare_prefill(cfg, got, ref)
    check_exact(got["ssm_state"], st["ssm_state"], "frozen ssm_state")


# ---------------------------------------------------------------- tensor-core edge cases
# bf16 I/O at headdim = d_state = 64 runs the tensor-core path

def _tc_case(seed, **kw):
    cfg = case("zamba2_2p7b_prefill", batch=2, seqlen=700, nheads=8, **kw)
    return cfg, W.make_params(cfg, seed), W.make_prefill_inputs(cfg, seed), W.make_states(cfg, seed)


def test_tc_dt_zero_freezes_state_and_gives_D_skip():
    # dt_raw = -inf in bf16: softplus gives 0 exactly, so the carried state passes
    # through every chunk unchanged (bit-exact) and y_pre = C h0 + D x
    cfg, params, inp, st = _tc_case(21)
    inp["dt_raw"][...] = float("-inf")
    got = gpu_prefill(cfg, inp, params, states={k: v.clone() for k, v in st.items()},
                      states_in=True)
    ref = oracle_prefill(cfg, inp, params, states=st)
    compare_prefill(cfg, got, ref)
    check_exact(got["ssm_state"], st["ssm_state"], "frozen ssm_state")
    assert m2.device_errors() == 0


def test_tc_strong_decay_forgets():
    # A = -1e4: exp(dt A) underflows to 0 after every token, so the state holds only
    # the last token's dt x B^T and y only the diagonal (plus D) term
    cfg, params, inp, st = _tc_case(22)
    params = dict(params, A=torch.full_like(params["A"], -1e4))
    got = gpu_prefill(cfg, inp, params, states={k: v.clone() for k, v in st.items()},
                      states_in=True)
    ref = oracle_prefill(cfg, inp, params, states=st)
    compare_prefill(cfg, got, ref)


@pytest.mark.parametrize("bias", [3.0, 8.0])
def test_tc_large_dt(bias):
    # dt ~ softplus(N(0,1) + bias): per-token decays of e^-3 .. e^-130, so the decay
    # span of a 32-token block exceeds what the factorised decay covers and the
    # output kernel takes its direct-exponential branch on the diagonal blocks
    cfg, params, inp, st = _tc_case(23)
    params = dict(params, dt_bias=torch.full_like(params["dt_bias"], bias))
    got = gpu_prefill(cfg, inp, params, states={k: v.clone() for k, v in st.items()},
                      states_in=True)
    ref = oracle_prefill(cfg, inp, params, states=st)
    compare_prefill(cfg, got, ref)


@pytest.mark.parametrize("mag", [1e5, 3e7])
def test_tc_large_carried_state(mag):
    # a carried SSM state far beyond the fp16 range: the output kernel's operand
    # holds each (chunk, head) state divided by a power of two and multiplies
    # C H_c^T back by it, so y and the final state still match the oracle
    cfg, params, inp, st = _tc_case(24)
    st = dict(st, ssm_state=st["ssm_state"] * (mag / 0.1))
    got = gpu_prefill(cfg, inp, params, states={k: v.clone() for k, v in st.items()},
                      states_in=True)
    ref = oracle_prefill(cfg, inp, params, states=st)
    compare_prefill(cfg, got, ref)
    assert m2.device_errors() == 0


def test_without_state_buffers():
    cfg = case("zamba2_2p7b_prefill", batch=2, seqlen=300, nheads=4)
    params = W.make_params(cfg, 2)
    inp = W.make_prefill_inputs(cfg, 2)
    got = gpu_prefill(cfg, inp, params, want_states=False)
    ref = oracle_prefill(cfg, inp, params)
    check_bf16_out(got["y"], ref["y"], "y")


def test_run_twice_is_bitwise_identical():
    cfg = case("zamba2_2p7b_prefill", batch=2, seqlen=600, nheads=8)
    params = W.make_params(cfg, 4)
    inp = W.make_prefill_inputs(cfg, 4)
    a = gpu_prefill(cfg, inp, params)
    b = gpu_prefill(cfg, inp, params)
    for k in a:
        check_exact(a[k], b[k], k)


# ---------------------------------------------------------------- continuation

@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_prefill_splits_into_two_prefills_on_gpu(io):
    cfg = case("zamba2_2p7b_prefill", batch=2, seqlen=600, nheads=4, ngroups=2, io_dtype=io)
    params = W.make_params(cfg, 6)
    inp = W.make_prefill_inputs(cfg, 6)
    st = W.make_states(cfg, 6)
    ref = oracle_prefill(cfg, inp, params, states=st)
    for L1 in (1, 255, 256, 300):
        c1 = cfg.with_(seqlen=L1)
        c2 = cfg.with_(seqlen=cfg.seqlen - L1)
        i1 = {k: v[:, :L1] for k, v in inp.items()}
        i2 = {k: v[:, L1:] for k, v in inp.items()}
        a = gpu_prefill(c1, {**i1, "zxbcdt": inp["zxbcdt"][:, :L1].contiguous()}, params,
                        states={k: v.clone() for k, v in st.items()}, states_in=True)
        b = gpu_prefill(c2, {**i2, "zxbcdt": inp["zxbcdt"][:, L1:].contiguous()}, params,
                        states={"conv_state": a["conv_state"], "ssm_state": a["ssm_state"]},
                        states_in=True)
        got = {"y": torch.cat([a["y"], b["y"]], dim=1), "conv_state": b["conv_state"],
               "ssm_state": b["ssm_state"]}
        compare_prefill(cfg, got, ref)


def _gpu_steps(cfg, params, st, step_inputs):
    dims = m2.dims_from_config(cfg)
    pt, pp = dev_params(params)
    cs = st["conv_state"].cuda().contiguous()
    hs = st["ssm_state"].cuda().contiguous()
    ys = []
    for si in step_inputs:
        v = W.split_packed(cfg, si["zxbcdt"].cuda())
        ys.append(m2.step(dims, pp, v["xBC"], v["z"], v["dt_raw"], cs, hs).cpu())
    torch.cuda.synchronize()
    return ys, cs.cpu(), hs.cpu()


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_prefill_then_decode_steps_equals_prefill(io):
    cfg = case("zamba2_2p7b_prefill", batch=2, seqlen=300, nheads=4, io_dtype=io)
    params = W.make_params(cfg, 7)
    inp = W.make_prefill_inputs(cfg, 7)
    ref = oracle_prefill(cfg, inp, params)
    k = 5
    c1 = cfg.with_(seqlen=cfg.seqlen - k)
    a = gpu_prefill(c1, {"zxbcdt": inp["zxbcdt"][:, :-k].contiguous()}, params)
    steps = [{"zxbcdt": inp["zxbcdt"][:, t].contiguous()} for t in range(cfg.seqlen - k,
                                                                          cfg.seqlen)]
    ys, cs, hs = _gpu_steps(cfg, params, a, steps)
    got = {"y": torch.cat([a["y"], torch.stack(ys, dim=1)], dim=1), "conv_state": cs,
           "ssm_state": hs}
    compare_prefill(cfg, got, ref)


# ---------------------------------------------------------------- decode vs oracle

@pytest.mark.parametrize("cfg", [
    case("zamba2_2p7b_decode", batch=3, nheads=6, ngroups=2),
    case("zamba2_2p7b_decode", batch=2, nheads=4, headdim=16, dstate=128, io_dtype="f32"),
    case("zamba2_2p7b_decode", batch=2, nheads=4, norm_before_gate=True),
    # a prime batch: clusters with one and with two rows (the deferred row finish)
    case("zamba2_2p7b_decode", batch=37, nheads=8),
], ids=lambda c: c.name)
def test_decode_small(cfg):
    params = W.make_params(cfg, 8)
    st = W.make_states(cfg, 8)
    steps = [W.make_step_inputs(cfg, 8, s) for s in range(6)]
    ys, cs, hs = _gpu_steps(cfg, params, st, steps)
    ocs, ohs = st["conv_state"], st["ssm_state"]
    dims = dict(nheads=cfg.nheads, headdim=cfg.headdim, dstate=cfg.dstate, ngroups=cfg.ngroups,
                norm_before_gate=cfg.norm_before_gate)
    for s, si in enumerate(steps):
        o = oracle.mixer_step(si["xBC"], si["z"], si["dt_raw"], params, ocs, ohs, **dims)
        ocs, ohs = o["conv_state"], o["ssm_state"]
        if cfg.io_dtype == "f32":
            check_f32(ys[s], o["y"], f"y step {s}")
        else:
            check_bf16_out(ys[s], o["y"], f"y step {s}")
    check_exact(cs, ocs, "conv_state")
    (check_f32 if cfg.io_dtype == "f32" else check_rms)(hs, ohs, "ssm_state")
    assert m2.device_errors() == 0
