"""GPU parity at the full benchmark sizes, through the same C-ABI calls and launch
configuration the benchmark times.

Prefill workloads are compared element by element over every output (the
oracle finishes them in seconds to a minute on the host cores).  The decode
workload (batch 256, 1024 steps) is compared on the rows the oracle can follow
one by one: batch rows {0, 1, 127, 255} for all 1024 steps, and every row for
the first 8 steps; y on every checked step, the states after step 8 and after
step 1024.
"""
import time

import numpy as np
import pytest
import torch

import mamba_ssd_scan_mixer_b200 as m2
import oracle
from mamba_ssd_scan_mixer_b200 import workloads as W

from harness import (check_bf16_out, check_exact, check_rms, compare_prefill, dev_params,
                     gpu_prefill, oracle_prefill)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["zamba2_2p7b_prefill", "zamba2_1p2b_prefill",
                                  "zamba2_7b_long_prefill"])
def test_full_size_prefill(name):
    cfg = W.CONFIGS[name]
    params = W.make_params(cfg, 0)
    inp = W.make_prefill_inputs(cfg, 0)
    got = gpu_prefill(cfg, inp, params)
    t = time.time()
    ref = oracle_prefill(cfg, inp, params)
    rep = compare_prefill(cfg, got, ref)
    print(name, rep, f"oracle {time.time() - t:.1f}s")


@pytest.mark.parametrize("L1", [2048, 1000])
def test_full_size_chunked_prefill_continuation(L1):
    # the 2.7B workload split into two prefills (the second continuing from the
    # first's conv and SSM states) equals the whole prefill (the cache test of
    # chunked prefill); compared with the oracle's whole-sequence result
    cfg = W.CONFIGS["zamba2_2p7b_prefill"]
    params = W.make_params(cfg, 1)
    inp = W.make_prefill_inputs(cfg, 1)
    st = W.make_states(cfg, 1)
    ref = oracle_prefill(cfg, inp, params, states=st)
    a = gpu_prefill(cfg.with_(seqlen=L1), {"zxbcdt": inp["zxbcdt"][:, :L1].contiguous()},
                    params, states={k: v.clone() for k, v in st.items()}, states_in=True)
    b = gpu_prefill(cfg.with_(seqlen=cfg.seqlen - L1),
                    {"zxbcdt": inp["zxbcdt"][:, L1:].contiguous()}, params,
                    states={"conv_state": a["conv_state"], "ssm_state": a["ssm_state"]},
                    states_in=True)
    got = {"y": torch.cat([a["y"], b["y"]], dim=1), "conv_state": b["conv_state"],
           "ssm_state": b["ssm_state"]}
    print(L1, compare_prefill(cfg, got, ref))
    assert m2.device_errors() == 0


def test_full_size_prefill_then_decode_steps():
    # prefill of the first 4096 - 8 tokens, then 8 single-token decode steps, equals
    # the whole prefill (the cached-decode test)
    cfg = W.CONFIGS["zamba2_2p7b_prefill"]
    k = 8
    params = W.make_params(cfg, 2)
    inp = W.make_prefill_inputs(cfg, 2)
    ref = oracle_prefill(cfg, inp, params)
    a = gpu_prefill(cfg.with_(seqlen=cfg.seqlen - k),
                    {"zxbcdt": inp["zxbcdt"][:, :-k].contiguous()}, params)
    dims = m2.dims_from_config(cfg)
    pt, pp = dev_params(params)
    cs = a["conv_state"].cuda().contiguous()
    hs = a["ssm_state"].cuda().contiguous()
    ys = []
    for t in range(cfg.seqlen - k, cfg.seqlen):
        v = W.split_packed(cfg, inp["zxbcdt"][:, t].contiguous().cuda())
        ys.append(m2.step(dims, pp, v["xBC"], v["z"], v["dt_raw"], cs, hs).cpu())
    torch.cuda.synchronize()
    got = {"y": torch.cat([a["y"], torch.stack(ys, dim=1)], dim=1), "conv_state": cs.cpu(),
           "ssm_state": hs.cpu()}
    print(compare_prefill(cfg, got, ref))
    assert m2.device_errors() == 0


def test_full_size_decode_1024_steps():
    cfg = W.CONFIGS["zamba2_2p7b_decode"]
    seed = 0
    params = W.make_params(cfg, seed)
    st = W.make_states(cfg, seed)
    dims = m2.dims_from_config(cfg)
    pt, pp = dev_params(params)
    cs = st["conv_state"].cuda().contiguous()
    hs = st["ssm_state"].cuda().contiguous()
    y = torch.empty(cfg.batch, cfg.d_inner, dtype=cfg.torch_dtype, device="cuda")
    rows = [0, 1, 127, 255]
    odims = dict(nheads=cfg.nheads, headdim=cfg.headdim, dstate=cfg.dstate,
                 ngroups=cfg.ngroups)
    o_cs, o_hs = st["conv_state"], st["ssm_state"]            # all rows, first 8 steps
    s_cs, s_hs = st["conv_state"][rows], st["ssm_state"][rows]  # checked rows, all steps
    worst = 0.0
    for s in range(cfg.decode_steps):
        si = W.make_step_inputs(cfg, seed, s)
        v = W.split_packed(cfg, si["zxbcdt"].cuda(non_blocking=True))
        m2.mamba2_ssd_step(dims, pp, v["xBC"], v["z"], v["dt_raw"], y, cs, hs)
        yg = y.cpu()
        if s < 8:
            o = oracle.mixer_step(si["xBC"], si["z"], si["dt_raw"], params, o_cs, o_hs, **odims)
            o_cs, o_hs = o["conv_state"], o["ssm_state"]
            worst = max(worst, check_bf16_out(yg, o["y"], f"y step {s} (all rows)")[0])
            if s == 7:
                check_exact(cs.cpu(), o_cs, "conv_state after 8 steps")
                check_rms(hs.cpu(), o_hs, "ssm_state after 8 steps")
        o = oracle.mixer_step(si["xBC"][rows], si["z"][rows], si["dt_raw"][rows], params, s_cs,
                              s_hs, **odims)
        s_cs, s_hs = o["conv_state"], o["ssm_state"]
        worst = max(worst, check_bf16_out(yg[rows], o["y"], f"y step {s} rows {rows}")[0])
    check_exact(cs.cpu()[rows], s_cs, "conv_state after 1024 steps")
    e = check_rms(hs.cpu()[rows], s_hs, "ssm_state after 1024 steps")
    print("decode worst y error beyond bf16 rounding", worst, "state", e)
    assert m2.device_errors() == 0
