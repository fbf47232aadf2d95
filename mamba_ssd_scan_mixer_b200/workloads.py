"""Synthetic, seeded workloads shaped like the Zamba2 Mamba-2 mixers.

This module only draws random numbers with fixed distributions; it holds none
of the mixer's arithmetic and imports neither the CUDA library nor the oracle,
so both sides can be fed the same values from it.

Shapes follow the Zamba2 family (1.2B / 2.7B / 7B) on the "Zamba2 hybrid
architecture in Transformers" page (qwbw.cn), section 五: d_state 64, d_conv 4,
chunk 256, mamba heads of headdim 64.  Distributions:

* x, z, B, C (the pre-conv xBC and the gate) ~ N(0, 1); dt_raw ~ N(0, 1)
* dt_bias = softplus^{-1}(u), u log-uniform on [time_step_min, time_step_max]
  = [1e-3, 1e-1] (section 五's dt initialisation range)
* A_h = -exp(U[0, ln 16]), D ~ N(0, 1)
* conv weight and bias ~ U(-0.5, 0.5); norm weight = 1 + 0.1 N(0, 1)
* decode: SSM state ~ N(0, 0.1^2) fp32, conv state ~ N(0, 1) in the I/O dtype

Everything is drawn in fp32 on the CPU from torch generators seeded by
(seed, stream) and rounded to the I/O dtype (round to nearest even).  The xBC,
z and dt_raw inputs are views into one packed buffer laid out like the
in_proj output, [z | xBC | dt], so the row strides of the library's
entry points are exercised.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class MixerConfig:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    d_conv: int = 4
    chunk_size: int = 256
    io_dtype: str = "bf16"  # "f32" or "bf16"
    norm_eps: float = 1e-5
    norm_before_gate: bool = False
    decode_steps: int = 0   # > 0: a decode workload of that many single-token steps
    states_in: bool = False  # prefill starts from carried (random) states

    @property
    def d_inner(self) -> int:
        return self.nheads * self.headdim

    @property
    def conv_dim(self) -> int:
        return self.d_inner + 2 * self.ngroups * self.dstate

    @property
    def d_in_proj(self) -> int:
        return self.d_inner + self.conv_dim + self.nheads

    @property
    def packed_width(self) -> int:
        """Row width of the packed [z | xBC | dt] buffer, padded to a multiple of 8
        elements (16 bytes in bf16) as the library's row strides require."""
        return -(-self.d_in_proj // 8) * 8

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.io_dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "MixerConfig":
        return replace(self, **kw)


CONFIGS = {
    "tiny_f32": MixerConfig("tiny_f32", batch=1, seqlen=256, nheads=4, headdim=16, dstate=16,
                            ngroups=1, chunk_size=64, io_dtype="f32"),
    "zamba2_2p7b_prefill": MixerConfig("zamba2_2p7b_prefill", batch=1, seqlen=4096, nheads=80,
                                       headdim=64, dstate=64, ngroups=1),
    "zamba2_1p2b_prefill": MixerConfig("zamba2_1p2b_prefill", batch=8, seqlen=2048, nheads=64,
                                       headdim=64, dstate=64, ngroups=1),
    "zamba2_7b_long_prefill": MixerConfig("zamba2_7b_long_prefill", batch=1, seqlen=32768,
                                          nheads=112, headdim=64, dstate=64, ngroups=2),
    "zamba2_2p7b_decode": MixerConfig("zamba2_2p7b_decode", batch=256, seqlen=1, nheads=80,
                                      headdim=64, dstate=64, ngroups=1, decode_steps=1024),
}

# Streams of the per-seed generator (keeps draws independent of one another).
_S_PARAMS, _S_INPUTS, _S_STATES, _S_STEP0 = 1, 2, 3, 1000


def generator(seed: int, stream: int) -> torch.Generator:
    return torch.Generator(device="cpu").manual_seed((seed * 1_000_003 + stream) % (2**63))


def make_params(cfg: MixerConfig, seed: int = 0) -> dict:
    """fp32 parameters: conv_w [conv_dim, K], conv_b [conv_dim], dt_bias, A, D [H],
    norm_w [d_inner]."""
    g = generator(seed, _S_PARAMS)
    H = cfg.nheads
    conv_w = torch.rand(cfg.conv_dim, cfg.d_conv, generator=g) - 0.5
    conv_b = torch.rand(cfg.conv_dim, generator=g) - 0.5
    lo, hi = math.log(1e-3), math.log(1e-1)
    u = torch.exp(lo + (hi - lo) * torch.rand(H, generator=g, dtype=torch.float64))
    dt_bias = (u + torch.log(-torch.expm1(-u))).float()  # inverse softplus of the init dt
    A = -torch.exp(math.log(16.0) * torch.rand(H, generator=g, dtype=torch.float64)).float()
    D = torch.randn(H, generator=g)
    norm_w = 1.0 + 0.1 * torch.randn(cfg.d_inner, generator=g)
    return {"conv_w": conv_w.contiguous(), "conv_b": conv_b, "dt_bias": dt_bias, "A": A, "D": D,
            "norm_w": norm_w}


def split_packed(cfg: MixerConfig, packed: torch.Tensor) -> dict:
    """Views z, xBC, dt_raw of a packed [..., packed_width] buffer (pad columns unused)."""
    di, cd, H = cfg.d_inner, cfg.conv_dim, cfg.nheads
    return {"zxbcdt": packed, "z": packed[..., :di], "xBC": packed[..., di:di + cd],
            "dt_raw": packed[..., di + cd:di + cd + H]}


def make_prefill_inputs(cfg: MixerConfig, seed: int = 0) -> dict:
    """Packed [b, L, d_in_proj] buffer in the I/O dtype and its views z, xBC, dt_raw.
    All entries ~ N(0, 1) (x, B, C, z and dt_raw alike)."""
    g = generator(seed, _S_INPUTS)
    packed = torch.randn(cfg.batch, cfg.seqlen, cfg.packed_width, generator=g)
    return split_packed(cfg, packed.to(cfg.torch_dtype))


def make_states(cfg: MixerConfig, seed: int = 0) -> dict:
    """Carried states: conv [b, conv_dim, K] ~ N(0, 1) in the I/O dtype, SSM
    [b, H, P, N] ~ N(0, 0.1^2) fp32."""
    g = generator(seed, _S_STATES)
    conv = torch.randn(cfg.batch, cfg.conv_dim, cfg.d_conv, generator=g).to(cfg.torch_dtype)
    ssm = 0.1 * torch.randn(cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate, generator=g)
    return {"conv_state": conv, "ssm_state": ssm}


def zero_states(cfg: MixerConfig) -> dict:
    return {"conv_state": torch.zeros(cfg.batch, cfg.conv_dim, cfg.d_conv, dtype=cfg.torch_dtype),
            "ssm_state": torch.zeros(cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate)}


def make_step_inputs(cfg: MixerConfig, seed: int, step: int) -> dict:
    """Inputs of decode step `step`: packed [b, d_in_proj] and its views."""
    g = generator(seed, _S_STEP0 + step)
    packed = torch.randn(cfg.batch, cfg.packed_width, generator=g)
    return split_packed(cfg, packed.to(cfg.torch_dtype))
