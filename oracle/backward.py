"""fp64 gradients of the Mamba-2 mixer core prefill -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of bench.py
may import this module; the product library never imports it and it imports
nothing from the product library.

The forward is written again here with plain PyTorch CPU float64 ops, token
by token, from the same definitions the C oracle follows (it shares no code
with ``mamba2_oracle.c``), and ``torch.autograd`` differentiates it:

* conv1d + SiLU over the x|B|C channels with the carried conv state as left
  context -- "Zamba2 hybrid architecture in Transformers" (qwbw.cn), section
  三 step 2, bias per section 五;
* dt = softplus(dt_raw + dt_bias) and h_t = exp(dt_t A) h_{t-1} + dt_t x_t B_t^T,
  y_t = C_t h_t + D x_t -- the Mamba-2 layer named on the state-spaces/mamba
  repository page (opendeer.net), "About the project";
* the gated group RMSNorm (either order) -- qwbw.cn section 三 step 4 and
  section 五 (eps).

Training through the mixer is what the qwbw.cn page's gradient-checkpointing
support (section 三) implies; the loss whose gradients are taken is
sum(y * dy) (+ sum(h_L * dh_L) when a gradient of the final state is given),
so the gradients are the vector-Jacobian products a framework's backward pass
would request.

Pins (tests/test_oracle_backward_pins.py): the forward equals the C oracle's,
and torch.autograd.gradcheck (central finite differences) accepts it.
"""
from __future__ import annotations

import numpy as np
import torch


def _t(a):
    """float64 CPU tensor (a copy), or None."""
    if a is None:
        return None
    if isinstance(a, torch.Tensor):
        return a.detach().to("cpu", torch.float64).clone()
    return torch.tensor(np.asarray(a, dtype=np.float64))


def _silu(s):
    return s / (1.0 + torch.exp(-s))


def _softplus(s):
    return torch.clamp(s, min=0.0) + torch.log1p(torch.exp(-torch.abs(s)))


def mixer_prefill_torch(xBC, z, dt_raw, conv_w, conv_b, dt_bias, A, D, norm_w, conv_state,
                        ssm_state, *, nheads, headdim, dstate, ngroups, eps=1e-5,
                        norm_before_gate=False):
    """The prefill of a batch as float64 torch ops.  xBC [b, L, conv_dim]; z [b, L, H*P];
    dt_raw [b, L, H]; conv_w [conv_dim, K]; conv_state [b, conv_dim, K] (oldest input
    first) or None; ssm_state [b, H, P, N] or None.  Returns (y [b, L, H*P], h_L)."""
    b, L, conv_dim = xBC.shape
    H, P, N, G = nheads, headdim, dstate, ngroups
    K = conv_w.shape[1]
    d_inner = H * P
    # the conv's left context: the state's newest K - 1 inputs, or zeros
    if conv_state is not None:
        left = conv_state[:, :, 1:].transpose(1, 2)
    else:
        left = torch.zeros(b, K - 1, conv_dim, dtype=xBC.dtype)
    xin = torch.cat([left, xBC], dim=1)  # [b, K - 1 + L, conv_dim]
    pre = conv_b.expand(b, L, conv_dim)
    for k in range(K):  # tap k multiplies the input K - 1 - k tokens back
        pre = pre + conv_w[:, k] * xin[:, k:k + L, :]
    u = _silu(pre)
    x = u[..., :d_inner].reshape(b, L, H, P)
    hpg = H // G
    Bh = u[..., d_inner:d_inner + G * N].reshape(b, L, G, N).repeat_interleave(hpg, dim=2)
    Ch = u[..., d_inner + G * N:].reshape(b, L, G, N).repeat_interleave(hpg, dim=2)
    dt = _softplus(dt_raw + dt_bias)  # [b, L, H]
    h = ssm_state if ssm_state is not None else torch.zeros(b, H, P, N, dtype=xBC.dtype)
    ys = []
    for t in range(L):
        a = torch.exp(dt[:, t] * A)  # [b, H]
        h = (a[:, :, None, None] * h
             + (dt[:, t, :, None] * x[:, t])[:, :, :, None] * Bh[:, t, :, None, :])
        ys.append((h * Ch[:, t, :, None, :]).sum(-1) + D[None, :, None] * x[:, t])
    ypre = torch.stack(ys, 1).reshape(b, L, d_inner) if L > 0 else torch.zeros(b, 0, d_inner,
                                                                              dtype=xBC.dtype)
    gs = d_inner // G
    v = ypre if norm_before_gate else ypre * _silu(z)
    v = v.reshape(b, L, G, gs)
    inv = 1.0 / torch.sqrt((v * v).mean(-1) + eps)
    out = (v * inv[..., None]).reshape(b, L, d_inner) * norm_w
    if norm_before_gate:
        out = out * _silu(z)
    return out, h


_NAMES = ("xBC", "z", "dt_raw", "conv_w", "conv_b", "dt_bias", "A", "D", "norm_w",
          "conv_state", "ssm_state")


def mixer_prefill_grads(xBC, z, dt_raw, params, dy, *, nheads, headdim, dstate, ngroups,
                        conv_state=None, ssm_state=None, d_ssm_state=None, eps=1e-5,
                        norm_before_gate=False):
    """Gradients of sum(y * dy) (+ sum(h_L * d_ssm_state)) with respect to every input.

    Returns a dict of float64 numpy arrays keyed like the inputs (conv_state and
    ssm_state only when given), plus "y" and "ssm_state_out" of the forward."""
    vals = {"xBC": _t(xBC), "z": _t(z), "dt_raw": _t(dt_raw),
            **{k: _t(params[k]) for k in ("conv_w", "conv_b", "dt_bias", "A", "D", "norm_w")},
            "conv_state": _t(conv_state), "ssm_state": _t(ssm_state)}
    leaves = {k: v.requires_grad_(True) for k, v in vals.items() if v is not None}
    y, hL = mixer_prefill_torch(*[vals[k] for k in _NAMES], nheads=nheads, headdim=headdim,
                                dstate=dstate, ngroups=ngroups, eps=eps,
                                norm_before_gate=norm_before_gate)
    loss = (y * _t(dy)).sum()
    if d_ssm_state is not None:
        loss = loss + (hL * _t(d_ssm_state)).sum()
    grads = torch.autograd.grad(loss, list(leaves.values()), allow_unused=True)
    out = {}
    for (k, v), g in zip(leaves.items(), grads):
        out[k] = (torch.zeros_like(v) if g is None else g).detach().numpy()
    out["y"] = y.detach().numpy()
    out["ssm_state_out"] = hL.detach().numpy()
    return out
