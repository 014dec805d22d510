"""fp64 reference gradients of the GDN scan.  TEST INFRASTRUCTURE ONLY.

The backward pass of the scan (the pages' bidirectional short training runs
the bidirectional GDN with gradients: "SANA-Streaming：基于混合扩散Transformer
的实时流式视频编辑系统", 方法步骤详情, second step) is the derivative of the
forward definition, so the reference is that definition written in plain
PyTorch CPU ops in float64 -- the same token recurrence as ``gdn_oracle.c``,
vectorised over (batch, head) only -- differentiated by autograd:

    q^ = q / sqrt(max(|q|^2, 1e-12)),  k^ likewise,  a_t = exp(g_t)
    S_t = a_t (I - beta_t k^_t k^_t^T) S_{t-1} + beta_t k^_t v_t^T,  o_t = S_t^T q^_t

Bidirectional mode adds the same recurrence over the time-reversed chunk from
a zero state; the state returned is the forward scan's.

``scan`` returns (out, state_out); ``grads`` returns the gradients of
<out, d_out> + <state_out, d_state_out> with respect to q, k, v, g, beta and
state_in.  ``tests/test_oracle_pins.py`` pins them to central finite
differences of the recurrence, to the pure-decay closed form, to the
single-token adjoint derived by hand and to linearity, and checks the forward
against the C oracle.
"""
from __future__ import annotations

import numpy as np
import torch


def _normalise(x):
    ss = (x * x).sum(-1, keepdim=True)
    return x / torch.sqrt(torch.clamp(ss, min=1e-12))


def _one_direction(q, k, v, g, beta, S, reverse):
    """q, k [B,T,H,Dk], v [B,T,H,Dv], g, beta [B,T,H], S [B,H,Dk,Dv];
    returns (out [B,T,H,Dv], final S)."""
    T = q.shape[1]
    qn, kn = _normalise(q), _normalise(k)
    outs = [None] * T
    order = range(T - 1, -1, -1) if reverse else range(T)
    for t in order:
        kt, qt, vt = kn[:, t], qn[:, t], v[:, t]                  # [B,H,D]
        a = torch.exp(g[:, t])[..., None, None]                   # [B,H,1,1]
        b = beta[:, t][..., None, None]
        x = torch.einsum("bhi,bhij->bhj", kt, S)                  # k^T S
        S = a * (S - b * kt[..., :, None] * x[..., None, :]) + b * kt[..., :, None] * vt[..., None, :]
        outs[t] = torch.einsum("bhi,bhij->bhj", qt, S)
    return torch.stack(outs, dim=1), S


def scan(q, k, v, g, beta, state_in=None, bidir=False):
    """The forward definition on float64 torch tensors."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    S0 = torch.zeros((B, H, Dk, Dv), dtype=torch.float64) if state_in is None else state_in
    out, S = _one_direction(q, k, v, g, beta, S0, reverse=False)
    if bidir:
        out_r, _ = _one_direction(q, k, v, g, beta, torch.zeros_like(S0), reverse=True)
        out = out + out_r
    return out, S


def grads(q, k, v, g, beta, state_in, d_out, d_state_out=None, bidir=False):
    """Reference gradients (numpy in, numpy float64 out): a dict with dq, dk,
    dv, dg, dbeta and dstate_in (None when state_in is None)."""
    t = lambda x: torch.tensor(np.asarray(x, np.float64), dtype=torch.float64,  # noqa: E731
                               requires_grad=True)
    ins = {"q": t(q), "k": t(k), "v": t(v), "g": t(g), "beta": t(beta)}
    if state_in is not None:
        ins["state_in"] = t(state_in)
    out, S = scan(ins["q"], ins["k"], ins["v"], ins["g"], ins["beta"], ins.get("state_in"), bidir)
    loss = (out * torch.tensor(np.asarray(d_out, np.float64))).sum()
    if d_state_out is not None:
        loss = loss + (S * torch.tensor(np.asarray(d_state_out, np.float64))).sum()
    names = list(ins)
    gs = torch.autograd.grad(loss, [ins[n] for n in names], allow_unused=True)
    res = {"d" + ("state_in" if n == "state_in" else n): (np.zeros(ins[n].shape) if gr is None else gr.numpy())
           for n, gr in zip(names, gs)}
    res.setdefault("dstate_in", None)
    return res


def forward_np(q, k, v, g, beta, state_in=None, bidir=False):
    """The forward of this transcription, numpy in and out (for cross-checks)."""
    t = lambda x: None if x is None else torch.tensor(np.asarray(x, np.float64))  # noqa: E731
    with torch.no_grad():
        out, S = scan(t(q), t(k), t(v), t(g), t(beta), t(state_in), bidir)
    return out.numpy(), S.numpy()
