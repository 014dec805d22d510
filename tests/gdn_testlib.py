"""Shared helpers for the GPU parity tests: device inputs from the seeded
workloads, the oracle on all or on sampled heads, and the error metric.

Metric: for each output tensor, max_i |x_i - ref_i| / max_i |ref_i| (the
"max relative error" of the parity bar), computed in fp64.  Thresholds:
1e-4 for fp32 I/O, 2e-2 for bf16 I/O with fp32 accumulation.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from gated_deltanet_linear_chunked_b200 import workloads as wl

TOL = {"f32": 1e-4, "bf16": 2e-2}


def max_rel(x, ref) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    den = np.max(np.abs(ref)) if ref.size else 0.0
    if den == 0.0:
        return float(np.max(np.abs(x))) if x.size else 0.0
    return float(np.max(np.abs(x - ref)) / den)


def max_rel_per_head(x, ref, head_axes) -> float:
    """The largest per-head max relative error: the metric taken separately
    over each (b, h) slice, so a wrong head of small magnitude cannot hide
    under another head's maximum.  `head_axes` are the (b, h) axes of the
    tensor: (0, 2) for outputs [B,T,H,D], (0, 1) for states [B,H,Dk,Dv]."""
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    ab, ah = head_axes
    worst = 0.0
    for b in range(x.shape[ab]):
        for h in range(x.shape[ah]):
            idx = [slice(None)] * x.ndim
            idx[ab], idx[ah] = b, h
            worst = max(worst, max_rel(x[tuple(idx)], ref[tuple(idx)]))
    return worst


def max_rel_rows(x, ref, rows) -> float:
    """Largest error over the given token rows of an output [B,T,H,D],
    relative to each (b, h, row)'s own largest reference value: rows whose
    reference is tiny or huge are measured on their own scale."""
    x = np.asarray(x, np.float64)[:, rows]
    ref = np.asarray(ref, np.float64)[:, rows]
    den = np.max(np.abs(ref), axis=-1)
    num = np.max(np.abs(x - ref), axis=-1)
    ok = den > 0
    worst = float(np.max(num[ok] / den[ok])) if ok.any() else 0.0
    if (~ok).any():
        worst = max(worst, float(np.max(num[~ok])))
    return worst


def torch_dtype(w: wl.Workload):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def device_inputs(w: wl.Workload, device="cuda"):
    """All inputs on the device, filled head by head (host peak = one head)."""
    dt = torch_dtype(w)
    q = torch.empty((w.B, w.T, w.H, w.Dk), dtype=dt, device=device)
    k = torch.empty_like(q)
    v = torch.empty((w.B, w.T, w.H, w.Dv), dtype=dt, device=device)
    g = torch.empty((w.B, w.T, w.H), dtype=torch.float32, device=device)
    beta = torch.empty_like(g)
    for b, h, d in wl.iter_heads(w):
        q[b, :, h] = torch.from_numpy(d["q"]).to(device=device, dtype=dt)
        k[b, :, h] = torch.from_numpy(d["k"]).to(device=device, dtype=dt)
        v[b, :, h] = torch.from_numpy(d["v"]).to(device=device, dtype=dt)
        g[b, :, h] = torch.from_numpy(d["g"]).to(device)
        beta[b, :, h] = torch.from_numpy(d["beta"]).to(device)
    s = wl.make_state(w)
    state_in = None if s is None else torch.from_numpy(s).to(device)
    return {"q": q, "k": k, "v": v, "g": g, "beta": beta, "state_in": state_in}


def host_inputs(w: wl.Workload):
    return wl.make_inputs(w)


def oracle_run(w: wl.Workload, x: dict, bidir: bool | None = None):
    """Oracle over every head of host inputs `x` (numpy)."""
    if bidir is None:
        bidir = w.mode == "bidir"
    fn = oracle.oracle_bidir if bidir else oracle.oracle_fwd
    return fn(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"])


def oracle_head(w: wl.Workload, b: int, h: int, state_in_head=None, bidir=None):
    """Oracle for one (b, h) head regenerated from the workload's seed."""
    if bidir is None:
        bidir = w.mode == "bidir"
    d = wl.make_head(w, b, h)
    shp = lambda a: a.reshape(1, w.T, 1, -1)  # noqa: E731
    fn = oracle.oracle_bidir if bidir else oracle.oracle_fwd
    return fn(shp(d["q"]), shp(d["k"]), shp(d["v"]), d["g"].reshape(1, w.T, 1),
              d["beta"].reshape(1, w.T, 1), state_in_head)


def to_np(t):
    return t.detach().float().cpu().numpy()
