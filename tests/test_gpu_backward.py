"""GPU parity of the backward pass: every gradient (q, k, v, g, beta,
state_in) of L = <out, d_out> + <state_out, d_state_out> against autograd of
the fp64 definition (oracle/backward.py), at the forward's bar applied to
each gradient tensor: max |x - ref| / max |ref| <= 1e-4 with fp32 I/O (the
token-serial kernel) and <= 2e-2 with bf16 I/O (the chunked tensor-core
kernel)."""
import numpy as np
import pytest
import torch

import gated_deltanet_linear_chunked_b200 as gdn
import oracle
from gated_deltanet_linear_chunked_b200 import workloads as wl

from gdn_testlib import TOL, max_rel, to_np

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dstate_in")


def run_and_check(w, with_state=True, with_dS=True, seed=0, heads=None):
    x = wl.make_inputs(w)
    rng = np.random.default_rng(90000 + seed)
    d_out = rng.standard_normal(x["v"].shape).astype(np.float32)
    d_S = rng.standard_normal((w.B, w.H, w.Dk, w.Dv)).astype(np.float32) if with_dS else None
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    if w.dtype == "bf16":
        d_out = wl.round_bf16(d_out)
    s_in = x["state_in"] if with_state else None
    d = {n: torch.from_numpy(np.ascontiguousarray(x[n])).cuda() for n in ("q", "k", "v", "g", "beta")}
    for n in ("q", "k", "v"):
        d[n] = d[n].to(tdt)
    fn = gdn.chunk_bidir_backward if w.mode == "bidir" else gdn.chunk_fwd_backward
    res = fn(d["q"], d["k"], d["v"], d["g"], d["beta"],
             None if s_in is None else torch.from_numpy(s_in).cuda(),
             torch.from_numpy(d_out).cuda().to(tdt),
             None if d_S is None else torch.from_numpy(d_S).cuda())
    torch.cuda.synchronize()
    hs = list(range(w.H)) if heads is None else heads  # heads compared with the oracle
    s0 = np.zeros((w.B, w.H, w.Dk, w.Dv)) if s_in is None else s_in
    ref = oracle.backward.grads(x["q"][:, :, hs], x["k"][:, :, hs], x["v"][:, :, hs],
                                x["g"][:, :, hs], x["beta"][:, :, hs], s0[:, hs],
                                d_out[:, :, hs], None if d_S is None else d_S[:, hs],
                                bidir=w.mode == "bidir")
    tol = TOL[w.dtype]
    got = {n: to_np(res[n]) for n in NAMES}
    got = {n: (v[:, hs] if n == "dstate_in" else v[:, :, hs]) for n, v in got.items()}
    errs = {n: max_rel(got[n], ref[n]) for n in NAMES}
    bad = {n: e for n, e in errs.items() if not e <= tol}
    assert not bad, f"{w.name}: {errs}"
    return errs


@pytest.mark.parametrize("mode", ["fwd", "bidir"])
def test_tiny_fp32_backward(mode):
    import dataclasses
    run_and_check(dataclasses.replace(wl.tiny(), mode=mode))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["fwd", "bidir"])
@pytest.mark.parametrize("D", [16, 64, 128])
@pytest.mark.parametrize("T", [1, 17, 65, 130])
def test_backward_sweep(T, D, mode, dtype):
    """Ragged lengths around the 64-token checkpoints and the 16-token groups,
    every head-dim class, carried state and a final-state gradient."""
    w = wl.Workload(f"bwd_T{T}_D{D}", 2, T, 2, D, D, dtype, 64, mode, ("uniform", -0.5, 0.0),
                    ("sigmoid",), ("normal", 0.3), 91000 + 7 * T + D)
    run_and_check(w, seed=T + D)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("Dk,Dv", [(32, 96), (128, 16), (48, 64)])
def test_backward_rectangular(Dk, Dv, dtype):
    w = wl.Workload("bwd_rect", 1, 100, 2, Dk, Dv, dtype, 64, "bidir", ("uniform", -0.5, 0.0),
                    ("sigmoid",), ("normal", 0.3), 92000 + Dk + Dv)
    run_and_check(w)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_zero_state_no_final_gradient(dtype):
    w = wl.Workload("bwd_zero", 1, 90, 3, 64, 64, dtype, 64, "fwd", ("neg_softplus",),
                    ("sigmoid",), ("zero",), 93000)
    run_and_check(w, with_state=False, with_dS=False)


@pytest.mark.parametrize("mode", ["fwd", "bidir"])
def test_backward_unnormalised_rows_bf16(mode):
    """q, k rows not unit-norm (N(0,1) rows with rows at 1e-3 and 1e3, rows
    under the 1e-12 clamp, an all-zero q row and k row): the chunked bf16
    backward's normalisation and the reduction's Jacobian."""
    w = wl.Workload("bwd_mixed", 1, 200, 2, 64, 64, "bf16", 64, mode, ("uniform", -0.5, 0.0),
                    ("sigmoid",), ("normal", 0.3), 94000, qk=("mixed",))
    run_and_check(w, seed=5)


def test_backward_empty_sequence():
    """T = 0: state_out = state_in, so d_state_in = d_state_out."""
    q = torch.empty(1, 0, 2, 16, device="cuda")
    g = torch.empty(1, 0, 2, device="cuda")
    s = torch.randn(1, 2, 16, 16, device="cuda")
    dS = torch.randn(1, 2, 16, 16, device="cuda")
    res = gdn.chunk_fwd_backward(q, q, q, g, g, s, q, dS)
    torch.cuda.synchronize()
    assert torch.equal(res["dstate_in"], dS)


@pytest.mark.parametrize("mode", ["fwd", "bidir"])
def test_backward_stream_chunk_full_size(mode):
    """The 2640-token x 20-head x d112 streaming chunk, bf16 I/O; heads 0
    and 19 compared with the oracle (heads are independent)."""
    run_and_check(wl.stream_chunk(mode), seed=1, heads=[0, 19])


@pytest.mark.parametrize("Dk,Dv", [(48, 80), (96, 32)])
def test_backward_many_chunks_rectangular(Dk, Dv):
    """Enough chunk tiles (2 x 24 chunks x 6 heads x 2 directions = 576) that
    each CTA of the persistent gradient pass walks several and prefetches the
    next; Dk or Dv below 64 gives the dX tiles buffers of their own.  Heads
    0 and 5 of both batch rows compared with the oracle."""
    w = wl.Workload(f"bwd_many_{Dk}_{Dv}", 2, 1500, 6, Dk, Dv, "bf16", 64, "bidir", ("uniform", -0.5, 0.0),
                    ("sigmoid",), ("normal", 0.3), 93000 + Dk + Dv)
    run_and_check(w, seed=4, heads=[0, 5])
