"""GPU parity of the fused GDN prologue: the gates formed inside the kernels
from the gate layer's logits, g = -softplus(x) and beta = sigmoid(y), against
the oracle's gate-logit mode (which evaluates both maps in fp64).

Same bar as the other parity tests: max relative error per tensor (and per
head at full size) <= 2e-2 with bf16 I/O, <= 1e-4 with fp32 I/O.
"""
import dataclasses

import numpy as np
import pytest
import torch

import gated_deltanet_linear_chunked_b200 as gdn
import oracle
from gated_deltanet_linear_chunked_b200 import workloads as wl

from gdn_testlib import TOL, max_rel, max_rel_per_head, to_np

pytestmark = pytest.mark.gpu


def to_dev(x, dtype):
    d = {}
    for n in ("q", "k", "v", "g_logit", "beta_logit"):
        d[n] = torch.from_numpy(np.ascontiguousarray(x[n])).cuda().to(dtype)
    d["state_in"] = None if x["state_in"] is None else torch.from_numpy(x["state_in"]).cuda()
    return d


def run_and_check(w, x=None, per_head=False):
    if x is None:
        x = wl.make_inputs(w)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    d = to_dev(x, tdt)
    fn = gdn.chunk_bidir_logits if w.mode == "bidir" else gdn.chunk_fwd_logits
    out, S = fn(d["q"], d["k"], d["v"], d["g_logit"], d["beta_logit"], d["state_in"], chunk=w.chunk)
    torch.cuda.synchronize()
    ofn = oracle.oracle_bidir_logits if w.mode == "bidir" else oracle.oracle_fwd_logits
    ro, rs = ofn(x["q"], x["k"], x["v"], x["g_logit"], x["beta_logit"], x["state_in"])
    o, s = to_np(out), to_np(S)
    tol = TOL[w.dtype]
    eo, es = max_rel(o, ro), max_rel(s, rs)
    assert eo <= tol and es <= tol, f"{w.name}: out {eo:.3e} state {es:.3e}"
    if per_head:
        assert max_rel_per_head(o, ro, (0, 2)) <= tol and max_rel_per_head(s, rs, (0, 1)) <= tol
    assert np.isfinite(o).all() and np.isfinite(s).all()
    return x, out, S


@pytest.mark.parametrize("mode", ["fwd", "bidir"])
def test_tiny_fp32_from_logits(mode):
    """The tiny fp32 scan (B1 H2 d16 T64) with its gates given as the logits
    they are stated as (g = -softplus(N(0,1)), beta = sigmoid(N(0,1)))."""
    w = dataclasses.replace(wl.tiny(), gate=("logit_normal",), beta=("logit_normal",), mode=mode)
    run_and_check(w)


@pytest.mark.parametrize("mode", ["fwd", "bidir"])
def test_stream_chunk_from_logits(mode):
    """The full 2640-token x 20-head x d112 streaming chunk, bf16, carried
    state, gates from bf16 logits: every head against the oracle."""
    run_and_check(wl.stream_chunk_logits(mode), per_head=True)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["fwd", "bidir"])
@pytest.mark.parametrize("D", [16, 64, 112, 128])
@pytest.mark.parametrize("T", [1, 17, 65, 200])
def test_logit_sweep(T, D, mode, dtype):
    w = wl.Workload(f"lsweep_T{T}_D{D}", 2, T, 3, D, D, dtype, 64, mode, ("logit_normal",),
                    ("logit_normal",), ("normal", 0.02), 72000 + 7 * T + D)
    run_and_check(w, per_head=True)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_extreme_logits(dtype):
    """Saturated logits: x = +-30 (g = -30, i.e. full decay, or g ~ -1e-13),
    y = +-30 (beta ~ 1 or ~ 1e-13), mixed along the sequence; nothing
    overflows and the result matches the oracle."""
    w = wl.Workload("lextreme", 1, 150, 2, 64, 64, dtype, 64, "fwd", ("logit_normal",),
                    ("logit_normal",), ("normal", 0.02), 4343)
    x = wl.make_inputs(w)
    rng = np.random.default_rng(9)
    x["g_logit"] = (30.0 * rng.choice([-1.0, 1.0], size=x["g_logit"].shape)).astype(np.float32)
    x["beta_logit"] = (30.0 * rng.choice([-1.0, 1.0], size=x["beta_logit"].shape)).astype(np.float32)
    run_and_check(w, x)


def test_fused_gates_equal_the_plain_entry_point():
    """The fused prologue computes the same scan as the plain entry point fed
    with the gates the oracle forms from the same logits (fp32): the two
    device results agree within the bf16 tolerance."""
    w = wl.stream_chunk_logits("fwd")
    x, out, S = run_and_check(w)
    g, b = oracle.gates_from_logits(x["g_logit"], x["beta_logit"])
    d = to_dev(x, torch.bfloat16)
    gt = torch.from_numpy(g.astype(np.float32)).cuda()
    bt = torch.from_numpy(b.astype(np.float32)).cuda()
    out2, S2 = gdn.chunk_fwd(d["q"], d["k"], d["v"], gt, bt, d["state_in"])
    torch.cuda.synchronize()
    assert max_rel(to_np(out), to_np(out2)) <= TOL["bf16"]
    assert max_rel(to_np(S), to_np(S2)) <= TOL["bf16"]
