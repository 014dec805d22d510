"""GPU parity of the time-segmented recurrence: segment maps formed in
parallel, a prefix over the segments, then every segment walked from its
true start state.  Compared with the fp64 oracle (and with the unsegmented
path) at the bf16 bar, 2e-2, per head."""
import contextlib

import numpy as np
import pytest
import torch

import gated_deltanet_linear_chunked_b200 as gdn
from gated_deltanet_linear_chunked_b200 import workloads as wl

from gdn_testlib import TOL, device_inputs, host_inputs, max_rel, max_rel_per_head, oracle_head, oracle_run, to_np

pytestmark = pytest.mark.gpu


@contextlib.contextmanager
def segments(n):
    old = gdn.set_time_segments(n)
    try:
        yield
    finally:
        gdn.set_time_segments(old)


def run(w, x, state_in="x"):
    fn = gdn.chunk_bidir if w.mode == "bidir" else gdn.chunk_fwd
    s = x["state_in"] if state_in == "x" else state_in
    out, S = fn(x["q"], x["k"], x["v"], x["g"], x["beta"], s)
    torch.cuda.synchronize()
    assert gdn.device_error() == 0
    return out, S


def dev(xh):
    d = {n: torch.from_numpy(np.ascontiguousarray(xh[n])).cuda() for n in ("q", "k", "v", "g", "beta")}
    for n in ("q", "k", "v"):
        d[n] = d[n].to(torch.bfloat16)
    d["state_in"] = None if xh["state_in"] is None else torch.from_numpy(xh["state_in"]).cuda()
    return d


@pytest.mark.parametrize("mode", ["fwd", "bidir"])
@pytest.mark.parametrize("G", [2, 3, 7])
@pytest.mark.parametrize("D,T", [(16, 650), (64, 650), (112, 1000), (128, 200)])
def test_forced_segments_match_oracle(D, T, G, mode):
    """Forced segment counts, ragged last segments and ragged last chunks."""
    w = wl.Workload(f"seg_D{D}_T{T}", 2, T, 3, D, D, "bf16", 64, mode, ("uniform", -0.5, 0.0),
                    ("sigmoid",), ("normal", 0.02), 81000 + D + T + G)
    xh = host_inputs(w)
    x = dev(xh)
    with segments(G):
        out, S = run(w, x)
    with segments(1):
        out1, S1 = run(w, x)
    ro, rs = oracle_run(w, xh)
    o, s = to_np(out), to_np(S)
    assert max_rel_per_head(o, ro, (0, 2)) <= TOL["bf16"]
    assert max_rel_per_head(s, rs, (0, 1)) <= TOL["bf16"]
    assert max_rel(o, to_np(out1)) <= TOL["bf16"] and max_rel(s, to_np(S1)) <= TOL["bf16"]


@pytest.mark.parametrize("gate", [("uniform", -1e-4, 0.0), ("uniform", -8.0, -4.0)])
def test_segments_at_gate_extremes(gate):
    """Near-identity decay (the segment maps stay close to products of
    reflections) and fast decay (they vanish), beta 0.99, forced G = 5."""
    w = wl.Workload("seg_gate", 1, 1400, 2, 64, 64, "bf16", 64, "fwd", gate, ("const", 0.99),
                    ("normal", 0.02), 82000)
    xh = host_inputs(w)
    with segments(5):
        out, S = run(w, dev(xh))
    ro, rs = oracle_run(w, xh)
    assert max_rel_per_head(to_np(out), ro, (0, 2)) <= TOL["bf16"]
    assert max_rel_per_head(to_np(S), rs, (0, 1)) <= TOL["bf16"]


def test_segments_zero_and_in_place_state():
    w = wl.Workload("seg_state", 1, 900, 2, 64, 64, "bf16", 64, "fwd", ("uniform", -0.5, 0.0),
                    ("sigmoid",), ("normal", 0.02), 83000)
    xh = host_inputs(w)
    x = dev(xh)
    with segments(4):
        S = x["state_in"].clone()
        out, S2 = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], S, state_out=S)
        out0, S0 = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None)
        torch.cuda.synchronize()
    ro, rs = oracle_run(w, xh)
    assert max_rel(to_np(out), ro) <= TOL["bf16"] and max_rel(to_np(S), rs) <= TOL["bf16"]
    ro0, rs0 = oracle_run(w, dict(xh, state_in=None))
    assert max_rel(to_np(out0), ro0) <= TOL["bf16"] and max_rel(to_np(S0), rs0) <= TOL["bf16"]


@pytest.mark.parametrize("mode", ["fwd", "bidir"])
def test_automatic_segments_single_head_stream(mode):
    """One head, 4096 tokens (64 chunks, 4 state slices): too few chains to
    fill the GPU, so the library segments on its own."""
    w = wl.Workload("seg_auto", 1, 4096, 1, 64, 64, "bf16", 64, mode, ("uniform", -0.5, 0.0),
                    ("sigmoid",), ("normal", 0.02), 84000)
    xh = host_inputs(w)
    out, S = run(w, dev(xh))
    ro, rs = oracle_run(w, xh)
    assert max_rel(to_np(out), ro) <= TOL["bf16"] and max_rel(to_np(S), rs) <= TOL["bf16"]


def test_long_stream_segmented():
    """B1 H2 d128 T65536 (1024 chunks), slow decay, automatic segments:
    both heads against the fp64 oracle."""
    w = wl.Workload("seg_long", 1, 65536, 2, 128, 128, "bf16", 64, "fwd", ("uniform", -1e-2, 0.0),
                    ("sigmoid",), ("normal", 0.02), 85000)
    x = device_inputs(w)
    out, S = run(w, x)
    s_in = wl.make_state(w)
    for h in range(2):
        ro, rs = oracle_head(w, 0, h, s_in[:, h:h + 1])
        assert max_rel(to_np(out[0, :, h]), ro[0, :, 0]) <= TOL["bf16"]
        assert max_rel(to_np(S[0, h]), rs[0, 0]) <= TOL["bf16"]
