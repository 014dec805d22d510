"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Every comparison is element by element on the same seeded inputs, with the
max-relative-error metric of gdn_testlib (1e-4 fp32, 2e-2 bf16), on the
outputs and on the final state.
"""
import numpy as np
import pytest
import torch

import gated_deltanet_linear_chunked_b200 as gdn
from gated_deltanet_linear_chunked_b200 import workloads as wl

from gdn_testlib import (TOL, device_inputs, host_inputs, max_rel, max_rel_per_head, max_rel_rows,
                         oracle_head, oracle_run, to_np)

pytestmark = pytest.mark.gpu


def run(w, x, state_in="from_x", chunk=None, bidir=None):
    if bidir is None:
        bidir = w.mode == "bidir"
    fn = gdn.chunk_bidir if bidir else gdn.chunk_fwd
    s = x["state_in"] if state_in == "from_x" else state_in
    out, S = fn(x["q"], x["k"], x["v"], x["g"], x["beta"], s,
                chunk=w.chunk if chunk is None else chunk)
    torch.cuda.synchronize()
    return out, S


def dev_from_host(x, dtype):
    d = {n: torch.from_numpy(np.ascontiguousarray(x[n])).cuda() for n in ("q", "k", "v", "g", "beta")}
    for n in ("q", "k", "v"):
        d[n] = d[n].to(dtype)
    d["state_in"] = None if x["state_in"] is None else torch.from_numpy(x["state_in"]).cuda()
    return d


def check(w, x_host, out, S, bidir=None, per_head=False):
    """Element-wise comparison with the oracle at the dtype's tolerance, on
    the whole tensors and, with per_head, on every (b, h) head alone."""
    ref_o, ref_S = oracle_run(w, x_host, bidir)
    o, s = to_np(out), to_np(S)
    eo, es = max_rel(o, ref_o), max_rel(s, ref_S)
    tol = TOL[w.dtype]
    assert eo <= tol and es <= tol, f"{w.name}: out {eo:.3e} state {es:.3e} tol {tol}"
    if per_head:
        ho, hs = max_rel_per_head(o, ref_o, (0, 2)), max_rel_per_head(s, ref_S, (0, 1))
        assert ho <= tol and hs <= tol, f"{w.name}: per head out {ho:.3e} state {hs:.3e} tol {tol}"
    return ref_o, ref_S


@pytest.mark.parametrize("mode", ["fwd", "bidir"])
def test_tiny_fp32_workload(mode):
    """Tiny fp32 scan (B1 H2 d16 T64, sub-chunk 16): tolerance 1e-4."""
    import dataclasses
    w = dataclasses.replace(wl.tiny(), mode=mode)
    xh = host_inputs(w)
    out, S = run(w, dev_from_host(xh, torch.float32))
    check(w, xh, out, S)


SWEEP_T = [1, 15, 16, 17, 63, 64, 65, 200]
SWEEP_D = [16, 64, 112, 128]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["fwd", "bidir"])
@pytest.mark.parametrize("D", SWEEP_D)
@pytest.mark.parametrize("T", SWEEP_T)
def test_small_sweep(T, D, mode, dtype):
    """Ragged lengths around the sub-chunk (tails of 1..63 tokens) and every
    supported head-dim class, both dtypes, both modes, carried state."""
    w = wl.Workload(f"sweep_T{T}_D{D}", 2, T, 3, D, D, dtype, 64, mode,
                    ("uniform", -0.5, 0.0), ("sigmoid",), ("normal", 0.02), 70000 + T * 7 + D)
    xh = host_inputs(w)
    out, S = run(w, dev_from_host(xh, torch.bfloat16 if dtype == "bf16" else torch.float32))
    check(w, xh, out, S)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["fwd", "bidir"])
@pytest.mark.parametrize("D", [16, 112, 128])
@pytest.mark.parametrize("T", [1, 17, 65, 200])
def test_small_sweep_unnormalised_qk(T, D, mode, dtype):
    """Ragged lengths and head-dim classes with the mixed un-normalised q/k
    recipe (rows at 1e-3 / 1e3 / under the clamp, zero rows)."""
    w = wl.Workload(f"sweepu_T{T}_D{D}", 2, T, 3, D, D, dtype, 64, mode,
                    ("uniform", -0.5, 0.0), ("sigmoid",), ("normal", 0.02), 71000 + T * 7 + D,
                    qk=("mixed",))
    xh = host_inputs(w)
    out, S = run(w, dev_from_host(xh, torch.bfloat16 if dtype == "bf16" else torch.float32))
    check(w, xh, out, S, per_head=True)


@pytest.mark.parametrize("Dk,Dv", [(32, 96), (128, 16), (64, 128), (48, 64), (80, 32), (96, 112)])
def test_rectangular_state(Dk, Dv):
    """Dk != Dv (the state is Dk x Dv; outputs are Dv wide)."""
    w = wl.Workload("rect", 1, 130, 2, Dk, Dv, "bf16", 64, "fwd",
                    ("uniform", -0.5, 0.0), ("sigmoid",), ("normal", 0.02), 808)
    xh = host_inputs(w)
    out, S = run(w, dev_from_host(xh, torch.bfloat16))
    check(w, xh, out, S)


@pytest.mark.parametrize("mode", ["fwd", "bidir"])
def test_stream_chunk_full_size(mode):
    """The 1280x704 streaming chunk (B1 H20 d112 T2640 bf16), every head
    compared with the oracle, as a whole and head by head; bidir adds the
    in-chunk reverse scan."""
    w = wl.stream_chunk(mode)
    xh = host_inputs(w)
    x = device_inputs(w)
    out, S = run(w, x)
    check(w, xh, out, S, per_head=True)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("mode", ["fwd", "bidir"])
@pytest.mark.parametrize("qk", ["raw", "mixed"])
def test_stream_chunk_unnormalised_qk(qk, mode, dtype):
    """The streaming chunk's shapes with q and k NOT pre-normalised, so the
    library's own L2 normalisation (q/|q|, k/|k|, |.|^2 clamped at 1e-12) is
    what makes the result right: raw N(0,1) rows (norm about sqrt(112)), and
    the mixed recipe with rows scaled by 1e-3 and 1e3, rows whose squared
    norm is under the clamp, and an all-zero q row and k row per head.
    Compared with the oracle on the whole tensors, head by head, and on the
    special rows each against its own scale."""
    import dataclasses
    w = dataclasses.replace(wl.stream_chunk(mode), qk=(qk,), dtype=dtype,
                            name=f"stream_{mode}_{qk}_{dtype}")
    xh = host_inputs(w)
    x = dev_from_host(xh, torch.bfloat16 if dtype == "bf16" else torch.float32)
    out, S = run(w, x)
    ref_o, _ = check(w, xh, out, S, per_head=True)
    if qk == "mixed":
        rows = wl.qk_rows(w.T)
        o = to_np(out)
        for name in ("small", "large", "subclamp", "zero_k"):
            e = max_rel_rows(o, ref_o, rows[name])
            assert e <= TOL[dtype], f"{name} rows: {e:.3e}"
        # an all-zero q row has an all-zero output (q^ = 0)
        assert not o[:, rows["zero_q"]].any()


def test_streaming_equals_one_scan_on_gpu():
    """N chunk calls with the state carried equal one call over the
    concatenation (GPU vs GPU, and both vs the oracle)."""
    w = wl.Workload("carry", 1, 700, 4, 64, 64, "bf16", 64, "fwd",
                    ("uniform", -0.5, 0.0), ("sigmoid",), ("normal", 0.02), 99)
    xh = host_inputs(w)
    x = dev_from_host(xh, torch.bfloat16)
    out_all, S_all = run(w, x)
    cuts = [0, 1, 64, 65, 300, 700]
    S = x["state_in"].clone()
    outs = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        sl = {n: x[n][:, a:b].contiguous() for n in ("q", "k", "v", "g", "beta")}
        o, S = gdn.chunk_fwd(sl["q"], sl["k"], sl["v"], sl["g"], sl["beta"], S, state_out=S)
        outs.append(o)
    torch.cuda.synchronize()
    out_cat = torch.cat(outs, dim=1)
    assert max_rel(to_np(out_cat), to_np(out_all)) <= 2e-2
    assert max_rel(to_np(S), to_np(S_all)) <= 2e-2
    check(w, xh, out_cat, S)


def test_in_place_state_and_zero_state():
    w = wl.Workload("inplace", 2, 150, 3, 32, 32, "bf16", 64, "fwd",
                    ("uniform", -0.5, 0.0), ("sigmoid",), ("normal", 0.02), 5)
    xh = host_inputs(w)
    x = dev_from_host(xh, torch.bfloat16)
    S = x["state_in"].clone()
    out, S2 = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], S, state_out=S)
    torch.cuda.synchronize()
    assert S2.data_ptr() == S.data_ptr()
    check(w, xh, out, S)
    # NULL state_in == zero state
    out0, S0 = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None)
    torch.cuda.synchronize()
    xh0 = dict(xh, state_in=None)
    check(w, xh0, out0, S0)


def test_empty_and_degenerate_calls():
    dev = "cuda"
    S_in = torch.randn(2, 3, 16, 16, device=dev)
    e = torch.empty(2, 0, 3, 16, device=dev, dtype=torch.bfloat16)
    ge = torch.empty(2, 0, 3, device=dev)
    out, S = gdn.chunk_fwd(e, e, e, ge, ge, S_in)
    torch.cuda.synchronize()
    assert torch.equal(S, S_in)
    out, S = gdn.chunk_fwd(e, e, e, ge, ge, None)
    torch.cuda.synchronize()
    assert not S.any()
    gdn.state_reset(S_in)
    torch.cuda.synchronize()
    assert not S_in.any()


def test_gate_extremes_small():
    """a = 1, beta = 0 on the GPU: the state is carried unchanged and
    o_t = S_in^T q^_t (closed form, no oracle needed)."""
    w = wl.Workload("p1", 1, 100, 2, 64, 64, "f32", 64, "fwd",
                    ("uniform", -0.5, 0.0), ("sigmoid",), ("normal", 0.5), 6)
    xh = host_inputs(w)
    xh["g"][:] = 0
    xh["beta"][:] = 0
    x = dev_from_host(xh, torch.float32)
    out, S = run(w, x)
    qn = xh["q"] / np.linalg.norm(xh["q"], axis=-1, keepdims=True)
    ref = np.einsum("bthi,bhij->bthj", qn.astype(np.float64), xh["state_in"].astype(np.float64))
    assert max_rel(to_np(out), ref) <= 1e-5
    assert max_rel(to_np(S), xh["state_in"]) <= 1e-6


def test_host_pointer_and_partial_alias_rejected():
    w = wl.Workload("err", 1, 32, 2, 16, 16, "bf16", 64, "fwd",
                    ("uniform", -0.5, 0.0), ("sigmoid",), ("normal", 0.02), 7)
    x = dev_from_host(host_inputs(w), torch.bfloat16)
    from gated_deltanet_linear_chunked_b200 import _lib
    lib = _lib.load()
    host_q = torch.empty_like(x["q"], device="cpu").pin_memory()
    out = torch.empty_like(x["v"])
    S = torch.empty(2, 2, 16, 16, device="cuda")
    args = lambda q, s_in, s_out: (q.data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(),  # noqa: E731
                                   x["g"].data_ptr(), x["beta"].data_ptr(), s_in, s_out,
                                   out.data_ptr(), 1, 32, 2, 16, 16, _lib.GDN_BF16, 0, None)
    assert lib.gdn_chunk_fwd(*args(host_q, None, S.data_ptr())) == _lib.GDN_ERR_INVALID_ARG
    # state_out starting 64 floats into state_in's range: partial overlap
    assert lib.gdn_chunk_fwd(*args(x["q"], S.data_ptr(), S.data_ptr() + 256)) == _lib.GDN_ERR_ALIAS
    assert lib.gdn_chunk_fwd(*args(x["q"], S.data_ptr(), S.data_ptr())) == _lib.GDN_OK
    torch.cuda.synchronize()
