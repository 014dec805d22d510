"""The allocation-free entry point, gdn_chunk_fwd_noalloc.

Some callers cannot let a library allocate device memory: a streaming server
that has already given all free HBM to its caches, where an allocation in the
middle of a stream can fail or stall, or a process without the CUDA
memory-pool API.  gdn_chunk_fwd_noalloc serves them by running the same
kernels as gdn_chunk_fwd on a fixed scratch array held in device memory.

These tests call it through the C ABI, twice in a row on different inputs
(so the second call runs on scratch the first one left behind), and compare
each result with gdn_chunk_fwd's on the same inputs within the bf16 parity
tolerance; they also check that an oversized problem is refused before
anything is launched.  This file is collected last so that a failure here
cannot hide any other test's result.
"""
import pytest
import torch

import gated_deltanet_linear_chunked_b200 as gdn
from gated_deltanet_linear_chunked_b200 import _lib
from gated_deltanet_linear_chunked_b200 import workloads as wl

from gdn_testlib import TOL, device_inputs, max_rel, to_np

pytestmark = pytest.mark.gpu


def _noalloc(x, out, S, w):
    lib = _lib.load()
    return lib.gdn_chunk_fwd_noalloc(
        x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), x["g"].data_ptr(),
        x["beta"].data_ptr(), x["state_in"].data_ptr(), S.data_ptr(), out.data_ptr(),
        w.B, w.T, w.H, w.Dk, w.Dv, _lib.GDN_BF16, 0, torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_allocating_entry_point_twice():
    for w in (wl.stream_chunk("fwd"), wl.stream_chunk("fwd", seed=77)):
        x = device_inputs(w)
        ref_out, ref_S = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"])
        out = torch.empty_like(ref_out)
        S = torch.empty_like(ref_S)
        assert _noalloc(x, out, S, w) == _lib.GDN_OK
        torch.cuda.synchronize()
        assert gdn.device_error() == _lib.GDN_OK
        assert max_rel(to_np(out), to_np(ref_out)) <= TOL["bf16"]
        assert max_rel(to_np(S), to_np(ref_S)) <= TOL["bf16"]


def test_noalloc_refuses_problem_beyond_its_scratch():
    import dataclasses
    w = dataclasses.replace(wl.stream_chunk("fwd"), B=2)   # 1680 chunk-heads
    q = torch.empty(w.B, w.T, w.H, w.Dk, dtype=torch.bfloat16, device="cuda")
    g = torch.empty(w.B, w.T, w.H, device="cuda")
    x = {"q": q, "k": torch.empty_like(q), "v": torch.empty_like(q), "g": g,
         "beta": torch.empty_like(g), "state_in": torch.zeros(w.B, w.H, w.Dk, w.Dv, device="cuda")}
    out = torch.empty_like(q)
    S = torch.empty_like(x["state_in"])
    assert _noalloc(x, out, S, w) == _lib.GDN_ERR_SCRATCH_LIMIT
    assert _lib.load().gdn_status_string(_lib.GDN_ERR_SCRATCH_LIMIT).decode() == "GDN_ERR_SCRATCH_LIMIT"
