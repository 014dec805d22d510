"""The allocation-free entry point, gdn_chunk_fwd_noalloc.

Some callers cannot let a library allocate device memory: a streaming server
that has already given all free HBM to its caches, where an allocation in the
middle of a stream can fail or stall, or a process without the CUDA
memory-pool API.  gdn_chunk_fwd_noalloc serves them by running the same
kernels as gdn_chunk_fwd on a fixed scratch array held in device memory.

These tests call it through the C ABI, twice in a row on different inputs (so
the second call runs on the scratch the first one left behind) and check:

* its results equal gdn_chunk_fwd's bit for bit (the same kernels on the same
  inputs) and are within the bf16 tolerance of the fp64 oracle;
* a NULL state_in (zero state) and an in-place state (state_out == state_in);
* that it allocates nothing: free device memory and the default memory
  pool's high-water mark are unchanged across the calls;
* that with GDN_DEBUG_SYNC=1 the call itself reports an expired bounded wait;
* that a problem beyond the scratch is refused before anything is launched.

This file is collected last so that a failure here cannot hide any other
test's result.
"""
import ctypes
import dataclasses
import glob
import os

import pytest
import torch

import gated_deltanet_linear_chunked_b200 as gdn
from gated_deltanet_linear_chunked_b200 import _lib
from gated_deltanet_linear_chunked_b200 import workloads as wl

from gdn_testlib import TOL, device_inputs, host_inputs, max_rel, oracle_run, to_np

pytestmark = pytest.mark.gpu

CUDA_MEMPOOL_ATTR_USED_MEM_HIGH = 0x8


def _cudart():
    try:
        return ctypes.CDLL("libcudart.so.12")
    except OSError:
        import nvidia
        root = os.path.dirname(nvidia.__path__[0])
        for p in glob.glob(os.path.join(root, "nvidia", "cuda_runtime", "lib", "libcudart.so*")):
            return ctypes.CDLL(p)
        raise


class DefaultPool:
    """The current device's default memory pool, through the CUDA runtime."""

    def __init__(self):
        self.rt = _cudart()
        self.pool = ctypes.c_void_p()
        assert self.rt.cudaDeviceGetDefaultMemPool(ctypes.byref(self.pool),
                                                   torch.cuda.current_device()) == 0

    def reset_high(self):
        zero = ctypes.c_uint64(0)
        assert self.rt.cudaMemPoolSetAttribute(self.pool, CUDA_MEMPOOL_ATTR_USED_MEM_HIGH,
                                               ctypes.byref(zero)) == 0

    def high(self) -> int:
        v = ctypes.c_uint64(0)
        assert self.rt.cudaMemPoolGetAttribute(self.pool, CUDA_MEMPOOL_ATTR_USED_MEM_HIGH,
                                               ctypes.byref(v)) == 0
        return v.value


def _noalloc(x, out, state_in, state_out, w):
    lib = _lib.load()
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    return lib.gdn_chunk_fwd_noalloc(
        p(x["q"]), p(x["k"]), p(x["v"]), p(x["g"]), p(x["beta"]), p(state_in), p(state_out),
        p(out), w.B, w.T, w.H, w.Dk, w.Dv, _lib.GDN_BF16, 0,
        torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_allocating_entry_point_twice():
    """Two calls in a row.  The first call on a device may load the module
    that holds the fixed array (the CUDA driver places it then, once), so free
    device memory is compared across the second call; the default pool's
    high-water mark across both."""
    pool = DefaultPool()
    for it, w in enumerate((wl.stream_chunk("fwd"), wl.stream_chunk("fwd", seed=77))):
        x = device_inputs(w)
        ref_out, ref_S = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"])
        out = torch.empty_like(ref_out)
        S = torch.empty_like(ref_S)
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        pool.reset_high()
        high0 = pool.high()
        assert _noalloc(x, out, x["state_in"], S, w) == _lib.GDN_OK
        torch.cuda.synchronize()
        assert pool.high() == high0
        if it == 1:
            assert torch.cuda.mem_get_info()[0] == free0
        assert gdn.device_error() == _lib.GDN_OK
        assert torch.equal(out, ref_out)
        assert torch.equal(S, ref_S)
        ref_o, ref_s = oracle_run(w, host_inputs(w))
        assert max_rel(to_np(out), ref_o) <= TOL["bf16"]
        assert max_rel(to_np(S), ref_s) <= TOL["bf16"]


def test_noalloc_zero_and_in_place_state():
    w = wl.Workload("noalloc_state", 2, 300, 3, 64, 64, "bf16", 64, "fwd",
                    ("uniform", -0.5, 0.0), ("sigmoid",), ("normal", 0.02), 4141)
    x = device_inputs(w)
    # NULL state_in: a zero state
    out0 = torch.empty_like(x["v"])
    S0 = torch.empty_like(x["state_in"])
    assert _noalloc(x, out0, None, S0, w) == _lib.GDN_OK
    ref_out0, ref_S0 = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None)
    torch.cuda.synchronize()
    assert torch.equal(out0, ref_out0) and torch.equal(S0, ref_S0)
    ro, rs = oracle_run(w, dict(host_inputs(w), state_in=None))
    assert max_rel(to_np(out0), ro) <= TOL["bf16"] and max_rel(to_np(S0), rs) <= TOL["bf16"]
    # in place: state_out == state_in
    S = x["state_in"].clone()
    out = torch.empty_like(x["v"])
    assert _noalloc(x, out, S, S, w) == _lib.GDN_OK
    ref_out, ref_S = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"])
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out) and torch.equal(S, ref_S)


def test_noalloc_debug_sync_reports_expired_wait(monkeypatch):
    """With GDN_DEBUG_SYNC=1 and a one-poll wait limit (a host setting: no
    bad address, no trap) the call returns GDN_ERR_TIMEOUT itself; with the
    default limit the next call is right again."""
    w = wl.Workload("noalloc_fail", 1, 2640, 4, 64, 64, "bf16", 64, "fwd",
                    ("uniform", -0.5, 0.0), ("sigmoid",), ("normal", 0.02), 31338)
    x = device_inputs(w)
    out = torch.empty_like(x["v"])
    S = torch.empty_like(x["state_in"])
    assert gdn.device_error() == _lib.GDN_OK
    monkeypatch.setenv("GDN_DEBUG_SYNC", "1")
    gdn.set_wait_limit(1)
    try:
        st = _noalloc(x, out, x["state_in"], S, w)
    finally:
        gdn.set_wait_limit(0)
    assert st == _lib.GDN_ERR_TIMEOUT
    assert gdn.device_error() == _lib.GDN_OK          # the call already cleared it
    assert _noalloc(x, out, x["state_in"], S, w) == _lib.GDN_OK
    monkeypatch.delenv("GDN_DEBUG_SYNC")
    torch.cuda.synchronize()
    ro, rs = oracle_run(w, host_inputs(w))
    assert max_rel(to_np(out), ro) <= TOL["bf16"] and max_rel(to_np(S), rs) <= TOL["bf16"]


def test_noalloc_refuses_problem_beyond_its_scratch():
    w = dataclasses.replace(wl.stream_chunk("fwd"), B=2)   # 1680 chunk-heads
    q = torch.empty(w.B, w.T, w.H, w.Dk, dtype=torch.bfloat16, device="cuda")
    g = torch.empty(w.B, w.T, w.H, device="cuda")
    x = {"q": q, "k": torch.empty_like(q), "v": torch.empty_like(q), "g": g,
         "beta": torch.empty_like(g)}
    s_in = torch.zeros(w.B, w.H, w.Dk, w.Dv, device="cuda")
    out = torch.empty_like(q)
    S = torch.empty_like(s_in)
    c0 = _lib.load().gdn_launch_count()
    assert _noalloc(x, out, s_in, S, w) == _lib.GDN_ERR_SCRATCH_LIMIT
    assert _lib.load().gdn_launch_count() == c0
    assert _lib.load().gdn_status_string(_lib.GDN_ERR_SCRATCH_LIMIT).decode() == "GDN_ERR_SCRATCH_LIMIT"
