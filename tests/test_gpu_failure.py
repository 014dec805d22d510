"""Failure detection and instrumentation on the GPU, without faulting it.

The tensor-core kernels bound every mbarrier wait; when a wait runs out the
CTA sets the device error word, drains what it was waiting for, frees its
tensor memory and returns.  The test makes the waits run out by setting the
poll limit to a single poll (a host-side setting, no bad address, no trap),
checks that the host sees GDN_ERR_TIMEOUT, and that the context stays usable:
the next call with the default limit matches the oracle.
"""
import ctypes

import pytest
import torch

import gated_deltanet_linear_chunked_b200 as gdn
from gated_deltanet_linear_chunked_b200 import _lib
from gated_deltanet_linear_chunked_b200 import workloads as wl

from gdn_testlib import TOL, device_inputs, host_inputs, max_rel, oracle_run, to_np

pytestmark = pytest.mark.gpu


def small_workload():
    return wl.Workload("fail", 1, 2640, 4, 64, 64, "bf16", 64, "fwd",
                       ("uniform", -0.5, 0.0), ("sigmoid",), ("normal", 0.02), 31337)


def test_wait_expiry_reports_timeout_and_context_survives():
    w = small_workload()
    x = device_inputs(w)
    assert gdn.device_error() == _lib.GDN_OK
    gdn.set_wait_limit(1)
    try:
        gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"])
        st = gdn.device_error()
    finally:
        gdn.set_wait_limit(0)
    assert st == _lib.GDN_ERR_TIMEOUT
    assert gdn.device_error() == _lib.GDN_OK          # read-and-clear
    out, S = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"])
    torch.cuda.synchronize()
    assert gdn.device_error() == _lib.GDN_OK
    ref_o, ref_S = oracle_run(w, host_inputs(w))
    assert max_rel(to_np(out), ref_o) <= TOL["bf16"]
    assert max_rel(to_np(S), ref_S) <= TOL["bf16"]


def test_error_words_are_per_stream():
    """An expired wait on one stream is reported on that stream only: a
    second stream's calls, before and after, see GDN_OK."""
    w = small_workload()
    x = device_inputs(w)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    for s in (s1, s2):  # give both streams their context before the fault injection
        gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"], stream=s)
        assert gdn.device_error(s) == _lib.GDN_OK
    gdn.set_wait_limit(1)
    try:
        gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"], stream=s1)
        s1.synchronize()
    finally:
        gdn.set_wait_limit(0)
    out2, S2 = gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"], stream=s2)
    assert gdn.device_error(s2) == _lib.GDN_OK
    assert gdn.device_error(s1) == _lib.GDN_ERR_TIMEOUT
    assert gdn.device_error(s1) == _lib.GDN_OK
    torch.cuda.synchronize()
    ref_o, ref_S = oracle_run(w, host_inputs(w))
    assert max_rel(to_np(out2), ref_o) <= TOL["bf16"]
    assert max_rel(to_np(S2), ref_S) <= TOL["bf16"]


def test_profile_hook_counts_each_kernel():
    w = small_workload()
    x = device_inputs(w)
    lib = _lib.load()
    assert lib.gdn_profile_begin(16) == _lib.GDN_OK
    for _ in range(2):
        gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"])
    ms = (ctypes.c_float * 4)()
    n = (ctypes.c_int * 4)()
    assert lib.gdn_profile_end(ctypes.addressof(ms), ctypes.addressof(n), 4) == _lib.GDN_OK
    assert list(n) == [0, 2, 2, 2]
    assert all(ms[i] > 0 for i in (1, 2, 3))
    assert lib.gdn_kernel_name(1).decode() == "gdn_prep_kernel"
