"""B200-native chunked Gated DeltaNet (GDN) scan, and the sink + sliding-window
softmax attention of the same hybrid DiT's softmax blocks.

The scan runs in ``libgdn.so`` (hand-written CUDA for sm_100a, C ABI in
``include/gdn.h``); this package is its thin torch binding plus the seeded
workload generators.  Importing the package does not load CUDA; the library
is loaded on the first call.
"""
from . import workloads  # noqa: F401

_API = ("chunk_fwd", "chunk_bidir", "chunk_fwd_logits", "chunk_bidir_logits",
        "chunk_fwd_backward", "chunk_bidir_backward", "sink_window_attention",
        "sink_window_cache", "sink_window_slot", "state_reset",
        "device_error", "set_wait_limit", "set_time_segments", "workspace_release")
__all__ = [*_API, "GDNError", "workloads"]


def __getattr__(name):
    if name in _API:
        from . import api
        return getattr(api, name)
    if name == "GDNError":
        from ._lib import GDNError
        return GDNError
    raise AttributeError(name)
