"""GPU parity of the softmax blocks' sink + sliding-window attention
(gdn_sink_window_attention) against the fp64 oracle.

Each test streams chunks 0, 1, 2, ... through the library on one KV cache,
exactly as a softmax block does, and after every call checks:

* the output against ``oracle.sink_window_attn.chunk_output`` on the same
  bf16 inputs, element by element, with the bf16 bar (max |x - ref| /
  max |ref| <= 2e-2), per (b, h) so a wrong head cannot hide;
* that the chunk's k and v landed in its cache slot bit for bit (byte work).

Shapes cover ragged tiles (Tc not a multiple of 64 or 128, Tc = 1), every
supported head width class, grids whose last pairs of query tiles run as
single tiles, several (n_sink, window) pairs including no sink
and a one-chunk window, the full streaming chunk (B1 H20 D112 Tc2640, one
sink chunk, window 2: 7920 keys from chunk 2 on), a sharp softmax that makes
the running maximum grow (the rescale path), inputs that are the cache slot
itself, and an expired bounded wait.
"""
import numpy as np
import pytest
import torch

import gated_deltanet_linear_chunked_b200 as gdn
from gated_deltanet_linear_chunked_b200 import _lib
from gated_deltanet_linear_chunked_b200 import workloads as wl
from oracle import sink_window_attn as swa

from gdn_testlib import TOL, max_rel, max_rel_per_head, to_np

pytestmark = pytest.mark.gpu


def _dev(x):
    return {n: torch.from_numpy(a).to("cuda", torch.bfloat16) for n, a in x.items()}


def _stream(w, heads_only=None):
    """Runs the stream; yields (c, got, ref) per chunk."""
    kc, vc = gdn.sink_window_cache(w.B, w.Tc, w.H, w.D, w.n_sink, w.window)
    ks, vs = [], []
    for c in range(w.chunks):
        x = wl.attn_chunk(w, c)
        ks.append(x["k"])
        vs.append(x["v"])
        d = _dev(x)
        out = gdn.sink_window_attention(d["q"], d["k"], d["v"], kc, vc, c, w.n_sink, w.window)
        torch.cuda.synchronize()
        assert gdn.device_error() == _lib.GDN_OK
        slot = gdn.sink_window_slot(c, w.n_sink, w.window)
        assert torch.equal(kc[:, slot], d["k"]) and torch.equal(vc[:, slot], d["v"]), c
        ref = swa.chunk_output(x["q"], np.concatenate(ks, 1), np.concatenate(vs, 1), c, w.Tc,
                               w.n_sink, w.window)
        yield c, to_np(out), ref


SMALL = [
    # B, Tc, H, D, n_sink, window, chunks
    (2, 200, 3, 64, 1, 2, 6),
    (1, 64, 2, 16, 0, 1, 3),
    (1, 129, 2, 128, 2, 3, 7),
    (3, 1, 2, 32, 1, 1, 4),
    (1, 300, 4, 112, 0, 4, 6),
    (1, 257, 2, 48, 3, 1, 5),
    (2, 640, 2, 96, 1, 3, 5),
    # pairs of query tiles just above a B200's 148 SMs: the last pairs run as
    # single tiles (a ragged pair of 128 + 72 rows; a pair whose second tile
    # is missing)
    (1, 200, 150, 32, 1, 2, 3),
    (1, 100, 160, 16, 0, 2, 3),
]


@pytest.mark.parametrize("B,Tc,H,D,n_sink,window,chunks", SMALL)
def test_streams_match_oracle(B, Tc, H, D, n_sink, window, chunks):
    w = wl.AttnStream(f"swa_{Tc}_{D}", B, Tc, H, D, n_sink, window, chunks, seed=100 + Tc + D)
    for c, got, ref in _stream(w):
        err = max_rel_per_head(got, ref, (0, 2))
        assert err <= TOL["bf16"], (c, err)


def test_full_streaming_chunk_matches_oracle():
    w = wl.sink_window_stream()
    seen = []
    for c, got, ref in _stream(w):
        err = max_rel_per_head(got, ref, (0, 2))
        seen.append(err)
        assert err <= TOL["bf16"], (c, err)
    assert len(seen) == w.chunks and w.chunks > w.steady_chunk


def test_sharp_softmax_matches_oracle():
    """q ~ N(0, 36): scores spread over about +-20, so a row's running maximum
    grows past the rescale headroom across tiles."""
    w = wl.AttnStream("swa_sharp", 1, 1000, 2, 64, 1, 2, 4, seed=77, q_scale=6.0)
    for c, got, ref in _stream(w):
        err = max_rel_per_head(got, ref, (0, 2))
        assert err <= TOL["bf16"], (c, err)


def test_extremely_sharp_softmax_matches_oracle():
    """q ~ N(0, 40^2): scores span hundreds of units of log2, so a row maximum
    that missed any column would overflow or underflow 2^(s - m)."""
    w = wl.AttnStream("swa_extreme", 1, 700, 2, 64, 1, 2, 3, seed=78, q_scale=40.0)
    for c, got, ref in _stream(w):
        assert np.isfinite(got).all(), c
        err = max_rel_per_head(got, ref, (0, 2))
        assert err <= TOL["bf16"], (c, err)


def test_inputs_that_are_the_cache_slot():
    """A projection may write k, v straight into the chunk's slot: the call
    then stores the same bytes over themselves and the result is the same."""
    w = wl.AttnStream("swa_inplace", 1, 333, 3, 64, 1, 2, 4, seed=31)
    kc, vc = gdn.sink_window_cache(w.B, w.Tc, w.H, w.D, w.n_sink, w.window)
    kc2, vc2 = gdn.sink_window_cache(w.B, w.Tc, w.H, w.D, w.n_sink, w.window)
    for c in range(w.chunks):
        d = _dev(wl.attn_chunk(w, c))
        ref = gdn.sink_window_attention(d["q"], d["k"], d["v"], kc, vc, c, w.n_sink, w.window)
        slot = gdn.sink_window_slot(c, w.n_sink, w.window)
        kc2[:, slot].copy_(d["k"])
        vc2[:, slot].copy_(d["v"])
        got = gdn.sink_window_attention(d["q"], kc2[:, slot], vc2[:, slot], kc2, vc2, c,
                                        w.n_sink, w.window)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), c
    assert torch.equal(kc, kc2) and torch.equal(vc, vc2)


def test_expired_wait_reports_timeout_and_next_call_is_right():
    """A one-poll wait limit (a host setting: no bad address, no trap) makes
    the kernel's first wait give up; the stream's error word reports it and
    the next call, with the default limit, is right."""
    w = wl.AttnStream("swa_fail", 1, 512, 2, 64, 1, 2, 1, seed=9)
    d = _dev(wl.attn_chunk(w, 0))
    kc, vc = gdn.sink_window_cache(w.B, w.Tc, w.H, w.D, w.n_sink, w.window)
    assert gdn.device_error() == _lib.GDN_OK
    gdn.set_wait_limit(1)
    try:
        gdn.sink_window_attention(d["q"], d["k"], d["v"], kc, vc, 0, w.n_sink, w.window)
        torch.cuda.synchronize()
    finally:
        gdn.set_wait_limit(0)
    assert gdn.device_error() == _lib.GDN_ERR_TIMEOUT
    assert gdn.device_error() == _lib.GDN_OK
    out = gdn.sink_window_attention(d["q"], d["k"], d["v"], kc, vc, 0, w.n_sink, w.window)
    torch.cuda.synchronize()
    ref = swa.chunk_output(*(wl.attn_chunk(w, 0)[n] for n in ("q", "k", "v")), 0, w.Tc, 1, 2)
    assert max_rel(to_np(out), ref) <= TOL["bf16"]


def test_device_side_rejections():
    """Arguments that pass the host checks but not the device ones."""
    lib = _lib.load()
    x = torch.zeros(1, 64, 2, 64, dtype=torch.bfloat16, device="cuda")
    kc, vc = gdn.sink_window_cache(1, 64, 2, 64, 1, 2)
    host = torch.zeros(1, 64, 2, 64, dtype=torch.bfloat16).pin_memory()
    s = torch.cuda.current_stream().cuda_stream
    p = [x.data_ptr(), x.data_ptr(), x.data_ptr(), kc.data_ptr(), vc.data_ptr()]
    out = torch.empty_like(x)
    assert lib.gdn_sink_window_attention(*p, host.data_ptr(), 1, 64, 2, 64, 1, 2, 0,
                                         _lib.GDN_BF16, s) == _lib.GDN_ERR_INVALID_ARG
    assert lib.gdn_sink_window_attention(*p, out.data_ptr(), 1, 64, 2, 64, 1, 2, 0,
                                         _lib.GDN_BF16, s) == _lib.GDN_OK
    torch.cuda.synchronize()
