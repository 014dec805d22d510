"""Thin torch-facing binding of the C ABI (include/gdn.h).

Argument marshalling only: each function checks that it was handed CUDA
tensors of the expected shapes and dtypes, allocates outputs the caller did
not supply, and passes raw pointers, sizes and the current CUDA stream to
libgdn.so.  Every step of the scan runs in the library's kernels; there is
no CPU or PyTorch fallback.

Layouts: q, k [B,T,H,Dk]; v, out [B,T,H,Dv] (bf16 or fp32); g, beta [B,T,H]
fp32; state [B,H,Dk,Dv] fp32.
"""
from __future__ import annotations

import torch

from . import _lib

_DTYPES = {torch.float32: _lib.GDN_F32, torch.bfloat16: _lib.GDN_BF16}


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check_tensor(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _scan(entry, q, k, v, g, beta, state_in, state_out, out, chunk, stream, logits=False):
    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k must be [B,T,H,Dk] and v [B,T,H,Dv]")
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    if q.dtype not in _DTYPES:
        raise TypeError(f"q/k/v must be bfloat16 or float32, got {q.dtype}")
    dt = q.dtype
    _check_tensor(q, "q", dt)
    _check_tensor(k, "k", dt, (B, T, H, Dk))
    _check_tensor(v, "v", dt, (B, T, H, Dv))
    gdt = dt if logits else torch.float32  # gate logits come in the I/O dtype
    _check_tensor(g, "g_logit" if logits else "g", gdt, (B, T, H))
    _check_tensor(beta, "beta_logit" if logits else "beta", gdt, (B, T, H))
    if state_in is not None:
        _check_tensor(state_in, "state_in", torch.float32, (B, H, Dk, Dv))
    if state_out is None:
        state_out = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device)
    else:
        _check_tensor(state_out, "state_out", torch.float32, (B, H, Dk, Dv))
    if out is None:
        out = torch.empty((B, T, H, Dv), dtype=dt, device=q.device)
    else:
        _check_tensor(out, "out", dt, (B, T, H, Dv))
    lib = _lib.load()
    st = getattr(lib, entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                             _ptr(state_in), _ptr(state_out), _ptr(out),
                             B, T, H, Dk, Dv, _DTYPES[dt], int(chunk), _stream(stream))
    _lib.check(st, entry)
    return out, state_out


def chunk_fwd(q, k, v, g, beta, state_in=None, state_out=None, out=None, chunk=0,
              stream=None):
    """Causal scan of one chunk from ``state_in`` (None = zero state).
    Returns ``(out, state_out)``; ``state_out`` may be ``state_in`` (in place)."""
    return _scan("gdn_chunk_fwd", q, k, v, g, beta, state_in, state_out, out, chunk, stream)


def chunk_bidir(q, k, v, g, beta, state_in=None, state_out=None, out=None, chunk=0,
                stream=None):
    """Forward scan from ``state_in`` plus the in-chunk reverse scan from zero,
    summed.  ``state_out`` is the forward scan's final state."""
    return _scan("gdn_chunk_bidir", q, k, v, g, beta, state_in, state_out, out, chunk, stream)


def chunk_fwd_logits(q, k, v, g_logit, beta_logit, state_in=None, state_out=None, out=None,
                     chunk=0, stream=None):
    """Causal scan with the fused gate prologue: ``g_logit`` and ``beta_logit``
    [B,T,H] (same dtype as q) are the gate layer's logits; the library forms
    g = -softplus(g_logit) and beta = sigmoid(beta_logit) itself."""
    return _scan("gdn_chunk_fwd_logits", q, k, v, g_logit, beta_logit, state_in, state_out, out,
                 chunk, stream, logits=True)


def chunk_bidir_logits(q, k, v, g_logit, beta_logit, state_in=None, state_out=None, out=None,
                       chunk=0, stream=None):
    """Bidirectional scan with the fused gate prologue (see chunk_fwd_logits)."""
    return _scan("gdn_chunk_bidir_logits", q, k, v, g_logit, beta_logit, state_in, state_out, out,
                 chunk, stream, logits=True)


def _backward(entry, q, k, v, g, beta, state_in, d_out, d_state_out, stream):
    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k must be [B,T,H,Dk] and v [B,T,H,Dv]")
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    if q.dtype not in _DTYPES:
        raise TypeError(f"q/k/v must be bfloat16 or float32, got {q.dtype}")
    dt = q.dtype
    _check_tensor(q, "q", dt)
    _check_tensor(k, "k", dt, (B, T, H, Dk))
    _check_tensor(v, "v", dt, (B, T, H, Dv))
    _check_tensor(g, "g", torch.float32, (B, T, H))
    _check_tensor(beta, "beta", torch.float32, (B, T, H))
    _check_tensor(d_out, "d_out", dt, (B, T, H, Dv))
    if state_in is not None:
        _check_tensor(state_in, "state_in", torch.float32, (B, H, Dk, Dv))
    if d_state_out is not None:
        _check_tensor(d_state_out, "d_state_out", torch.float32, (B, H, Dk, Dv))
    dev = q.device
    res = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
           "dg": torch.empty_like(g), "dbeta": torch.empty_like(beta),
           "dstate_in": torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=dev)}
    st = getattr(_lib.load(), entry)(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in), _ptr(d_out),
        _ptr(d_state_out), _ptr(res["dq"]), _ptr(res["dk"]), _ptr(res["dv"]), _ptr(res["dg"]),
        _ptr(res["dbeta"]), _ptr(res["dstate_in"]), B, T, H, Dk, Dv, _DTYPES[dt], _stream(stream))
    _lib.check(st, entry)
    return res


def chunk_fwd_backward(q, k, v, g, beta, state_in, d_out, d_state_out=None, stream=None):
    """Gradients of the causal scan: returns a dict with dq, dk, dv (q's dtype),
    dg, dbeta and dstate_in (fp32), given d_out and optionally d_state_out."""
    return _backward("gdn_chunk_fwd_backward", q, k, v, g, beta, state_in, d_out, d_state_out,
                     stream)


def chunk_bidir_backward(q, k, v, g, beta, state_in, d_out, d_state_out=None, stream=None):
    """Gradients of the bidirectional scan (see chunk_fwd_backward)."""
    return _backward("gdn_chunk_bidir_backward", q, k, v, g, beta, state_in, d_out, d_state_out,
                     stream)


def sink_window_cache(B, Tc, H, D, n_sink, window, device=None):
    """An empty (zeroed) KV cache pair for ``sink_window_attention``:
    two bf16 tensors [B, n_sink + window, Tc, H, D]."""
    shape = (B, n_sink + window, Tc, H, D)
    return (torch.zeros(shape, dtype=torch.bfloat16, device=device or "cuda"),
            torch.zeros(shape, dtype=torch.bfloat16, device=device or "cuda"))


def sink_window_slot(chunk_index, n_sink, window) -> int:
    """Cache slot that holds stream chunk ``chunk_index`` (-1: invalid)."""
    return int(_lib.load().gdn_sink_window_slot(int(chunk_index), int(n_sink), int(window)))


def sink_window_attention(q, k, v, k_cache, v_cache, chunk_index, n_sink, window, out=None,
                          stream=None):
    """Softmax attention of one streaming chunk over the sink chunks and the
    sliding window of chunks (its own included) held in ``k_cache`` /
    ``v_cache``; writes the chunk's k, v into its cache slot on the way.
    q, k, v [B, Tc, H, D] bf16; caches [B, n_sink + window, Tc, H, D] bf16.
    Returns ``out`` [B, Tc, H, D] bf16."""
    if q.dim() != 4:
        raise ValueError("q, k, v must be [B, Tc, H, D]")
    B, Tc, H, D = q.shape
    _check_tensor(q, "q", torch.bfloat16)
    _check_tensor(k, "k", torch.bfloat16, (B, Tc, H, D))
    _check_tensor(v, "v", torch.bfloat16, (B, Tc, H, D))
    cshape = (B, n_sink + window, Tc, H, D)
    _check_tensor(k_cache, "k_cache", torch.bfloat16, cshape)
    _check_tensor(v_cache, "v_cache", torch.bfloat16, cshape)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_tensor(out, "out", torch.bfloat16, (B, Tc, H, D))
    st = _lib.load().gdn_sink_window_attention(
        _ptr(q), _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(out), B, Tc, H, D,
        int(n_sink), int(window), int(chunk_index), _lib.GDN_BF16, _stream(stream))
    _lib.check(st, "gdn_sink_window_attention")
    return out


def state_reset(state, stream=None):
    """Zero a state tensor [B,H,Dk,Dv] in place (streaming restart)."""
    _check_tensor(state, "state", torch.float32)
    if state.dim() != 4:
        raise ValueError("state must be [B,H,Dk,Dv]")
    B, H, Dk, Dv = state.shape
    st = _lib.load().gdn_state_reset(_ptr(state), B, H, Dk, Dv, _stream(stream))
    _lib.check(st, "gdn_state_reset")
    return state


def device_error(stream=None) -> int:
    """Synchronise and read/clear the device error word (0 = none)."""
    return int(_lib.load().gdn_device_error(_stream(stream)))


def workspace_release() -> None:
    """Free the library's per-stream scratch and error words on the current
    device (after synchronising it).  No captured graph holding this
    library's launches may be replayed afterwards."""
    _lib.check(_lib.load().gdn_workspace_release(), "gdn_workspace_release")


def set_time_segments(segments: int) -> int:
    """Time segments of the bf16 path's recurrence: 0 = automatic, 1 = never,
    G >= 2 = exactly G.  Process-wide; returns the previous setting."""
    return int(_lib.load().gdn_set_time_segments(int(segments)))


def set_wait_limit(polls: int) -> int:
    """Polls a kernel's bounded wait makes before giving up (0 = default)."""
    return int(_lib.load().gdn_set_wait_limit(int(polls)))
