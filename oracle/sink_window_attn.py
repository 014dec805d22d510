"""fp64 reference for the softmax blocks' sink + sliding-window attention.
TEST INFRASTRUCTURE ONLY.

The hybrid DiT puts a softmax attention block among the GDN blocks at even
intervals, and each keeps a persistent sink plus a sliding window, so its
memory is fixed by the window size while it still sees fine correspondences
across chunk boundaries ("SANA-Streaming：基于混合扩散Transformer的实时流式
视频编辑系统", 核心方法).  Softmax attention itself is the dot-product,
softmax-normalised token interaction that the same page's background section
(线性注意力 vs Softmax注意力) contrasts with linear attention; its KV cache is
what the window bounds.

The pages fix neither the sink nor the window size, nor their unit.  Reading
taken here (the plainest one the streaming setup supports): the stream is
generated chunk by chunk (3 latent frames per chunk: same page, 方法步骤详情,
second step), so the sink and the window are counted in whole chunks.  With
``n_sink`` sink chunks and a window of ``window`` chunks (the current chunk
included), a query token in chunk c attends to every token of chunk m iff

    m <= c   and   (m < n_sink  or  m > c - window)

-- the chunk's own tokens in both directions, the ``window - 1`` chunks before
it, and the stream's first ``n_sink`` chunks forever.  The attention is
softmax(q k^T / sqrt(d)) v over exactly those keys.

``visible_chunks`` is that rule; ``attend`` the softmax over an explicit key
set; ``stream_outputs`` runs the rule over a whole stream held in memory (no
cache, no ring: the definition, not the streaming bookkeeping).
``tests/test_oracle_sink_window.py`` pins it to a hand-derived example, closed forms
(uniform weights when q = 0), invariances and PyTorch's own attention.
"""
from __future__ import annotations

import numpy as np


def visible_chunks(c: int, n_sink: int, window: int) -> list[int]:
    """The chunks a query in chunk c sees, in stream order."""
    return [m for m in range(c + 1) if m < n_sink or m > c - window]


def attend(q, k, v, scale=None):
    """softmax(q k^T * scale) v in float64 for one (batch, head):
    q [n, d], k [L, d], v [L, dv] -> [n, dv].  scale defaults to 1/sqrt(d)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    if scale is None:
        scale = 1.0 / np.sqrt(q.shape[-1])
    s = (q @ k.T) * scale
    s = s - s.max(axis=-1, keepdims=True)     # the same weights, no overflow
    p = np.exp(s)
    p = p / p.sum(axis=-1, keepdims=True)
    return p @ v


def chunk_output(q_c, k_stream, v_stream, c: int, chunk: int, n_sink: int, window: int):
    """Output of chunk c.  q_c [B, chunk, H, d]; k_stream, v_stream hold the
    stream's chunks 0..c (at least) as [B, >= (c+1)*chunk, H, d]."""
    B, n, H, _ = q_c.shape
    dv = v_stream.shape[-1]
    rows = np.concatenate([np.arange(m * chunk, (m + 1) * chunk)
                           for m in visible_chunks(c, n_sink, window)])
    out = np.empty((B, n, H, dv), np.float64)
    for b in range(B):
        for h in range(H):
            out[b, :, h] = attend(q_c[b, :, h], k_stream[b, rows, h], v_stream[b, rows, h])
    return out


def stream_outputs(q, k, v, chunk: int, n_sink: int, window: int):
    """Every chunk's output of a whole stream: q, k, v [B, C*chunk, H, d]."""
    C = q.shape[1] // chunk
    return np.concatenate([chunk_output(q[:, c * chunk:(c + 1) * chunk], k, v, c, chunk,
                                        n_sink, window) for c in range(C)], axis=1)
