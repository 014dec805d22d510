"""numpy fp64 transcriptions of the GDN scan.  TEST INFRASTRUCTURE ONLY.

``recurrence_fwd`` / ``recurrence_bidir``
    The definition, token by token, vectorised over (batch, head) only:

        q^ = q / sqrt(max(|q|^2, 1e-12)),  k^ likewise,  a_t = exp(g_t)
        S_t = a_t (I - beta_t k^_t k^_t^T) S_{t-1} + beta_t k^_t v_t^T
        o_t = S_t^T q^_t

    The pages describe the Gated DeltaNet only in words (a fixed-size memory
    updated recursively: "[논문리뷰] SANA-Streaming: Real-time Streaming Video
    Editing with Hybrid Diffusion Transformer", 1. Key Terms & Definitions);
    the streaming forward scan carries the previous chunk's cache and the
    bidirectional mode adds a backward scan inside the chunk
    ("SANA-Streaming：基于混合扩散Transformer的实时流式视频编辑系统",
    方法步骤详情, second step).  This is a second, independent transcription of
    the same definition as ``gdn_oracle.c``.

``chunked_fwd`` / ``chunked_bidir``
    The sub-chunked (WY / UT-transform) form of the same scan: the form the
    fused kernel's three stages compute (frame summaries, recurrent scan,
    state application: same page, 方法步骤详情, fourth step).  Derivation, per
    sub-chunk of n tokens entered with state S0 and gamma_r = sum_{i<=r} g_i:

      write u_t = beta_t (v_t - a_t S_{t-1}^T k^_t); then S_t = a_t S_{t-1} + k^_t u_t^T,
      so  S_r = e^{gamma_r} S0 + sum_{i<=r} e^{gamma_r - gamma_i} k^_i u_i^T.
      Substituting S_{t-1} into u_t gives the unit lower-triangular system
          (I + A) U = diag(beta) V - diag(beta e^gamma) K^ S0,
          A_ti = beta_t e^{gamma_t - gamma_i} k^_t . k^_i   (i < t, else 0),
      hence, with Tm = (I + A)^-1,
          W  = Tm diag(beta e^gamma) K^,   U~ = Tm diag(beta) V,   U = U~ - W S0,
          O  = diag(e^gamma) Q^ S0 + (Mask o Q^ K^^T) U,
               Mask_ti = e^{gamma_t - gamma_i} for i <= t, else 0,
          S_n = e^{gamma_n} S0 + (diag(e^{gamma_n - gamma}) K^)^T U.

    It reaches the recurrence exactly up to rounding, for every sub-chunk
    length including a ragged tail; ``tests/test_oracle_pins.py`` checks that
    by brute force.  Only differences of gamma are exponentiated where they
    can be positive, so fast decays do not overflow.
"""
from __future__ import annotations

import numpy as np


def gates_from_logits(g_logit, beta_logit):
    """Gate layer logits -> (g, beta) in fp64: g = -softplus(x) = -log(1 + e^x),
    beta = sigmoid(y) = 1 / (1 + e^-y).  The pages keep the gate layer in BF16
    ("SANA-Streaming：基于混合扩散Transformer的实时流式视频编辑系统", 实验结果)
    without writing its activations; these are the plainest maps onto g <= 0
    and beta in (0, 1).  A second transcription beside the C oracle's."""
    x = np.asarray(g_logit, np.float64)
    y = np.asarray(beta_logit, np.float64)
    g = -np.logaddexp(0.0, x)
    beta = np.exp(-np.logaddexp(0.0, -y))
    return g, beta


def _normalise(x):
    ss = np.sum(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(np.maximum(ss, 1e-12))


def _as64(*xs):
    return [np.asarray(x, dtype=np.float64) for x in xs]


def recurrence_fwd(q, k, v, g, beta, state_in=None):
    """Token-by-token forward scan.  Returns (out [B,T,H,Dv], state [B,H,Dk,Dv])."""
    q, k, v, g, beta = _as64(q, k, v, g, beta)
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    S = (np.zeros((B, H, Dk, Dv)) if state_in is None
         else np.array(state_in, dtype=np.float64, copy=True))
    out = np.zeros((B, T, H, Dv))
    for t in range(T):
        kh = _normalise(k[:, t])                       # [B,H,Dk]
        qh = _normalise(q[:, t])
        a = np.exp(g[:, t])[..., None, None]           # [B,H,1,1]
        b = beta[:, t][..., None, None]
        kkS = kh[..., :, None] * np.einsum("bhi,bhij->bhj", kh, S)[..., None, :]
        S = a * (S - b * kkS) + b * kh[..., :, None] * v[:, t][..., None, :]
        out[:, t] = np.einsum("bhi,bhij->bhj", qh, S)
    return out, S


def recurrence_bidir(q, k, v, g, beta, state_in=None):
    """Forward scan from state_in plus the reverse scan from zero, summed."""
    out_f, S = recurrence_fwd(q, k, v, g, beta, state_in)
    flip = lambda x: np.flip(np.asarray(x), axis=1)  # noqa: E731
    out_r, _ = recurrence_fwd(flip(q), flip(k), flip(v), flip(g), flip(beta), None)
    return out_f + np.flip(out_r, axis=1), S


def chunked_fwd(q, k, v, g, beta, state_in=None, chunk=64):
    """The WY / UT sub-chunked form of the forward scan (see module doc)."""
    q, k, v, g, beta = _as64(q, k, v, g, beta)
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    S_all = (np.zeros((B, H, Dk, Dv)) if state_in is None
             else np.array(state_in, dtype=np.float64, copy=True))
    out = np.zeros((B, T, H, Dv))
    for b in range(B):
        for h in range(H):
            S = S_all[b, h]
            for c0 in range(0, T, chunk):
                sl = slice(c0, min(c0 + chunk, T))
                Q = _normalise(q[b, sl, h])
                K = _normalise(k[b, sl, h])
                V = v[b, sl, h]
                bt = beta[b, sl, h]
                gam = np.cumsum(g[b, sl, h])
                n = gam.shape[0]
                diff = gam[:, None] - gam[None, :]
                lower_strict = np.tril(np.ones((n, n), dtype=bool), -1)
                lower_incl = np.tril(np.ones((n, n), dtype=bool), 0)
                A = np.where(lower_strict,
                             bt[:, None] * np.exp(np.where(lower_strict, diff, -np.inf)) * (K @ K.T),
                             0.0)
                Tm = np.linalg.inv(np.eye(n) + A)
                W = Tm @ ((bt * np.exp(gam))[:, None] * K)
                Ut = Tm @ (bt[:, None] * V)
                U = Ut - W @ S
                Mask = np.exp(np.where(lower_incl, diff, -np.inf))
                out[b, sl, h] = np.exp(gam)[:, None] * (Q @ S) + (Mask * (Q @ K.T)) @ U
                S = np.exp(gam[-1]) * S + (np.exp(gam[-1] - gam)[:, None] * K).T @ U
            S_all[b, h] = S
    return out, S_all


def chunked_bidir(q, k, v, g, beta, state_in=None, chunk=64):
    """Chunked forward scan from state_in plus chunked reverse scan from zero."""
    out_f, S = chunked_fwd(q, k, v, g, beta, state_in, chunk)
    flip = lambda x: np.flip(np.asarray(x), axis=1)  # noqa: E731
    out_r, _ = chunked_fwd(flip(q), flip(k), flip(v), flip(g), flip(beta), None, chunk)
    return out_f + np.flip(out_r, axis=1), S
