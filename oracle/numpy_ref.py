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

``chunked_backward``
    Reverse mode through that sub-chunked form (the derivation is in its
    docstring): the gradients the pages' bidirectional short training needs
    (same page, 方法步骤详情, second step), computed the way the chunked
    backward kernels do, in fp64.  Pinned by brute force against autograd of
    the recurrence (``oracle.backward``); it is not itself a reference.
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


def _normalise_vjp(x, dxh):
    """Gradient through x^ = x / sqrt(max(|x|^2, 1e-12)) on the last axis:
    (dx^ - x^ (x^ . dx^)) / |x|, or dx^ / 1e-6 where the clamp holds."""
    ss = np.sum(x * x, axis=-1, keepdims=True)
    n = np.sqrt(np.maximum(ss, 1e-12))
    xh = x / n
    proj = np.where(ss > 1e-12, np.sum(xh * dxh, axis=-1, keepdims=True), 0.0)
    return (dxh - xh * proj) / n


def _chunked_reverse_one(q, k, v, g, beta, S_init, d_out, dS_end, chunk):
    """One (batch, head, direction) in scan order: q, k [T,Dk], v, d_out
    [T,Dv], g, beta [T], S_init, dS_end [Dk,Dv].  Returns the gradients with
    respect to q^, k^ (before the normalisation), v, g, beta and S_init."""
    T = q.shape[0]
    Qh, Kh = _normalise(q), _normalise(k)
    fwd = []
    S = S_init.copy()
    for c0 in range(0, T, chunk):
        sl = slice(c0, min(c0 + chunk, T))
        Q, K, V, bt = Qh[sl], Kh[sl], v[sl], beta[sl]
        gam = np.cumsum(g[sl])
        n = gam.shape[0]
        diff = gam[:, None] - gam[None, :]
        strict = np.tril(np.ones((n, n), dtype=bool), -1)
        incl = np.tril(np.ones((n, n), dtype=bool), 0)
        E = np.exp(np.where(strict, diff, -np.inf))
        G = K @ K.T
        A = bt[:, None] * E * G
        Tm = np.linalg.inv(np.eye(n) + A)
        W = Tm @ ((bt * np.exp(gam))[:, None] * K)
        Ut = Tm @ (bt[:, None] * V)
        U = Ut - W @ S
        M = np.exp(np.where(incl, diff, -np.inf))
        Kt = np.exp(gam[-1] - gam)[:, None] * K
        fwd.append(dict(sl=sl, Q=Q, K=K, V=V, bt=bt, gam=gam, strict=strict, E=E, G=G, A=A,
                        Tm=Tm, W=W, Ut=Ut, U=U, M=M, P=M * (Q @ K.T), Kt=Kt, S0=S))
        S = np.exp(gam[-1]) * S + Kt.T @ U
    dqh, dkh = np.zeros_like(Qh), np.zeros_like(Kh)
    dv, dg, dbeta = np.zeros_like(v), np.zeros(T), np.zeros(T)
    dSe = dS_end.copy()
    for c in reversed(fwd):
        sl, Q, K, V, bt, gam = c["sl"], c["Q"], c["K"], c["V"], c["bt"], c["gam"]
        W, Ut, U, P, Kt, S0, Tm = c["W"], c["Ut"], c["U"], c["P"], c["Kt"], c["S0"], c["Tm"]
        dO = d_out[sl]
        e, eC = np.exp(gam), np.exp(gam[-1])
        # O = diag(e^g) Q^ S0 + P U  and  S_e = e^{g_C} S0 + K~^T U
        dU = P.T @ dO + Kt @ dSe
        dP = dO @ U.T
        dQK = c["M"] * dP
        dQ = dQK @ K + e[:, None] * (dO @ S0.T)
        dK = dQK.T @ Q
        dKt = U @ dSe.T
        dK += np.exp(gam[-1] - gam)[:, None] * dKt
        # U = U~ - W S0
        dS0 = eC * dSe + Q.T @ (e[:, None] * dO) - W.T @ dU
        dW = -dU @ S0.T
        # W = T diag(beta e^g) K^ and U~ = T diag(beta) V, T = (I + A)^-1:
        # the transposed solve, then dA = -T^T dT T^T = -(X_w W^T + X_u U~^T)
        Xw, Xu = Tm.T @ dW, Tm.T @ dU
        dK += (bt * e)[:, None] * Xw
        dv[sl] = bt[:, None] * Xu
        xk = np.sum(Xw * K, axis=1)
        dbt = e * xk + np.sum(Xu * V, axis=1)
        dgam = bt * e * xk
        dA = np.where(c["strict"], -(Xw @ W.T + Xu @ Ut.T), 0.0)
        # A = diag(beta) (E o K^ K^^T), E_ti = e^{g_t - g_i} below the diagonal
        dG = dA * bt[:, None] * c["E"]
        dK += (dG + dG.T) @ K
        dbt += np.sum(dA * c["E"] * c["G"], axis=1)
        dAA = dA * c["A"]
        dgam += dAA.sum(axis=1) - dAA.sum(axis=0)
        # the decays inside O and S_e
        dgam += np.sum(dO * (e[:, None] * (Q @ S0)), axis=1)
        dPP = dP * P
        dgam += dPP.sum(axis=1) - dPP.sum(axis=0)
        dKK = np.sum(dKt * Kt, axis=1)
        dgam -= dKK
        dgam[-1] += dKK.sum() + eC * np.sum(dSe * S0)
        # gamma_r = sum_{i<=r} g_i: dg is the suffix sum of dgamma
        dg[sl] = np.cumsum(dgam[::-1])[::-1]
        dbeta[sl] = dbt
        dqh[sl], dkh[sl] = dQ, dK
        dSe = dS0
    return dqh, dkh, dv, dg, dbeta, dSe


def chunked_backward(q, k, v, g, beta, state_in, d_out, d_state_out=None, bidir=False,
                     chunk=64):
    """Gradients of <out, d_out> + <state_out, d_state_out> by reverse mode
    through the sub-chunked form above: the derivation the chunked backward
    kernels compute, restated in fp64.  Per sub-chunk, walked in reverse
    scan order with dS_e the gradient reaching its end state:

      dU   = P^T dO + K~ dS_e                      (P = Mask o Q^ K^^T)
      dS0  = e^{gamma_n} dS_e + Q^^T diag(e^gamma) dO - W^T dU   (-> dS_e of
             the sub-chunk before)
      dq^  = (Mask o dO U^T) K^ + diag(e^gamma) dO S0^T
      dk^  = (Mask o dO U^T)^T Q^ + diag(e^{gamma_n - gamma}) U dS_e^T
             + diag(beta e^gamma) X_w + (dG + dG^T) K^
      [X_w | X_u] = T^T [-dU S0^T | dU],  dv = diag(beta) X_u
      dA   = -(X_w W^T + X_u U~^T) below the diagonal,  dG = dA o diag(beta) E
      dbeta, dgamma: row (and column) sums of the terms each factor enters;
      dg   = suffix sum of dgamma over the sub-chunk.

    q, k, v pass through the normalisation's Jacobian at the end; bidir adds
    the reverse scan from zero (no state gradient) on the flipped sequence.
    Returns the dict of ``oracle.backward.grads``."""
    q, k, v, g, beta, d_out = _as64(q, k, v, g, beta, d_out)
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    S_in = np.zeros((B, H, Dk, Dv)) if state_in is None else np.asarray(state_in, np.float64)
    dS_out = (np.zeros((B, H, Dk, Dv)) if d_state_out is None
              else np.asarray(d_state_out, np.float64))
    dqh, dkh = np.zeros_like(q), np.zeros_like(k)
    dv, dg, dbeta = np.zeros_like(v), np.zeros_like(g), np.zeros_like(beta)
    dstate = np.zeros((B, H, Dk, Dv))
    fwd_order, rev_order = np.arange(T), np.arange(T)[::-1]
    for b in range(B):
        for h in range(H):
            runs = [(fwd_order, S_in[b, h], dS_out[b, h])]
            if bidir:
                runs.append((rev_order, np.zeros((Dk, Dv)), np.zeros((Dk, Dv))))
            for r, (idx, S0, dSe) in enumerate(runs):
                res = _chunked_reverse_one(q[b, idx, h], k[b, idx, h], v[b, idx, h],
                                           g[b, idx, h], beta[b, idx, h], S0, d_out[b, idx, h],
                                           dSe, chunk)
                dqh[b, idx, h] += res[0]
                dkh[b, idx, h] += res[1]
                dv[b, idx, h] += res[2]
                dg[b, idx, h] += res[3]
                dbeta[b, idx, h] += res[4]
                if r == 0:
                    dstate[b, h] = res[5]
    return {"dq": _normalise_vjp(q, dqh), "dk": _normalise_vjp(k, dkh), "dv": dv, "dg": dg,
            "dbeta": dbeta, "dstate_in": None if state_in is None else dstate}
