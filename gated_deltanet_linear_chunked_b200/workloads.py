"""Seeded synthetic workloads for the GDN scan (numpy only).

This module only draws random inputs; it holds none of the scan's arithmetic
and imports nothing from the library or from the oracle, so tests, the
benchmark and the oracle can all take their inputs from it.

Shapes follow the pages' streaming workload: 1280x704 frames under a 32x
spatial latent give 40 x 22 = 880 tokens per latent frame (DCAE-V, F32T4C32:
SANA-Video blog "SANA-Video视频生成领域的效率革命", 3.2 多分辨率VAE设计), and a
streaming chunk is three
latent frames ("SANA-Streaming：基于混合扩散Transformer的实时流式视频编辑系统",
方法步骤详情, second step), i.e. 2640 tokens; the DiT has 15 GDN blocks
(same page, 核心方法).  Heads are 112 wide (SANA-Video-2B, same blog,
3.1 模型架构配置); 20 heads is the workload's stated head count.

Every (batch, head) pair draws from its own generator, seeded with
``[seed, b, h]``, in the fixed order q, k, v, gate, beta, so any single head
can be regenerated without drawing the rest.  Values are drawn in fp32 and,
for bf16 workloads, rounded to the nearest bf16 (ties to even) so that the
fp32 arrays returned hold exactly the values a bf16 tensor stores.
"""
from __future__ import annotations

import dataclasses
from typing import Iterator

import numpy as np

TOKENS_PER_LATENT_FRAME = 40 * 22  # 1280/32 x 704/32
FRAMES_PER_CHUNK = 3
CHUNK_TOKENS = FRAMES_PER_CHUNK * TOKENS_PER_LATENT_FRAME  # 2640
GDN_LAYERS = 15


@dataclasses.dataclass(frozen=True)
class Workload:
    """One scan call's shape and input distributions."""
    name: str
    B: int
    T: int
    H: int
    Dk: int
    Dv: int
    dtype: str            # "f32" or "bf16": dtype of q, k, v and out
    chunk: int            # sub-chunk length handed to the library
    mode: str             # "fwd" or "bidir"
    gate: tuple           # ("neg_softplus",), ("uniform", lo, hi): g = log decay;
                          # ("logit_normal",): the gate layer's decay logit ~ N(0,1)
    beta: tuple           # ("sigmoid",), ("const", value); ("logit_normal",): logit ~ N(0,1)
    state: tuple          # ("zero",) or ("normal", std)
    seed: int
    qk: tuple = ("unit",)  # ("unit",): rows L2-normalised; ("raw",): N(0,1) rows;
                           # ("mixed",): N(0,1) rows with special rows (see qk_rows)

    @property
    def head_tokens(self) -> int:
        return self.B * self.H * self.T


def tiny() -> Workload:
    """Tiny causal scan, fp32: B1 H2 d16 T64, sub-chunk 16, zero state."""
    return Workload("tiny_causal_f32", 1, 64, 2, 16, 16, "f32", 16, "fwd",
                    ("neg_softplus",), ("sigmoid",), ("zero",), 1)


def stream_chunk(mode: str = "fwd", seed: int | None = None) -> Workload:
    """One 1280x704 streaming chunk: B1 H20 d112 T2640 bf16, sub-chunk 64,
    g ~ U[-0.5, 0], beta = sigmoid(N(0,1)), state_in ~ N(0, 0.02^2)."""
    if seed is None:
        seed = 2 if mode == "fwd" else 3
    name = "stream_chunk_causal" if mode == "fwd" else "stream_chunk_bidir"
    return Workload(name, 1, CHUNK_TOKENS, 20, 112, 112, "bf16", 64, mode,
                    ("uniform", -0.5, 0.0), ("sigmoid",), ("normal", 0.02), seed)


def stream_chunk_logits(mode: str = "fwd", seed: int | None = None) -> Workload:
    """The streaming chunk with the gate layer's logits as inputs (fused
    prologue): decay and write-strength logits ~ N(0,1) rounded to bf16, so
    g = -softplus(logit) and beta = sigmoid(logit) have the tiny workload's
    stated gate distributions."""
    w = stream_chunk(mode, seed)
    return dataclasses.replace(w, name=w.name + "_logits", gate=("logit_normal",),
                               beta=("logit_normal",))


def stack_call(layer: int, chunk_index: int, mode: str = "bidir") -> Workload:
    """Chunk `chunk_index` of GDN layer `layer` in the 32-chunk x 15-layer
    stream; the state is carried per layer (zero before chunk 0)."""
    w = stream_chunk(mode, seed=1000 + 37 * layer + chunk_index)
    return dataclasses.replace(w, name=f"stack_l{layer}_c{chunk_index}", state=("zero",))


STRESS_DIMS = (64, 128)
STRESS_LENGTHS = (256, 4096, 65536)
STRESS_GATES = (("uniform", -1e-4, 0.0), ("uniform", -8.0, -4.0))
STRESS_BETAS = (0.01, 0.99)


def stress_cases() -> list[Workload]:
    """24 stress cases: B4 H16, d in {64,128}, T in {256,4096,65536}, bf16,
    near-identity (g in [-1e-4,0]) or fast (g in [-8,-4]) decay, constant
    beta in {0.01, 0.99}, state_in ~ N(0, 0.02^2)."""
    cases = []
    i = 0
    for d in STRESS_DIMS:
        for T in STRESS_LENGTHS:
            for gate in STRESS_GATES:
                for b in STRESS_BETAS:
                    tag = "slow" if gate[1] > -1.0 else "fast"
                    cases.append(Workload(f"stress_d{d}_T{T}_{tag}_b{b}", 4, T, 16, d, d,
                                          "bf16", 64, "fwd", gate, ("const", b),
                                          ("normal", 0.02), 5000 + i))
                    i += 1
    return cases


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32."""
    u = np.array(x, dtype=np.float32, copy=True).view(np.uint32)
    lsb = (u >> 16) & 1
    u += np.uint32(0x7FFF)          # finite inputs: no wrap-around
    u += lsb
    u &= np.uint32(0xFFFF0000)
    return u.view(np.float32)


def _l2_rows(x: np.ndarray) -> np.ndarray:
    # Part of the input recipe ("q, k ~ N(0,1), then L2-normalised"); the
    # library normalises again itself, so this only shapes the stored values.
    return (x / np.linalg.norm(x, axis=-1, keepdims=True)).astype(np.float32)


# Row scales of the ("mixed",) q/k recipe, which exercises the library's own
# L2 normalisation: rows at tiny and huge magnitudes, rows whose squared norm
# falls under the 1e-12 clamp, and all-zero rows.
MIXED_SMALL, MIXED_LARGE, MIXED_SUBCLAMP = 1e-3, 1e3, 3e-8


def qk_rows(T: int) -> dict:
    """Token indices of the special rows of the ("mixed",) recipe, the same
    for every head: q/k rows scaled by 1e-3 and 1e3, rows scaled by 3e-8
    (squared norm about 1e-13, under the clamp), one all-zero q row and one
    all-zero k row."""
    t = np.arange(T)
    return {"small": t[t % 7 == 3], "large": t[(t % 11 == 5) & (t % 7 != 3)],
            "subclamp": t[(t % 13 == 8) & (t % 7 != 3) & (t % 11 != 5)],
            "zero_q": np.array([T // 2]) if T >= 2 else np.array([], int),
            "zero_k": np.array([T // 3]) if T >= 3 else np.array([], int)}


def _shape_qk(x: np.ndarray, recipe: tuple, is_q: bool) -> np.ndarray:
    if recipe[0] == "unit":
        return _l2_rows(x)
    if recipe[0] == "raw":
        return x
    if recipe[0] == "mixed":
        rows = qk_rows(x.shape[0])
        x = x.copy()
        x[rows["small"]] *= np.float32(MIXED_SMALL)
        x[rows["large"]] *= np.float32(MIXED_LARGE)
        x[rows["subclamp"]] *= np.float32(MIXED_SUBCLAMP)
        x[rows["zero_q" if is_q else "zero_k"]] = 0.0
        return x
    raise ValueError(recipe)


def make_head(w: Workload, b: int, h: int) -> dict:
    """Inputs of one (batch, head) pair: q, k [T,Dk]; v [T,Dv]; g, beta [T]."""
    rng = np.random.default_rng([w.seed, b, h])
    q = _shape_qk(rng.standard_normal((w.T, w.Dk), dtype=np.float32), w.qk, True)
    k = _shape_qk(rng.standard_normal((w.T, w.Dk), dtype=np.float32), w.qk, False)
    v = rng.standard_normal((w.T, w.Dv), dtype=np.float32)
    if w.gate[0] == "logit_normal":
        # the gate layer's raw outputs: the library forms g and beta itself
        g_logit = rng.standard_normal(w.T, dtype=np.float32)
        beta_logit = rng.standard_normal(w.T, dtype=np.float32)
        if w.dtype == "bf16":
            q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
            g_logit, beta_logit = round_bf16(g_logit), round_bf16(beta_logit)
        return {"q": q, "k": k, "v": v, "g_logit": g_logit, "beta_logit": beta_logit}
    if w.gate[0] == "neg_softplus":
        z = rng.standard_normal(w.T, dtype=np.float32).astype(np.float64)
        g = -np.logaddexp(0.0, z)
    elif w.gate[0] == "uniform":
        lo, hi = w.gate[1], w.gate[2]
        g = lo + (hi - lo) * rng.random(w.T, dtype=np.float64)
    else:
        raise ValueError(w.gate)
    g = np.minimum(g.astype(np.float32), np.float32(0.0))
    if w.beta[0] == "sigmoid":
        z = rng.standard_normal(w.T, dtype=np.float32).astype(np.float64)
        beta = (1.0 / (1.0 + np.exp(-z))).astype(np.float32)
    elif w.beta[0] == "const":
        beta = np.full(w.T, w.beta[1], dtype=np.float32)
    else:
        raise ValueError(w.beta)
    if w.dtype == "bf16":
        q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
    return {"q": q, "k": k, "v": v, "g": g, "beta": beta}


def make_state(w: Workload) -> np.ndarray | None:
    """state_in [B,H,Dk,Dv] fp32, or None for a zero state."""
    if w.state[0] == "zero":
        return None
    rng = np.random.default_rng([w.seed, 0x57A7E])
    return (w.state[1] * rng.standard_normal((w.B, w.H, w.Dk, w.Dv))).astype(np.float32)


def iter_heads(w: Workload) -> Iterator[tuple[int, int, dict]]:
    for b in range(w.B):
        for h in range(w.H):
            yield b, h, make_head(w, b, h)


def make_inputs(w: Workload) -> dict:
    """All inputs in the library's layouts, fp32 numpy (bf16-exact for bf16
    workloads): q, k [B,T,H,Dk]; v [B,T,H,Dv]; g, beta [B,T,H]; state_in."""
    q = np.empty((w.B, w.T, w.H, w.Dk), np.float32)
    k = np.empty_like(q)
    v = np.empty((w.B, w.T, w.H, w.Dv), np.float32)
    gates = ("g_logit", "beta_logit") if w.gate[0] == "logit_normal" else ("g", "beta")
    ga = {n: np.empty((w.B, w.T, w.H), np.float32) for n in gates}
    for b, h, d in iter_heads(w):
        q[b, :, h], k[b, :, h], v[b, :, h] = d["q"], d["k"], d["v"]
        for n in gates:
            ga[n][b, :, h] = d[n]
    return {"q": q, "k": k, "v": v, **ga, "state_in": make_state(w)}


def slice_head(inputs: dict, b: int, h: int) -> dict:
    """One head of `make_inputs` output, shaped [1,T,1,D] for a B=H=1 call."""
    out = {n: np.ascontiguousarray(inputs[n][b:b + 1, :, h:h + 1]) for n in ("q", "k", "v", "g", "beta")}
    s = inputs.get("state_in")
    out["state_in"] = None if s is None else np.ascontiguousarray(s[b:b + 1, h:h + 1])
    return out


# --------------------------------------------------------------------------
# The softmax blocks' sink + sliding-window attention


@dataclasses.dataclass(frozen=True)
class AttnStream:
    """A stream of chunks through one softmax block: per chunk q, k, v
    [B, Tc, H, D] bf16, drawn N(0, 1) (k, v) and N(0, q_scale^2) (q), rounded
    to bf16; the block keeps ``n_sink`` sink chunks and a ``window`` of chunks
    (its own included)."""
    name: str
    B: int
    Tc: int
    H: int
    D: int
    n_sink: int
    window: int
    chunks: int           # chunks 0 .. chunks-1 of the stream
    seed: int
    q_scale: float = 1.0  # > 1 sharpens the softmax (scores ~ N(0, q_scale^2))

    @property
    def steady_chunk(self) -> int:
        """The first chunk whose query sees the full key set (sink + window)."""
        return self.n_sink + self.window - 1


def sink_window_stream(seed: int = 5, chunks: int = 4) -> AttnStream:
    """The streaming chunk through a softmax block: B1 H20 D112 Tc2640 (the
    GDN blocks' head layout), one sink chunk and a window of two chunks, so
    from chunk 2 on a query sees 3 x 2640 = 7920 keys."""
    return AttnStream("sink_window_chunk", 1, CHUNK_TOKENS, 20, 112, 1, 2, chunks, seed)


def attn_chunk(w: AttnStream, c: int) -> dict:
    """q, k, v of stream chunk c (fp32 arrays holding bf16 values), drawn from
    the generator seeded with [seed, c] in the order q, k, v."""
    rng = np.random.default_rng([w.seed, c])
    shape = (w.B, w.Tc, w.H, w.D)
    q = rng.standard_normal(shape, dtype=np.float32) * np.float32(w.q_scale)
    k = rng.standard_normal(shape, dtype=np.float32)
    v = rng.standard_normal(shape, dtype=np.float32)
    return {"q": round_bf16(q), "k": round_bf16(k), "v": round_bf16(v)}
