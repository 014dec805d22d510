"""The synthetic input recipe (CPU): shapes, distributions, seeding.

Every parity test and the benchmark draw their inputs from
gated_deltanet_linear_chunked_b200/workloads.py, so these checks tie the
generated data to the workloads they stand for: the 1280x704 streaming chunk
(3 latent frames of 40 x 22 tokens, 20 heads of dim 112), the tiny fp32
scan, the 32 x 15 stack and the stress sweep, with the distributions the
workload descriptions give.
"""
import numpy as np
import pytest

from gated_deltanet_linear_chunked_b200 import workloads as wl


def test_stream_chunk_shape_is_three_latent_frames():
    w = wl.stream_chunk()
    assert (w.B, w.T, w.H, w.Dk, w.Dv) == (1, 3 * 40 * 22, 20, 112, 112)
    assert (w.dtype, w.chunk, w.mode) == ("bf16", 64, "fwd")
    assert w.head_tokens == 2640 * 20
    wb = wl.stream_chunk("bidir")
    assert wb.mode == "bidir" and wb.seed != w.seed


def test_stream_chunk_distributions():
    w = wl.stream_chunk()
    d = wl.make_head(w, 0, 5)
    for n in ("q", "k"):
        nrm = np.linalg.norm(d[n].astype(np.float64), axis=-1)
        assert np.all(np.abs(nrm - 1.0) < 1e-2)          # L2-normalised, then bf16
    v = d["v"].astype(np.float64)
    assert abs(v.mean()) < 0.02 and abs(v.std() - 1.0) < 0.02
    assert d["g"].min() >= -0.5 and d["g"].max() <= 0.0
    assert abs(d["g"].mean() + 0.25) < 0.02                # U[-0.5, 0]
    assert 0.0 < d["beta"].min() and d["beta"].max() < 1.0
    assert abs(d["beta"].mean() - 0.5) < 0.02              # sigmoid(N(0, 1))
    s = wl.make_state(w)
    assert s.shape == (1, 20, 112, 112)
    assert abs(s.std() - 0.02) < 5e-4 and abs(s.mean()) < 5e-4


def test_bf16_inputs_are_exactly_representable():
    d = wl.make_head(wl.stream_chunk(), 0, 0)
    for n in ("q", "k", "v"):
        bits = d[n].view(np.uint32)
        assert np.all((bits & 0xFFFF) == 0)
    # round_bf16 is round-to-nearest-even on the dropped 16 bits
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)], np.float32)
    assert wl.round_bf16(x).tolist() == [1.0, 1.0 + 2.0 ** -6, -1.0]


def test_tiny_workload_recipe():
    w = wl.tiny()
    assert (w.B, w.T, w.H, w.Dk, w.Dv, w.dtype, w.chunk) == (1, 64, 2, 16, 16, "f32", 16)
    assert wl.make_state(w) is None
    d = wl.make_head(w, 0, 1)
    assert d["g"].max() <= 0.0                              # -softplus
    assert np.any((d["q"].view(np.uint32) & 0xFFFF) != 0)    # fp32: not rounded to bf16


def test_heads_are_seeded_independently_and_reproducibly():
    w = wl.stream_chunk()
    a = wl.make_head(w, 0, 3)
    b = wl.make_head(w, 0, 3)
    c = wl.make_head(w, 0, 4)
    for n in ("q", "k", "v", "g", "beta"):
        assert np.array_equal(a[n], b[n])
        assert not np.array_equal(a[n], c[n])


def test_make_inputs_layout_matches_per_head_draws():
    w = wl.Workload("layout", 2, 70, 3, 16, 32, "bf16", 64, "fwd",
                    ("uniform", -0.5, 0.0), ("sigmoid",), ("normal", 0.02), 77)
    x = wl.make_inputs(w)
    assert x["q"].shape == (2, 70, 3, 16) and x["v"].shape == (2, 70, 3, 32)
    assert x["g"].shape == (2, 70, 3) and x["state_in"].shape == (2, 3, 16, 32)
    d = wl.make_head(w, 1, 2)
    sl = wl.slice_head(x, 1, 2)
    assert np.array_equal(sl["q"][0, :, 0], d["q"])
    assert np.array_equal(sl["v"][0, :, 0], d["v"])
    assert np.array_equal(sl["beta"][0, :, 0], d["beta"])
    assert np.array_equal(sl["state_in"][0, 0], x["state_in"][1, 2])


def test_stack_calls_start_from_zero_with_per_layer_seeds():
    seeds = {wl.stack_call(l, c).seed for l in range(15) for c in range(32)}
    assert len(seeds) == 15 * 32
    w = wl.stack_call(4, 7)
    assert w.mode == "bidir" and wl.make_state(w) is None
    assert (w.T, w.H, w.Dk) == (2640, 20, 112)


def test_stress_sweep_covers_the_grid():
    cases = wl.stress_cases()
    assert len(cases) == 24
    grid = {(c.Dk, c.T, c.gate, c.beta[1]) for c in cases}
    assert len(grid) == 24
    assert {c.Dk for c in cases} == {64, 128}
    assert {c.T for c in cases} == {256, 4096, 65536}
    for c in cases:
        assert (c.B, c.H, c.dtype) == (4, 16, "bf16")
        d = wl.make_head(dataclass_replace_T(c, 512), 0, 0)
        lo, hi = c.gate[1], c.gate[2]
        assert d["g"].min() >= lo - 1e-6 and d["g"].max() <= hi
        assert np.all(d["beta"] == np.float32(c.beta[1]))


def dataclass_replace_T(w, T):
    import dataclasses
    return dataclasses.replace(w, T=T)


@pytest.mark.parametrize("mode", ["fwd", "bidir"])
def test_rank_streams_differ(mode):
    # bench.py gives every rank its own seed; different seeds, different data
    a = wl.make_head(wl.stream_chunk(mode, seed=10), 0, 0)
    b = wl.make_head(wl.stream_chunk(mode, seed=11), 0, 0)
    assert not np.array_equal(a["q"], b["q"])


def test_raw_and_mixed_qk_recipes():
    """The un-normalised q/k recipes used to exercise the library's own L2
    normalisation: raw N(0,1) rows (norm about sqrt(d)), and the mixed recipe
    with rows at 1e-3 and 1e3, rows under the 1e-12 clamp and zero rows."""
    import dataclasses
    base = wl.stream_chunk()
    raw = wl.make_head(dataclasses.replace(base, qk=("raw",)), 0, 3)
    for n in ("q", "k"):
        nrm = np.linalg.norm(raw[n].astype(np.float64), axis=-1)
        assert abs(np.median(nrm) - np.sqrt(112)) < 0.5
    w = dataclasses.replace(base, qk=("mixed",))
    d = wl.make_head(w, 0, 3)
    rows = wl.qk_rows(w.T)
    r = np.random.default_rng([w.seed, 0, 3])
    q0 = r.standard_normal((w.T, w.Dk), dtype=np.float32)
    for name, scale in (("small", 1e-3), ("large", 1e3), ("subclamp", 3e-8)):
        t = rows[name]
        assert len(t) > 10
        got = d["q"][t].astype(np.float64)
        want = wl.round_bf16(q0[t] * np.float32(scale)).astype(np.float64)
        assert np.array_equal(got, want), name
    sq = np.sum(d["q"][rows["subclamp"]].astype(np.float64) ** 2, axis=-1)
    assert np.all(sq < 1e-12) and np.all(sq > 0)
    assert not d["q"][rows["zero_q"]].any() and d["q"][rows["zero_k"]].any()
    assert not d["k"][rows["zero_k"]].any() and d["k"][rows["zero_q"]].any()
    # the special row sets are disjoint from one another
    sets = [set(rows[n].tolist()) for n in ("small", "large", "subclamp")]
    assert not (sets[0] & sets[1]) and not (sets[0] & sets[2]) and not (sets[1] & sets[2])


def test_logit_recipe_has_the_stated_gate_distributions():
    """The fused-prologue workload passes the gate layer's logits: decay and
    write-strength logits ~ N(0,1), bf16-exact, so that -softplus and sigmoid
    of them have the tiny workload's stated gate distributions; q, k, v are
    drawn exactly as in the streaming chunk."""
    w = wl.stream_chunk_logits()
    d = wl.make_head(w, 0, 4)
    assert set(d) == {"q", "k", "v", "g_logit", "beta_logit"}
    for n in ("g_logit", "beta_logit"):
        x = d[n].astype(np.float64)
        assert abs(x.mean()) < 0.05 and abs(x.std() - 1.0) < 0.05
        assert np.array_equal(d[n], wl.round_bf16(d[n]))
    plain = wl.make_head(wl.stream_chunk(), 0, 4)
    for n in ("q", "k", "v"):
        assert np.array_equal(d[n], plain[n])
    x = wl.make_inputs(wl.Workload("lg", 2, 33, 3, 16, 16, "f32", 16, "fwd", ("logit_normal",),
                                   ("logit_normal",), ("zero",), 3))
    assert x["g_logit"].shape == (2, 33, 3) and "g" not in x


def test_attention_stream_recipe():
    """The softmax blocks' stream: the GDN blocks' head layout, one sink
    chunk and a window of two (7920 keys from chunk 2 on), bf16 values with
    the stated distributions, each chunk seeded on its own."""
    w = wl.sink_window_stream()
    assert (w.B, w.Tc, w.H, w.D, w.n_sink, w.window) == (1, 2640, 20, 112, 1, 2)
    assert w.steady_chunk == 2 and (w.n_sink + w.window) * w.Tc == 7920
    small = wl.AttnStream("t", 1, 300, 2, 64, 1, 2, 3, 7)
    a0, a1 = wl.attn_chunk(small, 0), wl.attn_chunk(small, 1)
    for n in ("q", "k", "v"):
        assert a0[n].shape == (1, 300, 2, 64)
        assert np.all((a0[n].view(np.uint32) & 0xFFFF) == 0)          # bf16 values
        x = a0[n].astype(np.float64)
        assert abs(x.mean()) < 0.02 and abs(x.std() - 1.0) < 0.02      # N(0, 1)
        assert not np.array_equal(a0[n], a1[n])                        # per-chunk seeds
        assert np.array_equal(a0[n], wl.attn_chunk(small, 0)[n])       # reproducible
    sharp = wl.AttnStream("t", 1, 300, 2, 64, 1, 2, 3, 7, q_scale=6.0)
    qs = wl.attn_chunk(sharp, 0)["q"].astype(np.float64)
    assert abs(qs.std() - 6.0) < 0.1                                   # N(0, q_scale^2)
    np.testing.assert_array_equal(wl.attn_chunk(sharp, 0)["k"], a0["k"])  # k, v unscaled
