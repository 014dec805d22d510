"""Property-based pins of the CPU oracle (no GPU): the fixed-case pins of
test_oracle_pins.py, drawn over random small shapes instead.

Each example draws its sizes (T, Dk, Dv, heads), a sub-chunk length, the
mode, whether a start state is given, and a seed for the values; the
properties are ones the mathematics fixes for every such draw:

- the sub-chunked (WY / UT) forward form reaches the token recurrence;
- reverse mode through that form reaches autograd of the recurrence;
- streaming over arbitrary cut points equals one scan;
- the C oracle and the numpy recurrence agree;
- the library's cache-slot rule keeps every chunk the attention oracle's
  visibility rule shows a query in a slot of its own;
- gate logits up to +-60 give gates in range, and the C oracle's logit mode
  equals the numpy recurrence on numpy's gates;
- the attention oracle's outputs are convex combinations of the visible
  values, unchanged by a common shift of the keys, linear in the values;
- the bidirectional gradients are the forward scan's plus the flipped
  gradients of the flipped scan from zero.
"""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = settings(max_examples=25, deadline=None, derandomize=True)

shapes = st.fixed_dictionaries({
    "T": st.integers(1, 40),
    "Dk": st.integers(1, 7),
    "Dv": st.integers(1, 6),
    "H": st.integers(1, 2),
    "chunk": st.integers(1, 17),
    "bidir": st.booleans(),
    "state": st.booleans(),
    "g_lo": st.sampled_from([-0.05, -1.0, -6.0]),
    "seed": st.integers(0, 2 ** 31 - 1),
})


def draw(p):
    rng = np.random.default_rng(p["seed"])
    B, T, H, Dk, Dv = 1, p["T"], p["H"], p["Dk"], p["Dv"]
    q = rng.standard_normal((B, T, H, Dk))
    k = rng.standard_normal((B, T, H, Dk))
    v = rng.standard_normal((B, T, H, Dv))
    g = rng.uniform(p["g_lo"], 0.0, (B, T, H))
    beta = rng.uniform(0.0, 1.0, (B, T, H))
    s = rng.standard_normal((B, H, Dk, Dv)) if p["state"] else None
    return rng, q, k, v, g, beta, s


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


@SETTINGS
@given(shapes)
def test_chunked_form_reaches_the_recurrence(p):
    _, q, k, v, g, beta, s = draw(p)
    if p["bidir"]:
        want = oracle.recurrence_bidir(q, k, v, g, beta, s)
        got = oracle.numpy_ref.chunked_bidir(q, k, v, g, beta, s, chunk=p["chunk"])
    else:
        want = oracle.recurrence_fwd(q, k, v, g, beta, s)
        got = oracle.numpy_ref.chunked_fwd(q, k, v, g, beta, s, chunk=p["chunk"])
    assert rel(got[0], want[0]) < 1e-10 and rel(got[1], want[1]) < 1e-10


@SETTINGS
@given(shapes)
def test_chunked_reverse_mode_reaches_autograd(p):
    rng, q, k, v, g, beta, s = draw(p)
    do = rng.standard_normal(v.shape)
    dS = rng.standard_normal((1, p["H"], p["Dk"], p["Dv"]))
    want = oracle.backward.grads(q, k, v, g, beta, s, do, dS, bidir=p["bidir"])
    got = oracle.numpy_ref.chunked_backward(q, k, v, g, beta, s, do, dS, bidir=p["bidir"],
                                            chunk=p["chunk"])
    # with Dk = 1 the normalised q, k are +-1 and dq, dk vanish: compare
    # against a floor set by the largest gradient, not each tensor's own
    names = ["dq", "dk", "dv", "dg", "dbeta"] + ([] if s is None else ["dstate_in"])
    scale = max(np.max(np.abs(want[n])) for n in names)
    for name in names:
        np.testing.assert_allclose(got[name], want[name], rtol=1e-9, atol=1e-12 * scale,
                                   err_msg=name)
    if s is None:
        assert got["dstate_in"] is None and want["dstate_in"] is None


@SETTINGS
@given(shapes, st.lists(st.integers(0, 40), max_size=4))
def test_streaming_over_any_cuts_equals_one_scan(p, cuts):
    _, q, k, v, g, beta, s = draw(p)
    T = p["T"]
    out, S = oracle.recurrence_fwd(q, k, v, g, beta, s)
    edges = sorted({0, T, *[c for c in cuts if c <= T]})
    St = s
    for a, b in zip(edges[:-1], edges[1:]):
        o, St = oracle.recurrence_fwd(q[:, a:b], k[:, a:b], v[:, a:b], g[:, a:b], beta[:, a:b], St)
        assert rel(o, out[:, a:b]) < 1e-12 or np.max(np.abs(out[:, a:b])) == 0
    assert rel(St, S) < 1e-12


@SETTINGS
@given(shapes)
def test_c_and_numpy_recurrences_agree(p):
    _, q, k, v, g, beta, s = draw(p)
    q, k, v = (x.astype(np.float32) for x in (q, k, v))
    g, beta = g.astype(np.float32), beta.astype(np.float32)
    if p["bidir"]:
        c = oracle.oracle_bidir(q, k, v, g, beta, s, nthreads=1)
        n = oracle.recurrence_bidir(q, k, v, g, beta, s)
    else:
        c = oracle.oracle_fwd(q, k, v, g, beta, s, nthreads=1)
        n = oracle.recurrence_fwd(q, k, v, g, beta, s)
    assert rel(c[0], n[0]) < 1e-12 and rel(c[1], n[1]) < 1e-12


@SETTINGS
@given(st.integers(0, 6), st.integers(1, 8), st.integers(0, 60))
def test_cache_slots_of_the_visible_chunks_are_distinct(n_sink, window, c):
    """The library's cache-slot rule against the oracle's visibility rule:
    every chunk a query of chunk c sees (its own included) still sits in its
    own slot of the n_sink + window cache when chunk c runs, so no two visible
    chunks share a slot, and each visible chunk's slot is the one it was
    written to."""
    from gated_deltanet_linear_chunked_b200 import _lib
    lib = _lib.load()
    seen = oracle.sink_window_attn.visible_chunks(c, n_sink, window)
    assert len(seen) == min(c + 1, n_sink + window)
    slots = [lib.gdn_sink_window_slot(m, n_sink, window) for m in seen]
    assert all(0 <= x < n_sink + window for x in slots)
    assert len(set(slots)) == len(slots)
    # nothing written after chunk m (up to c) landed in m's slot
    for m, x in zip(seen, slots):
        later = [lib.gdn_sink_window_slot(j, n_sink, window) for j in range(m + 1, c + 1)]
        assert x not in later, (m, later)


@SETTINGS
@given(shapes, st.floats(0.1, 60.0))
def test_gate_logits_stay_in_range_and_transcriptions_agree(p, spread):
    """Gate logits anywhere in [-spread, spread] (up to +-60, far past what a
    bf16 gate layer emits) give g <= 0 and beta in [0, 1] with no NaN or
    overflow, and the C oracle's logit mode equals the numpy recurrence fed
    numpy's gates."""
    rng, q, k, v, _, _, s = draw(p)
    shape = q.shape[:3]
    x = rng.uniform(-spread, spread, shape).astype(np.float32)
    y = rng.uniform(-spread, spread, shape).astype(np.float32)
    g, beta = oracle.gates_from_logits(x, y)
    assert np.all(np.isfinite(g)) and np.all(g <= 0.0)
    assert np.all((beta >= 0.0) & (beta <= 1.0))
    q, k, v = (t.astype(np.float32) for t in (q, k, v))
    if p["bidir"]:
        c = oracle.oracle_bidir_logits(q, k, v, x, y, s, nthreads=1)
        n = oracle.recurrence_bidir(q, k, v, g, beta, s)
    else:
        c = oracle.oracle_fwd_logits(q, k, v, x, y, s, nthreads=1)
        n = oracle.recurrence_fwd(q, k, v, g, beta, s)
    assert np.all(np.isfinite(c[0])) and np.all(np.isfinite(c[1]))
    assert rel(c[0], n[0]) < 1e-11 and rel(c[1], n[1]) < 1e-11


attn = st.fixed_dictionaries({
    "chunk": st.integers(1, 6),
    "chunks": st.integers(1, 5),
    "d": st.integers(1, 8),
    "dv": st.integers(1, 5),
    "n_sink": st.integers(0, 2),
    "window": st.integers(1, 3),
    "scale": st.sampled_from([0.1, 1.0, 4.0]),
    "seed": st.integers(0, 2 ** 31 - 1),
})


@SETTINGS
@given(attn)
def test_attention_is_a_convex_combination_invariant_to_a_key_shift(p):
    """Softmax attention over the visible chunks: every output row lies in
    the per-coordinate range of the values it can see; adding one vector to
    every key moves each query's scores by a constant and leaves the output
    alone; scaling the values scales the output."""
    rng = np.random.default_rng(p["seed"])
    T = p["chunk"] * p["chunks"]
    q = p["scale"] * rng.standard_normal((1, T, 1, p["d"]))
    k = rng.standard_normal((1, T, 1, p["d"]))
    v = rng.standard_normal((1, T, 1, p["dv"]))
    args = (p["chunk"], p["n_sink"], p["window"])
    out = oracle.sink_window_attn.stream_outputs(q, k, v, *args)
    for c in range(p["chunks"]):
        rows = np.concatenate([np.arange(m * p["chunk"], (m + 1) * p["chunk"])
                               for m in oracle.sink_window_attn.visible_chunks(c, p["n_sink"],
                                                                                p["window"])])
        lo, hi = v[0, rows, 0].min(axis=0), v[0, rows, 0].max(axis=0)
        o = out[0, c * p["chunk"]:(c + 1) * p["chunk"], 0]
        assert np.all(o >= lo - 1e-12) and np.all(o <= hi + 1e-12)
    shift = rng.standard_normal(p["d"])
    out2 = oracle.sink_window_attn.stream_outputs(q, k + shift, v, *args)
    np.testing.assert_allclose(out2, out, rtol=1e-9, atol=1e-12)
    out3 = oracle.sink_window_attn.stream_outputs(q, k, -2.5 * v, *args)
    np.testing.assert_allclose(out3, -2.5 * out, rtol=1e-12, atol=1e-12)


@SETTINGS
@given(shapes)
def test_bidirectional_gradients_are_the_two_scans_gradients(p):
    """Bidirectional mode is the forward scan plus the forward scan of the
    flipped chunk from zero, so its gradients are the forward scan's plus the
    flipped gradients of the flipped scan (which has no state gradient)."""
    rng, q, k, v, g, beta, s = draw(p)
    do = rng.standard_normal(v.shape)
    dS = rng.standard_normal((1, p["H"], p["Dk"], p["Dv"]))
    both = oracle.backward.grads(q, k, v, g, beta, s, do, dS, bidir=True)
    fwd = oracle.backward.grads(q, k, v, g, beta, s, do, dS, bidir=False)
    f = lambda x: np.flip(x, axis=1).copy()  # noqa: E731
    rev = oracle.backward.grads(f(q), f(k), f(v), f(g), f(beta), None, f(do), None, bidir=False)
    names = ["dq", "dk", "dv", "dg", "dbeta"]
    scale = max(np.max(np.abs(both[n])) for n in names)
    for n in names:
        np.testing.assert_allclose(both[n], fwd[n] + f(rev[n]), rtol=1e-10, atol=1e-13 * scale,
                                   err_msg=n)
    if s is not None:
        np.testing.assert_allclose(both["dstate_in"], fwd["dstate_in"], rtol=1e-12, atol=1e-14)
