"""Pins of the sink + sliding-window attention oracle (CPU only).

Each pin checks the oracle against something other than itself, so that a
plausible slip -- an off-by-one in the window, a sink that is not kept, a
missing 1/sqrt(d), a softmax over the wrong axis, rows taken from the wrong
chunk -- fails at least one of them:

* the hand-derived example in ``tests/golden/sink_window_hand_d2.txt``;
* the visible chunk sets of a few (c, n_sink, window), written out by hand;
* q = 0 gives uniform weights, so the output is the plain mean of the visible
  values (closed form);
* values and keys of a chunk that has left the window do not matter, those of
  a visible chunk do; permuting the tokens of a visible past chunk (keys and
  values alike) does not matter;
* a key scaled far along q takes all the weight;
* two special cases reduce to PyTorch's own attention in float64: no sink and
  a window as long as the stream (block-causal over chunks), and no sink with
  a one-chunk window (each chunk on its own).
"""
import os

import numpy as np
import pytest
import torch

from oracle import sink_window_attn as swa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "sink_window_hand_d2.txt")


def _golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, rhs = (s.strip() for s in line.split("=", 1))
        vals[key] = rhs
    rows = lambda s: np.array([[float(x) for x in r.split()] for r in s.split(";")])  # noqa: E731
    return (int(vals["chunk"]), int(vals["n_sink"]), int(vals["window"]), rows(vals["q"]),
            rows(vals["k"]), rows(vals["v"]), rows(vals["out"]))


def _stream(rng, B, C, chunk, H, d):
    shape = (B, C * chunk, H, d)
    return rng.standard_normal(shape), rng.standard_normal(shape), rng.standard_normal(shape)


def test_hand_example():
    chunk, n_sink, window, q, k, v, out = _golden()
    as4 = lambda a: a[None, :, None, :]  # noqa: E731   [T, d] -> [1, T, 1, d]
    got = swa.stream_outputs(as4(q), as4(k), as4(v), chunk, n_sink, window)[0, :, 0, :]
    np.testing.assert_allclose(got, out, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("c,n_sink,window,expect", [
    (0, 1, 2, [0]),
    (1, 1, 2, [0, 1]),
    (5, 1, 2, [0, 4, 5]),
    (6, 2, 3, [0, 1, 4, 5, 6]),
    (3, 0, 1, [3]),
    (1, 2, 1, [0, 1]),
    (4, 0, 10, [0, 1, 2, 3, 4]),
    (4, 3, 1, [0, 1, 2, 4]),
])
def test_visible_sets_by_hand(c, n_sink, window, expect):
    assert swa.visible_chunks(c, n_sink, window) == expect


def test_zero_query_is_the_mean_of_the_visible_values():
    rng = np.random.default_rng(11)
    B, C, chunk, H, d = 2, 6, 5, 3, 8
    q, k, v = _stream(rng, B, C, chunk, H, d)
    q[:] = 0.0
    out = swa.stream_outputs(q, k, v, chunk, n_sink=1, window=2)
    sets = {0: [0], 1: [0, 1], 2: [0, 1, 2], 3: [0, 2, 3], 4: [0, 3, 4], 5: [0, 4, 5]}
    for c, ms in sets.items():
        mean = np.mean(np.concatenate([v[:, m * chunk:(m + 1) * chunk] for m in ms], axis=1), axis=1)
        for t in range(chunk):
            np.testing.assert_allclose(out[:, c * chunk + t], mean, rtol=1e-12, atol=1e-12)


def test_evicted_chunks_do_not_matter_and_visible_ones_do():
    rng = np.random.default_rng(12)
    B, C, chunk, H, d = 1, 5, 4, 2, 8
    q, k, v = _stream(rng, B, C, chunk, H, d)
    base = swa.chunk_output(q[:, 4 * chunk:], k, v, 4, chunk, n_sink=1, window=2)  # sees 0, 3, 4
    for m in (1, 2):                    # left the window
        k2, v2 = k.copy(), v.copy()
        k2[:, m * chunk:(m + 1) * chunk] += 3.0
        v2[:, m * chunk:(m + 1) * chunk] -= 7.0
        np.testing.assert_array_equal(swa.chunk_output(q[:, 4 * chunk:], k2, v2, 4, chunk, 1, 2), base)
    for m in (0, 3, 4):                 # sink, window, own chunk
        v2 = v.copy()
        v2[:, m * chunk:(m + 1) * chunk] += 1.0
        assert np.abs(swa.chunk_output(q[:, 4 * chunk:], k, v2, 4, chunk, 1, 2) - base).max() > 1e-3


def test_permuting_a_visible_past_chunk_does_not_matter():
    rng = np.random.default_rng(13)
    B, C, chunk, H, d = 1, 4, 6, 2, 8
    q, k, v = _stream(rng, B, C, chunk, H, d)
    base = swa.chunk_output(q[:, 3 * chunk:], k, v, 3, chunk, n_sink=1, window=3)
    perm = rng.permutation(chunk)
    k2, v2 = k.copy(), v.copy()
    k2[:, 2 * chunk:3 * chunk] = k[:, 2 * chunk + perm]
    v2[:, 2 * chunk:3 * chunk] = v[:, 2 * chunk + perm]
    np.testing.assert_allclose(swa.chunk_output(q[:, 3 * chunk:], k2, v2, 3, chunk, 1, 3), base,
                               rtol=1e-12, atol=1e-12)


def test_dominant_key_takes_all_the_weight():
    rng = np.random.default_rng(14)
    n, L, d = 3, 9, 8
    q = rng.standard_normal((n, d))
    k = rng.standard_normal((L, d))
    v = rng.standard_normal((L, d))
    k[5] = 200.0 * q[0] / np.linalg.norm(q[0])     # score ~ 200 |q0| / sqrt(8) for row 0
    out = swa.attend(q, k, v)
    np.testing.assert_allclose(out[0], v[5], rtol=0, atol=1e-9)


def _sdpa(q, k, v, mask):
    # torch's attention: [B, H, T, d] layout; boolean mask True = attend
    t = lambda a: torch.tensor(a, dtype=torch.float64).permute(0, 2, 1, 3)  # noqa: E731
    o = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=mask)
    return o.permute(0, 2, 1, 3).numpy()


def test_block_causal_special_case_matches_torch():
    rng = np.random.default_rng(15)
    B, C, chunk, H, d = 2, 4, 5, 3, 16
    q, k, v = _stream(rng, B, C, chunk, H, d)
    idx = np.arange(C * chunk) // chunk
    mask = torch.tensor(idx[:, None] >= idx[None, :])
    np.testing.assert_allclose(swa.stream_outputs(q, k, v, chunk, n_sink=0, window=C),
                               _sdpa(q, k, v, mask), rtol=1e-12, atol=1e-12)


def test_one_chunk_window_matches_torch_per_chunk():
    rng = np.random.default_rng(16)
    B, C, chunk, H, d = 1, 3, 7, 2, 16
    q, k, v = _stream(rng, B, C, chunk, H, d)
    out = swa.stream_outputs(q, k, v, chunk, n_sink=0, window=1)
    for c in range(C):
        s = slice(c * chunk, (c + 1) * chunk)
        np.testing.assert_allclose(out[:, s], _sdpa(q[:, s], k[:, s], v[:, s], None),
                                   rtol=1e-12, atol=1e-12)
