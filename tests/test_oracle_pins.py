"""Pins for the CPU oracle (no GPU).

The pages print no numeric example of the scan, so the oracle is pinned to
things other than itself: a hand-derived example, closed forms for special
gates, invariants of the delta rule, and brute force (the chunked WY form, an
independent algorithm, must reach the token recurrence).  Each pin is chosen
so that a plausible slip in the oracle (a dropped term, a wrong sign, the
decay on the wrong factor, a transposed state, the projection on the wrong
side, a missing normalisation) fails at least one of them.

Both transcriptions of the definition are pinned: the C oracle (double and
long double) and the numpy recurrence.
"""
import os

import numpy as np
import pytest

import oracle
from gated_deltanet_linear_chunked_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def c_fwd(q, k, v, g, beta, s=None):
    return oracle.oracle_fwd(q, k, v, g, beta, s, nthreads=2)


def c_bidir(q, k, v, g, beta, s=None):
    return oracle.oracle_bidir(q, k, v, g, beta, s, nthreads=2)


FWD = {"c": c_fwd, "numpy": oracle.recurrence_fwd}
BIDIR = {"c": c_bidir, "numpy": oracle.recurrence_bidir}


def rand_inputs(rng, B=2, T=23, H=3, Dk=8, Dv=6, g_lo=-1.0, unit=False):
    q = rng.standard_normal((B, T, H, Dk)).astype(np.float32)
    k = rng.standard_normal((B, T, H, Dk)).astype(np.float32)
    if unit:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, Dv)).astype(np.float32)
    g = rng.uniform(g_lo, 0.0, (B, T, H)).astype(np.float32)
    beta = rng.uniform(0.0, 1.0, (B, T, H)).astype(np.float32)
    s = (0.3 * rng.standard_normal((B, H, Dk, Dv))).astype(np.float64)
    return q, k, v, g, beta, s


def unit(x):
    x = np.asarray(x, np.float64)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def rel(a, b):
    return np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))) / max(
        np.max(np.abs(np.asarray(b, np.float64))), 1e-300)


def load_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rhs = line.split("=", 1)
            rows = [[float(x) for x in r.split()] for r in rhs.split(";")]
            vals[key.strip()] = np.array(rows)
    return vals


# --------------------------------------------------------------- hand example
@pytest.mark.parametrize("impl", ["c", "numpy"])
def test_hand_derived_example(impl):
    """Pin: the worked example in tests/golden/hand_d2_t2.txt, derived on
    paper from the definition (decay, unit-gate projection, normalisation of
    q and k, reverse scan and the bidirectional sum all exercised)."""
    G = load_golden("hand_d2_t2.txt")
    q = G["q"].reshape(1, 2, 1, 2).astype(np.float32)
    k = G["k"].reshape(1, 2, 1, 2).astype(np.float32)
    v = G["v"].reshape(1, 2, 1, 2).astype(np.float32)
    g = G["g"].reshape(1, 2, 1).astype(np.float32)
    beta = G["beta"].reshape(1, 2, 1).astype(np.float32)
    out, S = FWD[impl](q, k, v, g, beta)
    # g is stored in fp32, so a_1 = exp(fp32(ln 0.5)) differs from 0.5 by ~2e-9
    np.testing.assert_allclose(out[0, :, 0], G["out_fwd"], rtol=0, atol=1e-8)
    np.testing.assert_allclose(S[0, 0], G["state_fwd"], rtol=0, atol=1e-8)
    out_b, S_b = BIDIR[impl](q, k, v, g, beta)
    np.testing.assert_allclose(out_b[0, :, 0], G["out_bidir"], rtol=0, atol=1e-8)
    np.testing.assert_allclose(S_b[0, 0], G["state_fwd"], rtol=0, atol=1e-8)


# ------------------------------------------------------------- closed forms
@pytest.mark.parametrize("impl", ["c", "numpy"])
def test_p1_identity_gate_zero_beta_keeps_state(impl):
    """Pin p1: a = 1, beta = 0 -> S never changes and o_t = S_in^T q^_t."""
    rng = np.random.default_rng(11)
    q, k, v, g, beta, s = rand_inputs(rng)
    g[:] = 0
    beta[:] = 0
    out, S = FWD[impl](q, k, v, g, beta, s)
    np.testing.assert_allclose(S, s, rtol=0, atol=1e-14)
    expect = np.einsum("bthi,bhij->bthj", unit(q), s)
    np.testing.assert_allclose(out, expect, rtol=0, atol=1e-13)


@pytest.mark.parametrize("impl", ["c", "numpy"])
def test_p2_unit_gate_writes_value_exactly(impl):
    """Pin p2: a = 1, beta = 1, orthonormal keys k_t = e_{pi(t)} -> the state
    is S_in with row pi(t) replaced by v_t (the last write wins), so
    S^T e_{pi(t)} = v_t; every output follows from those row replacements."""
    rng = np.random.default_rng(12)
    B, T, H, Dk, Dv = 1, 6, 2, 8, 5
    q, k, v, g, beta, s = rand_inputs(rng, B, T, H, Dk, Dv)
    g[:] = 0
    beta[:] = 1
    perm = [3, 0, 6, 3, 1, 7]           # key 3 written twice
    k[:] = 0
    for t, i in enumerate(perm):
        k[:, t, :, i] = 2.5              # not unit: normalisation must fix it
    out, S = FWD[impl](q, k, v, g, beta, s)
    expect = s.copy()
    for t, i in enumerate(perm):
        expect[:, :, i, :] = v[:, t, :, :]
        np.testing.assert_allclose(out[:, t], np.einsum("bhi,bhij->bhj", unit(q[:, t]), expect),
                                   rtol=0, atol=1e-13)
    np.testing.assert_allclose(S, expect, rtol=0, atol=1e-13)


@pytest.mark.parametrize("impl", ["c", "numpy"])
def test_p2b_general_unit_key_projection(impl):
    """Pin p2 (general key): a = 1, beta = 1 -> after the update S^T k^ = v
    for any key direction, and S is unchanged on the complement of k^."""
    rng = np.random.default_rng(13)
    q, k, v, g, beta, s = rand_inputs(rng, 2, 1, 3, 16, 9)
    g[:] = 0
    beta[:] = 1
    out, S = FWD[impl](q, k, v, g, beta, s)
    kh = unit(k[:, 0])
    np.testing.assert_allclose(np.einsum("bhi,bhij->bhj", kh, S), v[:, 0], rtol=0, atol=1e-13)
    z = unit(rng.standard_normal(kh.shape))
    z = z - np.sum(z * kh, -1, keepdims=True) * kh          # orthogonal to k^
    np.testing.assert_allclose(np.einsum("bhi,bhij->bhj", z, S),
                               np.einsum("bhi,bhij->bhj", z, s), rtol=0, atol=1e-13)


@pytest.mark.parametrize("impl", ["c", "numpy"])
def test_p3_pure_decay(impl):
    """Pin p3: beta = 0 -> S_t = exp(sum_{s<=t} g_s) S_in and
    o_t = exp(sum_{s<=t} g_s) S_in^T q^_t."""
    rng = np.random.default_rng(14)
    q, k, v, g, beta, s = rand_inputs(rng, g_lo=-2.0)
    beta[:] = 0
    out, S = FWD[impl](q, k, v, g, beta, s)
    G = np.cumsum(g.astype(np.float64), axis=1)                 # [B,T,H]
    np.testing.assert_allclose(S, np.exp(G[:, -1])[..., None, None] * s, rtol=1e-13, atol=1e-300)
    expect = np.exp(G)[..., None] * np.einsum("bthi,bhij->bthj", unit(q), s)
    np.testing.assert_allclose(out, expect, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("impl", ["c", "numpy"])
def test_p9_single_token_formula(impl):
    """Pin p9a: T = 1 written out by hand:
    S1 = a S0 - a beta k^ (k^^T S0) + beta k^ v^T,  o = S1^T q^."""
    rng = np.random.default_rng(15)
    q, k, v, g, beta, s = rand_inputs(rng, 2, 1, 3, 12, 7)
    out, S = FWD[impl](q, k, v, g, beta, s)
    a = np.exp(g[:, 0].astype(np.float64))[..., None, None]
    b = beta[:, 0].astype(np.float64)[..., None, None]
    kh, qh = unit(k[:, 0]), unit(q[:, 0])
    kS = np.einsum("bhi,bhij->bhj", kh, s)
    S1 = a * s - a * b * kh[..., :, None] * kS[..., None, :] + b * kh[..., :, None] * v[:, 0][..., None, :]
    np.testing.assert_allclose(S, S1, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(out[:, 0], np.einsum("bhi,bhij->bhj", qh, S1), rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("impl", ["c", "numpy"])
def test_p9_scalar_state(impl):
    """Pin p9b: Dk = Dv = 1 reduces to the scalar recurrence
    s_t = a_t (1 - beta_t) s_{t-1} + beta_t sign(k_t) v_t, o_t = sign(q_t) s_t."""
    rng = np.random.default_rng(16)
    q, k, v, g, beta, s = rand_inputs(rng, 1, 40, 2, 1, 1)
    out, S = FWD[impl](q, k, v, g, beta, s)
    for h in range(2):
        st = s[0, h, 0, 0]
        for t in range(40):
            a = np.exp(np.float64(g[0, t, h]))
            b = np.float64(beta[0, t, h])
            st = a * (1.0 - b) * st + b * np.sign(k[0, t, h, 0]) * v[0, t, h, 0]
            assert abs(out[0, t, h, 0] - np.sign(q[0, t, h, 0]) * st) <= 1e-13 * max(1.0, abs(st))
        assert abs(S[0, h, 0, 0] - st) <= 1e-13 * max(1.0, abs(st))


@pytest.mark.parametrize("impl", ["c", "numpy"])
def test_p10_bidir_single_token(impl):
    """Pin p10: T = 1 bidirectional -> out = forward + beta (q^ . k^) v (the
    reverse scan from zero state sees only the token itself)."""
    rng = np.random.default_rng(17)
    q, k, v, g, beta, s = rand_inputs(rng, 2, 1, 3, 10, 4)
    out_f, S_f = FWD[impl](q, k, v, g, beta, s)
    out_b, S_b = BIDIR[impl](q, k, v, g, beta, s)
    qk = np.sum(unit(q[:, 0]) * unit(k[:, 0]), -1)
    expect = out_f[:, 0] + beta[:, 0, :, None] * qk[..., None] * v[:, 0]
    np.testing.assert_allclose(out_b[:, 0], expect, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S_b, S_f, rtol=0, atol=0)


# ---------------------------------------------------------------- invariants
@pytest.mark.parametrize("impl", ["c", "numpy"])
def test_p5_streaming_equals_one_scan(impl):
    """Pin p5: chunks scanned one after another with the state carried equal
    one scan over their concatenation (outputs and state)."""
    rng = np.random.default_rng(18)
    q, k, v, g, beta, s = rand_inputs(rng, 2, 37, 2, 8, 8)
    out, S = FWD[impl](q, k, v, g, beta, s)
    cuts = [0, 5, 6, 20, 37]
    St = s
    for a, b in zip(cuts[:-1], cuts[1:]):
        o, St = FWD[impl](q[:, a:b], k[:, a:b], v[:, a:b], g[:, a:b], beta[:, a:b], St)
        np.testing.assert_allclose(o, out[:, a:b], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(St, S, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("impl", ["c", "numpy"])
def test_p6_linearity_in_values_and_state(impl):
    """Pin p6: for fixed q, k, g, beta the map (V, S_in) -> (out, S_out) is
    linear."""
    rng = np.random.default_rng(19)
    q, k, v1, g, beta, s1 = rand_inputs(rng)
    # values on a 1/64 grid so the combination below is exact in fp32 inputs
    v1 = (np.round(v1 * 64) / 64).astype(np.float32)
    v2 = (np.round(rng.standard_normal(v1.shape) * 64) / 64).astype(np.float32)
    s2 = rng.standard_normal(s1.shape)
    al, be = np.float32(0.75), np.float32(-1.5)
    o1, S1 = FWD[impl](q, k, v1, g, beta, s1)
    o2, S2 = FWD[impl](q, k, v2, g, beta, s2)
    o3, S3 = FWD[impl](q, k, al * v1 + be * v2, g, beta, al * s1 + be * s2)
    np.testing.assert_allclose(o3, al * o1 + be * o2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S3, al * S1 + be * S2, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("impl", ["c", "numpy"])
def test_p7_columns_are_independent(impl):
    """Pin p7: column j of out and of S depends only on v[..., j] and
    S_in[..., j]; perturbing column 2 leaves every other column bit-equal."""
    rng = np.random.default_rng(20)
    q, k, v, g, beta, s = rand_inputs(rng, Dv=6)
    o1, S1 = FWD[impl](q, k, v, g, beta, s)
    v2, s2 = v.copy(), s.copy()
    v2[..., 2] += 1.0
    s2[..., 2] -= 0.5
    o2, S2 = FWD[impl](q, k, v2, g, beta, s2)
    keep = [0, 1, 3, 4, 5]
    assert np.array_equal(o1[..., keep], o2[..., keep])
    assert np.array_equal(S1[..., keep], S2[..., keep])
    assert np.max(np.abs(o1[..., 2] - o2[..., 2])) > 1e-3


@pytest.mark.parametrize("impl", ["c", "numpy"])
def test_p8_state_norm_bound(impl):
    """Pin p8: |I - b k^k^T|_2 = 1 for b in [0,1], so
    |S_t|_2 <= a_t |S_{t-1}|_2 + beta_t |v_t|.  Checked token by token."""
    rng = np.random.default_rng(21)
    q, k, v, g, beta, s = rand_inputs(rng, 1, 30, 2, 8, 8, g_lo=-0.3)
    St = s
    for t in range(30):
        _, Sn = FWD[impl](q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1], g[:, t:t + 1],
                          beta[:, t:t + 1], St)
        for h in range(2):
            lhs = np.linalg.norm(Sn[0, h], 2)
            rhs = (np.exp(np.float64(g[0, t, h])) * np.linalg.norm(St[0, h], 2)
                   + np.float64(beta[0, t, h]) * np.linalg.norm(v[0, t, h].astype(np.float64)))
            assert lhs <= rhs * (1 + 1e-12)
        St = Sn


def test_bidir_is_forward_plus_flipped_forward():
    """Reading of the bidirectional mode: out = fwd(state_in) + flip(fwd(flip(x),
    0)); the state comes from the forward scan only (C oracle vs its own
    forward entry point run on the flipped sequence)."""
    rng = np.random.default_rng(22)
    q, k, v, g, beta, s = rand_inputs(rng)
    out_b, S_b = c_bidir(q, k, v, g, beta, s)
    out_f, S_f = c_fwd(q, k, v, g, beta, s)
    fl = lambda x: np.ascontiguousarray(x[:, ::-1])  # noqa: E731
    out_r, _ = c_fwd(fl(q), fl(k), fl(v), fl(g), fl(beta), None)
    np.testing.assert_allclose(out_b, out_f + out_r[:, ::-1], rtol=1e-14, atol=1e-14)
    np.testing.assert_array_equal(S_b, S_f)


# --------------------------------------------------------------- brute force
@pytest.mark.parametrize("chunk", [1, 3, 16, 64])
@pytest.mark.parametrize("T", [1, 37, 100])
def test_p4_chunked_form_equals_recurrence(chunk, T):
    """Pin p4: the chunked WY/UT form (an independent algorithm) reaches the
    token recurrence to ~1e-13 for every sub-chunk length, ragged tails
    included."""
    rng = np.random.default_rng(100 + T + chunk)
    q, k, v, g, beta, s = rand_inputs(rng, 1, T, 2, 16, 12, g_lo=-1.0)
    o_c, S_c = oracle.chunked_fwd(q, k, v, g, beta, s, chunk)
    o_r, S_r = c_fwd(q, k, v, g, beta, s)
    assert rel(o_c, o_r) < 1e-12
    assert rel(S_c, S_r) < 1e-12
    ob_c, _ = oracle.chunked_bidir(q, k, v, g, beta, s, chunk)
    ob_r, _ = c_bidir(q, k, v, g, beta, s)
    assert rel(ob_c, ob_r) < 1e-12


def test_p4_chunked_form_fast_decay_does_not_overflow():
    """Pin p4 (fast decay): g in [-8,-4] over a 64-token sub-chunk drives
    exp(gamma) to ~e^-400; the chunked form must still equal the recurrence."""
    rng = np.random.default_rng(31)
    q, k, v, g, beta, s = rand_inputs(rng, 1, 130, 2, 16, 16)
    g[:] = rng.uniform(-8, -4, g.shape)
    with np.errstate(under="ignore"):
        o_c, S_c = oracle.chunked_fwd(q, k, v, g, beta, s, 64)
    o_r, S_r = c_fwd(q, k, v, g, beta, s)
    assert np.all(np.isfinite(o_c))
    assert rel(o_c, o_r) < 1e-12


def test_c_and_numpy_recurrences_agree_on_tiny_workload():
    """The two transcriptions agree on the tiny fp32 workload (fwd + bidir)."""
    w = wl.tiny()
    x = wl.make_inputs(w)
    args = (x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"])
    o1, S1 = c_fwd(*args)
    o2, S2 = oracle.recurrence_fwd(*args)
    assert rel(o1, o2) < 1e-13 and rel(S1, S2) < 1e-13
    o1, _ = c_bidir(*args)
    o2, _ = oracle.recurrence_bidir(*args)
    assert rel(o1, o2) < 1e-13


def test_p11_double_vs_long_double_error_floor():
    """Pin p11: on the stress gate extremes (near-identity and fast decay,
    beta 0.01 / 0.99) the double oracle agrees with a long-double rerun to
    far below the parity tolerances, so its own rounding is negligible."""
    rng = np.random.default_rng(41)
    for lo, hi in ((-1e-4, 0.0), (-8.0, -4.0)):
        for b in (0.01, 0.99):
            q, k, v, g, beta, s = rand_inputs(rng, 1, 512, 2, 32, 32, unit=True)
            g[:] = rng.uniform(lo, hi, g.shape)
            beta[:] = b
            o64, S64 = oracle.oracle_fwd(q, k, v, g, beta, s, nthreads=2)
            oLD, SLD = oracle.oracle_fwd(q, k, v, g, beta, s, nthreads=2, precision="long double")
            assert rel(o64, oLD.astype(np.float64)) < 1e-11
            assert rel(S64, SLD.astype(np.float64)) < 1e-11


def test_empty_sequence_passes_state_through():
    """T = 0: nothing to scan, state_out = state_in (or zero)."""
    rng = np.random.default_rng(5)
    q, k, v, g, beta, s = rand_inputs(rng, 1, 0, 2, 4, 4)
    out, S = c_fwd(q, k, v, g, beta, s)
    assert out.shape == (1, 0, 2, 4)
    np.testing.assert_array_equal(S, s)
    _, S0 = c_fwd(q, k, v, g, beta, None)
    assert not S0.any()


def test_oracle_planted_sign_error_is_caught():
    """The pins have teeth: an oracle with the decay applied after the delta
    correction instead of before (a plausible slip) fails pin p2's exact
    write-back once a < 1.  Planted in a CPU copy of the numpy recurrence."""
    def wrong_fwd(q, k, v, g, beta, s):
        q, k, v, g, beta = [np.asarray(x, np.float64) for x in (q, k, v, g, beta)]
        S = np.array(s, copy=True)
        out = np.zeros(v.shape)
        for t in range(q.shape[1]):
            kh = unit(k[:, t])
            a = np.exp(g[:, t])[..., None, None]
            b = beta[:, t][..., None, None]
            S = a * S
            S = S - b * kh[..., :, None] * np.einsum("bhi,bhij->bhj", kh, S)[..., None, :] \
                + a * b * kh[..., :, None] * v[:, t][..., None, :]
            out[:, t] = np.einsum("bhi,bhij->bhj", unit(q[:, t]), S)
        return out, S

    rng = np.random.default_rng(6)
    q, k, v, g, beta, s = rand_inputs(rng, 1, 3, 1, 4, 3)
    g[:] = -0.5
    beta[:] = 1.0
    _, S_ok = c_fwd(q, k, v, g, beta, s)
    _, S_bad = wrong_fwd(q, k, v, g, beta, s)
    kh = unit(k[:, -1])
    ok = np.einsum("bhi,bhij->bhj", kh, S_ok)
    bad = np.einsum("bhi,bhij->bhj", kh, S_bad)
    # with beta = 1 the right ordering gives S^T k^ = v for any a; the slip gives a v
    np.testing.assert_allclose(ok, v[:, -1], atol=1e-12)
    assert np.max(np.abs(bad - v[:, -1])) > 1e-2


# ---------------------------------------------------------------------------
# Gate activations of the fused prologue (g = -softplus(x), beta = sigmoid(y))
# ---------------------------------------------------------------------------
# The pages keep the gate layer in BF16 without writing its activations; the
# reading taken is g = -softplus(x) (so g <= 0 and a = e^g = 1 / (1 + e^x))
# and beta = sigmoid(y).  The pins below use only closed forms of those maps.

FWD_LOGITS = {
    "c": lambda q, k, v, x, y, s=None: oracle.oracle_fwd_logits(q, k, v, x, y, s, nthreads=2),
    "c_ld": lambda q, k, v, x, y, s=None: oracle.oracle_fwd_logits(q, k, v, x, y, s, nthreads=2,
                                                                   precision="long double"),
    "numpy": lambda q, k, v, x, y, s=None: oracle.recurrence_fwd(
        q, k, v, *oracle.gates_from_logits(x, y), s),
}


def test_gate_maps_closed_forms():
    """softplus(0) = ln 2 and sigmoid(0) = 1/2; softplus(x) - softplus(-x) = x;
    sigmoid(y) + sigmoid(-y) = 1; e^{-softplus(x)} = 1 / (1 + e^x); and the
    limits g -> -x for large x, g -> 0 for very negative x."""
    x = np.array([-30.0, -3.0, -0.5, 0.0, 0.5, 3.0, 30.0])
    g, b = oracle.gates_from_logits(x, x)
    assert g[3] == pytest.approx(-np.log(2.0), abs=1e-16)
    assert b[3] == pytest.approx(0.5, abs=1e-16)
    g_neg, b_neg = oracle.gates_from_logits(-x, -x)
    np.testing.assert_allclose(-g + g_neg, x, atol=1e-14)
    np.testing.assert_allclose(b + b_neg, 1.0, atol=1e-15)
    np.testing.assert_allclose(np.exp(g), 1.0 / (1.0 + np.exp(x)), rtol=1e-14)
    np.testing.assert_allclose(b, 1.0 / (1.0 + np.exp(-x)), rtol=1e-14)
    assert np.all(g <= 0) and np.all(np.diff(g) < 0) and np.all(np.diff(b) > 0)
    assert g[-1] == pytest.approx(-30.0, abs=1e-12) and g[0] == pytest.approx(0.0, abs=1e-12)


@pytest.mark.parametrize("impl", sorted(FWD_LOGITS))
def test_gate_logits_pure_decay(impl):
    """beta logit -800 (beta = 0 in double): the state only decays, by
    1 / (1 + e^x) per token: S_t = prod_{s<=t} 1/(1 + e^{x_s}) S_in and
    o_t = S_t^T q^_t."""
    rng = np.random.default_rng(11)
    B, T, H, D = 1, 9, 2, 5
    q = rng.standard_normal((B, T, H, D)).astype(np.float32)
    k = rng.standard_normal((B, T, H, D)).astype(np.float32)
    v = rng.standard_normal((B, T, H, D)).astype(np.float32)
    x = rng.uniform(-3, 3, (B, T, H)).astype(np.float32)
    y = np.full((B, T, H), -800.0, np.float32)
    s = rng.standard_normal((B, H, D, D))
    out, S = FWD_LOGITS[impl](q, k, v, x, y, s)
    dec = np.cumprod(1.0 / (1.0 + np.exp(x.astype(np.float64))), axis=1)  # [B,T,H]
    np.testing.assert_allclose(np.asarray(S, np.float64), s * dec[:, -1][:, :, None, None], rtol=1e-13)
    ref = np.einsum("bth,bthi,bhij->bthj", dec, unit(q), s)
    np.testing.assert_allclose(np.asarray(out, np.float64), ref, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("impl", sorted(FWD_LOGITS))
def test_gate_logits_write_strength(impl):
    """decay logit -800 (a = 1 in double) and orthonormal keys e_t: token t
    replaces row t by (1 - sigmoid(y_t)) S_in[t] + sigmoid(y_t) v_t, with
    sigmoid(y) = 1 / (1 + e^-y)."""
    rng = np.random.default_rng(12)
    B, T, H, D = 1, 6, 1, 6
    k = np.zeros((B, T, H, D), np.float32)
    for t in range(T):
        k[0, t, 0, t] = 1.0
    q = rng.standard_normal((B, T, H, D)).astype(np.float32)
    v = rng.standard_normal((B, T, H, D)).astype(np.float32)
    x = np.full((B, T, H), -800.0, np.float32)
    y = rng.uniform(-4, 4, (B, T, H)).astype(np.float32)
    s = rng.standard_normal((B, H, D, D))
    _, S = FWD_LOGITS[impl](q, k, v, x, y, s)
    bt = 1.0 / (1.0 + np.exp(-y[0, :, 0].astype(np.float64)))
    want = s[0, 0].copy()
    for t in range(T):
        want[t] = (1.0 - bt[t]) * s[0, 0, t] + bt[t] * v[0, t, 0]
    np.testing.assert_allclose(np.asarray(S, np.float64)[0, 0], want, rtol=1e-13, atol=1e-15)


def test_gate_logits_half_gates_scalar():
    """x = y = 0 gives a = beta = 1/2 exactly; with d = 1 the scan is the
    scalar recurrence s_t = a (1 - beta) s + beta sign(k_t) v_t = s / 4 +
    sign(k_t) v_t / 2, o_t = sign(q_t) s_t (forward and bidirectional)."""
    rng = np.random.default_rng(13)
    T = 7
    q = rng.standard_normal((1, T, 1, 1)).astype(np.float32)
    k = rng.standard_normal((1, T, 1, 1)).astype(np.float32)
    v = rng.standard_normal((1, T, 1, 1)).astype(np.float32)
    z = np.zeros((1, T, 1), np.float32)
    s0 = np.array([[[[0.7]]]])
    out, S = oracle.oracle_fwd_logits(q, k, v, z, z, s0, nthreads=1)
    sk, sq, vv = np.sign(k[0, :, 0, 0]), np.sign(q[0, :, 0, 0]), v[0, :, 0, 0].astype(np.float64)
    s, want = 0.7, []
    for t in range(T):
        s = s / 4 + sk[t] * vv[t] / 2
        want.append(sq[t] * s)
    np.testing.assert_allclose(out[0, :, 0, 0], want, rtol=1e-14)
    assert S[0, 0, 0, 0] == pytest.approx(s, rel=1e-14)
    outb, _ = oracle.oracle_bidir_logits(q, k, v, z, z, s0, nthreads=1)
    r, rev = 0.0, np.zeros(T)
    for t in reversed(range(T)):
        r = r / 4 + sk[t] * vv[t] / 2
        rev[t] = sq[t] * r
    np.testing.assert_allclose(outb[0, :, 0, 0], np.array(want) + rev, rtol=1e-13)


def test_gate_logits_c_matches_numpy_gates():
    """Both transcriptions agree: the C oracle's logit mode against the numpy
    gates fed to the numpy recurrence (all fp64), on random logits, both
    directions."""
    rng = np.random.default_rng(14)
    q, k, v, _, _, s = rand_inputs(rng, T=31)
    x = rng.standard_normal((2, 31, 3)).astype(np.float32) * 2
    y = rng.standard_normal((2, 31, 3)).astype(np.float32) * 2
    o1, S1 = oracle.oracle_fwd_logits(q, k, v, x, y, s, nthreads=2)
    g, b = oracle.gates_from_logits(x, y)
    o2, S2 = oracle.recurrence_fwd(q, k, v, g, b, s)
    assert rel(o1, o2) < 1e-12 and rel(S1, S2) < 1e-12
    ob1, _ = oracle.oracle_bidir_logits(q, k, v, x, y, s, nthreads=2)
    ob2, _ = oracle.recurrence_bidir(q, k, v, g, b, s)
    assert rel(ob1, ob2) < 1e-12


def test_planted_gate_slip_fails_the_decay_pin():
    """A plausible slip -- softplus of -x instead of x, i.e. a = sigmoid(x)
    instead of 1 - sigmoid(x) -- planted in a copy of the numpy gate map
    fails the pure-decay closed form."""
    rng = np.random.default_rng(11)
    B, T, H, D = 1, 9, 2, 5
    q = rng.standard_normal((B, T, H, D)).astype(np.float32)
    k = rng.standard_normal((B, T, H, D)).astype(np.float32)
    v = rng.standard_normal((B, T, H, D)).astype(np.float32)
    x = rng.uniform(-3, 3, (B, T, H)).astype(np.float32)
    s = rng.standard_normal((B, H, D, D))
    g_wrong = -np.logaddexp(0.0, -x.astype(np.float64))
    _, S = oracle.recurrence_fwd(q, k, v, g_wrong, np.zeros((B, T, H)), s)
    dec = np.prod(1.0 / (1.0 + np.exp(x.astype(np.float64))), axis=1)
    assert not np.allclose(S, s * dec[:, :, None, None], rtol=1e-6)


# ---------------------------------------------------------------------------
# Reference gradients (oracle/backward.py): autograd of the definition
# ---------------------------------------------------------------------------


def _fd_inputs(rng, B=1, T=5, H=2, Dk=3, Dv=2):
    q = rng.standard_normal((B, T, H, Dk))
    k = rng.standard_normal((B, T, H, Dk))
    v = rng.standard_normal((B, T, H, Dv))
    g = rng.uniform(-1.0, -0.05, (B, T, H))
    beta = rng.uniform(0.1, 0.9, (B, T, H))
    s = 0.5 * rng.standard_normal((B, H, Dk, Dv))
    return q, k, v, g, beta, s


@pytest.mark.parametrize("bidir", [False, True])
def test_backward_matches_central_differences(bidir):
    """Every gradient of L = <out, W1> + <state_out, W2> against central
    differences of the token recurrence (fp64, step 1e-6), element by
    element, for all six inputs."""
    rng = np.random.default_rng(21)
    q, k, v, g, beta, s = _fd_inputs(rng)
    W1 = rng.standard_normal(v.shape)
    W2 = rng.standard_normal(s.shape)
    gr = oracle.backward.grads(q, k, v, g, beta, s, W1, W2, bidir=bidir)

    def loss(xs):
        o, S = oracle.recurrence_bidir(*xs) if bidir else oracle.recurrence_fwd(*xs)
        return float(np.sum(o * W1) + np.sum(S * W2))
    base = [q, k, v, g, beta, s]
    h = 1e-6
    for idx, name in enumerate(["dq", "dk", "dv", "dg", "dbeta", "dstate_in"]):
        x = base[idx]
        fd = np.zeros_like(x)
        for e in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[e] += h
            xm[e] -= h
            bp, bm = list(base), list(base)
            bp[idx], bm[idx] = xp, xm
            fd[e] = (loss(bp) - loss(bm)) / (2 * h)
        np.testing.assert_allclose(gr[name], fd, rtol=1e-5, atol=1e-7, err_msg=name)


def test_backward_pure_decay_closed_form():
    """beta = 0: o_t = (prod_{s<=t} a_s) S_in^T q^_t and S_T = (prod a) S_in,
    so dv = 0 and dstate_in = sum_t (prod_{s<=t} a_s) q^_t do_t^T +
    (prod a) dS_T, in closed form."""
    rng = np.random.default_rng(22)
    q, k, v, g, _, s = _fd_inputs(rng, T=7, Dk=4, Dv=3)
    beta = np.zeros(g.shape)
    do = rng.standard_normal(v.shape)
    dS = rng.standard_normal(s.shape)
    gr = oracle.backward.grads(q, k, v, g, beta, s, do, dS)
    assert np.all(gr["dv"] == 0)
    dec = np.cumprod(np.exp(g), axis=1)                      # [B,T,H]
    qn = q / np.linalg.norm(q, axis=-1, keepdims=True)
    want = np.einsum("bth,bthi,bthj->bhij", dec, qn, do) + dec[:, -1][..., None, None] * dS
    np.testing.assert_allclose(gr["dstate_in"], want, rtol=1e-12, atol=1e-13)


def test_backward_is_linear_in_the_upstream_gradients():
    rng = np.random.default_rng(23)
    q, k, v, g, beta, s = _fd_inputs(rng, T=6)
    d1, d2 = rng.standard_normal(v.shape), rng.standard_normal(v.shape)
    e1, e2 = rng.standard_normal(s.shape), rng.standard_normal(s.shape)
    g1 = oracle.backward.grads(q, k, v, g, beta, s, d1, e1, bidir=True)
    g2 = oracle.backward.grads(q, k, v, g, beta, s, d2, e2, bidir=True)
    g12 = oracle.backward.grads(q, k, v, g, beta, s, 2 * d1 - 3 * d2, 2 * e1 - 3 * e2, bidir=True)
    for n in ("dq", "dk", "dv", "dg", "dbeta", "dstate_in"):
        np.testing.assert_allclose(g12[n], 2 * g1[n] - 3 * g2[n], rtol=1e-10, atol=1e-12, err_msg=n)


@pytest.mark.parametrize("bidir", [False, True])
def test_backward_forward_matches_c_oracle(bidir):
    """The torch transcription's forward is the C oracle's (both fp64)."""
    rng = np.random.default_rng(24)
    q, k, v, g, beta, s = rand_inputs(rng, T=19)
    o1, S1 = oracle.backward.forward_np(q, k, v, g, beta, s, bidir)
    o2, S2 = (c_bidir if bidir else c_fwd)(q, k, v, g, beta, s)
    assert rel(o1, o2) < 1e-12 and rel(S1, S2) < 1e-12


@pytest.mark.parametrize("bidir", [False, True])
def test_backward_single_token_adjoint_closed_form(bidir):
    """T = 1, worked out by hand from one update step.  With M = q^ do^T + dS
    (the gradient reaching S_1 = a (I - b k^k^T) S_0 + b k^ v^T):

        dS_0 = a (I - b k^k^T) M          dv = b M^T k^
        dg   = a <M, (I - b k^k^T) S_0>   db = <M, k^ v^T - a k^ k^T S_0>
        dq^  = S_1 do                      dk^ = b M v - a b (M S_0^T + S_0 M^T) k^

    and dx = (I - x^x^T) dx^ / |x| for the two normalised inputs.  The
    reverse scan of a one-token chunk starts from zero, so bidirectional mode
    adds o_r = b (k^.q^) v: dv += b (k^.q^) do, db += (k^.q^)(v.do),
    dq^ += b (v.do) k^, dk^ += b (v.do) q^.  Each term is a separate
    derivation, so a dropped term, a wrong sign or a transposed S_0 or M in
    the oracle's gradient moves one of the six outputs."""
    rng = np.random.default_rng(25)
    Dk, Dv = 4, 3
    q, k, v, g, beta, s = _fd_inputs(rng, B=1, T=1, H=1, Dk=Dk, Dv=Dv)
    do = rng.standard_normal(v.shape)
    dS = rng.standard_normal(s.shape)
    gr = oracle.backward.grads(q, k, v, g, beta, s, do, dS, bidir=bidir)

    qv, kv, vv, S0 = q[0, 0, 0], k[0, 0, 0], v[0, 0, 0], s[0, 0]
    a, b, dov = np.exp(g[0, 0, 0]), beta[0, 0, 0], do[0, 0, 0]
    nq, nk = np.linalg.norm(qv), np.linalg.norm(kv)
    qh, kh = qv / nq, kv / nk
    proj = np.eye(Dk) - b * np.outer(kh, kh)
    S1 = a * proj @ S0 + b * np.outer(kh, vv)
    M = np.outer(qh, dov) + dS[0, 0]
    want = {
        "dstate_in": a * proj @ M,
        "dv": b * M.T @ kh,
        "dg": a * np.sum(M * (proj @ S0)),
        "dbeta": np.sum(M * (np.outer(kh, vv) - a * np.outer(kh, kh @ S0))),
    }
    dqh = S1 @ dov
    dkh = b * M @ vv - a * b * (M @ S0.T + S0 @ M.T) @ kh
    if bidir:
        kq, vd = kh @ qh, vv @ dov
        want["dv"] = want["dv"] + b * kq * dov
        want["dbeta"] = want["dbeta"] + kq * vd
        dqh = dqh + b * vd * kh
        dkh = dkh + b * vd * qh
    want["dq"] = (np.eye(Dk) - np.outer(qh, qh)) @ dqh / nq
    want["dk"] = (np.eye(Dk) - np.outer(kh, kh)) @ dkh / nk
    for name, w in want.items():
        got = np.asarray(gr[name], np.float64).reshape(np.shape(w))
        np.testing.assert_allclose(got, w, rtol=1e-12, atol=1e-14, err_msg=name)


@pytest.mark.parametrize("impl", ["c", "numpy"])
def test_time_segments_compose_to_the_recurrence(impl):
    """The time-segmented scan's reading: the update is affine in the state,
    S_t = a_t (I - b_t k^k^T) S_{t-1} + b_t k^ v_t^T, so a segment of tokens
    maps its start state by S_out = P S_in + R.  P is the segment walked from
    the identity (Dk columns) with zero values, R the segment walked from a
    zero state; both come from the oracle itself.  Composing the maps in time
    order must give every segment's start state and the final state of one
    scan, and re-walking each segment from its start must give that scan's
    outputs -- exactly, up to fp64 rounding, for ragged segments too."""
    rng = np.random.default_rng(26)
    Bn, Hn, Dk, Dv = 2, 2, 6, 5
    q, k, v, g, beta, s = rand_inputs(rng, Bn, 41, Hn, Dk, Dv)
    out, S_end = FWD[impl](q, k, v, g, beta, s)
    cuts = [0, 9, 10, 27, 41]
    eye = np.broadcast_to(np.eye(Dk), (Bn, Hn, Dk, Dk)).copy()
    maps = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        sl = (slice(None), slice(a, b))
        zeros_v = np.zeros(q[sl].shape[:3] + (Dk,), np.float32)
        _, P = FWD[impl](q[sl], k[sl], zeros_v, g[sl], beta[sl], eye)
        _, R = FWD[impl](q[sl], k[sl], v[sl], g[sl], beta[sl], np.zeros_like(s))
        maps.append((P, R))
    St = s
    for (a, b), (P, R) in zip(zip(cuts[:-1], cuts[1:]), maps):
        o, _ = FWD[impl](q[:, a:b], k[:, a:b], v[:, a:b], g[:, a:b], beta[:, a:b], St)
        np.testing.assert_allclose(o, out[:, a:b], rtol=1e-12, atol=1e-13)
        St = np.einsum("bhij,bhjk->bhik", P, St) + R
    np.testing.assert_allclose(St, S_end, rtol=1e-12, atol=1e-13)
    # a map that skips its decay or its projection is visibly wrong
    P0 = maps[0][0]
    assert np.max(np.abs(P0 - eye)) > 1e-2


@pytest.mark.parametrize("bidir", [False, True])
@pytest.mark.parametrize("chunk,with_state", [(4, True), (7, True), (64, True), (7, False)])
def test_chunked_reverse_mode_reaches_the_reference_gradients(bidir, chunk, with_state):
    """Brute force: reverse mode through the sub-chunked (WY / UT) form --
    dU, dS0 carried backwards over the sub-chunks, the transposed solve
    T^T [dW | dU], dA = -(X_w W^T + X_u U~^T), row and column sums for dbeta
    and dgamma, dg as a suffix sum -- reaches autograd of the token
    recurrence for every input, sub-chunks of 4, 7 (ragged) and 64 tokens,
    with and without a start state; rows of zero and of tiny norm exercise
    the normalisation's clamp."""
    rng = np.random.default_rng(27)
    q, k, v, g, beta, s = _fd_inputs(rng, B=2, T=23, H=2, Dk=6, Dv=5)
    q[0, 3, 1] = 0.0
    k[1, 11, 0] = 0.0
    q[1, 5, 0] *= 1e-8
    s = s if with_state else None
    do = rng.standard_normal(v.shape)
    dS = rng.standard_normal((2, 2, 6, 5))
    want = oracle.backward.grads(q, k, v, g, beta, s, do, dS, bidir=bidir)
    got = oracle.numpy_ref.chunked_backward(q, k, v, g, beta, s, do, dS, bidir=bidir, chunk=chunk)
    for name in ("dq", "dk", "dv", "dg", "dbeta"):
        np.testing.assert_allclose(got[name], want[name], rtol=1e-10, atol=1e-10, err_msg=name)
    if with_state:
        np.testing.assert_allclose(got["dstate_in"], want["dstate_in"], rtol=1e-10, atol=1e-12)
    else:
        assert got["dstate_in"] is None


def test_planted_gradient_slip_fails_both_gradient_pins(monkeypatch):
    """The gradient pins have teeth: a copy of the gradient oracle's
    recurrence with the decay applied after the delta correction (the slip
    the forward's planted test uses) fails the hand-derived single-token
    adjoint and the chunked reverse mode alike."""
    import torch

    def slipped(q, k, v, g, beta, S, reverse):
        T = q.shape[1]
        qn, kn = oracle.backward._normalise(q), oracle.backward._normalise(k)
        outs = [None] * T
        for t in (range(T - 1, -1, -1) if reverse else range(T)):
            kt, qt, vt = kn[:, t], qn[:, t], v[:, t]
            a = torch.exp(g[:, t])[..., None, None]
            b = beta[:, t][..., None, None]
            S = a * S
            x = torch.einsum("bhi,bhij->bhj", kt, S)
            S = S - b * kt[..., :, None] * x[..., None, :] + a * b * kt[..., :, None] * vt[..., None, :]
            outs[t] = torch.einsum("bhi,bhij->bhj", qt, S)
        return torch.stack(outs, dim=1), S

    monkeypatch.setattr(oracle.backward, "_one_direction", slipped)
    with pytest.raises(AssertionError):
        test_backward_single_token_adjoint_closed_form(False)
    with pytest.raises(AssertionError):
        test_chunked_reverse_mode_reaches_the_reference_gradients(False, 7, True)
