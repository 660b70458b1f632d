"""Invariants of the oracle's functions over generated inputs (CPU).

Each property holds for the mathematics the function states, independently
of how the oracle computes it: scale invariance of RMSNorm, linearity of
attention in the values and its indifference to the order of the keys it
sees, equivariance of the router under a relabelling of the experts, the
LM-head statistics under a constant shift of every logit, the monotonicity
of the entropy budget, the sampler choosing between its two inputs, and the
MXFP8 encoding under powers of two."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import model as om

SETTINGS = settings(max_examples=40, deadline=None)
seeds = st.integers(min_value=0, max_value=2 ** 32 - 1)


@SETTINGS
@given(seeds, st.floats(min_value=1e-3, max_value=1e3))
def test_rms_norm_is_scale_invariant_and_odd(seed, c):
    r = np.random.default_rng(seed)
    h = r.standard_normal((3, 64))
    g = r.standard_normal(64)
    np.testing.assert_allclose(om.rms_norm(c * h, g, 0.0), om.rms_norm(h, g, 0.0), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(om.rms_norm(-h, g, 0.0), -om.rms_norm(h, g, 0.0), rtol=1e-12, atol=1e-15)


@SETTINGS
@given(seeds, st.sampled_from([(2, 1), (4, 2), (4, 4)]), st.booleans())
def test_attention_is_linear_in_values_and_ignores_key_order(seed, heads, causal):
    r = np.random.default_rng(seed)
    Hq, Hkv = heads
    n, P, D = 5, 7, 8
    q = r.standard_normal((Hq, n, D))
    k = r.standard_normal((Hkv, P + n, D))
    v1, v2 = r.standard_normal((2, Hkv, P + n, D))
    lim = P + 1 + np.arange(n) if causal else np.full(n, P + n)
    a = om.attention(q, k, v1 + v2, lim)
    np.testing.assert_allclose(a, om.attention(q, k, v1, lim) + om.attention(q, k, v2, lim), rtol=1e-10, atol=1e-12)
    if not causal:
        # the same visible keys in another order give the same output
        perm = r.permutation(P + n)
        np.testing.assert_allclose(om.attention(q, k[:, perm], v1[:, perm], lim), om.attention(q, k, v1, lim),
                                   rtol=1e-10, atol=1e-12)


@SETTINGS
@given(seeds, st.integers(min_value=1, max_value=6))
def test_router_is_equivariant_under_relabelled_experts(seed, k):
    r = np.random.default_rng(seed)
    E = 12
    logits = r.standard_normal((4, E))                  # continuous: no ties
    perm = r.permutation(E)                             # expert perm[j] is called j after relabelling
    idx, g = om.route_top_k(logits, k)
    idx2, g2 = om.route_top_k(logits[:, perm], k)
    np.testing.assert_array_equal(perm[idx2], idx)
    np.testing.assert_allclose(g2, g, rtol=1e-14)
    assert np.allclose(g.sum(axis=1), 1.0) and (np.diff(g, axis=1) <= 1e-15).all()   # gates descend


@SETTINGS
@given(seeds, st.floats(min_value=-50.0, max_value=50.0), st.sampled_from([0.3, 1.0, 2.0]))
def test_lm_head_stats_under_a_constant_logit_shift(seed, c, temp):
    """A constant column in the embedding matched by z adds c/T to every
    logit: lse and max move by c/T, nothing else changes."""
    r = np.random.default_rng(seed)
    z = r.standard_normal((3, 6))
    E = r.standard_normal((29, 6))
    a = om.lm_head_stats(z, E, temp)
    b = om.lm_head_stats(np.hstack([z, np.full((3, 1), c)]), np.hstack([E, np.ones((29, 1))]), temp)
    np.testing.assert_array_equal(a["argmax"], b["argmax"])
    np.testing.assert_allclose(b["lse"] - a["lse"], c / temp, rtol=1e-10, atol=1e-10)
    for key in ("conf", "logp", "margin", "gap", "entropy"):
        np.testing.assert_allclose(b[key], a[key], rtol=1e-9, atol=1e-9)


@SETTINGS
@given(seeds, st.floats(min_value=0.0, max_value=20.0), st.floats(min_value=0.0, max_value=20.0))
def test_entropy_budget_is_monotone(seed, g1, g2):
    r = np.random.default_rng(seed)
    e = r.exponential(1.0, 40).astype(np.float32)
    lo, hi = sorted((g1, g2))
    a, b = om.entropy_accept(e, lo), om.entropy_accept(e, hi)
    assert (a <= b).all() and a.sum() >= 1
    # what is accepted is a prefix of the (entropy, position) order
    order = sorted(range(40), key=lambda i: (e[i], i))
    assert b[order].tolist() == sorted(b[order].tolist(), reverse=True)


@SETTINGS
@given(seeds, st.floats(min_value=0.0, max_value=1.0))
def test_sampler_picks_one_of_its_inputs(seed, tau):
    r = np.random.default_rng(seed)
    n = 200
    a = r.integers(0, 1000, n)
    conf = r.random(n)
    noise = om.renoise_tokens(np.arange(n), int(r.integers(0, 48)), 0, int(r.integers(0, 2 ** 63)), 1000)
    out = om.sample(a, conf, tau, noise)
    assert ((out == a) | (out == noise)).all()
    assert (out[conf >= tau] == a[conf >= tau]).all()
    assert noise.min() >= 0 and noise.max() < 1000


@SETTINGS
@given(seeds, st.integers(min_value=-20, max_value=20))
def test_mx_encoding_commutes_with_powers_of_two(seed, k):
    """Scaling a block by 2^k shifts its shared exponent by k and nothing
    else, so the MXFP8 encoding commutes with it exactly (away from the
    float64 range limits), and encoding twice changes nothing."""
    from oracle import mx
    r = np.random.default_rng(seed)
    x = r.standard_normal((2, 96)) * np.exp(r.uniform(-6, 6, (2, 1)))
    y = mx.mx_round_trip(x)
    np.testing.assert_array_equal(mx.mx_round_trip(np.ldexp(x, k)), np.ldexp(y, k))
    np.testing.assert_array_equal(mx.mx_block_exponents(np.ldexp(x, k)), mx.mx_block_exponents(x) + k)
    np.testing.assert_array_equal(mx.mx_round_trip(y), y)
