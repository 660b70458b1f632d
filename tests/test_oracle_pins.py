"""Pins of the oracle against facts that do not come from the oracle itself.

Each test names what fixes the expected value: a published known-answer table,
an independent library routine (torch / scipy in float64), a closed form, an
invariant the pages state, or brute force on tiny inputs.  CPU only.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import model as om
from oracle.philox import philox4x32_10, uniform_token
import synth_inputs as si

GOLD = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


# --- Philox: published known answers (Random123 / SC'11) ------------------
def test_philox_known_answers():
    n = 0
    for line in open(os.path.join(GOLD, "philox4x32_10_kat.txt")):
        if line.startswith("#") or not line.strip():
            continue
        v = [int(x, 16) for x in line.split()]
        out = philox4x32_10(v[0], v[1], v[2], v[3], v[4], v[5])
        assert [int(o) for o in out] == v[6:]
        n += 1
    assert n == 3


def test_uniform_token_power_of_two_is_exact_mask():
    w = np.array([0, 1, 0xFFFFFFFF, 0x12345678], dtype=np.uint64)
    assert list(uniform_token(w, 8192)) == [0, 1, 8191, 0x12345678 & 8191]
    # non power of two: multiply-shift lands in range and is monotone in w
    t = uniform_token(np.array([0, 0x80000000, 0xFFFFFFFF], np.uint64), 1000)
    assert list(t) == [0, 500, 999]


# --- RMSNorm / SiLU against torch ------------------------------------------
def test_rms_norm_matches_torch_and_has_unit_rms():
    h = rng.standard_normal((7, 96)) * 3.0
    g = rng.standard_normal(96)
    ref = torch.nn.functional.rms_norm(torch.tensor(h), (96,), torch.tensor(g), eps=1e-6).numpy()
    np.testing.assert_allclose(om.rms_norm(h, g, 1e-6), ref, rtol=1e-12, atol=1e-12)
    u = om.rms_norm(h, np.ones(96), 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(u * u, axis=1)), 1.0, rtol=1e-12)


def test_silu_matches_torch():
    x = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(om.silu(x), torch.nn.functional.silu(torch.tensor(x)).numpy(),
                               rtol=1e-13, atol=1e-300)


# --- RoPE: complex-rotation form, identity at 0, relative-position property --
def test_rope_equals_complex_rotation():
    D, n, base = 12, 5, 10000.0
    x = rng.standard_normal((n, D))
    pos = np.array([0, 1, 7, 100, 4095])
    cos, sin = om.rope_angles(pos, D, base)
    got = om.apply_rope(x, cos, sin)
    half = D // 2
    zc = x[:, :half] + 1j * x[:, half:]
    theta = np.array([[p * base ** (-2.0 * j / D) for j in range(half)] for p in pos])
    rot = zc * np.exp(1j * theta)
    np.testing.assert_allclose(got[:, :half], rot.real, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got[:, half:], rot.imag, rtol=1e-12, atol=1e-12)


def test_rope_identity_at_zero_and_relative():
    D = 176
    q = rng.standard_normal(D)
    k = rng.standard_normal(D)
    c0, s0 = om.rope_angles(np.array([0]), D, 10000.0)
    np.testing.assert_array_equal(om.apply_rope(q[None], c0, s0)[0], q)

    def dot(m, n):
        cm, sm = om.rope_angles(np.array([m]), D, 10000.0)
        cn, sn = om.rope_angles(np.array([n]), D, 10000.0)
        return om.apply_rope(q[None], cm, sm)[0] @ om.apply_rope(k[None], cn, sn)[0]

    a = dot(5, 2)
    for m in (3, 17, 300, 2050):
        assert abs(dot(m, m - 3) - a) <= 1e-9 * max(1.0, abs(a))


# --- attention: textbook causal / full attention (torch SDPA, float64) -------
def _sdpa(q, k, v, causal):
    group = q.shape[0] // k.shape[0]
    kk = torch.tensor(k).repeat_interleave(group, 0)
    vv = torch.tensor(v).repeat_interleave(group, 0)
    o = torch.nn.functional.scaled_dot_product_attention(torch.tensor(q), kk, vv, is_causal=causal)
    return o.numpy().transpose(1, 0, 2).reshape(q.shape[1], -1)


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (4, 4), (8, 2)])
def test_attention_causal_reduces_to_sdpa(Hq, Hkv):
    n, D = 19, 16
    q, k, v = (rng.standard_normal((H, n, D)) for H in (Hq, Hkv, Hkv))
    got = om.attention(q, k, v, np.arange(1, n + 1))
    np.testing.assert_allclose(got, _sdpa(q, k, v, True), rtol=1e-11, atol=1e-12)


def test_attention_bidirectional_no_cache_is_full_sdpa():
    n, D = 23, 8
    q, k, v = rng.standard_normal((4, n, D)), rng.standard_normal((2, n, D)), rng.standard_normal((2, n, D))
    got = om.attention(q, k, v, np.full(n, n))
    np.testing.assert_allclose(got, _sdpa(q, k, v, False), rtol=1e-11, atol=1e-12)


def test_attention_with_cache_brute_force():
    Hq, Hkv, P, n, D = 2, 1, 3, 4, 4
    q = rng.standard_normal((Hq, n, D))
    k = rng.standard_normal((Hkv, P + n, D))
    v = rng.standard_normal((Hkv, P + n, D))
    for causal in (False, True):
        lim = P + 1 + np.arange(n) if causal else np.full(n, P + n)
        got = om.attention(q, k, v, lim)
        for h in range(Hq):
            for i in range(n):
                w = [math.exp(sum(q[h, i, t] * k[0, j, t] for t in range(D)) / math.sqrt(D))
                     for j in range(lim[i])]
                z = sum(w)
                for t in range(D):
                    ref = sum(w[j] * v[0, j, t] for j in range(lim[i])) / z
                    assert abs(got[i, h * D + t] - ref) < 1e-12


# --- router: brute-force ordering, ties to the lower index, gates -----------
def test_route_top_k_brute_force_and_ties():
    logits = np.array([[0.5, 2.0, 2.0, -1.0, 2.0, 0.5],
                       [1.0, 1.0, 1.0, 1.0, 1.0, 1.0],
                       [-3.0, -2.0, -1.0, 0.0, 1.0, 2.0]])
    idx, g = om.route_top_k(logits, 3)
    assert idx.tolist() == [[1, 2, 4], [0, 1, 2], [5, 4, 3]]
    np.testing.assert_allclose(g[0], [1 / 3] * 3, rtol=1e-15)
    e = np.exp([2.0, 1.0, 0.0])
    np.testing.assert_allclose(g[2], e / e.sum(), rtol=1e-14)
    # brute force over all k-subsets on random rows
    for _ in range(20):
        r = rng.standard_normal(7)
        best = max(itertools.combinations(range(7), 3), key=lambda c: sum(r[list(c)]))
        i2, _ = om.route_top_k(r[None], 3)
        assert sorted(i2[0].tolist()) == sorted(best)


# --- MoE: top-k = all experts equals the dense gate-weighted sum ------------
class _LW(dict):
    def expert(self, e, name):
        return self[name][e]


def _rand_layer(E, d, F, Fs):
    return _LW(w_gate=rng.standard_normal((E, F, d)) * 0.1, w_up=rng.standard_normal((E, F, d)) * 0.1,
               w_down=rng.standard_normal((E, d, F)) * 0.1, ws_gate=rng.standard_normal((Fs, d)) * 0.1,
               ws_up=rng.standard_normal((Fs, d)) * 0.1, ws_down=rng.standard_normal((d, Fs)) * 0.1)


def test_moe_all_experts_is_dense_softmax_mixture():
    E, d, F, Fs, n = 6, 10, 8, 12, 9
    lw = _rand_layer(E, d, F, Fs)
    u = rng.standard_normal((n, d))
    r = rng.standard_normal((n, E))
    idx, g = om.route_top_k(r, E)
    got = om.moe(u, lw, idx, g)
    # dense form: softmax over all experts, every expert applied to every row
    p = torch.softmax(torch.tensor(r), dim=1).numpy()
    t = torch.tensor(u)
    dense = torch.zeros(n, d, dtype=torch.float64)
    for e in range(E):
        a = t @ torch.tensor(lw["w_gate"][e]).T
        b = t @ torch.tensor(lw["w_up"][e]).T
        dense += torch.tensor(p[:, e:e + 1]) * ((torch.nn.functional.silu(a) * b) @ torch.tensor(lw["w_down"][e]).T)
    a = t @ torch.tensor(lw["ws_gate"]).T
    b = t @ torch.tensor(lw["ws_up"]).T
    dense += (torch.nn.functional.silu(a) * b) @ torch.tensor(lw["ws_down"]).T
    np.testing.assert_allclose(got, dense.numpy(), rtol=1e-11, atol=1e-12)


def test_moe_top1_is_single_expert():
    E, d, F, Fs, n = 5, 6, 4, 4, 7
    lw = _rand_layer(E, d, F, Fs)
    for k in ("ws_down",):
        lw[k] = np.zeros_like(lw[k])          # no shared expert
    u = rng.standard_normal((n, d))
    r = rng.standard_normal((n, E))
    idx, g = om.route_top_k(r, 1)
    np.testing.assert_array_equal(g, 1.0)
    got = om.moe(u, lw, idx, g)
    for i in range(n):
        e = int(np.argmax(r[i]))
        ref = om.swiglu_ffn(u[i:i + 1], lw["w_gate"][e], lw["w_up"][e], lw["w_down"][e])[0]
        np.testing.assert_allclose(got[i], ref, rtol=1e-12, atol=1e-14)


# --- LM-head statistics against scipy / brute force ------------------------
def test_lm_head_stats_match_logsumexp_and_ties():
    from scipy.special import logsumexp
    z = rng.standard_normal((5, 8))
    E = rng.standard_normal((37, 8))
    E[3] *= 10                                    # the longest row: a query along it peaks there (Cauchy-Schwarz)
    E[11] = E[3]                                  # exact tie between rows 3 and 11
    z[0] = E[3]
    st = om.lm_head_stats(z, E, 0.7, row_chunk=2, vocab_chunk=10)
    s = z @ E.T / 0.7
    np.testing.assert_allclose(st["lse"], logsumexp(s, axis=1), rtol=1e-13)
    assert st["argmax"][0] == 3                  # lowest index of the tied max
    assert st["margin"][0] == 0.0
    assert st["gap"][0] == 0.0
    for i in range(5):
        p = np.exp(s[i] - logsumexp(s[i]))
        srt = np.sort(p)[::-1]
        assert st["argmax"][i] == min(j for j in range(37) if s[i, j] == s[i].max())
        assert abs(st["conf"][i] - srt[0]) < 1e-14
        assert abs(st["margin"][i] - (srt[0] - srt[1])) < 1e-14
        ls = sorted(s[i], reverse=True)           # brute-force top-1 minus top-2 logit
        assert abs(st["gap"][i] - (ls[0] - ls[1])) < 1e-12


# --- sampler: fixed positions kept, re-noised tokens uniform (chi-square) ---
def test_sampler_keeps_confident_positions():
    n = 1000
    a = rng.integers(0, 8192, n)
    conf = rng.random(n)
    conf[::7] = 0.9                                # equality keeps the argmax
    conf[5] = np.nan                               # NaN re-noises
    noise = om.renoise_tokens(np.arange(n), 3, 0, 42, 8192)
    out = om.sample(a, conf, 0.9, noise)
    keep = conf >= 0.9
    np.testing.assert_array_equal(out[keep], a[keep])
    np.testing.assert_array_equal(out[~keep], noise[~keep])
    assert out[5] == noise[5]
    # deterministic in (position, step, sequence, seed)
    np.testing.assert_array_equal(noise, om.renoise_tokens(np.arange(n), 3, 0, 42, 8192))
    assert (noise != om.renoise_tokens(np.arange(n), 4, 0, 42, 8192)).mean() > 0.99


def test_renoise_tokens_are_uniform_chi_square():
    from scipy.stats import chi2
    n, V = 1 << 20, 262144
    pos = np.arange(n) % 65536
    seq = np.arange(n) // 65536
    t = om.renoise_tokens(pos, 5, seq, 0x1234567887654321, V)
    assert t.min() >= 0 and t.max() < V
    counts = np.bincount(t * 256 // V, minlength=256)
    stat = ((counts - n / 256) ** 2 / (n / 256)).sum()
    assert chi2.sf(stat, 255) > 1e-3


# --- harness arithmetic (codemajin.net section 5.1) --------------------------
def test_tpf_tps_definitions():
    # 4 blocks of 256 tokens, 40 steps in total: 3 extra commit forwards
    assert om.tokens_per_forward(1024, 40, 4) == 1024 / 43
    assert om.tokens_per_second(20.0, 0.01356) == pytest.approx(1474.9, rel=1e-4)


def test_tps_reproduces_the_printed_worked_example():
    """The pages' own numbers (tests/golden/codemajin_throughput_example.txt):
    TPS = TPF / t_fwd gives the printed 1,456 tok/s from TPF 19.74 and a
    13.56 ms step, and the printed speed-ups and sampling ratio follow from
    the printed rates and times, each at the precision it is printed to."""
    g = {}
    for line in open(os.path.join(GOLD, "codemajin_throughput_example.txt")):
        if line.strip() and not line.startswith("#"):
            name, value, dec = line.split()
            g[name] = (float(value), int(dec))

    def printed(x, name):
        v, dec = g[name]
        assert round(x, dec) == v, (name, x, v)

    tps = om.tokens_per_second(g["tpf"][0], g["t_fwd_ms"][0] * 1e-3)
    printed(tps, "tps")
    printed(g["tps"][0] / g["ar_tps"][0], "speedup_vs_ar")
    printed(g["tps"][0] / g["ar_mtp_tps"][0], "speedup_vs_ar_mtp")
    printed(g["sampling_diffusion_ms"][0] / g["sampling_ar_ms"][0], "sampling_ratio")
    # t_fwd must be in seconds: in milliseconds the same formula misses it
    assert round(om.tokens_per_second(g["tpf"][0], g["t_fwd_ms"][0])) != g["tps"][0]


# --- whole-model invariants on a tiny seeded workload ------------------------
def _tiny(**kw):
    w = si.workload("tiny").with_(**kw)
    return w


def test_commit_equals_prefill_of_concatenation():
    w = _tiny(prefix=40)
    x = si.uniform_tokens(w, "prefix", 1, 40).numpy()
    blk = si.uniform_tokens(w, "canvas", 1, 24).numpy()
    o1 = oracle.for_workload(w)
    o1.prefill(x)
    o1.commit_block(blk)
    o2 = oracle.for_workload(w)
    o2.prefill(np.concatenate([x, blk], axis=1))
    assert o1.P == o2.P == 64
    for l in range(w.shape.n_layers):
        np.testing.assert_allclose(o1.k_cache[l][0], o2.k_cache[l][0], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(o1.v_cache[l][0], o2.v_cache[l][0], rtol=1e-12, atol=1e-14)


def test_step_does_not_touch_cache_and_is_deterministic():
    w = _tiny(prefix=16)
    o = oracle.for_workload(w)
    o.prefill(si.uniform_tokens(w, "prefix", 1, 16).numpy())
    k0 = [c[0].copy() for c in o.k_cache]
    cv = si.uniform_tokens(w, "canvas", 1, 256).numpy()
    r1 = o.denoise_step(cv, 0, 7, 0.9)
    r2 = o.denoise_step(cv, 0, 7, 0.9)
    for l in range(w.shape.n_layers):
        np.testing.assert_array_equal(o.k_cache[l][0], k0[l])
    np.testing.assert_array_equal(r1.canvas_out, r2.canvas_out)
    np.testing.assert_array_equal(r1.hidden[-1], r2.hidden[-1])


def _zero_out_proj(l, t):
    t = dict(t)
    for k in ("wo", "w_down", "ws_down"):
        t[k] = torch.zeros_like(t[k])
    return t


def test_planted_identity_canvas_is_fixed_point():
    """With every output projection zero the residual stream stays E[x]; the
    tied LM head then peaks at x itself, and at a low temperature every
    position is confident, so the step returns its input canvas."""
    w = _tiny(prefix=8)
    o = oracle.for_workload(w, layer_override=_zero_out_proj)
    o.prefill(si.uniform_tokens(w, "prefix", 1, 8).numpy())
    cv = si.uniform_tokens(w, "canvas", 1, 256).numpy()
    r = o.denoise_step(cv, 0, 0, 0.9, temperature=0.01)
    emb = si.weight(w, "embed").to(torch.float64).numpy()
    np.testing.assert_array_equal(r.hidden[-1][0], emb[cv[0]])
    # brute force argmax of <rmsnorm(E[x]), E[v]>
    for i in range(0, 256, 17):
        e = emb[cv[0, i]]
        zz = e / np.sqrt(np.mean(e * e) + 1e-6)
        s = emb @ zz
        assert int(np.argmax(s)) == cv[0, i]
    assert (r.argmax == cv).all()
    assert (r.conf >= 0.9).all()
    np.testing.assert_array_equal(r.canvas_out, cv)


# --- the seeded generator itself ------------------------------------------------
def test_synth_slices_and_moments():
    w = si.workload("tiny")
    full = si.weight(w, "w_gate", 1)
    part = si.weight(w, "w_gate", 1, rows=slice(3, 9))
    assert torch.equal(full[3:9], part)
    x = full.to(torch.float64)
    assert abs(x.mean().item()) < 1e-3
    assert abs(x.std().item() - 0.02) < 5e-4
    wo = si.weight(w, "wo", 0).to(torch.float64)
    assert abs(wo.std().item() - 0.02 / 2) < 5e-4      # 1/sqrt(2*layers) on the tiny model
    t = si.uniform_tokens(w, "canvas", 1, 256)
    assert t.dtype == torch.int32 and int(t.min()) >= 0 and int(t.max()) < 8192


# --- entropy-constrained sampler (codemajin.net section 3.3) -----------------
def test_lm_head_entropy_matches_scipy():
    from scipy.special import softmax
    from scipy.stats import entropy
    z = rng.standard_normal((6, 8))
    E = rng.standard_normal((41, 8))
    st = om.lm_head_stats(z, E, 0.6, row_chunk=4, vocab_chunk=16)
    ref = entropy(softmax(z @ E.T / 0.6, axis=1), axis=1)
    # the oracle forms the entropy as lse - sum p s: when it is much smaller
    # than lse the two terms cancel, leaving an absolute rounding error of a
    # few ulps of lse (|lse| < 10 here), hence the absolute bound
    np.testing.assert_allclose(st["entropy"], ref, rtol=1e-12, atol=1e-12)
    # a one-hot distribution has zero entropy, a uniform one ln V
    st2 = om.lm_head_stats(np.zeros((1, 8)), E, 1.0)
    assert abs(st2["entropy"][0] - math.log(41)) < 1e-12


def test_entropy_accept_is_the_longest_low_entropy_prefix_within_budget():
    r2 = np.random.default_rng(7)
    for trial in range(300):
        n = int(r2.integers(1, 12))
        e = r2.choice([0.1, 0.25, 0.5, 1.0, 2.0], size=n).astype(np.float32)  # many exact ties
        gamma = float(r2.choice([0.0, 0.3, 0.75, 1.5, 100.0]))
        acc = om.entropy_accept(e, gamma)
        # brute force over the (entropy, position) order
        order = sorted(range(n), key=lambda i: (float(e[i]), i))
        k = 1
        while k < n and float(np.sum(e[order[:k + 1]], dtype=np.float64)) <= gamma + 1e-6:
            k += 1
        expect = np.zeros(n, dtype=bool)
        expect[order[:k]] = True
        np.testing.assert_array_equal(acc, expect)
    assert om.entropy_accept(np.array([3.0, 1.0, 1.0], np.float32), 0.0).tolist() == [False, True, False]
    assert om.entropy_accept(np.array([3.0, 1.0, 1.0], np.float32), 1e9).all()


def test_entropy_sample_stop_rule():
    a = np.array([5, 6, 7, 8])
    noise = np.array([100, 101, 102, 103])
    low = np.full(4, 0.01, np.float32)
    # first step of a block: no previous prediction, never stops
    out, stop = om.entropy_sample(a, low, None, 0.0, 1.0, noise)
    assert not stop and out.tolist() == [5, 101, 102, 103]
    # mean entropy below the threshold and argmax unchanged: stop, keep every argmax
    out, stop = om.entropy_sample(a, low, a.copy(), 0.0, 1.0, noise)
    assert stop and out.tolist() == [5, 6, 7, 8]
    # one argmax changed: no stop
    out, stop = om.entropy_sample(a, low, np.array([5, 6, 7, 9]), 0.0, 1.0, noise)
    assert not stop
    # mean entropy at the threshold: no stop (strictly below is required)
    out, stop = om.entropy_sample(a, np.full(4, 0.5, np.float32), a.copy(), 1.0, 0.5, noise)
    assert not stop and out.tolist() == [5, 6, 102, 103]


def test_anneal_temperature_linear_08_to_04():
    assert om.anneal_temperature(0, 48) == 0.8
    assert abs(om.anneal_temperature(47, 48) - 0.4) < 1e-15
    assert abs(om.anneal_temperature(23.5, 48) - 0.6) < 1e-15
    ts = [om.anneal_temperature(s, 48) for s in range(48)]
    assert all(b < a for a, b in zip(ts, ts[1:]))


def test_entropy_step_reuses_forward_and_noise():
    """The entropy step is the threshold step's forward pass plus another
    sampler: same argmax and entropies, re-noised positions take the same
    Philox draws."""
    w = _tiny(prefix=16)
    o = oracle.for_workload(w)
    o.prefill(si.uniform_tokens(w, "prefix", 1, 16).numpy())
    cv = si.uniform_tokens(w, "canvas", 1, 256).numpy()
    r1 = o.denoise_step(cv, 3, 11, 2.0, temperature=0.7)          # tau > 1: every position re-noised
    r2 = o.denoise_step_entropy(cv, 3, 11, 0.7, 0.5, 0.1)
    np.testing.assert_array_equal(r1.argmax, r2.argmax)
    acc = om.entropy_accept(r2.entropy[0].astype(np.float32), 0.5)
    np.testing.assert_array_equal(r2.canvas_out[0][acc], r2.argmax[0][acc])
    np.testing.assert_array_equal(r2.canvas_out[0][~acc], r1.canvas_out[0][~acc])
    assert not r2.stopped[0]


# --- self-conditioning (codemajin.net section 3.2) ----------------------------
def test_self_condition_matches_torch_restatement():
    z = rng.standard_normal((7, 12))
    E = rng.standard_normal((53, 12)) * 0.5
    wg, wu, wd = (rng.standard_normal(s) * 0.3 for s in ((9, 12), (9, 12), (12, 9)))
    got = om.self_condition(z, E, 0.7, wg, wu, wd, row_chunk=3, vocab_chunk=16)
    t = lambda a: torch.tensor(a, dtype=torch.float64)
    e = torch.softmax(t(z) @ t(E).T / 0.7, dim=1) @ t(E)
    ref = (torch.nn.functional.silu(e @ t(wg).T) * (e @ t(wu).T)) @ t(wd).T
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-14)


def test_self_condition_closed_forms():
    E = rng.standard_normal((40, 8))
    wg, wu, wd = (rng.standard_normal(s) for s in ((5, 8), (5, 8), (8, 5)))
    ffn = lambda e: om.swiglu_ffn(e, wg, wu, wd)
    # a flat distribution (z = 0): the mean embedding
    got = om.self_condition(np.zeros((2, 8)), E, 1.0, wg, wu, wd)
    np.testing.assert_allclose(got, ffn(np.tile(E.mean(axis=0), (2, 1))), rtol=1e-12, atol=1e-12)
    # a one-hot distribution (a very sharp temperature): that token's embedding
    z = E[[3, 17]]
    got = om.self_condition(z, E, 1e-6, wg, wu, wd)
    top = np.argmax(z @ E.T, axis=1)
    np.testing.assert_allclose(got, ffn(E[top]), rtol=1e-9, atol=1e-9)


def test_self_conditioned_step_adds_the_signal_to_the_input():
    w = _tiny(prefix=16)
    o = oracle.for_workload(w)
    o.prefill(si.uniform_tokens(w, "prefix", 1, 16).numpy())
    cv = si.uniform_tokens(w, "canvas", 1, 256).numpy()
    scw = si.self_cond_weights(w)
    r0 = o.denoise_step(cv, 0, 1, 0.9, sc_weights=scw)
    assert r0.self_cond.shape == (1, 256, w.shape.d_model)
    r1 = o.denoise_step(cv, 1, 1, 0.9, self_cond_in=r0.self_cond, sc_weights=scw)
    emb = si.weight(w, "embed").to(torch.float64).numpy()
    np.testing.assert_allclose(r1.hidden[0][0], emb[cv[0]] + r0.self_cond[0], rtol=1e-15, atol=0)
    # the signal is the oracle's own function of the step's final normalised rows
    z = om.rms_norm(r0.hidden[-1][0], o.final_norm, w.shape.rms_eps)
    np.testing.assert_allclose(r0.self_cond[0], om.self_condition(z, o.embed, 1.0, scw["sc_gate"], scw["sc_up"],
                                                                  scw["sc_down"]), rtol=1e-12, atol=1e-14)
