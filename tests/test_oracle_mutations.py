"""The oracle's pins bite: each plausible mistake below (a dropped term, a
wrong sign, index, exponent or comparison, a transposed or swapped operand)
is planted in the oracle on the CPU, and at least one pin of
test_oracle_pins.py / test_oracle_mx.py must then fail with an assertion.
Mistakes in the step's wiring (which keys a canvas row sees, where RoPE
positions start) are planted in the oracle too and must break its agreement
with the one-pass restatement of test_oracle_step_wiring.py.  The mutants are
test code; the oracle itself is restored after each case."""
import numpy as np
import pytest

import test_oracle_mx as mxpins
import test_oracle_pins as pins
from oracle import model as om
from oracle import mx


# --- mutants: (module, attribute, replacement built from the original) -------
def _rms_eps_outside(orig):
    return lambda h, g, eps: h / (np.sqrt(np.mean(h * h, axis=-1, keepdims=True)) + eps) * g


def _rms_sum(orig):
    return lambda h, g, eps: h / np.sqrt(np.sum(h * h, axis=-1, keepdims=True) + eps) * g


def _rms_no_gain(orig):
    return lambda h, g, eps: h / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + eps)


def _silu_sign(orig):
    return lambda x: x / (1.0 + np.exp(x))


def _rope_half_exponent(orig):
    def f(positions, head_dim, base):
        j = np.arange(head_dim // 2, dtype=np.float64)
        ang = np.asarray(positions, dtype=np.float64)[:, None] * (base ** (-j / head_dim))[None, :]
        return np.cos(ang), np.sin(ang)
    return f


def _rope_backwards(orig):
    def f(x, cos, sin):
        half = x.shape[-1] // 2
        x1, x2 = x[..., :half], x[..., half:]
        return np.concatenate([x1 * cos + x2 * sin, x2 * cos - x1 * sin], axis=-1)
    return f


def _rope_interleaved(orig):
    def f(x, cos, sin):
        x1, x2 = x[..., 0::2], x[..., 1::2]
        out = np.empty_like(x)
        out[..., 0::2] = x1 * cos - x2 * sin
        out[..., 1::2] = x2 * cos + x1 * sin
        return out
    return f


def _attention_variant(scale=True, kv_head=lambda h, group, Hkv: h // group, extra_key=0):
    def mutant(orig):
        def f(q, k, v, key_limit):
            Hq, n, D = q.shape
            Hkv, S, _ = k.shape
            group = Hq // Hkv
            visible = np.arange(S)[None, :] < np.asarray(key_limit)[:, None] + extra_key
            out = np.empty((n, Hq, D))
            for h in range(Hq):
                g = kv_head(h, group, Hkv)
                s = q[h] @ k[g].T / (np.sqrt(D) if scale else 1.0)
                s = np.where(visible, s, -np.inf)
                p = np.exp(s - s.max(axis=1, keepdims=True))
                out[:, h, :] = (p / p.sum(axis=1, keepdims=True)) @ v[g]
            return out.reshape(n, Hq * D)
        return f
    return mutant


def _topk_ties_high(orig):
    def f(logits, k):
        n, E = logits.shape
        idx = np.array([sorted(range(E), key=lambda e: (-logits[i, e], -e))[:k] for i in range(n)], dtype=np.int64)
        return idx, om.selected_gates(logits, idx)
    return f


def _gates_over_all_experts(orig):
    def f(logits, idx):
        p = np.exp(logits - logits.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        return np.take_along_axis(p, np.asarray(idx, dtype=np.int64), axis=1)
    return f


def _moe_without_shared(orig):
    def f(u, lw, idx, gates):
        return orig(u, lw, idx, gates) - om.swiglu_ffn(u, lw["ws_gate"], lw["ws_up"], lw["ws_down"])
    return f


def _moe_ungated(orig):
    return lambda u, lw, idx, gates: orig(u, lw, idx, np.ones_like(gates))


def _swiglu_swapped(orig):
    return lambda x, wg, wu, wd: (om.silu(x @ wu.T) * (x @ wg.T)) @ wd.T


def _lm_head_no_temperature(orig):
    return lambda z, embed, temperature, **kw: orig(z, embed, 1.0, **kw)


def _lm_head_last_argmax(orig):
    def f(z, embed, temperature, **kw):
        r = orig(z, embed, temperature, **kw)
        s = z @ np.asarray(embed, dtype=np.float64).T / temperature
        r["argmax"] = s.shape[1] - 1 - np.argmax(s[:, ::-1], axis=1)
        return r
    return f


def _lm_head_entropy_sign(orig):
    def f(z, embed, temperature, **kw):
        r = orig(z, embed, temperature, **kw)
        r["entropy"] = 2 * r["lse"] - r["entropy"]          # lse + sum p s instead of lse - sum p s
        return r
    return f


def _sample_strict(orig):
    return lambda argmax, conf, tau, noise: np.where(np.asarray(conf) > tau, argmax, noise)


def _sample_keeps_nan(orig):
    return lambda argmax, conf, tau, noise: np.where(~(np.asarray(conf) < tau), argmax, noise)


def _renoise_without_step(orig):
    return lambda positions, step, seq_ids, seed, vocab: orig(positions, 0, seq_ids, seed, vocab)


def _accept_strict_budget(orig):
    def f(entropy, gamma):
        e = np.asarray(entropy, dtype=np.float32)
        order = sorted(range(len(e)), key=lambda i: (e[i], i))
        acc = np.zeros(len(e), dtype=bool)
        run = np.float32(0.0)
        for rank, i in enumerate(order):
            run = np.float32(run + e[i])
            if rank > 0 and not (run < np.float32(gamma)):
                break
            acc[i] = True
        return acc
    return f


def _accept_first_not_forced(orig):
    def f(entropy, gamma):
        acc = orig(entropy, gamma)
        e = np.asarray(entropy, dtype=np.float32)
        first = min(range(len(e)), key=lambda i: (e[i], i))
        if e[first] > np.float32(gamma):
            acc[first] = False
        return acc
    return f


def _stop_at_threshold(orig):
    def f(argmax, entropy, prev_argmax, gamma, stop_entropy, noise):
        if prev_argmax is not None and om.mean_entropy(entropy) <= np.float32(stop_entropy) and \
                np.array_equal(argmax, prev_argmax):
            return np.asarray(argmax).copy(), True
        return np.where(om.entropy_accept(entropy, gamma), argmax, noise), False
    return f


def _stop_without_argmax_check(orig):
    def f(argmax, entropy, prev_argmax, gamma, stop_entropy, noise):
        if prev_argmax is not None and om.mean_entropy(entropy) < np.float32(stop_entropy):
            return np.asarray(argmax).copy(), True
        return np.where(om.entropy_accept(entropy, gamma), argmax, noise), False
    return f


def _anneal_over_max_steps(orig):
    return lambda step, max_steps=48, t_first=0.8, t_last=0.4: t_first + (t_last - t_first) * step / max_steps


def _tpf_without_commits(orig):
    return lambda total_tokens, total_steps, n_blocks: total_tokens / total_steps


def _self_cond_no_temperature(orig):
    return lambda z, embed, temperature, *a, **kw: orig(z, embed, 1.0, *a, **kw)


def _self_cond_argmax_embedding(orig):
    def f(z, embed, temperature, sc_gate, sc_up, sc_down, **kw):
        E = np.asarray(embed, dtype=np.float64)
        return om.swiglu_ffn(E[np.argmax(z @ E.T, axis=1)], sc_gate, sc_up, sc_down)
    return f


def _philox_nine_rounds(orig):
    def f(c0, c1, c2, c3, k0, k1):
        M = 0xFFFFFFFF
        c = [c0, c1, c2, c3]
        k = [k0, k1]
        for r in range(9):
            if r:
                k = [(k[0] + 0x9E3779B9) & M, (k[1] + 0xBB67AE85) & M]
            p0, p1 = 0xD2511F53 * c[0], 0xCD9E8D57 * c[2]
            c = [((p1 >> 32) ^ c[1] ^ k[0]) & M, p1 & M, ((p0 >> 32) ^ c[3] ^ k[1]) & M, p0 & M]
        return c
    return f


def _uniform_shift_off(orig):
    def f(w, vocab):
        w = np.asarray(w, dtype=np.uint64)
        if vocab & (vocab - 1) == 0:
            return (w & np.uint64(vocab - 1)).astype(np.int64)
        return ((w * np.uint64(vocab)) >> np.uint64(31)).astype(np.int64)
    return f


def _e4m3_ties_away(orig):
    def f(x):
        x = np.asarray(x, dtype=np.float64)
        a = np.abs(x)
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
        step = np.where(a >= mx.E4M3_MIN_NORMAL, 2.0 ** (np.minimum(e, mx.E4M3_EMAX) - 3), mx.E4M3_SUB_STEP)
        q = np.minimum(np.floor(a / step + 0.5) * step, mx.E4M3_MAX)
        return np.copysign(q, x)
    return f


def _e4m3_no_saturation(orig):
    def f(x):
        x = np.asarray(x, dtype=np.float64)
        big = np.abs(x) > mx.E4M3_MAX
        return np.where(big, x, orig(np.where(big, 0.0, x)))
    return f


def _mx_activations_unquantised(orig):
    return lambda x, w: np.asarray(x, dtype=np.float64) @ mx.mx_round_trip(w).T


def _mx_exponent_off_by_one(orig):
    return lambda x, block=mx.MX_BLOCK: orig(x, block) + 1


MUTANTS = {
    "rms_norm: eps outside the root": (om, "rms_norm", _rms_eps_outside, [pins.test_rms_norm_matches_torch_and_has_unit_rms]),
    "rms_norm: sum instead of mean": (om, "rms_norm", _rms_sum, [pins.test_rms_norm_matches_torch_and_has_unit_rms]),
    "rms_norm: gain dropped": (om, "rms_norm", _rms_no_gain, [pins.test_rms_norm_matches_torch_and_has_unit_rms]),
    "silu: exponent sign": (om, "silu", _silu_sign, [pins.test_silu_matches_torch]),
    "rope: base^(-j/D)": (om, "rope_angles", _rope_half_exponent, [pins.test_rope_equals_complex_rotation]),
    "rope: rotation backwards": (om, "apply_rope", _rope_backwards, [pins.test_rope_equals_complex_rotation]),
    "rope: interleaved pairs": (om, "apply_rope", _rope_interleaved, [pins.test_rope_equals_complex_rotation]),
    "attention: no 1/sqrt(D)": (om, "attention", _attention_variant(scale=False),
                                [pins.test_attention_bidirectional_no_cache_is_full_sdpa]),
    "attention: kv head h mod Hkv": (om, "attention", _attention_variant(kv_head=lambda h, g, Hkv: h % Hkv),
                                     [lambda: pins.test_attention_causal_reduces_to_sdpa(8, 2)]),
    "attention: one key too many": (om, "attention", _attention_variant(extra_key=1),
                                    [lambda: pins.test_attention_causal_reduces_to_sdpa(4, 2)]),
    "router: ties to the higher index": (om, "route_top_k", _topk_ties_high, [pins.test_route_top_k_brute_force_and_ties]),
    "router: gates over all experts": (om, "selected_gates", _gates_over_all_experts,
                                       [pins.test_route_top_k_brute_force_and_ties]),
    "moe: shared expert dropped": (om, "moe", _moe_without_shared, [pins.test_moe_all_experts_is_dense_softmax_mixture]),
    "moe: gates ignored": (om, "moe", _moe_ungated, [pins.test_moe_all_experts_is_dense_softmax_mixture]),
    "swiglu: SiLU on the up projection": (om, "swiglu_ffn", _swiglu_swapped,
                                          [pins.test_moe_all_experts_is_dense_softmax_mixture]),
    "lm head: temperature dropped": (om, "lm_head_stats", _lm_head_no_temperature,
                                     [pins.test_lm_head_stats_match_logsumexp_and_ties]),
    "lm head: last index of the maximum": (om, "lm_head_stats", _lm_head_last_argmax,
                                           [pins.test_lm_head_stats_match_logsumexp_and_ties]),
    "lm head: entropy sign": (om, "lm_head_stats", _lm_head_entropy_sign, [pins.test_lm_head_entropy_matches_scipy]),
    "sampler: conf == tau re-noised": (om, "sample", _sample_strict, [pins.test_sampler_keeps_confident_positions]),
    "sampler: NaN kept": (om, "sample", _sample_keeps_nan, [pins.test_sampler_keeps_confident_positions]),
    "re-noise: step not in the counter": (om, "renoise_tokens", _renoise_without_step,
                                          [pins.test_sampler_keeps_confident_positions]),
    "entropy accept: budget strict": (om, "entropy_accept", _accept_strict_budget,
                                      [pins.test_entropy_accept_is_the_longest_low_entropy_prefix_within_budget]),
    "entropy accept: first not forced": (om, "entropy_accept", _accept_first_not_forced,
                                         [pins.test_entropy_accept_is_the_longest_low_entropy_prefix_within_budget]),
    "stop rule: mean at the threshold stops": (om, "entropy_sample", _stop_at_threshold,
                                               [pins.test_entropy_sample_stop_rule]),
    "stop rule: argmax check dropped": (om, "entropy_sample", _stop_without_argmax_check,
                                        [pins.test_entropy_sample_stop_rule]),
    "temperature: / max_steps": (om, "anneal_temperature", _anneal_over_max_steps,
                                 [pins.test_anneal_temperature_linear_08_to_04]),
    "tpf: commit forwards dropped": (om, "tokens_per_forward", _tpf_without_commits, [pins.test_tpf_tps_definitions]),
    "self-conditioning: temperature dropped": (om, "self_condition", _self_cond_no_temperature,
                                               [pins.test_self_condition_matches_torch_restatement]),
    "self-conditioning: argmax embedding for p E": (om, "self_condition", _self_cond_argmax_embedding,
                                                    [pins.test_self_condition_closed_forms]),
    "philox: nine rounds": (pins, "philox4x32_10", _philox_nine_rounds, [pins.test_philox_known_answers]),
    "uniform token: shift by 31": (pins, "uniform_token", _uniform_shift_off,
                                   [pins.test_uniform_token_power_of_two_is_exact_mask]),
    "e4m3: ties away from zero": (mx, "e4m3_round", _e4m3_ties_away,
                                  [mxpins.test_e4m3_saturation_and_subnormal_ties]),
    "e4m3: no saturation": (mx, "e4m3_round", _e4m3_no_saturation, [mxpins.test_e4m3_saturation_and_subnormal_ties]),
    "mx: block exponent off by one": (mx, "mx_block_exponents", _mx_exponent_off_by_one,
                                      [mxpins.test_block_exponent_closed_forms]),
    "mx: activations left unquantised": (mx, "mx_linear", _mx_activations_unquantised,
                                         [mxpins.test_mx_linear_worked_example_by_hand]),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name, monkeypatch):
    module, attr, make, checks = MUTANTS[name]
    monkeypatch.setattr(module, attr, make(getattr(module, attr)))
    caught = 0
    for check in checks:
        try:
            check()
        except AssertionError:
            caught += 1
    assert caught, f"no pin fails when the oracle has: {name}"


def test_unmutated_pins_pass():
    """The same pin calls pass on the oracle as it is (so a failure above is
    the mutant's doing)."""
    for module, attr, make, checks in MUTANTS.values():
        for check in checks:
            check()


# --- wiring mistakes planted in the oracle's step, caught by the one-pass ----
# restatement of test_oracle_step_wiring.py (computed once, unmutated)
def _step_attention(transform):
    """attention() wrapper applying `transform` only to step-mode calls (every
    row sees the same number of keys: the cache plus the whole canvas)."""
    def mutant(orig):
        def f(q, k, v, key_limit):
            lim = np.asarray(key_limit)
            if lim.size > 1 and (lim == lim[0]).all():
                q, k, v, lim = transform(q, k, v, lim)
            return orig(q, k, v, lim)
        return f
    return mutant


def _causal_canvas(q, k, v, lim):
    n = q.shape[1]
    return q, k, v, lim[0] - n + 1 + np.arange(n)


def _canvas_only(q, k, v, lim):
    n = q.shape[1]
    return q, k[:, -n:], v[:, -n:], np.full(n, n)


def _cache_only(q, k, v, lim):
    n = q.shape[1]
    S = k.shape[1]
    return q, k[:, :S - n], v[:, :S - n], np.full(n, S - n)


def _rope_from_zero(orig):
    return lambda positions, head_dim, base: orig(np.asarray(positions) - np.min(positions), head_dim, base)


WIRING_MUTANTS = {
    "step: causal among canvas rows": (om, "attention", _step_attention(_causal_canvas)),
    "step: canvas sees only itself": (om, "attention", _step_attention(_canvas_only)),
    "step: canvas sees only the cache": (om, "attention", _step_attention(_cache_only)),
    "RoPE positions restart at 0 in every call": (om, "rope_angles", _rope_from_zero),
}


@pytest.fixture(scope="module")
def one_pass():
    import synth_inputs as si
    import test_oracle_step_wiring as wiring
    import torch
    w = si.workload("tiny").with_(prefix=48)
    weights = si.model_weights(w, "cpu")
    prompt = si.uniform_tokens(w, "prefix", 1, w.prefix)
    canvas = si.uniform_tokens(w, "canvas", 1, w.canvas)
    hidden, _, _ = wiring._sequence_forward(w, weights, torch.cat([prompt, canvas], 1)[0], w.prefix,
                                            "bidirectional")
    return w, prompt.numpy(), canvas.numpy(), [h[w.prefix:].numpy() for h in hidden]


def _step_matches_one_pass(w, prompt, canvas, hidden):
    import oracle
    orc = oracle.for_workload(w)
    orc.prefill(prompt)
    r = orc.denoise_step(canvas, 0, 1, 0.9, temperature=0.5)
    for l in range(w.shape.n_layers + 1):
        np.testing.assert_allclose(r.hidden[l][0], hidden[l], rtol=1e-10, atol=1e-12)


def test_unmutated_step_matches_one_pass(one_pass):
    _step_matches_one_pass(*one_pass)


@pytest.mark.parametrize("name", sorted(WIRING_MUTANTS))
def test_planted_wiring_mistake_in_the_oracle_fails(name, one_pass, monkeypatch):
    module, attr, make = WIRING_MUTANTS[name]
    monkeypatch.setattr(module, attr, make(getattr(module, attr)))
    with pytest.raises(AssertionError):
        _step_matches_one_pass(*one_pass)
