"""Pin of the oracle's step and commit wiring against a second, structurally
different statement of the same model (CPU, float64).

The oracle works the way the pages describe the decoder being used: a causal
encoder fills a per-layer KV cache for the prompt, then the bidirectional
decoder runs the canvas through every layer against that cache (codemajin.net
"DiffusionGemma architecture", section 3.2; aiboss88.com "hybrid attention
architecture").  The restatement here never builds a cache: it pushes the
whole sequence prompt || canvas through the layers in ONE pass with torch
routines (rms_norm, complex-number RoPE, scaled_dot_product_attention with an
explicit [S, S] mask, dense expert mixture), the mask saying which key each
row sees:

  * prompt rows: keys j <= i (causal);
  * canvas rows in the denoising step: every prompt row and every canvas row
    (bidirectional over the block, no mask among canvas rows);
  * canvas rows of a block commit: causal again, which is ordinary causal
    attention over prompt || block.

The two agree only if the oracle's step wiring is right: canvas positions
start at P (RoPE), the canvas keys are the cache rows [0, P) plus the whole
canvas, the step has no causal mask, the residual / norm / routing order is
the stated one, and a commit leaves in the cache exactly the keys/values of a
causal pass over the concatenation.  Plausible mistakes (RoPE from 0, canvas
attending only to itself, a causal mask in the step, a dropped residual) each
break the equality; the last tests plant such mistakes in a copy of the
restatement to show that they do.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth_inputs as si


def _f64(t):
    return t.to(torch.float64)


def _rope_complex(x, positions, base):
    """Rotate pairs (j, j + D/2) of x [H, S, D] as complex numbers z_j = x_j +
    i x_{j+D/2} multiplied by e^{i pos theta_j}, theta_j = base^(-2j/D)."""
    H, S, D = x.shape
    half = D // 2
    theta = base ** (-2.0 * torch.arange(half, dtype=torch.float64) / D)
    ang = positions.to(torch.float64)[:, None] * theta[None, :]
    rot = torch.polar(torch.ones_like(ang), ang)                   # e^{i ang}
    z = torch.complex(x[..., :half], x[..., half:]) * rot[None]
    return torch.cat([z.real, z.imag], dim=-1)


def _sequence_forward(w, weights, tokens, n_prompt, canvas_mode, plant=None):
    """Hidden states of every row of tokens [S] after each layer, and the
    post-RoPE keys/values of every layer, in one pass over the sequence.

    canvas_mode "bidirectional" (denoising step) or "causal" (block commit)
    decides the mask of rows >= n_prompt.  `plant` names a deliberate mistake
    (used only to show that the comparison catches it)."""
    s = w.shape
    d, Hq, Hkv, D = s.d_model, s.n_q_heads, s.n_kv_heads, s.head_dim
    S = tokens.shape[0]
    E = _f64(weights["embed"])
    h = E[tokens.long()]
    i = torch.arange(S)
    mask = i[None, :] <= i[:, None]                                # causal everywhere
    if canvas_mode == "bidirectional" and plant != "causal_step":
        mask[n_prompt:, :] = True                                  # canvas rows see every row
    if plant == "canvas_sees_only_itself":
        mask[n_prompt:, :n_prompt] = False
    positions = i.clone()
    if plant == "rope_from_zero":
        positions[n_prompt:] = torch.arange(S - n_prompt)
    hidden, keys, vals = [h.clone()], [], []
    for l in range(s.n_layers):
        lw = {k: _f64(v) for k, v in weights["layers"][l].items()}
        u = F.rms_norm(h, (d,), lw["attn_norm"], eps=s.rms_eps)
        qkv = u @ lw["wqkv"].T
        q = qkv[:, :Hq * D].reshape(S, Hq, D).transpose(0, 1)
        k = qkv[:, Hq * D:(Hq + Hkv) * D].reshape(S, Hkv, D).transpose(0, 1)
        v = qkv[:, (Hq + Hkv) * D:].reshape(S, Hkv, D).transpose(0, 1)
        q = _rope_complex(q, positions, s.rope_base)
        k = _rope_complex(k, positions, s.rope_base)
        keys.append(k)
        vals.append(v)
        G = Hq // Hkv
        o = F.scaled_dot_product_attention(q[None], k.repeat_interleave(G, 0)[None],
                                           v.repeat_interleave(G, 0)[None], attn_mask=mask[None, None])[0]
        o = o.transpose(0, 1).reshape(S, Hq * D)
        h = h + o @ lw["wo"].T
        u2 = F.rms_norm(h, (d,), lw["ffn_norm"], eps=s.rms_eps)
        r = u2 @ lw["w_router"].T
        if weights.get("router_bias") is not None:
            r = r + _f64(weights["router_bias"])
        top_v, top_i = torch.topk(r, s.top_k, dim=-1)
        mix = torch.zeros_like(r).scatter(1, top_i, torch.softmax(top_v, dim=-1))   # [S, E]
        y = (F.silu(u2 @ lw["ws_gate"].T) * (u2 @ lw["ws_up"].T)) @ lw["ws_down"].T
        for e in range(s.n_experts):
            ye = (F.silu(u2 @ lw["w_gate"][e].T) * (u2 @ lw["w_up"][e].T)) @ lw["w_down"][e].T
            y = y + mix[:, e:e + 1] * ye
        h = h + y if plant != "drop_moe_residual" else y
        hidden.append(h.clone())
    return hidden, keys, vals


def _lm_head(w, weights, h, temperature):
    z = F.rms_norm(h, (w.shape.d_model,), _f64(weights["final_norm"]), eps=w.shape.rms_eps)
    logits = z @ _f64(weights["embed"]).T / temperature
    logp = torch.log_softmax(logits, dim=-1)
    return logits.argmax(-1), logp.max(-1).values, torch.logsumexp(logits, -1)


@pytest.fixture(scope="module")
def setup():
    w = si.workload("tiny").with_(prefix=48)
    weights = si.model_weights(w, "cpu")
    prompt = si.uniform_tokens(w, "prefix", 1, w.prefix)
    canvas = si.uniform_tokens(w, "canvas", 1, w.canvas)
    seq = torch.cat([prompt, canvas], 1)[0]
    orc = oracle.for_workload(w)
    orc.prefill(prompt.numpy())
    r = orc.denoise_step(canvas.numpy(), 0, 1, 0.9, temperature=0.5)
    return w, weights, prompt, canvas, seq, orc, r


def test_step_equals_one_pass_with_block_mask(setup):
    w, weights, prompt, canvas, seq, orc, r = setup
    P = w.prefix
    hidden, _, _ = _sequence_forward(w, weights, seq, P, "bidirectional")
    for l in range(w.shape.n_layers + 1):
        np.testing.assert_allclose(r.hidden[l][0], hidden[l][P:].numpy(), rtol=1e-10, atol=1e-12)
    a, logp, lse = _lm_head(w, weights, hidden[-1][P:], 0.5)
    np.testing.assert_array_equal(r.argmax[0], a.numpy())
    np.testing.assert_allclose(r.logp[0], logp.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(r.lse[0], lse.numpy(), rtol=0, atol=1e-10)


def test_commit_equals_one_causal_pass_over_prompt_and_block(setup):
    """Bidirectional attention restricted by a causal mask is ordinary causal
    attention: the cache rows a block commit appends equal the keys/values of
    a causal pass over prompt || block."""
    w, weights, prompt, canvas, seq, _, _ = setup
    P, C = w.prefix, w.canvas
    orc = oracle.for_workload(w)
    orc.prefill(prompt.numpy())
    orc.commit_block(canvas.numpy())
    _, keys, vals = _sequence_forward(w, weights, seq, P, "causal")
    for l in range(w.shape.n_layers):
        np.testing.assert_allclose(orc.k_cache[l][0], keys[l].numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(orc.v_cache[l][0], vals[l].numpy(), rtol=1e-10, atol=1e-12)
    assert orc.P == P + C


def test_batch_rows_are_independent():
    """Two sequences denoised together give what each gives alone."""
    w = si.workload("tiny").with_(prefix=24, batch=2)
    prompt = si.uniform_tokens(w, "prefix", 2, 24).numpy()
    canvas = si.uniform_tokens(w, "canvas", 2, 256).numpy()
    both = oracle.for_workload(w)
    both.prefill(prompt)
    rb = both.denoise_step(canvas, 3, 9, 0.9)
    for b in range(2):
        # one sequence alone, told its index in the batch (the sampler's counter carries it)
        one = oracle.for_workload(w.with_(batch=1), seq_ids=[b])
        one.prefill(prompt[b:b + 1])
        r1 = one.denoise_step(canvas[b:b + 1], 3, 9, 0.9)
        np.testing.assert_allclose(rb.hidden[-1][b], r1.hidden[-1][0], rtol=1e-12, atol=1e-14)
        np.testing.assert_array_equal(rb.argmax[b], r1.argmax[0])
        np.testing.assert_array_equal(rb.canvas_out[b], r1.canvas_out[0])


def test_teacher_forced_layer_reproduces_free_running_layer(setup):
    """Fed its own hidden states, expert choices, router rows and LM-head rows,
    the teacher-forced mode gives the free-running results back (it changes
    where a layer's inputs come from, not what it computes)."""
    w, weights, prompt, canvas, seq, orc, r = setup
    s = w.shape
    router_rows = []
    for l in range(s.n_layers):
        # the router's input: RMSNorm of the residual after this layer's attention
        lw = orc.layer(l)
        hh, _, _ = orc._layer_forward(l, r.hidden[l][0], 0, orc.P, causal=False, need_ffn=False)
        router_rows.append(oracle.rms_norm(hh, lw["ffn_norm"], s.rms_eps)[None])
    lm_rows = oracle.rms_norm(r.hidden[-1], orc.final_norm, s.rms_eps)
    teacher = {"hidden": r.hidden, "experts": r.experts, "router_rows": router_rows, "lm_rows": lm_rows}
    rf = orc.denoise_step(canvas.numpy(), 0, 1, 0.9, temperature=0.5, teacher=teacher)
    for l in range(s.n_layers + 1):
        np.testing.assert_array_equal(rf.forced_hidden[l], r.hidden[l])
    for l in range(s.n_layers):
        np.testing.assert_array_equal(rf.forced_experts[l], r.experts[l])
        np.testing.assert_allclose(rf.forced_router_margin[l], r.router_margin[l], rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(rf.forced_lm["argmax"], r.argmax)
    np.testing.assert_allclose(rf.forced_lm["lse"], r.lse, rtol=1e-14)
    np.testing.assert_allclose(rf.forced_lm["gap"], r.gap, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("plant", ["rope_from_zero", "canvas_sees_only_itself", "causal_step",
                                   "drop_moe_residual"])
def test_planted_wiring_mistakes_are_caught(setup, plant):
    """Each plausible wiring mistake, planted in the restatement, moves the
    canvas hidden states far beyond the comparison's tolerance."""
    w, weights, prompt, canvas, seq, orc, r = setup
    P = w.prefix
    hidden, _, _ = _sequence_forward(w, weights, seq, P, "bidirectional", plant=plant)
    err = np.abs(r.hidden[-1][0] - hidden[-1][P:].numpy()).max()
    assert err > 1e-4, (plant, err)
