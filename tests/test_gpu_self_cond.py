"""GPU checks of the self-conditioning signal (codemajin.net "DiffusionGemma
architecture", section 3.2) through the C ABI: the signal a step computes
against the oracle's (on the GPU's own LM-head rows, and free-running), the
next step's input being the embedding plus that signal, and graph and eager
launches agreeing."""
import numpy as np
import pytest
import torch

import oracle
from oracle import model as om
import synth_inputs as si

from gpu_helpers import (HIDDEN_REL_L2, compare_step, device_weights_oracle, gpu_step, make_context, oracle_step,
                         rel_l2)

pytestmark = pytest.mark.gpu

SIGNAL_FREE_REL_L2 = 2e-2   # free-running signal (carries the hidden-state drift; see below)


def _sc_context(w, **kw):
    weights = si.model_weights(w, "cuda")
    weights.update(si.self_cond_weights(w, "cuda"))
    ctx, weights = make_context(w, weights=weights, **kw)
    return ctx, weights


def _signal(ctx, w):
    out = torch.empty(w.batch * w.canvas, w.shape.d_model, dtype=torch.float32, device="cuda")
    ctx.debug_self_cond(out)
    ctx.sync()
    return out.cpu().numpy().reshape(w.batch, w.canvas, -1)


@pytest.mark.parametrize("name,layers,temp", [("tiny", None, 1.0), ("tiny", None, 0.3), ("a4b_p2k", 1, 1.0)])
def test_self_conditioned_steps_match_oracle(name, layers, temp):
    w = si.workload(name)
    if layers:
        w = w.with_layers(layers).with_(prefix=256)
    ctx, weights = _sc_context(w, temperature=temp)
    scw = {k: weights[k].cpu() for k in ("sc_gate", "sc_up", "sc_down")}
    orc = device_weights_oracle(w, weights, keep_layers=True)
    prefix = si.uniform_tokens(w, "prefix", 1, w.prefix)
    ctx.prefill(prefix.cuda())
    orc.prefill(prefix.numpy())
    ctx.set_self_conditioning(True)
    canvas = si.uniform_tokens(w, "canvas", 1, w.canvas).numpy()
    # both sides take the same inputs every step: the canvas from the oracle,
    # the previous step's signal from the GPU (checked at that step)
    sc_prev = None
    for step in range(2):
        g = gpu_step(ctx, w, canvas, step, 5, 0.9, capture=True)
        sig = _signal(ctx, w)
        r = orc.denoise_step(canvas, step, 5, 0.9, temperature=temp,
                             self_cond_in=None if sc_prev is None else sc_prev.astype(np.float64), sc_weights=scw,
                             teacher={"hidden": g["hidden"], "experts": g["experts"],
                                      "router_rows": g["norm_rows"][:-1], "lm_rows": g["norm_rows"][-1]})
        # the step's input: embedding (+ the previous step's signal)
        emb = weights["embed"][torch.as_tensor(canvas[0]).long().cuda()].float().cpu().numpy()
        expect0 = emb if sc_prev is None else emb + sc_prev[0]
        np.testing.assert_allclose(g["hidden"][0][0], expect0, rtol=1e-6, atol=1e-6)
        res = compare_step(g, r, 0.9, orc=orc, temperature=temp)
        assert res["forced_hidden_rel_l2_max"] <= HIDDEN_REL_L2
        # the signal on the GPU's own LM-head rows (teacher-forced)
        forced = om.self_condition(g["norm_rows"][-1][0], orc.embed, temp, scw["sc_gate"], scw["sc_up"],
                                   scw["sc_down"])
        err_forced = rel_l2(sig[0], forced)
        # and free-running, on the tokens whose routing did not leave the oracle's.
        # The signal is a weighted mean of embeddings minus nearly all of its
        # mean, so its relative error amplifies the LM-head input drift: the
        # oracle's own signal moves by `propagated` between its rows and the
        # GPU's.  The kernel is held to 1e-2 teacher-forced; the free-running
        # signal, which carries that drift, to 2e-2.
        keep = ~res["diverged"][0]
        err_free = rel_l2(sig[0][keep], r.self_cond[0][keep])
        propagated = rel_l2(forced[keep], r.self_cond[0][keep])
        print(name, temp, "step", step, "signal rel-L2 forced", err_forced, "free", err_free,
              "drift-propagated", propagated, "tokens left out", int((~keep).sum()))
        assert err_forced <= HIDDEN_REL_L2
        assert err_free <= SIGNAL_FREE_REL_L2
        sc_prev = sig
        canvas = r.canvas_out
    ctx.close()


def test_self_conditioning_graph_matches_eager_and_resets():
    """Graph replay with the signal rebound per call gives the eager bits; a
    block commit or prefill starts the next canvas without a signal."""
    w = si.workload("small").with_(prefix=256)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        ctx, _ = _sc_context(w, temperature=0.5, stream=s.cuda_stream)
        ctx.prefill(si.uniform_tokens(w, "prefix", 1, 256, device="cuda"))
        ctx.set_self_conditioning(True)
        canvas = si.uniform_tokens(w, "canvas", 1, 256, device="cuda")

        def run(step, eager):
            out = torch.empty_like(canvas)
            conf = torch.empty(1, 256, dtype=torch.float32, device="cuda")
            if eager:
                ctx.debug_profile(["other"])
            ctx.denoise_step(canvas, step, 3, 0.9, out, conf)
            if eager:
                ctx.debug_profile([])
            ctx.sync()
            return out.cpu(), conf.cpu(), torch.as_tensor(_signal(ctx, w))

        # graph and eager from the same signal state: two chains of three steps
        chains = []
        for eager in (False, True):
            ctx.prefill(si.uniform_tokens(w, "prefix", 1, 256, device="cuda"))
            chains.append([run(st, eager) for st in range(3)])
        for a, b in zip(*chains):
            for x, y in zip(a, b):
                assert torch.equal(x, y)
        # the signal changes the next step (it is not ignored) ...
        assert not torch.equal(chains[0][0][1], chains[0][1][1])
        # ... and a commit starts the next block without it: same as a fresh prefill of prefix||block
        ctx.commit_block(canvas)
        first_after_commit = run(0, False)
        ctx.prefill(torch.cat([si.uniform_tokens(w, "prefix", 1, 256, device="cuda"), canvas], 1))
        first_after_prefill = run(0, False)
        assert torch.equal(first_after_commit[1], first_after_prefill[1]) or \
            (first_after_commit[1] - first_after_prefill[1]).abs().max() < 1e-3
        ctx.close()
