"""GPU checks of the entropy-constrained sampler (codemajin.net "DiffusionGemma
architecture", section 3.3) through the C ABI: the decision alone on given
float32 tensors (bit-exact), the step against the oracle, graph and eager
launches agreeing while the temperature changes from call to call, and the
adaptive stop on the planted closed form."""
import numpy as np
import pytest
import torch

import oracle
from oracle import model as om
import synth_inputs as si

from gpu_helpers import device_weights_oracle, make_context, rel_l2

pytestmark = pytest.mark.gpu

ENTROPY_ABS = 5e-2   # entropy (nats) of the GPU's LM head against the oracle's


def _zero_out(l, t):
    t = dict(t)
    for k in ("wo", "w_down", "ws_down"):
        t[k] = torch.zeros_like(t[k])
    return t


def test_entropy_sampler_decision_bit_exact():
    w = si.workload("tiny").with_(batch=3)
    ctx, _ = make_context(w)
    ctx.prefill(si.uniform_tokens(w, "prefix", 3, 16).cuda())
    C, V = w.canvas, w.shape.vocab
    g = torch.Generator().manual_seed(3)
    am = torch.randint(0, V, (3, C), generator=g, dtype=torch.int32)
    ent = (torch.rand(3, C, generator=g) * 2.0).to(torch.float32)
    ent[:, ::7] = 0.5                                   # exact ties
    ent[2] = 0.001                                      # a calm canvas
    prev = am.clone()
    prev[1, 17] += 1                                    # sequence 1: one argmax changed
    seed = 0x0123456789ABCDEF
    for gamma, stop, use_prev in ((3.0, 0.01, False), (0.0, 0.01, True), (50.0, 0.1, True), (1e9, 0.0, True)):
        out = torch.empty(3, C, dtype=torch.int32, device="cuda")
        stopped = torch.empty(3, dtype=torch.int32, device="cuda")
        ctx.debug_entropy_sample(am.cuda(), ent.cuda(), prev.cuda() if use_prev else None, 3, 5, seed, gamma,
                                 stop, out, stopped)
        ctx.sync()
        for b in range(3):
            noise = om.renoise_tokens(np.arange(16, 16 + C), 5, b, seed, V)
            ref, st = om.entropy_sample(am[b].numpy(), ent[b].numpy(), prev[b].numpy() if use_prev else None,
                                        gamma, stop, noise)
            np.testing.assert_array_equal(out[b].cpu().numpy(), ref)
            assert int(stopped[b]) == int(st), (gamma, stop, use_prev, b)
    ctx.close()


def _entropy_step(ctx, w, canvas, step, seed, temp, gamma, stop, prev=None, lm_rows=None):
    """One entropy step; with lm_rows (a list) the step is recorded and the
    bf16 rows its LM head consumed are appended to it."""
    B, C = canvas.shape
    if lm_rows is not None:
        ctx.debug_capture(True)
    cin = torch.as_tensor(canvas, dtype=torch.int32).cuda()
    out = torch.empty_like(cin)
    ent = torch.empty(B, C, dtype=torch.float32, device="cuda")
    am = torch.empty(B, C, dtype=torch.int32, device="cuda")
    stopped = torch.empty(B, dtype=torch.int32, device="cuda")
    ctx.denoise_step_entropy(cin, step, seed, temp, gamma, stop, out,
                             prev_argmax=None if prev is None else torch.as_tensor(prev).cuda(),
                             argmax_out=am, entropy=ent, stopped=stopped)
    if lm_rows is not None:
        z = torch.empty(B * C, w.shape.d_model, dtype=torch.bfloat16, device="cuda")
        ctx.debug_norm_rows(w.shape.n_layers, z)
        ctx.sync()
        lm_rows.append(z.cpu().to(torch.float64).numpy().reshape(B, C, -1))
        ctx.debug_capture(False)
    ctx.sync()
    return out.cpu().numpy(), ent.cpu().numpy(), am.cpu().numpy(), stopped.cpu().numpy()


@pytest.mark.parametrize("name,layers", [("tiny", None), ("a4b_p2k", 1)])
def test_entropy_step_matches_oracle(name, layers):
    """Entropies of the GPU's LM head against the oracle's (free-running); the
    decisions re-taken by the oracle on the GPU's own float32 entropies and
    argmax: identical tokens; the argmax of the oracle's LM head on the GPU's
    own LM-head rows: identical outside the rounding band.  Temperatures from
    the 0.8 -> 0.4 schedule."""
    w = si.workload(name)
    if layers:
        w = w.with_layers(layers).with_(prefix=256)
    ctx, weights = make_context(w)
    orc = device_weights_oracle(w, weights, keep_layers=True)
    prefix = si.uniform_tokens(w, "prefix", 1, w.prefix)
    ctx.prefill(prefix.cuda())
    orc.prefill(prefix.numpy())
    canvas = si.uniform_tokens(w, "canvas", 1, w.canvas).numpy()
    prev = None
    for step in (0, 30):
        temp = om.anneal_temperature(step, 48)
        gamma, stop = 40.0, 0.5
        rows = []
        out, ent, am, stopped = _entropy_step(ctx, w, canvas, step, 9, temp, gamma, stop, prev, lm_rows=rows)
        r = orc.denoise_step_entropy(canvas, step, 9, temp, gamma, stop, prev_argmax=prev, record=False)
        err = np.abs(ent.astype(np.float64) - r.entropy).max()
        print(name, "step", step, "T", temp, "entropy max abs err", err, "mean", ent.mean())
        assert err <= ENTROPY_ABS
        # the same decision on the GPU's own statistics
        noise = om.renoise_tokens(np.arange(w.prefix, w.prefix + w.canvas), step, 0, 9, w.shape.vocab)
        ref, st = om.entropy_sample(am[0], ent[0], None if prev is None else prev[0], gamma, stop, noise)
        np.testing.assert_array_equal(out[0], ref)
        assert int(stopped[0]) == int(st)
        # argmax against the oracle's LM head on the same rows, outside the rounding band
        f = om.lm_head_stats(rows[0][0], orc.embed, temp)
        clear = f["gap"] > 1e-3 / temp
        assert clear.sum() > 200
        np.testing.assert_array_equal(am[0][clear], f["argmax"][clear])
        assert np.abs(ent[0].astype(np.float64) - f["entropy"]).max() < 1e-3
        prev = am
    ctx.close()


def test_entropy_graph_matches_eager_across_temperatures():
    w = si.workload("small").with_(prefix=256)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        ctx, _ = make_context(w, stream=s.cuda_stream)
        ctx.prefill(si.uniform_tokens(w, "prefix", 1, 256, device="cuda"))
        canvas = si.uniform_tokens(w, "canvas", 1, 256).numpy()

        def run(step, temp, eager, prev=None):
            if eager:
                ctx.debug_profile(["other"])
            res = _entropy_step(ctx, w, canvas, step, 4, temp, 25.0, 0.2, prev)
            if eager:
                ctx.debug_profile([])
            return res

        prev = None
        for step in range(4):
            temp = om.anneal_temperature(step * 15, 48)
            g = run(step, temp, False, prev)
            e = run(step, temp, True, prev)
            for a, b in zip(g, e):
                np.testing.assert_array_equal(a, b)
            prev = g[2]
        ctx.close()


def test_entropy_adaptive_stop_planted_identity():
    """With every output projection zero the LM head peaks at the input token
    with entropy ~0: the first step accepts everything within the budget and
    keeps the canvas; the second, seeing the same argmax and a mean entropy
    below the threshold, stops."""
    w = si.workload("tiny").with_(prefix=32, batch=2)
    ctx, _ = make_context(w, layer_override=_zero_out)
    ctx.prefill(si.uniform_tokens(w, "prefix", 2, 32).cuda())
    canvas = si.uniform_tokens(w, "canvas", 2, 256).numpy()
    out, ent, am, stopped = _entropy_step(ctx, w, canvas, 0, 1, 0.1, 1.0, 0.05)
    np.testing.assert_array_equal(am, canvas)
    np.testing.assert_array_equal(out, canvas)
    assert (stopped == 0).all()
    assert ent.mean() < 1e-3
    out2, ent2, am2, stopped2 = _entropy_step(ctx, w, out, 1, 1, 0.1, 1.0, 0.05, prev=am)
    assert (stopped2 == 1).all()
    np.testing.assert_array_equal(out2, canvas)
    ctx.close()


def test_block_ar_loop_with_entropy_sampler_stops_early():
    """The block-AR driver with the entropy sampler and the 0.8 -> 0.4
    temperature schedule: on the planted closed form at the 26B-A4B shapes
    (depth 1, where the identity's logit gap is ~50 so T = 0.8 is still
    sharp) every block is accepted whole at its first step and stopped at its
    second."""
    import block_discrete_diffusion_denoise_b200 as dgp
    w = si.workload("a4b_blockar_b8").with_layers(1).with_(prefix=32, batch=2, blocks=3)
    ctx, _ = make_context(w, layer_override=_zero_out)
    init = lambda k: si.uniform_tokens(w, "canvas", 2, 256, block=k, device="cuda")
    out = dgp.generate_blocks(ctx, si.uniform_tokens(w, "prefix", 2, 32, device="cuda"), init, n_blocks=3,
                              max_steps=48, tau=None, seed=3,
                              entropy={"gamma": 1.0, "stop_entropy": 0.05})
    assert out["steps"] == [2, 2, 2] and out["settled"] == [True] * 3
    for k in range(3):
        assert torch.equal(out["blocks"][k].cpu(), init(k).cpu())
    assert ctx.cached_len == 32 + 2 * 256
    ctx.close()
