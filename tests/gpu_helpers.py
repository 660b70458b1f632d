"""Shared helpers of the GPU parity tests: build a context for a workload and
compare the CUDA path with the oracle under the stated criteria."""
from __future__ import annotations

import numpy as np
import torch

import block_discrete_diffusion_denoise_b200 as dgp
import oracle
import synth_inputs as si

# Acceptance criteria of the denoising step (GPU vs oracle):
HIDDEN_REL_L2 = 1e-2     # residual stream after every layer, relative L2
LOGP_ABS = 5e-2          # per-position log-probability of the argmax (and log-sum-exp)
EXCLUDE_BAND = 1e-3      # positions with top1-top2 margin or |conf - tau| below this are exempt
# Decisions re-taken by the oracle on the very operands the kernels consumed
# (teacher-forced): the two sides then differ only by fp32 accumulation order,
# far below these bands, so every decision outside them must agree.
ROUTER_GAP_BAND = 1e-3   # k-th minus (k+1)-th router logit
LM_GAP_BAND = 1e-3       # top-1 minus top-2 logit at T = 1 (scaled by 1/T)


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def make_context(w: si.Workload, temperature: float = 1.0, layer_override=None, max_seq: int | None = None,
                 prefill_rows: int = 0, weights=None, stream=None):
    if weights is None:
        weights = si.model_weights(w, "cuda", layer_override)
    if max_seq is None:
        max_seq = w.prefix + w.canvas * (w.blocks + 1)
    cfg = dgp.config_from_shape(w.shape, max_batch=w.batch, max_seq=max_seq, canvas=w.canvas,
                                temperature=temperature, prefill_rows=prefill_rows)
    return dgp.Context(cfg, weights, stream=stream), weights


def device_weights_oracle(w: si.Workload, weights: dict, keep_layers: bool = False, seqs=None):
    """Oracle over the seeded weights that already sit on the GPU: each layer
    is copied to the host when the oracle needs it (generating the 26B-shaped
    model on the CPU takes minutes per layer).  The generator gives the same
    bits on CPU and GPU; every copy is also checked here against a slice
    regenerated on the CPU, so the oracle reads the generator's values and
    nothing the kernels may have written.  seqs selects sequences of a batch
    (the oracle's sequences are independent of one another)."""
    rng = np.random.default_rng(0)

    def check(name, l, t):
        r0 = int(rng.integers(0, t.shape[0]))
        ref = si.weight(w, name, l, "cpu", rows=slice(r0, r0 + 1))
        assert torch.equal(t[r0:r0 + 1], ref), f"device copy of {name} (layer {l}) differs from the generator"

    def layer_fn(l):
        t = {k: v.cpu() for k, v in weights["layers"][l].items()}
        for name in ("wqkv", "wo", "w_router", "w_gate", "w_down", "ws_up"):
            check(name, l, t[name])
        return t

    embed = weights["embed"].cpu()
    check("embed", None, embed)
    rb = weights.get("router_bias")
    batch = w.batch if seqs is None else len(seqs)
    return oracle.Oracle(oracle.shape_of(w), layer_fn, embed, weights["final_norm"].cpu(),
                         None if rb is None else rb.cpu(), batch=batch, keep_layers=keep_layers,
                         seq_ids=seqs)


def gpu_step(ctx, w, canvas, step, seed, tau, capture=False):
    """Run one step; return dict of host arrays (and per-layer capture)."""
    B, C = canvas.shape
    cin = torch.as_tensor(canvas, dtype=torch.int32).cuda()
    cout = torch.empty_like(cin)
    conf = torch.empty(B, C, dtype=torch.float32, device="cuda")
    settled = torch.empty(B, dtype=torch.int32, device="cuda")
    if capture:
        ctx.debug_capture(True)
    ctx.denoise_step(cin, step, seed, tau, cout, conf, settled)
    res = {}
    T = B * C
    am = torch.empty(T, dtype=torch.int32, device="cuda")
    lse = torch.empty(T, dtype=torch.float32, device="cuda")
    cf = torch.empty(T, dtype=torch.float32, device="cuda")
    mg = torch.empty(T, dtype=torch.float32, device="cuda")
    ctx.debug_lmhead(am, lse, cf, mg)
    if capture:
        L = w.shape.n_layers
        hid, exp, nrm = [], [], []
        for l in range(L + 1):
            buf = torch.empty(T, w.shape.d_model, dtype=torch.float32, device="cuda")
            ctx.debug_hidden(l, buf)
            hid.append(buf)
            nb = torch.empty(T, w.shape.d_model, dtype=torch.bfloat16, device="cuda")
            ctx.debug_norm_rows(l, nb)
            nrm.append(nb)
        for l in range(L):
            buf = torch.empty(T, w.shape.top_k, dtype=torch.int32, device="cuda")
            ctx.debug_experts(l, buf)
            exp.append(buf)
        ctx.sync()
        res["hidden"] = [h.cpu().numpy().reshape(B, C, -1) for h in hid]
        res["experts"] = [e.cpu().numpy().reshape(B, C, -1) for e in exp]
        # bf16 rows exactly as consumed: routers (layers 0..L-1), LM head (L)
        res["norm_rows"] = [n.cpu().to(torch.float64).numpy().reshape(B, C, -1) for n in nrm]
    ctx.sync()
    res.update(canvas_out=cout.cpu().numpy(), conf=conf.cpu().numpy(), settled=settled.cpu().numpy(),
               argmax=am.cpu().numpy().reshape(B, C), lse=lse.cpu().numpy().reshape(B, C),
               conf_dbg=cf.cpu().numpy().reshape(B, C), margin=mg.cpu().numpy().reshape(B, C))
    return res


def _rms_rows(h):
    return np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + 1e-6)


def oracle_step(orc, canvas, step, seed, tau, temperature, g=None):
    """The oracle's step on the same canvas; with a captured GPU step `g`
    also teacher-forced on the GPU's per-layer inputs, expert choices,
    router rows and LM-head rows (one pass over the layers serves both)."""
    teacher = None
    if g is not None and "hidden" in g:
        L = len(g["experts"])
        teacher = {"hidden": g["hidden"], "experts": g["experts"],
                   "router_rows": g["norm_rows"][:L], "lm_rows": g["norm_rows"][L]}
    return orc.denoise_step(canvas, step, seed, tau, temperature=temperature, teacher=teacher)


def _embed_max_row_norm(orc) -> float:
    if getattr(orc, "_embed_max_norm", None) is None:
        e = orc.embed
        m = 0.0
        for r0 in range(0, e.shape[0], 16384):
            blk = e[r0:r0 + 16384]
            blk = blk.to(torch.float64) if isinstance(blk, torch.Tensor) else torch.as_tensor(blk, dtype=torch.float64)
            m = max(m, float(torch.linalg.vector_norm(blk, dim=1).max()))
        orc._embed_max_norm = m
    return orc._embed_max_norm


def teacher_forced_checks(g: dict, r, temperature: float, out: dict, fails: list):
    """Criteria on the teacher-forced results (every token, no exclusion
    beyond the decision bands):
      * each layer alone, fed the GPU's input rows and expert choices, within
        HIDDEN_REL_L2 of the GPU's output (relative L2 over all tokens);
      * the expert sets the GPU chose equal the oracle's top-k of the GPU's
        own router rows, except where that k-th/(k+1)-th logit gap is below
        ROUTER_GAP_BAND;
      * the full-vocabulary argmax equals the oracle's argmax of the GPU's
        own LM-head rows wherever that top-1/top-2 logit gap is above
        LM_GAP_BAND / min(1, T); log-sum-exp and log-probability within
        LOGP_ABS at every position."""
    L = len(g["experts"])
    errs = [rel_l2(g["hidden"][l + 1], r.forced_hidden[l + 1]) for l in range(L)]
    out["forced_hidden_rel_l2"] = errs
    out["forced_hidden_rel_l2_max"] = max(errs)
    if max(errs) > HIDDEN_REL_L2:
        fails.append(f"teacher-forced layer rel-L2 {max(errs):.4g} > {HIDDEN_REL_L2}")
    flips_in_band = 0
    for l in range(L):
        ge = np.sort(g["experts"][l], axis=-1)
        oe = np.sort(r.forced_experts[l], axis=-1)
        diff = (ge != oe).any(axis=-1)
        near = r.forced_router_margin[l] < ROUTER_GAP_BAND
        bad = diff & ~near
        flips_in_band += int((diff & near).sum())
        if bad.any():
            b, t = np.argwhere(bad)[0]
            fails.append(f"layer {l}: {int(bad.sum())} expert sets differ on identical router rows "
                         f"(token {b},{t}, gap {r.forced_router_margin[l][b, t]:.3g})")
    out["forced_router_flips_in_band"] = flips_in_band
    f = r.forced_lm
    band = LM_GAP_BAND / min(1.0, temperature)
    checked = f["gap"] > band
    am_bad = checked & (g["argmax"] != f["argmax"])
    out["forced_argmax_checked"] = int(checked.sum())
    out["forced_argmax_mismatch"] = int(am_bad.sum())
    if am_bad.any():
        fails.append(f"{int(am_bad.sum())} argmax differ on identical LM-head rows (gap > {band:.3g})")
    dl = np.abs(g["lse"].astype(np.float64) - f["lse"])
    dp = np.abs(np.log(np.maximum(g["conf"].astype(np.float64), 1e-38)) - f["logp"])
    out["forced_lse_abs_max"] = float(dl.max())
    out["forced_logp_abs_max"] = float(dp.max())
    if dl.max() > LOGP_ABS or dp.max() > LOGP_ABS:
        fails.append(f"teacher-forced LM head: lse {dl.max():.3g}, logp {dp.max():.3g} > {LOGP_ABS}")


def compare_step(g: dict, r: "oracle.StepResult", tau: float, orc=None, check_hidden=True, report=None,
                 temperature: float = 1.0, drift_tol: float | None = None):
    """Apply the criteria; returns a dict of measured errors (asserts at the end).

    Router near-ties.  The GPU feeds the router bf16 operands derived from its
    own fp32 residual stream, the oracle fp64 ones; where the oracle's k-th and
    (k+1)-th logits are closer than the perturbation those input differences
    can cause, the two may legitimately pick different experts.  The bound
    used is Cauchy-Schwarz: |d(r_a - r_b)| <= ||W_r[a] - W_r[b]|| * ||du||, with
    ||du|| = (drift of the normalised residual measured at the layer's input and
    output) + the bf16 rounding bound 2^-8 ||u||.  A flip beyond the bound is a
    failure; a token within it is counted and, from that layer on, left out of
    the hidden-state and log-probability comparisons (its residual stream has
    legitimately left the oracle's).

    The 1e-2 per-layer criterion is the error one layer adds: it is checked
    teacher-forced (teacher_forced_checks).  The free-running residual stream
    carries the rounding of every layer before it; it is held to the same 1e-2
    unless drift_tol is given (the 30-layer test gives 2e-2: a bf16-operand
    emulation of the first layer already reaches 0.7%, and the drift
    accumulates over depth).
    """
    out = {}
    B, C = r.canvas_out.shape
    diverged = np.zeros((B, C), dtype=bool)
    fails = []
    if check_hidden and "hidden" in g:
        errs = [rel_l2(g["hidden"][0], r.hidden[0])]
        errs_all = list(errs)
        flips = 0
        for l in range(len(r.experts)):
            ge = np.sort(g["experts"][l], axis=-1)
            oe = np.sort(r.experts[l], axis=-1)
            diff = (ge != oe).any(axis=-1) & ~diverged
            if diff.any():
                assert orc is not None, "router flip found; pass the oracle to bound it"
                wr = orc.layer(l)["w_router"]
                du = np.zeros((B, C))
                for hh in (l, l + 1):
                    ug = g["hidden"][hh] / _rms_rows(g["hidden"][hh])
                    uo = r.hidden[hh] / _rms_rows(r.hidden[hh])
                    du = np.maximum(du, np.linalg.norm(ug - uo, axis=-1))
                du = du + 2.0 ** -8 * np.sqrt(r.hidden[0].shape[-1])
                srt = np.argsort(-r.router_logits[l], axis=-1, kind="stable")
                k = r.experts[l].shape[-1]
                for b, t in zip(*np.nonzero(diff)):
                    ea, eb = srt[b, t, k - 1], srt[b, t, k]
                    bound = np.linalg.norm(wr[ea] - wr[eb]) * du[b, t]
                    gap = r.router_margin[l][b, t]
                    if gap > bound:
                        fails.append(f"layer {l} token {b},{t}: expert gap {gap:.4g} > bound {bound:.4g}")
            flips += int(diff.sum())
            diverged |= diff
            keep = ~diverged
            errs.append(rel_l2(g["hidden"][l + 1][keep], r.hidden[l + 1][keep]))
            errs_all.append(rel_l2(g["hidden"][l + 1], r.hidden[l + 1]))
        out["hidden_rel_l2_max"] = max(errs)
        out["hidden_rel_l2"] = errs
        out["hidden_rel_l2_all_tokens"] = errs_all
        out["expert_flips"] = flips
        tol = HIDDEN_REL_L2 if drift_tol is None else drift_tol
        if out["hidden_rel_l2_max"] > tol:
            fails.append(f"free-running hidden rel-L2 {out['hidden_rel_l2_max']:.4g} > {tol}")
    if check_hidden and "hidden" in g and r.forced_hidden:
        teacher_forced_checks(g, r, temperature, out, fails)
    keep = ~diverged
    logp_g = np.log(np.maximum(g["conf"].astype(np.float64), 1e-38))
    dlogp = np.abs(logp_g - r.logp)
    out["logp_abs_max"] = float(dlogp[keep].max()) if keep.any() else 0.0
    out["logp_abs_max_all_tokens"] = float(dlogp.max())
    # log-sum-exp on its own (free-running: same bound as logp, 5e-2 at T = 1;
    # the teacher-forced check above holds it to 5e-2 at every temperature)
    logp_tol = LOGP_ABS / min(1.0, temperature)
    dlse = np.abs(g["lse"].astype(np.float64) - r.lse)
    out["lse_abs_max"] = float(dlse[keep].max()) if keep.any() else 0.0
    if out["lse_abs_max"] > logp_tol:
        fails.append(f"lse max abs {out['lse_abs_max']:.4g} > {logp_tol:.4g}")
    # Free-running argmax, wherever the oracle's own top-1/top-2 logit gap
    # exceeds twice the largest logit change the GPU's LM-head input drift can
    # cause: |ds_v| <= ||z_gpu - z_oracle|| * max_v ||E_v|| / T (Cauchy-Schwarz).
    if "norm_rows" in g and orc is not None:
        z_o = oracle.rms_norm(r.hidden[-1], orc.final_norm, orc.s.rms_eps)
        dz = np.linalg.norm(g["norm_rows"][-1] - z_o, axis=-1)
        bound = dz * _embed_max_row_norm(orc) / temperature
        chk = (r.gap > 2.0 * bound) & keep
        am_bad = chk & (g["argmax"] != r.argmax)
        out["argmax_checked"] = int(chk.sum())
        out["argmax_mismatch"] = int(am_bad.sum())
        if am_bad.any():
            fails.append(f"{int(am_bad.sum())} free-running argmax differ beyond the drift bound")
    # logits are divided by the temperature before the softmax, so their
    # rounding error (and that of logp) scales with 1/T; the bound is stated at
    # T = 1 (the 1/T scaling below T = 1 goes beyond the stated criteria)
    if out["logp_abs_max"] > logp_tol:
        fails.append(f"logp max abs {out['logp_abs_max']:.4g} > {logp_tol:.4g}")
    excl = (r.margin < EXCLUDE_BAND) | (np.abs(r.conf - tau) < EXCLUDE_BAND) | diverged
    if temperature < 1.0:
        # Beyond the stated criteria (which are stated at T = 1): below T = 1 a
        # confidence moves by up to conf * (e^{logp error} - 1), far beyond the
        # 1e-3 band; a position whose two confidences fall on opposite sides of
        # tau while its logp agrees within the tolerance is exempt.  (The
        # decision given a confidence is checked bit-exact by the sampler hook
        # test, and the teacher-forced checks above hold at every T.)
        straddle = ((g["conf"] >= tau) != (r.conf >= tau)) & (dlogp <= logp_tol)
        out["straddle_exempt"] = int(straddle.sum())
        excl = excl | straddle
    mism = g["canvas_out"] != r.canvas_out
    out["token_mismatch"] = int((mism & ~excl).sum())
    out["excluded"] = int(excl.sum())
    out["excluded_mismatch"] = int((mism & excl).sum())
    if out["token_mismatch"]:
        fails.append(f"{out['token_mismatch']} token decisions differ outside the exclusion band")
    if report is not None:
        report.append(out)
    print({k: v for k, v in out.items()})
    assert not fails, fails
    res = dict(out)
    res["diverged"] = diverged   # tokens whose routing legitimately left the oracle's
    return res
