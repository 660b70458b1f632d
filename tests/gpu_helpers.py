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
LOGP_ABS = 5e-2          # per-position log-probability of the argmax
EXCLUDE_BAND = 1e-3      # positions with top1-top2 margin or |conf - tau| below this are exempt


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
        hid, exp = [], []
        for l in range(L + 1):
            buf = torch.empty(T, w.shape.d_model, dtype=torch.float32, device="cuda")
            ctx.debug_hidden(l, buf)
            hid.append(buf)
        for l in range(L):
            buf = torch.empty(T, w.shape.top_k, dtype=torch.int32, device="cuda")
            ctx.debug_experts(l, buf)
            exp.append(buf)
        ctx.sync()
        res["hidden"] = [h.cpu().numpy().reshape(B, C, -1) for h in hid]
        res["experts"] = [e.cpu().numpy().reshape(B, C, -1) for e in exp]
    ctx.sync()
    res.update(canvas_out=cout.cpu().numpy(), conf=conf.cpu().numpy(), settled=settled.cpu().numpy(),
               argmax=am.cpu().numpy().reshape(B, C), lse=lse.cpu().numpy().reshape(B, C),
               conf_dbg=cf.cpu().numpy().reshape(B, C), margin=mg.cpu().numpy().reshape(B, C))
    return res


def _rms_rows(h):
    return np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + 1e-6)


def compare_step(g: dict, r: "oracle.StepResult", tau: float, orc=None, check_hidden=True, report=None,
                 temperature: float = 1.0):
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
        if out["hidden_rel_l2_max"] > HIDDEN_REL_L2:
            fails.append(f"hidden rel-L2 {out['hidden_rel_l2_max']:.4g} > {HIDDEN_REL_L2}")
    keep = ~diverged
    logp_g = np.log(np.maximum(g["conf"].astype(np.float64), 1e-38))
    dlogp = np.abs(logp_g - r.logp)
    out["logp_abs_max"] = float(dlogp[keep].max()) if keep.any() else 0.0
    out["logp_abs_max_all_tokens"] = float(dlogp.max())
    # logits are divided by the temperature before the softmax, so their
    # rounding error (and that of logp) scales with 1/T; the bound is stated at T=1
    logp_tol = LOGP_ABS / min(1.0, temperature)
    if out["logp_abs_max"] > logp_tol:
        fails.append(f"logp max abs {out['logp_abs_max']:.4g} > {logp_tol:.4g}")
    excl = (r.margin < EXCLUDE_BAND) | (np.abs(r.conf - tau) < EXCLUDE_BAND) | diverged
    if temperature < 1.0:
        # Below T = 1 a confidence moves by up to conf * (e^{logp error} - 1),
        # far beyond the 1e-3 band; a position whose two confidences fall on
        # opposite sides of tau while its logp agrees within the tolerance is
        # exempt.  (The decision given a confidence is checked bit-exact by
        # the sampler hook test.)
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
    return out
