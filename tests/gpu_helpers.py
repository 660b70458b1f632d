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
                 prefill_rows: int = 0, weights=None):
    if weights is None:
        weights = si.model_weights(w, "cuda", layer_override)
    if max_seq is None:
        max_seq = w.prefix + w.canvas * (w.blocks + 1)
    cfg = dgp.config_from_shape(w.shape, max_batch=w.batch, max_seq=max_seq, canvas=w.canvas,
                                temperature=temperature, prefill_rows=prefill_rows)
    return dgp.Context(cfg, weights), weights


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


def compare_step(g: dict, r: "oracle.StepResult", tau: float, check_hidden=True, report=None):
    """Apply the criteria; returns a dict of measured errors (asserts inside)."""
    out = {}
    if check_hidden and "hidden" in g:
        errs = [rel_l2(g["hidden"][l], r.hidden[l]) for l in range(len(r.hidden))]
        out["hidden_rel_l2_max"] = max(errs)
        out["hidden_rel_l2"] = errs
        # expert sets: equal wherever the oracle's k-th/k+1-th logit gap is not a near tie
        flips = 0
        for l in range(len(r.experts)):
            ge = np.sort(g["experts"][l], axis=-1)
            oe = np.sort(r.experts[l], axis=-1)
            diff = (ge != oe).any(axis=-1)
            near = r.router_margin[l] < EXCLUDE_BAND
            bad = diff & ~near
            flips += int(diff.sum())
            assert not bad.any(), f"layer {l}: {int(bad.sum())} tokens with different experts (no near tie)"
        out["expert_flips"] = flips
        assert out["hidden_rel_l2_max"] <= HIDDEN_REL_L2, errs
    logp_g = -np.log(np.maximum(g["conf"].astype(np.float64), 1e-38))
    logp_o = -r.logp
    out["logp_abs_max"] = float(np.abs(logp_g - logp_o).max())
    assert out["logp_abs_max"] <= LOGP_ABS, out["logp_abs_max"]
    excl = (r.margin < EXCLUDE_BAND) | (np.abs(r.conf - tau) < EXCLUDE_BAND)
    mism = g["canvas_out"] != r.canvas_out
    out["token_mismatch"] = int((mism & ~excl).sum())
    out["excluded"] = int(excl.sum())
    out["excluded_mismatch"] = int((mism & excl).sum())
    assert out["token_mismatch"] == 0, out
    if report is not None:
        report.append(out)
    return out
