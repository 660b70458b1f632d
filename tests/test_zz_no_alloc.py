"""dg_lmhead_argmax_static: the LM-head reduction for callers that cannot
allocate device memory (e.g. while another framework records a CUDA graph, or
when their allocator already holds the whole device).  Its partials live in a
fixed array inside the library; this test checks it, through the C ABI, against
the LM-head outputs of the regular context-based path on the same rows, on two
calls in a row (the second call sees the first call's leftovers in the shared
array).  Kept in its own file, collected last."""
import numpy as np
import pytest
import torch

import block_discrete_diffusion_denoise_b200 as dgp
import synth_inputs as si

from gpu_helpers import LOGP_ABS, make_context

pytestmark = pytest.mark.gpu


def _zero_out(l, t):
    t = dict(t)
    for k in ("wo", "w_down", "ws_down"):
        t[k] = torch.zeros_like(t[k])
    return t


def test_static_scratch_lmhead_matches_context_path_on_two_calls():
    # With every output projection zero the residual stream of the step is the
    # embedding itself, so the rows the regular path feeds its LM head are
    # RMSNorm(E[canvas]) and can be rebuilt here.
    w = si.workload("tiny").with_(prefix=32)
    ctx, weights = make_context(w, temperature=1.0, layer_override=_zero_out)
    ctx.prefill(si.uniform_tokens(w, "prefix", 1, 32).cuda())
    canvas = si.uniform_tokens(w, "canvas", 1, 256).cuda()
    out = torch.empty_like(canvas)
    conf = torch.empty(1, 256, dtype=torch.float32, device="cuda")
    ctx.denoise_step(canvas, 0, 0, 0.9, out, conf)
    ref_am = torch.empty(256, dtype=torch.int32, device="cuda")
    ref_lse = torch.empty(256, dtype=torch.float32, device="cuda")
    ref_conf = torch.empty(256, dtype=torch.float32, device="cuda")
    ref_margin = torch.empty(256, dtype=torch.float32, device="cuda")
    ctx.debug_lmhead(ref_am, ref_lse, ref_conf, ref_margin)
    ctx.sync()

    embed = weights["embed"]
    h = embed[canvas[0].long()].float()
    z = (h * torch.rsqrt(h.pow(2).mean(-1, keepdim=True) + w.shape.rms_eps)
         * weights["final_norm"].float()).to(torch.bfloat16).contiguous()
    stream = torch.cuda.current_stream().cuda_stream
    decided = ref_margin.cpu().numpy() >= 1e-3
    for call in range(2):
        am = torch.full((256,), -7, dtype=torch.int32, device="cuda")
        lse = torch.full((256,), float("nan"), device="cuda")
        cf = torch.full((256,), float("nan"), device="cuda")
        st = dgp.lmhead_argmax_static(z, embed, 1.0, am, lse, cf, stream=stream)
        assert st == dgp.DG_OK, dgp.STATUS.get(st, st)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(am.cpu().numpy()[decided], ref_am.cpu().numpy()[decided])
        assert np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy()).max() <= LOGP_ABS
        assert np.abs(np.log(cf.cpu().numpy()) - np.log(ref_conf.cpu().numpy())).max() <= LOGP_ABS
    ctx.close()


def test_static_scratch_lmhead_rejects_oversize_without_launch():
    z = torch.zeros(512, 256, dtype=torch.bfloat16, device="cuda")
    embed = torch.zeros(262144, 256, dtype=torch.bfloat16, device="cuda")
    am = torch.empty(512, dtype=torch.int32, device="cuda")
    # 512 rows x 2048 vocabulary tiles exceeds the fixed 524288-entry array
    assert dgp.lmhead_argmax_static(z, embed, 1.0, am) == 3  # DG_ERR_CAPACITY
    assert dgp.lmhead_argmax_static(z[:, :100], embed, 1.0, am) == 1  # d_model not a multiple of 64
