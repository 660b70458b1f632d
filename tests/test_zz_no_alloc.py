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


def test_static_scratch_smaller_ragged_call_after_larger_one():
    """A call over fewer rows (100, not a multiple of the 128-row tile) and a
    narrower vocabulary right after a larger call: the shared array still
    holds the larger call's partials, none of which may be read.  Checked
    against float64 logits on the CPU."""
    g = torch.Generator().manual_seed(11)
    z1 = (torch.randn(256, 256, generator=g) * 1.0).to(torch.bfloat16).cuda()
    e1 = (torch.randn(8192, 256, generator=g) * 0.05).to(torch.bfloat16).cuda()
    z2 = (torch.randn(100, 256, generator=g) * 1.0).to(torch.bfloat16).cuda()
    e2 = (torch.randn(4096, 256, generator=g) * 0.05).to(torch.bfloat16).cuda()
    stream = torch.cuda.current_stream().cuda_stream
    big = torch.empty(256, dtype=torch.int32, device="cuda")
    assert dgp.lmhead_argmax_static(z1, e1, 0.7, big, stream=stream) == dgp.DG_OK
    am = torch.full((100,), -7, dtype=torch.int32, device="cuda")
    lse = torch.full((100,), float("nan"), device="cuda")
    cf = torch.full((100,), float("nan"), device="cuda")
    assert dgp.lmhead_argmax_static(z2, e2, 0.7, am, lse, cf, stream=stream) == dgp.DG_OK
    torch.cuda.synchronize()
    s = (z2.cpu().double() @ e2.cpu().double().T) / 0.7
    top2 = s.topk(2, dim=1).values
    ref_lse = torch.logsumexp(s, 1)
    clear = (top2[:, 0] - top2[:, 1]) > 1e-3
    np.testing.assert_array_equal(am.cpu()[clear].numpy(), s.argmax(1)[clear].numpy())
    assert (lse.cpu().double() - ref_lse).abs().max().item() < 1e-3
    assert (cf.cpu().double().log() - (top2[:, 0] - ref_lse)).abs().max().item() < 1e-3


def test_static_scratch_rejects_malformed_tensors_without_launch():
    z = torch.zeros(64, 256, dtype=torch.bfloat16, device="cuda")
    embed = torch.zeros(1024, 256, dtype=torch.bfloat16, device="cuda")
    am = torch.empty(64, dtype=torch.int32, device="cuda")
    ok_lse = torch.empty(64, dtype=torch.float32, device="cuda")
    bad = [
        (z.float(), embed, am, None),                                   # z not bf16
        (z, embed[:, :128], am, None),                                  # widths differ
        (torch.zeros(64, 512, dtype=torch.bfloat16, device="cuda")[:, :256], embed, am, None),  # z strided
        (z, embed, am[:10], None),                                      # argmax shorter than the rows
        (z, embed, am.float(), None),                                   # argmax not int32
        (z, embed, am, ok_lse[:63]),                                    # lse shorter than the rows
        (z.cpu(), embed, am, None),                                     # z on the host
    ]
    for zz, ee, a, l in bad:
        assert dgp.lmhead_argmax_static(zz, ee, 1.0, a, l) == 1        # DG_ERR_INVALID_ARG
    assert dgp.lmhead_argmax_static(z, embed, 1.0, am, ok_lse) == dgp.DG_OK
    torch.cuda.synchronize()
