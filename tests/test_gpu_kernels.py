"""Kernel-level GPU checks through the C ABI: the tcgen05 GEMM, the router
decision, the sampler decision and the bounded-wait failure path."""
import numpy as np
import pytest
import torch

import block_discrete_diffusion_denoise_b200 as dgp
import oracle
from oracle import model as om
import synth_inputs as si

from gpu_helpers import make_context

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny_ctx():
    w = si.workload("tiny")
    ctx, weights = make_context(w)
    yield ctx, w
    ctx.close()


def _bf16(t):
    return t.to(torch.bfloat16)


@pytest.mark.parametrize("M,K,T,splits", [(128, 64, 16, 1), (256, 256, 48, 1), (384, 2816, 256, 3),
                                          (5632, 2816, 256, 5), (16, 256, 200, 2), (2816, 704, 33, 1)])
def test_tcgen05_gemm_matches_fp64_matmul(tiny_ctx, M, K, T, splits):
    ctx, _ = tiny_ctx
    g = torch.Generator().manual_seed(M * 7 + K + T)
    w = _bf16(torch.randn(M, K, generator=g) * 0.05)
    x = _bf16(torch.randn(T, K, generator=g))
    out = torch.full((splits, T, M), float("nan"), dtype=torch.float32, device="cuda")
    ctx.debug_gemm(w.cuda(), x.cuda(), splits, out)
    ctx.sync()
    got = out.sum(0).cpu().double()
    ref = x.double() @ w.double().T
    err = (got - ref).abs().max().item()
    scale = ref.abs().max().item()
    assert err <= 1e-4 * scale + 1e-5, (err, scale)


def test_router_decision_bit_exact(tiny_ctx):
    ctx, w = tiny_ctx
    E, k = w.shape.n_experts, w.shape.top_k
    g = torch.Generator().manual_seed(5)
    logits = torch.randn(300, E, generator=g, dtype=torch.float32)
    logits[::3, 5] = logits[::3, 9]            # exact ties between experts
    logits[7] = 0.25                           # all equal
    idx = torch.empty(300, k, dtype=torch.int32, device="cuda")
    gates = torch.empty(300, k, dtype=torch.float32, device="cuda")
    ctx.debug_router(logits.cuda(), idx, gates)
    ctx.sync()
    ref_idx, ref_g = om.route_top_k(logits.double().numpy(), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_allclose(gates.cpu().numpy(), ref_g, rtol=2e-6, atol=1e-7)


def test_sampler_decision_bit_exact(tiny_ctx):
    ctx, w = tiny_ctx
    prefix = si.uniform_tokens(w, "prefix", 1, 16).cuda()
    ctx.prefill(prefix)
    T = 256
    g = torch.Generator().manual_seed(9)
    am = torch.randint(0, w.shape.vocab, (T,), generator=g, dtype=torch.int32)
    cf = torch.rand(T, generator=g)
    cf[::5] = 0.9
    cf[3] = float("nan")
    out = torch.empty(T, dtype=torch.int32, device="cuda")
    seed = 0xDEADBEEF12345678
    ctx.debug_sample(am.cuda(), cf.cuda(), 1, 11, seed, 0.9, out)
    ctx.sync()
    noise = om.renoise_tokens(np.arange(16, 16 + T), 11, 0, seed, w.shape.vocab)
    ref = om.sample(am.numpy(), cf.numpy(), 0.9, noise)
    np.testing.assert_array_equal(out.cpu().numpy(), ref)


def test_bounded_wait_reports_timeout_and_recovers(tiny_ctx):
    ctx, _ = tiny_ctx
    ctx.debug_wait_timeout(2_000_000)          # 2 ms
    with pytest.raises(dgp.DGError) as ei:
        ctx.sync()
    assert ei.value.status == 5
    ctx.sync()                                 # cleared; context still usable
    out = torch.empty(1, 16, 128, dtype=torch.float32, device="cuda")
    w = torch.ones(128, 64, dtype=torch.bfloat16, device="cuda")
    x = torch.ones(16, 64, dtype=torch.bfloat16, device="cuda")
    ctx.debug_gemm(w, x, 1, out)
    ctx.sync()
    assert torch.all(out == 64)


def test_synth_generator_same_bits_on_gpu():
    w = si.workload("a4b_p2k")
    a = si.weight(w, "w_down", 3, device="cpu", rows=slice(5, 7))
    b = si.weight(w, "w_down", 3, device="cuda", rows=slice(5, 7)).cpu()
    assert torch.equal(a, b)
    ta = si.uniform_tokens(w, "prefix", 1, 4096)
    tb = si.uniform_tokens(w, "prefix", 1, 4096, device="cuda").cpu()
    assert torch.equal(ta, tb)
