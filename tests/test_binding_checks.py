"""The binding's argument checks, on CPU.  The C ABI takes bare pointers, so
the binding refuses (DGError with DG_ERR_INVALID_ARG) any buffer the library
would read or write out of bounds or misread: wrong dtype, strided, on the
wrong device, or with fewer elements than the call touches.  Every call
pattern the GPU tests and bench.py make is replayed here on host tensors
against a stand-in library, and must pass; the malformed ones must not reach
the library."""
import math

import numpy as np
import pytest
import torch

import block_discrete_diffusion_denoise_b200 as dgp
import synth_inputs as si


def _refused(fn, *a, **kw):
    with pytest.raises(dgp.DGError) as ei:
        fn(*a, **kw)
    assert ei.value.status == dgp.DG_ERR_INVALID_ARG
    return str(ei.value)


@pytest.mark.parametrize("name", sorted(si.WORKLOADS))
def test_weight_numels_match_the_generator_layout(name):
    w = si.workload(name)
    n = dgp.weight_numels(dgp.config_from_shape(w.shape))
    for f, shape in si.layer_shapes(w.shape).items():
        assert n["layer"][f] == math.prod(shape), f
    s = w.shape
    assert n["embed"] == s.vocab * s.d_model and n["final_norm"] == s.d_model
    assert n["router_bias"] == s.n_experts
    assert n["sc_gate"] == n["sc_up"] == n["sc_down"] == s.expert_hidden * s.d_model
    assert set(n["layer"]) == set(dgp.LAYER_FIELDS)


def _tiny_weights(**kw):
    w = si.workload("tiny").with_(**kw)
    weights = si.model_weights(w, "cpu")
    return w, dgp.config_from_shape(w.shape), weights


def test_check_weights_accepts_the_generated_models():
    w, cfg, weights = _tiny_weights()
    dgp.check_weights(cfg, weights, "cpu")
    weights.update(si.self_cond_weights(w, "cpu"))               # with self-conditioning
    dgp.check_weights(cfg, weights, "cpu")
    w, cfg, weights = _tiny_weights(zipf_s=1.1)                  # with the fp32 router bias
    assert weights["router_bias"].dtype == torch.float32
    dgp.check_weights(cfg, weights, "cpu")

    def zero_out(l, t):                                          # the planted cases
        t = dict(t)
        for k in ("wo", "w_down", "ws_down"):
            t[k] = torch.zeros_like(t[k])
        return t
    dgp.check_weights(cfg, si.model_weights(w, "cpu", zero_out), "cpu")


def test_check_weights_refuses_what_the_library_would_misread():
    w, cfg, weights = _tiny_weights()
    assert "cuda" in _refused(dgp.check_weights, cfg, weights)   # host tensors for a device context

    def edited(path, value):
        out = dict(weights)
        out["layers"] = [dict(l) for l in weights["layers"]]
        if isinstance(path, tuple):
            out["layers"][path[0]][path[1]] = value
        elif value is None:
            out.pop(path)
        else:
            out[path] = value
        return out

    lw = weights["layers"][1]
    cases = {
        "embed dtype": edited("embed", weights["embed"].float()),
        "embed rows": edited("embed", weights["embed"][:-1]),
        "missing final norm": edited("final_norm", None),
        "wqkv short": edited((1, "wqkv"), lw["wqkv"][:-1].contiguous()),
        "wo strided": edited((1, "wo"), lw["wo"].t()),
        "w_down long": edited((1, "w_down"), torch.cat([lw["w_down"], lw["w_down"][:1]])),
        "w_up missing": edited((0, "w_up"), None),
        "router bias bf16": edited("router_bias", torch.zeros(16, dtype=torch.bfloat16)),
    }
    for what, bad in cases.items():
        _refused(dgp.check_weights, cfg, bad, "cpu")
    short = dict(weights, layers=weights["layers"][:1])
    assert "layer dicts" in _refused(dgp.check_weights, cfg, short, "cpu")
    sc = si.self_cond_weights(w, "cpu")
    partial = dict(weights, sc_gate=sc["sc_gate"], sc_up=sc["sc_up"])
    assert "none" in _refused(dgp.check_weights, cfg, partial, "cpu")


class _FakeLib:
    """Stands in for libdg.so: records the calls that got through."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if not name.startswith("dg_"):
            raise AttributeError(name)

        def call(*args):
            self.calls.append(name)
            return b"" if name == "dg_last_error" else 0
        return call


def _host_context(canvas=256):
    ctx = dgp.Context.__new__(dgp.Context)
    ctx._device_type = "cpu"
    ctx.lib = _FakeLib()
    ctx.ctx = None
    ctx.cfg = {"canvas": canvas}
    ctx._batch = None
    return ctx


def _i32(*shape):
    return torch.zeros(*shape, dtype=torch.int32)


def _f32(*shape):
    return torch.zeros(*shape, dtype=torch.float32)


def test_path_calls_of_the_tests_and_the_bench_pass():
    ctx = _host_context()
    ctx.prefill(_i32(2, 40))
    assert ctx._batch == 2 and ctx.lib.calls == ["dg_prefill"]
    cin = _i32(2, 256)
    ctx.denoise_step(cin, 0, 1, 0.9, torch.empty_like(cin), _f32(2, 256), _i32(2))
    ctx.denoise_step(cin, 0, 1, 0.9, cin, _f32(2, 256))                 # in place, no flags
    ctx.denoise_step(_i32(4, 256), 0, 1, 0.9, _i32(4, 256), _f32(4, 256), _i32(4))   # larger buffers
    ctx.denoise_step_entropy(cin, 1, 1, 0.8, 8.0, 0.5, _i32(2, 256))     # every optional output absent
    ctx.denoise_step_entropy(cin, 1, 1, 0.8, 8.0, 0.5, _i32(2, 256), prev_argmax=_i32(2, 256),
                             argmax_out=_i32(2, 256), entropy=_f32(2, 256), stopped=_i32(2))
    h = np.zeros((2, 256), np.int32)
    ctx.denoise_step_host(h, 0, 1, 0.9, np.empty_like(h), np.empty((2, 256), np.float32), np.empty(2, np.int32))
    ctx.denoise_step_host(h, 0, 1, 0.9, np.empty_like(h))
    ctx.denoise_step_host(torch.from_numpy(h), 0, 1, 0.9, _i32(2, 256), _f32(2, 256), _i32(2))
    ctx.commit_block(cin)
    ctx.prefill(torch.cat([_i32(2, 40), cin], 1))                      # prefix || block
    assert ctx.lib.calls == ["dg_prefill"] + ["dg_denoise_step"] * 3 + ["dg_denoise_step_entropy"] * 2 + \
        ["dg_denoise_step_host"] * 3 + ["dg_commit_block", "dg_prefill"]


def test_malformed_path_buffers_never_reach_the_library():
    ctx = _host_context()
    cin, conf = _i32(2, 256), _f32(2, 256)
    # before any prefill only dtype and layout are checked: the library refuses the state itself
    ctx.denoise_step(cin, 0, 1, 0.9, cin, conf)
    assert ctx.lib.calls == ["dg_denoise_step"]
    _refused(ctx.prefill, _i32(40))                                     # not [batch, length]
    _refused(ctx.prefill, torch.zeros(2, 40, dtype=torch.int64))
    ctx.prefill(_i32(2, 40))
    n0 = len(ctx.lib.calls)
    bad_steps = {
        "short canvas": (_i32(1, 256), cin, conf, None),
        "int64 canvas": (torch.zeros(2, 256, dtype=torch.int64), cin, conf, None),
        "strided canvas": (_i32(256, 2).t(), cin, conf, None),
        "short output": (cin, _i32(2, 255), conf, None),
        "no conf": (cin, cin, None, None),
        "fp64 conf": (cin, cin, torch.zeros(2, 256, dtype=torch.float64), None),
        "short flags": (cin, cin, conf, _i32(1)),
        "numpy canvas": (np.zeros((2, 256), np.int32), cin, conf, None),
    }
    for what, (a, o, c, s) in bad_steps.items():
        _refused(ctx.denoise_step, a, 0, 1, 0.9, o, c, s)
    _refused(ctx.denoise_step_entropy, cin, 1, 1, 0.8, 8.0, 0.5, cin, prev_argmax=_f32(2, 256))
    _refused(ctx.denoise_step_entropy, cin, 1, 1, 0.8, 8.0, 0.5, cin, entropy=_f32(2, 100))
    _refused(ctx.denoise_step_entropy, cin, 1, 1, 0.8, 8.0, 0.5, cin, stopped=_i32(1))
    h = np.zeros((2, 256), np.int32)
    _refused(ctx.denoise_step_host, h[:1], 0, 1, 0.9, h)
    _refused(ctx.denoise_step_host, h, 0, 1, 0.9, np.zeros((2, 512), np.int32)[:, ::2])
    _refused(ctx.denoise_step_host, h, 0, 1, 0.9, h.copy(), np.zeros((2, 256), np.float64))
    _refused(ctx.denoise_step_host, h, 0, 1, 0.9, h.copy(), None, np.zeros(1, np.int32))
    _refused(ctx.commit_block, _i32(1, 256))
    assert len(ctx.lib.calls) == n0

    dev = _host_context()
    dev._device_type = "cuda"                                           # a real context: host tensors refused
    _refused(dev.prefill, _i32(2, 40))
    assert dev.lib.calls == []
