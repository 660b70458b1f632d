"""The tracing build on the GPU: libdg_timeline.so records one entry per CTA of
every kernel, and the launch sequence rebuilt from them is the step's own
kernel sequence (the binding loads one library per process, so the check
runs in a child process with DG_LIBRARY pointing at the tracing build)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, os, sys
sys.path.insert(0, os.environ["DG_ROOT"]); sys.path.insert(0, os.path.join(os.environ["DG_ROOT"], "tests"))
import torch
import block_discrete_diffusion_denoise_b200 as dgp
import synth_inputs as si
from gpu_helpers import make_context
w = si.workload("tiny").with_(prefix=128)
s = torch.cuda.Stream()
with torch.cuda.stream(s):
    ctx, _ = make_context(w, stream=s.cuda_stream)
    ctx.prefill(si.uniform_tokens(w, "prefix", 1, 128, device="cuda"))
    cur = si.uniform_tokens(w, "canvas", 1, 256, device="cuda")
    out = torch.empty_like(cur); conf = torch.empty(1, 256, device="cuda")
    for st in range(3):                       # warm-up (the graph is captured)
        ctx.denoise_step(cur, st, 1, 0.9, out, conf)
    ctx.debug_timeline_reset()
    ctx.denoise_step(cur, 3, 1, 0.9, out, conf)
    rec, n = ctx.debug_timeline()
    launches = dgp.timeline_launches(rec)
    summ = dgp.timeline_summary(launches)
    print(json.dumps({"n": int(n), "names": [l["name"] for l in launches], "launch_count": ctx.launch_count,
                      "wall_us": summ["wall_us"], "ctas": [l["ctas"] for l in launches]}))
    ctx.close()
"""


def test_timeline_build_records_the_step_kernel_sequence():
    lib = os.path.join(ROOT, "block_discrete_diffusion_denoise_b200", "libdg_timeline.so")
    assert os.path.exists(lib), "libdg_timeline.so is not built"
    env = dict(os.environ, DG_LIBRARY=lib, DG_ROOT=ROOT)
    res = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    d = json.loads(res.stdout.strip().splitlines()[-1])
    names = d["names"]
    # embedding, then per layer: QKV, RoPE, attention (+ merge), O, residual norm,
    # router, dispatch, experts, combine; then the LM head and its merge + sampler
    assert names[0] == "embed_norm" and names[-2:] == ["gemm_lmhead", "lmhead_merge_sample"]
    layer = [n for n in names[1:-2] if n != "attn_merge"]
    per_layer = ["gemm_dense", "rope_qkv", "attention", "gemm_dense", "residual_norm", "gemm_dense",
                 "route_dispatch", "gemm_moe", "combine_norm"]
    assert len(layer) % len(per_layer) == 0 and len(layer) // len(per_layer) == 2
    assert layer == per_layer * 2
    assert d["n"] == sum(d["ctas"]) and d["wall_us"] > 0
