"""Oracle package — TEST INFRASTRUCTURE ONLY.

A plain float64 CPU statement of the block discrete-diffusion denoising step
(see `oracle.model`) and of the Philox4x32-10 generator its sampler draws from
(see `oracle.philox`).  Only `tests/`, `__graft_entry__.smoke()` and the
`cpu_baseline` / `--impl reference` legs of `bench.py` may import this package.
It shares no code with the CUDA library; the only thing both sides use is the
seeded input generator module `synth_inputs`.

Parity status of each function is recorded beside its pin in tests/.
"""
from .model import (Oracle, Shape, StepResult, anneal_temperature, apply_rope, attention, entropy_accept,
                    entropy_sample, lm_head_stats, mean_entropy, moe,
                    renoise_tokens, rms_norm, rope_angles, route_top_k, sample, selected_gates, self_condition, silu,
                    swiglu_ffn, tokens_per_forward, tokens_per_second)
from .mx import e4m3_round, moe_mx, mx_dequantize, mx_linear, mx_quantize, mx_round_trip, mx_swiglu_ffn
from .philox import philox4x32_10, uniform_token


def shape_of(w) -> Shape:
    """Oracle shape record from a synth_inputs.Workload."""
    s = w.shape
    return Shape(n_layers=s.n_layers, d_model=s.d_model, n_q_heads=s.n_q_heads,
                 n_kv_heads=s.n_kv_heads, head_dim=s.head_dim, n_experts=s.n_experts,
                 top_k=s.top_k, expert_hidden=s.expert_hidden, shared_hidden=s.shared_hidden,
                 vocab=s.vocab, rope_base=s.rope_base, rms_eps=s.rms_eps)


def for_workload(w, keep_layers: bool = True, layer_override=None, seq_ids=None,
                 expert_format: str = "bf16") -> Oracle:
    """Oracle over the seeded weights of workload `w` (generated on the CPU).

    layer_override(l, tensors) may edit a layer's tensors (planted cases);
    seq_ids gives the batch index of each of the oracle's sequences;
    expert_format "mxfp8" runs every expert GEMM in MXFP8 (oracle/mx.py)."""
    import synth_inputs as si

    def layer_fn(l):
        t = si.layer_weights(w, l, "cpu")
        if layer_override is not None:
            t = layer_override(l, t)
        return t

    g = si.global_weights(w, "cpu")
    return Oracle(shape_of(w), layer_fn, g["embed"], g["final_norm"], g["router_bias"],
                  batch=w.batch, keep_layers=keep_layers, seq_ids=seq_ids, expert_format=expert_format)
