"""Seeded synthetic inputs shared by the oracle and the CUDA path.

This module holds no arithmetic of the denoising method.  It only defines the
five workload shapes and produces seeded, bit-reproducible inputs for them:
random-init bf16 weights, uniform prefix tokens, uniform initial canvases and
the Zipf router skew.  Every generator is counter based (value = f(seed,
tensor id, flat index)), built from 32-bit integer mixing plus one table lookup,
so torch on the CPU and torch on a GPU produce the same bits and any slice of a
tensor can be regenerated on its own (the oracle regenerates only the layers it
checks).

Weights follow the model card of "DiffusionGemma Technical Report" as
summarised on codemajin.net, section 2.1 (MoE with 128 experts, top-8 plus one
shared expert, vocabulary ~262k); the exact dimensions are the five workload
shapes below.  The weight distribution is "bf16 N(0, 0.02)"; it is realised as
an Irwin-Hall sum of four uniform bytes, rescaled to standard deviation 0.02
(bounded at +-3.45 sigma), because that needs no transcendental function and is
therefore bit-identical on every device.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

__all__ = [
    "ModelShape", "Workload", "WORKLOADS", "workload", "tensor_id",
    "hash_u32", "weight", "layer_weights", "global_weights", "uniform_tokens",
    "router_bias", "tau_schedule", "norm_weight", "self_cond_weights",
]

MASK32 = 0xFFFFFFFF


@dataclass(frozen=True)
class ModelShape:
    n_layers: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n_experts: int
    top_k: int
    expert_hidden: int
    shared_hidden: int
    vocab: int
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    # output projections (Wo, routed Wd, shared Wd) multiplied by this factor
    out_scale: float = 1.0
    std: float = 0.02

    @property
    def qkv_dim(self) -> int:
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim


@dataclass(frozen=True)
class Workload:
    name: str
    shape: ModelShape
    batch: int
    prefix: int
    canvas: int = 256
    steps: int = 16
    tau0: float = 0.9
    tau1: float = 0.9          # linear schedule tau0 -> tau1 over the steps
    blocks: int = 1
    zipf_s: float = 0.0        # router skew exponent (0 = none)
    weight_seed: int = 0
    token_seed: int = 0
    sample_seed: int = 0
    temperature: float = 1.0
    description: str = ""

    def with_layers(self, n: int) -> "Workload":
        return replace(self, shape=replace(self.shape, n_layers=n),
                       name=f"{self.name}_L{n}")

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


_TINY = ModelShape(n_layers=2, d_model=256, n_q_heads=4, n_kv_heads=2, head_dim=64,
                   n_experts=16, top_k=2, expert_hidden=512, shared_hidden=512,
                   vocab=8192, out_scale=1.0 / math.sqrt(2 * 2))
_SMALL = ModelShape(n_layers=8, d_model=1024, n_q_heads=8, n_kv_heads=2, head_dim=128,
                    n_experts=32, top_k=4, expert_hidden=1024, shared_hidden=1024,
                    vocab=32768)
_A4B = ModelShape(n_layers=30, d_model=2816, n_q_heads=16, n_kv_heads=8, head_dim=176,
                  n_experts=128, top_k=8, expert_hidden=704, shared_hidden=2112,
                  vocab=262144)

WORKLOADS = {
    "tiny": Workload("tiny", _TINY, batch=1, prefix=128, steps=8, tau0=0.9, tau1=0.9,
                     description="tiny MoE decoder, 2 layers, d256, 16 experts top-2, V8192, "
                                 "prefix 128, 8 steps, tau 0.9"),
    "small": Workload("small", _SMALL, batch=1, prefix=1024, steps=16, tau0=0.95, tau1=0.5,
                      description="8 layers, d1024, 32 experts top-4, V32768, prefix 1024, "
                                  "16 steps, tau 0.95->0.5"),
    "a4b_p2k": Workload("a4b_p2k", _A4B, batch=1, prefix=2048, steps=16,
                        description="26B-A4B-shaped MoE (30 layers, d2816, 128 experts top-8 + "
                                    "shared, V262144), prefix 2048, batch 1, 256-token canvas"),
    "a4b_p32k": Workload("a4b_p32k", _A4B, batch=1, prefix=32768, steps=16,
                         description="26B-A4B-shaped MoE, prefix 32768, batch 1, 256-token canvas"),
    "a4b_blockar_b8": Workload("a4b_blockar_b8", _A4B, batch=8, prefix=4096, steps=24,
                               blocks=4, zipf_s=1.1,
                               description="26B-A4B-shaped MoE, batch 8, prefix 4096, 4 blocks of "
                                           "256, <=24 steps each, Zipf(1.1) router skew"),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def tau_schedule(w: Workload, step: int) -> float:
    """Threshold for denoising step `step` (linear from tau0 to tau1)."""
    if w.steps <= 1 or w.tau0 == w.tau1:
        return float(w.tau0)
    return float(w.tau0 + (w.tau1 - w.tau0) * step / (w.steps - 1))


# --------------------------------------------------------------------------
# counter-based 32-bit generator
# --------------------------------------------------------------------------
def _mix32_int(x: int) -> int:
    x &= MASK32
    x ^= x >> 16
    x = (x * 0x7FEB352D) & MASK32
    x ^= x >> 15
    x = (x * 0x846CA68B) & MASK32
    x ^= x >> 16
    return x


def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    # (x * c) mod 2^32 with every intermediate below 2^48 (no int64 overflow)
    lo = x * (c & 0xFFFF)
    hi = ((x * (c >> 16)) & 0xFFFF) << 16
    return (lo + hi) & MASK32


def _mix32(x: torch.Tensor) -> torch.Tensor:
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def _keys(seed: int, tid: int) -> tuple[int, int]:
    k1 = _mix32_int(seed ^ _mix32_int(tid * 0x9E3779B9 + 0x632BE5AB))
    k2 = _mix32_int(k1 ^ 0x85EBCA6B ^ (seed >> 32))
    return k1, k2


def hash_u32(seed: int, tid: int, start: int, n: int, device="cpu") -> torch.Tensor:
    """int64 tensor of n 32-bit hashes for flat indices [start, start+n)."""
    k1, k2 = _keys(seed, tid)
    idx = torch.arange(start, start + n, dtype=torch.int64, device=device)
    if start + n > (1 << 32):
        raise ValueError("flat index beyond 2^32")
    return _mix32(_mix32(idx ^ k1) ^ k2)


_TABLE_CACHE: dict = {}


def _irwin_hall_table(std: float, device) -> torch.Tensor:
    key = (std, str(device))
    if key not in _TABLE_CACHE:
        sigma = math.sqrt(4 * (256 * 256 - 1) / 12.0)
        vals = [(j - 510) * std / sigma for j in range(1021)]
        t = torch.tensor(vals, dtype=torch.float64).to(torch.float32).to(torch.bfloat16)
        _TABLE_CACHE[key] = t.to(device)
    return _TABLE_CACHE[key]


def _normalish(seed: int, tid: int, start: int, n: int, std: float, device) -> torch.Tensor:
    h = hash_u32(seed, tid, start, n, device)
    s = (h & 255) + ((h >> 8) & 255) + ((h >> 16) & 255) + ((h >> 24) & 255)
    return _irwin_hall_table(std, device)[s]


# tensor ids ----------------------------------------------------------------
_LAYER_NAMES = ["attn_norm", "wqkv", "wo", "ffn_norm", "w_router", "w_gate", "w_up",
                "w_down", "ws_gate", "ws_up", "ws_down"]
_GLOBAL_IDS = {"embed": 1_000_001, "final_norm": 1_000_002, "prefix": 2_000_001,
               "canvas": 2_000_002, "sc_gate": 1_000_003, "sc_up": 1_000_004, "sc_down": 1_000_005}
# the self-conditioning feed-forward layer: SwiGLU of the routed-expert width
_SELF_COND = ("sc_gate", "sc_up", "sc_down")


def tensor_id(name: str, layer: int | None = None) -> int:
    if layer is None:
        return _GLOBAL_IDS[name]
    return 1000 + layer * 32 + _LAYER_NAMES.index(name)


def layer_shapes(s: ModelShape) -> dict:
    d, E, F, Fs = s.d_model, s.n_experts, s.expert_hidden, s.shared_hidden
    return {
        "attn_norm": (d,), "wqkv": (s.qkv_dim, d), "wo": (d, s.n_q_heads * s.head_dim),
        "ffn_norm": (d,), "w_router": (E, d), "w_gate": (E, F, d), "w_up": (E, F, d),
        "w_down": (E, d, F), "ws_gate": (Fs, d), "ws_up": (Fs, d), "ws_down": (d, Fs),
    }


_OUT_PROJ = ("wo", "w_down", "ws_down")


def norm_weight(s: ModelShape, device="cpu") -> torch.Tensor:
    """RMSNorm gains are initialised to one."""
    return torch.ones(s.d_model, dtype=torch.bfloat16, device=device)


def weight(w: Workload, name: str, layer: int | None = None, device="cpu",
           rows: slice | None = None, chunk: int = 1 << 26) -> torch.Tensor:
    """One weight tensor (bf16).  `rows` selects a slice of the leading dim."""
    s = w.shape
    if name in ("attn_norm", "ffn_norm", "final_norm"):
        return norm_weight(s, device)
    if name == "embed":
        shape = (s.vocab, s.d_model)
    elif name in _SELF_COND:
        F = s.expert_hidden
        shape = (s.d_model, F) if name == "sc_down" else (F, s.d_model)
    else:
        shape = layer_shapes(s)[name]
    std = s.std * (s.out_scale if name in _OUT_PROJ else 1.0)
    inner = 1
    for x in shape[1:]:
        inner *= x
    r0, r1 = 0, shape[0]
    if rows is not None:
        r0, r1, _ = rows.indices(shape[0])
    n = (r1 - r0) * inner
    tid = tensor_id(name, layer)
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    base = r0 * inner
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        out[c0:c1] = _normalish(w.weight_seed, tid, base + c0, c1 - c0, std, device)
    return out.view((r1 - r0,) + tuple(shape[1:]))


def layer_weights(w: Workload, layer: int, device="cpu") -> dict:
    return {name: weight(w, name, layer, device) for name in _LAYER_NAMES}


def global_weights(w: Workload, device="cpu") -> dict:
    return {"embed": weight(w, "embed", None, device),
            "final_norm": norm_weight(w.shape, device),
            "router_bias": router_bias(w, device)}


def self_cond_weights(w: Workload, device="cpu") -> dict:
    """Weights of the self-conditioning feed-forward layer (bf16): sc_gate,
    sc_up [F, d] and sc_down [d, F], F the routed-expert width."""
    return {name: weight(w, name, None, device) for name in _SELF_COND}


def router_bias(w: Workload, device="cpu") -> torch.Tensor | None:
    """Zipf(s) skew of the router: expert e gets logit bias -s*ln(e+1) (fp32)."""
    if w.zipf_s == 0.0:
        return None
    b = [-w.zipf_s * math.log(e + 1.0) for e in range(w.shape.n_experts)]
    return torch.tensor(b, dtype=torch.float64).to(torch.float32).to(device)


def uniform_tokens(w: Workload, what: str, n_rows: int, n_cols: int, block: int = 0,
                   device="cpu") -> torch.Tensor:
    """int32 [n_rows, n_cols] tokens uniform over the vocabulary.

    `what` is "prefix" or "canvas"; `block` separates the initial canvases of
    consecutive blocks.
    """
    V = w.shape.vocab
    tid = tensor_id(what) + 7919 * block
    h = hash_u32(w.token_seed, tid, 0, n_rows * n_cols, device)
    if V & (V - 1) == 0:
        t = h & (V - 1)
    else:
        t = (h * V) >> 32
    return t.to(torch.int32).view(n_rows, n_cols)


def model_weights(w: Workload, device="cpu", layer_override=None, layers=None) -> dict:
    """All weights of workload `w` as bf16 tensors on `device`, in the layout of
    the C ABI (dg_weights / dg_layer_weights).  layer_override(l, dict) may
    replace tensors of a layer (planted cases)."""
    n = w.shape.n_layers if layers is None else layers
    out = global_weights(w, device)
    out["layers"] = []
    for l in range(n):
        t = layer_weights(w, l, device)
        if layer_override is not None:
            t = layer_override(l, t)
        out["layers"].append(t)
    return out
