"""Oracle for the block discrete-diffusion denoising step (TEST INFRASTRUCTURE ONLY).

A plain, slow, float64 CPU statement of what one denoising step, the causal
prefill and the block commit compute.  Only `tests/`, the `smoke()` entry of
`__graft_entry__` and the CPU-baseline leg of `bench.py` may import it; the
product path never does.  It shares no code with the CUDA library.

Sources ("DiffusionGemma Technical Report" as restated on five web pages):
  * codemajin.net "DiffusionGemma architecture", section 3.2: one weight-shared
    transformer used two ways: a causal encoder that turns the prompt and the
    committed blocks into a KV cache, and a bidirectional decoder that updates
    the whole 256-token block while attending to that cache; blocks are
    committed to the cache one after the other and never rewritten.
  * same page, section 3.1 (forward-process formula): at full noise every
    position is a uniformly random vocabulary token.
  * same page, section 3.3, and aibars.net "Uniform State Diffusion":
    confident predictions are accepted, the other positions are reset to
    uniformly random tokens; tokens of the current block may change again at
    later steps (section 3.2, multinomial diffusion).
  * same page, section 2.1: MoE, 128 experts of which 8 plus one shared expert
    are active per token, vocabulary ~262k.
  * aiboss88.com "hybrid attention architecture": prefill uses causal attention
    and writes the KV cache, denoising switches to bidirectional attention in
    which every canvas token sees every other one.
The pages leave the transformer's internals open; the readings taken here are
plain ones: pre-norm RMSNorm (gain initialised to one), rotate-half RoPE at
absolute positions, attention scale 1/sqrt(head_dim), GQA, top-k routing by
(logit desc, index asc) with a softmax over the k selected logits, an ungated
shared expert, SwiGLU experts, no embedding scaling, the LM head tied to the
embedding, confidence = maximum softmax probability.

Every function is written for clarity, not speed: each step below follows the
definition directly, with library matmuls as the only building block.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .mx import moe_mx
from .philox import philox4x32_10, uniform_token


# ---------------------------------------------------------------------------
# primitives
# ---------------------------------------------------------------------------
def rms_norm(h: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    """u = h / sqrt(mean(h^2) + eps) * gain, per row."""
    ms = np.mean(h * h, axis=-1, keepdims=True)
    return h / np.sqrt(ms + eps) * gain


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def rope_angles(positions: np.ndarray, head_dim: int, base: float):
    """cos/sin of angle pos * base^(-2j/D) for j < D/2 (rotate-half pairs j, j+D/2)."""
    half = head_dim // 2
    j = np.arange(half, dtype=np.float64)
    inv = base ** (-2.0 * j / head_dim)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv[None, :]
    return np.cos(ang), np.sin(ang)


def apply_rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate pairs (j, j+D/2) of x[..., n, D] by the angles of row n."""
    half = x.shape[-1] // 2
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, key_limit: np.ndarray) -> np.ndarray:
    """Grouped-query attention.

    q [Hq, n, D]; k, v [Hkv, S, D]; query row i sees keys j < key_limit[i].
    Returns o [n, Hq*D] (heads concatenated).
    """
    Hq, n, D = q.shape
    Hkv, S, _ = k.shape
    group = Hq // Hkv
    visible = np.arange(S)[None, :] < np.asarray(key_limit)[:, None]
    out = np.empty((n, Hq, D))
    for h in range(Hq):
        g = h // group
        s = q[h] @ k[g].T / np.sqrt(D)
        s = np.where(visible, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[g]
    return out.reshape(n, Hq * D)


def route_top_k(logits: np.ndarray, k: int):
    """Top-k experts per row ordered by (logit desc, index asc); gates are the
    softmax of the k selected logits.  Returns idx int64 [n,k], gates [n,k]."""
    n, E = logits.shape
    idx = np.empty((n, k), dtype=np.int64)
    for i in range(n):
        order = sorted(range(E), key=lambda e: (-logits[i, e], e))
        idx[i] = order[:k]
    return idx, selected_gates(logits, idx)


def selected_gates(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Softmax over the logits of the experts listed in idx [n, k]."""
    sel = np.take_along_axis(logits.astype(np.float64), np.asarray(idx, dtype=np.int64), axis=1)
    sel = sel - sel.max(axis=1, keepdims=True)
    g = np.exp(sel)
    return g / g.sum(axis=1, keepdims=True)


def swiglu_ffn(x: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray) -> np.ndarray:
    """(SiLU(x Wg^T) * (x Wu^T)) Wd^T with weights stored [out, in]."""
    return (silu(x @ wg.T) * (x @ wu.T)) @ wd.T


def moe(u: np.ndarray, lw, idx: np.ndarray, gates: np.ndarray) -> np.ndarray:
    """Shared expert (weight 1) plus the gate-weighted routed experts."""
    out = swiglu_ffn(u, lw["ws_gate"], lw["ws_up"], lw["ws_down"])
    for e in np.unique(idx):
        rows, slots = np.nonzero(idx == e)
        y = swiglu_ffn(u[rows], lw.expert(e, "w_gate"), lw.expert(e, "w_up"),
                       lw.expert(e, "w_down"))
        out[rows] += gates[rows, slots][:, None] * y
    return out


def lm_head_stats(z: np.ndarray, embed, temperature: float, row_chunk: int = 64,
                  vocab_chunk: int = 32768):
    """Per row of logits s = z E^T / T: max m, lowest argmax a, log-sum-exp,
    confidence exp(m - lse), log-probability m - lse, the top-1/top-2
    probability margin, the top-1/top-2 logit gap m - m2 and the entropy of
    the softmax, -sum_v p_v ln p_v = lse - sum_v p_v s_v (nats).  `embed` is
    the [V, d] tied embedding (any array or bf16 tensor); whole logit rows are
    formed before any statistic is taken."""
    n = z.shape[0]
    V = embed.shape[0]
    res = {k: np.empty(n) for k in ("max", "lse", "conf", "logp", "margin", "gap", "entropy")}
    res["argmax"] = np.empty(n, dtype=np.int64)
    logits = np.empty((min(n, row_chunk), V))
    for r0 in range(0, n, row_chunk):
        zr = z[r0:r0 + row_chunk]
        s = logits[:zr.shape[0]]
        for v0 in range(0, V, vocab_chunk):
            s[:, v0:v0 + vocab_chunk] = zr @ _f64(embed[v0:v0 + vocab_chunk]).T
        s /= temperature
        rows = np.arange(s.shape[0])
        a = np.argmax(s, axis=1)                      # first (lowest) index of the max
        m = s[rows, a]
        lse = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
        prob = np.exp(s - lse[:, None])
        ent = lse - (prob * s).sum(axis=1)
        s[rows, a] = -np.inf
        m2 = s.max(axis=1)
        sl = slice(r0, r0 + s.shape[0])
        res["argmax"][sl] = a
        res["max"][sl] = m
        res["lse"][sl] = lse
        res["conf"][sl] = np.exp(m - lse)
        res["logp"][sl] = m - lse
        res["margin"][sl] = np.exp(m - lse) - np.exp(m2 - lse)
        res["gap"][sl] = m - m2
        res["entropy"][sl] = ent
    return res


def self_condition(z: np.ndarray, embed, temperature: float, sc_gate, sc_up, sc_down,
                   row_chunk: int = 64, vocab_chunk: int = 32768) -> np.ndarray:
    """Self-conditioning signal of rows z [n, d] (codemajin.net "DiffusionGemma
    architecture", section 3.2): the predicted clean-token distribution
    p = softmax(z E^T / T) is passed through the embedding matrix, e = p E, and
    then through a small feed-forward layer, here SwiGLU:
    (SiLU(e Wg^T) * (e Wu^T)) Wd^T.  Returns [n, d]; the next step adds it to
    its input embeddings."""
    n, d = z.shape
    V = embed.shape[0]
    e = np.zeros((n, d))
    for r0 in range(0, n, row_chunk):
        zr = z[r0:r0 + row_chunk]
        s = np.empty((zr.shape[0], V))
        for v0 in range(0, V, vocab_chunk):
            s[:, v0:v0 + vocab_chunk] = zr @ _f64(embed[v0:v0 + vocab_chunk]).T
        s /= temperature
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        for v0 in range(0, V, vocab_chunk):
            e[r0:r0 + zr.shape[0]] += p[:, v0:v0 + vocab_chunk] @ _f64(embed[v0:v0 + vocab_chunk])
    return swiglu_ffn(e, _f64(sc_gate), _f64(sc_up), _f64(sc_down))


def renoise_tokens(positions, step: int, seq_ids, seed: int, vocab: int) -> np.ndarray:
    """Uniform replacement tokens: Philox4x32-10 with counter (absolute
    position, step, sequence, 0) and key (seed low word, seed high word)."""
    positions = np.asarray(positions, dtype=np.uint64)
    seq_ids = np.broadcast_to(np.asarray(seq_ids, dtype=np.uint64), positions.shape)
    w0, _, _, _ = philox4x32_10(positions, np.full(positions.shape, step, np.uint64),
                                seq_ids, np.zeros(positions.shape, np.uint64),
                                seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    return uniform_token(w0, vocab)


def sample(argmax: np.ndarray, conf: np.ndarray, tau: float, noise: np.ndarray) -> np.ndarray:
    """Keep the argmax where conf >= tau, else take the uniform draw (a NaN
    confidence re-noises)."""
    keep = np.asarray(conf) >= tau
    return np.where(keep, argmax, noise)


# ---------------------------------------------------------------------------
# entropy-constrained sampler (codemajin.net "DiffusionGemma architecture",
# section 3.3).  The page states: stop adaptively once the canvas's mean
# predicted entropy falls below a threshold AND the most likely token at every
# position is the one predicted at the previous step; otherwise accept tokens
# in order of low entropy and reset the rest to uniformly random tokens; the
# temperature falls linearly from 0.8 to 0.4; at most 48 steps.  It does not
# say how many tokens a step accepts; the sampler is called
# "entropy-constrained", read here as: the longest run of the lowest-entropy
# positions whose summed entropy stays within a budget gamma (at least one).
# Sums and comparisons are taken in float32, in the stated order, so that a
# decision is the same wherever it is taken from the same float32 entropies.
# ---------------------------------------------------------------------------
def anneal_temperature(step: int, max_steps: int = 48, t_first: float = 0.8, t_last: float = 0.4) -> float:
    """Temperature of denoising step `step` (0-based): linear from t_first at
    the first step to t_last at step max_steps - 1."""
    if max_steps <= 1:
        return t_first
    return t_first + (t_last - t_first) * step / (max_steps - 1)


def entropy_accept(entropy: np.ndarray, gamma: float) -> np.ndarray:
    """Boolean mask of the accepted positions of one canvas: positions taken
    in ascending (entropy, position) order while the float32 running sum of
    their entropies stays <= gamma; the first position is always taken."""
    e = np.asarray(entropy, dtype=np.float32)
    order = sorted(range(len(e)), key=lambda i: (e[i], i))
    acc = np.zeros(len(e), dtype=bool)
    run = np.float32(0.0)
    g = np.float32(gamma)
    for rank, i in enumerate(order):
        run = np.float32(run + e[i])
        if rank > 0 and not (run <= g):
            break
        acc[i] = True
    return acc


def mean_entropy(entropy: np.ndarray) -> np.float32:
    """Mean of one canvas's entropies: float32 sum in position order, / C."""
    run = np.float32(0.0)
    for x in np.asarray(entropy, dtype=np.float32):
        run = np.float32(run + x)
    return np.float32(run / np.float32(len(entropy)))


def entropy_sample(argmax: np.ndarray, entropy: np.ndarray, prev_argmax, gamma: float, stop_entropy: float,
                   noise: np.ndarray):
    """One canvas: returns (tokens, stopped).  stopped when prev_argmax is
    given (not the first step), the mean entropy is < stop_entropy and the
    argmax equals prev_argmax everywhere; then every position takes its
    argmax.  Otherwise the accepted positions take their argmax and the rest
    the uniform draws `noise`."""
    argmax = np.asarray(argmax)
    stopped = (prev_argmax is not None and bool(mean_entropy(entropy) < np.float32(stop_entropy))
               and bool(np.array_equal(argmax, np.asarray(prev_argmax))))
    if stopped:
        return argmax.copy(), True
    return np.where(entropy_accept(entropy, gamma), argmax, noise), False


def tokens_per_forward(total_tokens: int, total_steps: int, n_blocks: int) -> float:
    """TPF: generated tokens over (denoising steps + K - 1), the K - 1 being the
    extra forward that commits each finished block (codemajin.net section 5.1)."""
    return total_tokens / (total_steps + n_blocks - 1)


def tokens_per_second(tpf: float, t_fwd_s: float) -> float:
    """TPS = TPF / t_fwd (codemajin.net section 5.1)."""
    return tpf / t_fwd_s


# ---------------------------------------------------------------------------
# weights
# ---------------------------------------------------------------------------
class LayerWeights:
    """fp64 view of one layer's bf16 weights; routed experts are converted on
    demand so a 128-expert layer never sits in memory as fp64 all at once."""

    def __init__(self, tensors: dict):
        self._t = tensors
        self._cache = {}

    def __getitem__(self, name):
        if name not in self._cache:
            self._cache[name] = _f64(self._t[name])
        return self._cache[name]

    def expert(self, e: int, name: str) -> np.ndarray:
        return _f64(self._t[name][int(e)])

    def raw(self, name):
        return self._t[name]


def _index(tokens):
    try:
        import torch
        return torch.as_tensor(np.asarray(tokens, dtype=np.int64))
    except ImportError:  # pragma: no cover
        return np.asarray(tokens, dtype=np.int64)


def _f64(t) -> np.ndarray:
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float64)


@dataclass
class Shape:
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


# ---------------------------------------------------------------------------
# the model
# ---------------------------------------------------------------------------
@dataclass
class StepResult:
    canvas_out: np.ndarray
    conf: np.ndarray
    argmax: np.ndarray
    lse: np.ndarray
    logp: np.ndarray
    margin: np.ndarray
    hidden: list = field(default_factory=list)      # per layer boundary, [B, C, d]
    experts: list = field(default_factory=list)     # per layer, [B, C, k]
    router_logits: list = field(default_factory=list)
    router_margin: list = field(default_factory=list)  # k-th minus (k+1)-th logit
    gap: np.ndarray | None = None                    # top-1 minus top-2 logit (after /T)
    entropy: np.ndarray | None = None                # softmax entropy per position (nats)
    stopped: np.ndarray | None = None                # entropy sampler: adaptive stop per sequence
    self_cond: np.ndarray | None = None              # [B, C, d] signal for the next step (if enabled)
    forced_hidden: list = field(default_factory=list)  # teacher-forced layer outputs, [B, C, d]
    forced_experts: list = field(default_factory=list)  # top-k of given router rows, [B, C, k]
    forced_router_margin: list = field(default_factory=list)  # their k-th minus (k+1)-th logit
    forced_lm: dict | None = None                    # lm_head_stats of given LM-head rows, [B, C]


class Oracle:
    """Block discrete-diffusion decoder, fp64.

    layer_fn(l) -> dict of bf16 tensors for layer l (names as in the C ABI);
    embed: [V, d] bf16; router_bias: [E] fp32 or None.
    """

    def __init__(self, shape: Shape, layer_fn, embed, final_norm, router_bias=None,
                 batch: int = 1, keep_layers: bool = True, seq_ids=None, expert_format: str = "bf16"):
        self.s = shape
        # "bf16": experts as stored; "mxfp8": every expert GEMM with both
        # operands in MXFP8 (oracle/mx.py, the FP8 reading of section 5.2)
        assert expert_format in ("bf16", "mxfp8")
        self.expert_format = expert_format
        self.layer_fn = layer_fn
        self.embed = embed            # kept in storage precision; rows converted on use
        self.final_norm = _f64(final_norm)
        self.router_bias = None if router_bias is None else _f64(router_bias)
        self.B = batch
        # index of each of the oracle's sequences in the caller's batch (the
        # sampler's counter carries it): a subset of a batch can be checked
        self.seq_ids = np.arange(batch) if seq_ids is None else np.asarray(seq_ids)
        self.keep_layers = keep_layers
        self._layers = {}
        # KV cache per layer: list over sequences of (K [Hkv, P, D], V [Hkv, P, D])
        self.k_cache = [[np.zeros((shape.n_kv_heads, 0, shape.head_dim)) for _ in range(batch)]
                        for _ in range(shape.n_layers)]
        self.v_cache = [[np.zeros((shape.n_kv_heads, 0, shape.head_dim)) for _ in range(batch)]
                        for _ in range(shape.n_layers)]
        self.P = 0

    # -- weights --
    def layer(self, l: int) -> LayerWeights:
        if l in self._layers:
            return self._layers[l]
        last = getattr(self, "_last_layer", None)
        if last is not None and last[0] == l:
            return last[1]
        lw = LayerWeights(self.layer_fn(l))
        if self.keep_layers:
            self._layers[l] = lw
        else:
            self._last_layer = (l, lw)   # only the layer in use is held
        return lw

    # -- one transformer layer over new rows of one sequence --
    def _layer_forward(self, l: int, h: np.ndarray, b: int, pos0: int, causal: bool,
                       need_ffn: bool = True, dbg: dict | None = None, need_attn: bool = True,
                       forced_idx: np.ndarray | None = None):
        """One layer over n new rows at positions [pos0, pos0 + n).  Returns the
        updated residual and the rows' keys/values.  need_attn=False returns
        after the keys/values (h unchanged): the causal encoder's last layer
        only feeds the cache (codemajin.net "DiffusionGemma architecture",
        section 3.2).  forced_idx [n, k], when given, replaces the layer's own
        top-k choice by these experts (gates are still the softmax of this
        layer's logits at them): a test measures one layer's error on inputs
        and routing taken from elsewhere."""
        s = self.s
        lw = self.layer(l)
        n = h.shape[0]
        D, Hq, Hkv = s.head_dim, s.n_q_heads, s.n_kv_heads
        u = rms_norm(h, lw["attn_norm"], s.rms_eps)
        qkv = u @ lw["wqkv"].T
        q = qkv[:, :Hq * D].reshape(n, Hq, D).transpose(1, 0, 2)
        k = qkv[:, Hq * D:(Hq + Hkv) * D].reshape(n, Hkv, D).transpose(1, 0, 2)
        v = qkv[:, (Hq + Hkv) * D:].reshape(n, Hkv, D).transpose(1, 0, 2)
        cos, sin = rope_angles(np.arange(pos0, pos0 + n), D, s.rope_base)
        q = apply_rope(q, cos, sin)
        k = apply_rope(k, cos, sin)
        if not need_attn:
            return h, k, v
        keys = np.concatenate([self.k_cache[l][b][:, :pos0], k], axis=1)
        vals = np.concatenate([self.v_cache[l][b][:, :pos0], v], axis=1)
        if causal:
            limit = pos0 + 1 + np.arange(n)
        else:
            limit = np.full(n, pos0 + n)
        o = attention(q, keys, vals, limit)
        h = h + o @ lw["wo"].T
        if need_ffn:
            u2 = rms_norm(h, lw["ffn_norm"], s.rms_eps)
            r = u2 @ lw["w_router"].T
            if self.router_bias is not None:
                r = r + self.router_bias
            if forced_idx is None:
                idx, gates = route_top_k(r, s.top_k)
            else:
                idx = np.asarray(forced_idx, dtype=np.int64)
                gates = selected_gates(r, idx)
            h = h + (moe(u2, lw, idx, gates) if self.expert_format == "bf16" else moe_mx(u2, lw, idx, gates))
            if dbg is not None:
                dbg["idx"], dbg["logits"] = idx, r
                srt = -np.sort(-r, axis=1)
                dbg["margin"] = (srt[:, s.top_k - 1] - srt[:, s.top_k]
                                 if s.top_k < s.n_experts else np.full(n, np.inf))
        return h, k, v

    # -- causal encoder --
    def _causal_append(self, tokens: np.ndarray):
        """Causal forward of new rows at positions [P, P+n) for every sequence,
        appending their keys/values to the cache (the last layer's MoE does not
        feed the cache and is skipped)."""
        tokens = np.asarray(tokens)
        B, n = tokens.shape
        s = self.s
        for b in range(B):
            h = _f64(self.embed[_index(tokens[b])])
            for l in range(s.n_layers):
                last = l == s.n_layers - 1
                h, k, v = self._layer_forward(l, h, b, self.P, causal=True, need_ffn=not last,
                                              need_attn=not last)
                self.k_cache[l][b] = np.concatenate([self.k_cache[l][b][:, :self.P], k], axis=1)
                self.v_cache[l][b] = np.concatenate([self.v_cache[l][b][:, :self.P], v], axis=1)
        self.P += n

    def prefill(self, tokens: np.ndarray):
        """Reset the cache and encode the prompt causally."""
        s = self.s
        for l in range(s.n_layers):
            for b in range(self.B):
                self.k_cache[l][b] = np.zeros((s.n_kv_heads, 0, s.head_dim))
                self.v_cache[l][b] = np.zeros((s.n_kv_heads, 0, s.head_dim))
        self.P = 0
        self._causal_append(tokens)

    def commit_block(self, block: np.ndarray):
        """Append a finished block to the cache (one causal forward)."""
        self._causal_append(block)

    # -- bidirectional decoder + sampler --
    def denoise_step(self, canvas: np.ndarray, step: int, seed: int, tau: float,
                     temperature: float = 1.0, record: bool = True,
                     teacher: dict | None = None, self_cond_in=None,
                     sc_weights: dict | None = None) -> StepResult:
        """One denoising step of the canvas [B, C] (cache unchanged).

        teacher = {"hidden": [L+1 of [B, C, d]], "experts": [L of [B, C, k]]},
        when given, also runs every layer l on teacher["hidden"][l] with the
        experts teacher["experts"][l] and returns those outputs as
        forced_hidden[l + 1] (forced_hidden[0] is teacher["hidden"][0]): the
        error of each layer alone, free of the drift accumulated before it.
        Optional teacher["router_rows"] (L of [B, C, d], the normalised rows a
        layer's router consumed) give forced_experts / forced_router_margin,
        the top-k of those rows' logits; teacher["lm_rows"] ([B, C, d], the
        normalised rows the LM head consumed) give forced_lm, the LM-head
        statistics of those rows.

        Self-conditioning (codemajin.net section 3.2): self_cond_in [B, C, d]
        (the previous step's signal, or None at the first step of a block) is
        added to the input embeddings; with sc_weights (sc_gate, sc_up,
        sc_down) the step also returns self_cond, its own signal for the next
        step."""
        canvas = np.asarray(canvas)
        B, C = canvas.shape
        s = self.s
        hidden = [np.empty((B, C, s.d_model)) for _ in range(s.n_layers + 1)] if record else []
        experts = [np.empty((B, C, s.top_k), dtype=np.int64) for _ in range(s.n_layers)] if record else []
        rlog = [np.empty((B, C, s.n_experts)) for _ in range(s.n_layers)] if record else []
        rmar = [np.empty((B, C)) for _ in range(s.n_layers)] if record else []
        z = np.empty((B, C, s.d_model))
        forced, f_exp, f_mar, f_lm = [], [], [], None
        if teacher is not None:
            forced = [np.asarray(teacher["hidden"][0], dtype=np.float64)]
            forced += [np.empty((B, C, s.d_model)) for _ in range(s.n_layers)]
            if teacher.get("router_rows") is not None:
                f_exp = [np.empty((B, C, s.top_k), dtype=np.int64) for _ in range(s.n_layers)]
                f_mar = [np.empty((B, C)) for _ in range(s.n_layers)]
        for b in range(B):
            h = _f64(self.embed[_index(canvas[b])])
            if self_cond_in is not None:
                h = h + np.asarray(self_cond_in[b], dtype=np.float64)
            if record:
                hidden[0][b] = h
            for l in range(s.n_layers):
                dbg = {}
                h, _, _ = self._layer_forward(l, h, b, self.P, causal=False, dbg=dbg)
                if teacher is not None:
                    hf, _, _ = self._layer_forward(
                        l, np.asarray(teacher["hidden"][l][b], dtype=np.float64), b, self.P,
                        causal=False, forced_idx=teacher["experts"][l][b])
                    forced[l + 1][b] = hf
                    if teacher.get("router_rows") is not None:
                        rr = np.asarray(teacher["router_rows"][l][b], dtype=np.float64) @ \
                            self.layer(l)["w_router"].T
                        if self.router_bias is not None:
                            rr = rr + self.router_bias
                        fi, _ = route_top_k(rr, s.top_k)
                        srt = -np.sort(-rr, axis=1)
                        f_exp[l][b] = fi
                        f_mar[l][b] = (srt[:, s.top_k - 1] - srt[:, s.top_k] if s.top_k < s.n_experts
                                       else np.inf)
                if record:
                    hidden[l + 1][b] = h
                    experts[l][b] = dbg["idx"]
                    rlog[l][b] = dbg["logits"]
                    rmar[l][b] = dbg["margin"]
            z[b] = rms_norm(h, self.final_norm, s.rms_eps)
        st = lm_head_stats(z.reshape(B * C, s.d_model), self.embed, temperature)
        sc_next = None
        if sc_weights is not None:
            sc_next = self_condition(z.reshape(B * C, s.d_model), self.embed, temperature, sc_weights["sc_gate"],
                                     sc_weights["sc_up"], sc_weights["sc_down"]).reshape(B, C, s.d_model)
        if teacher is not None and teacher.get("lm_rows") is not None:
            zf = np.asarray(teacher["lm_rows"], dtype=np.float64).reshape(B * C, s.d_model)
            f_lm = {k: v.reshape(B, C) for k, v in lm_head_stats(zf, self.embed, temperature).items()}
        pos = np.tile(np.arange(self.P, self.P + C), B)
        seq = np.repeat(self.seq_ids[:B], C)
        noise = renoise_tokens(pos, step, seq, seed, s.vocab)
        out = sample(st["argmax"], st["conf"], tau, noise)
        rs = lambda a: a.reshape(B, C)
        return StepResult(canvas_out=rs(out), conf=rs(st["conf"]), argmax=rs(st["argmax"]),
                          lse=rs(st["lse"]), logp=rs(st["logp"]), margin=rs(st["margin"]),
                          hidden=hidden, experts=experts, router_logits=rlog,
                          router_margin=rmar, gap=rs(st["gap"]), entropy=rs(st["entropy"]),
                          forced_hidden=forced,
                          forced_experts=f_exp, forced_router_margin=f_mar, forced_lm=f_lm,
                          self_cond=sc_next)


def _entropy_step(self, canvas, step: int, seed: int, temperature: float, gamma: float, stop_entropy: float,
                  prev_argmax=None, record: bool = True, teacher: dict | None = None) -> StepResult:
    """One denoising step with the entropy-constrained sampler (codemajin.net
    section 3.3): the forward pass at this step's temperature, then per
    sequence the adaptive stop test against prev_argmax [B, C] (None at the
    first step of a block) or the entropy-ordered acceptance; re-noised
    positions take the same Philox draws as the threshold sampler."""
    r = self.denoise_step(canvas, step, seed, np.inf, temperature=temperature, record=record, teacher=teacher)
    B, C = r.argmax.shape
    noise = renoise_tokens(np.tile(np.arange(self.P, self.P + C), B), step, np.repeat(self.seq_ids[:B], C),
                           seed, self.s.vocab).reshape(B, C)
    out = np.empty_like(r.argmax)
    stopped = np.zeros(B, dtype=bool)
    for b in range(B):
        prev = None if prev_argmax is None else np.asarray(prev_argmax)[b]
        out[b], stopped[b] = entropy_sample(r.argmax[b], r.entropy[b].astype(np.float32), prev, gamma,
                                            stop_entropy, noise[b])
    r.canvas_out = out
    r.stopped = stopped
    return r


Oracle.denoise_step_entropy = _entropy_step
