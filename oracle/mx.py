"""FP8 expert weights for the oracle (test infrastructure only: nothing in the
product imports this module).

The pages measure the model at FP8 (codemajin.net "DiffusionGemma
architecture", section 5.2, H100 timings) and mention an 18 GB quantised model
(aibars.net), but give no format.  Reading taken here: MXFP8 as the OCP
Microscaling Formats (MX) specification v1.0 defines it, the FP8 format the
B200 tensor cores scale natively:

  * a block of 32 consecutive elements along the contraction (K) dimension
    shares one power-of-two scale X = 2^(floor(log2(max_i |x_i|)) - 8), where 8
    is the exponent of E4M3's largest normal (448 = 1.75 * 2^8); a block of
    zeros has X = 1;
  * each element is x_i / X rounded to nearest, ties to even, on the E4M3
    grid (sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals in
    steps of 2^-9, no infinities), saturating at +-448;
  * a product sums element products times the two blocks' scales; here it is
    formed exactly in float64 from the dequantised operands.

Both operands of an expert GEMM are quantised this way: the weight rows
([F, d] gate/up, [d, F] down: K contiguous) and the activation rows (the
normalised token rows for gate/up, the SwiGLU rows for down).  The shared
expert is quantised the same way; attention, the router and the LM head stay
bf16.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_EMAX = 8            # exponent of the largest normal
E4M3_MIN_NORMAL = 2.0 ** -6
E4M3_SUB_STEP = 2.0 ** -9
MX_BLOCK = 32


def e4m3_round(x) -> np.ndarray:
    """Nearest E4M3 value (ties to even), saturating at +-448; float64 in and out."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    # the step of the binade a lies in (3 mantissa bits), the subnormal step below 2^-6
    step = np.where(a >= E4M3_MIN_NORMAL, 2.0 ** (np.minimum(e, E4M3_EMAX) - 3), E4M3_SUB_STEP)
    q = np.round(a / step) * step            # numpy rounds halves to even
    q = np.minimum(q, E4M3_MAX)
    return np.copysign(q, x)


def mx_block_exponents(x: np.ndarray, block: int = MX_BLOCK) -> np.ndarray:
    """Shared exponent of every block of `block` elements along the last axis:
    floor(log2(max |x|)) - 8 (0 for an all-zero block)."""
    x = np.asarray(x, dtype=np.float64)
    assert x.shape[-1] % block == 0, "K must be a multiple of the block"
    amax = np.abs(x.reshape(*x.shape[:-1], -1, block)).max(axis=-1)
    _, e = np.frexp(amax)                    # amax = m * 2^e, m in [0.5, 1): floor(log2 amax) = e - 1
    return np.where(amax > 0, e - 1 - E4M3_EMAX, 0).astype(np.int64)


def mx_quantize(x: np.ndarray, block: int = MX_BLOCK):
    """(elements on the E4M3 grid, block exponents) of x along its last axis."""
    x = np.asarray(x, dtype=np.float64)
    ex = mx_block_exponents(x, block)
    scale = np.repeat(np.ldexp(1.0, ex), block, axis=-1)
    return e4m3_round(x / scale), ex


def mx_dequantize(elems: np.ndarray, exps: np.ndarray, block: int = MX_BLOCK) -> np.ndarray:
    return elems * np.repeat(np.ldexp(1.0, exps), block, axis=-1)


def mx_round_trip(x: np.ndarray, block: int = MX_BLOCK) -> np.ndarray:
    """x as its MXFP8 encoding represents it."""
    return mx_dequantize(*mx_quantize(x, block), block)


def mx_linear(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """x [n, K] times w [m, K]^T with both operands in MXFP8 along K."""
    return mx_round_trip(x) @ mx_round_trip(w).T


def mx_swiglu_ffn(x: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray) -> np.ndarray:
    """SwiGLU expert in MXFP8: SiLU(q(x) q(Wg)^T) * (q(x) q(Wu)^T), quantised
    again along F, times q(Wd)^T."""
    g = mx_linear(x, wg)
    h = g / (1.0 + np.exp(-g)) * mx_linear(x, wu)
    return mx_linear(h, wd)


def moe_mx(u: np.ndarray, lw, idx: np.ndarray, gates: np.ndarray) -> np.ndarray:
    """The oracle's MoE (shared expert plus gate-weighted routed experts) with
    every expert GEMM in MXFP8."""
    out = mx_swiglu_ffn(u, lw["ws_gate"], lw["ws_up"], lw["ws_down"])
    for e in np.unique(idx):
        rows, slots = np.nonzero(idx == e)
        y = mx_swiglu_ffn(u[rows], lw.expert(e, "w_gate"), lw.expert(e, "w_up"), lw.expert(e, "w_down"))
        out[rows] += gates[rows, slots][:, None] * y
    return out
