"""Pins of the oracle's MXFP8 expert path (oracle/mx.py): E4M3 rounding
against torch's float8_e4m3fn conversion, the MX block scale's closed forms
(OCP MX specification v1.0), the per-block error bound, exact products on
representable inputs, and the MoE structure (k = E reduces to the dense
gate-weighted mixture of MXFP8 experts)."""
import numpy as np
import torch

from oracle import model as om
from oracle import mx

rng = np.random.default_rng(11)


def test_e4m3_round_matches_torch_inside_the_finite_range():
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    x = np.concatenate([x, np.ldexp(rng.uniform(1, 2, 2000), rng.integers(-12, 9, 2000))])
    x = x[np.abs(x) < 464.0]                 # torch turns |x| >= 464 into NaN; MX saturates (below)
    # torch converts a float64 tensor to E4M3 through float32, so a value
    # within half a float32 ulp of an E4M3 midpoint would be rounded twice
    # there; on the float32 grid both sides round once
    x = x.astype(np.float32).astype(np.float64)
    ref = torch.tensor(x, dtype=torch.float64).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(mx.e4m3_round(x), ref)
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    codes = codes[np.isfinite(codes)]
    np.testing.assert_array_equal(mx.e4m3_round(codes), codes)   # every code point is its own rounding


def test_e4m3_saturation_and_subnormal_ties():
    np.testing.assert_array_equal(mx.e4m3_round([460.0, 464.0, 1000.0, -1e9]), [448.0, 448.0, 448.0, -448.0])
    # 2^-10 is halfway between 0 and the smallest subnormal 2^-9: ties to even gives 0
    np.testing.assert_array_equal(mx.e4m3_round([2.0 ** -10, 3 * 2.0 ** -10, 2.0 ** -9]), [0.0, 2.0 ** -8, 2.0 ** -9])
    assert mx.e4m3_round(-0.0) == 0.0


def test_block_exponent_closed_forms():
    for k in (-20, -3, 0, 5, 30):
        b = np.zeros((1, 32))
        b[0, 7] = 448.0 * 2.0 ** k
        assert mx.mx_block_exponents(b)[0, 0] == k
        b[0, 7] = 256.0 * 2.0 ** k           # any max in [256, 512) * 2^k shares exponent k
        assert mx.mx_block_exponents(b)[0, 0] == k
        b[0, 7] = 511.9 * 2.0 ** k
        assert mx.mx_block_exponents(b)[0, 0] == k
    assert mx.mx_block_exponents(np.zeros((2, 64))).tolist() == [[0, 0], [0, 0]]
    x = rng.standard_normal((3, 256)) * np.exp(rng.uniform(-8, 8, (3, 1)))
    ex = mx.mx_block_exponents(x)
    scaled_max = np.abs(x.reshape(3, 8, 32)).max(axis=-1) / np.ldexp(1.0, ex)
    assert ((scaled_max >= 256) & (scaled_max < 512)).all()


def test_round_trip_error_is_bounded_per_block():
    # blocks of very different magnitude: each is scaled on its own, so every
    # element keeps the relative precision of 3 mantissa bits (or the
    # subnormal step of its own block, or saturation at 448 * its scale)
    mags = np.exp(rng.uniform(-15, 15, (4, 8)))
    x = rng.standard_normal((4, 8, 32)) * mags[..., None]
    x = x.reshape(4, 256)
    y = mx.mx_round_trip(x)
    np.testing.assert_array_equal(mx.mx_round_trip(y), y)          # idempotent
    ex = np.repeat(mx.mx_block_exponents(x), 32, axis=-1)
    scale = np.ldexp(1.0, ex)
    bound = np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * scale)  # half a step, normal or subnormal
    bound = np.maximum(bound, np.abs(x) - 448.0 * scale)           # saturation of the block maximum
    assert (np.abs(x - y) <= bound * (1 + 1e-12)).all()
    # blocks far below their row's maximum keep their precision (one scale per
    # row instead of per block would flush them to zero)
    small = np.abs(x) < 1e-6 * np.abs(x).max(axis=-1, keepdims=True)
    assert small.any()
    assert (y[small] != 0).mean() > 0.9


def test_mx_linear_is_exact_on_representable_operands():
    # integers in [-8, 8] with an 8 in every block: the scale is 2^-5 and every
    # scaled element (a multiple of 32 up to 256) is an E4M3 value
    def ints(shape):
        a = rng.integers(-8, 9, shape).astype(np.float64)
        a.reshape(*shape[:-1], -1, 32)[..., 0] = 8.0
        return a
    x, w = ints((5, 96)), ints((7, 96))
    np.testing.assert_array_equal(mx.mx_linear(x, w), x @ w.T)


def test_mx_linear_worked_example_by_hand():
    """One 32-element block each, worked by hand.  x = (448, 1.06, 0...):
    max 448 = 1.75 * 2^8 gives exponent 0, scale 1; 448 is on the grid, 1.06
    lies in [1, 2) where the step is 1/8, nearest 1.0.  w = (1, 0.53, 0...):
    max 1 gives exponent -8, scale 2^-8; 0.53 * 256 = 135.68 lies in
    [128, 256) where the step is 16, nearest 128, i.e. 0.5.  So the product
    is 448 * 1 + 1.0 * 0.5 = 448.5, where unquantised operands give 448.5618."""
    x = np.zeros((1, 32))
    x[0, :2] = (448.0, 1.06)
    w = np.zeros((1, 32))
    w[0, :2] = (1.0, 0.53)
    assert mx.mx_block_exponents(x).tolist() == [[0]] and mx.mx_block_exponents(w).tolist() == [[-8]]
    np.testing.assert_array_equal(mx.mx_round_trip(x)[0, :2], [448.0, 1.0])
    np.testing.assert_array_equal(mx.mx_round_trip(w)[0, :2], [1.0, 0.5])
    assert mx.mx_linear(x, w)[0, 0] == 448.5


def test_moe_with_all_experts_is_the_dense_mixture_of_mxfp8_experts():
    d, F, E = 64, 32, 4

    class LW:
        def __init__(self):
            self.t = {n: rng.standard_normal(s) * 0.3 for n, s in
                      (("ws_gate", (F, d)), ("ws_up", (F, d)), ("ws_down", (d, F)),
                       ("w_gate", (E, F, d)), ("w_up", (E, F, d)), ("w_down", (E, d, F)))}

        def __getitem__(self, n):
            return self.t[n]

        def expert(self, e, n):
            return self.t[n][e]

    lw = LW()
    u = rng.standard_normal((6, d))
    logits = rng.standard_normal((6, E))
    idx, gates = om.route_top_k(logits, E)
    got = mx.moe_mx(u, lw, idx, gates)
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    ref = mx.mx_swiglu_ffn(u, lw["ws_gate"], lw["ws_up"], lw["ws_down"])
    for e in range(E):
        ref = ref + p[:, e:e + 1] * mx.mx_swiglu_ffn(u, lw.expert(e, "w_gate"), lw.expert(e, "w_up"),
                                                     lw.expert(e, "w_down"))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    # and it is the bf16 MoE up to the quantisation: a few per cent here, not zero
    exact = om.moe(u, lw, idx, gates)
    rel = np.linalg.norm(got - exact) / np.linalg.norm(exact)
    assert 1e-4 < rel < 0.2, rel


def test_oracle_step_with_mxfp8_experts_on_the_tiny_workload():
    """The step with MXFP8 experts is the bf16 step with moe replaced by
    moe_mx: the embedding is untouched, the layers move by the quantisation
    (E4M3 keeps 3 mantissa bits: ~3% rms per operand element, three GEMMs per
    expert, so 5-10% of the residual update), and a planted identity (every
    output projection zero) is still a fixed point."""
    import oracle
    import synth_inputs as si
    w = si.workload("tiny").with_(prefix=16)
    prefix = si.uniform_tokens(w, "prefix", 1, 16).numpy()
    canvas = si.uniform_tokens(w, "canvas", 1, 256).numpy()
    res = {}
    for fmt in ("bf16", "mxfp8"):
        o = oracle.for_workload(w, expert_format=fmt)
        o.prefill(prefix)
        res[fmt] = o.denoise_step(canvas, 0, 1, 0.9)
    a, b = res["bf16"], res["mxfp8"]
    np.testing.assert_array_equal(a.hidden[0], b.hidden[0])
    d = [np.linalg.norm(a.hidden[l] - b.hidden[l]) / np.linalg.norm(a.hidden[l] - a.hidden[0])
         for l in (1, 2)]
    assert all(1e-3 < x < 0.25 for x in d), d

    def zero_out(l, t):
        t = dict(t)
        for k in ("wo", "w_down", "ws_down"):
            t[k] = t[k] * 0
        return t
    o = oracle.for_workload(w, layer_override=zero_out, expert_format="mxfp8")
    o.prefill(prefix)
    r = o.denoise_step(canvas, 0, 1, 0.9, temperature=0.05)
    np.testing.assert_array_equal(r.argmax, canvas)
