"""The C-ABI library builds, loads without a GPU and exports every function
that include/dg.h declares (no compute call is made here)."""
import ctypes
import os
import re

import block_discrete_diffusion_denoise_b200 as dgp
from block_discrete_diffusion_denoise_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "dg.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dg_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    build.build()
    lib = ctypes.CDLL(dgp.LIB_PATH)
    declared = _declared()
    assert len(declared) >= 17
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(dgp.EXPORTS) == declared


def test_binding_declares_signatures():
    lib = dgp.load_library()
    assert lib.dg_last_error(None) == b"null context"
    assert lib.dg_cached_len(None) == -1
    assert lib.dg_debug_launch_count(None) == -1
    assert lib.dg_sync(None) == 1          # DG_ERR_INVALID_ARG, no device touched


def test_config_struct_matches_header_field_order():
    src = open(os.path.join(ROOT, "include", "dg.h")).read()
    body = src[src.index("typedef struct dg_config"):src.index("} dg_config;")]
    names = re.findall(r"\b(?:int32_t|float)\s+([a-z_]+);", body)
    assert names == [n for n, _ in dgp.dg_config._fields_]
    body = src[src.index("typedef struct dg_layer_weights"):src.index("} dg_layer_weights;")]
    names = re.findall(r"const void\*\s+([a-z_]+);", body)
    assert names == dgp.LAYER_FIELDS


def _tiny_config(**over):
    import synth_inputs as si
    cfg = dgp.config_from_shape(si.workload("tiny").shape, max_batch=1, max_seq=512, canvas=256)
    cfg.update(over)
    c = dgp.dg_config()
    for name, _ in dgp.dg_config._fields_:
        setattr(c, name, cfg[name])
    return c


def _fake_weights(n_layers, null_field=None):
    """Host addresses, 16-byte aligned and never dereferenced: dg_create checks
    shapes and pointers before it touches a device."""
    layers = (dgp.dg_layer_weights * n_layers)()
    for i in range(n_layers):
        for j, f in enumerate(dgp.LAYER_FIELDS):
            setattr(layers[i], f, None if f == null_field else 0x10000 + 0x100 * (i * 16 + j))
    w = dgp.dg_weights(embed=0x200000, final_norm=0x300000, router_bias=None,
                       layers=ctypes.cast(layers, ctypes.POINTER(dgp.dg_layer_weights)))
    return w, layers


def _create(cfg, w):
    lib = dgp.load_library()
    out = ctypes.c_void_p()
    st = lib.dg_create(ctypes.byref(cfg), ctypes.byref(w), None, ctypes.byref(out))
    return st, out.value, lib.dg_last_error(None).decode()


def test_create_rejects_unsupported_shapes_without_a_device():
    w, keep = _fake_weights(2)
    cases = {
        "head_dim": dict(head_dim=96),                      # not in {64, 128, 176}
        "gqa group vs attention tile": dict(n_q_heads=6, n_kv_heads=2),   # group 3 does not divide 128
        "experts": dict(n_experts=300, top_k=2),            # > 256
        "canvas": dict(canvas=200),                         # not a multiple of 16
        "d_model": dict(d_model=320),                       # not a multiple of 128
        "max_seq": dict(max_seq=128),                       # shorter than the canvas
        "d_model too wide": dict(d_model=4224),             # a row kernel holds at most 4096
        "vocab": dict(vocab=8000),                          # not a multiple of 128
        "expert width": dict(expert_hidden=500),            # not a multiple of 64
        "shared width": dict(shared_hidden=96 + 1),
        "experts not a multiple of 4": dict(n_experts=18),
        "top-k beyond 16": dict(n_experts=32, top_k=17),
        "top-k beyond the experts": dict(top_k=20),
        "canvas beyond 256": dict(canvas=272),
    }
    for what, over in cases.items():
        st, ctx, msg = _create(_tiny_config(**over), w)
        assert st == 7 and ctx is None, (what, st)          # DG_ERR_UNSUPPORTED, no context
        assert msg == "dg_create: unsupported shape", (what, msg)


def test_create_rejects_workspaces_beyond_the_row_limit_without_a_device():
    w, keep = _fake_weights(2)
    for over in (dict(max_batch=129), dict(prefill_rows=40000)):     # more than 32768 rows
        st, ctx, msg = _create(_tiny_config(**over), w)
        assert (st, ctx) == (7, None) and "32768" in msg, (over, st, msg)


def test_create_rejects_bad_arguments_without_a_device():
    w, keep = _fake_weights(2)
    st, ctx, msg = _create(_tiny_config(n_layers=0), w)
    assert (st, ctx) == (1, None) and "non-positive" in msg
    st, ctx, msg = _create(_tiny_config(temperature=0.0), w)
    assert (st, ctx) == (1, None) and "non-positive" in msg
    w2, keep2 = _fake_weights(2, null_field="w_down")
    st, ctx, msg = _create(_tiny_config(), w2)
    assert (st, ctx) == (1, None) and "layer weight" in msg
    w3 = dgp.dg_weights(embed=None, final_norm=0x300000, router_bias=None, layers=w.layers)
    st, ctx, msg = _create(_tiny_config(), w3)
    assert (st, ctx) == (1, None) and "null weights" in msg
    lib = dgp.load_library()
    assert lib.dg_create(None, ctypes.byref(w), None, None) == 1
    assert lib.dg_last_error(None) == b"dg_create: null argument"


def test_every_call_refuses_a_null_context_without_a_device():
    """Each entry point checks its context (and, for the no-allocation LM
    head, its operands) before anything else: with NULL it returns
    DG_ERR_INVALID_ARG, or -1 for the two counters, and touches no device."""
    lib = dgp.load_library()
    for name in dgp.EXPORTS:
        if name == "dg_create":
            continue                                   # its NULL arguments: test_create_rejects_bad_arguments
        f = getattr(lib, name)
        args = [None] * len(f.argtypes)
        for i, t in enumerate(f.argtypes):
            if t in (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64):
                args[i] = 0
            elif t is ctypes.c_float:
                args[i] = 0.0
        res = f(*args)
        if name in ("dg_cached_len", "dg_debug_launch_count"):
            assert res == -1, name
        elif name == "dg_last_error":
            assert isinstance(res, bytes), name
        else:
            assert res == 1, (name, res)


def test_static_lmhead_refuses_bad_arguments_without_a_device():
    """dg_lmhead_argmax_static checks shapes, alignment, temperature, outputs
    and its fixed scratch capacity before it asks for a device (the addresses
    below are never dereferenced)."""
    lib = dgp.load_library()
    z, e, out = 0x100000, 0x200000, ctypes.cast(0x300000, ctypes.POINTER(ctypes.c_int32))

    def call(n_rows=256, d=2816, vocab=262144, temp=1.0, zp=z, ep=e, am=out):
        return lib.dg_lmhead_argmax_static(zp, n_rows, d, ep, vocab, temp, am, None, None, None)

    assert call(d=100) == 1                      # d_model not a multiple of 64
    assert call(vocab=1000) == 1                 # vocab not a multiple of 128
    assert call(n_rows=0) == 1
    assert call(temp=0.0) == 1 and call(temp=float("nan")) == 1
    assert call(zp=z + 8) == 1 and call(ep=e + 4) == 1      # not 16-byte aligned
    assert call(zp=None) == 1
    assert call(am=None) == 1                    # no output at all
    assert call(n_rows=257) == 3                 # 257 x 262144 / 128 partials exceed the fixed scratch
