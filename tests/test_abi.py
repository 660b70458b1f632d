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
