"""Host side of the timeline (tracing) build: libdg_timeline.so exports the
same functions as libdg.so, the record layout matches the header, and the
launch sequence and per-kernel totals are rebuilt correctly from per-CTA
records (no device needed)."""
import ctypes
import os
import re

import numpy as np

import block_discrete_diffusion_denoise_b200 as dgp
from block_discrete_diffusion_denoise_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DT = np.dtype([("t0_ns", "<u8"), ("t1_ns", "<u8"), ("kernel", "<i4"), ("cta", "<i4")])


def test_timeline_library_exports_the_same_functions():
    build.build()
    lib = ctypes.CDLL(dgp.TIMELINE_LIB_PATH)
    for name in dgp.EXPORTS:
        assert hasattr(lib, name), name
    assert lib.dg_debug_timeline_reset(None) == 1      # DG_ERR_INVALID_ARG, no device touched
    n = ctypes.c_int64(5)
    assert lib.dg_debug_timeline(None, None, 0, ctypes.byref(n)) == 1


def test_record_layout_and_kernel_ids_match_the_header():
    assert ctypes.sizeof(dgp.dg_timeline_record) == 24 == DT.itemsize
    src = open(os.path.join(ROOT, "include", "dg.h")).read()
    ids = {int(v): k for k, v in re.findall(r"\b(DG_K_[A-Z_]+)\s*=\s*(\d+)", src)}
    assert set(ids) == set(dgp.TIMELINE_KERNELS)
    for v, name in ids.items():
        assert name[len("DG_K_"):].lower() == dgp.TIMELINE_KERNELS[v]


def _rec(rows):
    a = np.zeros(len(rows), DT)
    for i, (t0, t1, k) in enumerate(rows):
        a[i] = (t0, t1, k, i)
    return a


def test_launches_are_rebuilt_from_shuffled_cta_records():
    # three launches: dense (2 CTAs), dense again after it ended (a new launch), attention
    rows = [(100, 900, 10), (120, 1000, 10), (1300, 1800, 10), (1310, 2000, 10), (2500, 4000, 20),
            (2600, 3900, 20)]
    rng = np.random.default_rng(0)
    rec = _rec(rows)[rng.permutation(len(rows))]
    L = dgp.timeline_launches(rec)
    assert [(l["name"], l["t0_ns"], l["t1_ns"], l["ctas"]) for l in L] == [
        ("gemm_dense", 100, 1000, 2), ("gemm_dense", 1300, 2000, 2), ("attention", 2500, 4000, 2)]
    s = dgp.timeline_summary(L)
    assert s["launches"] == 3
    assert abs(s["wall_us"] - 3.9) < 1e-12
    assert abs(s["gaps_us"] - (0.3 + 0.5)) < 1e-12
    d = s["kernels"]["gemm_dense"]
    assert d["launches"] == 2 and abs(d["total_us"] - 1.6) < 1e-12 and abs(d["avg_us"] - 0.8) < 1e-12
    assert abs(d["gaps_before_us"] - 0.3) < 1e-12
    a = s["kernels"]["attention"]
    assert abs(a["total_us"] - 1.5) < 1e-12 and abs(a["share"] - 1.5 / 3.9) < 1e-12


def test_overlapping_ctas_of_one_kernel_stay_one_launch():
    # a CTA that starts before another of the same launch ends belongs to it
    rec = _rec([(0, 50, 11), (10, 60, 11), (55, 90, 11), (95, 99, 31)])
    L = dgp.timeline_launches(rec)
    assert [(l["name"], l["ctas"]) for l in L] == [("gemm_moe", 3), ("combine_norm", 1)]
    assert dgp.timeline_summary([])["launches"] == 0
