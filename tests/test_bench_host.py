"""Host-side arithmetic of bench.py, on CPU: the step's algorithmic bytes and
FLOPs (the roofline's numerator) and the clock sampler's timed window."""
import datetime
import tempfile

import pytest

import bench
import synth_inputs as si


def test_step_cost_matches_an_independent_count_of_the_26b_shape():
    """With every expert hit, the 26B-A4B step reads the whole model once plus
    the KV cache.  The count below is done parameter by parameter:

    - per layer, attention 23.79 M (QKV 5632 x 2816 plus O 2816 x 2816),
      router 0.36 M, 128 experts x 5.95 M, shared expert 17.84 M;
    - the tied LM head, 738 M;
    - the KV cache, 30 layers x (P + 256) keys x 8 heads x 176 x 2 (K and V)
      in bf16."""
    w = si.workload("a4b_p2k")
    by, fl, moe = bench.step_cost(w, [128] * 30)
    per_layer = (5632 * 2816 + 2816 * 2816) + 128 * 2816 + 128 * 3 * 704 * 2816 + 3 * 2112 * 2816
    weights = (30 * per_layer + 262144 * 2816) * 2
    kv = 30 * (2048 + 256) * 8 * 176 * 2 * 2
    assert by == weights + kv
    assert by / 1e9 == pytest.approx(50.06, abs=0.01)
    # FLOPs: 2 x active parameters per canvas token + attention 4*Hq*D*C*(P+C)*L
    active = 30 * ((5632 + 2816) * 2816 + 128 * 2816 + 8 * 3 * 704 * 2816 + 3 * 2112 * 2816) + 262144 * 2816
    assert fl == pytest.approx(2 * active * 256 + 4 * 16 * 176 * 256 * (2048 + 256) * 30)
    assert fl / 1e12 == pytest.approx(1.953, abs=0.001)
    assert moe == pytest.approx(128 * 3 * 704 * 2816 * 2 + 3 * 2112 * 2816 * 2)


def test_step_cost_counts_only_the_experts_hit_and_grows_with_the_cache():
    w = si.workload("a4b_p2k")
    full, _, _ = bench.step_cost(w, [128] * 30)
    half, _, _ = bench.step_cost(w, [64] * 30)
    assert full - half == 30 * 64 * 3 * 704 * 2816 * 2
    by32, fl32, _ = bench.step_cost(si.workload("a4b_p32k"), [128] * 30)
    assert by32 - full == 30 * (32768 - 2048) * 8 * 176 * 2 * 2
    assert fl32 / 1e12 == pytest.approx(4.611, abs=0.001)


class _DoneProcess:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def kill(self):
        pass


def _clocks_with_rows(rows):
    c = bench.Clocks.__new__(bench.Clocks)
    c.index = 0
    c.p = _DoneProcess()
    c.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
    c.f.write("\n".join(rows) + "\n")
    c.f.flush()
    return c


def _row(t, mhz, reasons=("Not Active",) * 4):
    stamp = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return ", ".join([stamp, "0", str(mhz), "1965", "700.00", "0x0"] + list(reasons))


def test_clock_samples_are_kept_inside_the_timed_window_only():
    t0 = 1_800_000_000.0
    rows = [_row(t0 - 1.0, 400),                      # warm-up, before the window
            _row(t0 + 0.05, 1965), _row(t0 + 0.10, 1950), _row(t0 + 0.15, 1965),
            _row(t0 + 2.0, 300, ("Not Active", "Not Active", "Active", "Not Active"))]  # after
    clk = _clocks_with_rows(rows).stop(t0, t0 + 0.2)
    assert clk["samples"] == 3
    assert clk["sm_mhz"] == 1965.0 and clk["sm_max_mhz"] == 1965.0
    assert clk["reasons"] == []


def test_clock_reasons_inside_the_window_are_reported():
    t0 = 1_800_000_000.0
    rows = [_row(t0 + 0.05, 1500, ("Not Active", "Not Active", "Not Active", "Active")),
            _row(t0 + 0.10, 1520, ("Not Active", "Not Active", "Not Active", "Active"))]
    clk = _clocks_with_rows(rows).stop(t0, t0 + 0.2)
    assert clk["reasons"] == ["sw_power_cap"]
    assert clk["sm_mhz"] == 1510.0


def test_mode_flags_parse_and_the_timeline_mode_selects_the_tracing_build(monkeypatch):
    """--timeline, --variants and --batch-sweep are modes with JSON lines of
    their own; --timeline points the binding at libdg_timeline.so before the
    package is imported (main() sets DG_LIBRARY)."""
    import sys
    monkeypatch.setattr(sys, "argv", ["bench.py", "--timeline", "--steps", "2"])
    args = bench.parse()
    assert args.timeline and not args.variants and args.steps == 2
    monkeypatch.setattr(sys, "argv", ["bench.py", "--variants"])
    assert bench.parse().variants
    monkeypatch.setattr(sys, "argv", ["bench.py", "--batch-sweep", "1,2"])
    assert bench.parse().batch_sweep == "1,2"
    src = open(bench.__file__).read()
    assert 'os.environ["DG_LIBRARY"] = os.path.join(ROOT, "block_discrete_diffusion_denoise_b200", "libdg_timeline.so")' in src


@pytest.mark.parametrize("mode", ["bounded", "full"])
def test_reference_arm_line_on_the_tiny_workload(mode, capsys):
    """--impl reference prints one line on the oracle's own clock: the bounded
    sample extrapolates to the full step; --reference-sample full times whole
    steps, so its value is the canvas over the measured step time."""
    import argparse
    import json
    args = argparse.Namespace(gpus=1, steps=1, warmup=0, reference_sample=mode)
    bench.run_reference(args, si.workload("tiny"))
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["dtype"] == "f64" and line["unit"] == bench.UNIT
    assert line["e2e"]["value"] == line["value"] == line["cpu_baseline"]["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    if mode == "full":
        assert "whole step" in line["cpu_baseline"]["sample"]
        assert line["value"] == pytest.approx(256 / line["step_seconds"][0], rel=1e-2)
        assert line["ms_per_step"] == pytest.approx(line["step_seconds"][0] * 1e3, rel=1e-2)
    else:
        assert line["extrapolated_ms_per_full_step"] > line["ms_per_step"] > 0
        assert line["value"] == pytest.approx(256 / (line["extrapolated_ms_per_full_step"] * 1e-3))


def test_code_hash_ignores_comments_and_layout_but_not_code(tmp_path):
    """The traffic record stays valid across comment edits of the kernel
    source and lapses with any code edit."""
    src = ("// header comment\n#include \"common.cuh\"\n/* block\n comment */\n"
           "constexpr int A = 4;  // trailing\n__global__ void k(int* p) { p[0] = A; }\n")
    variants = {
        "same": src,
        "comments": src.replace("header comment", "another header").replace("trailing", "changed"),
        "layout": src.replace("constexpr int A = 4;", "constexpr   int A =\n    4;"),
        "code": src.replace("A = 4", "A = 5"),
        "code in body": src.replace("p[0] = A", "p[1] = A"),
    }
    h = {}
    for name, text in variants.items():
        f = tmp_path / f"{name}.cuh"
        f.write_text(text)
        h[name] = bench.code_sha256(str(f))
    assert h["same"] == h["comments"] == h["layout"]
    assert h["code"] != h["same"] and h["code in body"] != h["same"]


def test_l2_note_follows_the_step_bytes():
    by, _, _ = bench.step_cost(si.workload("a4b_p2k"), [77] * 30)
    assert bench.l2_note(by).startswith("inputs larger than L2 (3") and "no flush" in bench.l2_note(by)
    tiny, _, _ = bench.step_cost(si.workload("tiny"), [16, 16])
    assert bench.l2_note(tiny).startswith("inputs fit in L2 (32 MB")
