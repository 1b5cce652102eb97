"""Host arithmetic of bench.py's per-kernel roofline rows (no GPU).

A row turns per-launch times into TFLOP/s (or GB/s), the fraction of the
measured peak (8-bit rows against twice the bf16 peak, the nominal ratio) and
the fraction of the nominal roofline max(FLOPs / dense rate, bytes / 8 TB/s).
"""
import math

import bench

PEAKS = (1600.0, 1400.0, 6500.0, "measured")


def test_tensor_row_bf16():
    # 1 TFLOP in 1 ms: 1000 TFLOP/s
    r = bench.kernel_row("k", "coda_x", [1.0, 1.0, 1.0], 1e12, 1e9, "tensor", 1, "bf16", None, PEAKS, None)
    assert math.isclose(r["tflops"], 1000.0)
    assert math.isclose(r["frac"], 1000.0 / 1600.0, rel_tol=1e-3)
    assert math.isclose(r["frac_of_sustained"], 1000.0 / 1400.0, rel_tol=1e-3)
    # nominal: max(1e12 / 2.25e15 s, 1e9 / 8e12 s) = 0.444 ms of 1 ms
    assert math.isclose(r["roofline_ms_nominal"], 1e12 / 2.25e15 * 1e3, rel_tol=1e-3)
    assert math.isclose(r["frac_of_nominal_roofline"], 0.4444, rel_tol=1e-3)


def test_eight_bit_rows_take_twice_the_bf16_peak():
    for dt in ("e4m3", "mxfp8"):
        r = bench.kernel_row("k", "coda_x", [0.5], 1e12, 1e9, "tensor", 1, dt, None, PEAKS, None)
        assert math.isclose(r["tflops"], 2000.0)
        assert math.isclose(r["peak"], 3200.0)
        assert math.isclose(r["frac"], 2000.0 / 3200.0, rel_tol=1e-3)
        assert math.isclose(r["roofline_ms_nominal"], 1e12 / 4.5e15 * 1e3, rel_tol=1e-3)
        assert "x 2" in r["peak_kind"] and dt in r["peak_kind"]


def test_hbm_row_and_clock_cycles():
    clk = {"sm_mhz": 1500.0, "reasons": ["sw_power_cap"]}
    r = bench.kernel_row("q", "coda_mx_quantize", [0.02, 0.03], 0.0, 1e8, "hbm", 1, "bf16", "note", PEAKS, clk)
    assert math.isclose(r["ms"], 0.025)
    assert math.isclose(r["gbs"], 1e8 / 0.025 / 1e6)          # 4000 GB/s
    assert r["unit"] == "GB/s" and math.isclose(r["frac"], 4000.0 / 6500.0, rel_tol=1e-3)
    assert math.isclose(r["kcycles"], 0.025 * 1500.0)          # ms x MHz = thousands of cycles
    assert r["reasons"] == ["sw_power_cap"] and r["note"] == "note"
    assert r["ms_median"] == 0.03 and r["ms_min"] == 0.02


def test_device_code_hash_ignores_comments_only():
    src = '''// a comment with "quotes" and 'ticks'
    asm volatile("mov.u64 %0, %%globaltimer; // not a comment" : "=l"(t));  /* block
    comment */ x = '/'; y = "a\\"b//c";
'''
    got = bench.strip_comments(src)
    assert got.count("\n") == src.count("\n")
    assert '"mov.u64 %0, %%globaltimer; // not a comment"' in got
    assert "'/'" in got and '"a\\"b//c"' in got
    assert "comment with" not in got and "block" not in got
    # the same code with other comments strips to the same text
    other = src.replace("a comment with", "another remark,").replace("block\n    comment", "x\n    y")
    assert bench.strip_comments(other) == got
    assert bench.strip_comments(src.replace("x = '/'", "x = '+'")) != got
