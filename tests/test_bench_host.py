"""Host-side arithmetic of bench.py's roofline object (no GPU): which step
time each timing mode reports, and the step overhead derived from it."""
import bench as B
from workloads import mla_workloads as W

PEAKS = {"hbm_gbs": 6545.0, "bf16_tflops": 1627.8}


def _measured(flushed):
    # 10 steps back to back in 1.2 ms; 0.105 ms between events around one
    # whole step; the decode kernel alone 0.1 ms
    return {"kernel_ms": 0.1, "combine_ms": 0.008, "metadata_ms": 0.009, "total_ms": 1.2, "steps": 10,
            "step_chained_ms": 0.105, "flushed": flushed, "clocks": {"sm_mhz": 1900.0}, "rows": 16}


def test_step_time_back_to_back_without_flush():
    r = B.roofline_of(W.make_inputs(W.get_workload("tiny")), _measured(False), PEAKS, "measured")
    assert abs(r["step_ms"] - 0.12) < 1e-12
    assert abs(r["step_overhead_ms"] - 0.02) < 1e-12


def test_step_time_between_events_with_flush():
    # the 256 MB L2 flush runs before each step, outside the step's events
    r = B.roofline_of(W.make_inputs(W.get_workload("tiny")), _measured(True), PEAKS, "measured")
    assert abs(r["step_ms"] - 0.105) < 1e-12
    assert abs(r["step_overhead_ms"] - 0.005) < 1e-12


def test_roofline_fraction_of_the_kernel_time():
    inp = W.make_inputs(W.get_workload("tiny"))
    work = W.algorithmic_work(inp)
    r = B.roofline_of(inp, _measured(False), PEAKS, "measured")
    assert r["bound"] == "hbm"
    assert abs(r["achieved"] - work["bytes"] / 1e-4 / 1e9) < 1e-6 * r["achieved"]
    assert abs(r["frac"] - r["achieved"] / PEAKS["hbm_gbs"]) < 1e-12


def test_kernel_hash_ignores_comments_but_not_code():
    code = "int f(int x) { return x + 1; }  // add one\n"
    a = B.strip_c_comments("/* header\n   two lines */\n" + code)
    b = B.strip_c_comments("// another header\n\n" + code.replace("// add one", "/* plus one */"))
    assert a == b == "int f(int x) { return x + 1; }"
    assert B.strip_c_comments(code.replace("x + 1", "x + 2")) != a
    # comment markers inside string literals (inline PTX) are code
    ptx = 'asm volatile("mov.b32 %0, 1; // kept /* kept */" : "=r"(v));'
    assert B.strip_c_comments(ptx) == ptx
    assert B.strip_c_comments("char q = '\"'; int y; // c") == "char q = '\"'; int y;"
