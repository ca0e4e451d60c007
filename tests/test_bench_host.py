"""Host-side logic of bench.py that needs no GPU: the code hash that keys the
committed DRAM-traffic figures to the kernel sources they were measured on."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_tokens_drops_comments_and_layout_only():
    src = ('asm volatile("ld.global.nc.v4.u32 {%0}, [%1]; // not a comment");  // comment\n'
           "int a = 1; /* block\n comment */ int b = '/';\n"
           '   const char* s = "/* kept */";   \n')
    assert bench.code_tokens(src) == (
        'asm volatile("ld.global.nc.v4.u32 {%0}, [%1]; // not a comment"); '
        "int a = 1; int b = '/'; const char* s = \"/* kept */\";")
    # an escaped quote does not end a string literal
    assert bench.code_tokens('x = "a\\"//b"; // c') == 'x = "a\\"//b";'


def test_code_changes_change_the_hash(tmp_path):
    d = tmp_path / "csrc"
    d.mkdir()
    (d / "k.cuh").write_text("int f() { return 1; }  // one\n")
    h0 = bench.kernel_source_hash(str(d))
    (d / "k.cuh").write_text("// reworded\nint f()  {\n  return 1;\n}\n")
    assert bench.kernel_source_hash(str(d)) == h0, "comments and layout are not code"
    (d / "k.cuh").write_text("int f() { return 2; }\n")
    assert bench.kernel_source_hash(str(d)) != h0
    (d / "k.cuh").write_text("int f() { return 1; }\n")
    (d / "notes.txt").write_text("ignored")
    assert bench.kernel_source_hash(str(d)) == h0, "only .cu / .cuh files count"


def test_traffic_is_reported_only_for_the_measured_kernels():
    """An entry of profiles/dram_traffic.json yields a figure exactly when its
    recorded code hash is that of the kernels in the tree."""
    import json
    d = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    now = bench.kernel_source_hash()
    for name, e in d.items():
        assert e["dram_bytes_per_launch"] > 0 and e["command"].startswith("ncu "), name
        got = bench.dram_traffic(name)
        assert got == (float(e["dram_bytes_per_launch"]) if e["csrc_sha256_16"] == now else None)
    assert bench.dram_traffic("no such workload") is None


def test_oracle_parity_leg_accepts_the_oracle_and_flags_a_planted_error():
    """The bench's parity report on the oracle's own outputs passes; a flipped
    code byte or a Y element off by far more than the tolerance fails it
    (the plant is made in the oracle's copy, on the CPU)."""
    import types

    import numpy as np
    import torch

    import oracle as orc
    name = "decode:3:256:384"
    o, w = bench.oracle_workload(name)
    amax = o.tensor_amax(w["x_bits"])
    qa = o.quantize(np.ascontiguousarray(w["x_bits"]), global_in=o.global_from_amax(amax))
    y = torch.from_numpy(o.gemm(qa, w["qw"])).to(torch.bfloat16)
    A = types.SimpleNamespace(codes=torch.from_numpy(qa.codes.copy()),
                              sf=torch.from_numpy(qa.sf_swizzled.copy()),
                              global_scale=torch.tensor([float(qa.g)], dtype=torch.float32), k=256)
    step = types.SimpleNamespace(y=y, A=A)
    good = bench.sample_outputs(step)
    rep = bench.oracle_parity(orc, w, name, good)
    assert rep["pass"] and rep["x_codes_scales_global_bit_exact"] and rep["rows"] == 3
    assert rep["y_rel_fro"] == 0.0

    bad = dict(good, codes=good["codes"].copy())
    bad["codes"][1, 7] ^= 0x01
    rep = bench.oracle_parity(orc, w, name, bad)
    assert not rep["pass"] and not rep["x_codes_scales_global_bit_exact"]

    bad = dict(good, y=good["y"].copy())
    bad["y"][2, 5] += 1.0e3
    rep = bench.oracle_parity(orc, w, name, bad)
    assert not rep["pass"] and rep["y_worst_excess_over_elem_bound"] > 0


def test_clock_summary_window_and_reasons():
    """The clock record: median SM clock and the throttle reasons seen in the
    timed window (extended by the extra second of the same step), idle
    samples outside it ignored; too few samples fall back to the whole run."""
    s = bench.ClockSampler(0)

    def row(mhz, power_cap="Not Active", thermal="Not Active"):
        return f"0, {mhz}, 1965, 900.0, 0x4, Not Active, Not Active, {thermal}, {power_cap}"

    s.samples = [(0.0, row(345)), (0.5, row(345))]                  # idle before the run
    s.samples += [(1.0 + 0.1 * i, row(1700 + i, power_cap="Active")) for i in range(10)]
    s.samples += [(5.0, row(300, thermal="Active"))]                 # idle after the run
    c = s.summary(1.0, 2.0, extended=True)
    assert c["samples"] == 10 and c["sm_mhz"] == 1704.5 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"] and c["window"].startswith("timed region + 1 s")
    c = s.summary(1.0, 1.15)                                         # 2 samples: whole run
    assert c["samples"] == 13 and c["window"].startswith("whole run")
    assert c["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]
    s.samples = [(1.0, "garbage"), (1.1, "0, N/A, N/A")]
    c = s.summary(0.0, 2.0)                                          # no usable sample
    assert c["sm_mhz"] is None and c["samples"] == 0 and "error" in c


def test_clock_sample_uses_nvidia_smi_timestamp():
    import time
    line = "2026/12/02 21:25:18.250, 0, 1700, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active\n"
    t, rest = bench.ClockSampler.parse(line, arrival=123.0)
    assert abs(t - (time.mktime(time.strptime("2026/12/02 21:25:18", "%Y/%m/%d %H:%M:%S")) + 0.25)) < 1e-6
    assert rest.startswith("0, 1700, 1965")
    assert bench.ClockSampler.parse("no stamp, 0, 1700", arrival=123.0) == (123.0, "0, 1700")


def test_linear_launch_count_follows_the_dispatch():
    """gpu_launches of the decode and linear lines: one kernel for at most 8
    tokens (quantized inside the GEMM), plus the quantizer above 8 tokens,
    plus the amax pass for a dynamic global over more than 64 KiB of X."""
    assert bench.linear_launches(1, 5120, False) == 1
    assert bench.linear_launches(8, 4096, False) == 1      # exactly 64 KiB
    assert bench.linear_launches(8, 5120, False) == 2      # amax pass
    assert bench.linear_launches(8, 5120, True) == 1       # static global
    assert bench.linear_launches(9, 2048, False) == 2      # quantizer takes the max
    assert bench.linear_launches(32, 5120, False) == 3
    assert bench.linear_launches(8192, 5120, True) == 2
    assert bench.linear_launches(8192, 5120, False) == 3
