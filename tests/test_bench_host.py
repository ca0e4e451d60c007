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
