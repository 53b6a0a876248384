"""Host-side helpers of bench.py (no GPU): the comment-insensitive source hash that ties a
recorded DRAM-traffic figure to the code it was measured on."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_comments_and_layout_do_not_change_the_code():
    a = "int a = 1;\nint b = a + 2; // add\n"
    b = "/* header\n * lines */\nint a =   1;   int b = a + 2;\n"
    assert bench.strip_c_comments(a) == bench.strip_c_comments(b)


def test_comment_markers_inside_literals_are_code():
    src = 'const char* s = "x // y /* z */"; char q = \'"\'; char e = \'\\\'\'; // tail'
    out = bench.strip_c_comments(src)
    assert '"x // y /* z */"' in out and "tail" not in out and "char e = '\\''" in out


def test_code_changes_do_change_the_stripped_text():
    assert bench.strip_c_comments("int a = 1;") != bench.strip_c_comments("int a = 2;")
    assert bench.strip_c_comments("a+b") != bench.strip_c_comments("a + b")



def test_the_recorded_dram_traffic_belongs_to_the_current_kernels():
    """profiles/dram_traffic.md's record carries the hash of the grouped-GEMM sources it
    was measured on; while those sources are unchanged bench.py reports its figures, and
    they are at least the algorithmic bytes of the kernels (each weight byte read once)."""
    gu = bench.recorded_traffic("mixtral_prefill", "moe_expert_gate_up")
    dn = bench.recorded_traffic("mixtral_prefill", "moe_expert_down")
    assert gu is not None and dn is not None, "the record's source hash no longer matches the GEMM sources"
    w13 = 8 * 2 * 14336 * 4096 * 2
    w2 = 8 * 4096 * 14336 * 2
    assert w13 <= gu <= 1.2 * (w13 + 2 * 8192 * 4096 * 2 + 8192 * 14336 * 2)
    assert w2 <= dn
    assert bench.recorded_traffic("no_such_workload", "moe_expert_gate_up") is None


def test_dispatch_path_names_match_the_library():
    import combine_warp_top_expert_b200 as moe
    assert bench.DISPATCH_PATHS == {"auto": moe.DISPATCH_AUTO, "two_pass": moe.DISPATCH_TWO_PASS,
                                    "one_pass": moe.DISPATCH_ONE_PASS}
