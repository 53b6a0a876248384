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

