"""The source hash that keys the DRAM traffic recorded for each bench kernel:
comment and whitespace edits keep it, code edits change it."""

import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402

CODE = 'int f(int a) {\n    return a + 1;  // one more\n}\n/* a\n   block */ const char* s = "x//y /* z */";\n'


def test_comments_and_whitespace_do_not_count():
    edited = CODE.replace("// one more", "// a different remark").replace("/* a\n   block */", "/* other */")
    edited = edited.replace("    return", "\treturn")
    assert bench.code_of(edited) == bench.code_of(CODE)


def test_code_edits_count():
    assert bench.code_of(CODE.replace("a + 1", "a + 2")) != bench.code_of(CODE)
    # a comment marker inside a string literal is code
    assert bench.code_of(CODE.replace('"x//y /* z */"', '"x//y /* w */"')) != bench.code_of(CODE)

