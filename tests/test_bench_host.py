"""Host-side pieces of bench.py: the code hash that ties an ncu traffic figure
under profiles/ to the kernel source it was taken from."""
from __future__ import annotations

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _write(tmp_path, name, text):
    p = tmp_path / name
    p.write_text(text, encoding="utf-8")
    return str(p)


def test_code_hash_ignores_comments_and_blank_lines(tmp_path):
    base = 'int f(int x) {\n  return x + 1;  // one more\n}\n'
    same = '// a header comment\n\nint f(int x) {\n  return x + 1;  // changed words\n}\n\n'
    other = 'int f(int x) {\n  return x + 2;  // one more\n}\n'
    a = bench._code_sha16(_write(tmp_path, "a.cu", base))
    b = bench._code_sha16(_write(tmp_path, "b.cu", same))
    c = bench._code_sha16(_write(tmp_path, "c.cu", other))
    assert a == b and a != c and len(a) == 16


def test_code_hash_keeps_slashes_inside_strings(tmp_path):
    # "//" inside a string literal is code, not a comment
    a = bench._code_sha16(_write(tmp_path, "a.cu", 'const char* s = "a//b";\n'))
    b = bench._code_sha16(_write(tmp_path, "b.cu", 'const char* s = "a//c";\n'))
    assert a != b
