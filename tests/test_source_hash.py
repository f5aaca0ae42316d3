"""The source hash that keys recorded ncu counters covers code, not comments:
comment edits keep it, any code edit changes it."""
import os

from attention_qk_norm_b200 import buildlib


def test_code_only_drops_comments_and_keeps_literals():
    text = ('int a = 1; // one\n/* block\n comment */ const char *s = "x // y /* z */";\n'
            "char c = '/'; const char *t = \"it's \\\" // still\";  \t\n")
    assert buildlib.code_only(text) == (
        'int a = 1; const char *s = "x // y /* z */"; char c = \'/\'; '
        'const char *t = "it\'s \\" // still";')


def test_hash_follows_code_only():
    files = {p: open(p, encoding="utf-8").read() for p in buildlib.kernel_sources()}
    base = buildlib.kernel_source_sha256(lambda p: files[p])
    some = sorted(files)[0]
    commented = dict(files)
    commented[some] = "// a new comment line\n" + files[some].replace("\n", "  \n", 3)
    assert buildlib.kernel_source_sha256(lambda p: commented[p]) == base
    changed = dict(files)
    changed[some] = files[some] + "\nstatic const int qkn_extra = 1;\n"
    assert buildlib.kernel_source_sha256(lambda p: changed[p]) != base
    assert all(os.path.basename(p).endswith((".cu", ".cuh", ".h")) for p in files)
