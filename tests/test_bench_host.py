"""Host-side logic of bench.py that needs no GPU: the code hash that ties a
committed ncu profile to the kernel sources it was captured on, and the
profile fields the bench reads back."""
import os
import re

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_strip_comments_keeps_code_and_literals():
    src = ('int a = 1; // trailing\n/* block\n comment */ int b = 2;\n'
           'asm("mov.u32 %0, 1; // not a comment"); char c = \'"\'; const char* s = "/*x*/";\n')
    out = bench.strip_comments(src)
    assert "trailing" not in out and "block" not in out
    assert "int a = 1;" in out and "int b = 2;" in out
    assert '"mov.u32 %0, 1; // not a comment"' in out
    assert "'\"'" in out and '"/*x*/"' in out


def test_comment_and_layout_edits_keep_the_hash_code_edits_change_it():
    base = "__device__ int f(int x) {\n  return x + 1;  // one more\n}\n"
    same = "// a new header line\n__device__ int f(int x)\n{\n    return x + 1; /* still one */\n}\n"
    other = "__device__ int f(int x) {\n  return x + 2;  // one more\n}\n"
    assert bench.strip_comments(base) == bench.strip_comments(same)
    assert bench.strip_comments(base) != bench.strip_comments(other)


def test_committed_profiles_name_a_hash_and_traffic():
    """Every per-kernel profile records the code hash and the per-launch DRAM
    bytes bench.py reads; a profile whose hash matches today's sources gives
    a positive traffic figure."""
    current = {k: bench.source_hash(k) for k in bench.KERNEL_SOURCES}
    pdir = os.path.join(ROOT, "profiles")
    seen = 0
    for name in sorted(os.listdir(pdir)):
        kernel = next((k for k in current if name.startswith(k)), None)
        if kernel is None:
            continue
        text = open(os.path.join(pdir, name)).read()
        h = re.search(r"source_sha256: `([0-9a-f]{16})`", text)
        b = re.search(r"dram_bytes_per_launch_full: `(\d+)`", text)
        assert h and b, name
        if h.group(1) == current[kernel]:
            assert bench.profile_traffic(name[:-3]) > 0
            seen += 1
    assert seen > 0
