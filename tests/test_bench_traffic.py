"""Host-side checks of how bench.py keys its DRAM-traffic records to the kernel code: a
record stays valid across comment and whitespace edits and is dropped when the code
changes; every committed record names sources that exist."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_comments_and_whitespace_do_not_count():
    a = "int f(int x) {\n    return x + 1;  // one more\n}\n"
    b = "/* the successor */\nint f(int x)\n{ return x + 1; }\n"
    assert bench._code_only(a) == bench._code_only(b)


def test_code_changes_count():
    assert bench._code_only("return x + 1;") != bench._code_only("return x + 2;")
    assert bench._code_only("a = b;") != bench._code_only("a = c;")


def test_string_and_char_literals_are_code():
    # comment markers inside literals are not comments; spaces inside them are kept
    assert bench._code_only('s = "// x";') == 's="// x";'
    assert bench._code_only('s = "a b";') != bench._code_only('s = "ab";')
    assert bench._code_only("c = '/'; // tail") == "c='/';"
    assert bench._code_only('s = "\\" // still a string";') == 's="\\" // still a string";'


def test_committed_records_name_existing_sources():
    d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    assert d, "no traffic records"
    for key, e in d.items():
        kernel, workload = key.split(":")
        assert e["bytes_per_launch"] > 0, key
        for n in e["sources"]:
            assert os.path.exists(os.path.join(ROOT, "bit_grouped_moe_gnf4_b200", "csrc", n)), (key, n)
        got = bench.recorded_traffic(kernel, workload)
        assert got is None or got == e["bytes_per_launch"], key
