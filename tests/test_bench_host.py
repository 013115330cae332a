"""Host logic of bench.py that needs no GPU: the code hash that ties a
recorded ncu traffic figure to the sources of the kernel it was taken on."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_comments_do_not_change_the_code():
    code = 'int a = 1; // note\n/* block\n   comment */ const char *s = "x // y /* z */";\nchar q = \'\\\'\';\n'
    stripped = bench.strip_c_comments(code)
    assert "note" not in stripped and "block" not in stripped
    assert '"x // y /* z */"' in stripped and "'\\''" in stripped
    assert bench.strip_c_comments(code.replace("note", "other note")) == stripped
    assert bench.strip_c_comments(code.replace("a = 1", "a = 2")) != stripped


def test_traffic_records_name_existing_sources():
    recs = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    assert recs
    for key, rec in recs.items():
        assert rec["dram_bytes_per_launch"] > 0, key
        assert len(bench.kernel_source_hash(rec["sources"])) == 16, key
