"""Host-side helpers of bench.py (no GPU): the kernel-source digest that ties committed ncu
counters to the code they were taken from."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_source_tokens_drop_comments_keep_literals():
    src = 'int a; // note\n/* block\n comment */ const char* s = "//kept /* too */";\n'
    assert bench.source_tokens(src) == 'int a; const char* s = "//kept /* too */";'


def test_digest_ignores_comments_and_tracks_code():
    files = {name: open(os.path.join(ROOT, "expert_routed_ffn_route_b200", "csrc", name)).read()
             for name in bench.KERNEL_SOURCES["tc_grouped"]}
    base = bench.kernel_source_digest("tc_grouped", files.__getitem__)
    assert base == bench.kernel_source_digest("tc_grouped")
    commented = dict(files)
    commented["common.cuh"] = "// a new comment\n" + files["common.cuh"].replace("\n", "\n\n", 3)
    assert bench.kernel_source_digest("tc_grouped", commented.__getitem__) == base
    changed = dict(files)
    changed["common.cuh"] = files["common.cuh"] + "\nconstexpr int kProbe = 1;\n"
    assert bench.kernel_source_digest("tc_grouped", changed.__getitem__) != base
