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


def test_bank_bytes_per_expert():
    """Algorithmic bytes of one expert (gate, up, down) per format: the bench's roofline
    numerators (d 2560, f 1024)."""
    import bench
    from expert_routed_ffn_route_b200 import synth
    cfg = synth.CONFIGS["prefill"]
    n = 3 * cfg.d * cfg.f
    assert bench.bank_bytes_per_expert(cfg, "int4") == (n // 2, n // 128 * 2)
    assert bench.bank_bytes_per_expert(cfg, "int8") == (n, n // 128 * 2)
    assert bench.bank_bytes_per_expert(cfg, "bf16") == (2 * n, 0)
    assert bench.bank_bytes_per_expert(cfg, "nvfp4") == (n // 2, n // 16 + 12)
    assert sum(bench.bank_bytes_per_expert(cfg, "int4")) == 4_055_040


def test_committed_traffic_summaries_match_the_sources():
    """The committed ncu summaries that feed roofline.traffic carry digests of the current
    kernel sources, and their byte counts are close to the algorithmic bytes they cover."""
    import bench
    dec = bench.profiled_traffic("decode", "decode_fused")
    pre = bench.profiled_traffic("prefill", "tc_grouped")
    nv = bench.profiled_traffic("prefill_nvfp4", "nv_grouped")
    assert dec is not None and abs(dec / 47.24e6 - 1) < 0.01
    assert pre is not None and 1.3e9 < pre < 1.5e9
    assert nv is not None and 1.5e9 < nv < 1.6e9


def test_workload_config_is_the_same_for_both_arms():
    import bench
    from expert_routed_ffn_route_b200 import synth
    for name in bench.ALL_WORKLOADS:
        cfg = synth.CONFIGS[name]
        a = bench.workload_config(cfg, 1)
        assert a == bench.workload_config(cfg, 1)
        assert a["workload"] == name and a["T"] == cfg.T
