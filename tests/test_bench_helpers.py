"""Host-side helpers of bench.py (CPU only): the kernel-source digest that
keys the committed traffic figures, the L2-flush rule and the shape options."""
import os
import sys
import types

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_code_only_drops_comments_and_blank_space_but_keeps_code():
    a = 'int a = 1; // note\n/* block\n comment */ int b = "s//t";\n'
    b = 'int a = 1;\n\n  int b = "s//t"; // another note\n'
    assert bench.code_only(a) == bench.code_only(b) == 'int a = 1; int b = "s//t";'
    assert bench.code_only("int a = 1;") != bench.code_only("int a = 2;")
    assert bench.code_only('x = "/* not a comment */";') == 'x = "/* not a comment */";'


def test_source_digest_is_stable_and_covers_the_kernel_files():
    d = bench.source_digest()
    assert len(d) == 16 and d == bench.source_digest()
    csrc = os.path.join(bench.ROOT, "paged_kv_cache_372_b200", "csrc")
    for name in bench.KERNEL_SOURCES:
        assert os.path.exists(os.path.join(csrc, name))


def test_committed_traffic_matches_the_current_kernels():
    # every committed entry names the digest of the sources it was captured on
    import json
    with open(bench.PROFILE_TRAFFIC) as f:
        entries = {k: v for k, v in json.load(f).items() if isinstance(v, dict)}
    assert entries
    for key, e in entries.items():
        assert e["dram_bytes_per_launch"] > 0
        assert os.path.exists(os.path.join(os.path.dirname(bench.PROFILE_TRAFFIC), e["summary"]))
        if e["source_digest"] == bench.source_digest():
            assert bench.profiled_traffic(key) == e["dram_bytes_per_launch"]


def test_shape_options_only_for_the_decode_batches():
    args = types.SimpleNamespace(block_size=32, head_dim=None, kv_heads=None, workload="llama7b")
    assert bench.shape_args(args) == {"block_size": 32}
    args = types.SimpleNamespace(block_size=None, head_dim=64, kv_heads=None, workload="llama3_8b")
    assert bench.shape_args(args) == {"head_dim": 64}
    args = types.SimpleNamespace(block_size=None, head_dim=None, kv_heads=4, workload="llama3_8b")
    assert bench.shape_args(args) == {"kv_heads": 4}
    from paged_kv_cache_372_b200 import workloads
    wl = workloads.llama3_8b(0, num_seqs=4, kv_heads=4)
    assert (wl.num_heads, wl.num_kv_heads, wl.name) == (32, 4, "llama3_8b_kv4")
    args = types.SimpleNamespace(block_size=32, head_dim=None, kv_heads=None, workload="beam")
    try:
        bench.shape_args(args)
    except SystemExit:
        pass
    else:
        raise AssertionError("beam takes no block-size option")


def test_cpu_baseline_and_reference_arm_time_the_same_sample():
    """Both arms run the oracle over the same bounded sample of the workload and
    report the same config keys."""
    from paged_kv_cache_372_b200 import workloads
    wl = workloads.tiny(0)
    cb = bench.cpu_baseline(wl, repeats=1)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["kv_gbs"] > 0
    assert cb["cores_1"]["seqs_per_s"] > 0 and cb["cores_all"]["seqs_per_s"] == cb["value"]
    args = types.SimpleNamespace(workload="tiny", seed=0, steps=2, warmup=1, gpus=1, block_size=None,
                                 head_dim=None)
    ref = bench.run_reference(args, 1, 0)
    assert ref["impl"] == "reference" and ref["config"] == bench.describe(wl)
    n = min(wl.num_seqs, bench.ORACLE_SAMPLE_SEQS)
    assert cb["sample"].startswith(f"{n} of ") and ref["cpu_baseline"]["sample"].startswith(f"{n} of ")


def test_non_kv_bytes_counts_each_part():
    """q/out rows, table entries, split partials and appended rows, against a
    count written out for the tiny workload (contexts 1, 7, 16, 33; H = Hkv = 2,
    D = 64, bs = 16)."""
    from paged_kv_cache_372_b200 import workloads
    wl = workloads.tiny(0)
    ctx = [int(c) for c in wl.steps[0].context_lens]
    assert sorted(ctx) == [1, 7, 16, 33]
    H, Hkv, D = 2, 2, 64
    nb = bench.non_kv_bytes(wl, 16, fused=True, shared=False)
    assert nb["q_and_out"] == 2 * 4 * H * D * 2
    assert nb["tables_and_contexts"] == 4 * (1 + 1 + 1 + 3) + 4 * 4
    assert nb["partials"] == 2 * 3 * H * (D * 4 + 8)  # only the 33-token sequence splits, into 3
    assert nb["appended_rows"] == 2 * 2 * 4 * Hkv * D * 2
    assert bench.non_kv_bytes(wl, 64, fused=False, shared=False)["partials"] == 0
    assert bench.non_kv_bytes(wl, 64, fused=False, shared=False)["appended_rows"] == 0
