"""Host-side helpers of bench.py that need no GPU: the code hash that keeps a committed
DRAM-traffic measurement tied to the kernel source it was taken on, the peak basis, the
converter's byte count, the index-statistics leg and the workload overrides."""
import json
import os

import pytest

import bench


def _write(tmp_path, name, text):
    p = tmp_path / name
    p.write_text(text)
    return str(p)


def test_code_hash_ignores_comments_and_layout(tmp_path):
    a = _write(tmp_path, "a.cu", "// header\nint f(int x) {\n  return x + 1;  \n}\n")
    b = _write(tmp_path, "b.cu", "// another header\n\n  // note\nint f(int x) {\n    return x + 1;\n}\n")
    assert bench.source_code_sha([a]) == bench.source_code_sha([b])


def test_code_hash_follows_code(tmp_path):
    a = _write(tmp_path, "a.cu", "int f(int x) {\n  return x + 1;\n}\n")
    b = _write(tmp_path, "b.cu", "int f(int x) {\n  return x + 2;\n}\n")
    assert bench.source_code_sha([a]) != bench.source_code_sha([b])
    # a trailing comment sits on a code line and counts as code
    c = _write(tmp_path, "c.cu", "int f(int x) {\n  return x + 1;  // one\n}\n")
    assert bench.source_code_sha([a]) != bench.source_code_sha([c])


def test_traffic_reported_only_for_the_measured_code(tmp_path, monkeypatch):
    """bench.py reports the committed figure while the hash matches, else null."""
    d = json.load(open(os.path.join(bench.ROOT, "profiles", "bwd_main_traffic.json")))
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "bwd_source_sha", lambda kernel: "abc")
    (prof / "bwd_main_traffic.json").write_text(json.dumps(dict(d, source_sha="abc")))
    assert bench.profiled_traffic(d["workload"]) == d["dram_bytes_per_launch"]
    assert bench.profiled_traffic("another_workload") is None
    (prof / "bwd_main_traffic.json").write_text(json.dumps(dict(d, source_sha="old")))
    assert bench.profiled_traffic(d["workload"]) is None


def test_peak_basis_follows_the_runs_own_clock_record():
    """Burst peak unless the timed region saw power capping; then the sustained one."""
    peaks = {"bf16_tflops": 1661.7, "bf16_tflops_sustained": 1406.6}
    assert bench.peak_basis(peaks, {"reasons": []}) == (1661.7, "bf16_tflops")
    assert bench.peak_basis(peaks, None) == (1661.7, "bf16_tflops")
    assert bench.peak_basis(peaks, {"reasons": ["sw_power_cap"]}) == (1406.6,
                                                                      "bf16_tflops_sustained")


def test_converter_bytes_index_workload():
    from index_sparse_attention_b200 import inputs as I
    w = I.WORKLOADS["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"]
    idx = 16384 * 4 * 2048 * 4          # 512 MiB of indices, read once
    bitmap = 4 * 16384 * 512 * 4        # 128 MiB, written and read back once
    lists = 4 * 4 * (128 * 130 + 128 * 130)
    assert bench.converter_bytes(w) == idx + 2 * bitmap + 2 * lists


def test_index_stats_leg_on_a_small_index_workload(capsys):
    """bench.py --op index_stats: counts on the seeded indices (no GPU)."""
    import types
    args = types.SimpleNamespace(workload="indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048",
                                 seq=1024)
    bench.run_index_stats(args)
    d = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert d["block_over_token"] >= 1.0
    assert 0.0 < d["nonempty_32key_subblocks_of_active_tiles"] <= 1.0
    assert 0.0 < d["tile_union_keys_over_causal_range"] <= 1.0
    # causal, 1024 tokens, top-2048: every (q, k <= q) pair is selected
    assert d["selected_pairs_per_kv_head"] == 1024 * 1025 // 2
    assert d["token_gather_forward_bytes"] == 4 * 1024 * 1025 // 2 * 2 * (192 + 128)


def test_head_count_override_makes_a_gqa_workload():
    """--heads HQ,HK turns a workload into GQA with those head counts (the mask is then
    drawn per KV head); invalid counts are refused before any work."""
    import argparse
    from index_sparse_attention_b200 import inputs as I
    ns = argparse.Namespace(workload="long_causal_blocksparse_h16_s32768_d256", seq=0,
                            heads="16,8")
    w = bench.get_workload(ns)
    assert (w.HQ, w.HK, w.Dqk, w.Sq) == (16, 8, 256, 32768)
    assert w.name.endswith("@H16x8")
    assert I.block_mask(I.scaled(w, Sq=512, Sk=512)).shape == (1, 8, 4, 4)
    for bad in ("16,5", "0,4", "8,16"):
        with pytest.raises(SystemExit):
            bench.get_workload(argparse.Namespace(workload=ns.workload, seq=0, heads=bad))
    ns.heads = ""
    assert bench.get_workload(ns) == I.WORKLOADS[ns.workload]


def test_reported_backward_kernel_follows_the_library_rule():
    """The roofline names the (192,128) backward instance the library picks: one CTA per
    key tile when B * HK * ceil(Sk / 128) is at least twice the SM count, else (and in
    deterministic mode, or when the split is forced) the head-dim split."""
    from index_sparse_attention_b200 import inputs as I
    w = I.WORKLOADS["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"]  # 128 tiles x 4 heads
    assert bench.bwd_kernel_name(w) == "sparse_bwd_kernel<192,128,1>"
    assert bench.bwd_kernel_name(w, deterministic=True) == "sparse_bwd_kernel<192,128,2>"
    assert bench.bwd_kernel_name(w, form="split") == "sparse_bwd_kernel<192,128,2>"
    small = I.scaled(w, Sq=4096, Sk=4096)  # 32 tiles x 4 heads = 128 < 2 x 148
    assert bench.bwd_kernel_name(small) == "sparse_bwd_kernel<192,128,2>"
    assert bench.bwd_kernel_name(small, form="whole") == "sparse_bwd_kernel<192,128,1>"
    edge = I.scaled(w, Sq=9472, Sk=9472)  # 74 tiles x 4 heads = 296 = 2 x 148
    assert bench.bwd_kernel_name(edge) == "sparse_bwd_kernel<192,128,1>"
    assert bench.bwd_kernel_name(I.scaled(w, Sq=9344, Sk=9344)) == "sparse_bwd_kernel<192,128,2>"
    assert bench.bwd_kernel_name(I.WORKLOADS["long_causal_blocksparse_h16_s32768_d256"]) == \
        "sparse_bwd_pair_kernel"
