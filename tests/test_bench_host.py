"""bench.py host logic on the CPU: the kernel-source hash that ties the
committed ncu counters to the code, FLOP counts, the L2-flush rule, the work
items and launches per call that follow the library's variant table, and the
stress-input recipe."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_code_tokens_drop_comments_keep_literals():
    src = 'int a = 1; // note\n/* block\n comment */ const char* s = "// kept /* too */";\n' \
          "char q = '\\''; char r = '\"';\n\n   b();"
    assert bench.code_tokens(src) == ('int a = 1; const char* s = "// kept /* too */"; '
                                      "char q = '\\''; char r = '\"'; b();")


def test_hash_ignores_comments_and_layout_only(tmp_path, monkeypatch):
    files = []
    for i, f in enumerate(bench.KERNEL_SOURCES):
        p = tmp_path / ("f%d" % i)
        p.write_text(open(f).read())
        files.append(str(p))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", files)
    h0 = bench.kernel_source_hash()
    text = open(files[0]).read()
    open(files[0], "w").write("// a new comment\n" + text.replace(";\n", ";   \n", 3))
    assert bench.kernel_source_hash() == h0
    open(files[0], "w").write(text + "\nint extra_code;\n")
    assert bench.kernel_source_hash() != h0


def test_flop_counts():
    assert bench.attn_flops(1, 1, 2, 4, False) == 4.0 * 2 * 2 * 4
    assert bench.attn_flops(64, 32, 8192, 128, True) == 2.0 * 64 * 32 * 8192 ** 2 * 128
    # LLaMA3-8B layer GEMMs: 2 * H * ((Hq + 2 Hkv) D + Hq D + 3 I) per token
    per_token = 2.0 * 4096 * (48 * 128 + 32 * 128 + 3 * 14336)
    assert bench.layer_flops(1, 1, 4096, 32, 8, 128, 14336) == per_token + \
        bench.attn_flops(1, 32, 1, 128, True)


def test_l2_flush_rule():
    from dnn_compiler_pipelining_b200.inputs import WORKLOADS
    # Q + K + V of the small single-batch workloads fit in twice the L2: flushed
    assert bench.needs_l2_flush(WORKLOADS["llama3-8b-s512-b1"])
    assert bench.needs_l2_flush(WORKLOADS["llama3-8b-s8192-b1"])
    # the batched workloads stream far more than the L2 holds
    assert not bench.needs_l2_flush(WORKLOADS["llama3-8b-s8192-b64"])
    assert not bench.needs_l2_flush(WORKLOADS["llama3-8b-s2048-b64"])


def test_items_and_launches_follow_the_variant_table():
    from dnn_compiler_pipelining_b200.build import build
    build()
    from dnn_compiler_pipelining_b200.inputs import WORKLOADS
    w = WORKLOADS["llama3-8b-s8192-b64"]            # variant 0: 256-row items
    assert bench.n_items(w) == 64 * 32 * 32
    assert bench.launches_per_call(w) == 1
    w = WORKLOADS["llama3-8b-s512-b1"]              # double-buffered kernel: 128-row items
    assert bench.n_items(w) == 32 * 4
    w = dict(B=1, Hq=32, Hkv=8, S=8192, D=128, causal=True)  # 256-row items fill the SMs
    assert bench.n_items(w) == 32 * 32
    w = dict(B=1, Hq=8, Hkv=8, S=2048, D=128, causal=False)  # too few 256-row items: 128
    assert bench.n_items(w) == 8 * 16
    # more items than one launch's per-CTA bit set holds: split over batch ranges
    w = dict(B=4096, Hq=32, Hkv=8, S=8192, D=128, causal=True)
    assert bench.launches_per_call(w) == -(-4096 * 32 * 32 // (148 * 2048 // (32 * 32) * 32 * 32))


def test_stress_inputs_recipe():
    assert bench.INPUTS["normal"][0] == 1.0 and bench.INPUTS["stress"][0] == 4.0
    cfg = bench.workload_config(dict(B=1, Hq=32, Hkv=8, S=512, D=128, causal=True), "x", 1,
                                "stress")
    assert "N(0,4^2)" in cfg["inputs"]


def test_profiled_traffic_needs_matching_source(tmp_path, monkeypatch):
    prof = tmp_path / "p.md"
    prof.write_text("kernel_source_sha256_16: %s\ndram_bytes_per_launch: 1.5e9\n"
                    % bench.kernel_source_hash())
    assert bench.profiled_traffic(str(prof)) == 1.5e9
    prof.write_text("kernel_source_sha256_16: 0123456789abcdef\ndram_bytes_per_launch: 1.5e9\n")
    assert bench.profiled_traffic(str(prof)) is None
    assert bench.profiled_traffic(str(tmp_path / "missing.md")) is None


def test_traffic_only_for_the_profiled_case(monkeypatch):
    monkeypatch.setattr(bench, "profiled_traffic", lambda *a, **k: 7.0e9)
    assert bench.attn_traffic(*bench.PROFILED_CASE) == 7.0e9
    from dnn_compiler_pipelining_b200.inputs import WORKLOADS
    assert bench.PROFILED_CASE[0] in WORKLOADS
    assert bench.attn_traffic(bench.PROFILED_CASE[0], "stress") is None
    other = next(n for n in WORKLOADS if n != bench.PROFILED_CASE[0])
    assert bench.attn_traffic(other, "normal") is None


def test_algorithmic_bytes_of_the_target_shape():
    # Q and O: 64*32*8192*128 fp16 each (4 GiB); K and V: 64*8*8192*128 fp16 each
    # (1 GiB); LSE: 64*32*8192 fp32 (64 MiB) -- 10.80 GB in all
    n = bench.algorithmic_bytes(64, 32, 8, 8192, 128)
    assert n == 2 * 2**32 + 2 * 2**30 + 2**26
    assert abs(n / 1e9 - 10.80) < 0.01
    h = bench.hbm_figure(n, 10.0, 6000.0, "measured")
    assert abs(h["achieved_gbs"] - n / 1e-2 / 1e9) < 1e-9
    assert abs(h["frac"] - h["achieved_gbs"] / 6000.0) < 1e-12
