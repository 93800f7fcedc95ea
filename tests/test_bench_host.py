"""bench.py host logic on the CPU: the kernel-source hash that ties the
committed ncu counters to the code, FLOP counts, and the L2-flush rule."""
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
