"""Fused-pass variant selection on the CPU: the compiled-in rule table, the
library's choice for every shape class, explicit-variant validation, and the
tuner's host logic (choice with a margin, rules over S ranges).  No compute
call runs here."""
import math
import os
import re

import pytest

from dnn_compiler_pipelining_b200 import attn, tune
from dnn_compiler_pipelining_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TABLE = os.path.join(ROOT, "dnn_compiler_pipelining_b200", "csrc", "variant_table.inc")

OK, NULL, SHAPE, ALIGN, UNSUP, CUDA = range(6)
FAKE = 0x10000


@pytest.fixture(scope="module")
def lib():
    build()
    return attn.load()


def table_rules(path=TABLE):
    text = re.sub(r"//[^\n]*", "", open(path).read())
    return [tuple(int(x) for x in m.groups()) for m in re.finditer(
        r"VARIANT_RULE\(\s*(-?\d+)\s*,\s*(-?\d+)\s*,\s*(-?\d+)\s*,\s*(-?\d+)\s*,\s*(-?\d+)\s*\)",
        text)]


def expected_variant(rules, D, causal, Sk):
    for d, c, lo, hi, var in rules:
        if d == D and c == causal and lo <= Sk <= hi:
            return var
    return 0


def test_count_and_names(lib):
    n = attn.variant_count()
    assert n == 20
    names = [attn.variant_name(i) for i in range(n)]
    structures = ["pingpong,row_pairs", "pingpong,head_pairs", "dbuf,softmax_split=1",
                  "dbuf,softmax_split=2"]
    assert names == ["%s,fma_exp2_pairs=%d/8" % (structures[i // 5], i % 5) for i in range(20)]
    assert attn.variant_name(-1) is None and attn.variant_name(n) is None


def test_table_well_formed(lib):
    rules = table_rules()
    n = attn.variant_count()
    for d, c, lo, hi, var in rules:
        assert d in (64, 128, 256) and c in (0, 1)
        assert 1 <= lo <= hi <= 2 ** 31 - 1
        assert 0 <= var < n
    # within one (D, causal) class the S ranges do not overlap
    for D in (64, 128, 256):
        for c in (0, 1):
            spans = sorted((lo, hi) for d, cc, lo, hi, _ in rules if d == D and cc == c)
            for (lo0, hi0), (lo1, hi1) in zip(spans, spans[1:]):
                assert hi0 < lo1


def test_select_follows_table(lib):
    rules = table_rules()
    probes = {1, 2, 127, 128, 129, 511, 512, 513, 700, 724, 725, 1023, 1024, 1448, 1449, 2048,
              2896, 2897, 4096, 5792, 5793, 8192, 16384, 65536}
    for lo_hi in rules:
        probes |= {lo_hi[2], lo_hi[3], max(1, lo_hi[2] - 1), lo_hi[3] + 1}
    for D in (64, 128, 256):
        for causal in (0, 1):
            for Sk in sorted(probes):
                if Sk < 1 or Sk > 2 ** 20:
                    continue
                got = attn.variant_select(1, 8, 2, Sk, Sk, D, causal)
                assert got == expected_variant(rules, D, causal, Sk), (D, causal, Sk)
                # non-causal, Sq != Sk: the key length decides
                assert attn.variant_select(1, 8, 2, 77, Sk, D, 0) == \
                    expected_variant(rules, D, 0, Sk)


def test_select_rejects_what_the_call_rejects(lib):
    assert attn.variant_select(0, 8, 2, 128, 128, 128, 1) == -1
    assert attn.variant_select(1, 8, 3, 128, 128, 128, 1) == -1    # Hq % Hkv
    assert attn.variant_select(1, 8, 2, 128, 128, 96, 1) == -1     # D
    assert attn.variant_select(1, 8, 2, 300, 200, 128, 1) == -1    # causal Sq > Sk
    assert attn.variant_select(1, 8, 2, 300, 200, 128, 0) >= 0


def test_explicit_variant_validation(lib):
    def call(variant, D=128, Sq=128, Sk=128, q=FAKE):
        return lib.attn_fwd_variant(q, FAKE, FAKE, FAKE, FAKE, 1, 4, 2, Sq, Sk, D, 1, variant,
                                    None)
    n = attn.variant_count()
    assert call(-1) == UNSUP and call(n) == UNSUP
    assert call(0, q=None) == NULL
    assert call(0, D=96) == UNSUP
    assert call(n, Sq=0) == SHAPE          # sizes are checked before the variant
    for var in range(n):
        assert call(var) in (CUDA, UNSUP)  # well-formed: reaches the runtime (no GPU here)


def test_tuner_choice_needs_margin():
    # variant 0 stays unless another agrees with it and is >= 2 % faster
    assert tune.choose([1.0, 0.99, 0.985], [True] * 3) == 0
    assert tune.choose([1.0, 0.97, 0.95], [True] * 3) == 2
    assert tune.choose([1.0, 0.97, 0.90], [True, True, False]) == 1
    assert tune.choose([1.0, 1.2], [True, True]) == 0


def test_tuner_rules_cover_all_sizes():
    choices = [(512, 0), (1024, 2), (2048, 2), (4096, 0), (8192, 1)]
    rules = tune.rules_for(choices)
    assert rules[0][0] == 1 and rules[-1][1] == 2 ** 31 - 1
    for (lo0, hi0, v0), (lo1, hi1, v1) in zip(rules, rules[1:]):
        assert lo1 == hi0 + 1 and v0 != v1
    # every measured S lands in a rule with its own choice
    for s, var in choices:
        assert [r[2] for r in rules if r[0] <= s <= r[1]] == [var]
    # boundaries sit at geometric midpoints: 724 (sqrt(512 * 1024) = 724.08) -> 512's rule
    assert rules[0] == (1, int(math.sqrt(512 * 1024)), 0)
    assert tune.rules_for([(512, 3)]) == [(1, 2 ** 31 - 1, 3)]


def test_tuner_writes_a_table_the_library_format_accepts(tmp_path, monkeypatch):
    """tune.main with the GPU timing replaced by a fake: the table it writes has
    one rule set per (D, causal), parses with the same pattern the library's
    macro takes, and picks a faster agreeing variant only past the margin."""
    fake = {}

    def fake_time_class(D, causal, S, reps, warmup, seed=0):
        med = [1.0, 1.0, 1.0, 1.0, 1.0]
        if D == 64 and causal and S >= 2048:
            med[2] = 0.9          # 10 % faster: chosen
        if D == 128 and not causal and S == 512:
            med[1] = 0.99         # 1 % faster: under the margin
        fake[(D, causal, S)] = med
        return max(1, tune.TOKENS // S), med, [True] * 5

    class Props:
        name, multi_processor_count = "fake GPU", 148

    monkeypatch.setattr(tune, "time_class", fake_time_class)
    monkeypatch.setattr(tune.torch.cuda, "is_available", lambda: True)
    monkeypatch.setattr(tune.torch.cuda, "get_device_properties", lambda i: Props())
    monkeypatch.setattr(tune.attn, "variant_count", lambda: 5)
    monkeypatch.setattr(tune.attn, "variant_name", lambda i: "v%d" % i)
    table, report = tmp_path / "t.inc", tmp_path / "r.md"
    tune.main(["--table", str(table), "--report", str(report)])
    text = open(table).read()
    rules = table_rules(str(table))
    assert len(fake) == 30   # D in {64, 128, 256} x causal x 5 sequence lengths
    assert expected_variant(rules, 64, 1, 8192) == 2 and expected_variant(rules, 64, 1, 2048) == 2
    # 1448 is the geometric midpoint of 1024 and 2048: the 2048 rule starts just above it
    assert expected_variant(rules, 64, 1, 1448) == 0 and expected_variant(rules, 64, 1, 1449) == 2
    assert expected_variant(rules, 128, 0, 512) == 0
    assert all(expected_variant(rules, d, c, s) == 0 for d in (64, 128) for c in (0, 1)
               for s in (1, 512, 1024) if not (d == 64 and c == 1 and s >= 1449))
    assert "VARIANT_RULE(" in text and "fake GPU" in text
    assert "| 64 | 1 | 8192 |" in open(report).read()
