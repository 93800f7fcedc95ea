"""The fp64 oracle against what the mathematics fixes (CPU only).

Each pin in ``pins.py`` runs against the real oracle.  Then a set of plausible
mistakes is planted in copies of the oracle's C source (on the CPU, in a
temporary folder), and every planted mistake must fail at least one pin.
"""
import importlib.util
import os
import shutil

import pytest

import oracle
from tests import pins

ORACLE_DIR = os.path.dirname(os.path.abspath(oracle.__file__))


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(check):
    check(oracle)


# (description, text in attn_oracle.c, replacement).  Every replacement keeps
# all memory accesses in bounds.
MUTATIONS = [
    ("dropped 1/sqrt(D) scale", "1.0 / sqrt((double)D)", "1.0"),
    ("causal window misses the diagonal", "causal ? i + 1 : S", "causal ? i : S"),
    ("causal mask ignored", "causal ? i + 1 : S", "causal ? S : S"),
    ("kv head by modulo instead of contiguous groups", "hq / group", "hq % Hkv"),
    ("LSE drops the max term", "m + log(l)", "log(l)"),
    ("max added instead of subtracted", "exp(p_out[j] - m)", "exp(p_out[j] + m)"),
    ("value rows read in reverse", "v[j * D + d]", "v[(n_keys - 1 - j) * D + d]"),
    ("probabilities not normalised", "p_out[j] /= l;", "p_out[j] /= 1.0;"),
    ("query/key operand index swapped", "q[d] * k[j * D + d]", "q[d] * k[j * D + (D - 1 - d)]"),
    # the different-length (Sq, Sk) entries
    ("causal window aligned top-left", "const int64_t last = i + (Sk - Sq);",
     "const int64_t last = i;"),
    ("causal offset sign flipped", "const int64_t last = i + (Sk - Sq);",
     "const int64_t last = i + (Sq - Sk);"),
    ("Sq/Sk weights not normalised", "o[d] /= sum;", "o[d] /= 1.0;"),
    ("Sq/Sk LSE drops the max term", "*lse = mx + log(sum);", "*lse = log(sum);"),
    ("Sq/Sk value rows shifted", "o[d] += scratch[j] * v[D * j + d];",
     "o[d] += scratch[j] * v[D * ((j + 1) % nk) + d];"),
    ("Sq/Sk scale dropped", "pow((double)D, -0.5)", "1.0"),
]


def _load_variant(tmp_path, name, src_text):
    d = tmp_path / name
    d.mkdir()
    shutil.copy(os.path.join(ORACLE_DIR, "__init__.py"), d / "__init__.py")
    (d / "attn_oracle.c").write_text(src_text)
    spec = importlib.util.spec_from_file_location("oracle_" + name, str(d / "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("desc,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(tmp_path, desc, old, new):
    src = open(os.path.join(ORACLE_DIR, "attn_oracle.c")).read()
    assert old in src, "mutation target missing: %r" % old
    mod = _load_variant(tmp_path, "mut", src.replace(old, new))
    failed = []
    for check in pins.ALL_CHECKS:
        try:
            check(mod)
        except (AssertionError, ValueError):
            failed.append(check.__name__)
    assert failed, "planted mistake '%s' passed every pin" % desc
