"""The decoder-layer oracle against its pins (CPU only), and planted mistakes
in copies of its source: every one must fail at least one pin."""
import importlib.util
import os

import pytest

import oracle
from oracle import decoder
from tests import decoder_pins

SRC = os.path.join(os.path.dirname(os.path.abspath(oracle.__file__)), "decoder.py")


@pytest.mark.parametrize("check", decoder_pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(check):
    check(decoder)


# (description, text in decoder.py, replacement)
MUTATIONS = [
    ("RMSNorm sums instead of averaging", "np.mean(x * x, axis=-1, keepdims=True)",
     "np.sum(x * x, axis=-1, keepdims=True)"),
    ("RMSNorm weight dropped", "/ np.sqrt(ms + eps) * np.asarray(w, dtype=np.float64)",
     "/ np.sqrt(ms + eps)"),
    ("RMSNorm eps outside the root", "np.sqrt(ms + eps)", "(np.sqrt(ms) + eps)"),
    ("rotation direction flipped", "a * c - b * s, b * c + a * s", "a * c + b * s, b * c - a * s"),
    ("interleaved pairs instead of halves", "a, b = x[..., : D // 2], x[..., D // 2:]",
     "a, b = x[..., 0::2], x[..., 1::2]"),
    ("frequency exponent halved", "-2.0 * i / D", "-1.0 * i / D"),
    ("silu with the wrong sign", "1.0 + np.exp(-a)", "1.0 + np.exp(a)"),
    ("value heads read from the key heads", "v = heads[:, Hq + Hkv:]", "v = heads[:, Hq:Hq + Hkv]"),
    ("no rotation of the keys", "k = r(rope(heads[:, Hq:Hq + Hkv], theta))",
     "k = r(heads[:, Hq:Hq + Hkv])"),
    ("attention not causal", "np.ascontiguousarray(v),\n                     True)",
     "np.ascontiguousarray(v),\n                     False)"),
    ("heads merged without the transpose", "o.transpose(0, 2, 1, 3).reshape(B, S, Hq * D)",
     "o.reshape(B, S, Hq * D)"),
    ("attention residual dropped", "h = r(x + o_tok @", "h = r(0 * x + o_tok @"),
    ("MLP norm applied to x", "n2 = r(rmsnorm(h, w_mlp_norm, eps))",
     "n2 = r(rmsnorm(x, w_mlp_norm, eps))"),
    ("gate and up swapped", "g = r(silu(gu[..., :inter]) * gu[..., inter:])",
     "g = r(silu(gu[..., inter:]) * gu[..., :inter])"),
    ("MLP residual dropped", "return r(h + g @", "return r(0 * h + g @"),
    ("rounding to fp16 skipped", "astype(np.float16).astype(np.float64)",
     "astype(np.float64).astype(np.float64)"),
]


@pytest.mark.parametrize("desc,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(tmp_path, desc, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation target missing or ambiguous: %r" % old
    path = tmp_path / "decoder_mut.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location("decoder_mut", str(path))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    failed = []
    for check in decoder_pins.ALL_CHECKS:
        try:
            check(mod)
        except (AssertionError, ValueError, IndexError):
            failed.append(check.__name__)
    assert failed, "planted mistake '%s' passed every pin" % desc
