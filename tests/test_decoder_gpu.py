"""GPU parity of the LLaMA3 decoder-layer proxy (attn_decoder_layer_fwd through
the C ABI) against the fp64 oracle, which rounds to fp16 at the same points
where the layer stores a tensor.  Needs a B200.

Tolerance, from the arithmetic.  Both sides round the same steps to fp16, so
they differ only by:
  * fp32-vs-fp64 arithmetic inside a step (relative ~1e-6);
  * the attention kernel's own error (up to 2e-3 on O);
  * one-step fp16 rounding flips of intermediates, which those differences
    trigger.
A difference in an intermediate reaches y in two ways:
  * through a projection sum, whose terms each carry up to 2^-11 relative
    error, giving an absolute error that scales with the RMS of the output
    row, not with the element itself;
  * through the residual h = x + ..., at most a fp16 step or two of |y|.
Bound per element: |y_gpu - y_ref| <= 4 ulp16(|y_ref|) + 8 * 2^-11 * rms(y_ref
row), where ulp16(v) is the fp16 spacing at v.  On average the difference is
at most one fp16 step: mean |y_gpu - y_ref| <= mean ulp16(|y_ref|)."""
import numpy as np
import pytest
import torch

from dnn_compiler_pipelining_b200 import attn
from dnn_compiler_pipelining_b200.inputs import DECODER_MODELS, make_decoder_inputs
from oracle import decoder as oracle_decoder

pytestmark = pytest.mark.gpu

EPS, THETA = 1e-5, 500000.0


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from dnn_compiler_pipelining_b200.build import build
    build()
    attn.load()
    torch.cuda.set_device(0)
    attn.device_status()


def ulp16(v):
    a = np.maximum(np.abs(v), 2.0 ** -14)
    return np.exp2(np.floor(np.log2(a)) - 10)


def _run(B, S, hidden, Hq, Hkv, D, inter, seed):
    x, w = make_decoder_inputs(B, S, hidden, Hq, Hkv, D, inter, seed=seed, device="cuda")
    y = attn.decoder_layer_fwd(x, w, Hq, Hkv, D, eps=EPS, rope_theta=THETA)
    st, site = attn.device_status()
    assert st == attn.ATTN_OK, "device status %d at site %#x" % (st, site)
    return x, w, y


def _check(x, w, y, Hq, Hkv, D, what):
    wc = {k: v.cpu().double().numpy() for k, v in w.items()}
    ref = oracle_decoder.decoder_layer(x.cpu().double().numpy(), Hq=Hq, Hkv=Hkv, D=D, eps=EPS,
                                       theta=THETA, **wc)
    got = y.cpu().double().numpy()
    assert np.all(np.isfinite(got)), what + ": non-finite output"
    err = np.abs(got - ref)
    rms = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
    bound = 4 * ulp16(ref) + 8 * 2.0 ** -11 * rms
    worst = np.unravel_index(np.argmax(err / bound), err.shape)
    assert np.all(err <= bound), "%s: err %.3e > bound %.3e at %s (ref %.4f)" % (
        what, err[worst], bound[worst], worst, ref[worst])
    assert err.mean() <= ulp16(ref).mean(), "%s: mean err %.3e > mean fp16 step %.3e" % (
        what, err.mean(), ulp16(ref).mean())
    print("%s: max err / bound %.2f, mean err %.2e" % (what, (err / bound).max(), err.mean()))


# (B, S, hidden, Hq, Hkv, D, inter): several tiles, ragged S, both head dims
SMALL = [(2, 200, 256, 4, 2, 64, 512), (1, 384, 512, 8, 2, 128, 1024),
         (3, 77, 128, 2, 1, 128, 384), (1, 1, 256, 4, 4, 64, 256)]


@pytest.mark.parametrize("B,S,hidden,Hq,Hkv,D,inter", SMALL)
def test_decoder_small(B, S, hidden, Hq, Hkv, D, inter):
    x, w, y = _run(B, S, hidden, Hq, Hkv, D, inter, seed=61)
    _check(x, w, y, Hq, Hkv, D, "B%d S%d hidden%d Hq%d Hkv%d D%d I%d" % (
        B, S, hidden, Hq, Hkv, D, inter))


def test_decoder_llama3_8b_dims():
    """The full LLaMA3-8B layer dimensions on a short ragged sequence."""
    m = DECODER_MODELS["llama3-8b"]
    x, w, y = _run(1, 130, m["hidden"], m["Hq"], m["Hkv"], m["D"], m["inter"], seed=67)
    _check(x, w, y, m["Hq"], m["Hkv"], m["D"], "llama3-8b dims, S=130")


def test_decoder_llama3_8b_dims_aligned():
    """The full LLaMA3-8B dimensions with S a multiple of 128: the output
    projection reads the attention output head-major (no merge step)."""
    m = DECODER_MODELS["llama3-8b"]
    x, w, y = _run(2, 256, m["hidden"], m["Hq"], m["Hkv"], m["D"], m["inter"], seed=69)
    _check(x, w, y, m["Hq"], m["Hkv"], m["D"], "llama3-8b dims, B=2 S=256")


def test_decoder_in_place_and_deterministic():
    B, S, hidden, Hq, Hkv, D, inter = 2, 256, 256, 4, 2, 128, 512
    x, w, y = _run(B, S, hidden, Hq, Hkv, D, inter, seed=71)
    y2 = attn.decoder_layer_fwd(x, w, Hq, Hkv, D, eps=EPS, rope_theta=THETA)
    xi = x.clone()
    attn.decoder_layer_fwd(xi, w, Hq, Hkv, D, eps=EPS, rope_theta=THETA, y=xi)
    torch.cuda.synchronize()
    assert torch.equal(y, y2) and torch.equal(y, xi)
