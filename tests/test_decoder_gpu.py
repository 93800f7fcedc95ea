"""GPU parity of the LLaMA3 decoder-layer proxy (attn_decoder_layer_fwd through
the C ABI) against the fp64 oracle, which rounds to fp16 at the same points
where the layer stores a tensor.  Needs a B200.

Tolerance: derived per output element from where the two sides can differ
(rounding flips, the attention's fp16 weights, and projections that carry
upstream differences); the budget and its constants are stated above _bound.
On average the difference is at most one fp16 step: mean |y_gpu - y_ref| <=
mean ulp16(|y_ref|)."""
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


# Error budget of one output element y_i, the GPU against the oracle (both
# round to fp16 at the same points; they differ only where a rounding
# decision flips or an upstream difference is carried along):
#   - the final rounding of y and the residual rounding of h can each land one
#     fp16 step apart: ulp16(y_i) + ulp16(h_i);
#   - a projection carries the per-element differences e_k of its input as
#     sum_k W_ik e_k.  The weights are drawn independently of those
#     differences, so the sum is distributed as N(0, |W_i|^2 rms(e)^2) and is
#     bounded by Z_SIGMA standard deviations;
#   - the attention output o differs by its own rounding plus the fp16
#     weights P (relative 2^-12 each, averaged over the row):
#     rms(e_o) <= C_O rms(ulp16(o)), C_O = 2;
#   - g = fp16(silu(gate) up) differs by its own rounding plus the fp16
#     roundings of gate and up carried through the product:
#     rms(e_g) <= C_G rms(ulp16(g)), C_G = 3.
# Z_SIGMA = 6.5: a two-sided Gaussian tail of 8e-11 per element, so a correct
# layer fails none of the ~10^7 checked elements but with probability < 1e-3.
Z_SIGMA = 6.5
C_O = 2.0
C_G = 3.0


def _bound(inter, wc, ref):
    rms = lambda a: np.sqrt(np.mean(a * a, axis=-1, keepdims=True))  # per token
    e_o = C_O * rms(ulp16(inter["o_tok"]))
    e_g = C_G * rms(ulp16(inter["g"]))
    n_o = np.linalg.norm(wc["w_o"], axis=1)      # |W_o row i|, [hidden]
    n_d = np.linalg.norm(wc["w_down"], axis=1)
    sigma = np.sqrt((n_o * e_o) ** 2 + (n_d * e_g) ** 2)
    return ulp16(ref) + ulp16(inter["h"]) + Z_SIGMA * sigma


def _check(x, w, y, Hq, Hkv, D, what):
    wc = {k: v.cpu().double().numpy() for k, v in w.items()}
    inter = {}
    ref = oracle_decoder.decoder_layer(x.cpu().double().numpy(), Hq=Hq, Hkv=Hkv, D=D, eps=EPS,
                                       theta=THETA, intermediates=inter, **wc)
    got = y.cpu().double().numpy()
    assert np.all(np.isfinite(got)), what + ": non-finite output"
    err = np.abs(got - ref)
    bound = _bound(inter, wc, ref)
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


def test_decoder_llama3_70b_dims():
    """The full LLaMA3-70B layer dimensions (K = 8192 in every projection but
    the down projection's 28672; a 57344-wide gate/up GEMM) on one short
    ragged sequence."""
    m = DECODER_MODELS["llama3-70b"]
    x, w, y = _run(1, 72, m["hidden"], m["Hq"], m["Hkv"], m["D"], m["inter"], seed=73)
    _check(x, w, y, m["Hq"], m["Hkv"], m["D"], "llama3-70b dims, S=72")
    del x, w, y
    torch.cuda.empty_cache()


def test_decoder_in_place_and_deterministic():
    B, S, hidden, Hq, Hkv, D, inter = 2, 256, 256, 4, 2, 128, 512
    x, w, y = _run(B, S, hidden, Hq, Hkv, D, inter, seed=71)
    y2 = attn.decoder_layer_fwd(x, w, Hq, Hkv, D, eps=EPS, rope_theta=THETA)
    xi = x.clone()
    attn.decoder_layer_fwd(xi, w, Hq, Hkv, D, eps=EPS, rope_theta=THETA, y=xi)
    torch.cuda.synchronize()
    assert torch.equal(y, y2) and torch.equal(y, xi)
