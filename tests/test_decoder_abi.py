"""attn_decoder_layer_fwd rejects bad arguments before launching anything (CPU)."""
import ctypes

import pytest

from dnn_compiler_pipelining_b200 import attn
from dnn_compiler_pipelining_b200.build import build

OK, NULL, SHAPE, ALIGN, UNSUP, CUDA, TIMEOUT, WORKSPACE = range(8)
FAKE = 0x10000   # 256-byte aligned stand-in address; never dereferenced


@pytest.fixture(scope="module")
def lib():
    build()
    return attn.load()


def call(lib, x=FAKE, y=FAKE + 0x1000, ws=FAKE + 0x2000, ws_bytes=None, B=1, S=16, hidden=256,
         Hq=4, Hkv=2, D=64, inter=512, eps=1e-5, theta=500000.0, w=FAKE):
    if ws_bytes is None:
        ws_bytes = lib.attn_decoder_layer_workspace_bytes(B, S, hidden, Hq, Hkv, D, inter)
    return lib.attn_decoder_layer_fwd(x, w, w, w, w, w, w, y, B, S, hidden, Hq, Hkv, D, inter,
                                      eps, theta, ws, ws_bytes, None)


def test_workspace_bytes(lib):
    f = lib.attn_decoder_layer_workspace_bytes
    r = lambda n: (n + 255) // 256 * 256
    B, S, H, Hq, Hkv, D, I = 2, 100, 256, 4, 2, 64, 512
    T = B * S
    # rotary table, RMSNorm output, Q, K, V, O, LSE, residual stream, SwiGLU
    # output (the fused GEMM epilogues keep no projection output around)
    want = (r(S * D // 2 * 8) + r(T * H * 2)
            + 2 * r(T * Hq * D * 2) + 2 * r(T * Hkv * D * 2) + r(T * Hq * 4) + r(T * H * 2)
            + r(T * I * 2))
    assert f(B, S, H, Hq, Hkv, D, I) == want
    assert f(0, S, H, Hq, Hkv, D, I) == 0
    assert f(B, S, 100, Hq, Hkv, D, I) == 0       # hidden % 8
    assert f(B, S, H, Hq, Hkv, 96, I) == 0        # D
    assert f(B, S, H, 4, 3, D, I) == 0            # Hq % Hkv


def test_validation_before_launch(lib):
    assert call(lib, x=None) == NULL
    assert call(lib, w=None) == NULL
    assert call(lib, ws=None) == NULL
    assert call(lib, B=0) == SHAPE
    assert call(lib, hidden=260) == SHAPE
    assert call(lib, inter=500) == SHAPE
    assert call(lib, Hq=4, Hkv=3) == SHAPE
    assert call(lib, D=96) == UNSUP
    assert call(lib, eps=-1.0) == SHAPE
    assert call(lib, eps=float("nan")) == SHAPE
    assert call(lib, theta=1.0) == SHAPE
    assert call(lib, x=FAKE + 8) == ALIGN
    assert call(lib, w=FAKE + 2) == ALIGN
    assert call(lib, ws=FAKE + 16) == ALIGN
    need = lib.attn_decoder_layer_workspace_bytes(1, 16, 256, 4, 2, 64, 512)
    assert call(lib, ws_bytes=need - 1) == WORKSPACE
    # well-formed: reaches the runtime, which has no device here
    assert call(lib) in (CUDA, UNSUP)
