"""The C-ABI library on the CPU: it loads, exports every symbol include/*.h
declares, and rejects bad arguments before touching a GPU.  No compute call
runs here (this machine has no GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from dnn_compiler_pipelining_b200 import attn
from dnn_compiler_pipelining_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, NULL, SHAPE, ALIGN, UNSUP, CUDA, TIMEOUT, WORKSPACE = range(8)


@pytest.fixture(scope="module")
def lib():
    build()
    return attn.load()


def declared_functions():
    text = "".join(open(os.path.join(ROOT, "include", f)).read()
                   for f in sorted(os.listdir(os.path.join(ROOT, "include"))) if f.endswith(".h"))
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 8, names
    for n in names:
        assert hasattr(lib, n), "missing export %s" % n


def test_version_and_strings(lib):
    assert attn.version() >> 16 == 2
    for code in range(8):
        s = attn.status_string(code)
        assert s.startswith(attn.STATUS_NAMES[code])
    assert "UNKNOWN" in attn.status_string(99)


FAKE = 0x10000  # 16-byte aligned stand-in address; never dereferenced (validation fails first)


def call(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=4, Hkv=2, S=128, D=128, causal=1):
    return lib.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, S, D, causal, None)


def test_validation_before_launch(lib):
    assert call(lib, q=None) == NULL
    assert call(lib, lse=None) == NULL
    assert call(lib, B=0) == SHAPE
    assert call(lib, S=0) == SHAPE            # empty sequence
    assert call(lib, Hkv=0) == SHAPE
    assert call(lib, B=-1) == SHAPE
    assert call(lib, S=-128) == SHAPE
    assert call(lib, Hkv=3) == SHAPE          # Hq % Hkv != 0
    assert call(lib, Hq=0) == SHAPE
    assert call(lib, D=96) == UNSUP
    assert call(lib, D=192) == UNSUP
    assert call(lib, D=512) == UNSUP
    assert call(lib, B=65536, Hq=1, Hkv=1, S=32768) == SHAPE  # key rows overflow 2^31
    assert call(lib, B=64, Hq=64, Hkv=8, S=1 << 20) == SHAPE  # row index overflow
    assert call(lib, q=FAKE + 8) == ALIGN
    assert call(lib, lse=FAKE + 2) == ALIGN


def test_qk_validation_before_launch(lib):
    lib.attn_fwd_qk.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 7 + [ctypes.c_void_p]

    def qk(Sq, Sk, causal, D=128):
        return lib.attn_fwd_qk(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, 2, Sq, Sk, D, causal, None)

    assert qk(300, 200, 1) == SHAPE         # a causal query would see no key
    assert qk(0, 200, 0) == SHAPE
    assert qk(200, 0, 0) == SHAPE
    assert qk(100, 200, 1, D=96) == UNSUP
    assert qk(100, 200, 1) in (CUDA, UNSUP)   # well-formed: reaches the runtime
    assert qk(300, 200, 0) in (CUDA, UNSUP)   # non-causal Sq > Sk is allowed


def test_valid_call_without_gpu_fails_loudly(lib):
    # well-formed arguments reach the CUDA runtime, which has no device here
    assert call(lib) in (CUDA, UNSUP)


def test_host_entry_validation(lib):
    need = lib.attn_fwd_host_workspace_bytes(1, 4, 2, 128, 128)
    # Q and O (1*4*128*128*2), K and V (1*2*128*128*2), LSE (4*128*4), each to 256 B
    assert need == 2 * 131072 + 2 * 65536 + 2048
    assert lib.attn_fwd_host_workspace_bytes(0, 4, 2, 128, 128) == 0
    buf = ctypes.create_string_buffer(64)
    a = ctypes.addressof(buf)
    args = [a, a, a, a, a, 1, 4, 2, 128, 128, 1]
    assert lib.attn_fwd_host(*args, FAKE, need - 1, None) == WORKSPACE
    assert lib.attn_fwd_host(*args, FAKE + 16, need, None) == ALIGN
    assert lib.attn_fwd_host(*args, None, need, None) == NULL


def test_binding_rejects_cpu_tensors(lib):
    q = torch.zeros(1, 4, 128, 128, dtype=torch.float16)
    k = torch.zeros(1, 2, 128, 128, dtype=torch.float16)
    with pytest.raises(ValueError):
        attn.attn_fwd(q, k, k)


def test_timeout_setting_roundtrip(lib):
    prev = attn.set_wait_timeout_ns(5_000_000)
    assert attn.set_wait_timeout_ns(10) == 5_000_000   # clamped up to 1 ms on the next set
    assert attn.set_wait_timeout_ns(prev) == 1_000_000


def _fastdiv_cases():
    """Divisors 1..300, powers of two and their neighbours, and large odd
    values; numerators at 0, 1, multiples of d and their neighbours, the top
    of the range (2^31 - 1) and seeded random values."""
    rng = np.random.default_rng(5)
    ds = list(range(1, 301)) + [2 ** k + e for k in range(9, 31) for e in (-1, 0, 1)]
    ds += [int(x) for x in rng.integers(1, 2 ** 31 - 1, 40)]
    for d in ds:
        ns = [0, 1, 2 ** 31 - 1, 2 ** 31 - 2, d - 1, d, d + 1]
        ks = np.unique(np.concatenate([np.arange(0, 50), rng.integers(0, (2 ** 31 - 1) // d + 1, 50)]))
        for k in ks:
            for e in (-1, 0, 1):
                ns.append(int(k) * d + e)
        ns += [int(x) for x in rng.integers(0, 2 ** 31, 200)]
        ns = np.array([x for x in ns if 0 <= x < 2 ** 31], dtype=np.int64)
        yield d, ns


def test_fastdiv_host_matches_floor_division(lib):
    """The multiply-shift division the kernels use to decode work items is
    exact floor division for every numerator below 2^31 (host evaluation of
    the same formula)."""
    for d, ns in _fastdiv_cases():
        q = attn.selftest_fastdiv(d, torch.from_numpy(ns.astype(np.int32)))
        assert np.array_equal(q.numpy().astype(np.int64), ns // d), d
    n = torch.zeros(4, dtype=torch.int32)
    assert lib.attn_selftest_fastdiv(0, n.data_ptr(), n.data_ptr(), 4, 0, None) == 2  # d == 0
    assert lib.attn_selftest_fastdiv(3, None, None, 4, 0, None) == 1
    assert lib.attn_selftest_fastdiv(3, None, None, 0, 0, None) == 0
