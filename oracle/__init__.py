"""fp64 CPU oracle for the fused attention forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
path (``dnn_compiler_pipelining_b200``) never imports it and shares no code
with it.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, OpenMP over rows):
the textbook definition of scaled dot-product attention with grouped-query
heads and an optional causal mask, which the PipeThreader pages evaluate as
"FlashAttention" on LLaMA3-8B/70B head shapes (papers.lqhl.me
"PipeThreader-OSDI25", "实验与结果", paper Sec. 6.2 / Fig. 12).  This module
only marshals numpy arrays into that library.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile ``attn_oracle.c`` into ``liboracle.so`` next to it (gcc, -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_attn_fwd_f64.argtypes = [_f64p, _f64p, _f64p, _f64p, _f64p] + \
            [ctypes.c_int64] * 5 + [ctypes.c_int]
        lib.oracle_attn_rows_f64.argtypes = [_f64p, _i64p, ctypes.c_int64, _f64p, _f64p,
                                             ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                             _f64p, _f64p]
        lib.oracle_attn_probs_row_f64.argtypes = [_f64p, _f64p, ctypes.c_int64, ctypes.c_int64,
                                                  ctypes.c_int64, ctypes.c_int, _f64p, _f64p]
        lib.oracle_attn_fwd_qk_f64.argtypes = [_f64p, _f64p, _f64p, _f64p, _f64p] + \
            [ctypes.c_int64] * 6 + [ctypes.c_int]
        lib.oracle_attn_rows_qk_f64.argtypes = [_f64p, _i64p, ctypes.c_int64, _f64p, _f64p,
                                                ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                                ctypes.c_int, _f64p, _f64p]
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray, t=_f64p):
    return a.ctypes.data_as(t)


def attention(q, k, v, causal: bool):
    """Whole tensors.  q: [B,Hq,S,D]; k, v: [B,Hkv,S,D].  Returns (O, LSE) in fp64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, S, D) or v.shape != k.shape:
        raise ValueError("shape mismatch: q %s k %s v %s" % (q.shape, k.shape, v.shape))
    o = np.empty_like(q)
    lse = np.empty((B, Hq, S), dtype=np.float64)
    rc = _load().oracle_attn_fwd_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                     B, Hq, Hkv, S, D, int(bool(causal)))
    if rc != 0:
        raise ValueError("oracle_attn_fwd_f64 failed (%d)" % rc)
    return o, lse


def attention_rows(q_rows, pos, k_head, v_head, causal: bool):
    """Selected query rows of one head.  q_rows: [n,D]; pos: [n] positions;
    k_head, v_head: [S,D] of that head's kv head.  Returns (O [n,D], LSE [n])."""
    q_rows, k_head, v_head = _f64(q_rows), _f64(k_head), _f64(v_head)
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    n, D = q_rows.shape
    S = k_head.shape[0]
    o = np.empty((n, D), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    rc = _load().oracle_attn_rows_f64(_ptr(q_rows), _ptr(pos, _i64p), n, _ptr(k_head),
                                      _ptr(v_head), S, D, int(bool(causal)), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attn_rows_f64 failed (%d)" % rc)
    return o, lse


def probs_row(q_vec, k_head, i: int, causal: bool):
    """Attention probabilities of one query row: (P [S], LSE)."""
    q_vec, k_head = _f64(q_vec), _f64(k_head)
    S, D = k_head.shape
    p = np.empty((S,), dtype=np.float64)
    lse = ctypes.c_double()
    rc = _load().oracle_attn_probs_row_f64(_ptr(q_vec), _ptr(k_head), int(i), S, D,
                                           int(bool(causal)), _ptr(p), ctypes.byref(lse))
    if rc != 0:
        raise ValueError("oracle_attn_probs_row_f64 failed (%d)" % rc)
    return p, lse.value


def attention_qk(q, k, v, causal: bool):
    """Sq query rows over Sk keys.  q: [B,Hq,Sq,D]; k, v: [B,Hkv,Sk,D].  The causal
    window is aligned at the bottom right (query i sees keys j <= i + Sk - Sq).
    Returns (O [B,Hq,Sq,D], LSE [B,Hq,Sq]) in fp64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    if k.shape != (B, Hkv, Sk, D) or v.shape != k.shape:
        raise ValueError("shape mismatch: q %s k %s v %s" % (q.shape, k.shape, v.shape))
    o = np.empty_like(q)
    lse = np.empty((B, Hq, Sq), dtype=np.float64)
    rc = _load().oracle_attn_fwd_qk_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                        B, Hq, Hkv, Sq, Sk, D, int(bool(causal)))
    if rc != 0:
        raise ValueError("oracle_attn_fwd_qk_f64 failed (%d)" % rc)
    return o, lse


def attention_rows_qk(q_rows, pos, k_head, v_head, Sq: int, causal: bool):
    """Selected query rows (positions in [0, Sq)) of one head over Sk keys."""
    q_rows, k_head, v_head = _f64(q_rows), _f64(k_head), _f64(v_head)
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    n, D = q_rows.shape
    Sk = k_head.shape[0]
    o = np.empty((n, D), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    rc = _load().oracle_attn_rows_qk_f64(_ptr(q_rows), _ptr(pos, _i64p), n, _ptr(k_head),
                                         _ptr(v_head), int(Sq), Sk, D, int(bool(causal)),
                                         _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attn_rows_qk_f64 failed (%d)" % rc)
    return o, lse


def num_threads() -> int:
    """OpenMP threads the oracle uses."""
    return int(_load().oracle_num_threads())
