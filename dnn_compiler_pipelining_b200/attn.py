"""Thin ctypes binding of libattn_b200.so (C ABI in include/attn.h).

Argument marshalling only: every step of the attention forward runs in the
library's CUDA kernels.  PyTorch supplies device memory and streams.  There is
no fallback: if the library is missing or the device is not an sm_100 GPU,
calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libattn_b200.so")

ATTN_OK = 0
ATTN_ERR_DEVICE_TIMEOUT = 6
ATTN_ERR_TOO_LARGE = 8
STATUS_NAMES = {0: "ATTN_OK", 1: "ATTN_ERR_NULL", 2: "ATTN_ERR_SHAPE", 3: "ATTN_ERR_ALIGN",
                4: "ATTN_ERR_UNSUPPORTED", 5: "ATTN_ERR_CUDA", 6: "ATTN_ERR_DEVICE_TIMEOUT",
                7: "ATTN_ERR_WORKSPACE", 8: "ATTN_ERR_TOO_LARGE"}

_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s" % (what, status_string(status) if _lib else STATUS_NAMES.get(status)))


def load() -> ctypes.CDLL:
    """Load libattn_b200.so from the package folder (raises if it is not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libattn_b200.so is not built (run `python -m "
                           "dnn_compiler_pipelining_b200.build`); there is no fallback path")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, u64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_size_t
    lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
    lib.attn_fwd.restype = i
    lib.attn_fwd_qk.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
    lib.attn_fwd_qk.restype = i
    lib.attn_fwd_variant.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp]
    lib.attn_fwd_variant.restype = i
    lib.attn_variant_count.argtypes = []
    lib.attn_variant_count.restype = i
    lib.attn_variant_name.argtypes = [i]
    lib.attn_variant_name.restype = ctypes.c_char_p
    lib.attn_variant_select.argtypes = [i, i, i, i, i, i, i]
    lib.attn_variant_select.restype = i
    lib.attn_decoder_layer_workspace_bytes.argtypes = [i] * 7
    lib.attn_decoder_layer_workspace_bytes.restype = sz
    lib.attn_decoder_layer_fwd.argtypes = [vp] * 8 + [i] * 7 + [ctypes.c_float] * 2 + [vp, sz, vp]
    lib.attn_decoder_layer_fwd.restype = i
    lib.attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
    lib.attn_fwd_noalloc.restype = i
    lib.attn_fwd_host.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, sz, vp]
    lib.attn_fwd_host.restype = i
    lib.attn_fwd_host_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.attn_fwd_host_workspace_bytes.restype = sz
    lib.attn_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.attn_device_status.restype = i
    lib.attn_device_status_ex.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32),
                                          ctypes.POINTER(ctypes.c_uint64)]
    lib.attn_device_status_ex.restype = i
    lib.attn_noalloc_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32),
                                        ctypes.POINTER(ctypes.c_uint64)]
    lib.attn_noalloc_status.restype = i
    lib.attn_set_wait_timeout_ns.argtypes = [u64]
    lib.attn_set_wait_timeout_ns.restype = u64
    lib.attn_selftest_exp2.argtypes = [vp, vp, i, vp]
    lib.attn_selftest_exp2.restype = i
    lib.attn_selftest_fastdiv.argtypes = [ctypes.c_uint32, vp, vp, i, i, vp]
    lib.attn_selftest_fastdiv.restype = i
    lib.attn_selftest_wait_timeout.argtypes = [u64, vp]
    lib.attn_selftest_wait_timeout.restype = i
    lib.attn_status_string.argtypes = [i]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_version.argtypes = []
    lib.attn_version.restype = i
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().attn_status_string(int(status)).decode()


def version() -> int:
    return int(load().attn_version())


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _check_dev(t: torch.Tensor, name: str, dtype):
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError("%s must be a contiguous CUDA %s tensor" % (name, dtype))


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True,
             o: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None):
    """O, LSE = attention(Q, K, V) on the GPU through the C ABI.

    q: [B,Hq,Sq,D] fp16; k, v: [B,Hkv,Sk,D] fp16 (contiguous, on the current
    device).  Returns (o [B,Hq,Sq,D] fp16, lse [B,Hq,Sq] fp32); o / lse may be
    passed in preallocated.  Sq == Sk calls attn_fwd, otherwise attn_fwd_qk
    (causal window aligned at the bottom right, Sq <= Sk).  Asynchronous on
    ``stream`` (default: the current torch stream).
    """
    lib = load()
    _check_dev(q, "q", torch.float16)
    _check_dev(k, "k", torch.float16)
    _check_dev(v, "v", torch.float16)
    B, Hq, S, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    if tuple(k.shape) != (B, Hkv, Sk, D) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("shape mismatch: q %s k %s v %s" % (tuple(q.shape), tuple(k.shape),
                                                             tuple(v.shape)))
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
    _check_dev(o, "o", torch.float16)
    _check_dev(lse, "lse", torch.float32)
    if Sk == S:
        st = lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                          B, Hq, Hkv, S, D, int(bool(causal)), _stream_ptr(stream))
    else:
        st = lib.attn_fwd_qk(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             lse.data_ptr(), B, Hq, Hkv, S, Sk, D, int(bool(causal)),
                             _stream_ptr(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd" if Sk == S else "attn_fwd_qk")
    return o, lse


def variant_count() -> int:
    """Number of compiled fused-pass variants."""
    return int(load().attn_variant_count())


def variant_name(variant: int) -> str | None:
    name = load().attn_variant_name(int(variant))
    return name.decode() if name is not None else None


def variant_select(B: int, Hq: int, Hkv: int, Sq: int, Sk: int, D: int, causal: bool) -> int:
    """The variant the library's measured table picks for these sizes (-1: invalid sizes).
    Host-only: touches no device."""
    return int(load().attn_variant_select(B, Hq, Hkv, Sq, Sk, D, int(bool(causal))))


def attn_fwd_variant(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool,
                     variant: int, o: torch.Tensor | None = None,
                     lse: torch.Tensor | None = None, stream=None):
    """attn_fwd with an explicit fused-pass variant (for the tuner and tests)."""
    lib = load()
    _check_dev(q, "q", torch.float16)
    _check_dev(k, "k", torch.float16)
    _check_dev(v, "v", torch.float16)
    B, Hq, S, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    if tuple(k.shape) != (B, Hkv, Sk, D) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("shape mismatch: q %s k %s v %s" % (tuple(q.shape), tuple(k.shape),
                                                             tuple(v.shape)))
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
    _check_dev(o, "o", torch.float16)
    _check_dev(lse, "lse", torch.float32)
    st = lib.attn_fwd_variant(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              lse.data_ptr(), B, Hq, Hkv, S, Sk, D, int(bool(causal)),
                              int(variant), _stream_ptr(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_variant")
    return o, lse


def attn_fwd_raw(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int, B: int, Hq: int,
                 Hkv: int, S: int, D: int, causal: bool, stream_ptr: int) -> int:
    """The C entry point with raw addresses; returns the status code."""
    return int(load().attn_fwd(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, Hq, Hkv, S, D,
                               int(bool(causal)), stream_ptr))


def attn_fwd_noalloc_raw(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int, B: int,
                        Hq: int, Hkv: int, S: int, D: int, causal: bool, stream_ptr: int) -> int:
    """The no-allocation C entry point with raw addresses; returns the status
    code.  For callers that cannot let the library call cudaMalloc (memory
    planned up front, their own caching allocator, or no tolerance for the
    device synchronization an allocation may cause): its per-call status
    words are a fixed array inside the library (read them with
    noalloc_status), shared by every such call on a device."""
    return int(load().attn_fwd_noalloc(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, Hq, Hkv, S, D,
                                       int(bool(causal)), stream_ptr))


DECODER_WEIGHTS = ("w_attn_norm", "w_qkv", "w_o", "w_mlp_norm", "w_gate_up", "w_down")


def decoder_layer_workspace_bytes(B: int, S: int, hidden: int, Hq: int, Hkv: int, D: int,
                                  inter: int) -> int:
    return int(load().attn_decoder_layer_workspace_bytes(B, S, hidden, Hq, Hkv, D, inter))


def decoder_layer_fwd(x: torch.Tensor, weights: dict, Hq: int, Hkv: int, D: int,
                      eps: float = 1e-5, rope_theta: float = 500000.0,
                      y: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """One LLaMA3 decoder layer (include/decoder_layer.h) on CUDA fp16 tensors.

    x: [B, S, hidden]; weights: the six tensors named in DECODER_WEIGHTS, laid
    out as the C ABI states.  y (default: new) may be x itself.  workspace:
    a CUDA uint8 tensor of at least decoder_layer_workspace_bytes(...) bytes
    (default: allocated here).  Asynchronous on ``stream``."""
    lib = load()
    _check_dev(x, "x", torch.float16)
    B, S, hidden = x.shape
    inter = weights["w_down"].shape[1]
    for name in DECODER_WEIGHTS:
        _check_dev(weights[name], name, torch.float16)
    if y is None:
        y = torch.empty_like(x)
    _check_dev(y, "y", torch.float16)
    need = decoder_layer_workspace_bytes(B, S, hidden, Hq, Hkv, D, inter)
    if need == 0:
        raise AttnError(2, "attn_decoder_layer_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    st = lib.attn_decoder_layer_fwd(
        x.data_ptr(), *[weights[n].data_ptr() for n in DECODER_WEIGHTS], y.data_ptr(), B, S,
        hidden, Hq, Hkv, D, inter, float(eps), float(rope_theta), workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_decoder_layer_fwd")
    return y


def host_workspace_bytes(B: int, Hq: int, Hkv: int, S: int, D: int) -> int:
    return int(load().attn_fwd_host_workspace_bytes(B, Hq, Hkv, S, D))


def attn_fwd_host(q_h: torch.Tensor, k_h: torch.Tensor, v_h: torch.Tensor, o_h: torch.Tensor,
                  lse_h: torch.Tensor, causal: bool, workspace: torch.Tensor, stream=None):
    """Host-buffer entry: CPU tensors in and out, device workspace from the caller.
    Synchronizes the stream before returning."""
    lib = load()
    for t, n in ((q_h, "q"), (k_h, "k"), (v_h, "v"), (o_h, "o"), (lse_h, "lse")):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("%s must be a contiguous CPU tensor" % n)
    B, Hq, S, D = q_h.shape
    Hkv = k_h.shape[1]
    st = lib.attn_fwd_host(q_h.data_ptr(), k_h.data_ptr(), v_h.data_ptr(), o_h.data_ptr(),
                           lse_h.data_ptr(), B, Hq, Hkv, S, D, int(bool(causal)),
                           workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                           _stream_ptr(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_host")


def device_status(stream=None):
    """(status, site): synchronizes the stream, reads and clears its status block."""
    site = ctypes.c_uint32(0)
    st = load().attn_device_status(_stream_ptr(stream), ctypes.byref(site))
    return int(st), int(site.value)


def device_status_ex(stream=None):
    """(status, site, exact_items): as device_status, plus how many work items
    the kernels recomputed in their exact pass since the last read."""
    site = ctypes.c_uint32(0)
    n = ctypes.c_uint64(0)
    st = load().attn_device_status_ex(_stream_ptr(stream), ctypes.byref(site), ctypes.byref(n))
    return int(st), int(site.value), int(n.value)


def noalloc_status(stream=None):
    """(status, site, exact_items) of the attn_fwd_noalloc calls on this device
    since the last read; synchronizes the stream, then clears the words."""
    site = ctypes.c_uint32(0)
    n = ctypes.c_uint64(0)
    st = load().attn_noalloc_status(_stream_ptr(stream), ctypes.byref(site), ctypes.byref(n))
    return int(st), int(site.value), int(n.value)


def set_wait_timeout_ns(ns: int) -> int:
    return int(load().attn_set_wait_timeout_ns(int(ns)))


def selftest_wait_timeout(ns: int, stream=None) -> int:
    return int(load().attn_selftest_wait_timeout(int(ns), _stream_ptr(stream)))


def selftest_fastdiv(d: int, n: torch.Tensor) -> torch.Tensor:
    """n // d through the kernels' multiply-shift division; n is an int32
    tensor of values in [0, 2^31), on the CPU (host arithmetic) or on the GPU
    (device arithmetic)."""
    n = n.contiguous()
    if n.dtype != torch.int32:
        raise ValueError("n must be int32")
    q = torch.empty_like(n)
    st = load().attn_selftest_fastdiv(int(d), n.data_ptr(), q.data_ptr(), n.numel(),
                                      1 if n.is_cuda else 0, _stream_ptr(None) if n.is_cuda else None)
    if st != ATTN_OK:
        raise AttnError(st, "attn_selftest_fastdiv")
    if n.is_cuda:
        torch.cuda.current_stream().synchronize()
    return q


def selftest_exp2(x: torch.Tensor) -> torch.Tensor:
    """The fused pass's FMA-pipe 2^x, evaluated on a CUDA fp32 tensor."""
    _check_dev(x, "x", torch.float32)
    y = torch.empty_like(x)
    st = load().attn_selftest_exp2(x.data_ptr(), y.data_ptr(), x.numel(), _stream_ptr(None))
    if st != ATTN_OK:
        raise AttnError(st, "attn_selftest_exp2")
    return y
