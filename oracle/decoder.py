"""fp64 CPU oracle of the LLaMA3 single-decoder-layer proxy -- TEST
INFRASTRUCTURE ONLY (same rule as the rest of ``oracle/``: only tests, smoke
and the bench's CPU legs may use it; the product path never does).

The PipeThreader pages report an FP16 single decoder layer of LLaMA3-8B / 70B
as a layer-level proxy (papers.lqhl.me "PipeThreader-OSDI25", section
实验与结果, paper Sec. 6.3 / Fig. 13) but do not spell the layer out.  This
module writes out the standard pre-norm LLaMA3 layer from the published
definitions of its parts: RMSNorm (Zhang & Sennrich, 2019), rotary position
embedding in the half-split pairing (Su et al., RoFormer, 2021, as LLaMA
applies it), grouped-query causal attention (this package's C oracle) and
the SwiGLU MLP (Shazeer, 2020).

Precision: the layer is FP16, so every tensor that the layer materialises
between steps is rounded to fp16 (``f16``) at the point where it is stored;
each step itself is computed in fp64.  ``round_fp16=False`` gives the pure
fp64 layer.
"""
from __future__ import annotations

import numpy as np

from oracle import attention


def f16(a):
    """Round to the nearest fp16 value (ties to even), kept as fp64."""
    return np.asarray(a, dtype=np.float64).astype(np.float16).astype(np.float64)


def rmsnorm(x, w, eps):
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * w."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(w, dtype=np.float64)


def rope_angles(S, D, theta):
    """[S, D/2] angles: position s, pair i turns by s * theta^(-2i/D)."""
    i = np.arange(D // 2, dtype=np.float64)
    inv_freq = np.power(float(theta), -2.0 * i / D)
    return np.arange(S, dtype=np.float64)[:, None] * inv_freq[None, :]


def rope(x, theta):
    """Rotary embedding of x [..., S, D]: the pair (i, i + D/2) of position s is
    rotated by s * theta^(-2i/D) (first half gets cos - sin, second sin + cos)."""
    x = np.asarray(x, dtype=np.float64)
    S, D = x.shape[-2], x.shape[-1]
    ang = rope_angles(S, D, theta)
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., : D // 2], x[..., D // 2:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def silu(a):
    """a * sigmoid(a) = a / (1 + e^-a)."""
    a = np.asarray(a, dtype=np.float64)
    return a / (1.0 + np.exp(-a))


def decoder_layer(x, w_attn_norm, w_qkv, w_o, w_mlp_norm, w_gate_up, w_down, Hq, Hkv, D, eps,
                  theta, round_fp16=True, intermediates=None):
    """One LLaMA3 decoder layer.  x [B, S, hidden]; weights as the C ABI lays
    them out (w_qkv [(Hq + 2 Hkv) D, hidden] with query, key, value heads in
    that order; w_o [hidden, Hq D]; w_gate_up [2 I, hidden] gate rows then up
    rows; w_down [hidden, I]).  Returns y [B, S, hidden] in fp64.  A dict
    passed as ``intermediates`` receives the stored tensors (o_tok: the
    attention output per token [B, S, Hq D], h, g) for error budgets; the
    arithmetic is the same either way."""
    r = f16 if round_fp16 else (lambda a: np.asarray(a, dtype=np.float64))
    x = np.asarray(x, dtype=np.float64)
    B, S, _ = x.shape
    inter = np.asarray(w_down).shape[1]
    # attention block
    n1 = r(rmsnorm(x, w_attn_norm, eps))
    qkv = r(n1 @ np.asarray(w_qkv, dtype=np.float64).T)
    heads = qkv.reshape(B, S, Hq + 2 * Hkv, D).transpose(0, 2, 1, 3)  # [B, heads, S, D]
    q = r(rope(heads[:, :Hq], theta))
    k = r(rope(heads[:, Hq:Hq + Hkv], theta))
    v = heads[:, Hq + Hkv:]
    o, _ = attention(np.ascontiguousarray(q), np.ascontiguousarray(k), np.ascontiguousarray(v),
                     True)
    o = r(o)
    o_tok = o.transpose(0, 2, 1, 3).reshape(B, S, Hq * D)
    h = r(x + o_tok @ np.asarray(w_o, dtype=np.float64).T)
    # MLP block
    n2 = r(rmsnorm(h, w_mlp_norm, eps))
    gu = r(n2 @ np.asarray(w_gate_up, dtype=np.float64).T)
    g = r(silu(gu[..., :inter]) * gu[..., inter:])
    if intermediates is not None:
        intermediates.update(o_tok=o_tok, h=h, g=g)
    return r(h + g @ np.asarray(w_down, dtype=np.float64).T)
