"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no attention arithmetic: it only draws i.i.d. normal numbers
and rounds them to fp16.  Both the CUDA path and the CPU oracle receive the
same fp16 tensors (the oracle reads them as exact fp64 values).

Recipe (the pages measure on synthetic LLaMA3-8B/70B head shapes, papers.lqhl.me
"PipeThreader-OSDI25", paper Sec. 6.2 / Fig. 12; no dataset or weights are
involved):
  * Q, K, V have shapes [B,Hq,S,D], [B,Hkv,S,D], [B,Hkv,S,D], dense row-major.
  * Each tensor has its own torch generator on ``device``: Q uses ``seed``,
    K ``seed + 1``, V ``seed + 2``.
  * Values are N(0, std^2) drawn in fp32 by ``torch.randn``, multiplied by std,
    then rounded to fp16 (round-to-nearest-even).  The standard workloads use
    std 1 for all three; the stress sweep uses std 4 for Q and K (large logits)
    and std 1 for V.
  * Large tensors are drawn in fixed chunks along the batch axis so the fp32
    temporary stays small; the chunking is part of the recipe, so a given
    (shape, seed, device) always yields the same values.
"""
from __future__ import annotations

import torch

_CHUNK_ELEMS = 1 << 26  # fp32 temporaries of at most 256 MiB


def _normal_fp16(shape, seed: int, std: float, device, mean: float = 0.0) -> torch.Tensor:
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    out = torch.empty(shape, dtype=torch.float16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    step = _CHUNK_ELEMS
    for start in range(0, n, step):
        m = min(step, n - start)
        x = torch.randn(m, generator=gen, dtype=torch.float32, device=device)
        if std != 1.0:
            x.mul_(std)
        if mean != 0.0:
            x.add_(mean)
        flat[start:start + m].copy_(x)
    return out


def make_qkv(B: int, Hq: int, Hkv: int, S: int, D: int, seed: int = 0,
             qk_std: float = 1.0, v_std: float = 1.0, device="cpu"):
    """Return fp16 (Q, K, V) on ``device`` following the recipe above."""
    q = _normal_fp16((B, Hq, S, D), seed, qk_std, device)
    k = _normal_fp16((B, Hkv, S, D), seed + 1, qk_std, device)
    v = _normal_fp16((B, Hkv, S, D), seed + 2, v_std, device)
    return q, k, v


# Workloads named by what they are (LLaMA3 head shapes from the pages).
WORKLOADS = {
    "llama3-8b-s512-b1": dict(B=1, Hq=32, Hkv=8, S=512, D=128, causal=True),
    "llama3-8b-s8192-b1": dict(B=1, Hq=32, Hkv=8, S=8192, D=128, causal=True),
    "llama3-8b-s2048-b64": dict(B=64, Hq=32, Hkv=8, S=2048, D=128, causal=True),
    "llama3-70b-s8192-b64": dict(B=64, Hq=64, Hkv=8, S=8192, D=128, causal=True),
    "llama3-8b-s8192-b64": dict(B=64, Hq=32, Hkv=8, S=8192, D=128, causal=True),
    # the large-head case: 8B head counts at head dimension 256
    "gqa32x8-d256-s8192-b16": dict(B=16, Hq=32, Hkv=8, S=8192, D=256, causal=True),
    # small cases of the same kernel for profiler captures (Q alone exceeds L2)
    "llama3-8b-s8192-b4": dict(B=4, Hq=32, Hkv=8, S=8192, D=128, causal=True),
    "llama3-8b-s2048-b8": dict(B=8, Hq=32, Hkv=8, S=2048, D=128, causal=True),
    "llama3-70b-s8192-b4": dict(B=4, Hq=64, Hkv=8, S=8192, D=128, causal=True),
    "gqa32x8-d256-s8192-b2": dict(B=2, Hq=32, Hkv=8, S=8192, D=256, causal=True),
}


def sweep_points():
    """The 40-point stress sweep: both head shapes x SEQ x BS x mask."""
    pts = []
    for Hq in (32, 64):
        for S in (512, 1024, 2048, 4096, 8192):
            for B in (1, 64):
                for causal in (True, False):
                    pts.append(dict(B=B, Hq=Hq, Hkv=8, S=S, D=128, causal=causal))
    return pts



# Decoder-layer proxy (the pages' second workload: an FP16 single LLaMA3-8B /
# 70B decoder layer, papers.lqhl.me "PipeThreader-OSDI25", paper Sec. 6.3 /
# Fig. 13): model dimensions of the two LLaMA3 sizes.
DECODER_MODELS = {
    "llama3-8b": dict(hidden=4096, Hq=32, Hkv=8, D=128, inter=14336),
    "llama3-70b": dict(hidden=8192, Hq=64, Hkv=8, D=128, inter=28672),
}


def make_decoder_inputs(B: int, S: int, hidden: int, Hq: int, Hkv: int, D: int, inter: int,
                        seed: int = 0, device="cpu"):
    """Synthetic activations and weights of one decoder layer, fp16 on ``device``.

    x ~ N(0, 1) [B, S, hidden]; each projection W [out, in] ~ N(0, 1/in), so
    every product keeps unit scale; the two RMSNorm weights ~ N(1, 0.1^2).
    Tensor k of (x, w_attn_norm, w_qkv, w_o, w_mlp_norm, w_gate_up, w_down)
    uses seed + k.  Returns (x, weights dict keyed as the C ABI names them).
    """
    x = _normal_fp16((B, S, hidden), seed, 1.0, device)
    w = {
        "w_attn_norm": _normal_fp16((hidden,), seed + 1, 0.1, device, mean=1.0),
        "w_qkv": _normal_fp16(((Hq + 2 * Hkv) * D, hidden), seed + 2, hidden ** -0.5, device),
        "w_o": _normal_fp16((hidden, Hq * D), seed + 3, (Hq * D) ** -0.5, device),
        "w_mlp_norm": _normal_fp16((hidden,), seed + 4, 0.1, device, mean=1.0),
        "w_gate_up": _normal_fp16((2 * inter, hidden), seed + 5, hidden ** -0.5, device),
        "w_down": _normal_fp16((hidden, inter), seed + 6, inter ** -0.5, device),
    }
    return x, w
