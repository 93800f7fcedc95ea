"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI,
run the fp64 oracle on the same fp16 inputs (all rows, or sampled rows), and
compare element by element.

Tolerances (fixed for the fp16 attention forward): max |O_gpu - O_ref| <= 2e-3
and max |LSE_gpu - LSE_ref| <= 1e-3, with O_gpu read as exact fp64 values of
the fp16 output and O_ref, LSE_ref the fp64 oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from dnn_compiler_pipelining_b200 import attn
from dnn_compiler_pipelining_b200.inputs import make_qkv

O_TOL = 2e-3
LSE_TOL = 1e-3


def run_gpu(q, k, v, causal):
    o = torch.full_like(q, float("nan"))  # poison: every element must be written
    lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device=q.device)
    attn.attn_fwd(q, k, v, causal, o=o, lse=lse)
    st, site = attn.device_status()
    assert st == attn.ATTN_OK, "device status %d at site %#x" % (st, site)
    return o, lse


def error_report(o_gpu, o_ref, lse_gpu, lse_ref):
    eo = np.abs(o_gpu - o_ref)
    el = np.abs(lse_gpu - lse_ref)
    mag = np.abs(o_ref)
    buckets = []
    for lo, hi in ((0, 1), (1, 2), (2, 4), (4, 8), (8, np.inf)):
        m = (mag >= lo) & (mag < hi)
        if m.any():
            buckets.append("|O| in [%g,%g): n=%d max err %.3e" % (lo, hi, m.sum(), eo[m].max()))
    return float(eo.max()), float(el.max()), "; ".join(buckets)


def assert_close(o_gpu, o_ref, lse_gpu, lse_ref, what=""):
    assert np.all(np.isfinite(o_gpu)) and np.all(np.isfinite(lse_gpu)), what + " non-finite output"
    eo, el, rep = error_report(o_gpu, o_ref, lse_gpu, lse_ref)
    assert eo <= O_TOL and el <= LSE_TOL, "%s: O err %.3e, LSE err %.3e (%s)" % (what, eo, el, rep)
    return eo, el


def full_check(B, Hq, Hkv, S, D, causal, seed=0, qk_std=1.0):
    q, k, v = make_qkv(B, Hq, Hkv, S, D, seed=seed, qk_std=qk_std, device="cuda")
    o, lse = run_gpu(q, k, v, causal)
    o_ref, lse_ref = oracle.attention(q.cpu().double().numpy(), k.cpu().double().numpy(),
                                      v.cpu().double().numpy(), causal)
    return assert_close(o.cpu().double().numpy(), o_ref, lse.cpu().double().numpy(), lse_ref,
                        "B%d Hq%d Hkv%d S%d causal=%d" % (B, Hq, Hkv, S, causal))


def sample_rows(B, Hq, S, n_random, seed):
    """(b, hq) heads checked in full, plus seeded random (b, hq, i) rows that
    always include positions 0, 127, 128 and S-1."""
    group_heads = {(0, 0), (0, Hq - 1), (B - 1, Hq // 2)}
    rng = np.random.default_rng(seed)
    # a head from a different kv group than head 0 (Hq/Hkv >= 1)
    group_heads.add((B // 2, int(rng.integers(Hq // 2, Hq))))
    rows = {}
    for bh in group_heads:
        rows.setdefault(bh, set()).update(range(S))
    fixed = [0, min(127, S - 1), min(128, S - 1), S - 1]
    for n in range(n_random):
        b, h = int(rng.integers(B)), int(rng.integers(Hq))
        i = fixed[n] if n < len(fixed) else int(rng.integers(S))
        rows.setdefault((b, h), set()).add(i)
    return {bh: np.array(sorted(s), dtype=np.int64) for bh, s in rows.items()}


def sampled_check(q, k, v, o, lse, causal, n_random=1024, seed=1234, full_heads=True):
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    group = Hq // Hkv
    rows = sample_rows(B, Hq, S, n_random, seed)
    if not full_heads:
        rows = {bh: r for bh, r in rows.items() if len(r) < S}
    worst_o = worst_l = 0.0
    n_rows = 0
    for (b, h), pos in rows.items():
        g = h // group
        pos_t = torch.from_numpy(pos).to(q.device)
        q_rows = q[b, h].index_select(0, pos_t).cpu().double().numpy()
        o_ref, lse_ref = oracle.attention_rows(q_rows, pos, k[b, g].cpu().double().numpy(),
                                               v[b, g].cpu().double().numpy(), causal)
        o_g = o[b, h].index_select(0, pos_t).cpu().double().numpy()
        l_g = lse[b, h].index_select(0, pos_t).cpu().double().numpy()
        eo, el = assert_close(o_g, o_ref, l_g, lse_ref, "head (%d,%d)" % (b, h))
        worst_o, worst_l = max(worst_o, eo), max(worst_l, el)
        n_rows += len(pos)
    return worst_o, worst_l, n_rows
