"""Checks that pin the fp64 oracle to facts the mathematics fixes.

Each ``check_*`` takes the oracle module (or a stand-in with the same API) and
raises AssertionError on a violation.  ``test_oracle_pins.py`` runs them
against the real oracle, and against deliberately broken copies to show that
each plausible mistake fails at least one of them.

Operator: scaled dot-product attention with an optional causal mask and
grouped-query heads (the PipeThreader pages' FlashAttention workload,
papers.lqhl.me "PipeThreader-OSDI25", paper Sec. 6.2 / Fig. 12; the pages do
not print the formula, the textbook definition is used).
"""
from __future__ import annotations

import glob
import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def check_golden(orc):
    """Hand-worked cases (tests/golden/*.json): exact closed forms."""
    files = sorted(glob.glob(os.path.join(GOLDEN, "*.json")))
    assert len(files) >= 4, files
    for f in files:
        c = json.load(open(f))
        B, Hq, Hkv, S, D = c["B"], c["Hq"], c["Hkv"], c["S"], c["D"]
        q = np.array(c["q"], dtype=np.float64).reshape(B, Hq, S, D)
        k = np.array(c["k"], dtype=np.float64).reshape(B, Hkv, S, D)
        v = np.array(c["v"], dtype=np.float64).reshape(B, Hkv, S, D)
        o, lse = orc.attention(q, k, v, c["causal"])
        eo = np.array(c["o"], dtype=np.float64).reshape(B, Hq, S, D)
        el = np.array(c["lse"], dtype=np.float64).reshape(B, Hq, S)
        assert np.allclose(o, eo, rtol=0, atol=1e-12), (c["name"], o, eo)
        assert np.allclose(lse, el, rtol=0, atol=1e-12), (c["name"], lse, el)


def check_row_sums(orc):
    """Each probability row sums to 1 and is zero outside the causal window."""
    r = _rng(1)
    S, D = 37, 16
    k = r.normal(size=(S, D)) * 2
    for causal in (True, False):
        for i in (0, 1, 17, S - 1):
            q = r.normal(size=(D,)) * 2
            p, _ = orc.probs_row(q, k, i, causal)
            assert abs(p.sum() - 1.0) < 1e-12, p.sum()
            assert np.all(p >= 0)
            if causal:
                assert np.all(p[i + 1:] == 0.0)
                assert np.all(p[: i + 1] > 0.0)


def check_constant_v(orc):
    """Every value row equal to c gives O = c on every row (softmax is convex)."""
    r = _rng(2)
    B, Hq, Hkv, S, D = 2, 4, 2, 29, 8
    q = r.normal(size=(B, Hq, S, D))
    k = r.normal(size=(B, Hkv, S, D))
    c = r.normal(size=(D,))
    v = np.broadcast_to(c, (B, Hkv, S, D)).copy()
    for causal in (True, False):
        o, _ = orc.attention(q, k, v, causal)
        assert np.allclose(o, np.broadcast_to(c, o.shape), rtol=0, atol=1e-12)


def check_zero_query(orc):
    """Q = 0: all logits are 0, so O_i is the mean of the visible values and
    LSE_i = ln(#visible keys): causal prefix mean / ln(i+1); non-causal mean / ln S."""
    r = _rng(3)
    B, Hq, Hkv, S, D = 1, 2, 1, 23, 4
    q = np.zeros((B, Hq, S, D))
    k = r.normal(size=(B, Hkv, S, D))
    v = r.normal(size=(B, Hkv, S, D))
    o, lse = orc.attention(q, k, v, True)
    prefix = np.cumsum(v[0, 0], axis=0) / np.arange(1, S + 1)[:, None]
    for h in range(Hq):
        assert np.allclose(o[0, h], prefix, rtol=0, atol=1e-12)
        assert np.allclose(lse[0, h], np.log(np.arange(1, S + 1)), rtol=0, atol=1e-12)
    o, lse = orc.attention(q, k, v, False)
    assert np.allclose(o[0, 0], np.broadcast_to(v[0, 0].mean(axis=0), (S, D)), rtol=0, atol=1e-12)
    assert np.allclose(lse, math.log(S), rtol=0, atol=1e-12)


def check_first_causal_row(orc):
    """Causal row 0 sees only key 0: O_0 = V_0 and LSE_0 = q_0.k_0/sqrt(D)."""
    r = _rng(4)
    B, Hq, Hkv, S, D = 1, 1, 1, 9, 16
    q = r.normal(size=(B, Hq, S, D))
    k = r.normal(size=(B, Hkv, S, D))
    v = r.normal(size=(B, Hkv, S, D))
    o, lse = orc.attention(q, k, v, True)
    assert np.allclose(o[0, 0, 0], v[0, 0, 0], rtol=0, atol=1e-13)
    assert abs(lse[0, 0, 0] - float(q[0, 0, 0] @ k[0, 0, 0]) / math.sqrt(D)) < 1e-12


def check_permutation(orc):
    """Non-causal: permuting key and value rows together leaves O and LSE unchanged."""
    r = _rng(5)
    B, Hq, Hkv, S, D = 1, 2, 2, 31, 8
    q = r.normal(size=(B, Hq, S, D)) * 2
    k = r.normal(size=(B, Hkv, S, D)) * 2
    v = r.normal(size=(B, Hkv, S, D))
    perm = r.permutation(S)
    o1, l1 = orc.attention(q, k, v, False)
    o2, l2 = orc.attention(q, k[:, :, perm], v[:, :, perm], False)
    assert np.allclose(o1, o2, rtol=0, atol=1e-12)
    assert np.allclose(l1, l2, rtol=0, atol=1e-12)


def check_key_shift(orc):
    """Adding one vector w to every key row adds q.w/sqrt(D) to every logit of a
    row: O is unchanged and LSE shifts by exactly that amount."""
    r = _rng(6)
    B, Hq, Hkv, S, D = 1, 2, 1, 19, 8
    q = r.normal(size=(B, Hq, S, D))
    k = r.normal(size=(B, Hkv, S, D))
    v = r.normal(size=(B, Hkv, S, D))
    w = r.normal(size=(D,))
    for causal in (True, False):
        o1, l1 = orc.attention(q, k, v, causal)
        o2, l2 = orc.attention(q, k + w, v, causal)
        assert np.allclose(o1, o2, rtol=0, atol=1e-11)
        assert np.allclose(l2 - l1, (q @ w) / math.sqrt(D), rtol=0, atol=1e-11)


def check_hard_attention(orc):
    """Scaling Q by 1e3 makes the softmax one-hot on the largest logit: O_i = V_argmax."""
    r = _rng(7)
    B, Hq, Hkv, S, D = 1, 1, 1, 17, 8
    q = r.normal(size=(B, Hq, S, D)) * 1e3
    k = r.normal(size=(B, Hkv, S, D))
    v = r.normal(size=(B, Hkv, S, D))
    for causal in (True, False):
        o, _ = orc.attention(q, k, v, causal)
        checked = 0
        for i in range(S):
            n = i + 1 if causal else S
            s = np.sort(k[0, 0, :n] @ q[0, 0, i] / math.sqrt(D))
            if n > 1 and s[-1] - s[-2] < 60.0:  # runner-up weight above e^-60: not one-hot
                continue
            j = int(np.argmax(k[0, 0, :n] @ q[0, 0, i]))
            assert np.allclose(o[0, 0, i], v[0, 0, j], rtol=0, atol=1e-12)
            checked += 1
        assert checked >= S // 2, checked


def check_gqa(orc):
    """Grouped-query heads equal multi-head attention with each kv head repeated
    for its contiguous group of Hq/Hkv query heads."""
    r = _rng(8)
    B, Hq, Hkv, S, D = 2, 8, 2, 13, 4
    q = r.normal(size=(B, Hq, S, D))
    k = r.normal(size=(B, Hkv, S, D))
    v = r.normal(size=(B, Hkv, S, D))
    kr = np.repeat(k, Hq // Hkv, axis=1)
    vr = np.repeat(v, Hq // Hkv, axis=1)
    for causal in (True, False):
        o1, l1 = orc.attention(q, k, v, causal)
        o2, l2 = orc.attention(q, kr, vr, causal)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def check_library(orc):
    """fp64 CPU torch scaled_dot_product_attention (kv heads repeated), with LSE
    rebuilt by torch.logsumexp of the scaled, masked logits."""
    import torch
    r = _rng(9)
    B, Hq, Hkv, S, D = 2, 4, 2, 45, 32
    q = r.normal(size=(B, Hq, S, D)) * 2
    k = r.normal(size=(B, Hkv, S, D)) * 2
    v = r.normal(size=(B, Hkv, S, D))
    tq = torch.from_numpy(q)
    tk = torch.from_numpy(np.repeat(k, Hq // Hkv, axis=1))
    tv = torch.from_numpy(np.repeat(v, Hq // Hkv, axis=1))
    for causal in (True, False):
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
        logits = tq @ tk.transpose(-1, -2) / math.sqrt(D)
        if causal:
            mask = torch.ones(S, S, dtype=torch.bool).triu(1)
            logits = logits.masked_fill(mask, float("-inf"))
        ref_lse = torch.logsumexp(logits, dim=-1)
        o, lse = orc.attention(q, k, v, causal)
        assert np.allclose(o, ref.numpy(), rtol=0, atol=1e-12)
        assert np.allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-12)


def check_rows_api(orc):
    """The per-row entry gives the same rows as the whole-tensor entry."""
    r = _rng(10)
    B, Hq, Hkv, S, D = 1, 4, 2, 33, 8
    q = r.normal(size=(B, Hq, S, D))
    k = r.normal(size=(B, Hkv, S, D))
    v = r.normal(size=(B, Hkv, S, D))
    for causal in (True, False):
        o, lse = orc.attention(q, k, v, causal)
        hq = 3
        g = hq // (Hq // Hkv)
        pos = np.array([0, 5, 32, 17])
        o2, l2 = orc.attention_rows(q[0, hq, pos], pos, k[0, g], v[0, g], causal)
        assert np.array_equal(o2, o[0, hq, pos]) and np.array_equal(l2, lse[0, hq, pos])


def check_qk_suffix(orc):
    """Bottom-right alignment: causal attention of the last Sq queries over all
    Sk keys equals the last Sq rows of the square causal problem (whose
    definition the pins above fix)."""
    r = _rng(11)
    B, Hq, Hkv, Sk, D = 1, 4, 2, 37, 16
    q = r.normal(size=(B, Hq, Sk, D)) * 2
    k = r.normal(size=(B, Hkv, Sk, D)) * 2
    v = r.normal(size=(B, Hkv, Sk, D))
    o_sq, l_sq = orc.attention(q, k, v, True)
    for sq in (1, 11, 36, 37):
        o, lse = orc.attention_qk(q[:, :, Sk - sq:], k, v, True)
        assert np.allclose(o, o_sq[:, :, Sk - sq:], rtol=0, atol=1e-12)
        assert np.allclose(lse, l_sq[:, :, Sk - sq:], rtol=0, atol=1e-12)


def check_qk_library(orc):
    """Sq != Sk against fp64 torch scaled_dot_product_attention: non-causal, and
    causal with the bottom-right boolean mask written out (j <= i + Sk - Sq)."""
    import torch
    r = _rng(12)
    B, Hq, Hkv, Sq, Sk, D = 2, 4, 2, 13, 29, 8
    q = r.normal(size=(B, Hq, Sq, D)) * 2
    k = r.normal(size=(B, Hkv, Sk, D)) * 2
    v = r.normal(size=(B, Hkv, Sk, D))
    tq = torch.from_numpy(q)
    tk = torch.from_numpy(np.repeat(k, Hq // Hkv, axis=1))
    tv = torch.from_numpy(np.repeat(v, Hq // Hkv, axis=1))
    ii = torch.arange(Sq).view(Sq, 1)
    jj = torch.arange(Sk).view(1, Sk)
    for causal in (True, False):
        keep = (jj <= ii + (Sk - Sq)) if causal else torch.ones(Sq, Sk, dtype=torch.bool)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=keep)
        logits = (tq @ tk.transpose(-1, -2) / math.sqrt(D)).masked_fill(~keep, float("-inf"))
        ref_lse = torch.logsumexp(logits, dim=-1)
        o, lse = orc.attention_qk(q, k, v, causal)
        assert np.allclose(o, ref.numpy(), rtol=0, atol=1e-12)
        assert np.allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-12)


def check_qk_edges(orc):
    """One causal query sees every key; a causal query with no visible key is
    rejected; the per-row entry agrees with the whole-tensor entry."""
    r = _rng(13)
    q = r.normal(size=(1, 2, 1, 8))
    k = r.normal(size=(1, 1, 20, 8))
    v = r.normal(size=(1, 1, 20, 8))
    oc, lc = orc.attention_qk(q, k, v, True)
    on, ln = orc.attention_qk(q, k, v, False)
    assert np.array_equal(oc, on) and np.array_equal(lc, ln)
    try:
        orc.attention_qk(r.normal(size=(1, 2, 21, 8)), k, v, True)
    except ValueError:
        pass
    else:
        raise AssertionError("causal Sq > Sk accepted")
    q2 = r.normal(size=(1, 2, 9, 8))
    o, lse = orc.attention_qk(q2, k, v, True)
    pos = np.array([0, 4, 8])
    o2, l2 = orc.attention_rows_qk(q2[0, 1, pos], pos, k[0, 0], v[0, 0], 9, True)
    assert np.array_equal(o2, o[0, 1, pos]) and np.array_equal(l2, lse[0, 1, pos])


ALL_CHECKS = [check_golden, check_row_sums, check_constant_v, check_zero_query,
              check_first_causal_row, check_permutation, check_key_shift,
              check_hard_attention, check_gqa, check_library, check_rows_api,
              check_qk_suffix, check_qk_library, check_qk_edges]
