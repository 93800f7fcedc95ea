"""Pins of the decoder-layer oracle (``oracle/decoder.py``) to what the
definitions of its parts fix, independent of the oracle's own code: closed
forms, special cases, invariants, and a brute-force loop version of the whole
layer on tiny inputs.  Each check takes the oracle module, so that the
planted-mistake tests can run it against altered copies."""
from __future__ import annotations

import math

import numpy as np


def _rng(seed):
    return np.random.default_rng(seed)


def check_rmsnorm(mod):
    # [3, 4]: mean square 12.5
    got = mod.rmsnorm(np.array([3.0, 4.0]), np.array([1.0, 1.0]), 0.0)
    assert np.allclose(got, [3 / math.sqrt(12.5), 4 / math.sqrt(12.5)], rtol=0, atol=1e-15)
    # a constant row normalises to its sign; the weight scales each column
    w = np.arange(1.0, 17.0)
    got = mod.rmsnorm(np.full(16, -2.5), w, 0.0)
    assert np.allclose(got, -w, rtol=0, atol=1e-14)
    # scale invariance (eps = 0) and eps keeps a zero row finite
    x = _rng(1).standard_normal((3, 32))
    assert np.allclose(mod.rmsnorm(7.0 * x, np.ones(32), 0.0), mod.rmsnorm(x, np.ones(32), 0.0),
                       rtol=0, atol=1e-13)
    z = mod.rmsnorm(np.zeros((1, 8)), np.ones(8), 1e-5)
    assert np.all(z == 0.0)
    # eps enters under the root: rms of [1, 1] with eps 3 is 2
    assert np.allclose(mod.rmsnorm(np.array([1.0, 1.0]), np.ones(2), 3.0), [0.5, 0.5], atol=1e-15)


def check_rope_conventions(mod):
    theta = 10000.0
    D = 4
    # position 0 is the identity
    x = _rng(2).standard_normal((1, 1, 3, D))
    assert np.allclose(mod.rope(x, theta)[..., 0, :], x[..., 0, :], rtol=0, atol=0)
    # half-split pairs (0, 2) and (1, 3); pair i turns by s * theta^(-2i/D)
    e = np.zeros((2, D))
    e[1, 0] = 1.0
    got = mod.rope(e, theta)[1]
    assert np.allclose(got, [math.cos(1.0), 0.0, math.sin(1.0), 0.0], rtol=0, atol=1e-15)
    e = np.zeros((2, D))
    e[1, 2] = 1.0
    got = mod.rope(e, theta)[1]
    assert np.allclose(got, [-math.sin(1.0), 0.0, math.cos(1.0), 0.0], rtol=0, atol=1e-15)
    e = np.zeros((4, D))
    e[3, 1] = 1.0
    a = 3.0 * theta ** -0.5
    got = mod.rope(e, theta)[3]
    assert np.allclose(got, [0.0, math.cos(a), 0.0, math.sin(a)], rtol=0, atol=1e-15)


def check_rope_invariants(mod):
    theta, S, D = 500000.0, 40, 64
    x = _rng(3).standard_normal((2, S, D))
    y = mod.rope(x, theta)
    # every (i, i + D/2) pair keeps its length
    n0 = x[..., : D // 2] ** 2 + x[..., D // 2:] ** 2
    n1 = y[..., : D // 2] ** 2 + y[..., D // 2:] ** 2
    assert np.allclose(n0, n1, rtol=1e-13, atol=1e-13)
    # <rope(q)_m, rope(k)_n> depends on m - n only
    q = _rng(4).standard_normal(D)
    k = _rng(5).standard_normal(D)
    X = np.zeros((S, D))
    X[3], X[10] = q, k
    Y = mod.rope(X, theta)
    d1 = float(Y[10] @ Y[3])
    X2 = np.zeros((S, D))
    X2[3 + 25], X2[10 + 25] = q, k
    Y2 = mod.rope(X2, theta)
    d2 = float(Y2[35] @ Y2[28])
    assert abs(d1 - d2) < 1e-10 * max(1.0, abs(d1))


def check_silu(mod):
    a = np.linspace(-8, 8, 33)
    s = mod.silu(a)
    assert mod.silu(np.array([0.0]))[0] == 0.0
    # silu(a) - silu(-a) = a, and silu(a) = a * sigmoid(a) at a = 1: 1 / (1 + 1/e)
    assert np.allclose(s - mod.silu(-a), a, rtol=0, atol=1e-14)
    assert abs(mod.silu(np.array([1.0]))[0] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15
    assert abs(mod.silu(np.array([-60.0]))[0]) < 1e-20


def check_f16(mod):
    assert mod.f16(1.0 + 2.0 ** -11) == 1.0           # a tie rounds to even
    assert mod.f16(1.0 + 3 * 2.0 ** -11) == 1.0 + 2.0 ** -9
    with np.errstate(over="ignore"):
        assert mod.f16(65519.0) == 65504.0 and np.isinf(mod.f16(65520.0))


def _weights(seed, hidden, Hq, Hkv, D, inter, norm_jitter=0.1):
    r = _rng(seed)
    return dict(
        w_attn_norm=1.0 + norm_jitter * r.standard_normal(hidden),
        w_qkv=r.standard_normal(((Hq + 2 * Hkv) * D, hidden)) / math.sqrt(hidden),
        w_o=r.standard_normal((hidden, Hq * D)) / math.sqrt(Hq * D),
        w_mlp_norm=1.0 + norm_jitter * r.standard_normal(hidden),
        w_gate_up=r.standard_normal((2 * inter, hidden)) / math.sqrt(hidden),
        w_down=r.standard_normal((hidden, inter)) / math.sqrt(inter))


def check_layer_zero_branches(mod):
    """W_o = 0 and W_down = 0: both residual branches vanish, y = x (rounded)."""
    hidden, Hq, Hkv, D, inter = 16, 2, 1, 8, 24
    w = _weights(6, hidden, Hq, Hkv, D, inter)
    w["w_o"] = np.zeros_like(w["w_o"])
    w["w_down"] = np.zeros_like(w["w_down"])
    x = _rng(7).standard_normal((2, 5, hidden))
    y = mod.decoder_layer(x, Hq=Hq, Hkv=Hkv, D=D, eps=1e-5, theta=10000.0, **w)
    assert np.array_equal(y, mod.f16(x))


def _rms(v, w, eps):
    return v / math.sqrt(sum(t * t for t in v) / len(v) + eps) * w


def check_layer_single_token(mod):
    """S = 1: each query sees only its own key, so attention returns V of the
    query head's group; the rest of the layer is then closed-form matmuls."""
    hidden, Hq, Hkv, D, inter, eps = 24, 4, 2, 8, 40, 1e-5
    w = _weights(8, hidden, Hq, Hkv, D, inter)
    x = _rng(9).standard_normal((3, 1, hidden))
    y = mod.decoder_layer(x, Hq=Hq, Hkv=Hkv, D=D, eps=eps, theta=500000.0, round_fp16=False, **w)
    group = Hq // Hkv
    for b in range(3):
        xv = x[b, 0]
        n1 = _rms(xv, w["w_attn_norm"], eps)
        proj = w["w_qkv"] @ n1
        o = np.concatenate([proj[(Hq + Hkv + hq // group) * D:(Hq + Hkv + hq // group + 1) * D]
                            for hq in range(Hq)])
        h = xv + w["w_o"] @ o
        n2 = _rms(h, w["w_mlp_norm"], eps)
        gate, up = w["w_gate_up"][:inter] @ n2, w["w_gate_up"][inter:] @ n2
        act = gate / (1.0 + np.exp(-gate)) * up
        ref = h + w["w_down"] @ act
        assert np.allclose(y[b, 0], ref, rtol=0, atol=1e-12), b


def _brute_layer(x, w, Hq, Hkv, D, inter, eps, theta):
    """The layer with explicit loops over tokens, heads and keys (fp64)."""
    B, S, hidden = x.shape
    group = Hq // Hkv
    y = np.zeros_like(x)
    for b in range(B):
        q = [[None] * S for _ in range(Hq)]
        k = [[None] * S for _ in range(Hkv)]
        v = [[None] * S for _ in range(Hkv)]
        for s in range(S):
            n1 = _rms(x[b, s], w["w_attn_norm"], eps)
            proj = [float(np.dot(w["w_qkv"][r], n1)) for r in range((Hq + 2 * Hkv) * D)]

            def rot(vec, pos):
                out = list(vec)
                for i in range(D // 2):
                    ang = pos * theta ** (-2.0 * i / D)
                    c, sn = math.cos(ang), math.sin(ang)
                    out[i] = vec[i] * c - vec[i + D // 2] * sn
                    out[i + D // 2] = vec[i + D // 2] * c + vec[i] * sn
                return out
            for hq in range(Hq):
                q[hq][s] = rot(proj[hq * D:(hq + 1) * D], s)
            for g in range(Hkv):
                k[g][s] = rot(proj[(Hq + g) * D:(Hq + g + 1) * D], s)
                v[g][s] = proj[(Hq + Hkv + g) * D:(Hq + Hkv + g + 1) * D]
        for s in range(S):
            o = []
            for hq in range(Hq):
                g = hq // group
                logits = [sum(q[hq][s][d] * k[g][j][d] for d in range(D)) / math.sqrt(D)
                          for j in range(s + 1)]
                mx = max(logits)
                p = [math.exp(t - mx) for t in logits]
                tot = sum(p)
                o += [sum(p[j] * v[g][j][d] for j in range(s + 1)) / tot for d in range(D)]
            h = x[b, s] + w["w_o"] @ np.array(o)
            n2 = _rms(h, w["w_mlp_norm"], eps)
            act = np.array([0.0] * inter)
            for j in range(inter):
                gt = float(np.dot(w["w_gate_up"][j], n2))
                up = float(np.dot(w["w_gate_up"][inter + j], n2))
                act[j] = gt / (1.0 + math.exp(-gt)) * up
            y[b, s] = h + w["w_down"] @ act
    return y


def check_layer_brute_force(mod):
    hidden, Hq, Hkv, D, inter, eps, theta = 8, 4, 2, 4, 12, 1e-5, 100.0
    w = _weights(10, hidden, Hq, Hkv, D, inter)
    # larger query/key weights give peaked attention, so the causal window and
    # the rotation matter
    w["w_qkv"] = w["w_qkv"] * 3.0
    x = _rng(11).standard_normal((2, 4, hidden))
    y = mod.decoder_layer(x, Hq=Hq, Hkv=Hkv, D=D, eps=eps, theta=theta, round_fp16=False, **w)
    ref = _brute_layer(x, w, Hq, Hkv, D, inter, eps, theta)
    assert np.allclose(y, ref, rtol=0, atol=1e-11), float(np.abs(y - ref).max())


def check_layer_rounds_like_fp16(mod):
    """With rounding on, the output is an fp16 value and within a few fp16
    steps of the fp64 layer."""
    hidden, Hq, Hkv, D, inter = 32, 4, 2, 8, 48
    w = _weights(12, hidden, Hq, Hkv, D, inter)
    x = _rng(13).standard_normal((2, 6, hidden))
    y16 = mod.decoder_layer(x, Hq=Hq, Hkv=Hkv, D=D, eps=1e-5, theta=10000.0, **w)
    y64 = mod.decoder_layer(x, Hq=Hq, Hkv=Hkv, D=D, eps=1e-5, theta=10000.0, round_fp16=False,
                            **w)
    assert np.array_equal(y16, y16.astype(np.float16).astype(np.float64))
    assert np.abs(y16 - y64).max() < 2e-2 and np.abs(y16 - y64).max() > 0


ALL_CHECKS = [check_rmsnorm, check_rope_conventions, check_rope_invariants, check_silu, check_f16,
              check_layer_zero_branches, check_layer_single_token, check_layer_brute_force,
              check_layer_rounds_like_fp16]
