"""Pins of the front-end oracle (oracle/front_end.py), CPU only.

Each pin is fixed by something other than the oracle itself: hand-worked
values (tests/golden/front_end_hand.json), closed forms (RoPE with angle 0
is the identity and keeps every pair's length; LayerNorm of a*v + c equals
LayerNorm of v when eps = 0), the relative-position property of RoPE with
angles proportional to the position, and brute-force Python loops for the
head-major projection. Planted mistakes in copies of the oracle's functions
must each fail a pin.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import front_end as fe

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "front_end_hand.json")


def pins_rope(rope):
    g = json.load(open(GOLDEN))
    for case in g["rope"]:
        out = rope(np.array(case["v"]), np.array(case["cos"]), np.array(case["sin"]),
                   case["rope_dim"])
        np.testing.assert_allclose(out, case["out"], rtol=0, atol=1e-12)
    rng = np.random.default_rng(0)
    v = rng.standard_normal((5, 3, 128))
    ones, zeros = np.ones((5, 1, 32)), np.zeros((5, 1, 32))
    np.testing.assert_array_equal(rope(v, ones, zeros, 64), v)
    ang = rng.uniform(-3, 3, (5, 1, 32))
    out = rope(v, np.cos(ang), np.sin(ang), 64)
    pair = lambda a: a[..., 0:64:2] ** 2 + a[..., 1:64:2] ** 2
    np.testing.assert_allclose(pair(out), pair(v), rtol=1e-12)
    np.testing.assert_array_equal(out[..., 64:], v[..., 64:])
    # angles proportional to the position: <rope(q, m), rope(k, n)> depends on m - n
    theta = 10000.0 ** (-np.arange(16) / 16)
    q, k = rng.standard_normal(32), rng.standard_normal(32)

    def at(x, pos):
        return rope(x, np.cos(pos * theta), np.sin(pos * theta), 32)
    for m, n in ((7, 3), (100, 96), (4, 0)):
        np.testing.assert_allclose(at(q, m) @ at(k, n), at(q, m - n) @ k, rtol=1e-10)


def pins_layernorm(layernorm):
    g = json.load(open(GOLDEN))
    for case in g["layernorm"]:
        out = layernorm(np.array(case["v"]), np.array(case["gain"]), np.array(case["bias"]),
                        case["eps"])
        np.testing.assert_allclose(out, case["out"], rtol=0, atol=1e-12)
    rng = np.random.default_rng(1)
    v = rng.standard_normal((4, 128)) * 3 + 1
    gain, bias = np.ones(128), np.zeros(128)
    y = layernorm(v, gain, bias, 0.0)
    np.testing.assert_allclose(y.mean(axis=-1), 0.0, atol=1e-12)
    np.testing.assert_allclose((y ** 2).mean(axis=-1), 1.0, rtol=1e-12)
    np.testing.assert_allclose(layernorm(2.5 * v - 7.0, gain, bias, 0.0), y, atol=1e-12)


def pins_front_end(front_end):
    """The projections against brute-force loops on a tiny problem (head-major
    output features, weights stored [out, in]), and w_scale."""
    rng = np.random.default_rng(2)
    T, H, D, hid, ql = 2, 2, 8, 6, 5
    bits = lambda a: (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    vals = lambda *s: rng.integers(-3, 4, s).astype(np.float32)
    x, qr = vals(T, hid), vals(T, ql)
    wq_b, wk, wp = vals(H * D, ql), vals(D, hid), vals(H, hid)
    gain, bias = np.ones(D), np.zeros(D)
    cos, sin = np.ones((T, 2)), np.zeros((T, 2))
    q, k, w = front_end(bits(x), bits(qr), bits(wq_b), bits(wk), bits(wp), gain, bias, cos, sin,
                        H=H, D=D, rope_dim=4, eps=0.0, w_scale=0.5)
    for t in range(T):
        for h in range(H):
            for d in range(D):
                assert q[t, h, d] == sum(float(qr[t, j]) * float(wq_b[h * D + d, j])
                                         for j in range(ql))
        for h in range(H):
            assert w[t, h] == 0.5 * sum(float(x[t, j]) * float(wp[h, j]) for j in range(hid))
        raw = [sum(float(x[t, j]) * float(wk[d, j]) for j in range(hid)) for d in range(D)]
        mean = sum(raw) / D
        var = sum((r - mean) ** 2 for r in raw) / D
        if var > 0:
            np.testing.assert_allclose(k[t], [(r - mean) / math.sqrt(var) for r in raw],
                                       atol=1e-12)


def test_rope_pins():
    pins_rope(fe.rope)


def test_layernorm_pins():
    pins_layernorm(fe.layernorm)


def test_front_end_pins():
    pins_front_end(fe.front_end)


# ---- planted mistakes: each must fail a pin ----------------------------------

def _rope_half_split(v, cos, sin, rope_dim):          # pairs (i, i + rope_dim/2)
    out = np.array(v, dtype=np.float64, copy=True)
    a, b = v[..., 0:rope_dim // 2], v[..., rope_dim // 2:rope_dim]
    out[..., 0:rope_dim // 2] = a * cos - b * sin
    out[..., rope_dim // 2:rope_dim] = a * sin + b * cos
    return out


def _rope_clockwise(v, cos, sin, rope_dim):           # sign of sin flipped
    return fe.rope(v, cos, -np.asarray(sin), rope_dim)


def _rope_all_features(v, cos, sin, rope_dim):        # rotates past rope_dim
    D = v.shape[-1]
    c = np.concatenate([np.broadcast_to(cos, v.shape[:-1] + (rope_dim // 2,)),
                        np.ones(v.shape[:-1] + ((D - rope_dim) // 2,))], -1)
    s = np.concatenate([np.broadcast_to(sin, v.shape[:-1] + (rope_dim // 2,)),
                        np.broadcast_to(sin[..., :1], v.shape[:-1] + ((D - rope_dim) // 2,))], -1)
    return fe.rope(v, c, s, D)


def _ln_unbiased(v, gain, bias, eps):                 # n - 1 in the variance
    v = np.asarray(v, np.float64)
    mean = v.mean(axis=-1, keepdims=True)
    var = ((v - mean) ** 2).sum(axis=-1, keepdims=True) / (v.shape[-1] - 1)
    return (v - mean) / np.sqrt(var + eps) * gain + bias


def _ln_no_centering(v, gain, bias, eps):             # an RMS norm instead
    v = np.asarray(v, np.float64)
    return v / np.sqrt((v ** 2).mean(axis=-1, keepdims=True) + eps) * gain + bias


def _ln_bias_before_gain(v, gain, bias, eps):
    v = np.asarray(v, np.float64)
    mean = v.mean(axis=-1, keepdims=True)
    var = ((v - mean) ** 2).mean(axis=-1, keepdims=True)
    return ((v - mean) / np.sqrt(var + eps) + bias) * gain


def _fe_feature_major(x, qr, wq_b, wk, wp, gain, bias, cos, sin, *, H, D, rope_dim, eps, w_scale):
    q, k, w = fe.front_end(x, qr, wq_b, wk, wp, gain, bias, cos, sin, H=H, D=D,
                           rope_dim=rope_dim, eps=eps, w_scale=w_scale)
    T = q.shape[0]                                    # features d-major instead of head-major
    return q.reshape(T, H * D).reshape(T, D, H).transpose(0, 2, 1), k, w


def _fe_no_w_scale(x, qr, wq_b, wk, wp, gain, bias, cos, sin, *, H, D, rope_dim, eps, w_scale):
    return fe.front_end(x, qr, wq_b, wk, wp, gain, bias, cos, sin, H=H, D=D, rope_dim=rope_dim,
                        eps=eps, w_scale=1.0)


@pytest.mark.parametrize("pin,mutant", [
    (pins_rope, _rope_half_split), (pins_rope, _rope_clockwise), (pins_rope, _rope_all_features),
    (pins_layernorm, _ln_unbiased), (pins_layernorm, _ln_no_centering),
    (pins_layernorm, _ln_bias_before_gain),
    (pins_front_end, _fe_feature_major), (pins_front_end, _fe_no_w_scale),
])
def test_planted_mistakes_fail_a_pin(pin, mutant):
    with pytest.raises(AssertionError):
        pin(mutant)
