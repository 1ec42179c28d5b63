"""Pins for the float64 definitions of the block steps around the layer (CPU only).

Each definition is tied to something other than itself: closed values (silu(0) = 0,
softplus(0) = ln 2), the odd-part identities silu(v) - silu(-v) = v and
softplus(v) - softplus(-v) = v, the large-|v| limits, library routines (np.convolve,
np.logaddexp, scipy.special.expit) and explicit per-element loops on tiny inputs.  The last
test swaps in plausible mistakes and checks that each fails at least one pin.
"""
import math

import numpy as np
import pytest
from scipy.special import expit

from oracle import glue


def _rng(seed):
    return np.random.default_rng(seed)


def pins_silu(silu):
    v = np.linspace(-30, 30, 601)
    yield "silu(0)", silu(np.array([0.0]))[0] == 0.0
    yield "odd part", np.allclose(silu(v) - silu(-v), v, rtol=0, atol=1e-12)
    yield "expit", np.allclose(silu(v), v * expit(v), rtol=1e-14, atol=1e-300)
    big = np.array([50.0, 700.0, -50.0, -700.0])
    yield "limits", np.allclose(silu(big), [50.0, 700.0, 0.0, 0.0], rtol=1e-15, atol=1e-18)


def pins_softplus(softplus):
    v = np.linspace(-40, 40, 801)
    yield "softplus(0)", abs(softplus(np.array([0.0]))[0] - math.log(2.0)) < 1e-16
    yield "odd part", np.allclose(softplus(v) - softplus(-v), v, rtol=0, atol=1e-12)
    yield "logaddexp", np.allclose(softplus(v), np.logaddexp(0.0, v), rtol=1e-14, atol=0)
    yield "limits", np.allclose(softplus(np.array([800.0, -800.0, -30.0])),
                                [800.0, 0.0, math.exp(-30.0)], rtol=1e-12, atol=0)


def pins_conv(conv):
    rng = _rng(7)
    for K in (1, 3, 4, 8):
        u = rng.standard_normal((2, 11, 5))
        w = rng.standard_normal((5, K))
        b = rng.standard_normal(5)
        got = conv(u, w, b)
        # library: the convolution sum[t] = sum_j u[j] w[K-1-(t-j)] is np.convolve with w reversed
        ref = np.empty_like(u)
        for bi in range(2):
            for c in range(5):
                ref[bi, :, c] = np.convolve(u[bi, :, c], w[c, ::-1])[:11] + b[c]
        yield f"np.convolve K={K}", np.allclose(got, ref * expit(ref), rtol=1e-13, atol=1e-14)
        # brute force, one element at a time
        t, c = 6, 3
        acc = b[c] + sum(w[c, k] * u[1, t - K + 1 + k, c] for k in range(K) if t - K + 1 + k >= 0)
        yield f"element K={K}", abs(got[1, t, c] - acc / (1 + math.exp(-acc))) < 1e-13
    # a unit weight on the oldest tap delays the sequence by K-1 tokens, zeros first
    u = rng.standard_normal((1, 9, 2))
    w = np.zeros((2, 4)); w[:, 0] = 1.0
    want = np.zeros_like(u); want[:, 3:, :] = u[:, :6, :]
    yield "delay", np.allclose(conv(u, w, None), want * expit(want), rtol=1e-14, atol=0)
    # a unit weight on the newest tap is SiLU alone; zero weights give silu(bias) everywhere
    w = np.zeros((2, 4)); w[:, 3] = 1.0
    yield "identity tap", np.allclose(conv(u, w, None), u * expit(u), rtol=1e-14, atol=0)
    yield "bias only", np.allclose(conv(u, np.zeros((2, 4)), np.array([0.5, -2.0])),
                                   np.broadcast_to(np.array([0.5, -2.0]) * expit([0.5, -2.0]),
                                                   u.shape), rtol=1e-14, atol=0)
    # a window longer than the sequence
    u = rng.standard_normal((1, 3, 1)); w = rng.standard_normal((1, 8))
    acc = np.array([sum(w[0, 7 - s] * u[0, t - s, 0] for s in range(t + 1)) for t in range(3)])
    yield "K > L", np.allclose(conv(u, w, None)[0, :, 0], acc * expit(acc), rtol=1e-13, atol=0)


def pins_gate(gate):
    rng = _rng(3)
    y, z = rng.standard_normal((4, 6)), rng.standard_normal((4, 6))
    yield "z = 0", np.all(gate(y, np.zeros_like(z)) == 0.0)
    yield "large z", np.allclose(gate(y, np.full_like(z, 60.0)), 60.0 * y, rtol=1e-15, atol=0)
    yield "expit", np.allclose(gate(y, z), y * z * expit(z), rtol=1e-14, atol=0)


def pins_dt(dt_softplus):
    rng = _rng(5)
    raw, bias = rng.standard_normal((2, 7, 3)) * 4, rng.standard_normal(3)
    got = dt_softplus(raw, bias)
    ok = all(abs(got[b, t, h] - math.log1p(math.exp(raw[b, t, h] + bias[h]))) < 1e-14
             for b in range(2) for t in range(7) for h in range(3))
    yield "per-element", ok
    yield "no bias", np.allclose(dt_softplus(raw), np.logaddexp(0.0, raw), rtol=1e-14, atol=0)


@pytest.mark.parametrize("name,pins,fn", [
    ("silu", pins_silu, glue.silu), ("softplus", pins_softplus, glue.softplus),
    ("conv_silu", pins_conv, glue.conv_silu), ("gate_silu", pins_gate, glue.gate_silu),
    ("dt_softplus", pins_dt, glue.dt_softplus)])
def test_glue_pins(name, pins, fn):
    failed = [what for what, ok in pins(fn) if not ok]
    assert not failed, f"{name}: {failed}"


def test_glue_bf16_inputs_widened():
    bits = np.array([0x3F80, 0xC000, 0x0000], dtype=np.uint16)  # 1.0, -2.0, 0.0
    np.testing.assert_array_equal(glue._f64(bits), [1.0, -2.0, 0.0])


# -- planted mistakes: each must fail at least one pin -------------------------------------

def _conv_off_by_one(u, w, bias=None):  # window one token too far back
    u = glue._f64(u); Bt, L, C = u.shape; K = w.shape[1]
    acc = np.zeros_like(u) if bias is None else np.broadcast_to(bias, u.shape).copy()
    for k in range(K):
        s = K - k
        if s < L:
            acc[:, s:, :] += w[None, None, :, k] * u[:, :L - s, :]
    return glue.silu(acc)


def _conv_taps_reversed(u, w, bias=None):
    return glue.conv_silu(u, np.asarray(w)[:, ::-1], bias)


def _conv_no_bias(u, w, bias=None):
    return glue.conv_silu(u, w, None)


def _conv_no_silu(u, w, bias=None):  # the pre-activation, SiLU left out
    u, w = glue._f64(u), np.asarray(w, float)
    Bt, L, C = u.shape; K = w.shape[1]
    acc = np.zeros_like(u) if bias is None else np.broadcast_to(bias, u.shape).copy()
    for k in range(K):
        s = K - 1 - k
        if s < L:
            acc[:, s:, :] += w[None, None, :, k] * u[:, :L - s, :]
    return acc


MUTANTS = [
    (pins_silu, lambda v: np.asarray(v, float) / (1 + np.exp(np.asarray(v, float)))),  # sign
    (pins_silu, lambda v: expit(np.asarray(v, float))),  # sigmoid, not silu
    (pins_softplus, lambda v: np.log(np.exp(np.asarray(v, float)))),  # dropped the 1
    (pins_softplus, lambda v: np.log1p(np.exp(-np.asarray(v, float)))),  # sign
    (pins_conv, _conv_off_by_one),
    (pins_conv, _conv_taps_reversed),
    (pins_conv, _conv_no_bias),
    (pins_conv, _conv_no_silu),
    (pins_gate, lambda y, z: np.asarray(y) * expit(np.asarray(z))),  # sigmoid gate
    (pins_gate, lambda y, z: np.asarray(z) * glue.silu(y)),  # operands swapped
    (pins_dt, lambda raw, bias=None: glue.softplus(raw)),  # bias dropped
    (pins_dt, lambda raw, bias=None: glue.softplus(raw) + (0 if bias is None else bias)),
]


@pytest.mark.parametrize("i", range(len(MUTANTS)))
def test_glue_pins_catch_mistakes(i):
    pins, fn = MUTANTS[i]
    with np.errstate(all="ignore"):
        results = [ok for _, ok in pins(fn)]
    assert not all(results)


def test_glue_input_recipe():
    from ssd_inputs import make_glue_inputs
    g = make_glue_inputs(2, 512, 64, 4, 8, 32, "f32")
    assert abs(g["u"].std() - 1) < 0.02 and abs(g["z"].std() - 1) < 0.02
    assert abs(g["w"].std() - 0.5) < 0.05  # N(0, 1) / sqrt(4)
    assert np.all(g["dt_bias"] >= -6) and np.all(g["dt_bias"] <= -2)
    h = make_glue_inputs(2, 512, 64, 4, 8, 32, "f32")
    for k in ("u", "w", "conv_bias", "raw", "dt_bias", "y", "z"):
        np.testing.assert_array_equal(g[k], h[k])
