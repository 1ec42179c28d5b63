"""Pins for the float64 gradients of the SSD layer (CPU only).

Every gradient is checked against central finite differences of the separate C forward oracle
(oracle.scan): for a random direction v in one input, (L(u + e v) - L(u - e v)) / 2e must equal
<grad, v>, with L = sum(dy * y) + sum(dh_final * h_final).  Shapes cover several heads per
group and groups > 1.  The last test plants plausible mistakes in the adjoint and checks that
each fails a pin.
"""
import numpy as np
import pytest

import oracle
from oracle import backward

NAMES = ["x", "dt", "A", "B", "C", "D", "init"]


def _inputs(seed=0, Bt=2, L=9, H=4, P=3, G=2, N=5):
    rng = np.random.default_rng(seed)
    return dict(x=rng.standard_normal((Bt, L, H, P)),
                dt=np.log1p(np.exp(rng.normal(-1.0, 0.5, (Bt, L, H)))),
                A=-np.exp(rng.uniform(0, np.log(4.0), H)),
                B=rng.standard_normal((Bt, L, G, N)) / np.sqrt(N),
                C=rng.standard_normal((Bt, L, G, N)) / np.sqrt(N),
                D=rng.standard_normal(H),
                init=0.3 * rng.standard_normal((Bt, H, P, N))), \
        rng.standard_normal((Bt, L, H, P)), rng.standard_normal((Bt, H, P, N))


def _loss(inp, dy, dh):
    # the C oracle reads float32 or bf16 storage; float64 values pass through float32 exactly
    # only if they are float32 values, so the probe inputs are rounded to float32 first.
    y, h = oracle.scan(*(inp[k].astype(np.float32) for k in ("x", "dt", "A", "B", "C", "D")),
                       init=inp["init"].astype(np.float32))
    return float(np.sum(dy * y) + np.sum(dh * h))


def _round32(inp):
    return {k: v.astype(np.float32).astype(np.float64) for k, v in inp.items()}


def fd_pins(grad_fn, seed=0, **shape):
    """Yield (input name, relative mismatch) for a random direction per input."""
    inp, dy, dh = _inputs(seed, **shape)
    inp = _round32(inp)
    g = grad_fn(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["init"], dy, dh)
    rng = np.random.default_rng(seed + 100)
    for name in NAMES:
        v = rng.standard_normal(inp[name].shape)
        # a step of ~1e-4 relative: float32 storage keeps 4 digits of it; the realised step
        # is what the prediction uses
        eps = 1e-4 * max(1e-3, float(np.max(np.abs(inp[name]))))
        up, dn = dict(inp), dict(inp)
        up[name] = inp[name] + eps * v
        dn[name] = inp[name] - eps * v
        # the float32 rounding of the probes changes the actual step: use the realised steps
        vu = up[name].astype(np.float32).astype(np.float64) - inp[name]
        vd = inp[name] - dn[name].astype(np.float32).astype(np.float64)
        fd = _loss(up, dy, dh) - _loss(dn, dy, dh)
        pred = float(np.sum(g[name] * (vu + vd)))
        yield name, abs(fd - pred) / max(1e-12, abs(fd) + abs(pred))


def _grad(x, dt, A, B, C, D, init, dy, dh):
    return backward.scan_backward(x, dt, A, B, C, D, init, dy, dh)


@pytest.mark.parametrize("shape", [dict(), dict(G=1), dict(H=2, G=2, L=5), dict(L=1)])
def test_backward_matches_finite_differences(shape):
    bad = [(n, r) for n, r in fd_pins(_grad, **shape) if r > 1e-5]
    assert not bad, bad


def test_backward_defaults_are_zeros():
    """D = None, init = None and dh_final = None mean zeros."""
    inp, dy, _ = _inputs(3)
    H, shp = inp["x"].shape[2], inp["init"].shape
    g = backward.scan_backward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], None, None, dy)
    g0 = backward.scan_backward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], np.zeros(H),
                                np.zeros(shp), dy, np.zeros(shp))
    for k in NAMES:
        np.testing.assert_array_equal(g[k], g0[k])


# -- planted mistakes: each must fail at least one finite-difference pin -------------------

def _mutant(kind):
    def fn(x, dt, A, B, C, D, init, dy, dh):
        g = backward.scan_backward(x, dt, A, B, C, D, init, dy, dh)
        if kind == "no_decay_term":       # ddt without the A exp(a) <G, h_{t-1}> part
            g0 = backward.scan_backward(x, dt, np.zeros_like(A), B, C, D, init, dy, dh)
            g["dt"] = g0["dt"]
        elif kind == "dA_sign":
            g["A"] = -g["A"]
        elif kind == "dB_one_head":       # group sum replaced by the first head's share
            g["B"] = g["B"] / (x.shape[2] // B.shape[2])
        elif kind == "dinit_undecayed":
            g["init"] = g["init"] / np.exp(dt[:, 0] * A[None, :])[..., None, None]
        elif kind == "dx_no_skip":
            g["x"] = g["x"] - D[None, None, :, None] * dy
        return g
    return fn


@pytest.mark.parametrize("kind", ["no_decay_term", "dA_sign", "dB_one_head", "dinit_undecayed",
                                  "dx_no_skip"])
def test_backward_pins_catch_mistakes(kind):
    assert any(r > 1e-5 for _, r in fd_pins(_mutant(kind)))
