"""Pins for the float64 selective-scan oracle (per-state transition), CPU only.

Tied to things other than itself: (1) with one decay rate shared by all states of a channel
the recurrence is the scalar-transition SSD layer with one-channel heads, whose oracle is the
separate C recurrence ``oracle.scan``; (2) with time-invariant dt, B and C the output is the
input convolved with the kernel sum_n C[n] exp(k dt A[d,n]) dt B[n] (np.convolve); (3) every
product of decays formed by an explicit loop on a tiny input; (4) the sequence split at any
token and resumed from the state gives the same outputs.  The last test plants plausible
mistakes and checks that each fails a pin.
"""
import math

import numpy as np
import pytest

import oracle
import ssd_inputs
from oracle import selective


def _small(io="f32", G=1, init="normal0.1", **kw):
    return ssd_inputs.make_selective_inputs(
        dict(name="t", batch=2, seqlen=kw.get("L", 40), dim=kw.get("dim", 8), dstate=16,
             ngroups=G, io=io, init=init))


def pin_scalar_rate(fn):
    """A[d, :] all equal -> the SSD oracle with H = dim heads of headdim 1."""
    inp = _small(G=2)
    A = np.repeat(inp["A"][:, :1], 16, axis=1)
    y, h = fn(inp["x"], inp["dt"], A, inp["B"], inp["C"], inp["D"], inp["init"])
    x4 = inp["x"][..., None]  # [Bt, L, H=dim, P=1]
    yo, ho = oracle.scan(x4, inp["dt"], A[:, 0].copy(), inp["B"], inp["C"], inp["D"],
                         init=inp["init"][:, :, None, :])
    return (np.allclose(y, yo[..., 0], rtol=1e-12, atol=1e-12)
            and np.allclose(h, ho[:, :, 0, :], rtol=1e-12, atol=1e-12))


def pin_lti(fn):
    """Constant dt, B, C: y = x * K + D x with K_k = sum_n C_n exp(k dt A_n) dt B_n."""
    rng = np.random.default_rng(11)
    L, dim, N = 50, 3, 16
    dtc = 0.2
    A = -np.exp(rng.uniform(0, math.log(16), size=(dim, N)))
    Bc, Cc = rng.standard_normal(N), rng.standard_normal(N)
    x = rng.standard_normal((1, L, dim))
    D = rng.standard_normal(dim)
    dt = np.full((1, L, dim), dtc)
    B = np.broadcast_to(Bc, (1, L, 1, N)).copy()
    C = np.broadcast_to(Cc, (1, L, 1, N)).copy()
    y, _ = fn(x, dt, A, B, C, D, None)
    ok = True
    for d in range(dim):
        K = np.array([np.sum(Cc * np.exp(k * dtc * A[d]) * dtc * Bc) for k in range(L)])
        ref = np.convolve(x[0, :, d], K)[:L] + D[d] * x[0, :, d]
        ok &= np.allclose(y[0, :, d], ref, rtol=1e-11, atol=1e-11)
    return ok


def pin_brute(fn):
    """y_t = sum_{s<=t} sum_n C_t[n] (prod_{k=s+1..t} e^{dt_k A[n]}) dt_s B_s[n] x_s
    + (prod_{k=0..t} e^{dt_k A[n]}) C_t[n] h0[n] + D x_t, products by explicit loops."""
    inp = _small(L=7, dim=4, G=2)
    x, dt, A, B, C, D, h0 = (selective._f64(inp[k]) for k in ("x", "dt", "A", "B", "C", "D",
                                                               "init"))
    y, _ = fn(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["init"])
    ok = True
    for b, d, t in [(0, 0, 0), (1, 3, 6), (0, 2, 4), (1, 1, 5)]:
        g = d // 2
        acc = D[d] * x[b, t, d]
        for n in range(16):
            p = 1.0
            for k in range(t, -1, -1):
                acc += C[b, t, g, n] * p * dt[b, k, d] * B[b, k, g, n] * x[b, k, d]
                p *= math.exp(dt[b, k, d] * A[d, n])
            acc += C[b, t, g, n] * p * h0[b, d, n]
        ok &= abs(y[b, t, d] - acc) < 1e-12 * (1 + abs(acc))
    return ok


def pin_split(fn):
    inp = _small(L=40, G=2)
    y, h = fn(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["init"])
    s = 17
    cut = lambda a, lo, hi: a[:, lo:hi]
    y1, h1 = fn(cut(inp["x"], 0, s), cut(inp["dt"], 0, s), inp["A"], cut(inp["B"], 0, s),
                cut(inp["C"], 0, s), inp["D"], inp["init"])
    y2, h2 = fn(cut(inp["x"], s, 40), cut(inp["dt"], s, 40), inp["A"], cut(inp["B"], s, 40),
                cut(inp["C"], s, 40), inp["D"], h1)
    return (np.allclose(np.concatenate([y1, y2], axis=1), y, rtol=1e-13, atol=1e-13)
            and np.allclose(h2, h, rtol=1e-13, atol=1e-13))


PINS = [pin_scalar_rate, pin_lti, pin_brute, pin_split]


def _oracle(x, dt, A, B, C, D, init):
    return selective.selective_scan(x, dt, A, B, C, D, init)


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_selective_pins(pin):
    assert pin(_oracle)


def test_selective_chain_subset_matches_whole():
    inp = _small(L=30, dim=8, G=2)
    y, h = _oracle(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["init"])
    rows, chans = np.array([1, 0, 1]), np.array([7, 0, 3])
    ys, hs = selective.selective_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                      inp["D"], inp["init"][rows, chans], rows=rows, chans=chans)
    np.testing.assert_array_equal(ys, y[rows, :, chans])
    np.testing.assert_array_equal(hs, h[rows, chans])


def test_selective_inputs_bf16_widen():
    inp = ssd_inputs.make_selective_inputs(0)
    assert inp["x"].dtype == np.uint16 and inp["A"].shape == (64, 16)
    assert np.all(inp["A"] <= -1.0) and np.all(inp["A"] >= -16.0)


# -- planted mistakes --------------------------------------------------------------------

def _variant(mistake):
    """The recurrence restated with one plausible mistake."""
    def fn(x, dt, A, B, C, D, init):
        x, dt, A, B, C, D = map(selective._f64, (x, dt, A, B, C, D))
        Bt, L, dim = x.shape
        G, N = B.shape[2], B.shape[3]
        g = np.arange(dim) % G if mistake == "group_map" else np.arange(dim) // (dim // G)
        if mistake == "transposed_A":
            A = A.T.reshape(dim, N)
        if mistake == "shared_decay":
            A = np.repeat(A[:, :1], N, axis=1)
        h = np.zeros((Bt, dim, N)) if init is None else selective._f64(init).copy()
        y = np.empty((Bt, L, dim))
        for t in range(L):
            dtt = dt[:, t, :, None]
            inp = (1.0 if mistake == "no_dt_input" else dtt) * B[:, t][:, g] * x[:, t, :, None]
            new = np.exp(dtt * A) * h + inp
            read = h if mistake == "pre_update" else new
            y[:, t] = np.sum(C[:, t][:, g] * read, axis=2) + D * x[:, t]
            h = new
        return y, h
    return fn


MUTANTS = ["transposed_A", "pre_update", "group_map", "no_dt_input", "shared_decay"]


def test_selective_variant_without_mistake_passes():
    assert all(pin(_variant(None)) for pin in PINS)


@pytest.mark.parametrize("mistake", MUTANTS)
def test_selective_pins_catch_mistakes(mistake):
    with np.errstate(all="ignore"):
        assert not all(pin(_variant(mistake)) for pin in PINS)


def test_selective_input_recipe():
    """The recipe the docstring of make_selective_inputs states: x ~ N(0,1), dt = softplus of
    N(-2, 0.5) (mean 0.1403), A in [-16, -1] independent per (channel, state), B and C with
    standard deviation 1/sqrt(16), init N(0, 0.1); deterministic for a seed."""
    inp = ssd_inputs.make_selective_inputs(dict(name="t", batch=2, seqlen=2048, dim=64,
                                                dstate=16, ngroups=1, io="f32",
                                                init="normal0.1"))
    assert abs(inp["x"].mean()) < 0.01 and abs(inp["x"].std() - 1) < 0.01
    assert abs(inp["dt"].mean() - 0.1403) < 0.003 and np.all(inp["dt"] > 0)
    assert np.all(inp["A"] <= -1) and np.all(inp["A"] >= -16)
    assert len(np.unique(inp["A"])) == inp["A"].size  # a rate per (channel, state)
    assert abs(inp["B"].std() - 0.25) < 0.01 and abs(inp["C"].std() - 0.25) < 0.01
    assert abs(inp["init"].std() - 0.1) < 0.005
    again = ssd_inputs.make_selective_inputs(dict(name="t", batch=2, seqlen=2048, dim=64,
                                                  dstate=16, ngroups=1, io="f32",
                                                  init="normal0.1"))
    for k in ("x", "dt", "A", "B", "C", "D", "init"):
        np.testing.assert_array_equal(inp[k], again[k])
