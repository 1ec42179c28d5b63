"""Float64 definitions of the steps either side of the SSD layer in a Mamba block -- TEST
INFRASTRUCTURE (only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` may use it).

"State Space Models (SSM)" (ultralytics.com glossary), section "Da S4 a Mamba": the
selective SSM sits inside a block that runs its input through a short convolution, derives the
step size from the input, and gates the output with a SiLU branch.  The pages name these steps
but give no formula beyond that; the readings taken here are the plainest ones:

* ``conv_silu``  -- depthwise causal convolution of width K over time, no history before the
  first token (zeros), plus a per-channel bias, followed by SiLU.
* ``dt_softplus`` -- dt = softplus(raw + bias), the usual way a positive step size is made
  from an unconstrained projection.
* ``gate_silu``  -- y * silu(z).

silu(v) = v * sigmoid(v) = v / (1 + e^-v); softplus(v) = log(1 + e^v).  Pinned in
``tests/test_oracle_glue.py`` against closed forms, limits and library routines
(``np.convolve``, ``np.logaddexp``, ``scipy.special.expit``).
"""
import numpy as np


def _f64(a):
    a = np.asarray(a)
    if a.dtype == np.uint16:  # bf16 bit patterns
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def silu(v):
    v = _f64(v)
    with np.errstate(over="ignore"):
        return v / (1.0 + np.exp(-v))


def softplus(v):
    v = _f64(v)
    # log(1 + e^v) = max(v, 0) + log(1 + e^-|v|): no exp overflows
    return np.maximum(v, 0.0) + np.log1p(np.exp(-np.abs(v)))


def conv_silu(u, w, bias=None):
    """u [Bt, L, C] (float32 or bf16 bits), w [C, K], bias [C] or None -> float64 [Bt, L, C].

    out[b, t, c] = silu(bias[c] + sum_{k<K} w[c, k] * u[b, t-K+1+k, c]), u = 0 for t < 0.
    """
    u, w = _f64(u), _f64(w)
    Bt, L, C = u.shape
    K = w.shape[1]
    acc = np.zeros((Bt, L, C)) if bias is None else np.broadcast_to(_f64(bias), (Bt, L, C)).copy()
    for k in range(K):
        shift = K - 1 - k  # tap k reads the token `shift` steps back
        if shift >= L:
            continue
        acc[:, shift:, :] += w[None, None, :, k] * u[:, :L - shift, :]
    return silu(acc)


def dt_softplus(raw, bias=None):
    """raw [Bt, L, H], bias [H] or None -> float64 dt [Bt, L, H]."""
    raw = _f64(raw)
    return softplus(raw if bias is None else raw + _f64(bias))


def gate_silu(y, z):
    """y, z of one shape -> float64 y * silu(z)."""
    return _f64(y) * silu(z)
