"""Float64 oracle of the selective scan with a per-state (diagonal) transition -- TEST
INFRASTRUCTURE (only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` may use it).

The first Mamba generation: "Architektury Mamba-2, State Space Models i liniowa atencja"
(tech.tersel.eu), section "Od S4 do Mamba-1: Wprowadzenie mechanizmu selektywnego" -- B, C and
the step dt become functions of the current input, and the recurrence is scanned on the GPU's
CUDA cores with the state kept on chip; "State Space Model" (book.paithon.it), overview of the
Mamba chapter (two linear steps merge into one step of the same kind; the state stays in the
GPU's fast memory).  The same pages contrast it with the scalar-transition (SSD) layer: there
the whole state fades at one rate, here every state n of every channel d fades at its own rate
exp(dt A[d, n]) (a diagonal A, "State Space Models (SSM)" (ultralytics.com), section "Come
funzionano gli SSM").

Per batch row b and channel d, with g = d // (dim // ngroups) the channel's group:

    h_t[n] = exp(dt_t[d] A[d, n]) h_{t-1}[n] + dt_t[d] B_t[g, n] x_t[d]
    y_t[d] = sum_n C_t[g, n] h_t[n] + D[d] x_t[d]

h_{-1} = init (zeros by default); the output reads the updated state, as in the SSD layer.
Pinned in ``tests/test_oracle_selective.py``.
"""
import numpy as np


def _f64(a):
    a = np.asarray(a)
    if a.dtype == np.uint16:  # bf16 bit patterns
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def selective_scan(x, dt, A, B, C, D=None, init=None, rows=None, chans=None):
    """Sequential float64 recurrence.

    x, dt [Bt, L, dim]; A [dim, N]; B, C [Bt, L, G, N]; D [dim] or None; init [Bt, dim, N] or
    None.  ``rows``/``chans`` (equal-length int arrays) restrict the scan to the chains
    (rows[i], chans[i]); then y is [n, L] and the final state [n, N] (init, if given, is then
    [n, N]).  Otherwise y is [Bt, L, dim] and the final state [Bt, dim, N].
    """
    x, dt, A, B, C = map(_f64, (x, dt, A, B, C))
    Bt, L, dim = x.shape
    G, N = B.shape[2], B.shape[3]
    D = np.zeros(dim) if D is None else _f64(D)
    if rows is None:
        rows = np.repeat(np.arange(Bt), dim)
        chans = np.tile(np.arange(dim), Bt)
        whole = True
        h = np.zeros((Bt * dim, N)) if init is None else _f64(init).reshape(Bt * dim, N).copy()
    else:
        rows, chans = np.asarray(rows), np.asarray(chans)
        whole = False
        h = np.zeros((len(rows), N)) if init is None else _f64(init).copy()
    grp = chans // (dim // G)
    Ad = A[chans]  # [n, N]
    y = np.empty((len(rows), L))
    for t in range(L):
        dtt = dt[rows, t, chans][:, None]
        xt = x[rows, t, chans]
        h = np.exp(dtt * Ad) * h + dtt * B[rows, t, grp] * xt[:, None]
        y[:, t] = np.sum(C[rows, t, grp] * h, axis=1) + D[chans] * xt
    if whole:
        return y.reshape(Bt, dim, L).transpose(0, 2, 1), h.reshape(Bt, dim, N)
    return y, h
