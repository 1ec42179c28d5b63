"""Float64 CPU oracle for the Mamba-2 SSD layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline and
reference arms) may import this package.  The product path (the CUDA library and its
binding in ``mamba_ssd_scan_03_b200``) never imports, loads or calls it, and the two share
no code; the only module both sides use is ``ssd_inputs`` (seeded input generation,
which holds none of the method's arithmetic).

Contents
--------
``scan``        the sequential float64 recurrence (C, OpenMP), one chain per (b, h, p):
                the plain definition of what the layer computes.
``step``        the same recurrence advanced by one token on a float64 state
                (the generation / decode form).
``forms``       independent small-case forms used to pin ``scan``: the explicit masked
                semiseparable (attention-like) matrix, brute-force products of decays,
                the LTI convolution kernel, and closed forms of special cases.
``glue``        float64 definitions of the block steps around the layer (short causal
                convolution + SiLU, dt softplus, SiLU output gate).
``selective``   the selective scan with a per-state transition (the first Mamba generation).
``backward``    the layer's gradients (reverse-mode adjoint of the recurrence).

Every function is pinned: ``tests/test_oracle.py``, ``tests/test_oracle_glue.py``,
``tests/test_oracle_selective.py``, ``tests/test_oracle_backward.py``; no function is "parity
unpinned".
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIBS = {}

F32 = 0
BF16 = 1


def _lib(mutation: int = 0):
    lib = _LIBS.get(mutation)
    if lib is None:
        path = _build.build(mutation)
        lib = ctypes.CDLL(path)
        fn = lib.ssd_oracle_scan_f64
        fn.restype = ctypes.c_int
        fn.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_void_p] + [ctypes.c_int64] * 6 + [
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_int]
        lib.ssd_oracle_mutation.restype = ctypes.c_int
        assert lib.ssd_oracle_mutation() == mutation
        _LIBS[mutation] = lib
    return lib


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _io_dtype(arr: np.ndarray) -> int:
    if arr.dtype == np.float32:
        return F32
    if arr.dtype == np.uint16:  # bf16 bit patterns
        return BF16
    raise TypeError(f"x/B/C must be float32 or uint16 (bf16 bits), got {arr.dtype}")


def _ptr(a):
    return None if a is None else a.ctypes.data


def scan(x, dt, A, B, C, D=None, init=None, chains=None, nthreads=None, mutation=0,
         want_state=True):
    """Sequential float64 recurrence.

    x [Bt,L,H,P] and B, C [Bt,L,G,N] are float32 arrays or uint16 arrays holding bf16 bits;
    dt [Bt,L,H], A [H], D [H] float32.  ``init`` is the state before token 0, float64 or
    float32, shaped [Bt,H,P,N] (all chains) or [n_chains,N] (with ``chains``).
    ``chains`` is an int64 array of flat ids (b*H + h)*P + p; None means every chain.

    Returns (y, h_final).  Without ``chains``: y [Bt,L,H,P] float64 and h_final
    [Bt,H,P,N] float64.  With ``chains``: y [n_chains,L], h_final [n_chains,N].
    """
    x = np.ascontiguousarray(x)
    B = np.ascontiguousarray(B)
    C = np.ascontiguousarray(C)
    dt = np.ascontiguousarray(dt, dtype=np.float32)
    A = np.ascontiguousarray(A, dtype=np.float32)
    D = None if D is None else np.ascontiguousarray(D, dtype=np.float32)
    io = _io_dtype(x)
    if _io_dtype(B) != io or _io_dtype(C) != io:
        raise TypeError("x, B and C must share one storage dtype")
    Bt, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if B.shape != (Bt, L, G, N) or C.shape != B.shape or dt.shape != (Bt, L, H):
        raise ValueError("inconsistent shapes")
    if chains is None:
        n = Bt * H * P
        ids = None
    else:
        ids = np.ascontiguousarray(chains, dtype=np.int64)
        n = ids.shape[0]
    h0 = None
    if init is not None:
        h0 = np.ascontiguousarray(np.asarray(init, dtype=np.float64).reshape(n, N))
    y = np.empty((n, L), dtype=np.float64)
    h1 = np.empty((n, N), dtype=np.float64) if want_state else None
    rc = _lib(mutation).ssd_oracle_scan_f64(
        _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), io, _ptr(h0), _ptr(y),
        _ptr(h1), Bt, L, H, P, N, G, _ptr(ids), n, nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    if chains is None:
        y = y.reshape(Bt, H, P, L).transpose(0, 3, 1, 2).copy()
        if h1 is not None:
            h1 = h1.reshape(Bt, H, P, N)
    return y, h1


def step(state, x, dt, A, B, C, D=None, chains=None, nthreads=None, mutation=0):
    """One token of the recurrence on a float64 state (the decode form).

    state: [Bt,H,P,N] (all chains) or [n_chains,N] float64; x [Bt,H,P]; dt [Bt,H];
    B, C [Bt,G,N].  Returns (y, new_state) with y [Bt,H,P] or [n_chains].
    """
    Bt, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    y, h1 = scan(x.reshape(Bt, 1, H, P), dt.reshape(Bt, 1, H), A, B.reshape(Bt, 1, G, N),
                 C.reshape(Bt, 1, G, N), D, init=state, chains=chains, nthreads=nthreads,
                 mutation=mutation)
    if chains is None:
        return y.reshape(Bt, H, P), h1
    return y.reshape(-1), h1


def chain_ids(b, h, p, nheads, headdim):
    """Flat chain id(s) for (batch, head, channel)."""
    return (np.asarray(b, dtype=np.int64) * nheads + np.asarray(h, dtype=np.int64)) * headdim \
        + np.asarray(p, dtype=np.int64)


def widen(a: np.ndarray) -> np.ndarray:
    """Exact float64 view of float32 data or of uint16 bf16 bit patterns."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


from . import forms  # noqa: E402  (re-export)
