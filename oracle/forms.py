"""Independent small-case forms of the SSD layer, float64 numpy (test infrastructure).

These do not share code with the sequential recurrence in ``ssd_oracle.c``; they are
other ways the pages say the same function can be written, used to pin that recurrence.

* ``quadratic``   -- the explicit lower-triangular semiseparable matrix, applied like
  masked attention: "Mamba-2 (2024): SSM e attention sono la stessa cosa" (paithon.it),
  sections "Due modi di guardare la stessa matrice" and "Il trucco a blocchi";
  "State Space Model" (book.paithon.it), section "Due strade, una meta" (a scalar
  transition computes the same function as a masked linear attention).
* ``brute_force`` -- the same matrix with every product of decays formed by an explicit
  loop instead of a difference of cumulative sums (tiny inputs only).
* ``lti_convolution`` -- for time-invariant parameters the output is the input convolved
  with the kernel C Abar^k Bbar: "State Space Model", section "Un sistema che riassume il
  passato"; "State Space Models (SSM)" (ultralytics.com glossary), section
  "Come funzionano gli SSM".
"""
import numpy as np


def _f64(a):
    if a is None:
        return None
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def quadratic(x, dt, A, B, C, D=None, init=None):
    """y = M X + exp(cumsum a)_t C_t^T h_{-1} + D x with M the masked semiseparable matrix.

    M[t, s] = (C_t . B_s) * dt_s * exp(sum_{k=s+1..t} a_k) for s <= t, else 0, with
    a_k = dt_k * A_h.  Shapes as in ``oracle.scan``; returns (y [Bt,L,H,P], h_final
    [Bt,H,P,N]).  The final state is the sum of every token's input decayed to the end,
    plus the decayed initial state (the state is the "summary" the block form passes on).
    """
    x, dt, A, B, C = map(_f64, (x, dt, A, B, C))
    D = np.zeros(x.shape[2]) if D is None else _f64(D)
    Bt, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    hpg = H // G
    y = np.zeros((Bt, L, H, P))
    hf = np.zeros((Bt, H, P, N))
    tri = np.tril(np.ones((L, L), dtype=bool))
    for b in range(Bt):
        for h in range(H):
            g = h // hpg
            a = dt[b, :, h] * A[h]                       # [L]
            cs = np.cumsum(a)                            # sum_{k<=t} a_k
            seg = cs[:, None] - cs[None, :]              # sum_{k=s+1..t} a_k
            Lmask = np.where(tri, np.exp(np.where(tri, seg, 0.0)), 0.0)
            CB = C[b, :, g, :] @ B[b, :, g, :].T         # [L(t), L(s)]
            M = Lmask * CB * dt[b, :, h][None, :]
            y[b, :, h, :] = M @ x[b, :, h, :] + D[h] * x[b, :, h, :]
            # final state: sum_s exp(cs_end - cs_s) dt_s x_s B_s^T  (+ decayed init)
            w = np.exp(cs[-1] - cs) * dt[b, :, h] if L else np.zeros(0)
            hf[b, h] = (x[b, :, h, :] * w[:, None]).T @ B[b, :, g, :]
            if init is not None:
                h0 = np.asarray(init, dtype=np.float64)[b, h]    # [P, N]
                y[b, :, h, :] += np.exp(cs)[:, None] * (C[b, :, g, :] @ h0.T)
                hf[b, h] += np.exp(cs[-1] if L else 0.0) * h0
    return y, hf


def brute_force(x, dt, A, B, C, D=None, init=None):
    """The semiseparable matrix with products of per-token decays taken by explicit loops."""
    x, dt, A, B, C = map(_f64, (x, dt, A, B, C))
    D = np.zeros(x.shape[2]) if D is None else _f64(D)
    Bt, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    hpg = H // G
    y = np.zeros((Bt, L, H, P))
    for b in range(Bt):
        for h in range(H):
            g = h // hpg
            dec = np.exp(dt[b, :, h] * A[h])
            for t in range(L):
                acc = D[h] * x[b, t, h, :].copy()
                for s in range(t + 1):
                    prod = 1.0
                    for k in range(s + 1, t + 1):
                        prod *= dec[k]
                    acc += prod * dt[b, s, h] * float(C[b, t, g] @ B[b, s, g]) * x[b, s, h, :]
                if init is not None:
                    prod = 1.0
                    for k in range(0, t + 1):
                        prod *= dec[k]
                    h0 = np.asarray(init, dtype=np.float64)[b, h]
                    acc += prod * (h0 @ C[b, t, g])
                y[b, t, h, :] = acc
    return y


def lti_convolution(x, dt_const, A, B_const, C_const, D=None):
    """Time-invariant case: y_t = sum_{k<=t} K_k x_{t-k} + D x_t, K_k = dt (C.B) exp(dt A)^k.

    x [L, H, P] one batch row; dt_const [H]; A [H]; B_const, C_const [G, N]; zero initial
    state (the convolution form holds from a zero state).
    """
    x = _f64(x)
    L, H, P = x.shape
    G = np.asarray(B_const).shape[0]
    hpg = H // G
    dtc, A, Bc, Cc = _f64(dt_const), _f64(A), _f64(B_const), _f64(C_const)
    D = np.zeros(H) if D is None else _f64(D)
    y = np.zeros((L, H, P))
    k = np.arange(L)
    for h in range(H):
        g = h // hpg
        K = dtc[h] * float(Cc[g] @ Bc[g]) * np.exp(dtc[h] * A[h]) ** k   # [L]
        for p in range(P):
            y[:, h, p] = np.convolve(x[:, h, p], K)[:L] + D[h] * x[:, h, p]
    return y


def diag_ssm_convolution(x, B_bar, C, Abar):
    """A diagonal SSM (one decay per state) on one channel, through its kernel.

    K_k = sum_n C_n Abar_n^k Bbar_n; y = causal convolution of x with K (zero start).
    """
    x = np.asarray(x, dtype=np.float64)
    L = len(x)
    powers = np.asarray(Abar, dtype=np.float64)[:, None] ** np.arange(L)[None, :]  # [N, L]
    K = (np.asarray(C, dtype=np.float64) * np.asarray(B_bar, dtype=np.float64)) @ powers
    return np.convolve(x, K)[:L]
