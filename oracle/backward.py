"""Float64 gradients of the SSD layer (the reverse-mode adjoint of the recurrence) -- TEST
INFRASTRUCTURE (only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` may use it).

The parallel (block) form exists so that the layer can be trained ("Mamba-2 (2024): SSM e
attention sono la stessa cosa" (paithon.it), "Due modi di guardare la stessa matrice": the
matrix form is the one used for training; "Architektury Mamba-2, State Space Models i liniowa
atencja" (tech.tersel.eu), "Rewolucja Mamba-2 i teoria State Space Duality SSD": 2-8x faster
training than the first generation).  The pages give no gradient formulas; these follow from
the recurrence by the chain rule.  Per batch row b and head h (group g), with a_t = dt_t A_h,
the state h_t = exp(a_t) h_{t-1} + dt_t x_t B_t^T ([P, N]) and y_t = h_t C_t + D_h x_t, and
upstream gradients dy_t ([P]) and dh_final ([P, N]):

    G_t   = dL/dh_t = dy_t C_t^T + exp(a_{t+1}) G_{t+1},   G_{L-1} = dy_{L-1} C_{L-1}^T + dh_final
    dx_t  = dt_t G_t B_t + D_h dy_t
    dB_t += dt_t G_t^T x_t            (summed over the heads of the group)
    dC_t += h_t^T dy_t                (summed over the heads of the group)
    ddt_t = x_t^T G_t B_t + A_h exp(a_t) <G_t, h_{t-1}>
    dA_h  = sum_t dt_t exp(a_t) <G_t, h_{t-1}>
    dD_h  = sum_t <dy_t, x_t>
    dh_init = exp(a_0) G_0

Pinned in ``tests/test_oracle_backward.py`` by central finite differences of the C forward
oracle (an independent implementation) in every input.
"""
import numpy as np


def _f64(a):
    a = np.asarray(a)
    if a.dtype == np.uint16:  # bf16 bit patterns
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def scan_backward(x, dt, A, B, C, D, init, dy, dh_final=None):
    """Gradients of L = sum(dy * y) + sum(dh_final * h_final) for small inputs.

    Shapes as for the forward oracle: x [Bt,L,H,P], dt [Bt,L,H], A [H], B, C [Bt,L,G,N],
    D [H] or None, init [Bt,H,P,N] or None; dy [Bt,L,H,P]; dh_final [Bt,H,P,N] or None.
    Returns a dict of float64 arrays: x, dt, A, B, C, D, init (each the gradient of L with
    respect to that input, same shape).
    """
    x, dt, A, B, C, dy = map(_f64, (x, dt, A, B, C, dy))
    Bt, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    D = np.zeros(H) if D is None else _f64(D)
    h0 = np.zeros((Bt, H, P, N)) if init is None else _f64(init)
    grp = np.arange(H) // (H // G)
    a = dt * A[None, None, :]                          # [Bt, L, H]
    Bh, Ch = B[:, :, grp], C[:, :, grp]                # [Bt, L, H, N]
    # forward, keeping every state (small inputs only)
    hs = np.empty((Bt, L + 1, H, P, N))
    hs[:, 0] = h0
    for t in range(L):
        hs[:, t + 1] = (np.exp(a[:, t])[..., None, None] * hs[:, t]
                        + (dt[:, t, :, None] * x[:, t])[..., None] * Bh[:, t, :, None, :])
    # reverse sweep
    gx, gdt = np.empty_like(x), np.empty_like(dt)
    gBh, gCh = np.zeros_like(Bh), np.zeros_like(Ch)
    gA, gD = np.zeros(H), np.zeros(H)
    Gt = np.zeros((Bt, H, P, N)) if dh_final is None else _f64(dh_final).copy()
    for t in range(L - 1, -1, -1):
        if t < L - 1:
            Gt = np.exp(a[:, t + 1])[..., None, None] * Gt
        Gt = Gt + dy[:, t, :, :, None] * Ch[:, t, :, None, :]
        h_new, h_old = hs[:, t + 1], hs[:, t]
        GB = np.einsum("bhpn,bhn->bhp", Gt, Bh[:, t])
        gx[:, t] = dt[:, t, :, None] * GB + D[None, :, None] * dy[:, t]
        gBh[:, t] = dt[:, t, :, None] * np.einsum("bhpn,bhp->bhn", Gt, x[:, t])
        gCh[:, t] = np.einsum("bhpn,bhp->bhn", h_new, dy[:, t])
        decay_term = np.exp(a[:, t]) * np.einsum("bhpn,bhpn->bh", Gt, h_old)
        gdt[:, t] = np.einsum("bhp,bhp->bh", x[:, t], GB) + A[None, :] * decay_term
        gA += np.sum(dt[:, t] * decay_term, axis=0)
        gD += np.einsum("bhp,bhp->h", dy[:, t], x[:, t])
    ginit = np.exp(a[:, 0])[..., None, None] * Gt
    gB, gC = np.zeros_like(B), np.zeros_like(C)
    for h in range(H):
        gB[:, :, grp[h]] += gBh[:, :, h]
        gC[:, :, grp[h]] += gCh[:, :, h]
    return dict(x=gx, dt=gdt, A=gA, B=gB, C=gC, D=gD, init=ginit)
