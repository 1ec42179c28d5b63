"""Helpers for the GPU parity tests: move seeded inputs to the device, run the float64 oracle
on all or on sampled chains, and compare with the tolerance the workloads fix
(max |err| <= tol * RMS(reference), tol = 1e-4 for float32 io, 2e-2 for bf16 io)."""
import numpy as np
import torch

import oracle

TOL = {"f32": 1e-4, "bf16": 2e-2}


def to_dev(a, bf16=False, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if bf16:
        t = t.view(torch.bfloat16)
    return t.to(device)


def dev_inputs(inp, device="cuda"):
    bf16 = inp["cfg"]["io"] == "bf16"
    out = {k: to_dev(inp[k], bf16 and k in ("x", "B", "C"), device)
           for k in ("x", "dt", "A", "B", "C", "D")}
    out["init"] = None if inp["init"] is None else to_dev(inp["init"], False, device)
    return out


def to_np(t):
    return t.float().cpu().numpy().astype(np.float64)


# A reference whose RMS lies below this is zero in float32 terms (the normal range of float32
# ends at 1.2e-38; a state decayed that far underflows on the GPU while the float64 oracle keeps
# it), so the relative error is taken against this floor instead.
RMS_FLOOR = 1e-30


def rel_err(got, ref):
    """max |got - ref| / RMS(ref), RMS over the compared elements (floored at RMS_FLOOR)."""
    rms = float(np.sqrt(np.mean(np.square(ref))))
    return float(np.max(np.abs(got - ref))) / max(rms, RMS_FLOOR)


def bf16_excess(got, ref, tol):
    """For a bf16 output: max over elements of (|got - ref| - 2^-8 |ref|) / RMS(ref), i.e. the
    error left after the output rounding itself (at most half a bf16 ulp <= 2^-8 |y|)."""
    rms = max(float(np.sqrt(np.mean(np.square(ref)))), RMS_FLOOR)
    return float(np.max(np.abs(got - ref) - 2.0 ** -8 * np.abs(ref))) / rms


def sample_chains(cfg, n, seed=0):
    """n distinct (b, h, p) chains, always including the first and last one."""
    Bt, H, P = cfg["batch"], cfg["nheads"], cfg["headdim"]
    total = Bt * H * P
    rng = np.random.default_rng(seed)
    ids = rng.choice(total, size=min(n, total), replace=False)
    ids = np.unique(np.concatenate([ids, [0, total - 1]])).astype(np.int64)
    p = ids % P
    h = (ids // P) % H
    b = ids // (P * H)
    return ids, b, h, p


def stratified_chains(cfg, per_pair, seed=0):
    """per_pair distinct channels p of every (batch row, head) pair: every head pair, and so every
    CTA range of the walk and every hand-off between ranges, is among the compared chains."""
    Bt, H, P = cfg["batch"], cfg["nheads"], cfg["headdim"]
    rng = np.random.default_rng(seed)
    ids = []
    for bb in range(Bt):
        for hh in range(H):
            for pp in rng.choice(P, size=min(per_pair, P), replace=False):
                ids.append((bb * H + hh) * P + int(pp))
    ids = np.unique(np.asarray(ids, dtype=np.int64))
    return ids, ids // (P * H), (ids // P) % H, ids % P


def oracle_chains(inp, ids, b, h, p):
    init = None if inp["init"] is None else inp["init"][b, h, p]
    return oracle.scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], init=init,
                       chains=ids)
