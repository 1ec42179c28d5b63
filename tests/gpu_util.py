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


def rel_err(got, ref):
    """max |got - ref| / RMS(ref), RMS over the compared elements."""
    rms = float(np.sqrt(np.mean(np.square(ref))))
    return float(np.max(np.abs(got - ref))) / max(rms, 1e-300)


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


def oracle_chains(inp, ids, b, h, p):
    init = None if inp["init"] is None else inp["init"][b, h, p]
    return oracle.scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], init=init,
                       chains=ids)
