"""GPU parity of the scan's gradients (ssd_chunk_scan_bwd) against the float64 oracle
(oracle/backward.py, itself pinned by finite differences of the C forward oracle).

Every gradient of L = sum(dy * y) + sum(dfinal * final_state) -- x, dt, A, B, C, D and the
initial state -- is compared element by element: max |err| <= tol * RMS(oracle gradient).  The
kernels read the stored inputs exactly (bf16 widens exactly) and compute in float32, so the bar
is float32-sized for both io dtypes.
"""
import numpy as np
import pytest
import torch

import mamba_ssd_scan_03_b200 as ssd
import ssd_inputs
from gpu_util import dev_inputs, rel_err, to_np
from oracle import backward

pytestmark = pytest.mark.gpu

TOL = 2e-4
NAMES = ("x", "dt", "A", "B", "C", "D", "init")


def make(seed, io="bf16", init="normal0.1", A_range=None, **shape):
    cfg = dict(batch=1, seqlen=256, nheads=4, headdim=64, dstate=128, ngroups=1, chunk=64,
               io=io, init=init)
    cfg.update(shape)
    inp = ssd_inputs.make_scan_inputs(cfg, seed=seed, A_range=A_range)
    rng = np.random.default_rng(seed + 1)
    Bt, L, H, P, N = cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"], cfg["dstate"]
    dy = rng.standard_normal((Bt, L, H, P)).astype(np.float32)
    dfin = (0.5 * rng.standard_normal((Bt, H, P, N))).astype(np.float32)
    return inp, dy, dfin


def run_bwd(inp, dy, dfin, with_init=True, with_D=True):
    t = dev_inputs(inp)
    g = ssd.chunk_scan_bwd(t["x"], t["dt"], t["A"], t["B"], t["C"],
                           t["D"] if with_D else None, torch.from_numpy(dy).cuda(),
                           init_state=t["init"] if with_init else None,
                           dfinal=None if dfin is None else torch.from_numpy(dfin).cuda())
    torch.cuda.synchronize()
    assert ssd.device_status() == 0
    return {k: to_np(v) for k, v in g.items()}


def check(inp, dy, dfin, got, with_init=True, with_D=True, tol=TOL, skip=()):
    ref = backward.scan_backward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                 inp["D"] if with_D else None,
                                 inp["init"] if with_init else None, dy, dfin)
    errs = {}
    for k in NAMES:
        if k in skip:
            continue
        errs[k] = rel_err(got[k], ref[k])
    bad = {k: v for k, v in errs.items() if v > tol}
    assert not bad, f"max|err|/RMS above {tol}: {bad} (all: {errs})"
    return errs


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [
    dict(batch=2, seqlen=200, nheads=4, headdim=16, dstate=16),            # ragged last chunk
    dict(batch=1, seqlen=300, nheads=4, headdim=64, dstate=128, ngroups=2),
    dict(batch=2, seqlen=130, nheads=6, headdim=32, dstate=64, ngroups=3),
    dict(batch=1, seqlen=64, nheads=2, headdim=64, dstate=128),             # one chunk
    dict(batch=3, seqlen=1, nheads=2, headdim=16, dstate=32),               # one token
    dict(batch=2, seqlen=100, nheads=2, headdim=18, dstate=30),             # widths not /4
])
def test_backward_small(io, shape):
    inp, dy, dfin = make(40 + shape["seqlen"], io=io, **shape)
    got = run_bwd(inp, dy, dfin)
    check(inp, dy, dfin, got)


def test_backward_without_init_D_and_final_gradient():
    inp, dy, _ = make(51, seqlen=333, nheads=4, headdim=32, dstate=64, init="zeros")
    got = run_bwd(inp, dy, None, with_init=False, with_D=False)
    check(inp, dy, None, got, with_init=False, with_D=False)


def test_backward_slow_decay():
    """Per-token decay >= 0.9: the adjoint and the forward state both carry across many chunks,
    so the chunk-to-chunk passes in both directions carry most of every gradient."""
    inp, dy, dfin = make(52, seqlen=700, nheads=4, headdim=32, dstate=64, A_range=(1e-3, 0.5))
    got = run_bwd(inp, dy, dfin)
    check(inp, dy, dfin, got)


def test_backward_tiny_f32_workload():
    inp = ssd_inputs.make_scan_inputs(0)
    rng = np.random.default_rng(5)
    c = inp["cfg"]
    dy = rng.standard_normal((c["batch"], c["seqlen"], c["nheads"], c["headdim"])).astype(
        np.float32)
    got = run_bwd(inp, dy, None, with_init=False)
    check(inp, dy, None, got, with_init=False)


def test_backward_130m_heads_shorter_sequence():
    """The 130M layer's heads (24 x 64, dstate 128, one group: dB and dC sum 24 heads), two
    batch rows of 256 tokens (the dense float64 oracle keeps every state)."""
    inp, dy, dfin = make(53, batch=2, seqlen=256, nheads=24, headdim=64, dstate=128,
                         init="zeros")
    got = run_bwd(inp, dy, dfin, with_init=False)
    check(inp, dy, dfin, got, with_init=False)


def test_backward_deterministic():
    inp, dy, dfin = make(54, batch=2, seqlen=500, nheads=4, headdim=64, dstate=128)
    a = run_bwd(inp, dy, dfin)
    b = run_bwd(inp, dy, dfin)
    for k in NAMES:
        assert np.array_equal(a[k], b[k]), k


def test_backward_argument_errors():
    inp, dy, dfin = make(55, seqlen=128, nheads=2, headdim=16, dstate=16)
    t = dev_inputs(inp)
    with pytest.raises(ValueError):  # dy of the wrong shape is caught by the binding
        ssd.chunk_scan_bwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"],
                           torch.zeros(1, device="cuda"))
    lib = ssd.load()
    # headdim 128 x dstate 256 does not fit one chunk's tiles: unsupported, nothing launched
    assert lib.ssd_chunk_scan_bwd_workspace_size(1, 128, 2, 128, 256, 1, ssd.SSD_BF16) == 0
