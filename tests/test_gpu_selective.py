"""GPU parity of the selective scan with a per-state transition (ssd_selective_scan_fwd)
against the float64 oracle recurrence (oracle.selective).  Bar as for the SSD layer:
max |err| <= tol * RMS(reference), tol = 1e-4 for float32 io and 2e-2 for bf16 io, for y and
for the final state; bf16 y is checked after removing its own rounding (bf16_excess)."""
import numpy as np
import pytest
import torch

import mamba_ssd_scan_03_b200 as ssd
import ssd_inputs
from gpu_util import TOL, bf16_excess, rel_err, to_dev, to_np
from oracle import selective

pytestmark = pytest.mark.gpu


def _dev(inp):
    bf16 = inp["cfg"]["io"] == "bf16"
    t = {k: to_dev(inp[k], bf16 and k in ("x", "B", "C")) for k in ("x", "dt", "A", "B", "C",
                                                                    "D")}
    t["init"] = None if inp["init"] is None else to_dev(inp["init"])
    return t


def _run(inp, y_dtype=torch.float32, with_D=True):
    t = _dev(inp)
    y, fin = ssd.selective_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"],
                                    t["D"] if with_D else None, t["init"], y_dtype=y_dtype)
    return to_np(y), to_np(fin)


@pytest.mark.parametrize("io,batch,seqlen,dim,G,init", [
    ("bf16", 2, 300, 64, 1, "normal0.1"),   # several chunks and a ragged tail
    ("f32", 2, 300, 64, 2, "normal0.1"),
    ("f32", 1, 37, 16, 2, "zeros"),
    ("bf16", 3, 1, 8, 1, "normal0.1"),     # one token
    ("bf16", 1, 64, 24, 3, "zeros"),       # exact chunks, three groups of 8 channels
    ("f32", 2, 33, 40, 5, "normal0.1"),
])
def test_selective_small_every_element(io, batch, seqlen, dim, G, init):
    inp = ssd_inputs.make_selective_inputs(dict(name="t", batch=batch, seqlen=seqlen, dim=dim,
                                                dstate=16, ngroups=G, io=io, init=init))
    y, fin = _run(inp)
    yo, ho = selective.selective_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                      inp["D"], inp["init"])
    assert rel_err(y, yo) <= TOL[io]
    assert rel_err(fin, ho) <= TOL[io]
    assert ssd.device_status() == 0


def test_selective_no_skip_and_bf16_y():
    inp = ssd_inputs.make_selective_inputs(0)
    y, _ = _run(inp, with_D=False)
    yo, _ = selective.selective_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], None,
                                     inp["init"])
    assert rel_err(y, yo) <= TOL["bf16"]
    yb, _ = _run(inp, y_dtype=torch.bfloat16)
    yo, _ = selective.selective_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                     inp["D"], inp["init"])
    assert bf16_excess(yb, yo, TOL["bf16"]) <= TOL["bf16"]


def test_selective_state_resume():
    """Two calls over the halves of a sequence (the second from the first's final state) give
    the whole sequence's y and state."""
    inp = ssd_inputs.make_selective_inputs(dict(name="t", batch=2, seqlen=200, dim=32, dstate=16,
                                                ngroups=1, io="f32", init="normal0.1"))
    t = _dev(inp)
    y, fin = ssd.selective_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], t["init"])
    s = 77
    cut = lambda a, lo, hi: a[:, lo:hi].contiguous()
    y1, f1 = ssd.selective_scan_fwd(cut(t["x"], 0, s), cut(t["dt"], 0, s), t["A"],
                                    cut(t["B"], 0, s), cut(t["C"], 0, s), t["D"], t["init"])
    y2, f2 = ssd.selective_scan_fwd(cut(t["x"], s, 200), cut(t["dt"], s, 200), t["A"],
                                    cut(t["B"], s, 200), cut(t["C"], s, 200), t["D"], f1)
    yo, ho = selective.selective_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                      inp["D"], inp["init"])
    assert rel_err(to_np(torch.cat([y1, y2], 1)), yo) <= 1e-4
    assert rel_err(to_np(f2), ho) <= 1e-4
    assert rel_err(to_np(y), yo) <= 1e-4


def test_selective_full_size_sampled():
    """The 5120-channel, 16-state workload at its full size (batch 4, seqlen 8192), in the
    launch configuration the benchmark times; 48 sampled chains compared over all tokens."""
    inp = ssd_inputs.make_selective_inputs(1)
    y, fin = _run(inp)
    rng = np.random.default_rng(5)
    Bt, dim = inp["cfg"]["batch"], inp["cfg"]["dim"]
    rows = np.concatenate([[0, Bt - 1], rng.integers(0, Bt, 46)])
    chans = np.concatenate([[0, dim - 1], rng.integers(0, dim, 46)])
    yo, ho = selective.selective_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                      inp["D"], None, rows=rows, chans=chans)
    assert rel_err(y[rows, :, chans], yo) <= TOL["bf16"]
    assert rel_err(fin[rows, chans], ho) <= TOL["bf16"]
    assert ssd.device_status() == 0


def test_selective_refuses_unsupported():
    x = torch.zeros(1, 4, 12, device="cuda", dtype=torch.bfloat16)  # dim 12: not 8-aligned
    z = lambda *s: torch.zeros(*s, device="cuda")
    with pytest.raises(ssd.SSDError):
        ssd.selective_scan_fwd(x, z(1, 4, 12), z(12, 16), x.new_zeros(1, 4, 1, 16),
                               x.new_zeros(1, 4, 1, 16))
    x = torch.zeros(1, 4, 16, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(ssd.SSDError):  # dstate 8
        ssd.selective_scan_fwd(x, z(1, 4, 16), z(16, 8), x.new_zeros(1, 4, 1, 8),
                               x.new_zeros(1, 4, 1, 8))
