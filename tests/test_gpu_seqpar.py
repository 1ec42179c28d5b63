"""GPU parity of the slice summary (ssd_chunk_state_fwd), the state passing between slices
(ssd_state_pass) and the sequence-sliced scan they make up, against the float64 oracle.  The
slices are run one after another on one GPU (no rank waits on another)."""
import numpy as np
import pytest
import torch

import mamba_ssd_scan_03_b200 as ssd
import oracle
import ssd_inputs
from gpu_util import TOL, dev_inputs, rel_err, to_np

pytestmark = pytest.mark.gpu


def _cfg(io, **kw):
    c = dict(batch=2, seqlen=700, nheads=4, headdim=64, dstate=128, ngroups=1, chunk=256,
             io=io, init="normal0.1")
    if io == "f32":
        c.update(headdim=24, dstate=40, ngroups=2, chunk=64)
    c.update(kw)
    return c


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("with_init", [False, True])
def test_chunk_state_matches_oracle(io, with_init):
    inp = ssd_inputs.make_scan_inputs(_cfg(io), seed=51)
    t = dev_inputs(inp)
    init = t["init"] if with_init else None
    fin, dec = ssd.chunk_state_fwd(t["x"], t["dt"], t["A"], t["B"], inp["cfg"]["chunk"],
                                   init_state=init)
    torch.cuda.synchronize()
    _, f_ref = oracle.scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                           init=inp["init"] if with_init else None)
    d_ref = (inp["dt"].astype(np.float64) * inp["A"].astype(np.float64)[None, None, :]).sum(1)
    assert rel_err(to_np(fin), f_ref) <= TOL[io]
    assert np.max(np.abs(to_np(dec) - d_ref) / np.abs(d_ref)) <= 1e-5
    assert ssd.device_status() == 0


def test_state_pass_matches_definition():
    rng = np.random.default_rng(52)
    R, Bt, H, P, N = 5, 3, 4, 24, 40
    S = rng.standard_normal((R, Bt, H, P, N)).astype(np.float32)
    dec = -rng.uniform(0.0, 3.0, (R, Bt, H)).astype(np.float32)
    init = rng.standard_normal((Bt, H, P, N)).astype(np.float32)
    st = torch.from_numpy(S).cuda()
    fin = ssd.state_pass(st, torch.from_numpy(dec).cuda(), torch.from_numpy(init).cuda())
    run = init.astype(np.float64)
    h_in = np.empty_like(S, dtype=np.float64)
    for r in range(R):
        h_in[r] = run
        run = np.exp(dec[r].astype(np.float64))[:, :, None, None] * run + S[r]
    torch.cuda.synchronize()
    assert rel_err(to_np(st), h_in) <= 1e-6
    assert rel_err(to_np(fin), run) <= 1e-6


@pytest.mark.parametrize("io,cuts", [("bf16", [0, 300, 550, 900]), ("bf16", [0, 128, 900]),
                                     ("f32", [0, 64, 400, 401, 900])])
def test_sliced_scan_equals_whole_scan(io, cuts):
    inp = ssd_inputs.make_scan_inputs(_cfg(io, seqlen=cuts[-1]), seed=53)
    t = dev_inputs(inp)
    Q = inp["cfg"]["chunk"]
    sl = [{k: t[k][:, lo:hi].contiguous() for k in ("x", "dt", "B", "C")}
          for lo, hi in zip(cuts[:-1], cuts[1:])]
    summ = [ssd.chunk_state_fwd(s["x"], s["dt"], t["A"], s["B"], Q) for s in sl]
    states = torch.stack([f for f, _ in summ])
    decays = torch.stack([d for _, d in summ])
    fin = ssd.state_pass(states, decays, t["init"])
    ys = [ssd.chunk_scan_fwd(s["x"], s["dt"], t["A"], s["B"], s["C"], t["D"], Q,
                             init_state=states[r].contiguous(), want_final=False)[0]
          for r, s in enumerate(sl)]
    y = torch.cat(ys, dim=1)
    torch.cuda.synchronize()
    y_ref, f_ref = oracle.scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                               init=inp["init"])
    assert rel_err(to_np(y), y_ref) <= TOL[io]
    assert rel_err(to_np(fin), f_ref) <= TOL[io]
    assert ssd.device_status() == 0
