"""GPU parity of the decode step (ssd_step) against the float64 oracle recurrence, which keeps
its own float64 state across steps.  Bar: per step, max |err(y)| <= 2e-2 * RMS(y_oracle) for
bf16 io (1e-4 for float32 io); the state to the same bound at checkpoints."""
import numpy as np
import pytest
import torch

import mamba_ssd_scan_03_b200 as ssd
import oracle
import ssd_inputs
from gpu_util import TOL, bf16_excess, dev_inputs, rel_err, sample_chains, to_dev, to_np

pytestmark = pytest.mark.gpu


def _step_dev(dec, k):
    s = ssd_inputs.decode_step_inputs(dec, k)
    bf16 = dec["cfg"]["io"] == "bf16"
    return s, {n: to_dev(s[n], bf16 and n != "dt") for n in ("x", "dt", "B", "C")}


@pytest.mark.parametrize("io,shape", [
    ("bf16", dict(batch=4, nheads=4, headdim=64, dstate=128)),
    ("f32", dict(batch=3, nheads=4, headdim=64, dstate=128, ngroups=2)),
    ("f32", dict(batch=2, nheads=3, headdim=24, dstate=40)),   # generic kernel
    ("bf16", dict(batch=2, nheads=4, headdim=32, dstate=128, ngroups=4)),
])
def test_decode_small_every_element(io, shape):
    dec = ssd_inputs.make_decode_inputs(4, io=io, **shape)
    A, D = to_dev(dec["A"]), to_dev(dec["D"])
    st = to_dev(dec["state"])
    so = dec["state"].astype(np.float64)
    for k in range(25):
        s, t = _step_dev(dec, k)
        y = ssd.step(st, t["x"], t["dt"], A, t["B"], t["C"], D)
        yo, so = oracle.step(so, s["x"], s["dt"], dec["A"], s["B"], s["C"], dec["D"])
        assert rel_err(to_np(y), yo) <= TOL[io], k
    torch.cuda.synchronize()
    assert rel_err(to_np(st), so) <= TOL[io]
    assert ssd.device_status() == 0


def test_decode_touches_only_state_and_y():
    dec = ssd_inputs.make_decode_inputs(4, batch=2, nheads=4)
    A, D = to_dev(dec["A"]), to_dev(dec["D"])
    n = dec["state"].size
    buf = torch.full((n + 2048,), 5.0, dtype=torch.float32, device="cuda")
    st = buf[1024:1024 + n].view(dec["state"].shape)
    st.copy_(to_dev(dec["state"]))
    s, t = _step_dev(dec, 0)
    ybuf = torch.full((t["x"].numel() + 512,), 9.0, dtype=torch.float32, device="cuda")
    y = ybuf[256:256 + t["x"].numel()].view(t["x"].shape)
    ssd.step(st, t["x"], t["dt"], A, t["B"], t["C"], D, out=y)
    torch.cuda.synchronize()
    assert torch.all(buf[:1024] == 5.0) and torch.all(buf[1024 + n:] == 5.0)
    assert torch.all(ybuf[:256] == 9.0) and torch.all(ybuf[256 + t["x"].numel():] == 9.0)


def test_prefill_then_decode():
    """Final state of a chunked scan over L tokens, then k decode steps == the recurrence over
    L + k tokens (the method's two forms hand over through the state)."""
    L, k = 500, 6
    inp = ssd_inputs.make_scan_inputs(dict(batch=2, seqlen=L + k, nheads=4, headdim=64,
                                           dstate=128, ngroups=1, chunk=256, io="bf16",
                                           init="normal0.1"), seed=21)
    t = dev_inputs(inp)
    pre = {n: t[n][:, :L].contiguous() for n in ("x", "dt", "B", "C")}
    _, st = ssd.chunk_scan_fwd(pre["x"], pre["dt"], t["A"], pre["B"], pre["C"], t["D"], 256,
                               init_state=t["init"])
    ys = []
    for j in range(L, L + k):
        ys.append(ssd.step(st, t["x"][:, j].contiguous(), t["dt"][:, j].contiguous(), t["A"],
                           t["B"][:, j].contiguous(), t["C"][:, j].contiguous(), t["D"]))
    torch.cuda.synchronize()
    yo, fo = oracle.scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                         init=inp["init"])
    for i, j in enumerate(range(L, L + k)):
        assert rel_err(to_np(ys[i]), yo[:, j]) <= TOL["bf16"]
    assert rel_err(to_np(st), fo) <= TOL["bf16"]


def test_decode_workload_1000_steps():
    """The decode workload: 1000 successive steps on 256 sequences x 80 heads x 64 x 128 state.
    y is compared at every step on 1024 sampled (b, h, p) chains; the state of those chains
    at steps 1, 10, 100 and 1000."""
    dec = ssd_inputs.make_decode_inputs(4)
    cfg = dec["cfg"]
    ids, b, h, p = sample_chains(cfg, 1024, seed=4)
    A, D = to_dev(dec["A"]), to_dev(dec["D"])
    st = to_dev(dec["state"])
    so = dec["state"][b, h, p].astype(np.float64)
    bi, hi, pi = (torch.as_tensor(v, device="cuda") for v in (b, h, p))
    worst = 0.0
    for k in range(cfg["decode_steps"]):
        s, t = _step_dev(dec, k)
        y = ssd.step(st, t["x"], t["dt"], A, t["B"], t["C"], D)
        yo, so = oracle.step(so, s["x"], s["dt"], dec["A"], s["B"], s["C"], dec["D"],
                             chains=ids)
        e = rel_err(to_np(y[bi, hi, pi]), yo)
        worst = max(worst, e)
        assert e <= TOL["bf16"], (k, e)
        if k + 1 in (1, 10, 100, 1000):
            assert rel_err(to_np(st[bi, hi, pi]), so) <= TOL["bf16"], k + 1
    assert ssd.device_status() == 0


def test_decode_bf16_output():
    dec = ssd_inputs.make_decode_inputs(4, batch=4, nheads=4)
    A, D = to_dev(dec["A"]), to_dev(dec["D"])
    st = to_dev(dec["state"])
    so = dec["state"].astype(np.float64)
    for k in range(10):
        s, t = _step_dev(dec, k)
        y = ssd.step(st, t["x"], t["dt"], A, t["B"], t["C"], D, y_dtype=torch.bfloat16)
        assert y.dtype == torch.bfloat16
        yo, so = oracle.step(so, s["x"], s["dt"], dec["A"], s["B"], s["C"], dec["D"])
        assert bf16_excess(to_np(y), yo, TOL["bf16"]) <= TOL["bf16"], k
