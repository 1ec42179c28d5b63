"""GPU parity of the chunked scan (ssd_chunk_scan_fwd / _simt) against the float64 oracle.

Bar: max |err| <= tol * RMS(oracle) for y and for the final state, tol = 1e-4 (float32 io) or
2e-2 (bf16 io).  Small cases compare every element; the full-size workloads compare sampled
(b, h, p) chains end to end (the whole sequence of each sampled chain and its final state),
in the same launch configuration bench.py times.
"""
import math

import numpy as np
import pytest
import torch

import mamba_ssd_scan_03_b200 as ssd
import oracle
import ssd_inputs
from gpu_util import (TOL, bf16_excess, dev_inputs, oracle_chains, rel_err, sample_chains,
                      to_dev, to_np)

pytestmark = pytest.mark.gpu


def run(inp, t, chunk=None, simt=False, init="auto", **kw):
    fn = ssd.chunk_scan_fwd_simt if simt else ssd.chunk_scan_fwd
    chunk = chunk or inp["cfg"]["chunk"] or 256
    init_t = t["init"] if init == "auto" else init
    y, fin = fn(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], chunk, init_state=init_t, **kw)
    torch.cuda.synchronize()
    assert ssd.device_status() == 0
    return y, fin


def check_full(inp, y, fin, tol=None):
    tol = tol or TOL[inp["cfg"]["io"]]
    yo, fo = oracle.scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                         init=inp["init"])
    ey, ef = rel_err(to_np(y), yo), rel_err(to_np(fin), fo)
    assert ey <= tol, f"y: max|err|/RMS = {ey:.3e} > {tol}"
    assert ef <= tol, f"final state: max|err|/RMS = {ef:.3e} > {tol}"
    return ey, ef


def small(io="bf16", seed=7, **shape):
    cfg = dict(batch=1, seqlen=256, nheads=4, headdim=64, dstate=128, ngroups=1, chunk=256,
               io=io, init="normal0.1")
    cfg.update(shape)
    return ssd_inputs.make_scan_inputs(cfg, seed=seed)


# ---- the tiny float32 workload, every element ------------------------------------------------
def test_tiny_f32_workload():
    inp = ssd_inputs.make_scan_inputs(0)
    assert ssd.path(1, 256, 4, 16, 16, 1, 64, ssd.SSD_F32) == ssd.SSD_PATH_SIMT
    y, fin = run(inp, dev_inputs(inp))
    check_full(inp, y, fin)


# ---- tensor-core path, every element, several tiles and ragged tails --------------------------
@pytest.mark.parametrize("shape", [
    dict(batch=1, seqlen=128, nheads=2),
    dict(batch=2, seqlen=300, nheads=4),
    dict(batch=1, seqlen=1000, nheads=8, ngroups=2),
    dict(batch=3, seqlen=777, nheads=6, init="zeros"),
    dict(batch=2, seqlen=1, nheads=2),
    dict(batch=1, seqlen=4500, nheads=4),     # several segments per sequence
])
def test_tensor_core_path_small(shape):
    inp = small(**shape)
    c = inp["cfg"]
    assert ssd.path(c["batch"], c["seqlen"], c["nheads"], 64, 128, c["ngroups"], 256) == \
        ssd.SSD_PATH_TCGEN05
    y, fin = run(inp, dev_inputs(inp))
    check_full(inp, y, fin)


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [
    dict(batch=2, seqlen=300, nheads=4),
    dict(batch=1, seqlen=513, nheads=4, ngroups=4),  # one group per head
    dict(batch=2, seqlen=200, nheads=3, headdim=24, dstate=40, ngroups=1),
])
def test_simt_path_small(io, shape):
    inp = small(io=io, **shape)
    y, fin = run(inp, dev_inputs(inp), simt=True)
    check_full(inp, y, fin)


@pytest.mark.parametrize("chunk", [64, 128, 256])
@pytest.mark.parametrize("simt", [False, True])
def test_chunk_size_invariance(chunk, simt):
    """The output does not depend on the block length (the duality's point); every admissible
    chunk gives the oracle's answer, including a partial last chunk."""
    inp = small(seed=11, batch=2, seqlen=700, nheads=4)
    y, fin = run(inp, dev_inputs(inp), chunk=chunk, simt=simt)
    check_full(inp, y, fin)


def test_slow_decay_stress():
    """Per-token decay >= 0.98: the inter-block states dominate y and the final state, so a
    broken state-passing path cannot hide behind the skip term."""
    inp = ssd_inputs.make_scan_inputs(1, seqlen=1024, A_range=(1e-3, 1e-1))
    t = dev_inputs(inp)
    y, fin = run(inp, t)
    check_full(inp, y, fin)
    # the stricter diagnostic: the SSM part alone (y - D x) against the oracle's
    yo, _ = oracle.scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], None)
    xd = oracle.widen(inp["x"]) * inp["D"][None, None, :, None]
    assert rel_err(to_np(y) - xd, yo) <= 4e-2


def test_initial_state_only():
    """x = 0 with a nonzero initial state: only the state-passing / off-diagonal path acts."""
    inp = small(seed=12, batch=2, seqlen=640, nheads=4)
    inp["x"] = np.zeros_like(inp["x"])
    y, fin = run(inp, dev_inputs(inp))
    check_full(inp, y, fin)


@pytest.mark.parametrize("simt", [False, True])
def test_water_tank_embedded(simt):
    """The pages' water tank (decay 1/2, inflow 2: 0, 2, 3, 3.5, 3.75, 3.875, 3.9375 -> 4)
    through the GPU path: one channel and one state coordinate carry the tank, the rest is
    zero; blocks of 128 tokens so the level crosses block boundaries."""
    L, H = 300, 2
    if simt:
        P, N, io, dt_np = 16, 16, "f32", np.float32
    else:
        P, N, io, dt_np = 64, 128, "bf16", np.float32
    x = np.zeros((1, L, H, P), dtype=np.float32)
    x[0, 1:, :, 0] = 2.0
    Bm = np.zeros((1, L, 1, N), dtype=np.float32)
    Bm[..., 0] = 1.0
    store = (lambda a: ssd_inputs.f32_to_bf16_bits(a)) if io == "bf16" else (lambda a: a)
    inp = dict(x=store(x), dt=np.ones((1, L, H), dt_np), A=np.full(H, -math.log(2.0), np.float32),
               B=store(Bm), C=store(Bm.copy()), D=np.zeros(H, np.float32), init=None,
               cfg=dict(io=io, chunk=64 if simt else 256))
    y, fin = run(inp, dev_inputs(inp), simt=simt)
    yy = to_np(y)[0, :, 0, 0]
    expect = [0, 2, 3, 3.5, 3.75, 3.875, 3.9375]
    tol = 1e-5 if simt else 2e-2
    assert np.allclose(yy[:7], expect, atol=tol * 4, rtol=0)
    assert abs(yy[-1] - 4.0) <= tol * 4
    assert abs(to_np(fin)[0, 0, 0, 0] - 4.0) <= tol * 4


def test_deterministic():
    inp = small(seed=13, batch=2, seqlen=900, nheads=4)
    t = dev_inputs(inp)
    y1, f1 = run(inp, t)
    y2, f2 = run(inp, t)
    assert torch.equal(y1, y2) and torch.equal(f1, f2)


def test_resume_from_final_state():
    """Scan [0, L1) then [L1, L) from the first part's final state == one scan over [0, L)."""
    inp = small(seed=14, batch=2, seqlen=1100, nheads=4)
    t = dev_inputs(inp)
    L1 = 517
    part = lambda a, sl: a[:, sl].contiguous()
    ya, fa = ssd.chunk_scan_fwd(part(t["x"], slice(0, L1)), part(t["dt"], slice(0, L1)), t["A"],
                                part(t["B"], slice(0, L1)), part(t["C"], slice(0, L1)), t["D"],
                                256, init_state=t["init"])
    yb, fb = ssd.chunk_scan_fwd(part(t["x"], slice(L1, None)), part(t["dt"], slice(L1, None)),
                                t["A"], part(t["B"], slice(L1, None)),
                                part(t["C"], slice(L1, None)), t["D"], 256, init_state=fa)
    torch.cuda.synchronize()
    check_full(inp, torch.cat([ya, yb], dim=1), fb)


def test_final_state_in_place():
    inp = small(seed=15, batch=1, seqlen=400, nheads=4)
    t = dev_inputs(inp)
    state = t["init"].clone()
    y, fin = ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], 256,
                                init_state=state, final_out=state)
    torch.cuda.synchronize()
    assert fin.data_ptr() == state.data_ptr()
    check_full(inp, y, state)


def test_output_canaries():
    """Nothing is written outside y (ragged last block) or the final state."""
    inp = small(seed=16, batch=2, seqlen=333, nheads=4)
    t = dev_inputs(inp)
    n = t["x"].numel()
    ybuf = torch.full((n + 4096,), 7.0, dtype=torch.float32, device="cuda")
    fbuf = torch.full((2 * 4 * 64 * 128 + 1024,), -3.0, dtype=torch.float32, device="cuda")
    y = ybuf[1024:1024 + n].view(t["x"].shape)
    fin = fbuf[256:256 + 2 * 4 * 64 * 128].view(2, 4, 64, 128)
    ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], 256,
                       init_state=t["init"], out=y, final_out=fin)
    torch.cuda.synchronize()
    assert torch.all(ybuf[:1024] == 7.0) and torch.all(ybuf[1024 + n:] == 7.0)
    assert torch.all(fbuf[:256] == -3.0) and torch.all(fbuf[256 + 2 * 4 * 64 * 128:] == -3.0)
    check_full(inp, y, fin)


def test_no_skip_and_no_final():
    inp = small(seed=17, batch=1, seqlen=260, nheads=2)
    inp["D"] = np.zeros_like(inp["D"])
    t = dev_inputs(inp)
    y, fin = ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], None, 256,
                                init_state=t["init"], want_final=False)
    torch.cuda.synchronize()
    assert fin is None
    yo, _ = oracle.scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], None, init=inp["init"])
    assert rel_err(to_np(y), yo) <= TOL["bf16"]


# ---- argument errors that need device pointers -------------------------------------------------
def test_device_argument_errors():
    inp = small(seed=18, batch=1, seqlen=256, nheads=2)
    t = dev_inputs(inp)
    lib = ssd.load()
    y = torch.empty(t["x"].shape, dtype=torch.float32, device="cuda")
    need = ssd.workspace_size(1, 256, 2, 64, 128, 1, 256)
    small_ws = torch.empty(max(need // 2, 256), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream

    def call(x=t["x"], yv=y, ws=small_ws, wsb=None, B=t["B"], ydt=0):
        return lib.ssd_chunk_scan_fwd(x.data_ptr(), t["dt"].data_ptr(), t["A"].data_ptr(),
                                      B.data_ptr(), t["C"].data_ptr(), t["D"].data_ptr(), None,
                                      yv.data_ptr(), None, 1, 256, 2, 64, 128, 1, 256, 1, ydt,
                                      ws.data_ptr(), ws.numel() if wsb is None else wsb, stream)
    assert call() == 3                                    # workspace too small
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    assert call(ws=ws) == 0
    assert call(ws=ws, yv=t["x"], ydt=1) == 1             # y aliases x
    host = torch.empty_like(t["x"], device="cpu")
    assert call(ws=ws, x=host) == 1                       # host pointer
    xb = torch.empty(t["x"].numel() + 8, dtype=torch.bfloat16, device="cuda")
    xm = xb[1:1 + t["x"].numel()].view(t["x"].shape)      # 2-byte aligned only
    xm.copy_(t["x"])
    assert call(ws=ws, x=xm) == 2                         # TMA needs 16-byte alignment
    torch.cuda.synchronize()
    assert ssd.device_status() == 0


# ---- full-size workloads: sampled chains, the launch configuration bench.py times -------------
@pytest.mark.parametrize("cfg_idx,n_chains", [(1, 96), (2, 96)])
def test_full_size_workload(cfg_idx, n_chains):
    inp = ssd_inputs.make_scan_inputs(cfg_idx)
    cfg = inp["cfg"]
    t = dev_inputs(inp)
    y, fin = run(inp, t)
    ids, b, h, p = sample_chains(cfg, n_chains, seed=cfg_idx)
    yo, fo = oracle_chains(inp, ids, b, h, p)
    yg = to_np(y[torch.as_tensor(b), :, torch.as_tensor(h), torch.as_tensor(p)])
    fg = to_np(fin[torch.as_tensor(b), torch.as_tensor(h), torch.as_tensor(p)])
    assert rel_err(yg, yo) <= TOL["bf16"]
    assert rel_err(fg, fo) <= TOL["bf16"]
    # every element: the tensor-core result against the float32 SIMT kernels
    ys, fs = run(inp, t, simt=True)
    assert rel_err(to_np(y), to_np(ys)) <= TOL["bf16"]
    assert rel_err(to_np(fin), to_np(fs)) <= TOL["bf16"]


def test_million_token_context():
    inp = ssd_inputs.make_scan_inputs(3)
    cfg = inp["cfg"]
    t = dev_inputs(inp)
    y, fin = run(inp, t)
    ids, b, h, p = sample_chains(cfg, 24, seed=3)
    yo, fo = oracle_chains(inp, ids, b, h, p)
    yg = to_np(y[torch.as_tensor(b), :, torch.as_tensor(h), torch.as_tensor(p)])
    fg = to_np(fin[torch.as_tensor(b), torch.as_tensor(h), torch.as_tensor(p)])
    assert rel_err(yg, yo) <= TOL["bf16"]
    assert rel_err(fg, fo) <= TOL["bf16"]


@pytest.mark.parametrize("simt", [False, True])
def test_bf16_output(simt):
    """y in the io dtype (bf16): the error beyond the output's own rounding (half a bf16 ulp,
    <= 2^-8 |y|) stays within the bf16 tolerance."""
    inp = small(seed=19, batch=2, seqlen=700, nheads=4)
    y, fin = run(inp, dev_inputs(inp), simt=simt, y_dtype=torch.bfloat16)
    assert y.dtype == torch.bfloat16
    yo, fo = oracle.scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                         init=inp["init"])
    assert bf16_excess(to_np(y), yo, TOL["bf16"]) <= TOL["bf16"]
    assert rel_err(to_np(fin), fo) <= TOL["bf16"]
