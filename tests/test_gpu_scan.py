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
                      stratified_chains, to_dev, to_np)

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


def small(io="bf16", seed=7, A_range=None, **shape):
    cfg = dict(batch=1, seqlen=256, nheads=4, headdim=64, dstate=128, ngroups=1, chunk=256,
               io=io, init="normal0.1")
    cfg.update(shape)
    return ssd_inputs.make_scan_inputs(cfg, seed=seed, A_range=A_range)


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
    dict(batch=2, seqlen=640, nheads=8, ngroups=4),  # one group per head pair
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
    # wide states (the chunk summaries stage 32 and 16 tokens at a time) and widths that are
    # not multiples of four (element-by-element loads, padded rows)
    dict(batch=1, seqlen=150, nheads=2, headdim=32, dstate=256, ngroups=1),
    dict(batch=1, seqlen=100, nheads=2, headdim=16, dstate=512, ngroups=2),
    dict(batch=2, seqlen=90, nheads=2, headdim=18, dstate=30, ngroups=1),
])
def test_simt_path_small(io, shape):
    inp = small(io=io, **shape)
    y, fin = run(inp, dev_inputs(inp), simt=True)
    check_full(inp, y, fin)


@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_chunk_size_invariance(chunk):
    """The output does not depend on the block length (the duality's point); every admissible
    chunk gives the oracle's answer, including a partial last chunk.  Only the SIMT kernels use
    `chunk` as their block length: the tensor-core path evaluates 128-token blocks (the tcgen05
    M = 128 tile) whatever the argument, so repeating it per chunk would rerun one computation."""
    inp = small(seed=11, batch=2, seqlen=700, nheads=4)
    y, fin = run(inp, dev_inputs(inp), chunk=chunk, simt=True)
    check_full(inp, y, fin)


def test_tensor_core_path_ignores_chunk():
    """The tensor-core path's blocks are 128 tokens for every admissible chunk: bit-identical."""
    inp = small(seed=11, batch=2, seqlen=700, nheads=4)
    t = dev_inputs(inp)
    ys = [run(inp, t, chunk=q) for q in (64, 128, 256)]
    check_full(inp, *ys[0])
    for y, fin in ys[1:]:
        assert torch.equal(y, ys[0][0]) and torch.equal(fin, ys[0][1])


# ---- the walk's plans ------------------------------------------------------------------------
# plan 1: whole sequences, cut into ranges across CTAs, so that a range starting inside a
# sequence takes the state published by the CTA that walked the sequence's head; plan 2: segments
# whose entering states come from the summary pass, with ranges that also start inside segments.
@pytest.mark.parametrize("plan,max_ctas,shape", [
    (1, 3, dict(batch=2, seqlen=1000, nheads=4)),            # 4 x 8 blocks over 3 CTAs
    (1, 3, dict(batch=1, seqlen=2100, nheads=8, ngroups=2)),  # 4 x 17 blocks, ragged tail
    (1, 2, dict(batch=3, seqlen=300, nheads=2, init="zeros")),
    (1, 5, dict(batch=2, seqlen=4500, nheads=6)),            # 6 x 36 blocks over 5 CTAs
    (2, 5, dict(batch=1, seqlen=3000, nheads=4)),            # 3 segments of 8, ranges of 9.6
    (2, 0, dict(batch=2, seqlen=777, nheads=6)),             # one-block segments
    (2, 9, dict(batch=1, seqlen=6000, nheads=2)),            # one sequence, 9 segments
])
def test_walk_plans(plan, max_ctas, shape):
    inp = small(seed=21 + max_ctas, **shape)
    t = dev_inputs(inp)
    y, fin = ssd.chunk_scan_fwd_ex(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], 256,
                                   init_state=t["init"], max_ctas=max_ctas, plan=plan)
    torch.cuda.synchronize()
    assert ssd.device_status() == 0
    check_full(inp, y, fin)


def test_walk_plans_agree():
    """Whole sequences and segments walk the same blocks with the same arithmetic per block;
    only where the entering state of a stretch comes from differs."""
    inp = small(seed=29, batch=2, seqlen=2000, nheads=4)
    t = dev_inputs(inp)
    out = []
    for plan, ctas in ((1, 0), (1, 3), (2, 6)):
        out.append(ssd.chunk_scan_fwd_ex(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], 256,
                                         init_state=t["init"], max_ctas=ctas, plan=plan))
    torch.cuda.synchronize()
    assert ssd.device_status() == 0
    for y, fin in out[1:]:
        assert rel_err(to_np(y), to_np(out[0][0])) <= TOL["bf16"]
        assert rel_err(to_np(fin), to_np(out[0][1])) <= TOL["bf16"]
    check_full(inp, *out[0])


def test_batch_rows_in_separate_calls():
    """Each batch row scanned by its own call on views of the same tensors (on its own streams,
    as bench.py's end-to-end leg does) matches the whole-batch call: rows are independent, only
    the plan (and so where boundary states are handed over) differs."""
    inp = small(seed=31, batch=3, seqlen=1500, nheads=4)
    t = dev_inputs(inp)
    y, fin = run(inp, t)
    yr = torch.empty_like(y)
    fr = torch.empty_like(fin)
    streams = [torch.cuda.Stream() for _ in range(3)]
    torch.cuda.synchronize()
    for r, st in enumerate(streams):
        with torch.cuda.stream(st):
            sl = slice(r, r + 1)
            ssd.chunk_scan_fwd(t["x"][sl], t["dt"][sl], t["A"], t["B"][sl], t["C"][sl], t["D"],
                               256, init_state=t["init"][sl], out=yr[sl], final_out=fr[sl])
    torch.cuda.synchronize()
    assert ssd.device_status() == 0
    assert rel_err(to_np(yr), to_np(y)) <= TOL["bf16"]
    assert rel_err(to_np(fr), to_np(fin)) <= TOL["bf16"]
    check_full(inp, yr, fr)


@pytest.mark.parametrize("plan", [1, 2])
def test_device_timeout_is_reported_and_recovered(plan):
    """A wait that gives up: with no waiting allowed every CTA's first wait on an event that has
    not happened yet expires.  The kernel latches SSD_ERR_DEVICE_TIMEOUT, lets its copies and
    MMAs land, frees its tensor memory and returns; the next normal call on the same stream
    is correct."""
    inp = small(seed=33, batch=2, seqlen=1000, nheads=4)
    t = dev_inputs(inp)
    ssd.chunk_scan_fwd_ex(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], 256,
                          init_state=t["init"], max_ctas=3, plan=plan, wait_limit_ns=-1)
    torch.cuda.synchronize()
    assert ssd.device_status() == 5  # SSD_ERR_DEVICE_TIMEOUT
    assert ssd.device_status() == 0  # read and cleared
    y, fin = run(inp, t)
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


def test_fast_decay_mix():
    """Heads whose decay per token ranges from mild to extreme (|A| log-uniform in [0.5, 300]):
    within one call, 16-token groups that decay by less than a factor 2^64 sit beside groups that
    decay by more than 2^128, where an exponential taken across the group leaves the float
    range, so the mask must take each one over the span between its own two tokens."""
    inp = small(seed=23, batch=1, seqlen=512, nheads=8, A_range=(0.5, 300.0))
    dt, A = inp["dt"].astype(np.float64), inp["A"].astype(np.float64)
    span = -(dt * A[None, None, :]).reshape(1, -1, 16, 8).sum(axis=2) / math.log(2.0)
    assert (span < 64).any() and (span > 128).any()  # both kinds of group occur
    y, fin = run(inp, dev_inputs(inp))
    check_full(inp, y, fin)


def test_initial_state_only():
    """x = 0 with a nonzero initial state: only the state-passing / off-diagonal path acts."""
    inp = small(seed=12, batch=2, seqlen=640, nheads=4)
    inp["x"] = np.zeros_like(inp["x"])
    y, fin = run(inp, dev_inputs(inp))
    check_full(inp, y, fin)


@pytest.mark.parametrize("plan,max_ctas", [(0, 0), (1, 2), (2, 4)])
def test_initial_state_only_survives(plan, max_ctas):
    """x = 0 with slow decays (A in [-0.5, -0.05]) over three and a half blocks: the initial state
    carries through every block and through the hand-offs between CTAs, and the final state is
    far from underflow (so its check has teeth)."""
    inp = small(seed=18, batch=2, seqlen=450, nheads=4, A_range=(0.05, 0.5))
    inp["x"] = np.zeros_like(inp["x"])
    t = dev_inputs(inp)
    y, fin = ssd.chunk_scan_fwd_ex(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], 256,
                                   init_state=t["init"], max_ctas=max_ctas, plan=plan)
    torch.cuda.synchronize()
    assert ssd.device_status() == 0
    _, fo = oracle.scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                        init=inp["init"])
    assert np.sqrt(np.mean(fo ** 2)) > 1e-3  # the state has not decayed away
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
@pytest.mark.parametrize("cfg_idx,per_pair", [(1, 4), (2, 3)])
def test_full_size_workload(cfg_idx, per_pair):
    """Configs 1 and 2 at full size, in bench.py's launch configuration: 768 and 960 chains (a few
    channels of every (batch row, head) pair) and their final states against the oracle."""
    inp = ssd_inputs.make_scan_inputs(cfg_idx)
    cfg = inp["cfg"]
    t = dev_inputs(inp)
    y, fin = run(inp, t)
    ids, b, h, p = stratified_chains(cfg, per_pair, seed=cfg_idx)
    assert len(ids) == cfg["batch"] * cfg["nheads"] * per_pair
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
    """2^20 tokens, 24 heads: 256 sampled chains (and their final states) against the oracle,
    compared 64 chains at a time; the RMS is taken over all compared elements."""
    inp = ssd_inputs.make_scan_inputs(3)
    cfg = inp["cfg"]
    t = dev_inputs(inp)
    y, fin = run(inp, t)
    ids, b, h, p = sample_chains(cfg, 256, seed=3)
    max_y = max_f = 0.0
    sq_y = sq_f = 0.0
    n_y = n_f = 0
    for s in range(0, len(ids), 64):
        sl = slice(s, s + 64)
        yo, fo = oracle_chains(inp, ids[sl], b[sl], h[sl], p[sl])
        bb, hh, pp = (torch.as_tensor(v[sl]) for v in (b, h, p))
        yg = to_np(y[bb, :, hh, pp])
        fg = to_np(fin[bb, hh, pp])
        max_y = max(max_y, float(np.max(np.abs(yg - yo))))
        max_f = max(max_f, float(np.max(np.abs(fg - fo))))
        sq_y += float(np.sum(yo ** 2))
        sq_f += float(np.sum(fo ** 2))
        n_y += yo.size
        n_f += fo.size
    assert max_y <= TOL["bf16"] * np.sqrt(sq_y / n_y)
    assert max_f <= TOL["bf16"] * np.sqrt(sq_f / n_f)


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
