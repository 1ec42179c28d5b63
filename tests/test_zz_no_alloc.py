"""ssd_chunk_scan_fwd_noalloc: the chunked scan for callers that cannot allocate device memory
(its scratch is a fixed device array inside the library instead of a caller workspace).

Called through the C ABI and compared with ssd_chunk_scan_fwd on the same inputs, within the
bf16 tolerance the parity tests use, on two calls in a row (the second call reuses the array the
first one left behind), and with the float64 oracle on sampled chains.  This file is collected
last so that a run stopping at the first failure has already run every other test; it also
passes alone in a fresh process.
"""
import ctypes

import pytest
import torch

import mamba_ssd_scan_03_b200 as ssd
import ssd_inputs
from gpu_util import TOL, dev_inputs, oracle_chains, rel_err, sample_chains, to_np

pytestmark = pytest.mark.gpu


def _noalloc_call(t, shape, y, fin):
    Bt, L, H, P, N, G, Q = shape
    lib = ssd.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.ssd_chunk_scan_fwd_noalloc(
        t["x"].data_ptr(), t["dt"].data_ptr(), t["A"].data_ptr(), t["B"].data_ptr(),
        t["C"].data_ptr(), t["D"].data_ptr(),
        None if t["init"] is None else t["init"].data_ptr(), y.data_ptr(),
        None if fin is None else fin.data_ptr(), Bt, L, H, P, N, G, Q, ssd.SSD_BF16,
        ssd.SSD_F32, stream)


@pytest.mark.parametrize("shape", [
    dict(batch=2, seqlen=1500, nheads=8),      # segments with a summary pass
    dict(batch=4, seqlen=2048, nheads=80),     # whole sequences handed between CTAs
])
def test_noalloc_matches_workspace_entry_point(shape):
    cfg = dict(headdim=64, dstate=128, ngroups=1, chunk=256, io="bf16", init="normal0.1")
    cfg.update(shape)
    inp = ssd_inputs.make_scan_inputs(cfg, seed=31)
    t = dev_inputs(inp)
    Bt, L, H = cfg["batch"], cfg["seqlen"], cfg["nheads"]
    y_ref, f_ref = ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], 256,
                                      init_state=t["init"])
    torch.cuda.synchronize()
    for call in range(2):
        y = torch.full(t["x"].shape, float("nan"), dtype=torch.float32, device="cuda")
        fin = torch.full((Bt, H, 64, 128), float("nan"), dtype=torch.float32, device="cuda")
        rc = _noalloc_call(t, (Bt, L, H, 64, 128, 1, 256), y, fin)
        assert rc == 0, ssd.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        assert ssd.device_status() == 0
        assert rel_err(to_np(y), to_np(y_ref)) <= TOL["bf16"], call
        assert rel_err(to_np(fin), to_np(f_ref)) <= TOL["bf16"], call
    # and against the float64 oracle on sampled (b, h, p) chains
    ids, b, h, p = sample_chains(cfg, 48, seed=5)
    yo, fo = oracle_chains(inp, ids, b, h, p)
    bb, hh, pp = (torch.as_tensor(v) for v in (b, h, p))
    assert rel_err(to_np(y[bb, :, hh, pp]), yo) <= TOL["bf16"]
    assert rel_err(to_np(fin[bb, hh, pp]), fo) <= TOL["bf16"]


def test_noalloc_rejects_what_does_not_fit():
    # 256 x 40 one-block sequences: a CTA walks at most 14 of them, so the walk needs at least
    # 732 CTAs and as many published 64 KiB states (46 MiB > the 32 MiB array): rejected before
    # any launch
    lib = ssd.load()
    rc = lib.ssd_chunk_scan_fwd_noalloc(*([None] * 9), 256, 128, 80, 64, 128, 1, 256,
                                        ssd.SSD_BF16, ssd.SSD_F32, None)
    assert rc == 2  # SSD_ERR_UNSUPPORTED
    # float32 io has no tensor-core path, so no fixed-scratch variant either
    rc = lib.ssd_chunk_scan_fwd_noalloc(*([None] * 9), 1, 256, 4, 16, 16, 1, 64, ssd.SSD_F32,
                                        ssd.SSD_F32, None)
    assert rc == 2
