"""GPU parity of the block steps around the layer (short convolution + SiLU, dt softplus,
SiLU output gate) against their float64 definitions.

The kernels compute in float32 and round once to the output dtype.  Bar: float32 outputs
within 1e-5 * (|ref| + scale) of the float64 value, scale = RMS of the reference (a few float32
ulps of the K-term sum and of exp/log); bf16 outputs within that plus 2^-8 |ref| (at most half
a bf16 ulp of rounding).
"""
import numpy as np
import pytest
import torch

import mamba_ssd_scan_03_b200 as ssd
import ssd_inputs
from gpu_util import to_dev, to_np
from oracle import glue

pytestmark = pytest.mark.gpu


def _check(got, ref, bf16):
    scale = float(np.sqrt(np.mean(np.square(ref)))) or 1.0
    bound = 1e-5 * (np.abs(ref) + scale) + (2.0 ** -8 * np.abs(ref) if bf16 else 0.0)
    excess = np.abs(got - ref) - bound
    assert float(excess.max()) <= 0.0, float(np.abs(got - ref).max())


@pytest.mark.parametrize("io,batch,seqlen,cdim,K", [
    ("bf16", 2, 300, 64, 4), ("f32", 2, 300, 64, 4), ("bf16", 1, 37, 8, 1),
    ("f32", 3, 5, 12, 8), ("bf16", 2, 1, 16, 4), ("bf16", 1, 129, 5376 // 8, 3)])
def test_conv_silu(io, batch, seqlen, cdim, K):
    g = ssd_inputs.make_glue_inputs(batch, seqlen, cdim, K, 2, 8, io)
    bf16 = io == "bf16"
    u = to_dev(g["u"], bf16)
    for bias in (g["conv_bias"], None):
        out = ssd.conv_silu(u, to_dev(g["w"]), None if bias is None else to_dev(bias))
        _check(to_np(out), glue.conv_silu(g["u"], g["w"], bias), bf16)
    assert ssd.device_status() == 0


def test_conv_silu_batches_do_not_mix():
    """The window of the first tokens of batch b must not reach into batch b-1."""
    g = ssd_inputs.make_glue_inputs(3, 6, 8, 4, 2, 8, "f32")
    u = g["u"].copy()
    u[1:, :, :] = 0.0
    out = ssd.conv_silu(to_dev(u), to_dev(g["w"]))
    assert torch.all(out[1:] == 0).item()


@pytest.mark.parametrize("batch,seqlen,H", [(2, 300, 80), (1, 7, 3), (4, 1, 24)])
def test_dt_softplus(batch, seqlen, H):
    g = ssd_inputs.make_glue_inputs(batch, seqlen, 8, 4, H, 8, "f32")
    raw = g["raw"].copy()
    raw[0, 0, : min(H, 3)] = [60.0, -60.0, 0.0][: min(H, 3)]  # both tails and 0
    for bias in (g["dt_bias"], None):
        dt = ssd.dt_softplus(to_dev(raw), None if bias is None else to_dev(bias))
        _check(to_np(dt), glue.dt_softplus(raw, bias), False)
    # in place
    t = to_dev(raw)
    ssd.dt_softplus(t, to_dev(g["dt_bias"]), out=t)
    _check(to_np(t), glue.dt_softplus(raw, g["dt_bias"]), False)
    assert ssd.device_status() == 0


@pytest.mark.parametrize("io,out_dtype", [("f32", torch.float32), ("bf16", torch.float32),
                                          ("bf16", torch.bfloat16)])
def test_gate_silu(io, out_dtype):
    g = ssd_inputs.make_glue_inputs(2, 131, 8, 4, 4, 64, io)
    z = g["z"].copy()
    big = [100.0, -100.0, 0.0, 20.0]
    z.reshape(-1)[:4] = ssd_inputs.f32_to_bf16_bits(np.float32(big)) if io == "bf16" else big
    out = ssd.gate_silu(to_dev(g["y"]), to_dev(z, io == "bf16"), out_dtype=out_dtype)
    _check(to_np(out), glue.gate_silu(g["y"], z), out_dtype == torch.bfloat16)
    # in place over y
    y = to_dev(g["y"])
    if out_dtype == torch.float32:
        ssd.gate_silu(y, to_dev(z, io == "bf16"), out=y)
        _check(to_np(y), glue.gate_silu(g["y"], z), False)
    assert ssd.device_status() == 0


def test_gate_silu_refuses_narrow_output_in_place():
    """out == y with a bf16 out would overwrite y elements that other threads have not read yet
    (a bf16 group of 8 covers the bytes of the first 4 float32 inputs of the same group):
    SSD_ERR_INVALID_ARG before any launch, and y is untouched."""
    y = torch.randn(4096, device="cuda")
    y0 = y.clone()
    z = torch.randn(4096, device="cuda").to(torch.bfloat16)
    lib = ssd.load()
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.ssd_gate_silu(y.data_ptr(), z.data_ptr(), y.data_ptr(), y.numel(), ssd.SSD_BF16,
                           ssd.SSD_BF16, stream)
    assert rc == 1  # SSD_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.equal(y, y0)
    assert ssd.device_status() == 0


def test_glue_refuses_unsupported():
    u = torch.zeros(1, 4, 6, device="cuda", dtype=torch.bfloat16)  # 6 channels: not 8-aligned
    with pytest.raises(ssd.SSDError):
        ssd.conv_silu(u, torch.zeros(6, 4, device="cuda"))
    w9 = torch.zeros(8, 9, device="cuda")
    with pytest.raises(ssd.SSDError):
        ssd.conv_silu(torch.zeros(1, 4, 8, device="cuda", dtype=torch.bfloat16), w9)
    with pytest.raises(ssd.SSDError):
        ssd.gate_silu(torch.zeros(12, device="cuda"), torch.zeros(12, device="cuda",
                                                                   dtype=torch.bfloat16))
