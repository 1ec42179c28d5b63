"""Host-only checks of the C ABI (no GPU needed): the library builds and loads, exports every
function include/ssd.h declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re
import subprocess

import pytest

import mamba_ssd_scan_03_b200 as ssd
from mamba_ssd_scan_03_b200 import build as ssd_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd.h")


@pytest.fixture(scope="module")
def lib():
    ssd_build.build()
    return ssd.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssd_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(ssd.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", ssd.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (ssd_[a-z_0-9]+)\b", out))
    for name in declared_functions():
        assert name in exported, name
        getattr(lib, name)  # resolvable through ctypes


def test_status_strings(lib):
    for code in range(6):
        assert lib.ssd_status_string(code).decode().startswith(ssd.STATUS[code])
    assert ssd.version().startswith("ssd-b200")


def test_path_selection(lib):
    # bf16, headdim 64, dstate 128, even heads per group -> tensor cores
    assert ssd.path(4, 8192, 80, 64, 128, 1, 256, ssd.SSD_BF16) == ssd.SSD_PATH_TCGEN05
    assert ssd.path(1, 1 << 20, 24, 64, 128, 1, 256, ssd.SSD_BF16) == ssd.SSD_PATH_TCGEN05
    assert ssd.path(1, 256, 4, 16, 16, 1, 64, ssd.SSD_F32) == ssd.SSD_PATH_SIMT
    assert ssd.path(4, 8192, 80, 64, 128, 1, 256, ssd.SSD_F32) == ssd.SSD_PATH_SIMT
    assert ssd.path(2, 512, 4, 64, 128, 4, 256, ssd.SSD_BF16) == ssd.SSD_PATH_SIMT  # 1 head/group
    assert ssd.path(2, 512, 4, 64, 128, 2, 256, ssd.SSD_BF16) == ssd.SSD_PATH_TCGEN05


def test_workspace_sizes(lib):
    # tensor-core path: one float32 state per (batch, segment, head) plus a decay per segment
    ws = ssd.workspace_size(4, 8192, 80, 64, 128, 1, 256)
    assert ws > 0 and ws % 256 == 0
    assert ws >= 4 * 80 * 64 * 128 * 4
    # SIMT path: cumsums + one state per chunk
    ws0 = ssd.workspace_size(1, 256, 4, 16, 16, 1, 64, ssd.SSD_F32)
    assert ws0 >= (4 * 4 * 64 + 4 * 4 * 16 * 16) * 4
    # invalid shapes report 0
    assert ssd.workspace_size(1, 256, 4, 16, 16, 1, 100, ssd.SSD_F32) == 0
    assert ssd.workspace_size(1, 256, 3, 16, 16, 2, 64, ssd.SSD_F32) == 0


def _scan_call(lib, **kw):
    args = dict(x=None, dt=None, A=None, B=None, C=None, D=None, init=None, y=None, fin=None,
                batch=1, seqlen=256, nheads=4, headdim=16, dstate=16, ngroups=1, chunk=64,
                io=ssd.SSD_F32, y_dtype=ssd.SSD_F32, ws=None, ws_bytes=0, stream=None)
    args.update(kw)
    return lib.ssd_chunk_scan_fwd(*args.values())


@pytest.mark.parametrize("bad", [
    dict(chunk=100), dict(chunk=0), dict(batch=0), dict(seqlen=0), dict(nheads=3, ngroups=2),
    dict(headdim=0), dict(dstate=-1), dict(io=7), dict(y_dtype=5),
    dict(),  # all pointers NULL
])
def test_scan_rejects_bad_arguments_on_host(lib, bad):
    assert _scan_call(lib, **bad) == 1  # SSD_ERR_INVALID_ARG


def test_step_rejects_bad_arguments_on_host(lib):
    assert lib.ssd_step(*([None] * 8), 0, 4, 16, 16, 1, 1, 0, None) == 1
    assert lib.ssd_step(*([None] * 8), 2, 4, 16, 16, 3, 1, 0, None) == 1
    assert lib.ssd_step(*([None] * 8), 2, 4, 16, 16, 1, 0, 1, None) == 1  # f32 io, bf16 y
    assert lib.ssd_step(*([None] * 8), 2, 4, 16, 16, 1, 1, 0, None) == 1  # NULL pointers


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16)
    with pytest.raises((ValueError, RuntimeError)):
        ssd.chunk_scan_fwd(x, torch.zeros(1, 4, 2), torch.zeros(2), torch.zeros(1, 4, 1, 128),
                           torch.zeros(1, 4, 1, 128), None, 256)


def test_state_entry_points_reject_bad_arguments_on_host(lib):
    # ssd_chunk_state_fwd(x, dt, A, B, init, final, total_decay, batch, seqlen, nheads, headdim,
    #                     dstate, ngroups, chunk, io, workspace, bytes, stream)
    shape = [2, 300, 4, 64, 128, 1, 256, 1]
    assert lib.ssd_chunk_state_fwd(*([None] * 7), *shape, None, 0, None) == 1  # NULL pointers
    bad = list(shape)
    bad[6] = 100  # chunk
    assert lib.ssd_chunk_state_fwd(*([None] * 7), *bad, None, 0, None) == 1
    bad = list(shape)
    bad[2], bad[5] = 3, 2  # 3 heads in 2 groups
    assert lib.ssd_chunk_state_fwd(*([None] * 7), *bad, None, 0, None) == 1
    # ssd_state_pass(states, decay, init, final, nslices, batch, nheads, headdim, dstate, stream)
    assert lib.ssd_state_pass(None, None, None, None, 0, 2, 4, 64, 128, None) == 1
    assert lib.ssd_state_pass(None, None, None, None, 3, 2, 4, 64, 128, None) == 1
    assert lib.ssd_state_pass(None, None, None, None, 3, 2, 0, 64, 128, None) == 1


def test_sliced_scan_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16)
    with pytest.raises((ValueError, RuntimeError)):
        ssd.chunk_state_fwd(x, torch.zeros(1, 4, 2), torch.zeros(2), torch.zeros(1, 4, 1, 128),
                            256)
    with pytest.raises((ValueError, RuntimeError)):
        ssd.state_pass(torch.zeros(2, 1, 2, 64, 128), torch.zeros(2, 1, 2))


def test_walk_plans_on_host(lib):
    # one walk over whole sequences unless a sequence is longer than every CTA's share of all
    # blocks plus the segment plan's overhead (9 blocks; a host without a GPU plans for 148
    # SMs); segments with a summary pass (seg_state + seg_pass + walk) otherwise
    assert ssd.plan_info(4, 8192, 80, 64, 128, 1, 256) == dict(launches=1, ctas=148, segments=1)
    # 130M layer: 96 sequences of 16 blocks, share 11 -> whole sequences on 96 CTAs
    assert ssd.plan_info(8, 2048, 24, 64, 128, 1, 256) == dict(launches=1, ctas=96, segments=1)
    # 40 sequences of 32 blocks, share 9 -> segments
    p = ssd.plan_info(1, 4096, 80, 64, 128, 1, 256)
    assert p["launches"] == 3 and p["segments"] >= 2 and p["ctas"] <= 148
    p = ssd.plan_info(1, 1 << 20, 24, 64, 128, 1, 256)
    assert p["launches"] == 3 and p["ctas"] == 148 and 8192 / p["segments"] <= 8192 * 12 / 148
    # forced plans and CTA caps
    assert ssd.plan_info(2, 1000, 4, 64, 128, 1, 256, max_ctas=3, plan=1) == \
        dict(launches=1, ctas=3, segments=1)
    assert ssd.plan_info(2, 1000, 4, 64, 128, 1, 256, max_ctas=3, plan=2)["segments"] >= 2
    # every range is at least one segment long: one sequence of 47 blocks over 9 CTAs in
    # segments of 6 blocks leaves 7 CTAs
    p = ssd.plan_info(1, 6000, 2, 64, 128, 1, 256, max_ctas=9, plan=2)
    assert p == dict(launches=3, ctas=7, segments=8)
    # not a tensor-core shape / invalid
    with pytest.raises(ssd.SSDError):
        ssd.plan_info(1, 256, 4, 16, 16, 1, 64, ssd.SSD_F32)
    with pytest.raises(ssd.SSDError):
        ssd.plan_info(1, 256, 4, 64, 128, 1, 100)


def test_scan_ex_rejects_bad_options_on_host(lib):
    import ctypes
    shape = [2, 300, 4, 64, 128, 1, 256, 1, 0]
    for opts in [(-1, 0, 0), (0, 3, 0), (0, -1, 0), (0, 0, -2)]:
        o = ssd.ScanOptions(*opts)
        assert lib.ssd_chunk_scan_fwd_ex(*([None] * 9), *shape, None, 0, ctypes.byref(o),
                                         None) == 1
    # valid options, NULL pointers: still an argument error, nothing launched
    o = ssd.ScanOptions(3, 1, -1)
    assert lib.ssd_chunk_scan_fwd_ex(*([None] * 9), *shape, None, 0, ctypes.byref(o), None) == 1
    # the float32 SIMT shapes have no tensor-core plan
    assert lib.ssd_chunk_scan_fwd_ex(*([None] * 9), 1, 256, 4, 16, 16, 1, 64, 0, 0, None, 0,
                                     None, None) == 2
    # the workspace of a forced segment plan covers the segments' states
    o1, o2 = ssd.ScanOptions(0, 1, 0), ssd.ScanOptions(0, 2, 0)
    w1 = lib.ssd_chunk_scan_workspace_size_ex(4, 8192, 80, 64, 128, 1, 256, 1, ctypes.byref(o1))
    w2 = lib.ssd_chunk_scan_workspace_size_ex(4, 8192, 80, 64, 128, 1, 256, 1, ctypes.byref(o2))
    assert w1 > 0 and w2 >= w1


def test_backward_rejects_bad_arguments_on_host(lib):
    # ssd_chunk_scan_bwd(x, dt, A, B, C, D, init, dy, dfinal, dx, ddt, dA, dB, dC, dD, dinit,
    #                    batch, seqlen, nheads, headdim, dstate, ngroups, io, ws, bytes, stream)
    shape = [2, 300, 4, 64, 128, 1, 1]
    assert lib.ssd_chunk_scan_bwd(*([None] * 16), *shape, None, 0, None) == 1  # NULL pointers
    bad = list(shape)
    bad[2], bad[5] = 3, 2  # 3 heads in 2 groups
    assert lib.ssd_chunk_scan_bwd(*([None] * 16), *bad, None, 0, None) == 1
    bad = list(shape)
    bad[6] = 9  # io
    assert lib.ssd_chunk_scan_bwd(*([None] * 16), *bad, None, 0, None) == 1
    # tiles too large for one chunk in shared memory
    assert lib.ssd_chunk_scan_bwd(*([None] * 16), 1, 128, 2, 128, 256, 1, 1, None, 0,
                                  None) == 2
    assert lib.ssd_chunk_scan_bwd_workspace_size(2, 300, 4, 64, 128, 1, 1) > 0
    assert lib.ssd_chunk_scan_bwd_workspace_size(2, 300, 4, 64, 128, 3, 1) == 0


def test_backward_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16)
    with pytest.raises((ValueError, RuntimeError)):
        ssd.chunk_scan_bwd(x, torch.zeros(1, 4, 2), torch.zeros(2), torch.zeros(1, 4, 1, 128),
                           torch.zeros(1, 4, 1, 128), None, torch.zeros(1, 4, 2, 64))


def test_glue_entry_points_reject_bad_arguments_on_host(lib):
    # ssd_conv_silu(u, w, bias, out, batch, seqlen, cdim, kwidth, io, stream)
    assert lib.ssd_conv_silu(None, None, None, None, 1, 8, 64, 4, 1, None) == 1  # NULL pointers
    assert lib.ssd_conv_silu(None, None, None, None, 1, 8, 64, 9, 1, None) == 1  # kwidth > 8
    assert lib.ssd_conv_silu(None, None, None, None, 1, 8, 64, 4, 7, None) == 1  # dtype code
    # ssd_dt_softplus(raw, bias, dt, batch, seqlen, nheads, stream)
    assert lib.ssd_dt_softplus(None, None, None, 1, 8, 4, None) == 1
    assert lib.ssd_dt_softplus(None, None, None, 1, 0, 4, None) == 1
    # ssd_gate_silu(y, z, out, n, z_dtype, out_dtype, stream): bf16 out needs bf16 z
    assert lib.ssd_gate_silu(None, None, None, 64, 0, 1, None) == 1
    assert lib.ssd_gate_silu(None, None, None, 0, 1, 1, None) == 1


def test_glue_binding_refuses_cpu_tensors(lib):
    import torch
    with pytest.raises((ValueError, RuntimeError)):
        ssd.conv_silu(torch.zeros(1, 4, 8, dtype=torch.bfloat16), torch.zeros(8, 4))
    with pytest.raises((ValueError, RuntimeError)):
        ssd.dt_softplus(torch.zeros(1, 4, 2))
    with pytest.raises((ValueError, RuntimeError)):
        ssd.gate_silu(torch.zeros(16), torch.zeros(16))


def test_selective_entry_point_rejects_bad_arguments_on_host(lib):
    # ssd_selective_scan_fwd(x, dt, A, B, C, D, init, y, final, batch, seqlen, dim, dstate,
    #                        ngroups, io, y_dtype, stream)
    shape = [2, 64, 64, 16, 1, 1, 0]
    assert lib.ssd_selective_scan_fwd(*([None] * 9), *shape, None) == 1  # NULL pointers
    bad = list(shape)
    bad[2], bad[4] = 64, 3  # 64 channels in 3 groups
    assert lib.ssd_selective_scan_fwd(*([None] * 9), *bad, None) == 1
    bad = list(shape)
    bad[5], bad[6] = 0, 1  # bf16 y with f32 io
    assert lib.ssd_selective_scan_fwd(*([None] * 9), *bad, None) == 1
    bad = list(shape)
    bad[1] = 0  # empty sequence
    assert lib.ssd_selective_scan_fwd(*([None] * 9), *bad, None) == 1


def test_selective_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 4, 16, dtype=torch.bfloat16)
    with pytest.raises((ValueError, RuntimeError)):
        ssd.selective_scan_fwd(x, torch.zeros(1, 4, 16), torch.zeros(16, 16),
                               torch.zeros(1, 4, 1, 16, dtype=torch.bfloat16),
                               torch.zeros(1, 4, 1, 16, dtype=torch.bfloat16))


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "ssd.h"
int main(void) {
  /* a plain C client: the header is valid C99 and every call links against libssd.so */
  if (strncmp(ssd_version(), "ssd-b200", 8) != 0) return 1;
  if (strcmp(ssd_status_string(SSD_OK), "SSD_OK") != 0) return 2;
  if (ssd_chunk_scan_path(2, 300, 4, 64, 128, 1, 256, SSD_BF16) != SSD_PATH_TCGEN05) return 3;
  if (ssd_chunk_scan_path(2, 300, 4, 64, 128, 1, 256, SSD_F32) != SSD_PATH_SIMT) return 4;
  if (ssd_chunk_scan_workspace_size(2, 300, 4, 64, 128, 1, 256, SSD_BF16) == 0) return 5;
  /* argument errors come back before anything touches a GPU */
  if (ssd_step(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 4, 64, 128, 1, SSD_BF16,
               SSD_F32, 0) != SSD_ERR_INVALID_ARG) return 6;
  if (ssd_selective_scan_fwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 8, 64, 16,
                             1, SSD_BF16, SSD_F32, 0) != SSD_ERR_INVALID_ARG) return 7;
  printf("%s\n", ssd_version());
  return 0;
}
"""


def test_plain_c_client_compiles_links_and_runs(lib, tmp_path):
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(ssd.LIB_PATH)
    cuda_inc = os.path.join(os.path.dirname(os.path.dirname(ssd_build.NVCC)), "include")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", cuda_inc, str(src), "-o", str(exe), "-L", libdir, "-l:libssd.so",
                    f"-Wl,-rpath,{libdir}"], check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stderr)
    assert r.stdout.startswith("ssd-b200")
