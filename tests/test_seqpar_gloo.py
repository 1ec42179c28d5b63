"""Host logic of the sequence-sliced scan on CPU: two gloo ranks each hold half of every
sequence; the slice operations are the float64 oracle (test stand-ins for the GPU kernels); the
result must equal the oracle's scan of the whole sequence."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import ssd_inputs


class OracleOps:
    """Slice operations from their definitions, on float64 CPU tensors."""

    def state(self, x, dt, A, B, chunk):
        Bt, L, H, P = x.shape
        _, h1 = oracle.scan(x.numpy(), dt.numpy(), A.numpy(), B.numpy(),
                            np.zeros_like(B.numpy()), None)
        decay = (dt.numpy().astype(np.float64) * A.numpy()[None, None, :]).sum(axis=1)
        return torch.from_numpy(h1), torch.from_numpy(decay)

    def identity(self, x, B):
        Bt, _, H, P = x.shape
        return (torch.zeros((Bt, H, P, B.shape[3]), dtype=torch.float64),
                torch.zeros((Bt, H), dtype=torch.float64))

    def state_pass(self, states, decay, init_state):
        run = torch.zeros_like(states[0]) if init_state is None else init_state.clone()
        for r in range(states.shape[0]):
            s = states[r].clone()
            states[r] = run
            run = torch.exp(decay[r])[:, :, None, None] * run + s
        return run

    def scan(self, x, dt, A, B, C, D, chunk, init_state, y_dtype):
        y, _ = oracle.scan(x.numpy(), dt.numpy(), A.numpy(), B.numpy(), C.numpy(), D.numpy(),
                           init=init_state.numpy())
        return torch.from_numpy(y)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, cuts, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from mamba_ssd_scan_03_b200.seqpar import seqpar_scan_fwd
        inp = ssd_inputs.make_scan_inputs(dict(batch=2, seqlen=cuts[-1], nheads=4, headdim=8,
                                               dstate=16, ngroups=2, chunk=64, io="f32",
                                               init="normal0.1"), seed=41)
        lo, hi = cuts[rank], cuts[rank + 1]
        t = {k: torch.from_numpy(np.ascontiguousarray(inp[k][:, lo:hi]))
             for k in ("x", "dt", "B", "C")}
        y, fin = seqpar_scan_fwd(t["x"], t["dt"], torch.from_numpy(inp["A"]), t["B"], t["C"],
                                 torch.from_numpy(inp["D"]), 64,
                                 init_state=torch.from_numpy(inp["init"]).double(),
                                 ops=OracleOps())
        q.put((rank, y.numpy(), fin.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts", [[0, 150, 300], [0, 1, 300], [0, 97, 211, 300],
                                  [0, 50, 100, 220, 300], [0, 0, 300], [0, 150, 150, 300]])
def test_sliced_scan_equals_whole_scan(cuts):
    world = len(cuts) - 1
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, cuts, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        r, y, fin = q.get(timeout=300)
        out[r] = (y, fin)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = ssd_inputs.make_scan_inputs(dict(batch=2, seqlen=cuts[-1], nheads=4, headdim=8,
                                           dstate=16, ngroups=2, chunk=64, io="f32",
                                           init="normal0.1"), seed=41)
    y_ref, f_ref = oracle.scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                               init=inp["init"])
    y = np.concatenate([out[r][0] for r in range(world)], axis=1)
    assert np.max(np.abs(y - y_ref)) <= 1e-9 * np.sqrt(np.mean(y_ref ** 2))
    for r in range(world):
        assert np.max(np.abs(out[r][1] - f_ref)) <= 1e-9 * np.sqrt(np.mean(f_ref ** 2))


def _dying_worker(rank, world, port, q):
    """Rank 1 leaves before the exchange; rank 0 must get an error, not wait for ever."""
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=10))
    if rank == 1:
        os._exit(0)  # gone between steps, no collective in flight
    from mamba_ssd_scan_03_b200.seqpar import seqpar_scan_fwd
    inp = ssd_inputs.make_scan_inputs(dict(batch=1, seqlen=64, nheads=4, headdim=8, dstate=16,
                                           ngroups=2, chunk=64, io="f32", init="zeros"), seed=3)
    t = {k: torch.from_numpy(np.ascontiguousarray(inp[k][:, :32]))
         for k in ("x", "dt", "B", "C")}
    try:
        seqpar_scan_fwd(t["x"], t["dt"], torch.from_numpy(inp["A"]), t["B"], t["C"],
                        torch.from_numpy(inp["D"]), 64, ops=OracleOps())
        q.put("no error")
    except Exception as e:  # the collective fails: the peer is gone
        q.put(type(e).__name__)


def test_exchange_fails_cleanly_when_a_rank_is_gone():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dying_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    assert res != "no error", res


def _cpu_tensor_worker(port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        from mamba_ssd_scan_03_b200.seqpar import seqpar_scan_fwd
        x = torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16)
        bc = torch.zeros(1, 8, 1, 128, dtype=torch.bfloat16)
        try:
            seqpar_scan_fwd(x, torch.zeros(1, 8, 2), torch.zeros(2), bc, bc, None, 256)
            q.put("no error")
        except (ValueError, RuntimeError) as e:
            q.put(str(e))
    finally:
        dist.destroy_process_group()


def test_library_ops_refuse_host_tensors():
    """The product path has no CPU fallback: host tensors are refused by the binding."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_cpu_tensor_worker, args=(_free_port(), q))
    p.start()
    res = q.get(timeout=120)
    p.join(timeout=60)
    assert res != "no error" and "CUDA" in res, res
