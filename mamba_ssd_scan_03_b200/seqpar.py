"""Sequence-sliced chunked scan over the ranks of a torch.distributed group.

Every rank holds a contiguous slice of the same sequences (rank r: tokens [r L/R, (r+1) L/R)
or any split in rank order).  A slice's steps compose like a single step, h_out =
exp(total_decay) h_in + S ("State Space Model" (book.paithon.it), "Un sistema che riassume il
passato": steps fuse pairwise by associativity), so the only exchange is one all-gather of the
slice summaries (S, total_decay); then each rank scans its slice from its entering state
("Architektury Mamba-2, State Space Models i liniowa atencja" (tech.tersel.eu), "Wyzwania
uczenia rozproszonego": only boundary states cross between devices).

    1. (S_r, decay_r) = chunk_state_fwd(own slice, zero state)     -- seg_state + seg_pass
    2. all-gather of (S_r, decay_r) over the group                   -- NCCL on GPUs
    3. H_in = state_pass(S, decay, init_state)                       -- exclusive scan
    4. y_r = chunk_scan_fwd(own slice, init_state = H_in[r])         -- the full scan kernels

Steps 1, 3 and 4 are the library's kernels (`ops` replaces them only in host-logic tests).
A rank whose slice is empty contributes the identity step (S = 0, total decay 0) and returns
an empty y.
"""
import torch
import torch.distributed as dist


class LibraryOps:
    """The slice operations on the GPU (libssd)."""

    def state(self, x, dt, A, B, chunk):
        from . import chunk_state_fwd
        return chunk_state_fwd(x, dt, A, B, chunk)

    def identity(self, x, B):
        """The summary of an empty slice: no input (S = 0) and no decay (total 0)."""
        Bt, _, H, P = x.shape
        S = torch.zeros((Bt, H, P, B.shape[3]), dtype=torch.float32, device=x.device)
        return S, torch.zeros((Bt, H), dtype=torch.float32, device=x.device)

    def state_pass(self, states, decay, init_state):
        from . import state_pass
        return state_pass(states, decay, init_state)

    def scan(self, x, dt, A, B, C, D, chunk, init_state, y_dtype):
        from . import chunk_scan_fwd
        y, _ = chunk_scan_fwd(x, dt, A, B, C, D, chunk, init_state=init_state,
                              want_final=False, y_dtype=y_dtype)
        return y


def seqpar_scan_fwd(x, dt, A, B, C, D, chunk, init_state=None, group=None, ops=None,
                    y_dtype=torch.float32):
    """This rank's slice: x [B,L_r,H,P], dt [B,L_r,H], B/C [B,L_r,G,N]; A, D [H]; init_state
    [B,H,P,N] (the state before the first slice, the same on every rank) or None.  Returns
    (y of the slice, state after the last slice) — the latter on every rank."""
    ops = LibraryOps() if ops is None else ops
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    empty = x.shape[1] == 0
    S, decay = ops.identity(x, B) if empty else ops.state(x, dt, A, B, chunk)
    all_s = [torch.empty_like(S) for _ in range(world)]
    all_d = [torch.empty_like(decay) for _ in range(world)]
    dist.all_gather(all_s, S.contiguous(), group=group)
    dist.all_gather(all_d, decay.contiguous(), group=group)
    states = torch.stack(all_s)
    decays = torch.stack(all_d)
    final = ops.state_pass(states, decays, init_state)
    if empty:
        return torch.empty(x.shape, dtype=y_dtype, device=x.device), final
    y = ops.scan(x, dt, A, B, C, D, chunk, states[rank].contiguous(), y_dtype)
    return y, final
