"""Sequence split of Laplacian-kernel Nystrom attention over several devices (bands of grid rows).

One (batch, head) unit's N = H W tokens are cut into bands of whole grid rows, one per rank; every
rank holds the Q, V and O rows of its band for all units. One forward is three exchanges between
the library's band calls (lfa_sp_pool, lfa_sp_pass1, lfa_sp_pass2 in include/lfa.h):
  1. all-reduce (sum) of the landmark shares: every rank then has the full landmarks L;
  2. all-reduce (sum, fp64) of the pass-1 partials: column sums of C and C^2, C^T V, sum V;
  3. the V rows just outside the band from the neighbouring ranks (one grid row each way) for DWC.
W, alpha, the Newton-Schulz chain and the combine are computed redundantly on every rank; each rank
writes its own rows of O. The messages are small (m d + 2 m + m d + d values per unit, one grid row
of V), so this split costs a few latency-bound collectives per call.

This module only sequences calls and exchanges: the arithmetic runs in the library's kernels. The
`compute` object it drives has pool / pass1 / pass2 methods (lfa.SeqSplitBand, or any object with
the same methods) and `comm` provides all_reduce_sum and the halo exchange.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple


def band_rows(H: int, world: int, rank: int) -> Tuple[int, int]:
    """(y0, ny): rank's band of the H grid rows, as even as possible (the first H % world ranks
    take one row more)."""
    base, extra = divmod(H, world)
    y0 = rank * base + min(rank, extra)
    return y0, base + (1 if rank < extra else 0)


def edge_rows(V, W: int):
    """(first grid row, last grid row) of a band's V, each [B, heads, W, d]."""
    return V[:, :, :W, :], V[:, :, V.shape[2] - W:, :]


class TorchComm:
    """Exchanges over torch.distributed (NCCL or gloo): one band per rank, bands in rank order."""

    def __init__(self, rank: int, world: int):
        self.rank, self.world = rank, world

    def all_reduce_sum(self, t):
        import torch.distributed as dist
        if self.world > 1:
            dist.all_reduce(t, op=dist.ReduceOp.SUM)
        return t

    def halo(self, V, W: int):
        """[B, heads, 2, W, d]: V row y0 - 1 from the rank above, row y0 + ny from the rank below
        (zeros at the grid's edges, where the library does not read them)."""
        import torch
        import torch.distributed as dist
        B, nh, _, d = V.shape
        out = torch.zeros((B, nh, 2, W, d), dtype=V.dtype, device=V.device)
        if self.world == 1:
            return out
        first, last = (x.contiguous() for x in edge_rows(V, W))
        top = torch.empty_like(first)
        bottom = torch.empty_like(first)
        ops = []
        if self.rank > 0:
            ops.append(dist.P2POp(dist.isend, first, self.rank - 1))
            ops.append(dist.P2POp(dist.irecv, top, self.rank - 1))
        if self.rank < self.world - 1:
            ops.append(dist.P2POp(dist.isend, last, self.rank + 1))
            ops.append(dist.P2POp(dist.irecv, bottom, self.rank + 1))
        for r in dist.batch_isend_irecv(ops):
            r.wait()
        if self.rank > 0:
            out[:, :, 0] = top
        if self.rank < self.world - 1:
            out[:, :, 1] = bottom
        return out


def forward_rank(compute, Q, V, O, comm, W: int):
    """One forward of this rank's band: pool, all-reduce, pass 1, all-reduce, halo, pass 2."""
    L = comm.all_reduce_sum(compute.pool(Q))
    part = comm.all_reduce_sum(compute.pass1(Q, V, L))
    compute.pass2(Q, V, comm.halo(V, W), part, O)
    return O


def forward_bands(computes: Sequence, Qs: Sequence, Vs: Sequence, Os: Sequence, W: int) -> List:
    """All bands in one process (the same exchanges, done as sums and slices): for one device that
    emulates the ranks, or for tests."""
    import torch
    L = computes[0].pool(Qs[0]).clone()
    for c, Q in zip(computes[1:], Qs[1:]):
        L += c.pool(Q)
    part = computes[0].pass1(Qs[0], Vs[0], L).clone()
    for c, Q, V in zip(computes[1:], Qs[1:], Vs[1:]):
        part += c.pass1(Q, V, L)
    n = len(computes)
    for k in range(n):
        B, nh, _, d = Vs[k].shape
        halo = torch.zeros((B, nh, 2, W, d), dtype=Vs[k].dtype, device=Vs[k].device)
        if k > 0:
            halo[:, :, 0] = edge_rows(Vs[k - 1], W)[1]
        if k < n - 1:
            halo[:, :, 1] = edge_rows(Vs[k + 1], W)[0]
        computes[k].pass2(Qs[k], Vs[k], halo, part, Os[k])
    return list(Os)
