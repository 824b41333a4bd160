"""The exchange set of a sequence split (one (batch, head) unit's tokens over two ranks) is exact.

Splitting one unit's N tokens across ranks by whole grid rows (a multiple of the pooling window r)
needs, per the design of the multi-GPU path:
  1. an all-gather of the landmarks (each rank pools the windows in its rows),
  2. an all-reduce of the pass-1 partials (column sums of C and C^2, C^T V, sum of V),
  3. a one-grid-row halo of V from each neighbour for the 3 x 3 DWC,
after which every rank forms W, X and the combine redundantly and writes its own rows of O.
This runs that decomposition with two gloo ranks on the CPU, using the oracle's building blocks
for the local arithmetic, and checks it against the single-rank oracle forward (reading A).
The library has no sequence-split path; this pins the exchange set it would implement.
"""
from __future__ import annotations

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

H, W, D, R, LAM, EPS, T = 16, 16, 8, 4, 2.0, 1e-6, 20


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((H * W, D))
    v = rng.standard_normal((H * W, D))
    w = rng.standard_normal((D, 3, 3)) * 0.1
    return q, v, w


def _worker(rank: int, world: int, port: int, out):
    from oracle import lfa_oracle as O

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, v, w = _inputs()
        rows = H // world                       # grid rows per rank, a multiple of R
        lo, hi = rank * rows * W, (rank + 1) * rows * W
        qk, vk = q[lo:hi], v[lo:hi]
        # 1. landmarks of this rank's windows, all-gathered in landmark (row-major) order
        Lk = torch.from_numpy(O.pool_landmarks(qk, rows, W, R))
        parts = [torch.empty_like(Lk) for _ in range(world)]
        dist.all_gather(parts, Lk)
        L = torch.cat(parts).numpy()
        # W, alpha and X on every rank
        Wm = O.landmark_gram(L, LAM, EPS)
        X, _, _ = O.newton_schulz(Wm, O.select_alpha(Wm).alpha, T)
        # 2. pass-1 partials, all-reduced
        Ck = O.laplacian_kernel(qk, L, LAM)
        part = torch.from_numpy(np.concatenate([Ck.sum(0), (Ck ** 2).sum(0), (Ck.T @ vk).ravel(), vk.sum(0)]))
        dist.all_reduce(part)
        m, N = L.shape[0], H * W
        S1, S2 = part[:m].numpy(), part[m:2 * m].numpy()
        P = part[2 * m:2 * m + m * D].numpy().reshape(m, D)
        SV = part[2 * m + m * D:].numpy()
        mu = S1 / N
        var = S2 / N - mu ** 2
        s = 1.0 / np.sqrt(var + EPS)
        A = s[:, None] * (P - np.outer(mu, SV)) + SV[None, :] / N     # C~^T V by rank-1 folding
        M = X @ A
        Ct = (Ck - mu) * s + 1.0 / N
        # 3. one grid row of V from each neighbour (zeros past the grid's edge)
        up = torch.from_numpy(vk[:W].copy())
        down = torch.from_numpy(vk[-W:].copy())
        above, below = torch.zeros_like(up), torch.zeros_like(down)
        reqs = []
        if rank > 0:
            reqs += [dist.isend(up, rank - 1), dist.irecv(above, rank - 1)]
        if rank < world - 1:
            reqs += [dist.isend(down, rank + 1), dist.irecv(below, rank + 1)]
        for r in reqs:
            r.wait()
        # rows + 2 halo rows; at the grid's top and bottom edges the halo stays zero (zero padding)
        ext = np.concatenate([above.numpy(), vk, below.numpy()])
        dwc = O.dwc3x3(ext, w, rows + 2, W)[W:-W]
        out[rank] = Ct @ M + dwc
    finally:
        dist.destroy_process_group()


def test_sequence_split_over_two_ranks_is_exact():
    from oracle import lfa_oracle as O

    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    got = np.concatenate([out[k] for k in range(world)])
    q, v, w = _inputs()
    ref = O.unit_forward(q, v, w, H, W, R, LAM, EPS, T).O
    assert np.allclose(got, ref, rtol=0, atol=1e-12 * np.abs(ref).max())
