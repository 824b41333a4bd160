"""The sequence-split driver (laplacian_nystr_attention_avg_b200.seqsplit) over real ranks is exact.

Four gloo ranks on the CPU run seqsplit.forward_rank with TorchComm, the exchanges the GPU ranks use
over NCCL (all-reduce of the landmark shares and of the pass-1 partials, neighbour send/receive of
the V halo rows), around band computations written here from the oracle's building blocks (the
library needs a GPU). Bands of uneven height that do not align with the pooling windows are used on
purpose: a landmark window shared by two ranks is summed across them. The assembled O must equal the
single-rank oracle forward (reading A) to rounding.
"""
from __future__ import annotations

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

H, W, D, R, LAM, EPS, T = 18, 15, 8, 3, 2.0, 1e-6, 20
WORLD = 4


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


class OracleBand:
    """pool / pass1 / pass2 of one band (grid rows [y0, y0 + ny)) in float64 from oracle pieces;
    tensors are [1, 1, rows, D] like the library's [B, heads, rows, d]."""

    def __init__(self, y0, ny, w):
        self.y0, self.ny, self.w = y0, ny, w

    def pool(self, Q):
        q = Q[0, 0].numpy()
        Wr = W // R
        L = np.zeros(((H // R) * Wr, D))
        for l in range(L.shape[0]):
            Y0, X0 = (l // Wr) * R, (l % Wr) * R
            for dy in range(R):
                yl = Y0 + dy - self.y0
                if 0 <= yl < self.ny:
                    L[l] += q[yl * W + X0:yl * W + X0 + R].sum(0)
        return torch.from_numpy(L / (R * R))[None, None]

    def pass1(self, Q, V, L):
        from oracle import lfa_oracle as O
        q, v, Lf = Q[0, 0].numpy(), V[0, 0].numpy(), L[0, 0].numpy()
        C = O.laplacian_kernel(q, Lf, LAM)
        self.C, self.L = C, Lf
        return torch.from_numpy(np.concatenate([C.sum(0), (C ** 2).sum(0), (C.T @ v).ravel(), v.sum(0)]))[None, None]

    def pass2(self, Q, V, halo, part, Out):
        from oracle import lfa_oracle as O
        m, N = self.L.shape[0], H * W
        pt = part[0, 0].numpy()
        S1, S2 = pt[:m], pt[m:2 * m]
        P = pt[2 * m:2 * m + m * D].reshape(m, D)
        SV = pt[2 * m + m * D:]
        Wm = O.landmark_gram(self.L, LAM, EPS)
        X, _, _ = O.newton_schulz(Wm, O.select_alpha(Wm).alpha, T)
        mu = S1 / N
        s = 1.0 / np.sqrt(S2 / N - mu ** 2 + EPS)
        A = s[:, None] * (P - np.outer(mu, SV)) + SV[None, :] / N     # C~^T V by rank-1 folding
        Ct = (self.C - mu) * s + 1.0 / N
        ext = np.concatenate([halo[0, 0, 0].numpy(), V[0, 0].numpy(), halo[0, 0, 1].numpy()])
        dwc = O.dwc3x3(ext, self.w, self.ny + 2, W)[W:-W]
        Out[0, 0] = torch.from_numpy(Ct @ (X @ A) + dwc)
        return Out


def _worker(rank: int, world: int, port: int, out):
    from laplacian_nystr_attention_avg_b200 import seqsplit

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, v, w = _inputs()
        y0, ny = seqsplit.band_rows(H, world, rank)
        sl = slice(y0 * W, (y0 + ny) * W)
        Q = torch.from_numpy(q[sl].copy())[None, None]
        V = torch.from_numpy(v[sl].copy())[None, None]
        Ob = torch.zeros_like(Q)
        seqsplit.forward_rank(OracleBand(y0, ny, w), Q, V, Ob, seqsplit.TorchComm(rank, world), W)
        out[rank] = Ob[0, 0].numpy()
    finally:
        dist.destroy_process_group()


def test_sequence_split_driver_over_four_ranks_is_exact():
    from oracle import lfa_oracle as O

    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(WORLD, _free_port(), out), nprocs=WORLD, start_method="spawn", join=True)
    got = np.concatenate([out[k] for k in range(WORLD)])
    q, v, w = _inputs()
    ref = O.unit_forward(q, v, w, H, W, R, LAM, EPS, T).O
    assert np.allclose(got, ref, rtol=0, atol=1e-12 * np.abs(ref).max())


def test_band_rows_cover_the_grid():
    from laplacian_nystr_attention_avg_b200 import seqsplit
    for Hh in (1, 7, 18, 256):
        for world in (1, 2, 3, 8):
            if world > Hh:
                continue
            rows = [seqsplit.band_rows(Hh, world, k) for k in range(world)]
            assert rows[0][0] == 0 and sum(n for _, n in rows) == Hh
            assert all(rows[k][0] + rows[k][1] == rows[k + 1][0] for k in range(world - 1))
            assert max(n for _, n in rows) - min(n for _, n in rows) <= 1
