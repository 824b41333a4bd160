"""Host logic of the multi-GPU benchmark path on CPU: two gloo ranks.

bench.py under torchrun runs the full batch on every rank (independent (batch, head) units, no
data-path collective; weak scaling) and reports the step time as the maximum over ranks. These
tests run the same helpers in two processes on the gloo backend.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r timed (r + 1) ms for the loop and (10 - r) ms end to end
        total, e2e = bench.max_over_ranks([rank + 1.0, 10.0 - rank], world)
        out[rank] = (total, e2e)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert dict(out) == {0: (2.0, 10.0), 1: (2.0, 10.0)}


def test_single_rank_is_identity():
    assert bench.max_over_ranks([3.5, 1.25], 1) == [3.5, 1.25]


def test_job_throughput_counts_every_rank():
    # 4 ranks, each 32 units of 3136 tokens per step, 100 steps in 10 ms (max over ranks)
    assert bench.job_tokens_per_s(4, 32, 3136, 100, 10.0) == pytest.approx(4 * 32 * 3136 * 100 / 0.01)


def test_ranks_draw_independent_inputs():
    # weak scaling: rank r seeds its synthetic batch with r, so ranks process different units
    from laplacian_nystr_attention_avg_b200.inputs import WORKLOADS, make_inputs
    wl = WORKLOADS["pr1"]
    a, b = make_inputs(wl, seed=0), make_inputs(wl, seed=1)
    assert not torch.equal(a.Q, b.Q)
