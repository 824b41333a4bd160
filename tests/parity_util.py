"""Shared helpers of the GPU parity tests: run the library and the oracle on the same inputs.

Tolerances (all per (batch, head) unit):
  * C, fp32 arithmetic: max |C_gpu - C| / C over entries with C >= 2^-126, and
    |C_gpu| <= 2^-126 where C underflows; bound 1e-4 (scaled by 4/lambda below lambda = 4,
    since the fp32 rounding of the distance sum enters C as D_err / lambda).
  * O, fp32 storage: max |O_gpu - O| / max |O| <= 1e-3, for O_attn (zero DWC weight) and O.
  * O, bf16 storage: ||O_gpu - O||_F / ||O||_F <= 2e-2, for O_attn and O.
"""
from __future__ import annotations

import functools
import os

import numpy as np
import torch

from laplacian_nystr_attention_avg_b200 import lfa
from laplacian_nystr_attention_avg_b200.inputs import WORKLOADS, Workload, make_inputs
from oracle import lfa_oracle as O

O.set_threads(os.cpu_count() or 8)

TINY = 2.0 ** -126


def c_tolerance(lam: float) -> float:
    return 1e-4 * max(1.0, 4.0 / lam)


def c_error(Cg: np.ndarray, Co: np.ndarray) -> float:
    big = Co >= TINY
    err = 0.0
    if big.any():
        err = float(np.max(np.abs(Cg[big] - Co[big]) / Co[big]))
    if (~big).any() and np.max(np.abs(Cg[~big])) > TINY:
        return float("inf")
    return err


def o_error(Og: np.ndarray, Oo: np.ndarray, bf16: bool) -> float:
    """Per-unit error, worst over units: Og, Oo are [U, N, d].

    A unit whose exact output lies entirely below the fp32 normal range (possible
    only when every C entry underflows, e.g. lambda = 0.25 without whitening) is
    compared absolutely: the fp32 result must be below 2^-126 as well.
    """
    worst = 0.0
    for u in range(Oo.shape[0]):
        a, b = Og[u].astype(np.float64), Oo[u]
        if np.max(np.abs(b)) < TINY:
            if np.max(np.abs(a)) > TINY:
                return float("inf")
            continue
        if bf16:
            e = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)
        else:
            e = np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)
        worst = max(worst, float(e))
    return worst


def o_tolerance(bf16: bool) -> float:
    return 2e-2 if bf16 else 1e-3


@functools.lru_cache(maxsize=8)
def inputs_for(wl: Workload, seed: int = 0):
    return make_inputs(wl, seed=seed)


@functools.lru_cache(maxsize=32)
def oracle_forward(wl: Workload, whiten: bool, zero_dwc: bool, units: tuple, seed: int = 0):
    x = inputs_for(wl, seed)
    w = np.zeros(x.dwc.shape) if zero_dwc else x.dwc.numpy()
    return O.forward(x.Q.numpy(), x.V.numpy(), w, wl, whiten=whiten, units=list(units))


def gpu_module(wl: Workload, whiten: bool, zero_dwc: bool, seed: int = 0):
    x = inputs_for(wl, seed)
    w = torch.zeros_like(x.dwc) if zero_dwc else x.dwc
    return lfa.LaplacianNystromAttention(lfa.make_config(wl, whiten), w, "cuda")


def run_gpu_forward(wl: Workload, whiten: bool, zero_dwc: bool, seed: int = 0):
    x = inputs_for(wl, seed)
    mod = gpu_module(wl, whiten, zero_dwc, seed)
    Q = x.Q_store.cuda()
    V = x.V_store.cuda()
    Og = mod.forward(Q, V)
    torch.cuda.synchronize()
    st, info = mod.info()
    return mod, Q, V, Og, st, info


def unit_rows(t: torch.Tensor, units) -> np.ndarray:
    """[B, heads, N, d] tensor -> float64 [len(units), N, d] for the listed flat units."""
    B, nh, N, d = t.shape
    flat = t.reshape(B * nh, N, d)
    return np.stack([flat[u].float().cpu().numpy() for u in units]).astype(np.float64)


def workload(name: str, **kw) -> Workload:
    wl = WORKLOADS[name]
    return wl.replace(**kw) if kw else wl
