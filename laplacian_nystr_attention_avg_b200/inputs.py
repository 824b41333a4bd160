"""Seeded synthetic workloads for Laplacian-kernel Nystrom attention.

This module only draws random numbers and names shapes. It holds none of the
method's arithmetic, so both the CUDA path's tests/benchmark and the CPU oracle
can take their inputs from here without sharing any computation.

Shapes follow the PVT-style stage shapes the attention block is used with
(LaplacianFormer note, §方法详解 / 整体框架: a PVT backbone whose query tensor
is reshaped into a spatial map and average-pooled into landmarks). There is no
public dataset on this path; these synthetic tensors stand in for activations.

Recipe (fixed, so every consumer sees identical bytes):
  * ``torch.Generator('cpu').manual_seed(seed)``; all draws are float32.
  * Draw order: Q, then V, then the depthwise-conv weight, then dO.
  * Q, V, dO have shape [B, heads, N, d] with token n = y*W + x (row-major grid).
  * Q ~ N(0, 1), or for the heavy-tailed workload a Student-t with nu = 3
    scaled to unit variance: t = z / sqrt(chi2_3 / 3) / sqrt(3), where
    chi2_3 is the sum of three squared N(0, 1) draws (z first, then the three
    chi-square components, each a full [B, heads, N, d] draw).
  * V ~ N(0, 1); dO ~ N(0, 1); DWC weight = 0.1 * N(0, 1), shape [heads, d, 3, 3].
  * bf16 workloads round Q, V and dO to bfloat16 (round-to-nearest-even) once;
    every consumer reads those rounded values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and hyper-parameters of one attention call.

    B, heads: independent (batch, head) units. H x W: token grid (N = H*W).
    d: channels per head. r: landmark pooling window (m = (H/r)*(W/r)).
    lam: Laplacian kernel scale lambda. eps: the regulariser added to W and
    inside the whitening square root. T: Newton-Schulz steps. dtype: 'f32' or
    'bf16' (storage type of Q, V, O; the library's arithmetic is set by the path, not by
    this field). qdist: 'normal' or
    'student_t3'. backward: whether the workload includes lfa_backward.
    """

    name: str
    B: int
    heads: int
    H: int
    W: int
    d: int
    r: int
    lam: float = 4.0
    eps: float = 1e-6
    T: int = 20
    dtype: str = "bf16"
    qdist: str = "normal"
    backward: bool = False

    @property
    def N(self) -> int:
        return self.H * self.W

    @property
    def m(self) -> int:
        return (self.H // self.r) * (self.W // self.r)

    @property
    def units(self) -> int:
        return self.B * self.heads

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads the path is specified on (plus the HR split into its two
# pooling choices). "pvt1" is the headline benchmark shape.
WORKLOADS: Dict[str, Workload] = {
    "pr1": Workload("pr1", B=1, heads=1, H=16, W=16, d=32, r=4, T=20, dtype="f32"),
    "pvt1": Workload("pvt1", B=32, heads=1, H=56, W=56, d=64, r=8, T=20),
    "pvt2": Workload("pvt2", B=32, heads=2, H=28, W=28, d=64, r=4, T=20, qdist="student_t3"),
    "hr49": Workload("hr49", B=4, heads=2, H=112, W=112, d=64, r=16, T=24),
    "hr196": Workload("hr196", B=4, heads=2, H=112, W=112, d=64, r=8, T=24),
    "long": Workload("long", B=1, heads=8, H=256, W=256, d=64, r=16, T=24, backward=True),
}

# lambda values swept on the heavy-tailed workload
PVT2_LAMBDA_SWEEP = (0.5, 1.0, 2.0, 4.0, 8.0)


@dataclasses.dataclass
class Inputs:
    """Host tensors of one workload (CPU, contiguous).

    Q, V, dO are float32 tensors holding the exact values the path consumes
    (already bf16-rounded for bf16 workloads); ``Q_store``/``V_store``/
    ``dO_store`` are the same values in the storage dtype handed to the
    library. ``dwc`` is float32 [heads, d, 3, 3].
    """

    wl: Workload
    Q: torch.Tensor
    V: torch.Tensor
    dwc: torch.Tensor
    dO: Optional[torch.Tensor]
    Q_store: torch.Tensor
    V_store: torch.Tensor
    dO_store: Optional[torch.Tensor]


def storage_dtype(wl: Workload) -> torch.dtype:
    return torch.bfloat16 if wl.dtype == "bf16" else torch.float32


def _draw_q(wl: Workload, g: torch.Generator, shape) -> torch.Tensor:
    if wl.qdist == "normal":
        return torch.randn(shape, generator=g, dtype=torch.float32)
    if wl.qdist == "student_t3":
        z = torch.randn(shape, generator=g, dtype=torch.float32)
        chi2 = torch.zeros(shape, dtype=torch.float32)
        for _ in range(3):
            c = torch.randn(shape, generator=g, dtype=torch.float32)
            chi2 += c * c
        return z / torch.sqrt(chi2 / 3.0) / math.sqrt(3.0)
    raise ValueError(f"unknown qdist {wl.qdist!r}")


def make_inputs(wl: Workload, seed: int = 0, with_dO: Optional[bool] = None) -> Inputs:
    """Draw the workload's inputs on the host, following the module recipe."""
    if with_dO is None:
        with_dO = wl.backward
    g = torch.Generator("cpu").manual_seed(seed)
    shape = (wl.B, wl.heads, wl.N, wl.d)
    Q = _draw_q(wl, g, shape)
    V = torch.randn(shape, generator=g, dtype=torch.float32)
    dwc = 0.1 * torch.randn((wl.heads, wl.d, 3, 3), generator=g, dtype=torch.float32)
    dO = torch.randn(shape, generator=g, dtype=torch.float32) if with_dO else None
    sd = storage_dtype(wl)
    Qs, Vs = Q.to(sd).contiguous(), V.to(sd).contiguous()
    dOs = dO.to(sd).contiguous() if dO is not None else None
    return Inputs(
        wl=wl,
        Q=Qs.float(),
        V=Vs.float(),
        dwc=dwc.contiguous(),
        dO=dOs.float() if dOs is not None else None,
        Q_store=Qs,
        V_store=Vs,
        dO_store=dOs,
    )


def crop_grid(x: torch.Tensor, H: int, W: int, h: int, w: int) -> torch.Tensor:
    """Top-left h x w crop of a [B, heads, H*W, d] token tensor (row-major grid)."""
    B, nh, N, d = x.shape
    assert N == H * W
    return x.reshape(B, nh, H, W, d)[:, :, :h, :w, :].reshape(B, nh, h * w, d).contiguous()


def make_crop_inputs(wl: Workload, h: int, w: int, r: int, seed: int = 0, name: Optional[str] = None):
    """A workload's own inputs cut down to the top-left h x w tokens of every (batch, head) grid.

    Draws the full workload's tensors with ``make_inputs`` (so the values are the workload's own,
    not a fresh draw), crops Q, V and dO with ``crop_grid`` and keeps the DWC weight. Returns the
    crop's Workload (same B, heads, d, lambda, eps, T, dtype; grid h x w; pooling window r) and
    its Inputs.
    """
    full = make_inputs(wl, seed=seed, with_dO=True)
    cw = wl.replace(name=name or f"{wl.name}_crop{h}x{w}_r{r}", H=h, W=w, r=r, backward=True)

    def crop(t):
        return crop_grid(t, wl.H, wl.W, h, w)

    return cw, Inputs(wl=cw, Q=crop(full.Q), V=crop(full.V), dwc=full.dwc, dO=crop(full.dO),
                      Q_store=crop(full.Q_store), V_store=crop(full.V_store), dO_store=crop(full.dO_store))


def make_spd_systems(m: int, kappa: float, U: int, nrhs: int, seed: int = 0):
    """U symmetric positive-definite m x m matrices with eigenvalues spaced geometrically from 1 to
    kappa (random orthogonal eigenvectors) and standard normal right-hand sides [U, m, nrhs]:
    float64 numpy arrays (the solver comparison's synthetic systems)."""
    rng = np.random.default_rng(seed)
    W = np.empty((U, m, m))
    for u in range(U):
        Qm, _ = np.linalg.qr(rng.standard_normal((m, m)))
        W[u] = (Qm * np.geomspace(1.0, kappa, m)) @ Qm.T
    B = rng.standard_normal((U, m, nrhs))
    return W, B

