"""GPU backward (lfa_backward) against the oracle's analytic gradient.

The oracle's gradient is pinned by central finite differences (tests/pins.py). Both sides
see the same seeded inputs; tolerances are the forward's: max-abs relative 1e-3 per unit
for fp32 storage, normwise 2e-2 per unit for bf16 storage, applied to dQ and dV.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from laplacian_nystr_attention_avg_b200 import lfa
from laplacian_nystr_attention_avg_b200.inputs import WORKLOADS, Workload, make_crop_inputs, make_inputs
from oracle import lfa_oracle as O
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


def _check_backward(wl: Workload, whiten: bool, units, zero_dwc: bool = False, seed: int = 0, x=None):
    if x is None:
        x = make_inputs(wl, seed=seed, with_dO=True)
    w = torch.zeros_like(x.dwc) if zero_dwc else x.dwc
    mod = lfa.LaplacianNystromAttention(lfa.make_config(wl, whiten), w, "cuda")
    Q, V, dO = x.Q_store.cuda(), x.V_store.cuda(), x.dO_store.cuda()
    mod.forward(Q, V)
    dQ, dV = mod.backward(Q, V, dO)
    torch.cuda.synchronize()
    gq, gv = O.backward(x.Q.numpy(), x.V.numpy(), w.numpy(), x.dO.numpy(), wl, whiten, units=list(units))
    bf16 = wl.dtype == "bf16"
    B, nh, N, d = gq.shape
    errs = {}
    for name, g, ref in (("dQ", dQ, gq), ("dV", dV, gv)):
        got = pu.unit_rows(g, units)
        want = ref.reshape(B * nh, N, d)[list(units)]
        errs[name] = pu.o_error(got, want, bf16)
        assert np.isfinite(got).all()
    tol = pu.o_tolerance(bf16)
    assert errs["dQ"] <= tol and errs["dV"] <= tol, f"{wl.name} whiten={whiten}: {errs} (tolerance {tol})"
    return mod, errs


CROPS = [
    # 16 x 16 grids shaped like the long-sequence workload (8 heads, d = 64, T = 24)
    Workload("crop_r16_f32", B=1, heads=8, H=16, W=16, d=64, r=16, T=24, dtype="f32", backward=True),
    Workload("crop_r4_f32", B=1, heads=8, H=16, W=16, d=64, r=4, T=24, dtype="f32", backward=True),
    Workload("crop_r4_bf16", B=1, heads=8, H=16, W=16, d=64, r=4, T=24, dtype="bf16", backward=True),
    Workload("crop_r2_f32", B=1, heads=2, H=16, W=16, d=64, r=2, T=24, dtype="f32", backward=True),
    # d = 32, ragged tiles, m > 64 (multi-chunk landmark loop), T = 0
    Workload("ragged_d32_f32", B=2, heads=1, H=12, W=12, d=32, r=4, T=20, dtype="f32", backward=True),
    Workload("m100_f32", B=1, heads=1, H=40, W=40, d=64, r=4, T=24, dtype="f32", backward=True),
    Workload("t0_f32", B=1, heads=2, H=16, W=16, d=64, r=4, T=0, dtype="f32", backward=True),
]


@pytest.mark.parametrize("wl", CROPS, ids=[w.name for w in CROPS])
@pytest.mark.parametrize("whiten", [True, False], ids=["whiten", "raw"])
def test_backward_small(wl, whiten):
    _check_backward(wl, whiten, tuple(range(wl.units)))


@pytest.mark.parametrize("r", [16, 4])
@pytest.mark.parametrize("whiten", [True, False], ids=["whiten", "raw"])
def test_backward_long_crop(r, whiten):
    # the long-sequence workload's own Q, V, dO (bf16) and DWC weight, cropped to the top-left
    # 16 x 16 tokens of all 8 heads' grids: r = 16 (one landmark) and r = 4 (16 landmarks); the
    # oracle's gradient on these same values is pinned by finite differences
    cw, x = make_crop_inputs(WORKLOADS["long"], 16, 16, r)
    _check_backward(cw, whiten, tuple(range(cw.units)), x=x)


@pytest.mark.parametrize("whiten", [True, False], ids=["whiten", "raw"])
def test_backward_long_full_size(whiten):
    # the long-sequence workload: 8 heads of a 256 x 256 grid, m = 256, bf16
    wl = pu.workload("long")
    _check_backward(wl, whiten, (0, 3, 7))


def test_backward_after_fused_forward():
    # PVT stage-1 shape: the forward takes the fused kernel; backward rebuilds the context
    wl = pu.workload("pvt1").replace(backward=True)
    mod, _ = _check_backward(wl, True, (0, 31))
    assert mod.path == "fused"


def test_backward_attn_only_and_deterministic():
    wl = CROPS[1]
    mod, _ = _check_backward(wl, True, tuple(range(wl.units)), zero_dwc=True)
    x = make_inputs(wl, with_dO=True)
    Q, V, dO = x.Q_store.cuda(), x.V_store.cuda(), x.dO_store.cuda()
    mod.forward(Q, V)
    a = [t.clone() for t in mod.backward(Q, V, dO)]
    b = mod.backward(Q, V, dO)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_backward_state_errors():
    wl = CROPS[1]
    x = make_inputs(wl, with_dO=True)
    mod = lfa.LaplacianNystromAttention(lfa.make_config(wl, True), x.dwc, "cuda")
    Q, V, dO = x.Q_store.cuda(), x.V_store.cuda(), x.dO_store.cuda()
    with pytest.raises(lfa.LfaError) as e:
        mod.backward(Q, V, dO)                   # no forward yet
    assert e.value.status == lfa.LFA_ERR_STATE
    mod.forward(Q, V)
    with pytest.raises(lfa.LfaError) as e:
        mod.backward(Q.clone(), V, dO)           # a different Q buffer
    assert e.value.status == lfa.LFA_ERR_STATE
