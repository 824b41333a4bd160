"""GPU parity of the batch-pooled whitening statistics (cfg.whiten = LFA_WHITEN_BATCH) against the
oracle's reading R12: the column mean and variance of each head pooled over the B*N rows of all
batch elements (LaplacianFormer note, 关键设计 1, statistics over a batch of similarity vectors).

Covers the heavy-tailed PVT stage-2 shape at full size (32 batch elements per head), a small fp32
shape with a ragged tile and d = 32, the pooled statistics themselves, the reduction to the
per-unit statistics at B = 1 (bit for bit on the GPU), the per-stage path choice, and the backward
(pooled whitening reverse mode) at three shapes and its reduction to the per-unit one at B = 1.
"""
import numpy as np
import pytest
import torch

from laplacian_nystr_attention_avg_b200 import lfa
from laplacian_nystr_attention_avg_b200.inputs import Workload, make_inputs
from oracle import lfa_oracle as O
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

SMALL = Workload("batch_small", B=3, heads=2, H=20, W=20, d=32, r=4, T=20, dtype="f32")


def _run(wl, zero_dwc=False):
    x = pu.inputs_for(wl)
    w = torch.zeros_like(x.dwc) if zero_dwc else x.dwc
    mod = lfa.LaplacianNystromAttention(lfa.make_config(wl, "batch"), w, "cuda")
    Og = mod.forward(x.Q_store.cuda(), x.V_store.cuda())
    torch.cuda.synchronize()
    st, _ = mod.info()
    ref = O.forward(x.Q.numpy(), x.V.numpy(), w.numpy(), wl, batch_stats=True)
    return mod, x, Og, st, ref


@pytest.mark.parametrize("wl", [pu.workload("pvt2"), SMALL], ids=["pvt2", "small_f32"])
@pytest.mark.parametrize("zero_dwc", [True, False], ids=["attn_only", "with_dwc"])
def test_batch_stats_forward(wl, zero_dwc):
    mod, x, Og, st, ref = _run(wl, zero_dwc)
    assert st == lfa.LFA_OK
    assert mod.path == "generic"
    units = tuple(range(wl.units))
    got = pu.unit_rows(Og, units)
    want = np.stack([ref.O[divmod(u, wl.heads)] for u in units])
    bf16 = wl.dtype == "bf16"
    err = pu.o_error(got, want, bf16)
    assert err <= pu.o_tolerance(bf16), f"{wl.name}: error {err:.3e}"


def test_batch_stats_pooled_statistics():
    mod, x, Og, st, ref = _run(SMALL)
    for u in range(SMALL.units):
        _, _, mu, s = (t.cpu().numpy().astype(np.float64) for t in mod.context(u))
        f = ref.units[u]
        np.testing.assert_allclose(mu, f.mu, rtol=1e-4)
        np.testing.assert_allclose(s, 1.0 / np.sqrt(f.var + SMALL.eps), rtol=1e-4)
    # units of one head share them; the two heads differ
    mu = [mod.context(u)[2].cpu() for u in range(SMALL.units)]
    for b in range(1, SMALL.B):
        for h in range(SMALL.heads):
            assert torch.equal(mu[b * SMALL.heads + h], mu[h])
    assert not torch.equal(mu[0], mu[1])


def test_batch_stats_single_batch_is_per_unit():
    wl = pu.workload("pr1")   # B = 1: the pooled sums are the unit's own, divided by 1
    x = pu.inputs_for(wl)
    outs = []
    for whiten in (True, "batch"):
        mod = lfa.LaplacianNystromAttention(lfa.make_config(wl, whiten), x.dwc, "cuda")
        assert mod.path == "generic"
        outs.append(mod.forward(x.Q_store.cuda(), x.V_store.cuda()))
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])


BWD = [SMALL.replace(backward=True),
       Workload("batch_bwd_bf16", B=4, heads=2, H=16, W=16, d=64, r=4, T=24, dtype="bf16", backward=True)]


@pytest.mark.parametrize("wl", BWD + [pu.workload("pvt2").replace(backward=True)],
                         ids=[w.name for w in BWD] + ["pvt2"])
def test_batch_stats_backward(wl):
    # the reverse mode of the pooled whitening (the oracle's R12 gradient, pinned by finite
    # differences): the column means of dC~ and dC~ o C^ over each head's B N rows
    x = make_inputs(wl, with_dO=True)
    mod = lfa.LaplacianNystromAttention(lfa.make_config(wl, "batch"), x.dwc, "cuda")
    Q, V, dO = x.Q_store.cuda(), x.V_store.cuda(), x.dO_store.cuda()
    mod.forward(Q, V)
    dQ, dV = mod.backward(Q, V, dO)
    torch.cuda.synchronize()
    gq, gv = O.backward(x.Q.numpy(), x.V.numpy(), x.dwc.numpy(), x.dO.numpy(), wl, True, batch_stats=True)
    bf16 = wl.dtype == "bf16"
    units = tuple(range(wl.units))
    for name, g, ref in (("dQ", dQ, gq), ("dV", dV, gv)):
        got = pu.unit_rows(g, units)
        want = ref.reshape(wl.units, wl.N, wl.d)
        assert np.isfinite(got).all()
        err = pu.o_error(got, want, bf16)
        assert err <= pu.o_tolerance(bf16), f"{wl.name} {name}: error {err:.3e}"


def test_batch_stats_backward_single_batch_is_per_unit():
    wl = pu.workload("pr1").replace(backward=True)   # B = 1: the pooled coefficients are the unit's own
    x = make_inputs(wl, with_dO=True)
    Q, V, dO = x.Q_store.cuda(), x.V_store.cuda(), x.dO_store.cuda()
    grads = []
    for whiten in (True, "batch"):
        mod = lfa.LaplacianNystromAttention(lfa.make_config(wl, whiten), x.dwc, "cuda")
        mod.forward(Q, V)
        grads.append([t.clone() for t in mod.backward(Q, V, dO)])
    torch.cuda.synchronize()
    assert torch.equal(grads[0][0], grads[1][0]) and torch.equal(grads[0][1], grads[1][1])
