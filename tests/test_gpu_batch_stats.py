"""GPU parity of the batch-pooled whitening statistics (cfg.whiten = LFA_WHITEN_BATCH) against the
oracle's reading R12: the column mean and variance of each head pooled over the B*N rows of all
batch elements (LaplacianFormer note, 关键设计 1, statistics over a batch of similarity vectors).

Covers the heavy-tailed PVT stage-2 shape at full size (32 batch elements per head), a small fp32
shape with a ragged tile and d = 32, the pooled statistics themselves, the reduction to the
per-unit statistics at B = 1 (bit for bit on the GPU), the per-stage path choice and the
unsupported backward.
"""
import numpy as np
import pytest
import torch

from laplacian_nystr_attention_avg_b200 import lfa
from laplacian_nystr_attention_avg_b200.inputs import Workload
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


def test_batch_stats_backward_unsupported():
    wl = SMALL
    x = pu.inputs_for(wl)
    mod = lfa.LaplacianNystromAttention(lfa.make_config(wl, "batch"), x.dwc, "cuda")
    Q, V = x.Q_store.cuda(), x.V_store.cuda()
    mod.forward(Q, V)
    with pytest.raises(lfa.LfaError) as e:
        mod.backward(Q, V, torch.ones_like(Q))
    assert e.value.status == lfa.LFA_ERR_UNSUPPORTED
