"""GPU parity of Reading B (cfg.whiten = LFA_WHITEN_FULL) against the oracle's reading R13: the
columns of the whole Nystrom matrix G^ = C X C^T whitened, O_attn = G~ V (LaplacianFormer note,
关键设计 1 applied to 关键设计 2's G^), in the factored form the per-stage kernels compute.

Covers the PVT stage-1 and stage-2 shapes at full size (bf16, several tiles per CTA), the HR-196
shape (m = 196: four 64-landmark blocks, the last one ragged), a small fp32 shape with a ragged tile
and d = 32, and an fp32 shape with m = 247 (not a multiple of 4) and a ragged last tile, with and
without the DWC term; the per-stage path choice; and the unsupported backward.
"""
import numpy as np
import pytest
import torch

from laplacian_nystr_attention_avg_b200 import lfa
from laplacian_nystr_attention_avg_b200.inputs import Workload
from oracle import lfa_oracle as O
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

SMALL = Workload("reading_b_small", B=3, heads=2, H=20, W=20, d=32, r=4, T=20, dtype="f32")
# 13 x 19 landmarks (m = 247) over a 52 x 76 grid: N = 3952 is 61 tiles and a 48-row tail
M247 = Workload("reading_b_m247", B=1, heads=2, H=52, W=76, d=32, r=4, lam=4.0, T=24, dtype="f32")


@pytest.mark.parametrize("wl", [pu.workload("pvt1"), pu.workload("pvt2"), SMALL, pu.workload("hr196"), M247],
                         ids=["pvt1", "pvt2", "small_f32", "hr196", "m247_f32"])
@pytest.mark.parametrize("zero_dwc", [True, False], ids=["attn_only", "with_dwc"])
def test_reading_b_forward(wl, zero_dwc):
    x = pu.inputs_for(wl)
    w = torch.zeros_like(x.dwc) if zero_dwc else x.dwc
    mod = lfa.LaplacianNystromAttention(lfa.make_config(wl, "full"), w, "cuda")
    assert mod.path == "generic"
    Og = mod.forward(x.Q_store.cuda(), x.V_store.cuda())
    torch.cuda.synchronize()
    st, _ = mod.info()
    assert st == lfa.LFA_OK
    # every unit of the smaller workloads; the first and last of HR-196 (eight units of 12544 rows)
    units = tuple(range(wl.units)) if wl.units * wl.N <= 32768 else (0, wl.units - 1)
    Oref, _, _ = O.forward_reading_b(x.Q.numpy(), x.V.numpy(), w.numpy(), wl, units)
    got = pu.unit_rows(Og, units)
    want = np.stack([Oref[divmod(u, wl.heads)] for u in units])
    bf16 = wl.dtype == "bf16"
    err = pu.o_error(got, want, bf16)
    assert err <= pu.o_tolerance(bf16), f"{wl.name}: error {err:.3e}"


def test_reading_b_backward_unsupported():
    x = pu.inputs_for(SMALL)
    mod = lfa.LaplacianNystromAttention(lfa.make_config(SMALL, "full"), x.dwc, "cuda")
    Q, V = x.Q_store.cuda(), x.V_store.cuda()
    mod.forward(Q, V)
    with pytest.raises(lfa.LfaError) as e:
        mod.backward(Q, V, torch.ones_like(Q))
    assert e.value.status == lfa.LFA_ERR_UNSUPPORTED
