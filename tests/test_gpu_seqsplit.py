"""The sequence-split band calls (lfa_sp_*), all bands emulated on one device, against the whole-grid
forward and the oracle.

laplacian_nystr_attention_avg_b200.seqsplit.forward_bands runs the same three exchanges as the
multi-rank driver (sums of the landmark shares and of the fp64 pass-1 partials, neighbouring V rows
as the DWC halo) in one process. The assembled O must match the per-stage whole-grid forward and the oracle
within the forward tolerances (1e-3 max-relative for fp32, 2e-2 normwise for bf16). Against the
whole-grid forward:
  * fp32 tokens (CUDA-core passes): only the order of the sums differs, max |diff| / max |O| <= 1e-5
    per unit;
  * bf16 tokens with d = 64 (tensor-core passes): pass 1 multiplies bf16(C - c), c the column mean of
    C over each thread block's first tile, so the band split (other blocks, other c) changes the
    rounding. Unwhitened, that rounding is relative to C - c, far below the mean part of C that
    dominates O: max |diff| / max |O| <= 2^-8 (one bf16 rounding of the result). Whitened, O keeps
    only the centred part, of the size of C - c, so each side carries the bf16 unit roundoff 2^-8 of
    its products: normwise |diff| / |O| <= 2 x 2^-8 = 2^-7 per unit.
"""
import numpy as np
import pytest
import torch

from laplacian_nystr_attention_avg_b200 import lfa, seqsplit
from laplacian_nystr_attention_avg_b200.inputs import Workload
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

CASES = [
    (Workload("sp_f32", B=2, heads=1, H=24, W=20, d=32, r=4, T=20, dtype="f32"), 3),
    (Workload("sp_bf16", B=2, heads=2, H=28, W=28, d=64, r=4, T=20, qdist="student_t3"), 4),
    (pu.workload("pvt1").replace(B=4), 2),
    (pu.workload("long"), 4),
]


def _bands(wl, nb, x, whiten):
    cfg = lfa.make_config(wl, whiten)
    bands, Qs, Vs, Os = [], [], [], []
    for k in range(nb):
        y0, ny = seqsplit.band_rows(wl.H, nb, k)
        band = lfa.SeqSplitBand(cfg, y0, ny, x.dwc, "cuda")
        sl = slice(y0 * wl.W, (y0 + ny) * wl.W)
        Qs.append(x.Q_store[:, :, sl].contiguous().cuda())
        Vs.append(x.V_store[:, :, sl].contiguous().cuda())
        Os.append(torch.empty_like(Qs[-1]))
        bands.append(band)
    seqsplit.forward_bands(bands, Qs, Vs, Os, wl.W)
    torch.cuda.synchronize()
    return torch.cat(Os, dim=2)


@pytest.mark.parametrize("wl,nb", CASES, ids=[f"{w.name}-{n}bands" for w, n in CASES])
@pytest.mark.parametrize("whiten", [True, False], ids=["whitened", "unwhitened"])
def test_bands_match_whole_grid(wl, nb, whiten, monkeypatch):
    x = pu.inputs_for(wl)
    O_sp = _bands(wl, nb, x, whiten)
    monkeypatch.setenv("LFA_FORWARD_PATH", "generic")
    mod = pu.gpu_module(wl, whiten, False)
    O_full = mod.forward(x.Q_store.cuda(), x.V_store.cuda())
    torch.cuda.synchronize()
    units = tuple(range(wl.units))
    a, b = pu.unit_rows(O_sp, units), pu.unit_rows(O_full, units)
    bf16 = wl.dtype == "bf16"
    for u in units:
        if bf16 and whiten:
            assert np.linalg.norm(a[u] - b[u]) <= 2.0 ** -7 * np.linalg.norm(b[u]), f"unit {u}"
        else:
            ulp = 2.0 ** -8 if bf16 else 1e-5
            assert np.max(np.abs(a[u] - b[u])) <= ulp * np.max(np.abs(b[u])), f"unit {u}"
    check = (0, wl.units - 1)
    ref = pu.oracle_forward(wl, whiten, False, check)
    want = np.stack([ref.O[divmod(u, wl.heads)] for u in check])
    err = pu.o_error(pu.unit_rows(O_sp, check), want, wl.dtype == "bf16")
    assert err <= pu.o_tolerance(wl.dtype == "bf16"), f"{wl.name}: error {err:.3e}"


def test_band_handles_reject_the_whole_grid_calls():
    wl = Workload("sp_f32", B=1, heads=1, H=16, W=16, d=32, r=4, T=20, dtype="f32")
    x = pu.inputs_for(wl)
    band = lfa.SeqSplitBand(lfa.make_config(wl), 0, 8, x.dwc, "cuda")
    Q = x.Q_store[:, :, :128].contiguous().cuda()
    assert band.lib.lfa_forward(band.handle, Q.data_ptr(), Q.data_ptr(), Q.data_ptr(), None) == \
        lfa.LFA_ERR_INVALID_ARG
    # a band needs its halo unless it is the whole grid
    L = band.pool(Q)
    part = band.pass1(Q, Q, L)
    st = band.lib.lfa_sp_pass2(band.handle, Q.data_ptr(), Q.data_ptr(), None, part.data_ptr(), Q.data_ptr(), None)
    assert st == lfa.LFA_ERR_INVALID_ARG
    bad = lfa.make_config(wl.replace(H=16))
    assert band.lib.lfa_sp_workspace_size(bad, 10, 8) == 0      # rows beyond the grid
    batch = lfa.make_config(wl, "batch")
    assert band.lib.lfa_sp_workspace_size(batch, 0, 8) == 0     # batch-pooled statistics: unsupported
