"""The cross kernel C that the fused forward itself computes and multiplies, against the oracle.

lfa_debug_capture_cross arms a one-shot copy of one unit's C from inside the next forward. The fused
kernel keeps bf16(C - c) on chip between pass 1 and pass 2, with c a per-column shift of each thread
block's rows (pass 2's bias adds c back exactly), so the copy is that bf16 value widened to fp32 plus c,
and the call also returns the c of every entry. The oracle computes C = exp(-||q - l||_1 / lambda) in
float64 from the same bf16 inputs (LaplacianFormer note, §关键设计 2).

Bound per entry on |C_gpu - C|, with e_C = 2^-16 (1 + D / lambda) C and D = ||q - l||_1:
  * e_C: the fp32 distance sum of d = 64 rounded |q - l| terms (relative error <= 64 u D with
    u = 2^-24, entering C as 2^-18 D / lambda), the fp32 landmark average (<= 64 u per coordinate, of
    the same order), the fp32 product with -log2(e) / lambda and ex2.approx (<= 2^-22 relative), with
    a 4x margin;
  * 2^-8 (|C - c| + e_C): round-to-nearest-even of the fp32 C - c to bf16 (8 significant bits, unit
    roundoff 2^-8);
  * 2^-23 C: the fp32 sum that adds c back;
  * 2^-126: ex2.approx.ftz flushes results below the fp32 normal range to zero.
"""
import numpy as np
import pytest
import torch

from laplacian_nystr_attention_avg_b200 import lfa
from oracle import lfa_oracle as O
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

def fused_c_error(Cg: np.ndarray, Sg: np.ndarray, q: np.ndarray, L: np.ndarray, lam: float) -> float:
    """Worst ratio of |C_gpu - C| to the bound above (<= 1 passes)."""
    D = O.l1_distances(q, L)
    C = np.exp(-D / lam)
    eC = 2.0 ** -16 * (1.0 + D / lam) * C
    bound = 2.0 ** -8 * (np.abs(C - Sg) + eC) + eC + 2.0 ** -23 * C + 2.0 ** -126
    return float(np.max(np.abs(Cg - C) / bound))


CASES = [("pvt1", 4.0), ("pvt2", 0.5), ("pvt2", 1.0), ("pvt2", 2.0), ("pvt2", 4.0), ("pvt2", 8.0),
         ("pvt2", 32.0), ("hr49", 4.0)]


@pytest.mark.parametrize("name,lam", CASES)
def test_fused_cross_kernel(name, lam):
    wl = pu.workload(name, lam=lam)
    x = pu.inputs_for(wl)
    mod = pu.gpu_module(wl, True, False)
    assert mod.path == "fused"
    Q, V = x.Q_store.cuda(), x.V_store.cuda()
    for u in sorted({0, wl.units // 2, wl.units - 1}):
        Cg, Sg = (t.cpu().numpy().astype(np.float64) for t in mod.capture_cross(Q, V, u))
        b, h = divmod(u, wl.heads)
        q = x.Q[b, h].double().numpy()
        L = O.pool_landmarks(q, wl.H, wl.W, wl.r)
        r = fused_c_error(Cg, Sg, q, L, wl.lam)
        assert r <= 1.0, f"{name} lam={lam} unit {u}: C error {r:.3f} of the bound"


# Per-stage path with bf16 tokens and d = 64: pass 2 multiplies bf16(C - mu) on the tensor cores, mu
# the column mean; the copy is that value widened plus mu, under the same bound (shift mu). Large grids
# are checked on a row sample (every 7th row and the last rows).
STREAM_CASES = [("pvt2", 4.0, "generic"), ("pvt2", 32.0, "generic"), ("hr196", 4.0, None), ("long", 4.0, None)]


@pytest.mark.parametrize("name,lam,path", STREAM_CASES)
def test_stream_cross_kernel(name, lam, path, monkeypatch):
    wl = pu.workload(name, lam=lam)
    x = pu.inputs_for(wl)
    if path:
        monkeypatch.setenv("LFA_FORWARD_PATH", path)
    mod = pu.gpu_module(wl, True, False)
    monkeypatch.delenv("LFA_FORWARD_PATH", raising=False)
    assert mod.path == "generic"
    Q, V = x.Q_store.cuda(), x.V_store.cuda()
    rows = np.unique(np.concatenate([np.arange(0, wl.H * wl.W, 7), np.arange(wl.H * wl.W - 70, wl.H * wl.W)]))
    for u in sorted({0, wl.units - 1}):
        Cg, Sg = (t.cpu().numpy().astype(np.float64)[rows] for t in mod.capture_cross(Q, V, u))
        b, h = divmod(u, wl.heads)
        q = x.Q[b, h].double().numpy()
        L = O.pool_landmarks(q, wl.H, wl.W, wl.r)
        mu_ref = O.laplacian_kernel(q, L, wl.lam).mean(axis=0)
        assert np.allclose(Sg, mu_ref[None, :], rtol=1e-4, atol=0.0), f"{name}: shift is not the column mean"
        r = fused_c_error(Cg, Sg, q[rows], L, wl.lam)
        assert r <= 1.0, f"{name} lam={lam} unit {u}: C error {r:.3f} of the bound"


def test_capture_on_cuda_core_path_matches_debug_kernel():
    # fp32 tokens take the CUDA-core passes, which copy C with their own tile code: identical to
    # lfa_debug_cross_kernel
    wl = pu.workload("pr1")
    x = pu.inputs_for(wl)
    mod = pu.gpu_module(wl, True, False)
    assert mod.path == "generic"
    Q, V = x.Q_store.cuda(), x.V_store.cuda()
    a, sh = mod.capture_cross(Q, V, 0)
    b = mod.cross_kernel(Q, 0)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert not sh.any()
    # lfa_debug_cross_kernel pooled into the workspace: the saved context is gone until a forward
    with pytest.raises(lfa.LfaError) as e:
        mod.backward(Q, V, torch.zeros_like(Q))
    assert e.value.status == lfa.LFA_ERR_STATE


@pytest.mark.parametrize("lam", [16.0, 32.0])
@pytest.mark.parametrize("zero_dwc", [True, False], ids=["attn_only", "with_dwc"])
def test_forward_large_lambda(lam, zero_dwc):
    # larger lambda raises mu / sigma of every column of C, so the bf16 rounding of the resident C
    # weighs more after whitening; the fused forward must still meet the bf16 bound
    wl = pu.workload("pvt2", lam=lam)
    mod, Q, V, Og, st, info = pu.run_gpu_forward(wl, True, zero_dwc)
    assert st == lfa.LFA_OK and mod.path == "fused"
    units = tuple(range(wl.units))
    ref = pu.oracle_forward(wl, True, zero_dwc, units)
    got = pu.unit_rows(Og, units)
    want = np.stack([ref.O[divmod(u, wl.heads)] for u in units])
    err = pu.o_error(got, want, True)
    assert err <= pu.o_tolerance(True), f"lambda={lam}: error {err:.3e}"
