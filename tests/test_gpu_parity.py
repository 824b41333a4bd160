"""GPU parity: the CUDA library (through the C-ABI) against the CPU oracle on the same seeded inputs.

Covers every workload at full size (all units), both whitening readings, the DWC term
separately, the cross kernel C, the Newton-Schulz context, the lambda sweep of the
heavy-tailed workload, and edge cases (ragged tiles, d = 32 in bf16, one landmark,
T = 0, eps = 0, underflowing C, constant inputs, m = 256 on a small grid).
"""
import numpy as np
import pytest
import torch

from laplacian_nystr_attention_avg_b200 import lfa
from laplacian_nystr_attention_avg_b200.inputs import PVT2_LAMBDA_SWEEP, WORKLOADS, Workload
from oracle import lfa_oracle as O
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

FULL = ["pr1", "pvt1", "pvt2", "hr49", "hr196", "long"]


def _check_forward(wl: Workload, whiten: bool, zero_dwc: bool, units=None):
    units = tuple(range(wl.units)) if units is None else tuple(units)
    mod, Q, V, Og, st, info = pu.run_gpu_forward(wl, whiten, zero_dwc)
    assert st == lfa.LFA_OK
    ref = pu.oracle_forward(wl, whiten, zero_dwc, units)
    got = pu.unit_rows(Og, units)
    want = np.stack([ref.O[divmod(u, wl.heads)] for u in units])
    err = pu.o_error(got, want, wl.dtype == "bf16")
    tol = pu.o_tolerance(wl.dtype == "bf16")
    assert err <= tol, f"{wl.name} whiten={whiten} zero_dwc={zero_dwc}: error {err:.3e} > {tol:.0e}"
    for k, u in enumerate(units):
        assert info[u].alpha_fallback == int(ref.units[k].alpha.fallback)
    return err


@pytest.mark.parametrize("name", FULL)
@pytest.mark.parametrize("whiten", [True, False], ids=["whitened", "unwhitened"])
@pytest.mark.parametrize("zero_dwc", [True, False], ids=["attn_only", "with_dwc"])
def test_forward_full_size(name, whiten, zero_dwc):
    _check_forward(pu.workload(name), whiten, zero_dwc)


@pytest.mark.parametrize("lam", PVT2_LAMBDA_SWEEP)
@pytest.mark.parametrize("zero_dwc", [True, False], ids=["attn_only", "with_dwc"])
def test_forward_lambda_sweep(lam, zero_dwc):
    _check_forward(pu.workload("pvt2", lam=lam), True, zero_dwc)


@pytest.mark.parametrize("name,lam", [("pr1", 4.0), ("pvt1", 4.0), ("pvt2", 0.5), ("pvt2", 1.0),
                                      ("pvt2", 8.0), ("hr49", 4.0), ("hr196", 4.0), ("long", 4.0)])
def test_cross_kernel(name, lam):
    wl = pu.workload(name, lam=lam)
    x = pu.inputs_for(wl)
    mod = pu.gpu_module(wl, True, False)
    Q = x.Q_store.cuda()
    for u in sorted({0, wl.units - 1}):
        Cg = mod.cross_kernel(Q, u).cpu().numpy().astype(np.float64)
        b, h = divmod(u, wl.heads)
        q = x.Q[b, h].double().numpy()
        L = O.pool_landmarks(q, wl.H, wl.W, wl.r)
        Co = O.laplacian_kernel(q, L, wl.lam)
        err = pu.c_error(Cg, Co)
        assert err <= pu.c_tolerance(wl.lam), f"{name} lam={lam} unit {u}: C error {err:.3e}"


@pytest.mark.parametrize("name", FULL)
def test_newton_schulz_context(name):
    wl = pu.workload(name)
    mod, Q, V, Og, st, info = pu.run_gpu_forward(wl, True, False)
    ref = pu.oracle_forward(wl, True, False, tuple(range(wl.units)))
    for u in sorted({0, wl.units // 2, wl.units - 1}):
        L, X, mu, s = (t.cpu().numpy().astype(np.float64) for t in mod.context(u))
        f = ref.units[u]
        assert np.max(np.abs(L - f.L)) <= 1e-5 * np.max(np.abs(f.L))
        kappa = np.linalg.cond(f.W)
        errX = np.max(np.abs(X - f.X)) / np.max(np.abs(f.X))
        # First-order error of the last printed Newton-Schulz step is ~ c * kappa * u for unit
        # roundoff u of the products (c = 33). Every path runs the m x m products on the tensor cores
        # as split TF32 (hi + lo, the lo part truncated to 11 bits): u = 2^-21.
        u_eff = 2.0 ** -21
        assert errX <= 33 * u_eff * kappa + 1e-5, f"{name} unit {u}: X error {errX:.2e} (kappa {kappa:.0f})"
        assert abs(info[u].lambda_max - f.alpha.norm2) <= 1e-4 * f.alpha.norm2
        assert info[u].alpha_fallback == int(f.alpha.fallback) == 1
        # ||I - W X_gpu||_F, computed on the device, against a bound from its parts: the oracle's own
        # residual after T steps, the distance of X_gpu from the oracle's X (times ||W||_F), and the
        # rounding of the device product W X_gpu (at most m u_eff ||W||_F ||X_gpu||_F per side)
        Wn, Xn = np.linalg.norm(f.W), np.linalg.norm(X)
        res_o = np.linalg.norm(np.eye(wl.m) - f.W @ f.X)
        bound = res_o + Wn * np.linalg.norm(X - f.X) + 2 * wl.m * u_eff * Wn * Xn
        assert info[u].ns_residual_fro <= bound, f"{name} unit {u}: residual {info[u].ns_residual_fro:.2e} > {bound:.2e}"
        np.testing.assert_allclose(mu, f.mu, rtol=1e-4)
        np.testing.assert_allclose(s, 1.0 / np.sqrt(f.var + wl.eps), rtol=1e-4)


def test_deterministic():
    wl = pu.workload("pvt1")
    x = pu.inputs_for(wl)
    mod = pu.gpu_module(wl, True, False)
    Q, V = x.Q_store.cuda(), x.V_store.cuda()
    a = mod.forward(Q, V).clone()
    b = mod.forward(Q, V)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


EDGE = [
    # ragged last row tile (N = 144), fp32
    Workload("ragged_f32", B=2, heads=1, H=12, W=12, d=32, r=4, T=20, dtype="f32"),
    # ragged, bf16, d = 64, several heads
    Workload("ragged_bf16", B=1, heads=3, H=20, W=12, d=64, r=4, T=20),
    # d = 32 in bf16
    Workload("d32_bf16", B=2, heads=2, H=32, W=32, d=32, r=8, T=20),
    # one landmark (r = H = W)
    Workload("m1", B=2, heads=1, H=16, W=16, d=64, r=16, T=20),
    # no Newton-Schulz steps: X = alpha W^T
    Workload("T0", B=1, heads=1, H=16, W=16, d=32, r=4, T=0, dtype="f32"),
    # eps = 0
    Workload("eps0", B=1, heads=1, H=16, W=16, d=32, r=4, T=20, eps=0.0, dtype="f32"),
    # strong underflow of C (lambda = 0.25)
    Workload("underflow", B=1, heads=2, H=28, W=28, d=64, r=4, T=20, lam=0.25),
    # the largest landmark count (m = 256) on a small grid, fp32
    Workload("m256", B=1, heads=1, H=32, W=32, d=32, r=2, T=24, dtype="f32"),
    # m between 64 and 256, not a multiple of 16 (m = 81)
    Workload("m81", B=1, heads=2, H=36, W=36, d=64, r=4, T=24),
    # non-square grid
    Workload("rect", B=1, heads=1, H=24, W=40, d=64, r=8, T=20),
    # more units than SMs: the per-stage path with one streaming thread block per unit, in two waves
    Workload("many_units", B=80, heads=2, H=16, W=16, d=64, r=4, T=20),
    # one landmark on the streaming passes (80 units: past the fused kernel's unit limit), 15 of 16 warps
    # without a landmark
    Workload("m1_stream", B=80, heads=1, H=16, W=16, d=64, r=16, T=20),
]


@pytest.mark.parametrize("wl", EDGE, ids=[w.name for w in EDGE])
@pytest.mark.parametrize("whiten", [True, False], ids=["whitened", "unwhitened"])
def test_edge_cases(wl, whiten):
    _check_forward(wl, whiten, True)
    _check_forward(wl, whiten, False)


def test_constant_queries():
    # identical queries: C is constant per column, var = 0, s = 1/sqrt(eps)
    wl = Workload("const", B=1, heads=1, H=16, W=16, d=32, r=4, T=20, dtype="f32")
    x = pu.inputs_for(wl)
    Q = torch.full_like(x.Q_store, 0.5)
    mod = pu.gpu_module(wl, True, False)
    Og = mod.forward(Q.cuda(), x.V_store.cuda())
    ref = O.forward(Q.double().numpy(), x.V.numpy(), x.dwc.numpy(), wl)
    got = pu.unit_rows(Og, [0])
    assert pu.o_error(got, ref.O[0][None], False) <= 1e-3


def test_info_and_state_errors():
    wl = pu.workload("pr1")
    x = pu.inputs_for(wl)
    mod = pu.gpu_module(wl, True, False)
    Q, V = x.Q_store.cuda(), x.V_store.cuda()
    dO = torch.zeros_like(Q)
    with pytest.raises(lfa.LfaError) as e:
        mod.backward(Q, V, dO)
    assert e.value.status == lfa.LFA_ERR_STATE
    mod.forward(Q, V)
    with pytest.raises(lfa.LfaError) as e:
        mod.backward(Q.clone(), V, dO)      # different Q pointer than the forward
    assert e.value.status == lfa.LFA_ERR_STATE
    st, info = mod.info()
    assert st == lfa.LFA_OK and len(info) == 1
    # misaligned pointers are rejected on the host
    raw = torch.empty(Q.numel() + 4, dtype=Q.dtype, device="cuda")
    with pytest.raises(lfa.LfaError) as e:
        mod.forward(raw[1:1 + Q.numel()].view(Q.shape), V)
    assert e.value.status == lfa.LFA_ERR_INVALID_ARG


def test_forward_host_buffers():
    wl = pu.workload("pvt1")
    x = pu.inputs_for(wl)
    mod = pu.gpu_module(wl, True, False)
    Qh, Vh = x.Q_store.pin_memory(), x.V_store.pin_memory()
    Oh = torch.empty(Qh.shape, dtype=Qh.dtype).pin_memory()
    Qd, Vd, Od = torch.empty_like(Qh, device="cuda"), torch.empty_like(Vh, device="cuda"), \
        torch.empty_like(Qh, device="cuda")
    mod.forward_host(Qh, Vh, Oh, Qd, Vd, Od)
    ref = mod.forward(x.Q_store.cuda(), x.V_store.cuda()).cpu()
    assert torch.equal(Oh, ref)


@pytest.mark.parametrize("name", ["pvt1", "hr196"])
def test_forward_host_async_on_two_streams(name):
    # two handles on two streams, alternate steps with their own pinned buffers: every step's O equals the
    # one-stream forward's (fused launches are ordered per device; the copies overlap)
    wl = pu.workload(name)
    x = pu.inputs_for(wl)
    mods = [pu.gpu_module(wl, True, False) for _ in range(2)]
    ref = mods[0].forward(x.Q_store.cuda(), x.V_store.cuda()).cpu()
    streams = [torch.cuda.current_stream(), torch.cuda.Stream()]
    host = [(x.Q_store.pin_memory(), x.V_store.pin_memory(), torch.empty(x.Q_store.shape, dtype=x.Q_store.dtype).pin_memory())
            for _ in range(2)]
    dev = [tuple(torch.empty(x.Q_store.shape, dtype=x.Q_store.dtype, device="cuda") for _ in range(3)) for _ in range(2)]
    outs = []
    for k in range(6):
        i = k % 2
        host[i][2].zero_()
        mods[i].forward_host_async(*host[i], *dev[i], stream=streams[i])
        if k >= 1:
            j = 1 - i
            streams[j].synchronize()
            outs.append(host[j][2].clone())
    streams[1 - (5 % 2)].synchronize()
    streams[5 % 2].synchronize()
    outs.append(host[5 % 2][2].clone())
    for o in outs:
        assert torch.equal(o, ref)


@pytest.mark.parametrize("name", ["pvt1", "pvt2", "hr49"])
def test_fused_and_generic_paths_agree(name, monkeypatch):
    wl = pu.workload(name)
    x = pu.inputs_for(wl)
    fused = pu.gpu_module(wl, True, False)
    monkeypatch.setenv("LFA_FORWARD_PATH", "generic")
    generic = pu.gpu_module(wl, True, False)
    monkeypatch.delenv("LFA_FORWARD_PATH")
    assert fused.path == "fused" and generic.path == "generic"
    Q, V = x.Q_store.cuda(), x.V_store.cuda()
    a = pu.unit_rows(fused.forward(Q, V), range(wl.units))
    b = pu.unit_rows(generic.forward(Q, V), range(wl.units))
    assert pu.o_error(a, b, True) <= 1e-2
    # repeated calls reuse the cross-CTA flags (epochs) and give identical results
    c = pu.unit_rows(fused.forward(Q, V), range(wl.units))
    assert np.array_equal(a, c)
