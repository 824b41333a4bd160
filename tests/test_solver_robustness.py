"""Newton-Schulz against conjugate gradients on ill-conditioned landmark systems (CPU, oracle).

The LaplacianFormer note (关键设计 3 and its solver ablation) prefers Newton-Schulz to CG because
CG degrades on ill-conditioned systems (condition number 50 is its example) while Newton-Schulz
converges stably after a warm-up. This measures both solvers on W Y = B with W symmetric
positive definite, m = 49 (the PVT landmark count), condition number 50, 64 right-hand sides,
in float64 and in float32 arithmetic: relative error ||Y - W^-1 B||_F / ||W^-1 B||_F after a
number of Newton-Schulz steps (Y = X_T B, alpha by the fallback rule) or CG iterations. One
Newton-Schulz step costs 2 m^3 = 235 k multiply-adds, one CG iteration m^2 * 64 = 154 k, so 20
steps cost about as much as 30 iterations.

Run with -s to print the table.
"""
import numpy as np
import pytest

from oracle import lfa_oracle as O
from tests import pins

M, D, KAPPA, SEEDS = 49, 64, 50.0, (0, 1, 2)


def _errors():
    rows = []
    for seed in SEEDS:
        W = pins._spd(M, KAPPA, 100 + seed)
        B = np.random.default_rng(seed).standard_normal((M, D))
        Y = np.linalg.solve(W, B)
        alpha = O.select_alpha(W).alpha
        rel = lambda Z: float(np.linalg.norm(np.asarray(Z, np.float64) - Y) / np.linalg.norm(Y))
        r = {}
        for T in (5, 10, 15, 20):
            r["ns", T, 64] = rel(O.newton_schulz(W, alpha, T)[0] @ B)
            r["ns", T, 32] = rel(O.newton_schulz_dtype(W, alpha, T, np.float32).astype(np.float64) @ B)
        for k in (5, 10, 15, 20, 30, 49):
            r["cg", k, 64] = rel(O.cg_solve(W, B, k))
            r["cg", k, 32] = rel(O.cg_solve(W, B, k, np.float32))
        rows.append(r)
    return rows


@pytest.fixture(scope="module")
def errors():
    rows = _errors()
    keys = sorted(rows[0], key=lambda k: (k[0], k[2], k[1]))
    print("\nsolver steps precision: relative error per seed")
    for k in keys:
        print(f"  {k[0]} {k[1]:3d} fp{k[2]}: " + "  ".join(f"{r[k]:.1e}" for r in rows))
    return rows


def test_newton_schulz_warm_up_then_quadratic(errors):
    for r in errors:
        assert r["ns", 10, 64] > r["cg", 10, 64]          # CG is ahead during the warm-up
        assert r["ns", 15, 64] < 1e-5
        assert r["ns", 20, 64] < 1e-13                     # converged to fp64 rounding
        assert r["ns", 20, 32] < 2e-6                      # and to fp32 rounding


def test_newton_schulz_ahead_at_equal_steps_and_equal_cost(errors):
    for r in errors:
        for p in (64, 32):
            assert r["ns", 20, p] * 100 < r["cg", 20, p]
            assert r["ns", 20, p] < r["cg", 30, p]         # about equal multiply-add counts


def test_cg_linear_rate_at_kappa_50(errors):
    rho = (np.sqrt(KAPPA) - 1) / (np.sqrt(KAPPA) + 1)
    for r in errors:
        for k in (10, 20, 30):
            # the energy-norm bound, carried to the 2-norm by sqrt(kappa)
            assert r["cg", k, 64] <= 2 * rho ** k * np.sqrt(KAPPA)
        assert r["cg", 49, 64] < 1e-7                      # m steps: exact up to rounding
