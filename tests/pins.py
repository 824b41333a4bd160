"""Pins of the CPU oracle to things other than itself.

Each ``check_*`` raises AssertionError on failure. tests/test_oracle_pins.py runs
them on the real oracle; tests/test_oracle_mutations.py plants plausible
mistakes in the oracle (on the CPU) and asserts that some pin catches each one.

Anchors used (none of them re-types an oracle formula):
  * closed forms: k(x, x) = 1, k(0, 1_d) = exp(-d/lam), the 1-D factorisation,
    the window-centre value of a pooled ramp, the eigen closed form of every
    Newton-Schulz iterate, R_{k+1} = R_k^2.
  * library routines: scipy cdist(cityblock), torch avg_pool2d / conv2d (float64),
    scipy Cholesky, numpy solve, sklearn StandardScaler.
  * brute force: the dense O(N^2) kernel product at r = 1.
  * finite differences of the forward for the backward pass.
"""
from __future__ import annotations

import numpy as np
import scipy.linalg
import torch
from scipy.spatial.distance import cdist

from oracle import lfa_oracle as O


def _rng(seed):
    return np.random.default_rng(seed)


# --- Laplacian kernel ------------------------------------------------------

def check_kernel_closed_forms():
    rng = _rng(1)
    for d in (1, 8, 32, 64):
        for lam in (0.5, 4.0):
            x = rng.standard_normal((5, d))
            y = rng.standard_normal((7, d))
            K = O.laplacian_kernel(x, x, lam)
            assert np.allclose(np.diag(K), 1.0, rtol=0, atol=1e-15), "k(x, x) != 1"
            Kxy = O.laplacian_kernel(x, y, lam)
            Kyx = O.laplacian_kernel(y, x, lam)
            assert np.array_equal(Kxy, Kyx.T), "kernel not symmetric"
            # hand value: x = 0, y = 1_d gives exp(-d/lam)
            h = O.laplacian_kernel(np.zeros((1, d)), np.ones((1, d)), lam)[0, 0]
            assert abs(h - np.exp(-d / lam)) <= 1e-15 * max(1.0, np.exp(-d / lam)), "hand value"
            # product of 1-D Laplace kernels
            prod = np.ones((5, 7))
            for k in range(d):
                prod *= np.exp(-np.abs(x[:, k][:, None] - y[:, k][None, :]) / lam)
            assert np.allclose(Kxy, prod, rtol=1e-12, atol=0), "1-D factorisation"


def check_kernel_vs_cdist():
    rng = _rng(2)
    x = rng.standard_normal((300, 64))
    y = rng.standard_normal((49, 64)) * 0.2
    for lam in (0.5, 1.0, 4.0, 8.0):
        ref = np.exp(-cdist(x, y, "cityblock") / lam)
        got = O.laplacian_kernel(x, y, lam)
        assert np.allclose(got, ref, rtol=1e-12, atol=0), "kernel vs cdist"


# --- landmark pooling -------------------------------------------------------

def check_pool_ramp():
    for H, W, r in ((16, 16, 4), (56, 56, 8), (28, 28, 4), (8, 12, 4)):
        d = 3
        yy, xx, kk = np.meshgrid(np.arange(H), np.arange(W), np.arange(d), indexing="ij")
        q = (yy * W + xx + 1000.0 * kk).reshape(H * W, d).astype(np.float64)
        L = O.pool_landmarks(q, H, W, r)
        Y, X = np.meshgrid(np.arange(H // r), np.arange(W // r), indexing="ij")
        cy = Y.reshape(-1) * r + (r - 1) / 2.0
        cx = X.reshape(-1) * r + (r - 1) / 2.0
        expect = (cy * W + cx)[:, None] + 1000.0 * np.arange(d)[None, :]
        assert np.allclose(L, expect, rtol=0, atol=1e-9), "ramp pool != window centre"


def check_pool_vs_torch():
    rng = _rng(3)
    H, W, r, d = 56, 56, 8, 16
    q = rng.standard_normal((H * W, d))
    L = O.pool_landmarks(q, H, W, r)
    t = torch.from_numpy(q.reshape(H, W, d)).permute(2, 0, 1)[None]
    ref = torch.nn.functional.avg_pool2d(t, r, r)[0].permute(1, 2, 0).reshape(-1, d).numpy()
    assert np.allclose(L, ref, rtol=1e-13, atol=1e-15), "pool vs avg_pool2d"


# --- landmark kernel W and alpha --------------------------------------------

def _landmarks(H, W, r, d, seed, scale=1.0):
    q = _rng(seed).standard_normal((H * W, d)) * scale
    return O.pool_landmarks(q, H, W, r)


def check_gram_spd():
    for (H, W, r, d, lam, eps) in ((16, 16, 4, 32, 4.0, 1e-6), (56, 56, 8, 64, 4.0, 1e-6),
                                   (112, 112, 8, 64, 4.0, 1e-6), (28, 28, 4, 64, 0.5, 1e-6)):
        L = _landmarks(H, W, r, d, seed=H + r)
        Wm = O.landmark_gram(L, lam, eps)
        assert np.array_equal(Wm, Wm.T), "W not symmetric"
        assert np.allclose(np.diag(Wm), 1.0 + eps, rtol=0, atol=1e-15), "diag(W) != 1 + eps"
        scipy.linalg.cholesky(Wm)  # raises if not positive definite


def check_alpha_rule():
    # The printed alpha = 2/||W||_2 is tested, and it fails whenever ||W||_2 > 1.
    for (H, W, r, d) in ((16, 16, 4, 32), (56, 56, 8, 64), (112, 112, 16, 64)):
        Wm = O.landmark_gram(_landmarks(H, W, r, d, seed=7), 4.0, 1e-6)
        ac = O.select_alpha(Wm)
        lmax = np.linalg.eigvalsh(Wm).max()
        assert abs(ac.norm2 - lmax) <= 1e-12 * lmax, "||W||_2 != lambda_max for SPD W"
        assert abs(ac.alpha_pages - 2.0 / lmax) <= 1e-12 / lmax
        # eigenvalue 1 - 2 lmax of I - (2/lmax) W^2 lies below -1
        assert abs(ac.cond_pages - (2.0 * lmax - 1.0)) <= 1e-9 * lmax, "printed condition value"
        assert ac.fallback and abs(ac.alpha - 1.0 / lmax ** 2) <= 1e-12 / lmax ** 2
        assert np.linalg.norm(np.eye(len(Wm)) - ac.alpha * Wm @ Wm.T, 2) < 1.0
    # a matrix with ||W||_2 < 1 keeps the printed alpha
    Wm = 0.5 * np.eye(4)
    ac = O.select_alpha(Wm)
    assert not ac.fallback and ac.alpha == 4.0


# --- Newton-Schulz ------------------------------------------------------------

def _spd(m, kappa, seed):
    Qm, _ = np.linalg.qr(_rng(seed).standard_normal((m, m)))
    return (Qm * np.geomspace(1.0, kappa, m)) @ Qm.T


def check_ns_eigen_closed_form():
    # X_k = U diag((1 - (1 - alpha w^2)^(2^k)) / w) U^T for every step k
    for Wm, T in ((O.landmark_gram(_landmarks(16, 16, 4, 32, 5), 4.0, 1e-6), 20),
                  (_spd(49, 50.0, 11), 20)):
        ac = O.select_alpha(Wm)
        X, res, its = O.newton_schulz(Wm, ac.alpha, T, keep_iterates=True)
        w, U = np.linalg.eigh(Wm)
        r0 = 1.0 - ac.alpha * w ** 2
        for k, Xk in enumerate(its):
            xk = (1.0 - r0 ** (2 ** k)) / w
            ref = (U * xk) @ U.T
            assert np.allclose(Xk, ref, rtol=0, atol=1e-10 * np.abs(ref).max()), f"NS step {k}"


def check_ns_vs_cholesky():
    for Wm in (O.landmark_gram(_landmarks(56, 56, 8, 64, 9), 4.0, 1e-6), _spd(64, 50.0, 12)):
        ac = O.select_alpha(Wm)
        X, res, _ = O.newton_schulz(Wm, ac.alpha, 20)
        inv = scipy.linalg.cho_solve(scipy.linalg.cho_factor(Wm), np.eye(len(Wm)))
        kappa = np.linalg.cond(Wm)
        err = np.abs(X - inv).max() / np.abs(inv).max()
        assert err < 50 * kappa * np.finfo(float).eps, f"NS vs Cholesky {err}"


def check_ns_kappa50_and_quadratic():
    # kappa = 50 converges within 20 steps with the fallback alpha; R_{k+1} = R_k^2
    Wm = _spd(49, 50.0, 13)
    ac = O.select_alpha(Wm)
    X, res, _ = O.newton_schulz(Wm, ac.alpha, 20)
    assert res[-1][1] < 1e-12, "kappa=50 did not converge in 20 steps"
    for k in range(len(res) - 1):
        r2, r2n = res[k][1], res[k + 1][1]
        if r2 ** 2 > 1e-12:
            assert abs(r2n - r2 ** 2) <= 1e-9 + 1e-7 * r2 ** 2, f"||R_k+1|| != ||R_k||^2 at {k}"


def check_cg_vs_solve():
    # in exact arithmetic CG terminates in m steps; with a small condition number fp64 gets there
    rng = _rng(71)
    Wm = _spd(16, 5.0, 14)
    Bm = rng.standard_normal((16, 6))
    Y = O.cg_solve(Wm, Bm, 24)
    ref = np.linalg.solve(Wm, Bm)
    assert np.allclose(Y, ref, rtol=0, atol=1e-10 * np.abs(ref).max())


def check_cg_error_bound():
    # the classical bound ||e_k||_W <= 2 ((sqrt k - 1) / (sqrt k + 1))^k ||e_0||_W at kappa = 50
    kappa = 50.0
    Wm = _spd(49, kappa, 15)
    b = _rng(72).standard_normal((49, 1))
    y = np.linalg.solve(Wm, b)
    e0 = float(np.sqrt((y.T @ Wm @ y).item()))
    rho = (np.sqrt(kappa) - 1.0) / (np.sqrt(kappa) + 1.0)
    for k in range(1, 25):
        e = O.cg_solve(Wm, b, k) - y
        ek = float(np.sqrt((e.T @ Wm @ e).item()))
        assert ek <= 2.0 * rho ** k * e0 * (1 + 1e-9) + 1e-13 * e0, f"CG bound at step {k}"


# --- Nystrom assembly -----------------------------------------------------------

def check_nystrom_r1_dense():
    # r = 1: landmarks are the tokens, C = W - eps I = G, so C X C^T V = G V at eps = 0
    for (H, W, d, lam) in ((4, 4, 4, 4.0), (8, 8, 8, 4.0), (8, 8, 16, 2.0)):
        rng = _rng(H * d)
        q = rng.standard_normal((H * W, d))
        v = rng.standard_normal((H * W, d))
        w = np.zeros((d, 3, 3))
        G = np.exp(-cdist(q, q, "cityblock") / lam)
        dense = G @ v
        f = O.unit_forward(q, v, w, H, W, 1, lam, 0.0, 60, whiten=False)
        assert np.allclose(f.O_attn, dense, rtol=0, atol=1e-8 * np.abs(dense).max()), "r=1, eps=0"
        eps = 1e-6
        f = O.unit_forward(q, v, w, H, W, 1, lam, eps, 60, whiten=False)
        ref = dense - eps * v   # G (G + eps I)^-1 G = G - eps I + O(eps^2)
        assert np.allclose(f.O_attn, ref, rtol=0, atol=1e-8 * np.abs(dense).max()), "r=1, eps>0"


def check_whitening_moments():
    rng = _rng(21)
    C = np.exp(-rng.gamma(3.0, 4.0, size=(784, 49)))
    for eps in (0.0, 1e-6, 1e-2):
        Ct, mu, var = O.whiten_columns(C, eps)
        N = C.shape[0]
        Z = Ct - 1.0 / N
        assert np.allclose(Z.mean(axis=0), 0.0, atol=1e-12 * np.abs(Z).max())
        assert np.allclose(Ct.mean(axis=0), 1.0 / N, rtol=1e-9)
        assert np.allclose(Z.var(axis=0), C.var(axis=0) / (C.var(axis=0) + eps), rtol=1e-9)
        assert np.allclose(mu, C.mean(axis=0), rtol=1e-13)


def check_whitening_vs_sklearn():
    from sklearn.preprocessing import StandardScaler
    rng = _rng(22)
    C = np.exp(-rng.gamma(3.0, 2.0, size=(256, 16)))
    Ct, _, _ = O.whiten_columns(C, 0.0)
    ref = StandardScaler().fit_transform(C) + 1.0 / C.shape[0]
    assert np.allclose(Ct, ref, rtol=1e-10, atol=1e-12)


def check_whitened_assembly_vs_solve():
    # converged X = W^-1, so O_attn = C~ solve(W, C~^T V): independent of the NS code
    rng = _rng(23)
    H = W = 16
    d, r, lam, eps = 32, 4, 4.0, 1e-6
    q = rng.standard_normal((H * W, d))
    v = rng.standard_normal((H * W, d))
    w = rng.standard_normal((d, 3, 3)) * 0.1
    f = O.unit_forward(q, v, w, H, W, r, lam, eps, 30, whiten=True)
    ref = f.Ct @ np.linalg.solve(f.W, f.Ct.T @ v)
    assert np.allclose(f.O_attn, ref, rtol=0, atol=1e-9 * np.abs(ref).max())
    # the unwhitened product is the same assembly with C
    g = O.unit_forward(q, v, w, H, W, r, lam, eps, 30, whiten=False)
    ref = g.C @ np.linalg.solve(g.W, g.C.T @ v)
    assert np.allclose(g.O_attn, ref, rtol=0, atol=1e-9 * np.abs(ref).max())


# --- batch-pooled whitening statistics (reading R12) ----------------------------

class _BatchWl:
    """Minimal workload record for the oracle's whole-call forward."""

    def __init__(self, H, W, r, lam, eps, T):
        self.H, self.W, self.r, self.lam, self.eps, self.T = H, W, r, lam, eps, T


def _batch_case(B, heads, seed, H=8, W=8, d=8, r=2, replicate=False):
    rng = _rng(seed)
    N = H * W
    shape = (1 if replicate else B, heads, N, d)
    q = rng.standard_normal(shape)
    v = rng.standard_normal(shape)
    if replicate:
        q = np.repeat(q, B, axis=0)
        v = np.repeat(v, B, axis=0)
    w = rng.standard_normal((heads, d, 3, 3)) * 0.1
    return q, v, w, _BatchWl(H, W, r, 2.0, 1e-6, 16)


def check_batch_stats_single_batch():
    # B = 1: the pooled statistics are the unit's own, so the two readings coincide
    q, v, w, wl = _batch_case(1, 3, 51)
    a = O.forward(q, v, w, wl)
    b = O.forward(q, v, w, wl, batch_stats=True)
    assert np.allclose(a.O, b.O, rtol=0, atol=1e-12 * np.abs(a.O).max())


def check_batch_stats_replicated():
    # identical batch elements: pooling copies of the same rows leaves mean and variance unchanged
    q, v, w, wl = _batch_case(4, 2, 52, replicate=True)
    a = O.forward(q, v, w, wl)
    b = O.forward(q, v, w, wl, batch_stats=True)
    assert np.allclose(a.O, b.O, rtol=0, atol=1e-10 * np.abs(a.O).max())


def check_batch_stats_vs_sklearn():
    # per head: standard scaling of the vertically stacked C of all batch elements
    from sklearn.preprocessing import StandardScaler
    B, heads = 3, 2
    q, v, w, wl = _batch_case(B, heads, 53)
    wl.eps = 0.0
    f = O.forward(q, v, w, wl, batch_stats=True)
    N = q.shape[2]
    for h in range(heads):
        units = [b * heads + h for b in range(B)]
        Cs = [f.units[u].C for u in units]
        ref = StandardScaler().fit_transform(np.concatenate(Cs, axis=0)) + 1.0 / N
        got = np.concatenate([f.units[u].Ct for u in units], axis=0)
        assert np.allclose(got, ref, rtol=1e-10, atol=1e-12), f"head {h}"


# --- Reading B: column whitening of the full Nystrom matrix (reading R13) --------

def check_reading_b_vs_dense():
    # materialise G^ = C X C^T (N x N), standard-scale its columns, add 1/N, multiply by V
    from sklearn.preprocessing import StandardScaler
    rng = _rng(61)
    H = W = 8
    d, r, lam, T = 8, 2, 2.0, 30
    q = rng.standard_normal((H * W, d))
    v = rng.standard_normal((H * W, d))
    w = rng.standard_normal((d, 3, 3)) * 0.1
    f = O.unit_forward_reading_b(q, v, w, H, W, r, lam, 0.0, T)
    G = f.C @ f.X @ f.C.T
    ref = (StandardScaler().fit_transform(G) + 1.0 / G.shape[0]) @ v
    assert np.allclose(f.O_attn, ref, rtol=0, atol=1e-10 * np.abs(ref).max())
    assert np.allclose(f.col_var, G.var(axis=0), rtol=1e-10)


def check_reading_b_r1_is_whitened_kernel():
    # r = 1 and eps = 0: the landmarks are the tokens, W = G, X -> G^-1 and G^ = G G^-1 G = G, so
    # Reading B is the column-whitened Laplacian kernel matrix itself applied to V
    rng = _rng(62)
    H = W = 4
    d, lam = 8, 2.0
    q = rng.standard_normal((H * W, d))
    v = rng.standard_normal((H * W, d))
    w = np.zeros((d, 3, 3))
    f = O.unit_forward_reading_b(q, v, w, H, W, 1, lam, 0.0, 40)
    G = np.exp(-np.abs(q[:, None, :] - q[None, :, :]).sum(-1) / lam)
    Z = (G - G.mean(axis=0)) / G.std(axis=0) + 1.0 / G.shape[0]
    ref = Z @ v
    assert np.allclose(f.O_attn, ref, rtol=0, atol=1e-9 * np.abs(ref).max())


# --- DWC ------------------------------------------------------------------------

def check_dwc_vs_conv2d():
    rng = _rng(31)
    for (H, W, d) in ((16, 16, 32), (7, 9, 5)):
        v = rng.standard_normal((H * W, d))
        w = rng.standard_normal((d, 3, 3))
        out = O.dwc3x3(v, w, H, W)
        t = torch.from_numpy(v.reshape(H, W, d)).permute(2, 0, 1)[None]
        ref = torch.nn.functional.conv2d(t, torch.from_numpy(w)[:, None], padding=1, groups=d)
        ref = ref[0].permute(1, 2, 0).reshape(H * W, d).numpy()
        assert np.allclose(out, ref, rtol=1e-12, atol=1e-13)
        # adjoint: <dwc(v), g> = <v, dwc^T(g)>
        g = rng.standard_normal((H * W, d))
        lhs = np.sum(out * g)
        rhs = np.sum(v * O.dwc3x3_transpose(g, w, H, W))
        assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs))


def check_dwc_taps():
    rng = _rng(32)
    H, W, d = 6, 5, 3
    v = rng.standard_normal((H * W, d))
    w = np.zeros((d, 3, 3))
    w[:, 1, 1] = [2.0, -1.0, 0.5]
    assert np.allclose(O.dwc3x3(v, w, H, W), v * w[:, 1, 1][None, :], rtol=0, atol=0)
    # single tap at (dy, dx) = (-1, +1): out[y, x] = v[y-1, x+1], zero outside
    w = np.zeros((d, 3, 3))
    w[:, 0, 2] = 1.0
    out = O.dwc3x3(v, w, H, W).reshape(H, W, d)
    g = v.reshape(H, W, d)
    exp = np.zeros_like(g)
    exp[1:, :-1] = g[:-1, 1:]
    assert np.array_equal(out, exp)


# --- backward -------------------------------------------------------------------

def _fd_case(H, W, d, r, lam, eps, T, seed, whiten, n_samples=40, h=1e-6):
    rng = _rng(seed)
    q = rng.standard_normal((H * W, d))
    v = rng.standard_normal((H * W, d))
    w = rng.standard_normal((d, 3, 3)) * 0.1
    dO = rng.standard_normal((H * W, d))
    return _fd_check(q, v, w, dO, H, W, r, lam, eps, T, whiten, rng, n_samples, n_samples // 2, h)


def _fd_check(q, v, w, dO, H, W, r, lam, eps, T, whiten, rng, n_q, n_v, h=1e-6):
    """Worst |central difference - analytic| / max|analytic| over sampled Q and V coordinates."""
    dQ, dV, f = O.unit_backward(q, v, w, dO, H, W, r, lam, eps, T, whiten)

    def loss(qq, vv):
        return float(np.sum(dO * O.unit_forward(qq, vv, w, H, W, r, lam, eps, T, whiten).O))

    def loss_attn(qq):
        # DWC(V) does not depend on Q; leaving it out keeps the difference quotient
        # above the rounding floor of the loss when the attention part is small
        return float(np.sum(dO * O.unit_forward(qq, v, w, H, W, r, lam, eps, T, whiten).O_attn))

    d = q.shape[1]
    L = f.L
    pooled_dist = np.abs(L[:, None, :] - L[None, :, :])
    off = ~np.eye(len(L), dtype=bool)
    checked = 0
    worst_q = 0.0
    scale_q = np.abs(dQ).max()
    for idx in rng.permutation(H * W * d):
        i, k = divmod(int(idx), d)
        # skip coordinates within reach of a kink of |q - l| or of |l - l'|
        if np.min(np.abs(q[i, k] - L[:, k])) < 20 * h:
            continue
        if np.min(pooled_dist[:, :, k][off], initial=np.inf) < 20 * h / (r * r):
            continue
        qp = q.copy(); qp[i, k] += h
        qm = q.copy(); qm[i, k] -= h
        fd = (loss_attn(qp) - loss_attn(qm)) / (2 * h)
        worst_q = max(worst_q, abs(fd - dQ[i, k]) / scale_q)
        checked += 1
        if checked >= n_q:
            break
    assert checked >= n_q // 2, "too few kink-free coordinates"
    worst_v = 0.0
    scale_v = np.abs(dV).max()
    for idx in rng.choice(H * W * d, size=n_v, replace=False):
        i, k = divmod(int(idx), d)
        vp = v.copy(); vp[i, k] += h
        vm = v.copy(); vm[i, k] -= h
        fd = (loss(q, vp) - loss(q, vm)) / (2 * h)
        worst_v = max(worst_v, abs(fd - dV[i, k]) / scale_v)
    return worst_q, worst_v


def check_backward_fd_long_crop(n_per_head=64, heads=None):
    """The long-sequence workload's own Q, V, dO and DWC weight, cropped to the top-left 16 x 16
    tokens of every head's 256 x 256 grid (bf16-rounded values, as the library consumes them), at
    the literal pooling window r = 16 (one landmark) and at r = 4 (16 landmarks, so that the
    Newton-Schulz chain is not trivial). Central differences in float64 against the analytic
    gradient, 64 Q and 64 V coordinates per head."""
    from laplacian_nystr_attention_avg_b200.inputs import WORKLOADS, make_crop_inputs

    wl = WORKLOADS["long"]
    for r in (16, 4):
        cw, x = make_crop_inputs(wl, 16, 16, r)
        for hh in (range(cw.heads) if heads is None else heads):
            q = x.Q[0, hh].double().numpy()
            v = x.V[0, hh].double().numpy()
            w = x.dwc[hh].double().numpy()
            dO = x.dO[0, hh].double().numpy()
            wq, wv = _fd_check(q, v, w, dO, cw.H, cw.W, r, cw.lam, cw.eps, cw.T, True,
                               _rng(1000 + 16 * r + hh), n_per_head, n_per_head)
            assert wq < 1e-6, f"dQ vs finite differences: {wq} (long crop, r={r}, head {hh})"
            assert wv < 1e-6, f"dV vs finite differences: {wv} (long crop, r={r}, head {hh})"


def check_backward_fd(cases=None):
    if cases is None:
        # 16 x 16 crops shaped like the long-sequence workload (d = 64, lam = 4):
        # r = 16 (one landmark) and r = 4 (16 landmarks, non-trivial NS), both readings
        cases = [(16, 16, 64, 16, 4.0, 1e-6, 24, 41, True),
                 (16, 16, 64, 4, 4.0, 1e-6, 24, 42, True),
                 (16, 16, 64, 4, 4.0, 1e-6, 24, 43, False),
                 (8, 8, 8, 2, 2.0, 1e-3, 24, 44, True)]
    for c in cases:
        wq, wv = _fd_case(*c)
        assert wq < 1e-6, f"dQ vs finite differences: {wq} for {c}"
        assert wv < 1e-6, f"dV vs finite differences: {wv} for {c}"


def check_backward_batch_stats_fd(n_samples=24, h=1e-6):
    # reading R12: two batch elements share the head's whitening statistics, so a token of one
    # unit moves the other unit's output too; the gradient is checked through the whole call
    B, heads = 2, 1
    q, v, w, wl = _batch_case(B, heads, 81)
    wl.eps = 1e-3
    rng = _rng(82)
    dO = rng.standard_normal(q.shape)
    dQ, dV = O.backward(q, v, w, dO, wl, batch_stats=True)

    def loss(qq, vv, attn_only=False):
        f = O.forward(qq, vv, w, wl, batch_stats=True)
        return float(np.sum(dO * (f.O_attn if attn_only else f.O)))

    N, d = q.shape[2], q.shape[3]
    Ls = [O.pool_landmarks(q[b, 0], wl.H, wl.W, wl.r) for b in range(B)]
    worst_q, checked = 0.0, 0
    scale_q = np.abs(dQ).max()
    for idx in rng.permutation(B * N * d):
        b, rest = divmod(int(idx), N * d)
        i, k = divmod(rest, d)
        L = Ls[b]
        if np.min(np.abs(q[b, 0, i, k] - L[:, k])) < 20 * h:
            continue
        pd = np.abs(L[:, None, k] - L[None, :, k])[~np.eye(len(L), dtype=bool)]
        if np.min(pd, initial=np.inf) < 20 * h / (wl.r * wl.r):
            continue
        qp = q.copy(); qp[b, 0, i, k] += h
        qm = q.copy(); qm[b, 0, i, k] -= h
        fd = (loss(qp, v, True) - loss(qm, v, True)) / (2 * h)
        worst_q = max(worst_q, abs(fd - dQ[b, 0, i, k]) / scale_q)
        checked += 1
        if checked >= n_samples:
            break
    assert checked >= n_samples // 2, "too few kink-free coordinates"
    assert worst_q < 1e-6, f"dQ vs finite differences: {worst_q}"
    worst_v, scale_v = 0.0, np.abs(dV).max()
    for idx in rng.choice(B * N * d, size=n_samples // 2, replace=False):
        b, rest = divmod(int(idx), N * d)
        i, k = divmod(rest, d)
        vp = v.copy(); vp[b, 0, i, k] += h
        vm = v.copy(); vm[b, 0, i, k] -= h
        fd = (loss(q, vp) - loss(q, vm)) / (2 * h)
        worst_v = max(worst_v, abs(fd - dV[b, 0, i, k]) / scale_v)
    assert worst_v < 1e-6, f"dV vs finite differences: {worst_v}"


# --- injectivity (the pages' claim for the exact map; see the counterexample) --------

def check_injectivity_generic():
    rng = _rng(51)
    H = W = 16
    d, r, lam, eps = 32, 4, 4.0, 1e-6
    q = rng.standard_normal((H * W, d))
    v = rng.standard_normal((H * W, d))
    f = O.unit_forward(q, v, np.zeros((d, 3, 3)), H, W, r, lam, eps, 20)
    Z = f.Ct @ f.X @ f.Ct.T            # rows z_i of the attention map
    D = cdist(Z, Z, "euclidean")
    np.fill_diagonal(D, np.inf)
    assert D.min() > 0.0, "two distinct queries produced identical attention rows"
    return float(D.min())


def nystrom_collision_example():
    """Two distinct queries with identical Nystrom rows: q + t (e_a + e_b) with
    q_a above every landmark's coordinate a and q_b below every landmark's
    coordinate b keeps every |q - l|_1, hence every C row, unchanged.
    Returns (max |C_row1 - C_row2|, ||q1 - q2||)."""
    rng = _rng(52)
    H = W = 16
    d, r, lam = 32, 4, 4.0
    q = rng.standard_normal((H * W, d))
    L = O.pool_landmarks(q, H, W, r)
    q1 = q[0].copy()
    a, b = 0, 1
    q1[a] = L[:, a].max() + 1.0
    q1[b] = L[:, b].min() - 1.0
    q2 = q1.copy()
    q2[a] += 0.25
    q2[b] += 0.25
    c1 = O.laplacian_kernel(q1[None], L, lam)
    c2 = O.laplacian_kernel(q2[None], L, lam)
    return float(np.abs(c1 - c2).max()), float(np.linalg.norm(q1 - q2))


ALL_PINS = [
    check_kernel_closed_forms, check_kernel_vs_cdist, check_pool_ramp, check_pool_vs_torch,
    check_gram_spd, check_alpha_rule, check_ns_eigen_closed_form, check_ns_vs_cholesky,
    check_ns_kappa50_and_quadratic, check_nystrom_r1_dense, check_whitening_moments,
    check_whitening_vs_sklearn, check_whitened_assembly_vs_solve, check_dwc_vs_conv2d,
    check_dwc_taps, check_backward_fd, check_injectivity_generic,
    check_batch_stats_single_batch, check_batch_stats_replicated, check_batch_stats_vs_sklearn,
    check_reading_b_vs_dense, check_reading_b_r1_is_whitened_kernel, check_cg_vs_solve,
    check_cg_error_bound, check_backward_batch_stats_fd, check_backward_fd_long_crop,
]
