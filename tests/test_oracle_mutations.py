"""Plant plausible mistakes in the CPU oracle and check that a pin catches each one.

Every mistake is planted with monkeypatch into the oracle module on the CPU; the
oracle file itself is never edited.
"""
import numpy as np
import pytest

from oracle import lfa_oracle as O
from tests import pins

_orig = {name: getattr(O, name) for name in (
    "laplacian_kernel", "l1_distances", "pool_landmarks", "landmark_gram", "newton_schulz",
    "whiten_columns", "dwc3x3", "_sign_contractions", "select_alpha", "pooled_column_stats",
    "batch_groups", "unit_forward_reading_b", "cg_solve", "_whitening_backward")}


def _kernel_no_lambda(X, Y, lam):
    return np.exp(-_orig["l1_distances"](X, Y))


def _kernel_l2(X, Y, lam):
    X = np.asarray(X, float)
    Y = np.asarray(Y, float)
    return np.exp(-np.sqrt(((X[:, None, :] - Y[None, :, :]) ** 2).sum(-1)) / lam)


def _pool_transposed_window(Qu, H, W, r):
    N, d = Qu.shape
    g = Qu.reshape(r, H // r, r, W // r, d)     # window/grid axes swapped
    return g.mean(axis=(0, 2)).reshape(-1, d)


def _gram_without_eps(L, lam, eps):
    return O.laplacian_kernel(L, L, lam)


def _ns_wrong_update(W, alpha, T, keep_iterates=False):
    m = W.shape[0]
    X = alpha * W.T
    its = [X]
    for _ in range(T):
        X = X @ (np.eye(m) - W @ X)          # "I" where the update needs "2I"
        its.append(X)
    res = [(0.0, 0.0)] * (T + 1)
    return X, res, (its if keep_iterates else None)


def _ns_wrong_x0(W, alpha, T, keep_iterates=False):
    # X_0 = alpha W W^T (the condition's matrix) instead of alpha W^T
    m = W.shape[0]
    X = alpha * W @ W.T
    its = [X]
    for _ in range(T):
        X = X @ (2.0 * np.eye(m) - W @ X)
        its.append(X)
    res = [(0.0, 0.0)] * (T + 1)
    return X, res, (its if keep_iterates else None)


def _alpha_pages_always(W):
    ac = _orig["select_alpha"](W)
    ac.alpha = ac.alpha_pages
    ac.fallback = False
    return ac


def _whiten_plus_mu(C, eps):
    N = C.shape[0]
    mu = C.mean(axis=0)
    var = ((C - mu) ** 2).mean(axis=0)
    return (C + mu) / np.sqrt(var + eps) + 1.0 / N, mu, var


def _whiten_no_offset(C, eps):
    Ct, mu, var = _orig["whiten_columns"](C, eps)
    return Ct - 1.0 / C.shape[0], mu, var


def _whiten_sample_var(C, eps):
    N = C.shape[0]
    mu = C.mean(axis=0)
    var = ((C - mu) ** 2).sum(axis=0) / (N - 1)
    return (C - mu) / np.sqrt(var + eps) + 1.0 / N, mu, var


def _pooled_sample_var(Cs):
    S = np.concatenate(Cs, axis=0)
    mu = S.mean(axis=0)
    return mu, ((S - mu) ** 2).sum(axis=0) / (S.shape[0] - 1)


def _pooled_first_unit_only(Cs):
    return _orig["pooled_column_stats"](Cs[:1])


def _groups_across_heads(B, heads):
    return [list(range(B * heads))]


def _reading_b_variant(uncentred_cov=False, no_offset=False, sample_var=False):
    def f(Qu, Vu, w, H, W, r, lam, eps, T):
        Qu = np.asarray(Qu, float)
        Vu = np.asarray(Vu, float)
        L = O.pool_landmarks(Qu, H, W, r)
        C = O.laplacian_kernel(Qu, L, lam)
        Wm = O.landmark_gram(L, lam, eps)
        X, _, _ = O.newton_schulz(Wm, O.select_alpha(Wm).alpha, T)
        N = C.shape[0]
        cbar = C.mean(axis=0)
        Cc = C - cbar
        S = (C.T @ C if uncentred_cov else Cc.T @ Cc) / (N - 1 if sample_var else N)
        var = np.einsum("jl,lk,jk->j", C, X.T @ S @ X, C)
        M = X @ (C.T @ (Vu / np.sqrt(var + eps)[:, None]))
        Oa = Cc @ M + (0.0 if no_offset else Vu.sum(axis=0)[None, :] / N)
        return O.UnitForwardB(C, X, cbar, S, C @ (X.T @ cbar), var, Oa, Oa)
    return f


def _cg_steepest_descent(W, B, iters, dtype=np.float64):
    # beta = 0: every direction is the residual (steepest descent), no conjugacy
    W = np.asarray(W, dtype=dtype)
    Y = np.zeros_like(np.asarray(B, dtype=dtype))
    R = np.asarray(B, dtype=dtype).copy()
    for _ in range(iters):
        WR = W @ R
        a = (R * R).sum(axis=0) / (R * WR).sum(axis=0)
        Y = Y + a * R
        R = R - a * WR
    return Y


def _whitening_backward_per_unit(dCts, Cs, mu, var, eps):
    # each unit's reverse mode on its own rows although the statistics are shared
    return [_orig["_whitening_backward"]([g], [C], mu, var, eps)[0] for g, C in zip(dCts, Cs)]


def _dwc_convolution(Vu, w, H, W):
    return _orig["dwc3x3"](Vu, w[:, ::-1, ::-1].copy(), H, W)


def _sign_as_printed(Qu, L, dD):
    dq, dl = _orig["_sign_contractions"](Qu, L, dD)
    return -dq, -dl


MUTATIONS = [
    ("kernel_missing_lambda", "laplacian_kernel", _kernel_no_lambda, [pins.check_kernel_closed_forms]),
    ("kernel_l2_distance", "laplacian_kernel", _kernel_l2, [pins.check_kernel_vs_cdist]),
    ("pool_transposed_window", "pool_landmarks", _pool_transposed_window, [pins.check_pool_ramp]),
    ("gram_without_eps", "landmark_gram", _gram_without_eps, [pins.check_gram_spd]),
    ("ns_wrong_update", "newton_schulz", _ns_wrong_update, [pins.check_ns_eigen_closed_form]),
    ("ns_wrong_x0", "newton_schulz", _ns_wrong_x0, [pins.check_ns_eigen_closed_form]),
    ("alpha_printed_without_check", "select_alpha", _alpha_pages_always, [pins.check_alpha_rule]),
    ("whiten_plus_mu", "whiten_columns", _whiten_plus_mu, [pins.check_whitening_moments]),
    ("whiten_no_offset", "whiten_columns", _whiten_no_offset, [pins.check_whitening_moments]),
    ("whiten_sample_variance", "whiten_columns", _whiten_sample_var, [pins.check_whitening_vs_sklearn]),
    ("dwc_convolution_not_correlation", "dwc3x3", _dwc_convolution, [pins.check_dwc_vs_conv2d]),
    ("batch_stats_sample_variance", "pooled_column_stats", _pooled_sample_var, [pins.check_batch_stats_vs_sklearn]),
    ("batch_stats_first_unit_only", "pooled_column_stats", _pooled_first_unit_only,
     [pins.check_batch_stats_vs_sklearn]),
    ("batch_stats_pooled_across_heads", "batch_groups", _groups_across_heads, [pins.check_batch_stats_vs_sklearn]),
    ("batch_stats_backward_per_unit", "_whitening_backward", _whitening_backward_per_unit,
     [pins.check_backward_batch_stats_fd]),
    ("cg_without_conjugacy", "cg_solve", _cg_steepest_descent, [pins.check_cg_vs_solve, pins.check_cg_error_bound]),
    ("reading_b_uncentred_covariance", "unit_forward_reading_b", _reading_b_variant(uncentred_cov=True),
     [pins.check_reading_b_vs_dense]),
    ("reading_b_no_offset", "unit_forward_reading_b", _reading_b_variant(no_offset=True),
     [pins.check_reading_b_vs_dense]),
    ("reading_b_sample_variance", "unit_forward_reading_b", _reading_b_variant(sample_var=True),
     [pins.check_reading_b_vs_dense, pins.check_reading_b_r1_is_whitened_kernel]),
    ("kernel_gradient_sign_as_printed", "_sign_contractions", _sign_as_printed,
     [lambda: pins.check_backward_fd([(8, 8, 8, 2, 2.0, 1e-3, 24, 44, True)])]),
]


@pytest.mark.parametrize("name,attr,fn,catchers", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, name, attr, fn, catchers):
    monkeypatch.setattr(O, attr, fn)
    caught = False
    for check in catchers:
        try:
            check()
        except (AssertionError, np.linalg.LinAlgError, ValueError, FloatingPointError):
            caught = True
    assert caught, f"planted mistake {name!r} passed every pin"
