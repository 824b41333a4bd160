"""CPU oracle for Laplacian-kernel Nystrom attention -- TEST INFRASTRUCTURE ONLY.

Plain, slow, float64 numpy restatement of what the attention block computes.
Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference legs may import it. The CUDA library never calls it and shares no
code, header, table or helper with it.

Sources (cited below by these tags, page title + section):
  [P1] papernotes.org ICLR 2026 note "LaplacianFormer：用拉普拉斯核重新思考线性注意力"
       sections: 研究背景与动机 (核心 idea), 方法详解 / 整体框架 (flowchart),
       关键设计 1 (injective whitened map), 关键设计 2 (Nystrom),
       关键设计 3 (Newton-Schulz + CUDA).
  [P2] shd-paper.top summary "LaplacianFormer:Rethinking Linear Attention with
       Laplacian Kernel" (abstract; pipeline summary in §方法详解).

Readings taken where the pages are silent or garbled (each one is listed in the
design notes with its reason):
  R1  keys are the queries: landmarks are pooled from Q and C is query-vs-landmark
      ([P1] 关键设计 2), so one point set feeds both C and W.
  R2  pooling: non-overlapping r x r windows, stride r, landmark order row-major.
  R3  the same eps regularises W (关键设计 3) and the whitening root (关键设计 1).
  R4  alpha = 2/||W||_2 is tested against ||I - alpha W W^T||_2 < 1 as printed; when
      the test fails (it always does: W has unit diagonal so ||W||_2 > 1) the
      oracle uses alpha = 1/||W||_2^2 and raises a flag.
  R5  whitening statistics are per landmark column over the N rows of one
      (batch, head) unit, population variance (divide by N).
  R6  "Reading A": the whitened C~ = (C - mu)/sqrt(var + eps) + 1/N replaces C on
      both sides of the Nystrom product, O_attn = C~ (X (C~^T V)).
  R7  no row normalisation of Z V (the pages give none).
  R8  DWC: 3x3 depthwise cross-correlation, zero padding 1, stride 1, no bias,
      weights fixed (no weight gradient).
  R9  the printed kernel gradient (+1/lam) sign(x - y) k has the wrong sign; the
      oracle differentiates k = exp(-||x - y||_1 / lam) itself, giving
      -(1/lam) sign(x - y) k, with sign(0) = 0.
  R10 alpha is held constant in the backward pass (stop-gradient).
  R11 exactly T Newton-Schulz steps, no early exit.
  R12 (alternative reading of R5, selected by batch_stats=True) the note's whitening
      statistics "over a batch" of similarity vectors: mu and var of landmark column l
      are taken over the B*N rows of every unit that shares the head h (all batch
      elements), population variance; C~ of each unit is then formed as in R6 with
      that unit's own N in the 1/N offset. Its reverse mode shares the whitening's
      batch-norm backward across those units (backward(..., batch_stats=True)).
  R13 (alternative reading of R6, "Reading B", unit_forward_reading_b) the whitening acts
      on the columns of the whole Nystrom similarity matrix G^ = C X C^T (N x N, one
      column per key token j): g~_j = (g_j - mean_i g_ij) / sqrt(var_i g_ij + eps) + 1/N,
      population variance, and O_attn = G~ V. In factored form, with c_j the j-th row
      of C, c- the column mean of C, Cc = C - 1 c-^T and S = Cc^T Cc / N:
      mean_i g_ij = c-^T X c_j, var_i g_ij = c_j^T X^T S X c_j, and
      O_attn = Cc X C^T D^-1/2 V + (1/N) 1 (1^T V), D = diag(var_j + eps). Forward only.

Parity pins (tests/test_oracle_*.py): closed forms of the kernel, scipy cdist,
torch avg_pool2d / conv2d in float64, the per-step eigen closed form of
Newton-Schulz, a Cholesky inverse, the r = 1 Nystrom identity against a dense
O(N^2) product, sklearn's StandardScaler, whitening moments, and central finite
differences for the backward pass. The whitening placement (R6) itself is
"parity unpinned": nothing on the pages fixes it beyond self-consistency.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor
from typing import List, Optional, Tuple

import numpy as np

_ROW_CHUNK = 512
_THREADS = 8


def set_threads(n: int) -> None:
    """Threads used for the row-chunked distance loops (numpy releases the GIL)."""
    global _THREADS
    _THREADS = max(1, int(n))


def _chunked(n_rows: int, fn, threads: Optional[int] = None):
    starts = list(range(0, n_rows, _ROW_CHUNK))
    t = _THREADS if threads is None else threads
    if t <= 1 or len(starts) == 1:
        return [fn(s, min(s + _ROW_CHUNK, n_rows)) for s in starts]
    with ThreadPoolExecutor(max_workers=t) as ex:
        return list(ex.map(lambda s: fn(s, min(s + _ROW_CHUNK, n_rows)), starts))


# ---------------------------------------------------------------------------
# Building blocks
# ---------------------------------------------------------------------------

def pool_landmarks(Qu: np.ndarray, H: int, W: int, r: int) -> np.ndarray:
    """Landmarks L = r x r average pool of the query map ([P1] 关键设计 2, R2).

    Qu: [N, d] tokens of one unit, token n = y*W + x. Returns L [m, d] with
    landmark index l = Y*(W/r) + X for window (Y, X).
    """
    N, d = Qu.shape
    assert N == H * W and H % r == 0 and W % r == 0
    g = Qu.reshape(H // r, r, W // r, r, d)
    L = np.zeros((H // r, W // r, d))
    for dy in range(r):
        for dx in range(r):
            L += g[:, dy, :, dx, :]
    return (L / (r * r)).reshape(-1, d)


def l1_distances(X: np.ndarray, Y: np.ndarray) -> np.ndarray:
    """D[i, j] = sum_k |x_ik - y_jk| ([P1] 研究背景与动机, 核心 idea: the l1 norm)."""
    X = np.asarray(X, dtype=np.float64)
    Y = np.asarray(Y, dtype=np.float64)

    def rows(a, b):
        return np.abs(X[a:b, None, :] - Y[None, :, :]).sum(axis=2)

    return np.concatenate(_chunked(X.shape[0], rows), axis=0)


def laplacian_kernel(X: np.ndarray, Y: np.ndarray, lam: float) -> np.ndarray:
    """k(x, y) = exp(-||x - y||_1 / lam) for every pair ([P1] 核心 idea; 关键设计 2)."""
    return np.exp(-l1_distances(X, Y) / lam)


def landmark_gram(L: np.ndarray, lam: float, eps: float) -> np.ndarray:
    """W = [k(l_a, l_b)] + eps I ([P1] 关键设计 2 defines W; 关键设计 3 adds eps I)."""
    return laplacian_kernel(L, L, lam) + eps * np.eye(L.shape[0])


@dataclasses.dataclass
class AlphaChoice:
    alpha: float            # the alpha actually used for X_0 = alpha W^T
    alpha_pages: float      # 2 / ||W||_2, as printed
    cond_pages: float       # ||I - alpha_pages W W^T||_2
    fallback: bool          # True when the printed condition fails (R4)
    norm2: float            # ||W||_2


def select_alpha(W: np.ndarray) -> AlphaChoice:
    """alpha per [P1] 关键设计 3, with the R4 fallback alpha = 1/||W||_2^2."""
    norm2 = float(np.linalg.norm(W, 2))
    a = 2.0 / norm2
    m = W.shape[0]
    cond = float(np.linalg.norm(np.eye(m) - a * (W @ W.T), 2))
    if cond < 1.0:
        return AlphaChoice(a, a, cond, False, norm2)
    return AlphaChoice(1.0 / norm2 ** 2, a, cond, True, norm2)


def newton_schulz(W: np.ndarray, alpha: float, T: int, keep_iterates: bool = False):
    """X_0 = alpha W^T; X_{k+1} = X_k (2I - W X_k), exactly T steps ([P1] 关键设计 3, R11).

    Returns (X_T, residuals, iterates) where residuals[k] = (||I - W X_k||_F,
    ||I - W X_k||_2) for k = 0..T and iterates = [X_0..X_T] when requested.
    """
    m = W.shape[0]
    I = np.eye(m)
    X = alpha * W.T
    its = [X] if keep_iterates else None
    res = []
    for _ in range(T):
        R = I - W @ X
        res.append((float(np.linalg.norm(R, "fro")), float(np.linalg.norm(R, 2))))
        X = X @ (2.0 * I - W @ X)
        if keep_iterates:
            its.append(X)
    R = I - W @ X
    res.append((float(np.linalg.norm(R, "fro")), float(np.linalg.norm(R, 2))))
    return X, res, its


def cg_solve(W: np.ndarray, B: np.ndarray, iters: int, dtype=np.float64) -> np.ndarray:
    """Conjugate gradients for the SPD system W Y = B: the solver the note ablates against
    Newton-Schulz ([P1] 关键设计 3 and its ablation). One independent Hestenes-Stiefel recursion
    per right-hand-side column, Y_0 = 0, exactly ``iters`` iterations, every operation in
    ``dtype`` (float64, or float32 to see the single-precision behaviour).
    """
    W = np.asarray(W, dtype=dtype)
    B = np.asarray(B, dtype=dtype)
    Y = np.zeros_like(B)
    R = B.copy()
    P = R.copy()
    rr = (R * R).sum(axis=0)
    for _ in range(iters):
        WP = W @ P
        pwp = (P * WP).sum(axis=0)
        a = np.divide(rr, pwp, out=np.zeros_like(rr), where=pwp > 0)
        Y = Y + a * P
        R = R - a * WP
        rr_new = (R * R).sum(axis=0)
        beta = np.divide(rr_new, rr, out=np.zeros_like(rr), where=rr > 0)
        P = R + beta * P
        rr = rr_new
    return Y


def newton_schulz_dtype(W: np.ndarray, alpha: float, T: int, dtype=np.float32) -> np.ndarray:
    """newton_schulz's X_T with every product in ``dtype`` (the single-precision counterpart
    used to compare the two solvers' robustness)."""
    W = np.asarray(W, dtype=dtype)
    I2 = 2.0 * np.eye(W.shape[0], dtype=dtype)
    X = dtype(alpha) * W.T
    for _ in range(T):
        X = X @ (I2 - W @ X)
    return X


def whiten_columns(C: np.ndarray, eps: float):
    """Diagonal centring + whitening of [P1] 关键设计 1 (R5): per column mean mu and
    population variance var over the N rows; C~ = (C - mu)/sqrt(var + eps) + 1/N.

    Returns (C~, mu, var).
    """
    N = C.shape[0]
    mu = C.mean(axis=0)
    var = ((C - mu) ** 2).mean(axis=0)
    return (C - mu) / np.sqrt(var + eps) + 1.0 / N, mu, var


def pooled_column_stats(Cs: List[np.ndarray]):
    """R12: per-column mean and population variance over the stacked rows of several
    units' cross kernels ([P1] 关键设计 1, statistics over a batch). Returns (mu, var)."""
    S = np.concatenate([np.asarray(C, dtype=np.float64) for C in Cs], axis=0)
    mu = S.mean(axis=0)
    var = ((S - mu) ** 2).mean(axis=0)
    return mu, var


def batch_groups(B: int, heads: int) -> List[List[int]]:
    """R12: the units u = b*heads + h that pool their statistics: one group per head."""
    return [[b * heads + h for b in range(B)] for h in range(heads)]


def dwc3x3(Vu: np.ndarray, w: np.ndarray, H: int, W: int) -> np.ndarray:
    """DWC(V): per-channel 3x3 cross-correlation with zero padding 1 ([P1] 整体框架
    flowchart node "DWC(V) 深度卷积"; 关键设计 1 output ZV + DWC(V); R8).

    Vu: [N, d]; w: [d, 3, 3] with w[k, dy+1, dx+1] multiplying V[y+dy, x+dx, k].
    """
    N, d = Vu.shape
    g = Vu.reshape(H, W, d)
    pad = np.zeros((H + 2, W + 2, d))
    pad[1:-1, 1:-1] = g
    out = np.zeros((H, W, d))
    for a in range(3):
        for b in range(3):
            out += w[:, a, b][None, None, :] * pad[a:a + H, b:b + W, :]
    return out.reshape(N, d)


def dwc3x3_transpose(G: np.ndarray, w: np.ndarray, H: int, W: int) -> np.ndarray:
    """Adjoint of dwc3x3 in its input: dV[y', x'] = sum_{a,b} w[a,b] G[y'-a+1, x'-b+1]."""
    N, d = G.shape
    g = G.reshape(H, W, d)
    pad = np.zeros((H + 2, W + 2, d))
    pad[1:-1, 1:-1] = g
    out = np.zeros((H, W, d))
    for a in range(3):
        for b in range(3):
            out += w[:, a, b][None, None, :] * pad[2 - a:2 - a + H, 2 - b:2 - b + W, :]
    return out.reshape(N, d)


# ---------------------------------------------------------------------------
# One (batch, head) unit
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class UnitForward:
    L: np.ndarray           # [m, d] landmarks
    C: np.ndarray           # [N, m] cross kernel
    W: np.ndarray           # [m, m] landmark kernel + eps I
    alpha: AlphaChoice
    X: np.ndarray           # [m, m] X_T
    ns_residuals: List[Tuple[float, float]]
    Ct: np.ndarray          # [N, m] the matrix used in the product (whitened or raw C)
    mu: Optional[np.ndarray]
    var: Optional[np.ndarray]
    A: np.ndarray           # Ct^T V   [m, d]
    M: np.ndarray           # X A      [m, d]
    O_attn: np.ndarray      # Ct M     [N, d]
    O: np.ndarray           # O_attn + DWC(V)
    iterates: Optional[List[np.ndarray]] = None


def unit_forward(Qu, Vu, w, H, W, r, lam, eps, T, whiten=True, keep_iterates=False,
                 stats=None) -> UnitForward:
    """Forward pass of one unit, in the pages' order ([P1] 整体框架 flowchart):
    pool -> Laplacian kernels -> Newton-Schulz W^+ -> whitening -> C~ (X (C~^T V)) + DWC(V).

    ``stats`` = (mu, var) replaces the unit's own column statistics (R12).
    """
    Qu = np.asarray(Qu, dtype=np.float64)
    Vu = np.asarray(Vu, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    L = pool_landmarks(Qu, H, W, r)
    C = laplacian_kernel(Qu, L, lam)
    Wm = landmark_gram(L, lam, eps)
    ac = select_alpha(Wm)
    X, res, its = newton_schulz(Wm, ac.alpha, T, keep_iterates)
    if whiten and stats is not None:
        mu, var = stats
        Ct = (C - mu) / np.sqrt(var + eps) + 1.0 / C.shape[0]
    elif whiten:
        Ct, mu, var = whiten_columns(C, eps)
    else:
        Ct, mu, var = C, None, None
    A = Ct.T @ Vu
    M = X @ A
    O_attn = Ct @ M
    O = O_attn + dwc3x3(Vu, w, H, W)
    return UnitForward(L, C, Wm, ac, X, res, Ct, mu, var, A, M, O_attn, O, its)


def _sign_contractions(Qu, L, dD):
    """dq[i,k] = sum_l dD[i,l] sign(q_ik - l_lk);  dl[l,k] = -sum_i dD[i,l] sign(q_ik - l_lk)."""
    N, d = Qu.shape

    def rows(a, b):
        S = np.sign(Qu[a:b, None, :] - L[None, :, :])           # [rows, m, d]
        dq = np.einsum("il,ilk->ik", dD[a:b], S)
        dl = -np.einsum("il,ilk->lk", dD[a:b], S)
        return dq, dl

    parts = _chunked(N, rows)
    dQ = np.concatenate([p[0] for p in parts], axis=0)
    dL = np.sum([p[1] for p in parts], axis=0)
    return dQ, dL


def _backward_to_ct(Qu, Vu, w, dOu, H, W, r, lam, eps, T, whiten, stats=None):
    """First half of the reverse mode: through O = Ct M + DWC(V), M = X A, A = Ct^T V.
    Returns (fwd, dCt, dX, dV)."""
    Qu = np.asarray(Qu, dtype=np.float64)
    Vu = np.asarray(Vu, dtype=np.float64)
    dO = np.asarray(dOu, dtype=np.float64)
    f = unit_forward(Qu, Vu, w, H, W, r, lam, eps, T, whiten, keep_iterates=True, stats=stats)
    dV = dwc3x3_transpose(dO, np.asarray(w, dtype=np.float64), H, W)
    dM = f.Ct.T @ dO
    dX = dM @ f.A.T
    dA = f.X.T @ dM
    dCt = dO @ f.M.T + Vu @ dA.T
    dV = dV + f.Ct @ dA
    return f, dCt, dX, dV


def _backward_from_c(Qu, f, dC, dX, H, W, r, lam, eps, T):
    """Second half: through C = exp(-D/lam), the Newton-Schulz chain, W and the pooling.
    Returns dQ."""
    Qu = np.asarray(Qu, dtype=np.float64)
    N, d = Qu.shape
    m = f.L.shape[0]
    dD = -(f.C * dC) / lam
    dQ, dL = _sign_contractions(Qu, f.L, dD)
    # Newton-Schulz: X_{k+1} = 2 X_k - X_k W X_k, X_0 = alpha W^T (alpha held constant)
    Wm = f.W
    G = dX
    dW = np.zeros((m, m))
    for k in range(T - 1, -1, -1):
        Xk = f.iterates[k]
        dW -= Xk.T @ G @ Xk.T
        G = 2.0 * G - G @ Xk.T @ Wm.T - Wm.T @ Xk.T @ G
    dW += f.alpha.alpha * G.T
    # W = exp(-E/lam) + eps I,  E_ab = sum_k |l_ak - l_bk|
    dE = -(Wm - eps * np.eye(m)) * dW / lam
    Sl = np.sign(f.L[:, None, :] - f.L[None, :, :])            # [m, m, d]
    dL = dL + np.einsum("ab,abk->ak", dE, Sl) - np.einsum("ab,abk->bk", dE, Sl)
    # L = pool(Q): every token of window l receives dL_l / r^2
    Wr = W // r
    g = dL.reshape(H // r, 1, Wr, 1, d) / (r * r)
    return dQ + np.broadcast_to(g, (H // r, r, Wr, r, d)).reshape(N, d)


def _whitening_backward(dCts, Cs, mu, var, eps):
    """Batch-norm form of the whitening's reverse mode (population variance) over the stacked
    rows of the listed units, whose statistics (mu, var) are shared: returns one dC per unit."""
    s = 1.0 / np.sqrt(var + eps)
    Chat = np.concatenate([(C - mu) * s for C in Cs])
    dCt = np.concatenate(dCts)
    dC = s * (dCt - dCt.mean(axis=0) - Chat * (dCt * Chat).mean(axis=0))
    return np.split(dC, np.cumsum([len(C) for C in Cs])[:-1])


def unit_backward(Qu, Vu, w, dOu, H, W, r, lam, eps, T, whiten=True):
    """Reverse mode through unit_forward (R9 kernel sign, R10 alpha constant).

    Returns (dQ [N, d], dV [N, d], fwd). The loss is <dO, O>.
    """
    f, dCt, dX, dV = _backward_to_ct(Qu, Vu, w, dOu, H, W, r, lam, eps, T, whiten)
    # whitening (population-variance batch-norm form), then C = exp(-D/lam)
    dC = _whitening_backward([dCt], [f.C], f.mu, f.var, eps)[0] if whiten else dCt
    dQ = _backward_from_c(Qu, f, dC, dX, H, W, r, lam, eps, T)
    return dQ, dV, f


@dataclasses.dataclass
class UnitForwardB:
    C: np.ndarray           # [N, m] cross kernel
    X: np.ndarray           # [m, m] X_T
    cbar: np.ndarray        # [m] column mean of C
    S: np.ndarray           # [m, m] covariance of the columns of C
    col_mean: np.ndarray    # [N] mean over i of column j of G^ = C X C^T
    col_var: np.ndarray     # [N] its population variance
    O_attn: np.ndarray      # G~ V
    O: np.ndarray           # O_attn + DWC(V)


def unit_forward_reading_b(Qu, Vu, w, H, W, r, lam, eps, T) -> UnitForwardB:
    """R13: column whitening of the full Nystrom similarity matrix ([P1] 关键设计 1 applied to
    关键设计 2's G^), in the O(N m^2) factored form; the steps before X as in unit_forward."""
    Qu = np.asarray(Qu, dtype=np.float64)
    Vu = np.asarray(Vu, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    L = pool_landmarks(Qu, H, W, r)
    C = laplacian_kernel(Qu, L, lam)
    Wm = landmark_gram(L, lam, eps)
    ac = select_alpha(Wm)
    X, _, _ = newton_schulz(Wm, ac.alpha, T)
    N = C.shape[0]
    cbar = C.mean(axis=0)
    Cc = C - cbar
    S = Cc.T @ Cc / N
    K = X.T @ S @ X
    col_mean = C @ (X.T @ cbar)                       # c-^T X c_j for every j
    col_var = np.einsum("jl,lk,jk->j", C, K, C)       # c_j^T K c_j
    dinv = 1.0 / np.sqrt(col_var + eps)
    M = X @ (C.T @ (dinv[:, None] * Vu))              # X C^T D^-1/2 V
    O_attn = Cc @ M + Vu.sum(axis=0)[None, :] / N
    O = O_attn + dwc3x3(Vu, w, H, W)
    return UnitForwardB(C, X, cbar, S, col_mean, col_var, O_attn, O)


def forward_reading_b(Q, V, dwc, wl, units=None):
    """R13 over all (or the listed) units of a workload: returns (O, O_attn, [UnitForwardB])."""
    Q = np.asarray(Q, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    w = np.asarray(dwc, dtype=np.float64)
    B, nh, N, d = Q.shape
    O = np.zeros_like(Q)
    Oa = np.zeros_like(Q)
    us = []
    for u in (range(B * nh) if units is None else units):
        b, h = divmod(u, nh)
        f = unit_forward_reading_b(Q[b, h], V[b, h], w[h], wl.H, wl.W, wl.r, wl.lam, wl.eps, wl.T)
        O[b, h] = f.O
        Oa[b, h] = f.O_attn
        us.append(f)
    return O, Oa, us


# ---------------------------------------------------------------------------
# Whole calls ([B, heads, N, d] tensors)
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Forward:
    O: np.ndarray           # [B, heads, N, d]
    O_attn: np.ndarray
    units: List[UnitForward]


def forward(Q, V, dwc, wl, whiten=True, units=None, keep_units=True, batch_stats=False) -> Forward:
    """Oracle forward over all (or the listed) units of a workload.

    Q, V: [B, heads, N, d] array-likes (float values already in the storage
    precision); dwc: [heads, d, 3, 3]. ``units`` restricts to a list of flat
    unit indices u = b*heads + h (others are left zero). ``batch_stats`` selects
    the R12 reading: whitening statistics pooled over the batch, per head (the
    pooled statistics always use every batch element, also when ``units`` is set).
    """
    Q = np.asarray(Q, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    w = np.asarray(dwc, dtype=np.float64)
    B, nh, N, d = Q.shape
    O = np.zeros_like(Q)
    Oa = np.zeros_like(Q)
    us = []
    todo = range(B * nh) if units is None else units
    pooled = {}
    if whiten and batch_stats:
        for grp in batch_groups(B, nh):
            Cs = []
            for u in grp:
                b, h = divmod(u, nh)
                L = pool_landmarks(Q[b, h], wl.H, wl.W, wl.r)
                Cs.append(laplacian_kernel(Q[b, h], L, wl.lam))
            st = pooled_column_stats(Cs)
            for u in grp:
                pooled[u] = st
    for u in todo:
        b, h = divmod(u, nh)
        f = unit_forward(Q[b, h], V[b, h], w[h], wl.H, wl.W, wl.r, wl.lam, wl.eps, wl.T, whiten,
                         stats=pooled.get(u))
        O[b, h] = f.O
        Oa[b, h] = f.O_attn
        us.append(f if keep_units else None)
    return Forward(O, Oa, us)


def backward(Q, V, dwc, dO, wl, whiten=True, units=None, batch_stats=False):
    """Oracle gradients (dQ, dV), [B, heads, N, d], for the loss <dO, O>.

    ``batch_stats`` (R12): the statistics, and so the whitening's reverse mode, are shared by
    the units of a head; every unit is then computed (``units`` is ignored).
    """
    if whiten and batch_stats:
        return _backward_batch_stats(Q, V, dwc, dO, wl)
    Q = np.asarray(Q, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    w = np.asarray(dwc, dtype=np.float64)
    B, nh, N, d = Q.shape
    dQ = np.zeros_like(Q)
    dV = np.zeros_like(Q)
    todo = range(B * nh) if units is None else units
    for u in todo:
        b, h = divmod(u, nh)
        gq, gv, _ = unit_backward(Q[b, h], V[b, h], w[h], dO[b, h], wl.H, wl.W, wl.r,
                                  wl.lam, wl.eps, wl.T, whiten)
        dQ[b, h] = gq
        dV[b, h] = gv
    return dQ, dV


def _backward_batch_stats(Q, V, dwc, dO, wl):
    """R12 reverse mode: per head, the whitening backward runs over the stacked rows of all
    batch elements (their shared mean and variance), the rest per unit."""
    Q = np.asarray(Q, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    w = np.asarray(dwc, dtype=np.float64)
    B, nh, N, d = Q.shape
    dQ = np.zeros_like(Q)
    dV = np.zeros_like(Q)
    for grp in batch_groups(B, nh):
        Cs = []
        for u in grp:
            b, h = divmod(u, nh)
            L = pool_landmarks(Q[b, h], wl.H, wl.W, wl.r)
            Cs.append(laplacian_kernel(Q[b, h], L, wl.lam))
        mu, var = pooled_column_stats(Cs)
        halves = []
        for u in grp:
            b, h = divmod(u, nh)
            halves.append(_backward_to_ct(Q[b, h], V[b, h], w[h], dO[b, h], wl.H, wl.W, wl.r, wl.lam,
                                          wl.eps, wl.T, True, stats=(mu, var)))
        dCs = _whitening_backward([hv[1] for hv in halves], [hv[0].C for hv in halves], mu, var, wl.eps)
        for u, (f, _, dX, dVu), dC in zip(grp, halves, dCs):
            b, h = divmod(u, nh)
            dQ[b, h] = _backward_from_c(Q[b, h], f, dC, dX, wl.H, wl.W, wl.r, wl.lam, wl.eps, wl.T)
            dV[b, h] = dVu
    return dQ, dV
