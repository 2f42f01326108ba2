"""fp64 CPU oracle for the fitter that produces the decomposition's factors
from a dense matrix (the step before the GEMV).

TEST INFRASTRUCTURE ONLY: only tests/, ``__graft_entry__.smoke()`` and the
CPU legs of ``bench.py`` may import this module.  The library never imports
it, and it imports nothing from the library.

The FluxBin page (Methodology, 1. Algorithm innovation: the decoupled
row-column binary decomposition and the Hessian-guided saliency-aware hybrid
bases) defines what the factors are -- W_hat = sum_k (alpha_r^(k)
alpha_c^(k)^T) (.) B^(k), plus extra bases on a salient column set S chosen
with second-order (Hessian) information -- but prints no fitting procedure.
This module takes the plainest reading of it:

* Saliency, with the diagonal of the Hessian as the proxy.  For calibration
  activations X [T][N] the layer's Hessian is proportional to X^T X; its
  diagonal is h_j = sum_t X[t][j]^2, and the loss increase of dropping column
  j under a diagonal Hessian is proportional to h_j * sum_i W[i][j]^2, the
  column's score.  S is the nS columns of largest score (equal scores: the
  lower column first), listed in ascending order.
* Greedy residual bases.  Starting from R = W, each base takes
  B = sign(R) (R >= 0 gives +1) and the row and column scales that best fit
  |R| = R (.) B as a rank-one matrix alpha_r alpha_c^T in least squares, found
  by `sweeps` alternating least-squares sweeps from alpha_c = 1:
  alpha_r = |R| alpha_c / ||alpha_c||^2, then alpha_c = |R|^T alpha_r /
  ||alpha_r||^2 (a zero norm gives zero scales).  With B fixed to sign(R)
  this is the least-squares choice of the scales, and for scales of fixed
  positive product sign(R) is the least-squares choice of B.  Then
  R -= (alpha_r alpha_c^T) (.) B.
* Salient refinement: after the K global bases, Ks more bases fitted the same
  way to the residual's salient columns R[:, S] (the global bases still cover
  every column; the two terms are summed).

Parity status: every function is pinned by ``tests/test_fit_oracle.py``
(exact recovery of a rank-one magnitude, the leading singular pair from
numpy's SVD, never-growing residuals, constructed saliency cases, and the
fitted factors run through the GEMV oracle); none is "parity unpinned".
"""

from __future__ import annotations

from typing import Dict

import numpy as np


def _sign(R: np.ndarray) -> np.ndarray:
    """+1 where R >= 0 (zero and negative zero included), else -1."""
    return np.where(R >= 0, 1, -1).astype(np.int8)


def _magnitude(R: np.ndarray) -> np.ndarray:
    return np.abs(R)


def _norm2(v: np.ndarray) -> float:
    return float(np.dot(v, v))


def _scaled(num: np.ndarray, den: float) -> np.ndarray:
    return num / den if den > 0 else np.zeros_like(num)


def saliency_scores(W: np.ndarray, X: np.ndarray) -> np.ndarray:
    """score_j = (sum_t X[t][j]^2) * (sum_i W[i][j]^2), in fp64."""
    W = np.asarray(W, np.float64)
    X = np.asarray(X, np.float64)
    h = np.einsum("tj,tj->j", X, X)
    w = np.einsum("ij,ij->j", W, W)
    return h * w


def select_salient(score: np.ndarray, nS: int) -> np.ndarray:
    """The nS columns of largest score, equal scores taking the lower column
    first, returned in ascending column order (uint32)."""
    score = np.asarray(score)
    N = score.shape[0]
    if not 0 <= nS <= N:
        raise ValueError("nS out of range")
    # descending score, then ascending column: a stable sort on -score
    order = np.argsort(-score, kind="stable")
    return np.sort(order[:nS]).astype(np.uint32)


def fit_base(R: np.ndarray, sweeps: int):
    """One greedy base on the residual R [M][N].

    Returns (signs int8 [M][N], alpha_r [M], alpha_c [N], R_next [M][N]), all
    scales and the new residual in fp64."""
    if sweeps < 1:
        raise ValueError("at least one sweep")
    R = np.asarray(R, np.float64)
    M, N = R.shape
    B = _sign(R)
    A = _magnitude(R)
    ac = np.ones(N)
    ar = np.zeros(M)
    for _ in range(sweeps):
        ar = _scaled(A @ ac, _norm2(ac))
        ac = _scaled(A.T @ ar, _norm2(ar))
    R_next = R - np.outer(ar, ac) * B
    return B, ar, ac, R_next


def fit(W: np.ndarray, X: np.ndarray, K: int, Ks: int, nS: int, sweeps: int) -> Dict[str, np.ndarray]:
    """The whole fit: K global bases, then the salient set and Ks bases on its
    columns.  Returns the factors in the shapes of the GEMV's inputs (signs
    int8 [K][M][N], alpha_r [K][M], alpha_c [K][N], s_idx [nS], s_signs
    [Ks][M][nS], s_alpha_r [Ks][M], s_alpha_c [Ks][nS]), the scores, and the
    final residual W - W_hat."""
    W = np.asarray(W, np.float64)
    M, N = W.shape
    score = saliency_scores(W, X)
    S = select_salient(score, nS)
    R = W.copy()
    signs = np.empty((K, M, N), np.int8)
    alpha_r = np.empty((K, M))
    alpha_c = np.empty((K, N))
    for k in range(K):
        signs[k], alpha_r[k], alpha_c[k], R = fit_base(R, sweeps)
    s_signs = np.empty((Ks, M, nS), np.int8)
    s_alpha_r = np.empty((Ks, M))
    s_alpha_c = np.empty((Ks, nS))
    if nS and Ks:
        RS = R[:, S.astype(np.int64)]
        for k in range(Ks):
            s_signs[k], s_alpha_r[k], s_alpha_c[k], RS = fit_base(RS, sweeps)
        R[:, S.astype(np.int64)] = RS
    return {"signs": signs, "alpha_r": alpha_r, "alpha_c": alpha_c, "score": score, "s_idx": S,
            "s_signs": s_signs, "s_alpha_r": s_alpha_r, "s_alpha_c": s_alpha_c, "residual": R}
