"""fp64 CPU oracle for group-wise row scales (the "g128" format variant).

TEST INFRASTRUCTURE ONLY: only tests/ may import this module (the GPU
variant, fb_gemv_group_scales, is checked against it there).  The library
never imports it, and it imports nothing from the library.

The FluxBin page (Experimental results, the accuracy paragraph) names a
"2b-s16-g128" setting without defining it.  Reading taken: "g128" is the
usual group-wise scale of post-training quantisation, one row scale per
group of G = 128 consecutive input columns, so the row scale of base k
becomes alpha_r[k][i][j // G]:

    W_hat[i][j] = sum_k alpha_r[k][i][j // G] * alpha_c[k][j] * B[k][i][j]
                  (+ the salient term, unchanged: its row scales stay per row)

With one group (G = N) this is the ordinary decomposition.

Parity status: pinned by ``tests/test_groupwise_oracle.py`` (one group
against the C oracle; every group against the C oracle on its column slice;
hand-sized brute force).
"""

from __future__ import annotations

from typing import Optional

import numpy as np


def group_of(N: int, G: int) -> np.ndarray:
    """The group index of every column."""
    if G < 1 or N % G:
        raise ValueError("G must divide N")
    return np.arange(N) // G


def dequant(signs: np.ndarray, alpha_r: np.ndarray, alpha_c: Optional[np.ndarray], G: int) -> np.ndarray:
    """signs int8 [K][M][N] (+1/-1), alpha_r [K][M][N/G], alpha_c [K][N] or
    None (ones) -> the global term of W_hat [M][N] in fp64."""
    K, M, N = signs.shape
    grp = group_of(N, G)
    if alpha_r.shape != (K, M, N // G):
        raise ValueError("alpha_r must be [K][M][N/G]")
    ar = np.asarray(alpha_r, np.float64)[:, :, grp]                  # [K][M][N]
    ac = np.ones((K, N)) if alpha_c is None else np.asarray(alpha_c, np.float64)
    return np.einsum("kmn,kn,kmn->mn", ar, ac, signs.astype(np.float64))


def gemv(signs, alpha_r, alpha_c, G, x, s_idx=None, s_signs=None, s_alpha_r=None, s_alpha_c=None) -> np.ndarray:
    """y = W_hat x in fp64 for one activation vector x [N] (its exact values);
    the salient term, when given, is the ordinary one (per-row scales)."""
    W = dequant(signs, alpha_r, alpha_c, G)
    if s_idx is not None and len(s_idx):
        S = np.asarray(s_idx, np.int64)
        nS = S.size
        Ws = np.einsum("km,kt,kmt->mt", np.asarray(s_alpha_r, np.float64),
                       np.asarray(s_alpha_c, np.float64)[:, :nS], np.asarray(s_signs, np.float64)[:, :, :nS])
        W[:, S] += Ws
    return W @ np.asarray(x, np.float64)
