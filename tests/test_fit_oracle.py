"""Pins of the fitter oracle (``oracle/fit.py``) to things other than itself:
exact recovery of a rank-one magnitude, numpy's SVD for the leading singular
pair, the never-growing residual of a least-squares step, constructed
saliency cases, and the fitted factors run through the GEMV oracle.  Planted
mistakes in the oracle's helpers must fail a pin."""

import numpy as np
import pytest

import oracle
import workloads as wl
from oracle import fit as F


def _rank_one_signed(M, N, seed):
    rng = np.random.default_rng(seed)
    a = rng.uniform(0.5, 2.0, M)
    b = rng.uniform(0.5, 2.0, N)
    B0 = np.where(rng.random((M, N)) < 0.5, 1, -1).astype(np.int8)
    return a, b, B0, np.outer(a, b) * B0


def test_fit_base_recovers_an_exact_rank_one_magnitude():
    """|W| = a b^T exactly: one sweep from alpha_c = 1 lands on it (alpha_r =
    a (sum b)/N, then alpha_c = b N / sum b), the signs are W's, and the
    residual vanishes."""
    a, b, B0, W = _rank_one_signed(9, 13, 0)
    B, ar, ac, R = F.fit_base(W, sweeps=1)
    assert np.array_equal(B, B0)
    np.testing.assert_allclose(np.outer(ar, ac), np.outer(a, b), rtol=1e-13)
    np.testing.assert_allclose(ar, a * b.sum() / b.size, rtol=1e-13)
    assert np.max(np.abs(R)) <= 1e-13 * np.max(np.abs(W))


def test_fit_base_converges_to_the_leading_singular_pair():
    """Alternating least squares on a positive matrix is the power method:
    the rank-one fit is sigma_1 u_1 v_1^T of |R| (numpy's SVD)."""
    rng = np.random.default_rng(1)
    R = rng.normal(size=(40, 30))
    _, ar, ac, _ = F.fit_base(R, sweeps=200)
    U, s, Vt = np.linalg.svd(np.abs(R))
    np.testing.assert_allclose(np.outer(ar, ac), s[0] * np.outer(U[:, 0], Vt[0]), rtol=1e-9, atol=1e-12)


def test_fit_base_sign_convention_and_zero_matrix():
    R = np.array([[0.0, -0.0, 1.5], [-2.0, 3.0, -1e-30]])
    B, ar, ac, Rn = F.fit_base(R, sweeps=3)
    assert B.tolist() == [[1, 1, 1], [-1, 1, -1]]
    B, ar, ac, Rn = F.fit_base(np.zeros((3, 4)), sweeps=2)   # zero norms give zero scales
    assert np.all(B == 1) and not ar.any() and not ac.any() and not Rn.any()


@pytest.mark.parametrize("sweeps", [1, 2, 8])
def test_residual_never_grows(sweeps):
    """Each sweep is a least-squares update from a start no worse than zero
    scales, so no base can increase the residual."""
    fi = wl.fit_inputs(48, 64, T=16, seed=3)
    R = fi.W.astype(np.float64)
    norms = [np.linalg.norm(R)]
    for _ in range(6):
        _, _, _, R = F.fit_base(R, sweeps)
        norms.append(np.linalg.norm(R))
    assert all(n1 <= n0 * (1 + 1e-12) for n0, n1 in zip(norms, norms[1:]))
    assert norms[-1] < 0.9 * norms[0]


def test_saliency_constructed_cases():
    rng = np.random.default_rng(4)
    W = rng.normal(size=(8, 12))
    # activations only on column 5: every other column has zero score
    X = np.zeros((3, 12))
    X[:, 5] = [1.0, -2.0, 0.5]
    assert F.select_salient(F.saliency_scores(W, X), 1).tolist() == [5]
    # equal activations everywhere and column j of W scaled by j + 1: the
    # largest nS columns are the last nS
    Wc = np.ones((4, 12)) * (np.arange(12) + 1.0)
    s = F.saliency_scores(Wc, np.ones((5, 12)))
    assert F.select_salient(s, 4).tolist() == [8, 9, 10, 11]
    np.testing.assert_allclose(s, 5 * 4 * (np.arange(12) + 1.0) ** 2)
    # equal weight columns: the activation term is the Hessian's diagonal,
    # diag(X^T X) (a matrix product here), so a single large activation
    # (3: 9) outranks spread ones (2, 2: 8; 1, 1, 1, 1: 4)
    Xd = np.array([[3.0, 1.0, 2.0], [0.0, 1.0, 2.0], [0.0, 1.0, 0.0], [0.0, -1.0, 0.0]])
    sd = F.saliency_scores(np.ones((4, 3)), Xd)
    np.testing.assert_array_equal(sd, 4 * np.diag(Xd.T @ Xd))
    assert F.select_salient(sd, 1).tolist() == [0] and F.select_salient(sd, 2).tolist() == [0, 2]


def test_select_equal_scores_take_the_lower_column_and_list_ascending():
    assert F.select_salient(np.ones(10), 3).tolist() == [0, 1, 2]
    assert F.select_salient(np.array([1.0, 5.0, 5.0, 2.0, 5.0]), 2).tolist() == [1, 2]
    assert F.select_salient(np.array([3.0, 1.0, 2.0]), 0).tolist() == []
    with pytest.raises(ValueError):
        F.select_salient(np.ones(3), 4)


def _as_problem(f, M, N, x):
    K, Ks, nS = f["signs"].shape[0], f["s_signs"].shape[0], f["s_idx"].size
    nS_pad = wl.round_up(nS, 32) if nS else 0
    s_signs = np.full((Ks, M, nS_pad), -1, np.int8)   # pad bits 0
    s_signs[:, :, :nS] = f["s_signs"]
    return wl.Problem(
        name="fit", M=M, N=N, K=K, g=4, nS=nS, Ks=Ks, batch=1, x_dtype="f32",
        sign_bits=wl.pack_signs(f["signs"]), alpha_r=f["alpha_r"].astype(np.float32),
        alpha_c=f["alpha_c"].astype(np.float32), s_idx=f["s_idx"],
        s_sign_bits=wl.pack_signs(s_signs), s_alpha_r=f["s_alpha_r"].astype(np.float32),
        s_alpha_c=f["s_alpha_c"].astype(np.float32),
        x=x[None, :].astype(np.float32))


def test_fitted_factors_through_the_gemv_oracle():
    """The fit's factors, packed in the GEMV's input format, make the GEMV
    oracle compute (W - residual) x: the fitter's output means what the
    GEMV's inputs mean.  The scales are rounded to fp32 on the way, so the
    comparison uses the dequantised fp32 factors."""
    M, N = 40, 64
    fi = wl.fit_inputs(M, N, T=8, seed=5)
    f = F.fit(fi.W, fi.X, K=2, Ks=2, nS=7, sweeps=4)
    x = np.random.default_rng(6).normal(size=N)
    p = _as_problem(f, M, N, x)
    y = oracle.gemv(oracle.OracleWeights.from_problem(p), p.x_f32().astype(np.float64))[0][0]
    Wh = np.einsum("km,kn,kmn->mn", p.alpha_r.astype(np.float64), p.alpha_c.astype(np.float64),
                   f["signs"].astype(np.float64))
    S = f["s_idx"].astype(np.int64)
    Wh[:, S] += np.einsum("km,kn,kmn->mn", p.s_alpha_r.astype(np.float64),
                          p.s_alpha_c.astype(np.float64), f["s_signs"].astype(np.float64))
    np.testing.assert_allclose(y, Wh @ x.astype(np.float32).astype(np.float64), rtol=1e-12, atol=1e-15)
    # and, before fp32 rounding of the scales, W_hat = W - residual
    Wh64 = np.einsum("km,kn,kmn->mn", f["alpha_r"], f["alpha_c"], f["signs"].astype(np.float64))
    Wh64[:, S] += np.einsum("km,kn,kmn->mn", f["s_alpha_r"], f["s_alpha_c"], f["s_signs"].astype(np.float64))
    np.testing.assert_allclose(Wh64, fi.W.astype(np.float64) - f["residual"], rtol=0, atol=1e-15)


def test_more_bases_and_salient_bases_fit_better():
    M, N = 64, 96
    fi = wl.fit_inputs(M, N, T=16, seed=8)
    errs = [np.linalg.norm(F.fit(fi.W, fi.X, K=k, Ks=0, nS=0, sweeps=6)["residual"]) for k in (1, 2, 3, 4)]
    assert all(b < a for a, b in zip(errs, errs[1:]))
    f0 = F.fit(fi.W, fi.X, K=2, Ks=0, nS=10, sweeps=6)
    f2 = F.fit(fi.W, fi.X, K=2, Ks=2, nS=10, sweeps=6)
    S = f2["s_idx"].astype(np.int64)
    assert np.array_equal(f0["s_idx"], f2["s_idx"])
    assert np.linalg.norm(f2["residual"][:, S]) < 0.8 * np.linalg.norm(f0["residual"][:, S])
    rest = np.setdiff1d(np.arange(N), S)
    assert np.array_equal(f2["residual"][:, rest], f0["residual"][:, rest])


# ---- planted mistakes: each must fail one of the pins above -----------------

def _pins_pass():
    try:
        test_fit_base_recovers_an_exact_rank_one_magnitude()
        test_fit_base_converges_to_the_leading_singular_pair()
        test_fit_base_sign_convention_and_zero_matrix()
        test_saliency_constructed_cases()
        test_select_equal_scores_take_the_lower_column_and_list_ascending()
        for s in (1, 2, 8):
            test_residual_never_grows(s)
        test_more_bases_and_salient_bases_fit_better()
        test_fitted_factors_through_the_gemv_oracle()
    except (AssertionError, ValueError, FloatingPointError, IndexError):
        return False
    return True


@pytest.mark.parametrize("mutation", ["sign_strict", "no_magnitude", "norm_not_squared",
                                      "score_no_activation", "select_descending_ties"])
def test_planted_mistakes_fail_a_pin(monkeypatch, mutation):
    assert _pins_pass()
    if mutation == "sign_strict":        # zero taken as -1
        monkeypatch.setattr(F, "_sign", lambda R: np.where(R > 0, 1, -1).astype(np.int8))
    elif mutation == "no_magnitude":     # fitting R instead of |R|
        monkeypatch.setattr(F, "_magnitude", lambda R: R)
    elif mutation == "norm_not_squared":
        monkeypatch.setattr(F, "_norm2", lambda v: float(np.sqrt(np.dot(v, v))))
    elif mutation == "score_no_activation":
        monkeypatch.setattr(F, "saliency_scores", lambda W, X: np.einsum("ij,ij->j", np.asarray(W, float), np.asarray(W, float)))
    elif mutation == "select_descending_ties":
        monkeypatch.setattr(F, "select_salient",   # equal scores take the higher column
                            lambda s, n: np.sort(np.lexsort((-np.arange(len(s)), -np.asarray(s)))[:n]).astype(np.uint32))
    assert not _pins_pass()


SOURCE_MUTATIONS = [
    ("residual update sign", "R_next = R - np.outer(ar, ac) * B", "R_next = R + np.outer(ar, ac) * B"),
    ("one sweep too few", "for _ in range(sweeps):", "for _ in range(sweeps - 1):"),
    ("column scale from the old row scale", "        ar = _scaled(A @ ac, _norm2(ac))\n        ac = _scaled(A.T @ ar, _norm2(ar))",
     "        ac_old = ac\n        ar = _scaled(A @ ac, _norm2(ac))\n        ac = _scaled(A.T @ ar, _norm2(ac_old))"),
    ("activation energy not squared", 'np.einsum("tj,tj->j", X, X)', 'np.einsum("tj->j", np.abs(X))'),
    ("weight energy over rows", 'np.einsum("ij,ij->j", W, W)', 'np.einsum("ij,ij->j", W, np.abs(W) ** 0.5)'),
    ("smallest scores selected", "np.argsort(-score, kind=\"stable\")", "np.argsort(score, kind=\"stable\")"),
    ("salient set not listed ascending", "return np.sort(order[:nS]).astype(np.uint32)",
     "return order[:nS].astype(np.uint32)"),
    ("salient residual not written back", "        R[:, S.astype(np.int64)] = RS\n", ""),
    ("salient bases fitted before the global ones", "    for k in range(K):\n        signs[k], alpha_r[k], alpha_c[k], R = fit_base(R, sweeps)\n",
     ""),
    ("salient set shifted by one rank", "return np.sort(order[:nS]).astype(np.uint32)",
     "return np.sort(order[1:nS + 1]).astype(np.uint32)"),
    ("residual started from |W|", "    R = W.copy()\n", "    R = np.abs(W)\n"),
    ("salient bases fitted to W", "RS = R[:, S.astype(np.int64)]", "RS = W[:, S.astype(np.int64)]"),
    ("score as a sum", "return h * w", "return h + w"),
    ("sweeps started from alpha_c = 2", "    ac = np.ones(N)\n", "    ac = np.full(N, 2.0)\n"),
    ("residual update without the signs", "R_next = R - np.outer(ar, ac) * B", "R_next = R - np.outer(ar, ac) * np.abs(B)"),
]


@pytest.mark.parametrize("name,old,new", SOURCE_MUTATIONS, ids=[m[0] for m in SOURCE_MUTATIONS])
def test_planted_source_mistakes_fail_a_pin(monkeypatch, name, old, new):
    """Each edits one step of a copy of ``oracle/fit.py`` (loaded as a new
    module; the real one is untouched) and the pins, run against the copy,
    must fail."""
    import sys
    import types
    src = open(F.__file__).read()
    assert src.count(old) == 1, name
    mod = types.ModuleType("fit_mutant")
    mod.__file__ = F.__file__
    exec(compile(src.replace(old, new), F.__file__, "exec"), mod.__dict__)
    monkeypatch.setattr(sys.modules[__name__], "F", mod)
    assert not _pins_pass(), name
