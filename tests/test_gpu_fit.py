"""GPU parity of the fitter (``fb_fit_saliency``, ``fb_fit_base`` and the
``fit`` sequence, through the C ABI) against the fp64 oracle in
``oracle/fit.py``.

Bars, from the arithmetic: the GPU sums in fp64 and rounds each scale once to
fp32, so on the same fp32 residual the signs are bit-exact (both sides decide
R >= 0 on the same values), the scales agree to 1e-5 relative (sums of
positive terms: no cancellation; the fp32 rounding of one sweep's scales feeds
the next), and the new residual to 1e-5 * (|R| + alpha_r alpha_c).  Across a
chain of bases each side follows its own residual, so signs are compared
where the oracle's residual is not within rounding of zero."""

import numpy as np
import pytest
import torch

import lut_binary_gemv_b200 as fb
import workloads as wl
from oracle import fit as F

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gpu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


@pytest.mark.parametrize("M,N,sweeps", [(1, 1, 1), (37, 45, 3), (64, 96, 8), (300, 257, 2), (1024, 4096, 8)])
def test_fit_base_matches_oracle(M, N, sweeps):
    R0 = wl.fit_inputs(M, N, T=4, seed=M * 7 + N).W
    R = _gpu(R0)
    signs, ar, ac = fb.fb_fit_base(R, sweeps)
    B, ar_o, ac_o, Rn_o = F.fit_base(R0.astype(np.float64), sweeps)
    assert np.array_equal(signs.cpu().numpy(), B)
    np.testing.assert_allclose(ar.cpu().numpy(), ar_o, rtol=1e-5, atol=0)
    np.testing.assert_allclose(ac.cpu().numpy(), ac_o, rtol=1e-5, atol=0)
    bound = 1e-5 * (np.abs(R0) + np.outer(ar_o, ac_o))
    assert np.all(np.abs(R.cpu().numpy() - Rn_o) <= bound)


def test_fit_base_zero_and_signed_zero_residual():
    R0 = np.zeros((33, 40), np.float32)
    R0[0, :5] = [-0.0, 0.0, 1.0, -1.0, -0.0]
    R = _gpu(R0)
    signs, ar, ac = fb.fb_fit_base(R, 2)
    B, ar_o, ac_o, Rn_o = F.fit_base(R0.astype(np.float64), 2)
    assert np.array_equal(signs.cpu().numpy(), B)
    np.testing.assert_allclose(ar.cpu().numpy(), ar_o, rtol=1e-6, atol=0)
    np.testing.assert_allclose(ac.cpu().numpy(), ac_o, rtol=1e-6, atol=0)
    R = _gpu(np.zeros((8, 8), np.float32))
    signs, ar, ac = fb.fb_fit_base(R, 3)
    assert bool((signs == 1).all()) and not ar.any() and not ac.any() and not R.any()


def test_fit_base_chain_of_bases():
    M, N = 512, 768
    W = wl.fit_inputs(M, N, T=4, seed=11).W
    R = _gpu(W)
    Ro = W.astype(np.float64)
    for _ in range(4):
        signs, ar, ac = fb.fb_fit_base(R, 6)
        B, ar_o, ac_o, Rn = F.fit_base(Ro, 6)
        clear = np.abs(Ro) > 1e-4 * np.abs(Ro).max()
        assert np.array_equal(signs.cpu().numpy()[clear], B[clear])
        np.testing.assert_allclose(ar.cpu().numpy(), ar_o, rtol=1e-4)
        np.testing.assert_allclose(ac.cpu().numpy(), ac_o, rtol=1e-4)
        Ro = Rn
    np.testing.assert_allclose(np.linalg.norm(R.cpu().numpy()), np.linalg.norm(Ro), rtol=1e-5)


def _same_selection(got, want, score_o, nS, rtol=1e-6):
    """Equal sets, or sets that differ only in columns tied (within rtol) at
    the selection boundary."""
    got, want = set(got.tolist()), set(want.tolist())
    if got == want:
        return True
    edge = np.sort(score_o)[::-1][nS - 1]
    return all(abs(score_o[j] - edge) <= rtol * edge for j in got ^ want)


@pytest.mark.parametrize("M,N,T,nS", [(8, 64, 3, 5), (64, 1000, 16, 0), (256, 4096, 64, 128),
                                      (128, 11008, 32, 330), (16, 300, 4, 300)])
def test_fit_saliency_matches_oracle(M, N, T, nS):
    fi = wl.fit_inputs(M, N, T=T, seed=N + nS)
    score, s_idx = fb.fb_fit_saliency(_gpu(fi.W), _gpu(fi.X), nS)
    s_o = F.saliency_scores(fi.W, fi.X)
    S_o = F.select_salient(s_o, nS)
    np.testing.assert_allclose(score.cpu().numpy(), s_o, rtol=1e-6, atol=0)
    got = s_idx.cpu().numpy().astype(np.int64)
    assert np.all(np.diff(got) > 0)                      # ascending, distinct
    assert _same_selection(got, S_o.astype(np.int64), s_o, nS)


def test_fit_saliency_equal_scores_take_the_lower_column():
    W = np.ones((4, 100), np.float32)
    X = np.ones((2, 100), np.float32)
    _, s_idx = fb.fb_fit_saliency(_gpu(W), _gpu(X), 7)
    assert s_idx.cpu().tolist() == list(range(7))


@pytest.mark.parametrize("M,N,T,nS,levels", [(16, 5000, 2, 1234, 3), (8, 65536, 2, 4096, 7), (4, 100003, 1, 50001, 2),
                                             (32, 4096, 4, 128, 0), (8, 777, 3, 777, 4)])
def test_fit_saliency_selection_is_exact_on_its_scores(M, N, T, nS, levels):
    """The selection itself, bit for bit: on the GPU's own fp32 scores, the
    nS largest with equal scores taken lower column first (a stable sort of
    the negated scores), ascending.  levels > 0: W in {0, 1} with `levels`
    distinct column counts of ones, so most scores tie exactly and the cut
    falls inside a run of equal scores."""
    rng = np.random.default_rng(N + nS)
    if levels:
        ones_per_col = rng.integers(0, levels, N)
        W = (np.arange(M)[:, None] < ones_per_col[None, :]).astype(np.float32)
        X = np.ones((T, N), np.float32)
    else:
        fi = wl.fit_inputs(M, N, T=T, seed=N)
        W, X = fi.W, fi.X
    score, s_idx = fb.fb_fit_saliency(_gpu(W), _gpu(X), nS)
    sc = score.cpu().numpy()
    want = np.sort(np.argsort(-sc, kind="stable")[:nS])
    assert np.array_equal(s_idx.cpu().numpy().astype(np.int64), want)


def test_fit_end_to_end_4096():
    """The whole fit of a 4096 x 4096 layer (K = 2, Ks = 2, 128 salient
    columns, 8 sweeps): the same salient set, global scales within 1e-4, the
    salient scales' products (the padded gather scales each factor by the
    same constant, only the product is unique) within 1e-4, and the same
    reconstruction error."""
    M = N = 4096
    fi = wl.fit_inputs(M, N, T=64, seed=21)
    g = fb.fit(_gpu(fi.W), _gpu(fi.X), K=2, Ks=2, nS=128, sweeps=8)
    o = F.fit(fi.W, fi.X, K=2, Ks=2, nS=128, sweeps=8)
    assert _same_selection(g["s_idx"].cpu().numpy().astype(np.int64), o["s_idx"].astype(np.int64), o["score"], 128)
    np.testing.assert_allclose(g["alpha_r"].cpu().numpy(), o["alpha_r"], rtol=1e-4)
    np.testing.assert_allclose(g["alpha_c"].cpu().numpy(), o["alpha_c"], rtol=1e-4)
    for k in range(2):
        pg = np.outer(g["s_alpha_r"][k].cpu().numpy(), g["s_alpha_c"][k].cpu().numpy())
        np.testing.assert_allclose(pg, np.outer(o["s_alpha_r"][k], o["s_alpha_c"][k]), rtol=1e-4)
    agree = (g["signs"].cpu().numpy() == o["signs"]).mean()
    assert agree > 0.9999
    S = o["s_idx"].astype(np.int64)
    res = g["residual"].cpu().numpy().astype(np.float64)
    res[:, S] = g["s_residual"].cpu().numpy()
    np.testing.assert_allclose(np.linalg.norm(res), np.linalg.norm(o["residual"]), rtol=1e-4)
