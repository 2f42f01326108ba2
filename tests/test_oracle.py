"""Pins for the fp64 CPU oracle (CPU only).

Each test ties the oracle to something other than itself: a worked example
derived by hand, closed forms of the LUT entries, special cases with exact
integer answers from numpy/torch integer routines, exact rational brute force
built by a different route (matrix algebra instead of loops), and invariants.
Together they are chosen so that a plausible slip in the oracle (a dropped
term, a wrong sign, bit order or index, a transposed operand) fails at least
one of them; ``test_oracle_mutations.py`` checks exactly that by planting such
slips in a copy of ``oracle.c``.
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _weights_from_signs(signs, alpha_r, alpha_c=None, s_idx=None, s_signs=None,
                        s_alpha_r=None, s_alpha_c=None):
    K, M, N = signs.shape
    sb = wl.pack_signs(signs)[..., : N // 8]
    if s_idx is not None and len(s_idx):
        ssb = wl.pack_signs(s_signs)
        return oracle.OracleWeights(M, N, K, sb, alpha_r, alpha_c, s_idx, ssb,
                                    s_alpha_r, s_alpha_c, s_signs.shape[0])
    return oracle.OracleWeights(M, N, K, sb, alpha_r, alpha_c)


# --- activations -----------------------------------------------------------

def test_f16_decode_all_bit_patterns():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.x_to_f64(bits.view(np.float16), "f16")
    want = bits.view(np.float16).astype(np.float64)      # numpy's own conversion
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])


# --- the worked example ------------------------------------------------------

def test_hand_worked_example():
    ex = json.load(open(os.path.join(GOLDEN, "hand_example_2x8.json")))
    w = _weights_from_signs(np.array(ex["signs"], np.int8), np.array(ex["alpha_r"], np.float32),
                            np.array(ex["alpha_c"], np.float32), np.array(ex["s_idx"], np.uint32),
                            np.array(ex["s_signs"], np.int8), np.array(ex["s_alpha_r"], np.float32),
                            np.array(ex["s_alpha_c"], np.float32))
    x = np.array(ex["x"], np.float64)
    W = oracle.dequant(w)
    assert np.array_equal(W, np.array(ex["expected"]["W"]))
    y, d, e = oracle.gemv(w, x)
    assert np.array_equal(y[0], ex["expected"]["y"])
    assert np.array_equal(d[0], ex["expected"]["d"])
    assert np.array_equal(e[0], ex["expected"]["e"])
    for g in (1, 2, 4, 8):
        assert np.array_equal(oracle.gemv_lut(w, g, x)[0], ex["expected"]["y"])
    T = oracle.lut_tables(x, np.array(ex["alpha_c"], np.float32), 2, 4)
    lg = ex["expected"]["lut_g4_base1_row0"]
    assert T[1, 0, lg["group0_pattern"]] == lg["group0_entry"]
    assert T[1, 1, lg["group1_pattern"]] == lg["group1_entry"]


# --- LUT-BSF closed forms ----------------------------------------------------

@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_lut_closed_forms(g):
    rng = np.random.default_rng(10 + g)
    N, K = 8 * 4, 2
    x = rng.standard_normal(N)
    ac = (np.abs(rng.standard_normal((K, N))) + 0.1).astype(np.float32)
    T = oracle.lut_tables(x, ac, K, g)
    z = (ac.astype(np.float64) * x[None, :]).reshape(K, N // g, g)
    P = 1 << g
    # all bits set: every column enters with +1; no bit set: every column with -1
    np.testing.assert_allclose(T[:, :, P - 1], z.sum(-1), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(T[:, :, 0], -z.sum(-1), rtol=1e-14, atol=1e-14)
    # complement symmetry T[~p] = -T[p]
    np.testing.assert_allclose(T[:, :, ::-1], -T, rtol=1e-14, atol=1e-14)
    # bit t of the pattern belongs to column t of the group, and +1 <=> set bit
    for p in range(P):
        for t in range(g):
            if not (p >> t) & 1:
                np.testing.assert_allclose(T[:, :, p | (1 << t)] - T[:, :, p], 2 * z[:, :, t],
                                           rtol=1e-12, atol=1e-12)


def test_lut_alpha_c_none_is_ones():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(64)
    np.testing.assert_array_equal(oracle.lut_tables(x, None, 2, 4),
                                  oracle.lut_tables(x, np.ones((2, 64), np.float32), 2, 4))


# --- exact special cases -----------------------------------------------------

@pytest.mark.parametrize("M,N", [(8, 8), (37, 96), (5, 256)])
def test_k1_unit_scales_is_integer_Bx(M, N):
    rng = np.random.default_rng(M * N)
    signs = np.where(rng.integers(0, 2, (1, M, N)) > 0, 1, -1).astype(np.int8)
    xi = rng.integers(-50, 51, N)
    w = _weights_from_signs(signs, np.ones((1, M), np.float32), np.ones((1, N), np.float32))
    y, _, _ = oracle.gemv(w, xi.astype(np.float64))
    assert np.array_equal(y[0], signs[0].astype(np.int64) @ xi)
    w_none = _weights_from_signs(signs, np.ones((1, M), np.float32), None)
    assert np.array_equal(oracle.gemv(w_none, xi.astype(np.float64))[0][0], signs[0].astype(np.int64) @ xi)
    for g in (1, 2, 4, 8):
        assert np.array_equal(oracle.gemv_lut(w, g, xi.astype(np.float64))[0], signs[0].astype(np.int64) @ xi)


def test_ternary_is_exact_dense_ternary_matvec():
    p = wl.make_problem(96, 160, 2, ternary=True, integer_mode=True, x_dtype="f16", seed=7)
    xi = p.x_f32()[0].astype(np.int64)
    ar = 2.0 * p.alpha_r[0].astype(np.float64)           # the per-row scale alpha_r
    want = ar * (p.ternary.astype(np.int64) @ xi)          # integer matvec, then exact dyadic scale
    y, _, _ = oracle.problem_reference(p)
    assert np.array_equal(y[0], want)
    for g in (4, 8):
        assert np.array_equal(oracle.gemv_lut(oracle.OracleWeights.from_problem(p), g,
                                              oracle.x_to_f64(p.x, p.x_dtype))[0], want)


def test_ternary_float_matches_ternary_matvec():
    p = wl.make_problem(64, 256, 2, ternary=True, x_dtype="bf16", seed=8)
    x = p.x_f32()[0].astype(np.float64)
    want = 2.0 * p.alpha_r[0].astype(np.float64) * (p.ternary.astype(np.float64) @ x)
    y, d, _ = oracle.problem_reference(p)
    assert np.all(np.abs(y[0] - want) <= 1e-13 * d[0] + 1e-300)


# --- brute force by another route ---------------------------------------------

def _dense_by_matrix_algebra(signs, ar, ac, s_idx, s_signs, s_ar, s_ac):
    """W = sum_k outer(alpha_r, alpha_c) * B  +  (sum_k' outer(s_ar, s_ac) * Bs) @ P,
    with P the 0/1 matrix that places compact column t at column S[t]; exact
    rationals throughout."""
    K, M, N = signs.shape
    F = np.vectorize(Fraction, otypes=[object])
    W = np.zeros((M, N), dtype=object)
    W[:] = Fraction(0)
    for k in range(K):
        W = W + np.outer(F(ar[k].astype(np.float64)), F(ac[k].astype(np.float64))) * signs[k].astype(object)
    if s_idx is not None and len(s_idx):
        P = np.zeros((len(s_idx), N), dtype=object)
        P[:] = Fraction(0)
        P[np.arange(len(s_idx)), s_idx] = Fraction(1)
        for k in range(s_signs.shape[0]):
            Ws = np.outer(F(s_ar[k].astype(np.float64)), F(s_ac[k].astype(np.float64))) * s_signs[k].astype(object)
            W = W + Ws.dot(P)
    return W


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_8x8_exact_rationals(seed):
    rng = np.random.default_rng(100 + seed)
    K, M, N, nS, Ks = 2, 8, 8, 3, 2
    signs = np.where(rng.integers(0, 2, (K, M, N)) > 0, 1, -1).astype(np.int8)
    ar = (np.abs(rng.standard_normal((K, M))) + 0.1).astype(np.float32)
    ac = (np.abs(rng.standard_normal((K, N))) + 0.1).astype(np.float32)
    s_idx = np.sort(rng.choice(N, nS, replace=False)).astype(np.uint32)
    s_signs = np.where(rng.integers(0, 2, (Ks, M, nS)) > 0, 1, -1).astype(np.int8)
    s_ar = (np.abs(rng.standard_normal((Ks, M))) + 0.1).astype(np.float32)
    s_ac = (np.abs(rng.standard_normal((Ks, nS))) + 0.1).astype(np.float32)
    x = rng.standard_normal(N).astype(np.float32).astype(np.float64)
    W = _dense_by_matrix_algebra(signs, ar, ac, s_idx, s_signs, s_ar, s_ac)
    y_exact = W.dot(np.vectorize(Fraction, otypes=[object])(x))
    w = _weights_from_signs(signs, ar, ac, s_idx, s_signs, s_ar, s_ac)
    Wo = oracle.dequant(w)
    np.testing.assert_allclose(Wo, W.astype(np.float64), rtol=4e-16, atol=0)
    y, d, _ = oracle.gemv(w, x)
    err = np.abs(y[0] - np.array([float(v) for v in y_exact]))
    assert np.all(err <= 32 * 2.0**-53 * d[0])
    for g in (1, 2, 4, 8):
        yl = oracle.gemv_lut(w, g, x)[0]
        assert np.all(np.abs(yl - np.array([float(v) for v in y_exact])) <= 64 * 2.0**-53 * np.abs(
            np.abs(W).dot(np.abs(x)).astype(np.float64)) + 1e-300)


# --- the two formulations, and the dense matvec against numpy -----------------

@pytest.mark.parametrize("g", [1, 2, 4, 8])
@pytest.mark.parametrize("shape", [(33, 64, 1, 0), (70, 288, 3, 40), (17, 512, 4, 512)])
def test_lut_formulation_equals_dequant(g, shape):
    M, N, K, nS = shape
    p = wl.make_problem(M, N, K, g=g, nS=nS, Ks=2, x_dtype="f16", alpha_dist="unit",
                        seed=hash((M, N, K, g)) % 1000)
    w = oracle.OracleWeights.from_problem(p)
    x = oracle.x_to_f64(p.x, p.x_dtype)
    y, d, e = oracle.gemv(w, x)
    yl = oracle.gemv_lut(w, g, x)
    assert np.all(np.abs(yl - y) <= 1e-12 * e)


def test_gemv_equals_numpy_matvec_of_dequant():
    p = wl.make_problem(45, 192, 3, nS=20, Ks=2, x_dtype="f32", alpha_dist="unit", seed=5)
    w = oracle.OracleWeights.from_problem(p)
    x = oracle.x_to_f64(p.x, p.x_dtype)
    W = oracle.dequant(w)
    y, d, _ = oracle.gemv(w, x)
    np.testing.assert_allclose(y[0], W @ x[0], rtol=0, atol=1e-13 * d[0].max())
    np.testing.assert_allclose(d[0], np.abs(W * x[0][None, :]).sum(1), rtol=1e-13)


def test_dequant_structure_single_base():
    rng = np.random.default_rng(11)
    M, N = 24, 40
    signs = np.where(rng.integers(0, 2, (1, M, N)) > 0, 1, -1).astype(np.int8)
    ar = (np.abs(rng.standard_normal((1, M))) + 0.1).astype(np.float32)
    ac = (np.abs(rng.standard_normal((1, N))) + 0.1).astype(np.float32)
    W = oracle.dequant(_weights_from_signs(signs, ar, ac))
    # elementwise product of the rank-one scale matrix with the signs
    np.testing.assert_array_equal(W, np.outer(ar[0].astype(np.float64), ac[0].astype(np.float64)) * signs[0])
    W1 = oracle.dequant(_weights_from_signs(signs, np.ones_like(ar), np.ones_like(ac)))
    np.testing.assert_array_equal(W1, signs[0])


def test_sampled_rows_match_full():
    p = wl.make_problem(77, 96, 2, nS=9, Ks=3, x_dtype="f16", seed=12, batch=3)
    w = oracle.OracleWeights.from_problem(p)
    x = oracle.x_to_f64(p.x, p.x_dtype)
    y, d, e = oracle.gemv(w, x)
    rows = np.array([76, 0, 31, 32, 5])
    ys, ds, es = oracle.gemv(w, x, rows)
    np.testing.assert_array_equal(ys, y[:, rows])
    np.testing.assert_array_equal(ds, d[:, rows])
    np.testing.assert_array_equal(oracle.gemv_lut(w, 4, x, rows), oracle.gemv_lut(w, 4, x)[:, rows])
    np.testing.assert_array_equal(oracle.dequant(w, rows), oracle.dequant(w)[rows])
    for b in range(3):   # batch rows are independent problems
        np.testing.assert_array_equal(oracle.gemv(w, x[b])[0][0], y[b])
        np.testing.assert_array_equal(oracle.gemv_lut(w, 4, x[b])[0], oracle.gemv_lut(w, 4, x)[b])


# --- invariants ---------------------------------------------------------------

def test_salient_over_all_columns_equals_extra_global_bases():
    K, Ks, M, N = 2, 2, 40, 64
    p = wl.make_problem(M, N, K, nS=N, Ks=Ks, integer_mode=True, x_dtype="f16", seed=21)
    assert np.array_equal(p.s_idx, np.arange(N))
    y, _, _ = oracle.problem_reference(p)
    # the same weight as a (K+Ks)-base global matrix
    bits = np.concatenate([p.sign_bits, p.s_sign_bits[..., : N // 8]], axis=0)
    w2 = oracle.OracleWeights(M, N, K + Ks, bits, np.concatenate([p.alpha_r, p.s_alpha_r]),
                              np.concatenate([p.alpha_c, p.s_alpha_c]))
    y2, _, _ = oracle.gemv(w2, oracle.x_to_f64(p.x, p.x_dtype))
    assert np.array_equal(y, y2)


def test_negating_a_base_and_its_scale_changes_nothing():
    """(-alpha_r) alpha_c^T (.) (-B) is the same term: flipping every sign of
    a base (global or salient) and negating its row scales leaves W, y and
    both tolerance magnitudes d and e unchanged (e sums |alpha_r alpha_c x|)."""
    p = wl.make_problem(40, 128, 3, nS=17, Ks=2, x_dtype="f32", seed=27, batch=2)
    x = oracle.x_to_f64(p.x, p.x_dtype)
    W0 = oracle.dequant(oracle.OracleWeights.from_problem(p))
    y0, d0, e0 = oracle.problem_reference(p)
    signs, s_signs = p.signs(), p.s_signs()
    signs[1] *= -1
    s_signs[0] *= -1
    ar, s_ar = p.alpha_r.copy(), p.s_alpha_r.copy()
    ar[1] *= -1
    s_ar[0] *= -1
    w = _weights_from_signs(signs, ar, p.alpha_c, p.s_idx, s_signs, s_ar, p.s_alpha_c)
    assert np.array_equal(oracle.dequant(w), W0)
    y, d, e = oracle.gemv(w, x)
    assert np.array_equal(y, y0) and np.array_equal(d, d0) and np.array_equal(e, e0)
    assert np.array_equal(oracle.gemv_lut(w, 4, x), oracle.gemv_lut(oracle.OracleWeights.from_problem(p), 4, x))


def test_empty_salient_equals_global_term():
    p = wl.make_problem(50, 128, 2, nS=30, Ks=2, x_dtype="f16", seed=22)
    x = oracle.x_to_f64(p.x, p.x_dtype)
    w0 = oracle.OracleWeights(p.M, p.N, p.K, p.sign_bits, p.alpha_r, p.alpha_c)
    p.s_alpha_r[:] = 0
    w1 = oracle.OracleWeights.from_problem(p)
    assert np.array_equal(oracle.gemv(w0, x)[0], oracle.gemv(w1, x)[0])


def test_power_of_two_scaling_is_exact():
    p = wl.make_problem(30, 96, 3, nS=11, Ks=2, x_dtype="f32", alpha_dist="unit", seed=23)
    w = oracle.OracleWeights.from_problem(p)
    x = oracle.x_to_f64(p.x, p.x_dtype)
    y = oracle.gemv(w, x)[0]
    assert np.array_equal(oracle.gemv(w, 8.0 * x)[0], 8.0 * y)
    assert np.array_equal(oracle.gemv_lut(w, 4, 0.25 * x), 0.25 * oracle.gemv_lut(w, 4, x))
    p.alpha_r *= 2
    p.s_alpha_r *= 2
    assert np.array_equal(oracle.gemv(oracle.OracleWeights.from_problem(p), x)[0], 2.0 * y)


def test_column_permutation_invariance():
    p = wl.make_problem(36, 128, 2, nS=13, Ks=2, x_dtype="f32", alpha_dist="unit", seed=24)
    rng = np.random.default_rng(0)
    perm = rng.permutation(p.N)               # new column c holds old column perm[c]
    inv = np.argsort(perm)
    signs = p.signs()[:, :, perm]
    new_s = inv[p.s_idx]                       # old salient column -> its new position
    order = np.argsort(new_s)                  # keep S ascending: reorder compact columns
    w = _weights_from_signs(signs, p.alpha_r, p.alpha_c[:, perm], new_s[order].astype(np.uint32),
                            p.s_signs()[:, :, order], p.s_alpha_r, p.s_alpha_c[:, order])
    x = oracle.x_to_f64(p.x, p.x_dtype)
    y, d, _ = oracle.problem_reference(p)
    y2, _, _ = oracle.gemv(w, x[:, perm])
    assert np.all(np.abs(y2 - y) <= 1e-12 * d)


def test_linearity_in_x():
    p = wl.make_problem(20, 64, 2, nS=5, Ks=1, x_dtype="f32", seed=25, batch=2)
    w = oracle.OracleWeights.from_problem(p)
    x = oracle.x_to_f64(p.x, p.x_dtype)
    y, _, e = oracle.gemv(w, x)
    ysum, _, _ = oracle.gemv(w, x[0] + x[1])
    assert np.all(np.abs(ysum[0] - y[0] - y[1]) <= 1e-12 * (e[0] + e[1]))


def test_vcm_gather_matches_fancy_indexing():
    rng = np.random.default_rng(26)
    x = rng.standard_normal(300)
    s = np.sort(rng.choice(300, 45, replace=False)).astype(np.uint32)
    got = oracle.vcm_gather(x, s, 64)
    assert np.array_equal(got[:45], x[s]) and np.all(got[45:] == 0)
    assert oracle.vcm_gather(x, np.zeros(0, np.uint32), 0).shape == (0,)


def test_rejects_bad_arguments():
    p = wl.make_problem(8, 32, 1, nS=3, Ks=1, seed=27)
    w = oracle.OracleWeights.from_problem(p)
    w.arrays["s_idx"][0] = 32                  # out of range salient column
    with pytest.raises(ValueError):
        oracle.gemv(w, np.zeros(32))
    with pytest.raises(ValueError):
        oracle.gemv_lut(oracle.OracleWeights.from_problem(p), 3, np.zeros(32))
    with pytest.raises(ValueError):
        oracle.gemv(oracle.OracleWeights.from_problem(p), np.zeros(32), rows=[8])
    # more salient columns than columns (each index in range)
    many = oracle.OracleWeights(8, 32, 1, p.sign_bits, p.alpha_r, p.alpha_c, np.arange(33, dtype=np.uint32) % 32,
                                np.zeros((1, 8, 8), np.uint8), np.ones((1, 8), np.float32),
                                np.ones((1, 33), np.float32), 1)
    with pytest.raises(ValueError):
        oracle.gemv(many, np.zeros(32))


def test_integer_mode_stays_below_2_24():
    """The integer-valued mode is exact in fp32 only if every partial sum is an
    integer (or dyadic) below 2^24; check the worst workload shape."""
    K, Ks = 3, 2
    for M, N in wl.SHAPES70B:
        # |alpha_r| <= 2, |alpha_c| <= 4, |x| <= 4 over N columns and K+Ks bases
        assert (K + Ks) * 2.0 * N * 4 * 4 < 2**24


# torch is imported last so that failing mutants stop before paying for it
def test_bf16_decode_all_bit_patterns():
    import torch
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.x_to_f64(bits, "bf16")
    want = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
