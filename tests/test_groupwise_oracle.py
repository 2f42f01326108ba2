"""Pins of the group-wise row-scale oracle (``oracle/groupwise.py``): one
group is the ordinary format (the C oracle), every group is the ordinary
format on its own column slice (the C oracle again), and a hand-sized case
by explicit loops.  A planted mistake in the group index must fail."""

import numpy as np
import pytest

import oracle
import workloads as wl
from oracle import groupwise as GW


def _problem(M, N, K, seed, nS=0, Ks=2):
    return wl.make_problem(M, N, K, nS=nS, Ks=Ks, seed=seed, x_dtype="f32")


def _c_oracle_y(p):
    return oracle.gemv(oracle.OracleWeights.from_problem(p), p.x_f32().astype(np.float64))[0][0]


def _salient_args(p):
    if not p.nS:
        return {}
    return {"s_idx": p.s_idx, "s_signs": p.s_signs(), "s_alpha_r": p.s_alpha_r, "s_alpha_c": p.s_alpha_c}


@pytest.mark.parametrize("nS", [0, 37])
def test_one_group_is_the_ordinary_format(nS):
    p = _problem(48, 256, 2, seed=31, nS=nS)
    ar = p.alpha_r[:, :, None]                                  # [K][M][1]: G = N
    y = GW.gemv(p.signs(), ar, p.alpha_c, p.N, p.x_f32()[0], **_salient_args(p))
    np.testing.assert_allclose(y, _c_oracle_y(p), rtol=1e-12, atol=1e-15)


def test_each_group_is_the_ordinary_format_on_its_columns():
    """y = sum over groups of the ordinary GEMV of the group's column slice
    with that group's row scales, each computed by the C oracle."""
    M, N, K, G = 40, 512, 3, 128
    p = _problem(M, N, K, seed=32)
    rng = np.random.default_rng(33)
    ar = np.abs(rng.normal(0.0, 0.02, size=(K, M, N // G))).astype(np.float32) + 1e-3
    x = p.x_f32()[0]
    y = GW.gemv(p.signs(), ar, p.alpha_c, G, x)
    total = np.zeros(M)
    for gi in range(N // G):
        cols = slice(gi * G, (gi + 1) * G)
        q = wl.Problem(name="slice", M=M, N=G, K=K, g=4, nS=0, Ks=0, batch=1, x_dtype="f32",
                       sign_bits=np.ascontiguousarray(p.sign_bits[:, :, gi * G // 8:(gi + 1) * G // 8]),
                       alpha_r=np.ascontiguousarray(ar[:, :, gi]), alpha_c=np.ascontiguousarray(p.alpha_c[:, cols]),
                       s_idx=np.zeros(0, np.uint32), s_sign_bits=np.zeros((0, M, 0), np.uint8),
                       s_alpha_r=np.zeros((0, M), np.float32), s_alpha_c=np.zeros((0, 0), np.float32),
                       x=np.ascontiguousarray(p.x[:, cols]))
        total += _c_oracle_y(q)
    np.testing.assert_allclose(y, total, rtol=1e-12, atol=1e-15)


def test_hand_sized_case_by_loops():
    """2 rows, 8 columns, groups of 4, one base: written out with loops."""
    signs = np.array([[[1, -1, 1, 1, -1, -1, 1, -1], [1, 1, 1, 1, -1, 1, -1, 1]]], np.int8)
    ar = np.array([[[2.0, 0.5], [1.0, 3.0]]])                    # [K=1][M=2][N/G=2]
    ac = np.array([[1.0, 2.0, 3.0, 4.0, 1.0, 1.0, 2.0, 2.0]])
    x = np.array([1.0, -1.0, 0.5, 2.0, 4.0, -2.0, 1.0, 0.25])
    want = []
    for i in range(2):
        s = 0.0
        for j in range(8):
            s += ar[0][i][j // 4] * ac[0][j] * signs[0][i][j] * x[j]
        want.append(s)
    assert GW.gemv(signs, ar, ac, 4, x).tolist() == want
    # by hand, row 0: group 0 = 1*1*1 + 2*(-1)*(-1) + 3*1*0.5 + 4*1*2 = 12.5, scaled by 2;
    # group 1 = 1*(-1)*4 + 1*(-1)*(-2) + 2*1*1 + 2*(-1)*0.25 = -0.5, scaled by 0.5
    assert want[0] == 24.75
    # row 1: group 0 = 1*1*1 + 2*1*(-1) + 3*1*0.5 + 4*1*2 = 8.5, scaled by 1;
    # group 1 = 1*(-1)*4 + 1*1*(-2) + 2*(-1)*1 + 2*1*0.25 = -7.5, scaled by 3
    assert want[1] == -14.0


def test_bad_grouping_is_rejected():
    with pytest.raises(ValueError):
        GW.group_of(100, 128)
    with pytest.raises(ValueError):
        GW.dequant(np.ones((1, 2, 8), np.int8), np.ones((1, 2, 3)), None, 4)


def test_planted_group_index_mistake_fails(monkeypatch):
    monkeypatch.setattr(GW, "group_of", lambda N, G: np.minimum((np.arange(N) + 1) // G, N // G - 1))
    with pytest.raises(AssertionError):
        test_each_group_is_the_ordinary_format_on_its_columns()
    with pytest.raises(AssertionError):
        test_hand_sized_case_by_loops()


SOURCE_MUTATIONS = [
    ("groups in reverse order", "np.asarray(alpha_r, np.float64)[:, :, grp]", "np.asarray(alpha_r, np.float64)[:, :, grp[::-1]]"),
    ("column scales ignored", "ac = np.ones((K, N)) if alpha_c is None else np.asarray(alpha_c, np.float64)",
     "ac = np.ones((K, N))"),
    ("salient term dropped", "W[:, S] += Ws", "W[:, S] += 0.0 * Ws"),
    ("salient term on the compact columns", "W[:, S] += Ws", "W[:, :nS] += Ws"),
    ("row scales of base 0 for every base", "ar = np.asarray(alpha_r, np.float64)[:, :, grp]",
     "ar = np.asarray(alpha_r, np.float64)[[0] * K][:, :, grp]"),
]


@pytest.mark.parametrize("name,old,new", SOURCE_MUTATIONS, ids=[m[0] for m in SOURCE_MUTATIONS])
def test_planted_source_mistakes_fail_a_pin(monkeypatch, name, old, new):
    """Each edits one step of a copy of ``oracle/groupwise.py`` (loaded as a
    new module; the real one is untouched); one of the pins must fail."""
    import sys
    import types
    src = open(GW.__file__).read()
    assert src.count(old) == 1, name
    mod = types.ModuleType("groupwise_mutant")
    exec(compile(src.replace(old, new), GW.__file__, "exec"), mod.__dict__)
    monkeypatch.setattr(sys.modules[__name__], "GW", mod)
    failed = 0
    for pin in (lambda: test_one_group_is_the_ordinary_format(37), test_each_group_is_the_ordinary_format_on_its_columns,
                test_hand_sized_case_by_loops):
        try:
            pin()
        except (AssertionError, IndexError, ValueError):
            failed += 1
    assert failed, name
