"""Checks of the seeded input generators (``workloads/``), which both the
CUDA path's tests and bench and the oracle's tests read: the interchange
formats, the recipe's structure (salient sets, ternary encoding, integer
mode, seeds) and the algorithmic byte counts the roofline divides by.
CPU only."""

import numpy as np
import pytest
import torch

import workloads as wl


def test_salient_counts_round_half_up():
    # 3% of 4096 = 122.88, of 11008 = 330.24; 5% of 8192 = 409.6, of 28672 = 1433.6
    assert [wl.salient_count(0.03, 4096), wl.salient_count(0.03, 11008)] == [123, 330]
    assert [wl.salient_count(0.05, 8192), wl.salient_count(0.05, 28672)] == [410, 1434]
    assert wl.salient_count(0.5, 3) == 2 and wl.salient_count(0.25, 2) == 1 and wl.salient_count(0.0, 99) == 0


def test_sign_bits_are_lsb_first_and_round_trip():
    signs = np.array([[1, -1, -1, -1, -1, -1, -1, -1, -1, 1] + [-1] * 22], np.int8)
    bits = wl.pack_signs(signs)
    assert bits.shape == (1, 4) and bits[0].tolist() == [0x01, 0x02, 0, 0]   # column 0 and column 9
    rng = np.random.default_rng(0)
    s = np.where(rng.random((3, 5, 70)) < 0.5, 1, -1).astype(np.int8)
    b = wl.pack_signs(s)
    assert b.shape == (3, 5, 12)                                            # 70 columns padded to 96
    assert np.array_equal(wl.unpack_signs(b, 70), s)
    assert not np.unpackbits(b, axis=-1, bitorder="little")[..., 70:].any()  # pad bits are 0


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 20000),
                        np.array([0.0, -0.0, 1.0, -2.5, 3.0e38, 1e-40], np.float32)]).astype(np.float32)
    ties = (np.arange(64, dtype=np.uint32) << 16 | 0x8000).view(np.float32)  # exactly halfway
    v = np.concatenate([v, ties, -ties])
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(wl.f32_to_bf16_bits(v), want)
    assert np.array_equal(wl.bf16_bits_to_f32(want), torch.from_numpy(want.view(np.int16)).view(torch.bfloat16)
                          .float().numpy())


def test_problem_structure():
    p = wl.make_problem(70, 544, 3, nS=45, Ks=2, batch=3, x_dtype="bf16", seed=5)
    assert p.sign_bits.shape == (3, 70, 68) and p.alpha_r.shape == (3, 70) and p.alpha_c.shape == (3, 544)
    assert p.s_sign_bits.shape == (2, 70, 8) and p.s_alpha_r.shape == (2, 70) and p.s_alpha_c.shape == (2, 45)
    assert p.x.shape == (3, 544) and p.x.dtype == np.uint16
    assert np.all(np.diff(p.s_idx.astype(np.int64)) > 0) and p.s_idx.max() < 544 and p.s_idx.dtype == np.uint32
    assert not np.unpackbits(p.s_sign_bits, axis=-1, bitorder="little")[..., 45:].any()
    assert np.all(p.alpha_r >= np.float32(1e-3)) and np.all(p.s_alpha_c >= np.float32(1e-3))
    q = wl.make_problem(70, 544, 3, nS=45, Ks=2, batch=3, x_dtype="bf16", seed=5)
    r = wl.make_problem(70, 544, 3, nS=45, Ks=2, batch=3, x_dtype="bf16", seed=6)
    for f in ("sign_bits", "alpha_r", "alpha_c", "s_idx", "s_sign_bits", "s_alpha_r", "s_alpha_c", "x"):
        assert np.array_equal(getattr(p, f), getattr(q, f)), f                 # same seed, same draw
    assert not np.array_equal(p.sign_bits, r.sign_bits) and not np.array_equal(p.x, r.x)
    with pytest.raises(ValueError):
        wl.make_problem(8, 40, 1)                                              # N % 32 != 0


def test_integer_mode_values():
    p = wl.make_problem(64, 256, 2, nS=20, Ks=2, x_dtype="f16", integer_mode=True, seed=7)
    assert set(np.unique(p.alpha_r)) <= {0.5, 1.0, 1.5, 2.0}
    assert set(np.unique(p.alpha_c)) <= {1.0, 2.0, 3.0, 4.0}
    assert set(np.unique(p.s_alpha_r)) <= {0.5, 1.0, 1.5, 2.0}
    assert set(np.unique(p.s_alpha_c)) <= {1.0, 2.0, 3.0, 4.0}
    assert set(np.unique(p.x_f32())) <= set(range(-4, 5))


def test_ternary_encoding():
    p = wl.make_problem(40, 96, 2, x_dtype="bf16", ternary=True, seed=8)
    s = p.signs().astype(np.int64)
    assert np.array_equal((s[0] + s[1]) // 2, p.ternary)                      # +1:(+,+)  -1:(-,-)  0:(+,-)
    assert np.array_equal(s[0][p.ternary == 0], np.ones(int((p.ternary == 0).sum())))
    assert p.alpha_c is None and np.array_equal(p.alpha_r[0], p.alpha_r[1])
    counts = np.bincount(wl.ternary11008().ternary.ravel() + 1, minlength=3)
    assert np.all(np.abs(counts / counts.sum() - 1 / 3) < 0.005)             # p = 1/3 each
    with pytest.raises(ValueError):
        wl.make_problem(8, 32, 3, ternary=True)


@pytest.mark.parametrize("build,want", [
    # planes 2*4096*4096/8 = 4,194,304; alpha_r, alpha_c 2*4*4096 each = 32,768 + 32,768; x 8,192 (fp16);
    # y 16,384; salient planes 2*4096*128/8 = 131,072; alpha_r^s 32,768; alpha_c^s 1,024; s_idx 512
    (lambda: wl.layer4096(), 4_449_792),
    # planes 2*11008*4096/8 = 11,272,192; alpha_r 88,064; no alpha_c; x 8,192 (bf16); y 44,032
    (lambda: wl.ternary11008(), 11_412_480),
    # planes 3*8192*8192/8 = 25,165,824; alpha_r, alpha_c 98,304 each; x 16,384; y 32,768;
    # salient planes 2*8192*410/8 = 839,680; alpha_r^s 65,536; alpha_c^s 3,280; s_idx 1,640
    (lambda: wl.layer70b(0, 1), 26_321_720),
])
def test_algorithmic_bytes_by_hand(build, want):
    assert build().algorithmic_bytes() == want


def test_step7b_recipe_and_bytes():
    """32 layers of q, k, v, o (4096^2), gate, up (11008x4096) and down
    (4096x11008), 3% salient; the seeds are 1000 + 7*layer + matrix.  Bytes by
    hand, as planes + alpha_r + alpha_c + x + y + salient planes + alpha_r^s +
    alpha_c^s + s_idx:
      4096^2, nS 123:     4,194,304 + 32,768 + 32,768 + 8,192 + 16,384 + 125,952
                          + 32,768 + 984 + 492 = 4,444,612
      11008x4096, nS 123: 11,272,192 + 88,064 + 32,768 + 8,192 + 44,032 + 338,496
                          + 88,064 + 984 + 492 = 11,873,284
      4096x11008, nS 330: 11,272,192 + 32,768 + 88,064 + 22,016 + 16,384 + 337,920
                          + 32,768 + 2,640 + 1,320 = 11,806,072
    one layer 53,331,088 B, the step 32 times that."""
    p = wl.step7b_matrix(3, 5)
    assert (p.M, p.N, p.nS, p.K, p.g, p.Ks, p.x_dtype) == (11008, 4096, 123, 2, 4, 2, "f16")
    q = wl.make_problem(11008, 4096, 2, g=4, nS=123, Ks=2, x_dtype="f16", seed=1000 + 7 * 3 + 5)
    assert np.array_equal(p.sign_bits[:, :4], q.sign_bits[:, :4]) and np.array_equal(p.x, q.x)
    layer = [wl.step7b_matrix(0, m).algorithmic_bytes() for m in range(7)]
    assert layer == [4_444_612] * 4 + [11_873_284] * 2 + [11_806_072]
    assert 32 * sum(layer) == 1_706_594_816
